"""Guard bands around every output of the hot-path calls (the stand-in for a memory checker on
this hardware): each output buffer is a view into a larger allocation whose bytes before and
after it hold a sentinel; after the call (on ragged shapes) the sentinels must be intact."""
import numpy as np
import pytest
import torch

from nvfp4_w4a4_moe_02_b200 import nvfp4rac as R
from nvfp4_w4a4_moe_02_b200 import synthetic as syn

pytestmark = pytest.mark.gpu

GUARD = 4096  # bytes on each side (keeps the 16-byte alignment of the view)
SENTINEL = 0xA5


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    R.load()
    return torch.device("cuda:0")


class Guarded:
    """nbytes of device memory with GUARD sentinel bytes on both sides."""

    def __init__(self, nbytes, dev, fill=None):
        self.n = nbytes
        self.raw = torch.full((nbytes + 2 * GUARD,), SENTINEL, dtype=torch.uint8, device=dev)
        if fill is not None:
            self.raw[GUARD:GUARD + nbytes].fill_(fill)

    def view(self, dtype=torch.uint8):
        return self.raw[GUARD:GUARD + self.n].view(dtype)

    def intact(self):
        lo = self.raw[:GUARD].cpu().numpy()
        hi = self.raw[GUARD + self.n:].cpu().numpy()
        return bool(np.all(lo == SENTINEL) and np.all(hi == SENTINEL))


def guarded_packed(rows, cols, dev, rows_padded=None, layout=R.SF_ATOM128, slabs=1):
    group = 16 if layout == R.SF_SLAB16 else 128
    rp = R.round_up(rows, group) if rows_padded is None else rows_padded
    gc = Guarded(slabs * rp * cols // 2, dev, fill=0)
    gs = Guarded(slabs * R.sf_bytes(rp, cols, layout), dev, fill=0)
    gg = Guarded(slabs * 4, dev, fill=0)
    p = R.Packed(gc.view(), gs.view(), gg.view(torch.float32), slabs, rows, rp, cols, layout)
    return p, [gc, gs, gg]


def to_dev(a, dev):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to(dev).view(torch.bfloat16)


def test_quantise_and_gemm_outputs_stay_inside(dev, orc):
    M, N, K, Kp = 301, 384, 704, 192
    x = syn.normal_bf16(21, 1, M, K, 1.0, syn.outlier_colscale(21, K))
    w = syn.normal_bf16(21, 2, N, K, 0.02)
    sel = np.sort(np.random.default_rng(21).choice(K, Kp, replace=False)).astype(np.int32)
    seld = torch.from_numpy(sel).to(dev)
    st = R.new_status(dev)
    q, gq = guarded_packed(M, K, dev)
    qr, gqr = guarded_packed(M, Kp, dev, rows_padded=q.rows_padded)
    R.nvfp4_quantize(to_dev(x, dev), seld, out=q, out_res=qr, status=st)
    wq, gw = guarded_packed(N, K, dev, rows_padded=N)
    ws, gws = guarded_packed(N, Kp, dev, rows_padded=N)
    R.pack_weights(to_dev(w, dev), seld, out=wq, out_sel=ws, status=st)
    for dt in (torch.float32, torch.bfloat16):
        gy = Guarded(M * N * (4 if dt == torch.float32 else 2), dev)
        y = gy.view(dt).view(M, N)
        R.w4a4_rac_gemm(q, qr, wq, ws, M, y=y, status=st)
        torch.cuda.synchronize()
        R.check_status(st)
        assert gy.intact(), dt
    for g in gq + gqr + gw + gws:
        assert g.intact()


def test_moe_outputs_stay_inside(dev, orc):
    """Scatter quantiser, grouped GEMM (SwiGLU), segment quantiser, grouped GEMM, combine, on a
    layout made by the device plan."""
    wl = syn.moe_block(T=96, H=512, E=8, topk=2, I=128, T_cal=64)
    T, k = wl.topk_ids.shape
    st = R.new_status(dev)
    ids = torch.from_numpy(np.ascontiguousarray(wl.topk_ids, dtype=np.int32)).to(dev)
    cap = R.moe_rows_capacity(T, k, wl.E, 128)
    g_er = Guarded(wl.E * 4, dev)
    er = g_er.view(torch.int32)
    off, rs, _, _ = R.moe_dispatch_plan(ids, wl.E, 128, rows_capacity=cap, status=st, expert_rows=er)
    sel_gu = torch.from_numpy(orc.calibrate(wl.x_cal, wl.Kp_gu)[0]).to(dev)
    sel_dn = torch.from_numpy(orc.calibrate(syn.moe_down_calibration_batch(wl), wl.Kp_dn)[0]).to(dev)
    pgu, pgus = R.pack_weights(to_dev(wl.wgu, dev), sel_gu, gate_up_interleave=True, status=st)
    pdn, pdns = R.pack_weights(to_dev(wl.wdn, dev), sel_dn, status=st)
    a, ga = guarded_packed(cap, wl.H, dev, rows_padded=cap)
    ar, gar = guarded_packed(cap, wl.Kp_gu, dev, rows_padded=cap)
    R.nvfp4_quantize_scatter(to_dev(wl.x, dev), rs, cap, sel_gu, out=a, out_res=ar, status=st)
    gh = Guarded(cap * wl.I * 2, dev, fill=0)
    h = gh.view(torch.bfloat16).view(cap, wl.I)
    gam = Guarded(4, dev)
    amax = gam.view(torch.float32)
    R.grouped_w4a4_rac_moe(a, ar, off, pgu, pgus, swiglu=True, y=h, amax_out=amax, status=st, expert_rows=er)
    hq, ghq = guarded_packed(cap, wl.I, dev, rows_padded=cap)
    hqr, ghqr = guarded_packed(cap, wl.Kp_dn, dev, rows_padded=cap)
    R.nvfp4_quantize_segments(h, off, er, sel_dn, amax_in=amax, out=hq, out_res=hqr, status=st)
    gy = Guarded(cap * wl.H * 2, dev)
    y = gy.view(torch.bfloat16).view(cap, wl.H)
    R.grouped_w4a4_rac_moe(hq, hqr, off, pdn, pdns, y=y, status=st, expert_rows=er)
    gout = Guarded(T * wl.H * 2, dev)
    out = gout.view(torch.bfloat16).view(T, wl.H)
    wts = torch.full((T, k), 0.5, dtype=torch.float32, device=dev)
    R.moe_combine(y, rs, wts, out=out, status=st)
    torch.cuda.synchronize()
    R.check_status(st)
    for g in ga + gar + [gh, gam, g_er] + ghq + ghqr + [gy, gout]:
        assert g.intact()


def test_decode_and_qdq_outputs_stay_inside(dev, orc):
    wl = syn.moe_block(T=40, H=1024, E=12, topk=2, I=256, T_cal=64)
    T, k = wl.topk_ids.shape
    st = R.new_status(dev)
    ids = torch.from_numpy(np.ascontiguousarray(wl.topk_ids, dtype=np.int32)).to(dev)
    cap = R.moe_rows_capacity(T, k, wl.E, 16)
    _, rs, se, sc = R.moe_dispatch_plan(ids, wl.E, 16, rows_capacity=cap, n_slots=cap // 16, status=st)
    sel = torch.from_numpy(orc.calibrate(wl.x_cal, wl.Kp_gu)[0]).to(dev)
    pgu, pgus = R.pack_weights(to_dev(wl.wgu, dev), sel, gate_up_interleave=True, status=st)
    a, ga = guarded_packed(cap, wl.H, dev, rows_padded=cap, layout=R.SF_SLAB16)
    ar, gar = guarded_packed(cap, wl.Kp_gu, dev, rows_padded=cap, layout=R.SF_SLAB16)
    R.nvfp4_quantize_scatter(to_dev(wl.x, dev), rs, cap, sel, out=a, out_res=ar, status=st)
    gy = Guarded(cap * wl.I * 2, dev)
    y = gy.view(torch.bfloat16).view(cap, wl.I)
    gam = Guarded(4, dev)
    R.grouped_w4a4_rac_moe_decode(a, ar, se, sc, pgu, pgus, swiglu=True, y=y, amax_out=gam.view(torch.float32),
                                  status=st)
    n = 3 * 4096 + 48
    wq = torch.from_numpy(syn.normal_bf16(5, 2, 3, n // 3, 0.02).view(np.int16)).to(dev).view(torch.bfloat16)
    gq = Guarded(n * 2, dev)
    gs = Guarded(3 * 4, dev)
    R.weight_qdq(wq, out=gq.view(torch.bfloat16).view(3, n // 3), s_g=gs.view(torch.float32), status=st)
    gc = Guarded(cap * wl.H, dev)
    gsf = Guarded(cap * wl.H // 16, dev)
    lib = R.load()
    import ctypes
    c = a.c()
    R._check(lib.nvfp4_unpack_logical(ctypes.byref(c), 0, gc.view().data_ptr(), gsf.view().data_ptr(),
                                      R._stream(None)))
    torch.cuda.synchronize()
    R.check_status(st)
    for g in ga + gar + [gy, gam, gq, gs, gc, gsf]:
        assert g.intact()
