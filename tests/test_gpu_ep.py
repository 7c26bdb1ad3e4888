"""GPU side of expert parallelism (one GPU: the exchange itself is covered on CPU ranks).

The grouped GEMM over source-major segments with a segment -> expert map (what a rank
receives) against the oracle, the standalone amax, and the whole expert-parallel layer on a
one-rank NCCL group against the single-GPU layer, bit for bit."""
import os
import socket

import numpy as np
import pytest
import torch

from nvfp4_w4a4_moe_02_b200 import nvfp4rac as R
from nvfp4_w4a4_moe_02_b200 import synthetic as syn

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    R.load()
    return torch.device("cuda:0")


def to_dev(a, dev):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to(dev).view(torch.bfloat16)


def test_amax_matches_oracle(dev, orc):
    x = syn.normal_bf16(3, 1, 777, 320, 1.0, syn.outlier_colscale(3, 320))
    a = R.nvfp4_amax(to_dev(x, dev))
    torch.cuda.synchronize()
    assert np.float32(a.item()) == orc.amax_bf16(x)


def test_segments_gemm_matches_oracle(dev, orc):
    """Rows in segments (source, expert) of 128-padded blocks, several segments per expert, the
    weight slab of each given by seg_expert; plain and SwiGLU epilogues."""
    wl = syn.moe_block(T=120, H=512, E=4, topk=2, I=128, T_cal=64)
    sel = orc.calibrate(wl.x_cal, wl.Kp_gu)[0]
    rng = np.random.default_rng(7)
    # segment list: (expert, tokens) with two "sources" per expert, one of them empty for expert 3
    segs = []
    for src in range(2):
        for e in range(4):
            n = 0 if (e == 3 and src == 1) else int(rng.integers(1, 140))
            segs.append((e, rng.integers(0, wl.x.shape[0], n)))
    off = [0]
    for _, toks in segs:
        off.append(off[-1] + (len(toks) + 127) // 128 * 128)
    rows = off[-1]
    gather = np.full(rows, -1, np.int32)
    for (e, toks), o in zip(segs, off):
        gather[o:o + len(toks)] = toks
    st = R.new_status(dev)
    seld = torch.from_numpy(sel).to(dev)
    a, ar = R.nvfp4_quantize(to_dev(wl.x, dev), seld, row_gather=torch.from_numpy(gather).to(dev), M_out=rows,
                             status=st)
    w, ws = R.pack_weights(to_dev(wl.wgu, dev), seld, gate_up_interleave=True, status=st)
    seg_off = torch.tensor(off, dtype=torch.int32, device=dev)
    seg_rows = torch.tensor([len(t) for _, t in segs], dtype=torch.int32, device=dev)
    seg_exp = torch.tensor([e for e, _ in segs], dtype=torch.int32, device=dev)
    y = R.grouped_w4a4_rac_moe_segments(a, ar, seg_off, seg_rows, seg_exp, w, ws, out_dtype=torch.float32,
                                        status=st)
    h, amax = R.grouped_w4a4_rac_moe_segments(a, ar, seg_off, seg_rows, seg_exp, w, ws, swiglu=True, status=st)
    torch.cuda.synchronize()
    R.check_status(st)
    s_x = orc.global_scale(orc.amax_bf16(wl.x))
    yg = y.cpu().numpy()
    n = np.arange(2 * wl.I)
    logical = np.where((n % 128) < 64, (n // 128) * 64 + n % 128, wl.I + (n // 128) * 64 + n % 128 - 64)
    for (e, toks), o in zip(segs, off):
        if len(toks) == 0:
            continue
        ac, aS, rc, rS, _ = orc.act_quant_rac(wl.x[toks], s_x, sel)
        s_w = orc.global_scale(orc.amax_bf16(wl.wgu[e]))
        y_ref, ad = orc.gemm_rac(ac, aS, rc, rS, *orc.weight_pack(wl.wgu[e], s_w, sel), s_x, s_w)
        got = np.empty((len(toks), 2 * wl.I))
        got[:, logical] = yg[o:o + len(toks)]
        err = np.abs(got - y_ref)
        assert (err <= 1e-3 * ad + 1e-6).all(), (e, err.max())
    # a segment naming a slab outside the weights is reported
    bad = torch.tensor([0, 9, 1, 2, 3, 0, 1, 2], dtype=torch.int32, device=dev)
    st2 = R.new_status(dev)
    R.grouped_w4a4_rac_moe_segments(a, ar, seg_off, seg_rows, bad, w, ws, out_dtype=torch.float32, status=st2)
    torch.cuda.synchronize()
    assert int(st2.item()) == 1
    assert h.shape == (rows, wl.I) and amax.item() > 0


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_expert_parallel_one_rank_equals_the_layer(dev, orc):
    """EPMoEBlock on a one-rank NCCL group (global amax reductions, count and row all-to-alls,
    segment GEMMs, reverse all-to-all, combine) gives the single-GPU layer's output bit for bit."""
    import torch.distributed as dist

    from nvfp4_w4a4_moe_02_b200.ep import EPMoEBlock, ExpertParallel

    wl = syn.moe_block(T=256, H=512, E=8, topk=2, I=256, T_cal=64)
    T, k = wl.topk_ids.shape
    sel_gu = torch.from_numpy(orc.calibrate(wl.x_cal, wl.Kp_gu)[0]).to(dev)
    sel_dn = torch.from_numpy(orc.calibrate(syn.moe_down_calibration_batch(wl), wl.Kp_dn)[0]).to(dev)
    st = R.new_status(dev)
    pgu, pgus = R.pack_weights(to_dev(wl.wgu, dev), sel_gu, gate_up_interleave=True, status=st)
    pdn, pdns = R.pack_weights(to_dev(wl.wdn, dev), sel_dn, status=st)
    logits = torch.from_numpy(syn.normal_f64(wl.seed, syn.STREAM_ROUTER, T * wl.E).reshape(T, wl.E)
                              .astype(np.float32)).to(dev)
    x = to_dev(wl.x, dev)
    # the single-GPU layer
    cap = R.moe_rows_capacity(T, k, wl.E, 128)
    ids, wts = R.moe_route_topk(logits, k, status=st)
    er = torch.empty(wl.E, dtype=torch.int32, device=dev)
    off, rows, _, _ = R.moe_dispatch_plan(ids, wl.E, 128, rows_capacity=cap, status=st, expert_rows=er)
    a, ar = R.nvfp4_quantize_scatter(x, rows, cap, sel_gu, status=st)
    h, amax_h = R.grouped_w4a4_rac_moe(a, ar, off, pgu, pgus, swiglu=True, status=st, expert_rows=er)
    hq = R.Packed.empty(cap, wl.I, rows_padded=cap, device=dev, zero=True)
    hqr = R.Packed.empty(cap, wl.Kp_dn, rows_padded=cap, device=dev, zero=True)
    R.nvfp4_quantize_segments(h, off, er, sel_dn, amax_in=amax_h, out=hq, out_res=hqr, status=st)
    ye = R.grouped_w4a4_rac_moe(hq, hqr, off, pdn, pdns, status=st, expert_rows=er)
    y_ref = R.moe_combine(ye, rows, wts, status=st)
    torch.cuda.synchronize()
    R.check_status(st)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_free_port()))
    dist.init_process_group("nccl", rank=0, world_size=1)
    try:
        ep = ExpertParallel(wl.E)
        blk = EPMoEBlock(ep, T, k, wl.H, wl.I, (pgu, pgus, pdn, pdns), sel_gu, sel_dn, dev)
        y = blk.run(x, logits)
        torch.cuda.synchronize()
        R.check_status(blk.status)
        assert torch.equal(y.view(torch.int16), y_ref.view(torch.int16))
    finally:
        dist.destroy_process_group()
