"""GPU parity of the bulk-copy activation quantiser against the oracle (through the C ABI):
every tile shape it can pick (rows per tile, consumer warps), every row map (plain rows with
zero padding rows, gather, scatter, expert segments), both scale layouts, and the calls around
it that inspect or differentiate the packed data (nvfp4_unpack_logical, weight_qdq_backward)."""
import numpy as np
import pytest
import torch

from nvfp4_w4a4_moe_02_b200 import nvfp4rac as R
from nvfp4_w4a4_moe_02_b200 import synthetic as syn
from nvfp4_layout import expert_layout, scatter_map, unpack_codes, unpack_sf

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    R.load()
    yield torch.device("cuda:0")
    R.set_act_tile(0, 0)


def to_dev(a, dev):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to(dev).view(torch.bfloat16)


def logical(p, rows=None):
    rows = p.rows if rows is None else rows
    codes = p.codes.cpu().numpy()
    sf = p.sf.cpu().numpy()
    return (unpack_codes(codes, rows, p.rows_padded, p.cols),
            unpack_sf(sf, rows, p.rows_padded, p.cols, slab16=p.sf_layout == R.SF_SLAB16))


def ref_quant(orc, x, sel, s_g=None):
    s = orc.global_scale(orc.amax_bf16(x)) if s_g is None else s_g
    c, S, rc, rS, _ = orc.act_quant_rac(x, s, sel)
    return s, c, S, rc, rS


@pytest.mark.parametrize("rows,warps", [(1, 4), (3, 6), (5, 7), (16, 8), (0, 0)])
@pytest.mark.parametrize("K,Kp", [(768, 384), (1024, 192), (2048, 1024), (576, 0)])
def test_every_tile_shape_matches_oracle(dev, orc, rows, warps, K, Kp):
    """Forced tile shapes (rows per tile x consumer warps, 0 = automatic) on a ragged row count:
    codes, scales, residual bit-exact; rows past M (to rows_padded) come out zero."""
    M = 301
    rng = np.random.default_rng(K + Kp)
    x = syn.normal_bf16(K, 1, M, K, 1.0, np.exp(rng.standard_normal(K)))
    sel = np.sort(rng.choice(K, Kp, replace=False)).astype(np.int32)
    R.set_act_tile(rows, warps)
    try:
        st = R.new_status(dev)
        q, qr = R.nvfp4_quantize(to_dev(x, dev), torch.from_numpy(sel).to(dev) if Kp else None, status=st)
        torch.cuda.synchronize()
        R.check_status(st)
    finally:
        R.set_act_tile(0, 0)
    s, c, S, rc, rS = ref_quant(orc, x, sel)
    assert q.s_g.item() == float(s)
    gc, gS = logical(q, rows=q.rows_padded)
    assert np.array_equal(gc[:M], c) and np.array_equal(gS[:M], S)
    assert not gc[M:].any() and not gS[M:].any()
    if Kp:
        grc, grS = logical(qr, rows=qr.rows_padded)
        assert np.array_equal(grc[:M], rc) and np.array_equal(grS[:M], rS)
        assert not grc[M:].any() and not grS[M:].any()


def test_gather_rows_and_zero_rows(dev, orc):
    """Gather map with repeated, negative and out-of-range entries (those give zero rows)."""
    K, Kp, M = 1024, 512, 90
    rng = np.random.default_rng(5)
    x = syn.normal_bf16(7, 1, M, K, 1.0, syn.outlier_colscale(7, K))
    sel = np.sort(rng.choice(K, Kp, replace=False)).astype(np.int32)
    g = rng.integers(-5, M + 5, 200).astype(np.int32)
    g[:3] = [0, 0, M - 1]
    st = R.new_status(dev)
    q, qr = R.nvfp4_quantize(to_dev(x, dev), torch.from_numpy(sel).to(dev), row_gather=torch.from_numpy(g).to(dev),
                             M_out=g.size, status=st)
    torch.cuda.synchronize()
    R.check_status(st)
    s, c, S, rc, rS = ref_quant(orc, x, sel)
    ok = (g >= 0) & (g < M)
    gc, gS = logical(q)
    grc, grS = logical(qr)
    assert np.array_equal(gc[ok], c[g[ok]]) and np.array_equal(gS[ok], S[g[ok]])
    assert np.array_equal(grc[ok], rc[g[ok]]) and np.array_equal(grS[ok], rS[g[ok]])
    assert not gc[~ok].any() and not gS[~ok].any() and not grc[~ok].any() and not grS[~ok].any()


@pytest.mark.parametrize("layout", [R.SF_ATOM128, R.SF_SLAB16])
def test_scatter_fanout_matches_oracle(dev, orc, layout):
    """Each token's codes land in all its expert rows (fanout 8), untouched rows stay zero."""
    T, K, Kp, E = 200, 2048, 1024, 16
    wl = syn.moe_block(T=T, H=K, E=E, topk=8, I=128, T_cal=64)
    sel = orc.calibrate(wl.x_cal, Kp)[0]
    off, rows_padded, pair_rows = expert_layout(wl.counts, 128 if layout == R.SF_ATOM128 else 16)
    sm = scatter_map(wl.pair_token, pair_rows, T, 8)
    st = R.new_status(dev)
    q, qr = R.nvfp4_quantize_scatter(to_dev(wl.x, dev), torch.from_numpy(sm).to(dev), rows_padded,
                                     torch.from_numpy(sel).to(dev), status=st, sf_layout=layout)
    torch.cuda.synchronize()
    R.check_status(st)
    s, c, S, rc, rS = ref_quant(orc, wl.x, sel)
    gc, gS = logical(q, rows=rows_padded)
    grc, grS = logical(qr, rows=rows_padded)
    tok = wl.pair_token
    assert np.array_equal(gc[pair_rows], c[tok]) and np.array_equal(gS[pair_rows], S[tok])
    assert np.array_equal(grc[pair_rows], rc[tok]) and np.array_equal(grS[pair_rows], rS[tok])
    pad = np.ones(rows_padded, bool)
    pad[pair_rows] = False
    assert not gc[pad].any() and not gS[pad].any() and not grc[pad].any()


def test_segments_quantise_token_rows_only(dev, orc):
    """nvfp4_quantize_segments: the token rows of each padded expert segment are quantised (the
    tensor scale from amax_in), every other row keeps its previous contents; an empty segment and
    a segment longer than 128 rows are included."""
    K, Kp = 768, 384
    counts = np.array([5, 0, 128, 131, 1, 64, 0, 7], np.int64)
    off, rows_padded, pair_rows = expert_layout(counts, 128)
    rng = np.random.default_rng(9)
    h = syn.normal_bf16(9, 1, rows_padded, K, 0.5, np.exp(rng.standard_normal(K)))
    sel = np.sort(rng.choice(K, Kp, replace=False)).astype(np.int32)
    amax = np.float32(orc.amax_bf16(h[pair_rows]))
    st = R.new_status(dev)
    q = R.Packed.empty(rows_padded, K, device=dev)
    qr = R.Packed.empty(rows_padded, Kp, rows_padded=q.rows_padded, device=dev)
    for t in (q.codes, q.sf, qr.codes, qr.sf):
        t.fill_(0xA5)  # sentinel in the rows that must stay untouched
    R.nvfp4_quantize_segments(to_dev(h, dev), torch.from_numpy(off[:-1].astype(np.int32)).to(dev),
                              torch.from_numpy(counts.astype(np.int32)).to(dev), torch.from_numpy(sel).to(dev),
                              amax_in=torch.tensor([amax], device=dev), out=q, out_res=qr, status=st)
    torch.cuda.synchronize()
    R.check_status(st)
    s = orc.global_scale(amax)
    assert q.s_g.item() == float(s) and qr.s_g.item() == float(s)
    _, c, S, rc, rS = ref_quant(orc, h[pair_rows], sel, s_g=s)
    codes = q.codes.cpu().numpy().reshape(rows_padded, K // 2)
    rcodes = qr.codes.cpu().numpy().reshape(rows_padded, Kp // 2)
    gc, gS = logical(q, rows=rows_padded)
    grc, grS = logical(qr, rows=rows_padded)
    assert np.array_equal(gc[pair_rows], c) and np.array_equal(gS[pair_rows], S)
    assert np.array_equal(grc[pair_rows], rc) and np.array_equal(grS[pair_rows], rS)
    pad = np.ones(rows_padded, bool)
    pad[pair_rows] = False
    assert np.all(codes[pad] == 0xA5) and np.all(rcodes[pad] == 0xA5)
    assert np.all(gS[pad] == 0xA5) and np.all(grS[pad] == 0xA5)


def test_segment_past_the_rows_is_an_error(dev):
    K = 256
    x = torch.zeros(256, K, dtype=torch.bfloat16, device=dev)
    st = R.new_status(dev)
    off = torch.tensor([0, 200], dtype=torch.int32, device=dev)
    rows = torch.tensor([10, 100], dtype=torch.int32, device=dev)  # 200 + 100 > 256
    R.nvfp4_quantize_segments(x, off, rows, amax_in=torch.ones(1, device=dev), status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 1


@pytest.mark.parametrize("layout", [R.SF_ATOM128, R.SF_SLAB16])
def test_unpack_logical_matches_layout_definition(dev, orc, layout):
    """nvfp4_unpack_logical against the test-side decoder of the storage definition, on
    activations (both scale layouts) and on one slab of a packed weight."""
    M, K = 150, 512
    x = syn.normal_bf16(4, 1, M, K, 1.0)
    rp = R.round_up(M, 128 if layout == R.SF_ATOM128 else 16)
    q = R.Packed.empty(M, K, rows_padded=rp, device=dev, sf_layout=layout)
    R.nvfp4_quantize(to_dev(x, dev), out=q)
    codes, sf = R.unpack_logical(q)
    gc, gS = logical(q)
    assert np.array_equal(codes.cpu().numpy(), gc) and np.array_equal(sf.cpu().numpy(), gS)
    w = syn.normal_bf16(4, 2, 3 * 256, K, 0.02).reshape(3, 256, K)
    pw, _ = R.pack_weights(to_dev(w, dev))
    codes, sf = R.unpack_logical(pw, slab=2)
    cb = pw.rows_padded * K // 2
    sb = R.sf_bytes(pw.rows_padded, K)
    ref_c = unpack_codes(pw.codes[2 * cb:3 * cb].cpu().numpy(), 256, 256, K)
    ref_s = unpack_sf(pw.sf[2 * sb:3 * sb].cpu().numpy(), 256, 256, K)
    assert np.array_equal(codes.cpu().numpy(), ref_c) and np.array_equal(sf.cpu().numpy(), ref_s)
    s_w = orc.global_scale(orc.amax_bf16(w[2]))
    c2, S2, _, _ = orc.weight_pack(w[2], s_w, np.zeros(0, np.int32))
    assert np.array_equal(codes.cpu().numpy(), c2) and np.array_equal(sf.cpu().numpy(), S2)


def test_weight_qdq_backward_is_straight_through(dev):
    """The fake-quant's backward: grad_w is grad_fq bit for bit, grad_acc += grad_fq in binary32,
    and torch autograd through FakeQuantSTE hands the upstream gradient to the weights."""
    n = 1000 * 16 + 5  # a tail past the 8-element vectors
    g = torch.from_numpy(syn.normal_bf16(3, 9, 1, n, 1.0)[0].view(np.int16)).to(dev).view(torch.bfloat16)
    gw = R.weight_qdq_backward(g)
    assert torch.equal(gw.view(torch.int16), g.view(torch.int16))
    acc0 = torch.randn(n, device=dev)
    acc = acc0.clone()
    R.weight_qdq_backward(g, grad_acc=acc)
    ref = (acc0.cpu().numpy() + g.float().cpu().numpy()).astype(np.float32)
    assert np.array_equal(acc.cpu().numpy(), ref)
    w = torch.from_numpy(syn.normal_bf16(3, 2, 64, 256, 0.02).view(np.int16)).to(dev).view(torch.bfloat16)
    w.requires_grad_(True)
    y = R.FakeQuantSTE.apply(w)
    ref_fq, _ = R.weight_qdq(w.detach())
    assert torch.equal(y.detach().view(torch.int16), ref_fq.view(torch.int16))
    up = torch.randn(64, 256, device=dev).to(torch.bfloat16)
    y.backward(up)
    assert torch.equal(w.grad.view(torch.int16), up.view(torch.int16))
    assert w.grad.dtype == torch.bfloat16 and w.grad.shape == w.shape


@pytest.mark.parametrize("n,elems", [(1, 16), (5, 512 * 3 + 48), (37, 4096), (600, 1040), (3, 4 << 20)])
def test_weight_qdq_one_pass_equals_two_pass(dev, orc, n, elems):
    """The one-pass fake-quant (CTA groups meeting at a per-tensor counter) and the two-pass form
    give the same bits and scales; sampled tensors also against the oracle."""
    w = syn.normal_bf16(5, 11, n, elems, 0.02)
    w[n - 1, : min(16, elems)] = syn.normal_bf16(5, 12, 1, min(16, elems), 2.0)[0]
    wd = to_dev(w, dev)
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    try:
        R.set_qdq_one_pass(True)
        o1, s1 = R.weight_qdq(wd, status=st)
        R.set_qdq_one_pass(False)
        o2, s2 = R.weight_qdq(wd, status=st)
    finally:
        R.set_qdq_one_pass(True)
    torch.cuda.synchronize()
    assert st.item() == 0
    assert torch.equal(s1, s2)
    assert torch.equal(o1.view(torch.int16), o2.view(torch.int16))
    got = o1.view(torch.int16).cpu().numpy().view(np.uint16).reshape(n, elems)
    for t in sorted({0, n // 2, n - 1}):
        ref, s_ref = orc.weight_qdq(w[t])
        assert s1[t].item() == float(s_ref)
        assert np.array_equal(got[t], ref), (t, np.argwhere(got[t] != ref)[:5])
