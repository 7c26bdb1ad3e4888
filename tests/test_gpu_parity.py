"""Parity of the CUDA path (through the C ABI) with the CPU oracle, on a B200.

Bit-exact: E2M1/E4M3 codes, block scales, per-tensor scales, channel selections,
fake-quantised weights.  GEMM outputs: |y - y_ref| <= 1e-3 * sum_k |a_k b_k| + 1e-6 per
element (plus one bf16 ulp of y_ref in bf16-output mode), y_ref being the exact product of
the identical quantised operands.
"""
import numpy as np
import pytest
import torch

from nvfp4_w4a4_moe_02_b200 import nvfp4rac as R
import nvfp4_layout as L
from nvfp4_w4a4_moe_02_b200 import synthetic as syn
from nvfp4_layout import unpack_codes, unpack_sf

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    R.load()
    return torch.device("cuda:0")


def to_dev(a: np.ndarray, dev) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to(dev).view(torch.bfloat16)


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def logical(p: R.Packed, slab: int = 0, rows: int | None = None):
    rows = p.rows if rows is None else rows
    cb = p.rows_padded * p.cols // 2
    sb = R.sf_bytes(p.rows_padded, p.cols, p.sf_layout)
    codes = p.codes[slab * cb:(slab + 1) * cb].cpu().numpy()
    sf = p.sf[slab * sb:(slab + 1) * sb].cpu().numpy()
    return (unpack_codes(codes, rows, p.rows_padded, p.cols),
            unpack_sf(sf, rows, p.rows_padded, p.cols, slab16=p.sf_layout == R.SF_SLAB16))


def f32(v):
    return np.float32(v)


def bf16_ulp(y: np.ndarray) -> np.ndarray:
    a = np.abs(y).astype(np.float64)
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -126)))
    return 2.0 ** (e - 7)


def assert_gemm_close(y_gpu: np.ndarray, y_ref: np.ndarray, absdot: np.ndarray, bf16_out: bool):
    tol = 1e-3 * absdot + 1e-6
    if bf16_out:
        tol = tol + bf16_ulp(y_ref)
    err = np.abs(y_gpu.astype(np.float64) - y_ref)
    bad = np.argwhere(err > tol)
    assert bad.size == 0, (f"{len(bad)} of {err.size} outside tolerance; first {bad[:5].tolist()} "
                           f"gpu {y_gpu[tuple(bad[0])]} ref {y_ref[tuple(bad[0])]} tol {tol[tuple(bad[0])]}")


# ------------------------------------------------------------------------------------------ codecs
def test_codec_e2m1_matches_oracle(dev, orc):
    rng = np.random.default_rng(0)
    pts = [np.float32(0.0), np.float32(-0.0)]
    for g in [0, .25, .5, .75, 1, 1.25, 1.5, 1.75, 2, 2.5, 3, 3.5, 4, 5, 6, 7, 8, 1e4]:
        v = np.float32(g)
        for _ in range(6):
            pts += [v, -v]
            v = np.nextafter(v, np.float32(np.inf))
        v = np.float32(g)
        for _ in range(6):
            pts += [v, -v]
            v = np.nextafter(v, np.float32(-np.inf))
    arr = np.concatenate([np.array(pts, np.float32), rng.uniform(-9, 9, 1 << 20).astype(np.float32),
                          (rng.standard_normal(1 << 16) * 1e-20).astype(np.float32)])
    got = R.encode_e2m1(torch.from_numpy(arr).to(dev)).cpu().numpy()
    ref = orc.e2m1_encode_array(arr)
    bad = np.nonzero(got != ref)[0]
    assert bad.size == 0, [(float(arr[i]), int(got[i]), int(ref[i])) for i in bad[:8]]


def test_codec_e4m3_matches_oracle(dev, orc):
    rng = np.random.default_rng(1)
    vals = [orc.e4m3_decode(c) for c in range(0x7F)]
    pts = []
    for a, b in zip(vals, vals[1:]):
        m = np.float32((a + b) / 2)
        for d in (-2, -1, 0, 1, 2):
            v = m
            for _ in range(abs(d)):
                v = np.nextafter(v, np.float32(np.inf if d > 0 else -np.inf))
            pts.append(v)
        pts.append(np.float32(b))
    arr = np.concatenate([np.array(pts, np.float32), rng.uniform(0, 500, 1 << 20).astype(np.float32),
                          np.exp(rng.uniform(-14, 7, 1 << 18)).astype(np.float32)])
    got = R.encode_e4m3(torch.from_numpy(arr).to(dev)).cpu().numpy()
    ref = orc.e4m3_encode_array(arr)
    bad = np.nonzero(got != ref)[0]
    assert bad.size == 0, [(float(arr[i]), int(got[i]), int(ref[i])) for i in bad[:8]]


def _bit_patterns(lo: int, n: int, dev):
    """float32 values with the bit patterns lo .. lo + n - 1 (as int32), on the device and on the host."""
    d = torch.arange(lo, lo + n, dtype=torch.int64, device=dev).to(torch.int32).view(torch.float32)
    h = np.arange(lo, lo + n, dtype=np.int64).astype(np.int32).view(np.float32)
    return d, h


def test_codec_e2m1_exhaustive(dev, orc):
    """The device E2M1 encoder (the conversion instruction the quantisers use) against the
    oracle's nearest-with-ties-to-even encoder on every float32 bit pattern except NaNs (the
    quantisers never convert a NaN: a non-finite input is an error of the call)."""
    chunk = 1 << 26
    for lo in range(-(1 << 31), 1 << 31, chunk):
        vd, vh = _bit_patterns(lo, chunk, dev)
        got = R.encode_e2m1(vd).cpu().numpy()
        ref = orc.e2m1_encode_array(vh)
        bad = np.nonzero((got != ref) & ~np.isnan(vh))[0]
        assert bad.size == 0, [(hex(int(vh[i:i + 1].view(np.uint32)[0])), int(got[i]), int(ref[i])) for i in bad[:8]]


def test_codec_e4m3_exhaustive_scale_range(dev, orc):
    """The device E4M3 scale encoder against the oracle on every non-negative float32 up to 2^9
    (bit patterns 0 .. 0x44000000): the scale rule feeds it RN(b / RN(6 s_g)) <= 448 (up to
    rounding), so this covers every input it can receive, saturation included."""
    end = 0x44000000 + 1
    chunk = 1 << 26
    for lo in range(0, end, chunk):
        n = min(chunk, end - lo)
        vd, vh = _bit_patterns(lo, n, dev)
        got = R.encode_e4m3(vd).cpu().numpy()
        ref = orc.e4m3_encode_array(vh)
        bad = np.nonzero(got != ref)[0]
        assert bad.size == 0, [(float(vh[i]), int(got[i]), int(ref[i])) for i in bad[:8]]


# ------------------------------------------------------------------------------------------ quantiser
def check_act_quant(dev, orc, x: np.ndarray, sel: np.ndarray, rows_padded=None):
    xd = to_dev(x, dev)
    seld = torch.from_numpy(sel.astype(np.int32)).to(dev) if sel.size else None
    st = R.new_status(dev)
    q, qr = R.nvfp4_quantize(xd, seld, rows_padded=rows_padded, status=st)
    torch.cuda.synchronize()
    R.check_status(st)
    s_ref = orc.global_scale(orc.amax_bf16(x))
    assert q.s_g.item() == float(s_ref)
    codes, S, rcodes, rS, _ = orc.act_quant_rac(x, s_ref, sel.astype(np.int32))
    gc, gS = logical(q)
    assert np.array_equal(gS, S), np.argwhere(gS != S)[:5]
    assert np.array_equal(gc, codes), np.argwhere(gc != codes)[:5]
    # padded rows are zero
    full_c, full_s = logical(q, rows=q.rows_padded)
    assert not full_c[x.shape[0]:].any() and not full_s[x.shape[0]:].any()
    if sel.size:
        assert qr.s_g.item() == float(s_ref)
        grc, grS = logical(qr)
        assert np.array_equal(grS, rS), np.argwhere(grS != rS)[:5]
        assert np.array_equal(grc, rcodes), np.argwhere(grc != rcodes)[:5]
    return q, qr


def test_quantize_tiny(dev, orc):
    wl = syn.dense_tiny()
    sel, _ = orc.calibrate(wl.x_cal, wl.Kp)
    check_act_quant(dev, orc, wl.x, sel)


def test_quantize_ragged_rows_and_tail(dev, orc):
    rng = np.random.default_rng(2)
    M, K = 200, 704  # 704 = 512 + 192: a ragged last iteration; 200 rows: a partial row block
    x = syn.normal_bf16(3, 1, M, K, 1.0, np.exp(rng.standard_normal(K)))
    x[5] = 0  # an all-zero row
    sel = np.sort(rng.choice(K, 192, replace=False)).astype(np.int32)
    check_act_quant(dev, orc, x, sel)
    check_act_quant(dev, orc, x, np.zeros(0, np.int32), rows_padded=384)


def test_quantize_zero_tensor(dev, orc):
    x = np.zeros((64, 128), np.uint16)
    q, qr = check_act_quant(dev, orc, x, np.arange(0, 128, 2, dtype=np.int32))
    assert q.s_g.item() == 0.0


def test_quantize_dense_prefill_full(dev, orc):
    wl = syn.dense_prefill()
    sel, _ = orc.calibrate(wl.x_cal[:256], wl.Kp)  # any ascending set of the right size
    check_act_quant(dev, orc, wl.x, sel)


def test_quantize_row_gather(dev, orc):
    wl = syn.moe_block(T=300, H=1024, E=16, topk=4, I=256, T_cal=64, materialize_weights=False)
    g, off, pair_rows = L.gather_map(wl.pair_token, wl.counts)
    xd = to_dev(wl.x, dev)
    sel = np.arange(1, 1024, 2, dtype=np.int32)
    gd = torch.from_numpy(g).to(dev)
    q, qr = R.nvfp4_quantize(xd, torch.from_numpy(sel).to(dev), row_gather=gd, M_out=g.size)
    torch.cuda.synchronize()
    s_ref = orc.global_scale(orc.amax_bf16(wl.x))
    rows_x = np.where(g >= 0, g, 0)
    xg = wl.x[rows_x].copy()
    xg[g < 0] = 0
    codes, S, rcodes, rS, _ = orc.act_quant_rac(xg, s_ref, sel)
    gc, gS = logical(q)
    grc, grS = logical(qr)
    assert np.array_equal(gc, codes) and np.array_equal(gS, S)
    assert np.array_equal(grc, rcodes) and np.array_equal(grS, rS)


def test_quantize_scatter_matches_gather(dev, orc):
    """Scatter mode (each token quantised once, written to its expert rows) gives the same bytes
    as the gather mode and as the oracle; unnamed (padding) rows stay zero."""
    wl = syn.moe_block(T=300, H=1024, E=16, topk=4, I=256, T_cal=64, materialize_weights=False)
    g, off, pair_rows = L.gather_map(wl.pair_token, wl.counts)
    sm = L.scatter_map(wl.pair_token, pair_rows, wl.x.shape[0], 4)
    xd = to_dev(wl.x, dev)
    sel = np.arange(3, 1024, 2, dtype=np.int32)[:448]
    seld = torch.from_numpy(sel).to(dev)
    qg, qgr = R.nvfp4_quantize(xd, seld, row_gather=torch.from_numpy(g).to(dev), M_out=g.size)
    qs, qsr = R.nvfp4_quantize_scatter(xd, torch.from_numpy(sm).to(dev), g.size, seld)
    torch.cuda.synchronize()
    assert torch.equal(qg.codes, qs.codes) and torch.equal(qg.sf, qs.sf) and torch.equal(qg.s_g, qs.s_g)
    assert torch.equal(qgr.codes, qsr.codes) and torch.equal(qgr.sf, qsr.sf)
    s_ref = orc.global_scale(orc.amax_bf16(wl.x))
    codes, S, rcodes, rS, _ = orc.act_quant_rac(wl.x, s_ref, sel)
    gc, gS = logical(qs, rows=qs.rows_padded)
    assert np.array_equal(gc[pair_rows], codes[wl.pair_token]) and np.array_equal(gS[pair_rows], S[wl.pair_token])
    grc, grS = logical(qsr, rows=qsr.rows_padded)
    assert np.array_equal(grc[pair_rows], rcodes[wl.pair_token])
    pad = np.ones(qs.rows_padded, bool)
    pad[pair_rows] = False
    assert not gc[pad].any() and not gS[pad].any() and not grc[pad].any()


# ------------------------------------------------------------------------------------------ calibration
@pytest.mark.parametrize("shape", [(64, 256, 128), (2048, 4096, 2048), (100, 704, 320)])
def test_calibrate_matches_oracle(dev, orc, shape):
    T, K, Kp = shape
    rng = np.random.default_rng(T)
    x = syn.normal_bf16(5, 3, T, K, 1.0, np.exp(rng.standard_normal(K)))
    sel_ref, err_ref = orc.calibrate(x, Kp)
    sel, err = R.rac_calibrate(to_dev(x, dev), Kp, want_err=True)
    torch.cuda.synchronize()
    assert np.array_equal(err.cpu().numpy(), err_ref)
    assert np.array_equal(sel.cpu().numpy(), sel_ref)


def test_calibrate_full_ratio_selects_all(dev):
    x = syn.normal_bf16(1, 3, 32, 256, 1.0)
    sel, _ = R.rac_calibrate(to_dev(x, dev), 256)
    assert np.array_equal(sel.cpu().numpy(), np.arange(256))


# ------------------------------------------------------------------------------------------ weights
@pytest.mark.parametrize("interleave", [False, True])
def test_pack_weights_matches_oracle(dev, orc, interleave):
    E, N, K, Kp = 3, 256, 512, 256
    w = syn.normal_bf16(0, 2, E * N, K, 0.02).reshape(E, N, K)
    w[1] *= 0  # an all-zero expert: s_g = 0
    sel = np.sort(np.random.default_rng(9).choice(K, Kp, replace=False)).astype(np.int32)
    wq, wsq = R.pack_weights(to_dev(w, dev), torch.from_numpy(sel).to(dev), gate_up_interleave=interleave)
    torch.cuda.synchronize()
    for e in range(E):
        s_ref = orc.global_scale(orc.amax_bf16(w[e]))
        assert wq.s_g[e].item() == float(s_ref) and wsq.s_g[e].item() == float(s_ref)
        we = w[e]
        if interleave:
            p = np.arange(N)
            q, j = p // 128, p % 128
            src = np.where(j < 64, q * 64 + j, N // 2 + q * 64 + j - 64)
            we = we[src]
        c, S, sc, sS = orc.weight_pack(we, s_ref, sel)
        gc, gS = logical(wq, e)
        gsc, gsS = logical(wsq, e)
        assert np.array_equal(gc, c) and np.array_equal(gS, S)
        assert np.array_equal(gsc, sc) and np.array_equal(gsS, sS)


def test_weight_qdq_matches_oracle(dev, orc):
    n, elems = 5, 4096 + 16 * 3
    w = syn.normal_bf16(0, 9, n, elems, 0.02)
    w[2, :96] = syn.normal_bf16(0, 10, 1, 96, 1.28)[0]  # one tensor with a heavier head
    out, s_g = R.weight_qdq(to_dev(w, dev))
    torch.cuda.synchronize()
    got = bf16_bits(out).reshape(n, elems)
    for t in range(n):
        ref, s_ref = orc.weight_qdq(w[t])
        assert s_g[t].item() == float(s_ref)
        assert np.array_equal(got[t], ref), np.argwhere(got[t] != ref)[:5]


@pytest.mark.parametrize("n,elems", [(3, 16), (300, 512 * 7 + 16), (7, 512 * 5), (2, 2 << 20)])
def test_weight_qdq_shapes_match_oracle(dev, orc, n, elems):
    """Tensor boundaries inside and at the edges of 512-element chunks, tiny and 4 MB tensors."""
    w = syn.normal_bf16(1, 9, n, elems, 0.02)
    h = min(32, elems)
    w[0, :h] = syn.normal_bf16(1, 10, 1, h, 1.28)[0]  # a heavier head in one tensor
    out, s_g = R.weight_qdq(to_dev(w, dev))
    torch.cuda.synchronize()
    got = bf16_bits(out).reshape(n, elems)
    for t in sorted({0, 1 % n, n // 2, n - 1}):
        ref, s_ref = orc.weight_qdq(w[t])
        assert s_g[t].item() == float(s_ref)
        assert np.array_equal(got[t], ref), (t, np.argwhere(got[t] != ref)[:5])


def test_weight_qdq_trainer_full_sampled(dev, orc):
    """The trainer fake-quant configuration at full size: 2^31 bf16 N(0, 0.02) weights as 1024
    tensors of 1024 x 2048 (one scale each), then as a single tensor (one scale); sampled tensors
    and chunks against the oracle, every per-tensor scale exact."""
    w = syn.trainer_weights()
    n, elems = w.shape
    wd = to_dev(w, dev)
    out, s_g = R.weight_qdq(wd)
    torch.cuda.synchronize()
    s_all = s_g.cpu().numpy()
    for t in range(n):
        assert s_all[t] == orc.global_scale(orc.amax_bf16(w[t:t + 1]))
    for t in (0, 1, 511, n - 1):
        ref, s_ref = orc.weight_qdq(w[t])
        assert s_all[t] == s_ref
        got = bf16_bits(out[t])
        assert np.array_equal(got, ref), (t, np.argwhere(got != ref)[:5])
    # one tensor of 2^31 elements: a single scale over everything (int64 indexing throughout)
    out1, s1 = R.weight_qdq(wd.view(1, -1), out=out.view(1, -1))
    torch.cuda.synchronize()
    s_ref = orc.global_scale(orc.amax_bf16(w))
    assert s1.item() == float(s_ref)
    flat = out1.view(-1)
    for start in (0, (1 << 30) + 48, (1 << 31) - (1 << 20)):
        chunk = w.reshape(-1)[start:start + (1 << 20)]
        ref, _ = orc.weight_qdq(chunk, s_ref)
        got = bf16_bits(flat[start:start + (1 << 20)])
        assert np.array_equal(got, ref), (start, np.argwhere(got != ref)[:5])


def test_shared_weight_path_gpu(dev):
    """DQ(pack_weights(W)) == weight_qdq(W), bitwise, both computed on the GPU."""
    N, K = 256, 1024
    w = syn.normal_bf16(4, 2, N, K, 0.02)
    wd = to_dev(w, dev)
    wq, _ = R.pack_weights(wd)
    fq, s_g = R.weight_qdq(wd.reshape(1, -1))
    torch.cuda.synchronize()
    c, S = logical(wq)
    mag = np.array([0, .5, 1, 1.5, 2, 3, 4, 6], np.float32)
    e = mag[c & 7] * np.where(c & 8, np.float32(-1), np.float32(1))
    from oracle import e4m3_decode  # decode table only

    table = np.array([e4m3_decode(i) if i != 0x7F else np.nan for i in range(128)], np.float32)
    d = (table[S] * np.float32(wq.s_g[0].item())).astype(np.float32)
    dq = (e * np.repeat(d, 16, axis=1)).astype(np.float32)
    ref = torch.from_numpy(dq).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(bf16_bits(fq).reshape(N, K), ref)


# ------------------------------------------------------------------------------------------ GEMM
def run_dense(dev, orc, x, w, x_cal, Kp, out_dtype, rows=None):
    sel_np, _ = orc.calibrate(x_cal, Kp)
    sel_gpu, _ = R.rac_calibrate(to_dev(x_cal, dev), Kp)
    assert np.array_equal(sel_gpu.cpu().numpy(), sel_np)
    xd, wd = to_dev(x, dev), to_dev(w, dev)
    st = R.new_status(dev)
    q, qr = R.nvfp4_quantize(xd, sel_gpu if Kp else None, status=st)
    wq, wsq = R.pack_weights(wd, sel_gpu if Kp else None, status=st)
    y = R.w4a4_rac_gemm(q, qr, wq, wsq, x.shape[0], out_dtype=out_dtype, status=st)
    torch.cuda.synchronize()
    R.check_status(st)
    f = orc.dense_rac_forward(x, w, sel_np if Kp else np.zeros(0, np.int32), rows=rows)
    yg = y.float().cpu().numpy()
    if rows is not None:
        yg = yg[rows]
    assert_gemm_close(yg, f["y"], f["absdot"], out_dtype == torch.bfloat16)
    return y, f


def test_gemm_tiny_fp32(dev, orc):
    wl = syn.dense_tiny()
    run_dense(dev, orc, wl.x, wl.w, wl.x_cal, wl.Kp, torch.float32)


def test_gemm_tiny_r0_is_plain_w4a4(dev, orc):
    wl = syn.dense_tiny()
    run_dense(dev, orc, wl.x, wl.w, wl.x_cal, 0, torch.float32)


@pytest.mark.parametrize("M,N,K,Kp", [(300, 384, 768, 384), (128, 256, 320, 64), (520, 512, 1024, 1024)])
def test_gemm_ragged_shapes(dev, orc, M, N, K, Kp):
    rng = np.random.default_rng(M + N)
    cs = np.exp(rng.standard_normal(K))
    x = syn.normal_bf16(11, 1, M, K, 1.0, cs)
    w = syn.normal_bf16(11, 2, N, K, 0.02)
    x_cal = syn.normal_bf16(11, 3, 128, K, 1.0, cs)
    run_dense(dev, orc, x, w, x_cal, Kp, torch.float32)
    run_dense(dev, orc, x, w, x_cal, Kp, torch.bfloat16)


def tile_order_blocks(m_blocks: int, n_blocks: int, grid: int = 148):
    """128-row m-blocks spread over a persistent GEMM's tile order (grid CTAs; tile
    t = m_block * n_blocks + n_block runs on CTA t % grid as its (t // grid)-th tile, into
    accumulator buffer (t // grid) % 2): the first and the last m-block, the middle one, and the
    m-blocks holding the first tiles of the CTAs' second and third turns."""
    picks = {0, m_blocks - 1, m_blocks // 2}
    for turn in (1, 2):
        picks.add(min(m_blocks - 1, (turn * grid + n_blocks - 1) // n_blocks))
    return sorted(picks)


def test_gemm_dense_prefill_sampled(dev, orc):
    """The dense prefill projection at full size: every row of whole m-blocks spread over the
    tile order (both accumulator buffers, first and last tiles of CTAs)."""
    wl = syn.dense_prefill()
    blocks = tile_order_blocks(wl.M // 128, wl.N // 256)
    assert len(blocks) >= 4
    rows = np.concatenate([np.arange(128 * b, 128 * b + 128) for b in blocks])
    run_dense(dev, orc, wl.x, wl.w, wl.x_cal, wl.Kp, torch.bfloat16, rows=rows)


# ------------------------------------------------------------------------------------------ MoE
def moe_pipeline(dev, wl, sel_gu, sel_dn):
    g, off, pair_rows = L.gather_map(wl.pair_token, wl.counts)
    st = R.new_status(dev)
    offd = torch.from_numpy(off.astype(np.int32)).to(dev)
    wgu = to_dev(wl.wgu, dev)
    wdn = to_dev(wl.wdn, dev)
    seld_gu = torch.from_numpy(sel_gu).to(dev)
    seld_dn = torch.from_numpy(np.ascontiguousarray(sel_dn)).to(dev)  # 2-D: one list per expert
    pgu, pgus = R.pack_weights(wgu, seld_gu, gate_up_interleave=True, status=st)
    pdn, pdns = R.pack_weights(wdn, seld_dn, status=st)
    sm = torch.from_numpy(L.scatter_map(wl.pair_token, pair_rows, wl.x.shape[0], wl.topk_ids.shape[1])).to(dev)
    a, ar = R.nvfp4_quantize_scatter(to_dev(wl.x, dev), sm, g.size, seld_gu, status=st)
    h, amax_h = R.grouped_w4a4_rac_moe(a, ar, offd, pgu, pgus, swiglu=True, status=st)
    row_group = R.moe_row_groups(offd, wl.E, g.size) if seld_dn.dim() == 2 else None
    hq, hqr = R.nvfp4_quantize(h, seld_dn, amax_in=amax_h, status=st, row_group=row_group)
    y = R.grouped_w4a4_rac_moe(hq, hqr, offd, pdn, pdns, status=st)
    torch.cuda.synchronize()
    R.check_status(st)
    return dict(g=g, off=off, pair_rows=pair_rows, a=a, ar=ar, h=h, amax_h=amax_h, hq=hq, hqr=hqr, y=y, pgu=pgu,
                pdn=pdn)


def check_moe(orc, wl, sel_gu, sel_dn, out, sample_pairs, wgu_of=None, wdn_of=None):
    """Sampled (token, expert) rows of an MoE pipeline against the oracle.  wgu_of / wdn_of give
    an expert's bf16 weight bits (default: the workload's host copies)."""
    wgu_of = wgu_of or wl.gate_up_expert
    wdn_of = wdn_of or wl.down_expert
    I, H = wl.I, wl.H
    s_x = orc.global_scale(orc.amax_bf16(wl.x))
    assert out["a"].s_g.item() == float(s_x)
    h_gpu = bf16_bits(out["h"])
    # amax of the SwiGLU output over the real rows equals the device amax; padding rows are 0
    valid = np.zeros(h_gpu.shape[0], bool)
    valid[out["pair_rows"]] = True
    assert not h_gpu[~valid].any()
    hv = syn.bf16_to_f32(h_gpu[valid])
    assert np.float32(np.abs(hv).max()) == np.float32(out["amax_h"].item())
    s_h = orc.global_scale(np.float32(out["amax_h"].item()))
    assert out["hq"].s_g.item() == float(s_h)
    gq_c, gq_S = logical(out["hq"], rows=out["hq"].rows_padded)
    if out["hqr"] is not None:
        gqr_c, gqr_S = logical(out["hqr"], rows=out["hqr"].rows_padded)
    for e in sorted(set(int(wl.pair_expert[i]) for i in sample_pairs)):
        pidx = [i for i in sample_pairs if wl.pair_expert[i] == e]
        rows = out["pair_rows"][pidx]
        toks = wl.pair_token[pidx]
        # gate_up on the oracle: quantise the token rows, exact GEMM against the expert's weights
        xa = wl.x[toks]
        a_c, a_S, r_c, r_S, _ = orc.act_quant_rac(xa, s_x, sel_gu)
        wgu = wgu_of(e)
        s_w = orc.global_scale(orc.amax_bf16(wgu))
        wc, wS, wsc, wsS = orc.weight_pack(wgu, s_w, sel_gu)
        gu, ad = orc.gemm_rac(a_c, a_S, r_c, r_S, wc, wS, wsc, wsS, s_x, s_w)
        # bound on h from the GEMM bound on g and u
        tol_gu = 1e-3 * ad + 1e-6 + bf16_ulp(gu)
        g, u = gu[:, :I], gu[:, I:]
        tg, tu = tol_gu[:, :I], tol_gu[:, I:]
        sig = 1.0 / (1.0 + np.exp(-g))
        silu = g * sig
        dsilu = np.abs(sig * (1 + g * (1 - sig))) + 0.1
        h_ref = silu * u
        tol_h = 2.0 * (dsilu * tg * (np.abs(u) + tu) + np.abs(silu) * tu) + 2 * bf16_ulp(h_ref) + 1e-30
        h_g = syn.bf16_to_f32(h_gpu[rows]).astype(np.float64)
        bad = np.argwhere(np.abs(h_g - h_ref) > tol_h)
        assert bad.size == 0, (e, bad[:5], h_g[tuple(bad[0])], h_ref[tuple(bad[0])])
        # down: the GPU's h rows quantised by the oracle must match the GPU codes bit for bit
        sel_e = sel_dn[e] if sel_dn.ndim == 2 else sel_dn  # per-expert lists: the expert's own
        hrows = h_gpu[rows]
        hc, hS, hrc, hrS, _ = orc.act_quant_rac(hrows, s_h, sel_e)
        assert np.array_equal(gq_c[rows], hc) and np.array_equal(gq_S[rows], hS)
        if out["hqr"] is not None:
            assert np.array_equal(gqr_c[rows], hrc) and np.array_equal(gqr_S[rows], hrS)
        else:
            assert len(sel_e) == 0
        wdn = wdn_of(e)
        s_wd = orc.global_scale(orc.amax_bf16(wdn))
        dc, dS, dsc, dsS = orc.weight_pack(wdn, s_wd, sel_e)
        y_ref, ad2 = orc.gemm_rac(hc, hS, hrc, hrS, dc, dS, dsc, dsS, s_h, s_wd)
        y_g = out["y"][torch.from_numpy(rows).to(out["y"].device)].float().cpu().numpy()
        assert_gemm_close(y_g, y_ref, ad2, True)


def test_moe_small_ragged(dev, orc):
    """Small MoE block with empty, single-row and >128-row experts."""
    wl = syn.moe_block(T=96, H=512, E=8, topk=2, I=128, T_cal=64)
    # force a skewed routing: expert 7 gets nothing, expert 0 gets most tokens
    wl.topk_ids[:, 0] = np.where(np.arange(96) % 3 == 0, 0, wl.topk_ids[:, 0])
    wl.topk_ids[wl.topk_ids == 7] = 6
    wl.topk_ids[:, 1] = np.where(wl.topk_ids[:, 1] == wl.topk_ids[:, 0], (wl.topk_ids[:, 0] + 1) % 7,
                                 wl.topk_ids[:, 1])
    wl.pair_token, wl.pair_expert, wl.counts = syn.sort_pairs(wl.topk_ids, wl.E)
    assert wl.counts[7] == 0
    sel_gu, _ = orc.calibrate(wl.x_cal, wl.Kp_gu)
    h_cal = syn.moe_down_calibration_batch(wl)
    sel_dn, _ = orc.calibrate(h_cal, wl.Kp_dn)
    out = moe_pipeline(dev, wl, sel_gu, sel_dn)
    check_moe(orc, wl, sel_gu, sel_dn, out, list(range(wl.pair_token.size)))


def test_moe_per_expert_down_lists(dev, orc):
    """The per-expert variant: the down projection's channel lists come from each expert's own
    calibration rows (GPU calibration bit-exact against the oracle), the weights are packed with
    them, h is quantised with its row's list, and the outputs match the oracle per expert."""
    wl = syn.moe_block(T=96, H=512, E=8, topk=2, I=128, T_cal=64)
    sel_gu, _ = orc.calibrate(wl.x_cal, wl.Kp_gu)
    h_cal = syn.moe_down_calibration_batch(wl)
    off_cal = syn.moe_down_calibration_offsets(wl)
    sel_dn, err_dn = orc.calibrate_grouped(h_cal, off_cal, wl.Kp_dn)
    gsel, gerr = R.rac_calibrate_grouped(to_dev(h_cal, dev), torch.from_numpy(off_cal.astype(np.int32)).to(dev),
                                         wl.Kp_dn, want_err=True)
    torch.cuda.synchronize()
    assert np.array_equal(gerr.cpu().numpy(), err_dn) and np.array_equal(gsel.cpu().numpy(), sel_dn)
    assert len({tuple(r) for r in sel_dn}) > 1  # the lists really differ between experts
    out = moe_pipeline(dev, wl, sel_gu, sel_dn)
    check_moe(orc, wl, sel_gu, sel_dn, out, list(range(wl.pair_token.size)))
    # padding rows (row group -1) carry an all-zero residual
    gqr_c, gqr_S = logical(out["hqr"], rows=out["hqr"].rows_padded)
    pad = np.ones(gqr_c.shape[0], bool)
    pad[out["pair_rows"]] = False
    assert not gqr_c[pad].any() and not gqr_S[pad].any()


@pytest.mark.parametrize("which", ["tiny", "ragged", "aligned_full"])
def test_masked_residual_variant_matches_oracle(dev, orc, which):
    """The masked full-K residual variant: codes and scales bit-exact, and the GEMM with the main
    packed weight as the residual weight within the GEMM tolerance."""
    if which == "tiny":
        wl = syn.dense_tiny()
        x, w = wl.x, wl.w
        sel, _ = orc.calibrate(wl.x_cal, wl.Kp)
    else:
        x = syn.normal_bf16(2, 1, 300, 1024, 1.0, syn.outlier_colscale(2, 1024))
        w = syn.normal_bf16(2, 2, 384, 1024, 0.02)
        sel = np.arange(5, 1024, 3, dtype=np.int32)[:320] if which == "ragged" else np.arange(1024, dtype=np.int32)
    s_x = orc.global_scale(orc.amax_bf16(x))
    st = R.new_status(dev)
    seld = torch.from_numpy(sel).to(dev)
    q, qm = R.nvfp4_quantize(to_dev(x, dev), seld, masked=True, status=st)
    wq, _ = R.pack_weights(to_dev(w, dev), status=st)
    y = R.w4a4_rac_gemm(q, qm, wq, wq, x.shape[0], out_dtype=torch.float32, status=st)
    torch.cuda.synchronize()
    R.check_status(st)
    c, S, mc, mS = orc.act_quant_masked(x, s_x, sel)
    gc, gS = logical(q)
    gmc, gmS = logical(qm)
    assert np.array_equal(gc, c) and np.array_equal(gS, S)
    assert np.array_equal(gmc, mc) and np.array_equal(gmS, mS), np.argwhere(gmc != mc)[:5]
    y_ref, ad = orc.masked_rac_forward(x, w, sel)
    assert_gemm_close(y.cpu().numpy(), y_ref, ad, False)


def test_grouped_expert_rows_skips_padding_boxes(dev, orc):
    """With per-expert token counts, output boxes of padding only keep their old contents, every
    token row is bit-identical to the call without counts, and the SwiGLU amax is unchanged."""
    wl = syn.moe_block(T=300, H=512, E=6, topk=2, I=128, T_cal=64)
    sel_gu, _ = orc.calibrate(wl.x_cal, wl.Kp_gu)
    st = R.new_status(dev)
    g, off, pair_rows = L.gather_map(wl.pair_token, wl.counts)
    seld = torch.from_numpy(sel_gu).to(dev)
    a, ar = R.nvfp4_quantize(to_dev(wl.x, dev), seld, row_gather=torch.from_numpy(g).to(dev), M_out=g.size, status=st)
    w, ws = R.pack_weights(to_dev(wl.wgu, dev), seld, gate_up_interleave=True, status=st)
    offd = torch.from_numpy(off.astype(np.int32)).to(dev)
    rows = torch.from_numpy(np.asarray(wl.counts, dtype=np.int32)).to(dev)
    for swiglu in (False, True):
        ycols = wl.I if swiglu else 2 * wl.I
        y_ref = torch.full((a.rows_padded, ycols), 7.0, dtype=torch.bfloat16, device=dev)
        y_new = y_ref.clone()
        out_ref = R.grouped_w4a4_rac_moe(a, ar, offd, w, ws, swiglu=swiglu, y=y_ref, status=st)
        out_new = R.grouped_w4a4_rac_moe(a, ar, offd, w, ws, swiglu=swiglu, y=y_new, status=st, expert_rows=rows)
        torch.cuda.synchronize()
        R.check_status(st)
        tok = torch.from_numpy(pair_rows).to(dev)
        assert torch.equal(y_new[tok].view(torch.int16), y_ref[tok].view(torch.int16))
        if swiglu:
            assert out_new[1].item() == out_ref[1].item()
        yn = y_new.float().cpu().numpy()
        for e in range(wl.E):
            lo, n = int(off[e]), int(wl.counts[e])
            live_end = lo + (n + 31) // 32 * 32 if n else lo  # boxes that hold a token row
            assert np.all(yn[live_end:int(off[e + 1])] == 7.0), e      # padding boxes untouched
            assert np.all(yn[lo + n:live_end] == 0.0), e               # padding rows of live boxes


def whole_block_pairs(pair_rows: np.ndarray, rows_padded: int, n_blocks: int, grid: int = 148):
    """The (token, expert) pairs whose rows lie in the m-blocks tile_order_blocks picks for the
    grouped GEMM: every token row of those blocks."""
    picks = tile_order_blocks(rows_padded // 128, n_blocks, grid)
    pairs = np.nonzero(np.isin(pair_rows // 128, picks))[0]
    return picks, pairs.tolist()


def test_moe_prefill_full_sampled(dev, orc):
    """The MoE prefill block at full size, r = 0.5: every row of whole m-blocks spread over the
    tile order (both accumulator buffers, first and last tiles) plus random pairs."""
    wl = syn.moe_prefill()
    sel_gu, _ = orc.calibrate(wl.x_cal, wl.Kp_gu)
    h_cal = syn.moe_down_calibration_batch(wl)
    sel_dn, _ = orc.calibrate(h_cal, wl.Kp_dn)
    out = moe_pipeline(dev, wl, sel_gu, sel_dn)
    rng = np.random.default_rng(0)
    P = wl.pair_token.size
    blocks, pairs = whole_block_pairs(out["pair_rows"], out["g"].size, 1536 // 256)
    assert len(blocks) >= 4 and len(pairs) >= 3 * 100
    sample = sorted(set(rng.choice(P, 96, replace=False).tolist() + [0, P - 1] + pairs))
    check_moe(orc, wl, sel_gu, sel_dn, out, sample)


@pytest.mark.parametrize("r", [0.0, 0.25, 1.0])
def test_moe_prefill_ratio_sweep_matches_oracle(dev, orc, r):
    """The RAC ratio sweep on the MoE prefill shapes (r = 0 is plain W4A4, K' = 0 in both GEMMs;
    r = 0.25 gives K' = 512 / 192, a partial last residual k-tile in the down GEMM; r = 1 the
    residual over every channel): every row of whole m-blocks spread over the tile order
    against the oracle, as at r = 0.5."""
    import dataclasses

    base = syn.moe_prefill()
    wl = dataclasses.replace(base, r=r, Kp_gu=syn.kp_from_ratio(base.H, r), Kp_dn=syn.kp_from_ratio(base.I, r))
    empty = np.zeros(0, np.int32)
    sel_gu = orc.calibrate(wl.x_cal, wl.Kp_gu)[0] if wl.Kp_gu else empty
    sel_dn = orc.calibrate(syn.moe_down_calibration_batch(wl), wl.Kp_dn)[0] if wl.Kp_dn else empty
    out = moe_pipeline(dev, wl, sel_gu, sel_dn)
    if wl.Kp_gu == 0:
        assert out["ar"] is None and out["hqr"] is None
    blocks, pairs = whole_block_pairs(out["pair_rows"], out["g"].size, 1536 // 256)
    assert len(blocks) >= 4
    check_moe(orc, wl, sel_gu, sel_dn, out, pairs + [0, wl.pair_token.size - 1])


# ------------------------------------------------------------------------------------------ MoE decode
def decode_pipeline(dev, wl, sel_gu, sel_dn, packed, counts=None):
    """quantise (scatter into 16-token expert slabs) -> decode gate_up + SwiGLU -> quantise h ->
    decode down, all through the C ABI."""
    st = R.new_status(dev)
    pgu, pgus, pdn, pdns = packed
    counts = wl.counts if counts is None else counts
    se, sc, pair_rows = L.decode_slots(counts)
    rows = 16 * se.size
    sed = torch.from_numpy(se).to(dev)
    scd = torch.from_numpy(sc).to(dev)
    seld_gu = torch.from_numpy(sel_gu).to(dev) if sel_gu.size else None
    seld_dn = torch.from_numpy(sel_dn).to(dev) if sel_dn.size else None
    sm = torch.from_numpy(L.scatter_map(wl.pair_token, pair_rows, wl.x.shape[0], wl.topk_ids.shape[1])).to(dev)
    a, ar = R.nvfp4_quantize_scatter(to_dev(wl.x, dev), sm, rows, seld_gu, status=st, sf_layout=R.SF_SLAB16)
    h, amax_h = R.grouped_w4a4_rac_moe_decode(a, ar, sed, scd, pgu, pgus, swiglu=True, status=st)
    hq = R.Packed.empty(rows, wl.I, rows_padded=rows, device=dev, sf_layout=R.SF_SLAB16)
    hqr = R.Packed.empty(rows, sel_dn.size, rows_padded=rows, device=dev, sf_layout=R.SF_SLAB16) if sel_dn.size \
        else None
    R.nvfp4_quantize(h, seld_dn, amax_in=amax_h, out=hq, out_res=hqr, status=st)
    y = R.grouped_w4a4_rac_moe_decode(hq, hqr, sed, scd, pdn, pdns, status=st)
    torch.cuda.synchronize()
    R.check_status(st)
    return dict(pair_rows=pair_rows, slot_expert=se, slot_count=sc, a=a, ar=ar, h=h, amax_h=amax_h, hq=hq, hqr=hqr,
                y=y)


def pack_host_weights(dev, wl, sel_gu, sel_dn):
    st = R.new_status(dev)
    seld_gu = torch.from_numpy(sel_gu).to(dev) if sel_gu.size else None
    seld_dn = torch.from_numpy(sel_dn).to(dev) if sel_dn.size else None
    pgu, pgus = R.pack_weights(to_dev(wl.wgu, dev), seld_gu, gate_up_interleave=True, status=st)
    pdn, pdns = R.pack_weights(to_dev(wl.wdn, dev), seld_dn, status=st)
    torch.cuda.synchronize()
    R.check_status(st)
    return pgu, pgus, pdn, pdns


def skewed_decode_workload():
    """Decode-sized routing with every slab shape: experts with 1, 4, 7, 16, 17 and 33 tokens
    and experts with none."""
    wl = syn.moe_block(T=40, H=1024, E=12, topk=2, I=256, T_cal=64)
    ids = np.zeros((40, 2), np.int64)
    ids[:, 0] = np.repeat([0, 1, 2], [17, 16, 7])          # 17, 16 tokens
    ids[:33, 1] = 3                                       # 33 tokens
    ids[33:, 1] = np.array([4, 4, 4, 4, 5, 6, 11])        # 4 tokens, singles; 7..10 empty
    ids[33:40, 0] = np.where(ids[33:40, 1] == 4, 2, ids[33:40, 0])
    wl.topk_ids = ids
    wl.pair_token, wl.pair_expert, wl.counts = syn.sort_pairs(ids, wl.E)
    return wl


def test_decode_small_every_slab_shape(dev, orc):
    wl = skewed_decode_workload()
    assert {1, 16, 17, 33}.issubset(set(wl.counts.tolist())) and (wl.counts == 0).any()
    sel_gu, _ = orc.calibrate(wl.x_cal, wl.Kp_gu)
    sel_dn, _ = orc.calibrate(syn.moe_down_calibration_batch(wl), wl.Kp_dn)
    out = decode_pipeline(dev, wl, sel_gu, sel_dn, pack_host_weights(dev, wl, sel_gu, sel_dn))
    check_moe(orc, wl, sel_gu, sel_dn, out, list(range(wl.pair_token.size)))
    # rows of a slab past its count come out as zeros in both projections
    y = bf16_bits(out["y"])
    valid = np.zeros(y.shape[0], bool)
    valid[out["pair_rows"]] = True
    assert not y[~valid].any()


@pytest.mark.parametrize("r", [0.0, 0.5])
def test_decode_plain_epilogue_fp32(dev, orc, r):
    """No-SwiGLU epilogue with FP32 output (the tolerance without the bf16 ulp), r = 0 included."""
    wl = skewed_decode_workload()
    Kp = syn.kp_from_ratio(wl.H, r)
    sel = orc.calibrate(wl.x_cal, Kp)[0] if Kp else np.zeros(0, np.int32)
    st = R.new_status(dev)
    seld = torch.from_numpy(sel).to(dev) if Kp else None
    w, ws = R.pack_weights(to_dev(wl.wgu, dev), seld, status=st)
    se, sc, pair_rows = L.decode_slots(wl.counts)
    sm = torch.from_numpy(L.scatter_map(wl.pair_token, pair_rows, wl.x.shape[0], 2)).to(dev)
    a, ar = R.nvfp4_quantize_scatter(to_dev(wl.x, dev), sm, 16 * se.size, seld, status=st, sf_layout=R.SF_SLAB16)
    y = R.grouped_w4a4_rac_moe_decode(a, ar, torch.from_numpy(se).to(dev), torch.from_numpy(sc).to(dev), w, ws,
                                      out_dtype=torch.float32, status=st)
    torch.cuda.synchronize()
    R.check_status(st)
    yg = y.cpu().numpy()
    s_x = orc.global_scale(orc.amax_bf16(wl.x))
    for e in np.nonzero(wl.counts)[0]:
        idx = np.nonzero(wl.pair_expert == e)[0]
        ac, aS, rc, rS, _ = orc.act_quant_rac(wl.x[wl.pair_token[idx]], s_x, sel)
        s_w = orc.global_scale(orc.amax_bf16(wl.wgu[e]))
        wc, wS, wsc, wsS = orc.weight_pack(wl.wgu[e], s_w, sel)
        y_ref, ad = orc.gemm_rac(ac, aS, rc, rS, wc, wS, wsc, wsS, s_x, s_w)
        assert_gemm_close(yg[pair_rows[idx]], y_ref, ad, False)


def test_decode_no_slots_and_bad_expert(dev):
    wl = skewed_decode_workload()
    st = R.new_status(dev)
    w, _ = R.pack_weights(to_dev(wl.wgu[:2], dev), status=st)
    a = R.Packed.empty(32, wl.H, rows_padded=32, device=dev, zero=True, sf_layout=R.SF_SLAB16)
    a.s_g.fill_(1.0)
    empty = torch.zeros(0, dtype=torch.int32, device=dev)
    y = R.grouped_w4a4_rac_moe_decode(a, None, empty, empty, w, None, status=st)
    assert y.shape[0] == 0
    torch.cuda.synchronize()
    R.check_status(st)
    # an expert index outside [0, E) stops the call with an error status; the context stays usable
    bad = torch.tensor([1, 2], dtype=torch.int32, device=dev)
    cnt = torch.tensor([16, 16], dtype=torch.int32, device=dev)
    R.grouped_w4a4_rac_moe_decode(a, None, bad, cnt, w, None, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 1
    assert float(torch.ones(8, device=dev).sum().item()) == 8.0


def test_moe_decode_full_sampled(dev, orc):
    """The decode configuration at full size (64 tokens, hidden 7168, 256 experts, top-8,
    intermediate 2048, r = 0.5), weights made on the device; sampled rows vs the oracle on
    the exact weight bytes the device used."""
    wl = syn.moe_decode()
    touched = np.nonzero(wl.counts)[0]
    st = R.new_status(dev)
    sel_gu, _ = orc.calibrate(wl.x_cal, wl.Kp_gu)
    h_cal = syn.moe_down_calibration_batch_torch(wl, dev, max_pairs=2048)
    sel_dn, _ = orc.calibrate(h_cal, wl.Kp_dn)
    seld_gu, seld_dn = torch.from_numpy(sel_gu).to(dev), torch.from_numpy(sel_dn).to(dev)
    N_gu = 2 * wl.I
    pgu = R.Packed.empty(N_gu, wl.H, slabs=wl.E, rows_padded=N_gu, device=dev)
    pgus = R.Packed.empty(N_gu, wl.Kp_gu, slabs=wl.E, rows_padded=N_gu, device=dev)
    pdn = R.Packed.empty(wl.H, wl.I, slabs=wl.E, rows_padded=wl.H, device=dev)
    pdns = R.Packed.empty(wl.H, wl.Kp_dn, slabs=wl.E, rows_padded=wl.H, device=dev)
    wbuf = torch.empty(N_gu, wl.H, dtype=torch.bfloat16, device=dev)
    dbuf = torch.empty(wl.H, wl.I, dtype=torch.bfloat16, device=dev)
    for e in touched:
        R.pack_weights(wl.gate_up_expert_torch(int(e), dev, out=wbuf), seld_gu, gate_up_interleave=True,
                       out=pgu.slab(int(e)), out_sel=pgus.slab(int(e)), status=st)
        R.pack_weights(wl.down_expert_torch(int(e), dev, out=dbuf), seld_dn, out=pdn.slab(int(e)),
                       out_sel=pdns.slab(int(e)), status=st)
    torch.cuda.synchronize()
    R.check_status(st)
    out = decode_pipeline(dev, wl, sel_gu, sel_dn, (pgu, pgus, pdn, pdns))
    rng = np.random.default_rng(1)
    P = wl.pair_token.size
    # the busiest expert, and a spread of others
    busiest = int(np.argmax(wl.counts))
    sample = set(np.nonzero(wl.pair_expert == busiest)[0].tolist())
    sample |= set(rng.choice(P, 10, replace=False).tolist()) | {0, P - 1}
    dev_bits = lambda t: bf16_bits(t.contiguous())
    check_moe(orc, wl, sel_gu, sel_dn, out, sorted(sample),
              wgu_of=lambda e: dev_bits(wl.gate_up_expert_torch(int(e), dev)),
              wdn_of=lambda e: dev_bits(wl.down_expert_torch(int(e), dev)))


# ------------------------------------------------------------------------------------------ failure path
def test_bounded_wait_reports_timeout(dev):
    st = R.new_status(dev)
    R.selftest_wait_timeout(1_000_000, st)  # 1 ms on a barrier nothing completes
    torch.cuda.synchronize()
    assert int(st.item()) == 6
    # the context is still usable
    x = torch.ones(4, device=dev)
    assert float(x.sum().item()) == 4.0


def test_range_error_reported(dev):
    x = np.zeros((16, 64), np.uint16)
    x[3, 5] = 0x7F80  # +inf
    st = R.new_status(dev)
    R.nvfp4_quantize(to_dev(x, dev), status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 4
