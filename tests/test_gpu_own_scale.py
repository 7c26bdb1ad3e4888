"""GPU parity of the own-scale residual variant (the residual R_sel quantised with its own tensor
scale s_r = amax(R_sel) / 2688, two accumulators in the GEMM) against the oracle: the quantise
calls for every row map (codes and scales bit-exact, s_r exact), the dense GEMM, the grouped
GEMM with the plain and the SwiGLU epilogue, and K' = 0."""
import numpy as np
import pytest
import torch

from nvfp4_w4a4_moe_02_b200 import nvfp4rac as R
from nvfp4_w4a4_moe_02_b200 import synthetic as syn
import nvfp4_layout as L
import test_gpu_parity as P

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    R.load()
    return torch.device("cuda:0")


def test_own_scale_quantise_rows_matches_oracle(dev, orc):
    M, K, Kp = 300, 1024, 384
    x = syn.normal_bf16(41, 1, M, K, 1.0, syn.outlier_colscale(41, K))
    sel = np.sort(np.random.default_rng(41).choice(K, Kp, replace=False)).astype(np.int32)
    st = R.new_status(dev)
    q, qr = R.nvfp4_quantize(P.to_dev(x, dev), torch.from_numpy(sel).to(dev), status=st, own_scale=True)
    torch.cuda.synchronize()
    R.check_status(st)
    s_x = orc.global_scale(orc.amax_bf16(x))
    c, S, rc, rS, s_r = orc.act_quant_rac_own(x, s_x, sel)
    assert q.s_g.item() == float(s_x) and qr.s_g.item() == float(s_r) and s_r != s_x
    gc, gS = P.logical(q)
    grc, grS = P.logical(qr)
    assert np.array_equal(gc, c) and np.array_equal(gS, S)
    assert np.array_equal(grc, rc) and np.array_equal(grS, rS)
    assert grS.max() == 0x7E  # the residual's own amax block


def test_own_scale_scatter_and_segments_match_oracle(dev, orc):
    wl = syn.moe_block(T=160, H=1024, E=8, topk=2, I=256, T_cal=64)
    sel_gu = orc.calibrate(wl.x_cal, wl.Kp_gu)[0]
    off, rows_padded, pair_rows = L.expert_layout(wl.counts, 128)
    sm = L.scatter_map(wl.pair_token, pair_rows, wl.x.shape[0], 2)
    st = R.new_status(dev)
    a, ar = R.nvfp4_quantize_scatter(P.to_dev(wl.x, dev), torch.from_numpy(sm).to(dev), rows_padded,
                                     torch.from_numpy(sel_gu).to(dev), status=st, own_scale=True)
    # segments: the token rows of a padded h
    I, Kd = wl.I, wl.Kp_dn
    h = syn.normal_bf16(42, 1, rows_padded, I, 0.3, syn.outlier_colscale(42, I))
    sel_dn = np.sort(np.random.default_rng(42).choice(I, Kd, replace=False)).astype(np.int32)
    amax_h = np.float32(orc.amax_bf16(h[pair_rows]))
    hq, hqr = R.nvfp4_quantize_segments(P.to_dev(h, dev), torch.from_numpy(off[:-1].astype(np.int32)).to(dev),
                                        torch.from_numpy(wl.counts.astype(np.int32)).to(dev),
                                        torch.from_numpy(sel_dn).to(dev), amax_in=torch.tensor([amax_h], device=dev),
                                        status=st, own_scale=True)
    torch.cuda.synchronize()
    R.check_status(st)
    s_x = orc.global_scale(orc.amax_bf16(wl.x))
    c, S, rc, rS, s_r = orc.act_quant_rac_own(wl.x, s_x, sel_gu)
    assert a.s_g.item() == float(s_x) and ar.s_g.item() == float(s_r)
    gc, gS = P.logical(a, rows=rows_padded)
    grc, grS = P.logical(ar, rows=rows_padded)
    tok = wl.pair_token
    assert np.array_equal(gc[pair_rows], c[tok]) and np.array_equal(gS[pair_rows], S[tok])
    assert np.array_equal(grc[pair_rows], rc[tok]) and np.array_equal(grS[pair_rows], rS[tok])
    s_h = orc.global_scale(amax_h)
    hc, hS, hrc, hrS, s_hr = orc.act_quant_rac_own(h[pair_rows], s_h, sel_dn)
    assert hq.s_g.item() == float(s_h) and hqr.s_g.item() == float(s_hr)
    gc, gS = P.logical(hq, rows=rows_padded)
    grc, grS = P.logical(hqr, rows=rows_padded)
    assert np.array_equal(gc[pair_rows], hc) and np.array_equal(gS[pair_rows], hS)
    assert np.array_equal(grc[pair_rows], hrc) and np.array_equal(grS[pair_rows], hrS)


@pytest.mark.parametrize("M,N,K,Kp", [(300, 384, 768, 384), (257, 256, 1024, 1024), (128, 128, 512, 0)])
def test_own_scale_dense_gemm_matches_oracle(dev, orc, M, N, K, Kp):
    rng = np.random.default_rng(M + K)
    x = syn.normal_bf16(43, 1, M, K, 1.0, np.exp(rng.standard_normal(K)))
    w = syn.normal_bf16(43, 2, N, K, 0.02)
    sel = np.sort(rng.choice(K, Kp, replace=False)).astype(np.int32)
    seld = torch.from_numpy(sel).to(dev) if Kp else None
    st = R.new_status(dev)
    q, qr = R.nvfp4_quantize(P.to_dev(x, dev), seld, status=st, own_scale=True)
    wq, wsq = R.pack_weights(P.to_dev(w, dev), seld, status=st)
    for dt in (torch.float32, torch.bfloat16):
        y = R.w4a4_rac_gemm(q, qr, wq, wsq, M, out_dtype=dt, status=st, own_scale=True)
        torch.cuda.synchronize()
        R.check_status(st)
        s_x = orc.global_scale(orc.amax_bf16(x))
        s_w = orc.global_scale(orc.amax_bf16(w))
        c, S, rc, rS, s_r = orc.act_quant_rac_own(x, s_x, sel)
        y_ref, ad = orc.gemm_rac_own(c, S, rc, rS, *orc.weight_pack(w, s_w, sel), s_x, s_r, s_w)
        P.assert_gemm_close(y.float().cpu().numpy(), y_ref, ad, dt == torch.bfloat16)


def test_own_scale_grouped_gemm_plain_and_swiglu(dev, orc):
    """Grouped gate_up with the own-scale residual: FP32 output against the oracle per expert, and
    the SwiGLU epilogue (64-byte boxes) equal to SwiGLU of the GPU's own FP32 output."""
    wl = syn.moe_block(T=200, H=512, E=6, topk=2, I=256, T_cal=64)
    sel = orc.calibrate(wl.x_cal, wl.Kp_gu)[0]
    g, off, pair_rows = L.gather_map(wl.pair_token, wl.counts)
    st = R.new_status(dev)
    seld = torch.from_numpy(sel).to(dev)
    a, ar = R.nvfp4_quantize(P.to_dev(wl.x, dev), seld, row_gather=torch.from_numpy(g).to(dev), M_out=g.size,
                             status=st, own_scale=True)
    w, ws = R.pack_weights(P.to_dev(wl.wgu, dev), seld, gate_up_interleave=True, status=st)
    offd = torch.from_numpy(off.astype(np.int32)).to(dev)
    y = R.grouped_w4a4_rac_moe(a, ar, offd, w, ws, out_dtype=torch.float32, status=st, own_scale=True)
    h, amax = R.grouped_w4a4_rac_moe(a, ar, offd, w, ws, swiglu=True, status=st, own_scale=True)
    torch.cuda.synchronize()
    R.check_status(st)
    # the residual scale of the gathered rows equals that of the token rows (gather duplicates rows)
    s_x = orc.global_scale(orc.amax_bf16(wl.x))
    _, _, _, _, s_r = orc.act_quant_rac_own(wl.x[wl.pair_token], s_x, sel)
    assert ar.s_g.item() == float(s_r)
    yg = y.cpu().numpy()
    n = np.arange(2 * wl.I)
    logical = np.where((n % 128) < 64, (n // 128) * 64 + n % 128, wl.I + (n // 128) * 64 + n % 128 - 64)
    for e in range(wl.E):
        idx = np.nonzero(wl.pair_expert == e)[0]
        if idx.size == 0:
            continue
        c, S, rc, rS, _ = orc.act_quant_rac_own(wl.x[wl.pair_token[idx]], s_x, sel, s_r=s_r)
        s_w = orc.global_scale(orc.amax_bf16(wl.wgu[e]))
        y_ref, ad = orc.gemm_rac_own(c, S, rc, rS, *orc.weight_pack(wl.wgu[e], s_w, sel), s_x, s_r, s_w)
        got = np.empty((idx.size, 2 * wl.I))
        got[:, logical] = yg[pair_rows[idx]]
        P.assert_gemm_close(got, y_ref, ad, False)
    # SwiGLU of the FP32 output with the epilogue's own roundings (bf16 g and u, bf16 h)
    gu = torch.from_numpy(yg).to(dev)
    gate = torch.cat([gu[:, 128 * q:128 * q + 64] for q in range(wl.I // 64)], dim=1).to(torch.bfloat16).float()
    up = torch.cat([gu[:, 128 * q + 64:128 * q + 128] for q in range(wl.I // 64)], dim=1).to(torch.bfloat16).float()
    h_ref = ((gate / (1.0 + torch.exp(-gate))).to(torch.float32) * up).to(torch.bfloat16).float()
    hv = h.float()
    rows = torch.from_numpy(pair_rows).to(dev)
    diff = (hv[rows] - h_ref[rows]).abs()
    ulp = torch.clamp(h_ref[rows].abs(), min=2.0 ** -126) * 2.0 ** -7
    assert bool((diff <= 2 * ulp + 1e-30).all())
    assert float(amax.item()) == float(hv[rows].abs().max().item())
