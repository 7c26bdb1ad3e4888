"""Parity of the FP8 comparison path (through the C ABI) with the oracle on a B200: codes and
power-of-two scales bit-exact; GEMM outputs within |y - y_ref| <= 1e-3 * sum_k |a_k b_k| + 1e-6
(plus one bf16 ulp of y_ref for bf16 output), y_ref the oracle's sum over the identical
quantised operands."""
import numpy as np
import pytest
import torch

from nvfp4_w4a4_moe_02_b200 import mxfp8 as F
from nvfp4_w4a4_moe_02_b200 import nvfp4rac as R
import nvfp4_layout as L
from nvfp4_w4a4_moe_02_b200 import synthetic as syn
from test_gpu_parity import assert_gemm_close, bf16_bits, bf16_ulp, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    F.load()
    return torch.device("cuda:0")


def logical(p: F.Mx8Packed, slab: int = 0, rows: int | None = None):
    """codes [rows, K] and scale codes [rows, K/32] of one slab, from the storage definition: the
    scale of (row r, 32-block b) sits in atom (r // 128, b // 4) at byte (r % 32) * 16 +
    ((r // 32) % 4) * 4 + b % 4."""
    rows = p.rows if rows is None else rows
    K, rp = p.cols, p.rows_padded
    codes = p.codes[slab * rp * K:(slab + 1) * rp * K].cpu().numpy().reshape(rp, K)[:rows]
    sf = p.sf[slab * rp * K // 32:(slab + 1) * rp * K // 32].cpu().numpy()
    r = np.arange(rows)[:, None]
    b = np.arange(K // 32)[None, :]
    idx = (r // 128) * (K // 128) * 512 + (b // 4) * 512 + (r % 32) * 16 + ((r // 32) % 4) * 4 + b % 4
    return codes, sf[idx]


@pytest.mark.parametrize("rows,K", [(64, 256), (300, 768), (4100, 2048)])
def test_fp8_quantize_matches_oracle(dev, orc, rows, K):
    rng = np.random.default_rng(rows)
    x = syn.normal_bf16(rows, 1, rows, K, 1.0, np.exp(3 * rng.standard_normal(K)))
    x[0, :32] = 0           # a zero block
    x[1, 40] = 0x8000       # a negative zero
    x[2, 64:96] = 0x0001    # a block of the smallest bf16 subnormal
    st = R.new_status(dev)
    rp = (rows + 127) // 128 * 128 + 128
    q = F.quantize(to_dev(x, dev), rows_padded=rp, status=st)
    torch.cuda.synchronize()
    R.check_status(st)
    c_ref, S_ref = orc.mx8_quantize(x)
    c, S = logical(q)
    assert np.array_equal(S, S_ref), np.argwhere(S != S_ref)[:5]
    assert np.array_equal(c, c_ref), np.argwhere(c != c_ref)[:5]
    cp, Sp = logical(q, rows=rp)
    assert not cp[rows:].any() and not Sp[rows:].any()


@pytest.mark.parametrize("interleave", [False, True])
def test_fp8_pack_matches_oracle(dev, orc, interleave):
    E, N, K = 2, 256, 512
    w = syn.normal_bf16(7, 2, E * N, K, 0.02).reshape(E, N, K)
    wq = F.pack_weights(to_dev(w, dev), gate_up_interleave=interleave)
    torch.cuda.synchronize()
    for e in range(E):
        we = w[e]
        if interleave:
            p = np.arange(N)
            q, j = p // 128, p % 128
            we = we[np.where(j < 64, q * 64 + j, N // 2 + q * 64 + j - 64)]
        c_ref, S_ref = orc.mx8_quantize(we)
        c, S = logical(wq, e)
        assert np.array_equal(c, c_ref) and np.array_equal(S, S_ref)


def test_fp8_scatter_matches_gather(dev, orc):
    M, K, fan = 50, 256, 3
    x = syn.normal_bf16(2, 1, M, K, 1.0)
    rows_padded = 256
    rng = np.random.default_rng(2)
    dest = rng.permutation(rows_padded)[:M * fan].reshape(M, fan).astype(np.int32)
    dest[4, 1] = -1
    q = F.quantize_scatter(to_dev(x, dev), torch.from_numpy(dest).to(dev), rows_padded)
    torch.cuda.synchronize()
    c_ref, S_ref = orc.mx8_quantize(x)
    c, S = logical(q, rows=rows_padded)
    for m in range(M):
        for j in range(fan):
            d = dest[m, j]
            if d >= 0:
                assert np.array_equal(c[d], c_ref[m]) and np.array_equal(S[d], S_ref[m])
    untouched = np.setdiff1d(np.arange(rows_padded), dest[dest >= 0])
    assert not c[untouched].any() and not S[untouched].any()


@pytest.mark.parametrize("M,N,K,bf16", [(64, 128, 128, False), (300, 384, 768, True), (520, 512, 1024, False)])
def test_fp8_gemm_matches_oracle(dev, orc, M, N, K, bf16):
    x = syn.normal_bf16(M, 1, M, K, 1.0)
    w = syn.normal_bf16(N, 2, N, K, 0.02)
    st = R.new_status(dev)
    a = F.quantize(to_dev(x, dev), status=st)
    wq = F.pack_weights(to_dev(w, dev), status=st)
    y = F.gemm(a, wq, M, out_dtype=torch.bfloat16 if bf16 else torch.float32, status=st)
    torch.cuda.synchronize()
    R.check_status(st)
    ac, aS = orc.mx8_quantize(x)
    wc, wS = orc.mx8_quantize(w)
    y_ref, ad = orc.mx8_gemm(ac, aS, wc, wS)
    assert_gemm_close(y.float().cpu().numpy(), y_ref, ad, bf16)


def test_fp8_moe_block_matches_oracle(dev, orc):
    """gate_up (SwiGLU epilogue) and down on FP8 operands over ragged expert segments."""
    wl = syn.moe_block(T=96, H=512, E=8, topk=2, I=128, T_cal=64)
    g, off, pair_rows = L.gather_map(wl.pair_token, wl.counts)
    offd = torch.from_numpy(off.astype(np.int32)).to(dev)
    rows = torch.from_numpy(np.asarray(wl.counts, np.int32)).to(dev)
    st = R.new_status(dev)
    wgu = F.pack_weights(to_dev(wl.wgu, dev), gate_up_interleave=True, status=st)
    wdn = F.pack_weights(to_dev(wl.wdn, dev), status=st)
    sm = torch.from_numpy(L.scatter_map(wl.pair_token, pair_rows, wl.x.shape[0], wl.topk_ids.shape[1])).to(dev)
    a = F.quantize_scatter(to_dev(wl.x, dev), sm, g.size, status=st)
    # padding-only output boxes are skipped: h starts zeroed so its padding rows stay finite zeros
    h = torch.zeros(g.size, wl.I, dtype=torch.bfloat16, device=dev)
    F.grouped_moe(a, offd, wgu, swiglu=True, y=h, status=st, expert_rows=rows)
    hq = F.quantize(h, status=st)
    y = F.grouped_moe(hq, offd, wdn, status=st, expert_rows=rows)
    torch.cuda.synchronize()
    R.check_status(st)
    I = wl.I
    h_gpu = bf16_bits(h)
    hq_c, hq_S = logical(hq, rows=hq.rows_padded)
    for e in range(wl.E):
        pidx = np.nonzero(wl.pair_expert == e)[0]
        if pidx.size == 0:
            continue
        prow = pair_rows[pidx]
        ac, aS = orc.mx8_quantize(wl.x[wl.pair_token[pidx]])
        wc, wS = orc.mx8_quantize(wl.gate_up_expert(e))
        gu, ad = orc.mx8_gemm(ac, aS, wc, wS)
        tol = 1e-3 * ad + 1e-6 + bf16_ulp(gu)
        gg, uu = gu[:, :I], gu[:, I:]
        tg, tu = tol[:, :I], tol[:, I:]
        sig = 1.0 / (1.0 + np.exp(-gg))
        silu = gg * sig
        dsilu = np.abs(sig * (1 + gg * (1 - sig))) + 0.1
        h_ref = silu * uu
        tol_h = 2.0 * (dsilu * tg * (np.abs(uu) + tu) + np.abs(silu) * tu) + 2 * bf16_ulp(h_ref) + 1e-30
        h_g = syn.bf16_to_f32(h_gpu[prow]).astype(np.float64)
        assert np.all(np.abs(h_g - h_ref) <= tol_h), e
        # down: the GPU's h rows quantised by the oracle match the GPU codes bit for bit
        hc, hS = orc.mx8_quantize(h_gpu[prow])
        assert np.array_equal(hq_c[prow], hc) and np.array_equal(hq_S[prow], hS)
        dc, dS = orc.mx8_quantize(wl.down_expert(e))
        y_ref, ad2 = orc.mx8_gemm(hc, hS, dc, dS)
        assert_gemm_close(y[torch.from_numpy(prow).to(dev)].float().cpu().numpy(), y_ref, ad2, True)


def test_fp8_non_finite_block_is_reported(dev):
    x = syn.normal_bf16(1, 1, 16, 128, 1.0)
    x[3, 35] = 0x7F80  # +inf
    st = R.new_status(dev)
    q = F.quantize(to_dev(x, dev), status=st)
    torch.cuda.synchronize()
    assert st.item() == 4  # NVFP4_ERR_RANGE
    c, S = logical(q)
    assert not c[3, 32:64].any() and S[3, 1] == 0
