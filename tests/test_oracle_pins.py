"""Pins of the CPU oracle to facts that do not come from the oracle itself.

Each test checks an oracle routine against something independent: the format
facts stated on the pages (8 E2M1 magnitudes per sign), closed forms of the
E4M3 / E2M1 encodings, brute-force searches written here in plain Python,
hand-worked fixtures, exact rational arithmetic, and invariants of the method
(on-grid round trip, r = 0 reduces to plain W4A4, r = 1 selects every channel,
compensation lowers the error on the calibration data).
"""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest

from nvfp4_w4a4_moe_02_b200 import synthetic as syn

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")

E2M1_GRID = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


# ------------------------------------------------------------------ independent reference encoders
def brute_e2m1(v: float) -> int:
    """Nearest grid magnitude by exhaustive exact comparison; ties to even index; saturate."""
    m = abs(Fraction(v))
    best = None
    for i, g in enumerate(E2M1_GRID):
        d = abs(m - Fraction(g))
        key = (d, i % 2)  # smaller distance first, then even index
        if best is None or key < best[0]:
            best = (key, i)
    idx = best[1]
    if m > 6:
        idx = 7
    sign = 8 if math.copysign(1.0, v) < 0 else 0
    return idx | sign


def e4m3_value_closed_form(code: int) -> float:
    e, m = (code >> 3) & 15, code & 7
    if e == 0:
        return m * 2.0 ** -9
    return (1 + m / 8) * 2.0 ** (e - 7)


E4M3_POS = [e4m3_value_closed_form(c) for c in range(0x7F)]  # 0x00 .. 0x7E


def brute_e4m3(raw: float) -> int:
    r = Fraction(raw)
    if r >= 448:
        return 0x7E
    best = None
    for c, val in enumerate(E4M3_POS):
        d = abs(r - Fraction(val))
        key = (d, c % 2)
        if best is None or key < best[0]:
            best = (key, c)
    return best[1]


def f32(x):
    return float(np.float32(x))


def neighbours(x: float, k: int = 3):
    """x and its k nearest float32 neighbours on both sides."""
    out = [np.float32(x)]
    up = dn = np.float32(x)
    for _ in range(k):
        up = np.nextafter(up, np.float32(np.inf), dtype=np.float32)
        dn = np.nextafter(dn, np.float32(-np.inf), dtype=np.float32)
        out += [up, dn]
    return [float(v) for v in out]


# ------------------------------------------------------------------ E2M1
def test_e2m1_has_eight_magnitudes_per_sign(orc):
    """The failure-mode section: E2M1 gives 8 representable magnitude levels per sign."""
    pos = [orc.e2m1_decode(c) for c in range(8)]
    neg = [orc.e2m1_decode(c) for c in range(8, 16)]
    assert pos == E2M1_GRID
    assert [-v for v in neg] == E2M1_GRID
    assert all(math.copysign(1.0, v) < 0 for v in neg)  # -0 included
    assert len(set(pos)) == 8 and len(set(abs(v) for v in neg)) == 8


def test_e2m1_encode_matches_brute_force(orc):
    pts = []
    mids = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0]
    for g in E2M1_GRID + mids + [6.5, 7.0, 1e3, 1e30]:
        for s in (1.0, -1.0):
            pts += [s * v for v in neighbours(g, 4)]
    rng = np.random.default_rng(0)
    pts += list(rng.uniform(-8, 8, 20000).astype(np.float32).astype(float))
    pts += list((rng.standard_normal(2000) * 1e-30).astype(np.float32).astype(float))
    pts += [0.0, -0.0, float(np.float32(1.4e-45)), -float(np.float32(1.4e-45))]
    arr = np.array(pts, dtype=np.float32)
    got = orc.e2m1_encode_array(arr)
    exp = np.array([brute_e2m1(float(v)) for v in arr], dtype=np.uint8)
    bad = np.nonzero(got != exp)[0]
    assert bad.size == 0, [(float(arr[i]), int(got[i]), int(exp[i])) for i in bad[:10]]


def test_e2m1_ties_go_to_even(orc):
    assert orc.e2m1_encode(0.25) == 0 and orc.e2m1_encode(0.75) == 2
    assert orc.e2m1_encode(1.25) == 2 and orc.e2m1_encode(1.75) == 4
    assert orc.e2m1_encode(2.5) == 4 and orc.e2m1_encode(3.5) == 6 and orc.e2m1_encode(5.0) == 6
    assert orc.e2m1_encode(-0.2) == 8  # sign kept on a zero result
    assert orc.e2m1_encode(100.0) == 7 and orc.e2m1_encode(-100.0) == 15


# ------------------------------------------------------------------ E4M3
def test_e4m3_decode_closed_form(orc):
    for c in range(256):
        v = orc.e4m3_decode(c)
        if c & 0x7F == 0x7F:
            assert math.isnan(v)
            continue
        ref = e4m3_value_closed_form(c & 0x7F) * (-1 if c & 0x80 else 1)
        assert v == ref, (c, v, ref)
    assert orc.e4m3_decode(0x7E) == 448.0
    assert orc.e4m3_decode(0x01) == 2.0 ** -9
    assert orc.e4m3_decode(0x08) == 2.0 ** -6
    assert orc.e4m3_decode(0x38) == 1.0
    vals = [orc.e4m3_decode(c) for c in range(0x7F)]
    assert all(a < b for a, b in zip(vals, vals[1:]))
    # 256 code points: 2 zeros, 2 NaN, 252 finite non-zero values (the 256-level comparison format)
    assert len({orc.e4m3_decode(c) for c in range(256) if c & 0x7F not in (0, 0x7F)}) == 252


def test_e4m3_encode_matches_brute_force(orc):
    pts = []
    for a, b in zip(E4M3_POS, E4M3_POS[1:]):
        pts += neighbours((a + b) / 2, 2) + neighbours(b, 1)
    pts += neighbours(2.0 ** -10, 3) + neighbours(448.0, 3) + neighbours(464.0, 3) + [1e6, 0.0]
    rng = np.random.default_rng(1)
    pts += list(rng.uniform(0, 460, 5000).astype(np.float32).astype(float))
    pts += list(np.exp(rng.uniform(-12, 6, 5000)).astype(np.float32).astype(float))
    arr = np.array([p for p in pts if p >= 0], dtype=np.float32)
    got = orc.e4m3_encode_array(arr)
    exp = np.array([brute_e4m3(float(v)) for v in arr], dtype=np.uint8)
    bad = np.nonzero(got != exp)[0]
    assert bad.size == 0, [(float(arr[i]), int(got[i]), int(exp[i])) for i in bad[:10]]


def test_e4m3_saturation_and_underflow(orc):
    assert orc.e4m3_encode(448.0) == 0x7E and orc.e4m3_encode(1e9) == 0x7E
    assert orc.e4m3_encode(2.0 ** -10) == 0  # tie between 0 and 2^-9 goes to even code 0
    assert orc.e4m3_encode(f32(np.nextafter(np.float32(2.0 ** -10), np.float32(1)))) == 1


# ------------------------------------------------------------------ bf16 storage
def test_bf16_rounding_matches_torch(orc):
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(2)
    v = np.concatenate([rng.standard_normal(3000) * 10.0 ** rng.integers(-30, 30, 3000),
                        np.array([1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -(1.0 + 2 ** -8), 3.3895e38])]).astype(np.float32)
    ref = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().astype(np.uint16)
    got = np.array([orc.f64_to_bf16(float(x)) for x in v], dtype=np.uint16)
    assert np.array_equal(got, ref)


# ------------------------------------------------------------------ scales and blocks
def test_global_scale_power_of_two(orc):
    for j in range(-20, 20):
        assert float(orc.global_scale(2688.0 * 2.0 ** j)) == 2.0 ** j
    assert float(orc.global_scale(0.0)) == 0.0


def test_hand_worked_fixture(orc):
    g = json.load(open(os.path.join(GOLDEN, "nvfp4_hand_worked_blocks.json")))
    x = np.array(g["x"], dtype=np.float32)
    xb = (x.view(np.uint32) >> 16).astype(np.uint16).reshape(1, -1)
    assert np.array_equal(syn.bf16_to_f32(xb).reshape(-1), x)  # inputs are bf16-exact
    amax = orc.amax_bf16(xb)
    s_g = orc.global_scale(amax)
    assert float(s_g) == g["s_g"]
    sel = np.array(g["sel"], dtype=np.int32)
    codes, S, rcodes, rS, resid = orc.act_quant_rac(xb, s_g, sel)
    assert codes.reshape(-1).tolist() == g["codes"]
    assert S.reshape(-1).tolist() == g["S"]
    assert rS.reshape(-1).tolist() == g["rS"]
    assert rcodes.reshape(-1).tolist() == g["rcodes"]
    assert resid.reshape(-1).tolist() == g["resid"]
    _, _, dq = orc.quantize_f32(x.reshape(1, -1), s_g)
    assert dq.reshape(-1).tolist() == g["dq"]


def test_quantize_matches_float32_numpy_steps(orc):
    """Each block decision re-derived with numpy float32 arithmetic and the brute-force encoders."""
    rng = np.random.default_rng(3)
    t = (rng.standard_normal((6, 64)) * np.exp(rng.standard_normal((6, 1)) * 2)).astype(np.float32)
    t[0, :16] = 0.0
    amax = np.float32(np.abs(t).max())
    s_g = np.float32(amax / np.float32(2688.0))
    codes, S, dq = orc.quantize_f32(t, s_g)
    t6 = np.float32(np.float32(6.0) * s_g)
    for r in range(t.shape[0]):
        for b in range(4):
            blk = t[r, 16 * b:16 * b + 16]
            bmax = np.float32(np.abs(blk).max())
            raw = np.float32(bmax / t6)
            s_exp = brute_e4m3(float(raw))
            assert S[r, b] == s_exp
            if s_exp == 0:
                assert not codes[r, 16 * b:16 * b + 16].any()
                continue
            d = np.float32(np.float32(E4M3_POS[s_exp]) * s_g)
            inv = np.float32(np.float32(1.0) / d)
            for i in range(16):
                v = np.float32(blk[i] * inv)
                q = brute_e2m1(float(v))
                assert codes[r, 16 * b + i] == q
                val = E2M1_GRID[q & 7] * (-1 if q & 8 else 1)
                assert dq[r, 16 * b + i] == np.float32(np.float32(val) * d)


def test_on_grid_values_round_trip_exactly(orc):
    """Values built from the grid (s_g = 2^j, any E4M3 block scale, a +-6 in every block) are
    reproduced exactly and leave a zero residual."""
    rng = np.random.default_rng(4)
    for j in (-6, 0, 3):
        rows, K = 8, 128
        s_g = 2.0 ** j
        S = rng.integers(1, 0x7F, size=(rows, K // 16))
        S[0, 0] = 0x7E  # the amax block: 6 * 448 * s_g = 2688 * s_g
        e_idx = rng.integers(0, 8, size=(rows, K))
        sign = rng.integers(0, 2, size=(rows, K))
        e_idx[:, ::16] = 7
        vals = np.array(E2M1_GRID)[e_idx] * np.where(sign, -1, 1)
        svals = np.array(E4M3_POS)[S]
        x = (vals * np.repeat(svals, 16, axis=1) * s_g).astype(np.float32)
        assert np.array_equal(x.astype(np.float64), vals * np.repeat(svals, 16, axis=1) * s_g)
        xb = (x.view(np.uint32) >> 16).astype(np.uint16)
        assert np.array_equal(syn.bf16_to_f32(xb), x)
        assert float(orc.global_scale(orc.amax_bf16(xb))) == s_g
        sel = np.arange(0, K, 2, dtype=np.int32)
        codes, Sq, rcodes, rS, resid = orc.act_quant_rac(xb, s_g, sel)
        assert np.array_equal(Sq, S)
        assert np.array_equal(codes & 7, e_idx)
        _, _, dq = orc.quantize_f32(x, s_g)
        assert np.array_equal(dq, x)
        assert not resid.any() and not rS.any()


def test_residual_is_input_minus_dequant(orc):
    wl = syn.dense_tiny()
    x = wl.x
    s_g = orc.global_scale(orc.amax_bf16(x))
    sel = np.arange(0, wl.K, 3, dtype=np.int32)[:64]
    codes, S, rcodes, rS, resid = orc.act_quant_rac(x, s_g, sel)
    xf = syn.bf16_to_f32(x)
    e = np.array(E2M1_GRID, np.float32)[codes & 7] * np.where(codes & 8, np.float32(-1), np.float32(1))
    d = (np.array(E4M3_POS, np.float32)[S] * np.float32(s_g)).astype(np.float32)
    dq = (e * np.repeat(d, 16, axis=1)).astype(np.float32)
    assert np.array_equal(resid, (xf[:, sel] - dq[:, sel]).astype(np.float32))
    # the residual of a kept channel is what the residual codes approximate
    rq = orc.dequant(rcodes, rS, s_g)
    assert np.abs(rq - resid).max() <= np.abs(resid).max() / 6 + 1e-12


# ------------------------------------------------------------------ GEMM
def test_gemm_exact_vs_fraction_brute_force(orc):
    rng = np.random.default_rng(5)
    M, N, K, Kp = 3, 4, 32, 16
    a = rng.integers(0, 16, (M, K), dtype=np.uint8)
    w = rng.integers(0, 16, (N, K), dtype=np.uint8)
    r = rng.integers(0, 16, (M, Kp), dtype=np.uint8)
    ws = rng.integers(0, 16, (N, Kp), dtype=np.uint8)
    aS = rng.integers(0, 0x7F, (M, K // 16), dtype=np.uint8)
    wS = rng.integers(0, 0x7F, (N, K // 16), dtype=np.uint8)
    rS = rng.integers(0, 0x7F, (M, Kp // 16), dtype=np.uint8)
    wsS = rng.integers(0, 0x7F, (N, Kp // 16), dtype=np.uint8)
    s_a, s_w = 0.37109375, 1.5 * 2 ** -7
    y, ad = orc.gemm_rac(a, aS, r, rS, w, wS, ws, wsS, s_a, s_w)

    def val(q, s):
        e = Fraction(E2M1_GRID[q & 7]) * (-1 if q & 8 else 1)
        return e * Fraction(E4M3_POS[s])

    for i in range(M):
        for j in range(N):
            acc = sum(val(a[i, k], aS[i, k // 16]) * val(w[j, k], wS[j, k // 16]) for k in range(K))
            acc += sum(val(r[i, k], rS[i, k // 16]) * val(ws[j, k], wsS[j, k // 16]) for k in range(Kp))
            ref = acc * Fraction(s_a) * Fraction(s_w)
            assert y[i, j] == float(ref)


def test_gemm_matches_dequantized_float_matmul(orc):
    wl = syn.dense_tiny()
    sel, _ = orc.calibrate(wl.x_cal, wl.Kp)
    f = orc.dense_rac_forward(wl.x, wl.w, sel)
    A = orc.dequant(f["a"], f["aS"], f["s_x"])
    R = orc.dequant(f["r"], f["rS"], f["s_x"])
    W = orc.dequant(f["wc"], f["wS"], f["s_w"])
    WS = orc.dequant(f["wsc"], f["wsS"], f["s_w"])
    ref = A @ W.T + R @ WS.T
    assert np.abs(f["y"] - ref).max() <= 1e-12 * f["absdot"].max()


def test_r0_reduces_to_plain_w4a4(orc):
    """The native W4A4 GEMM path stays intact: with no selected channel the result is plain W4A4."""
    wl = syn.dense_tiny()
    empty = np.zeros(0, np.int32)
    f0 = orc.dense_rac_forward(wl.x, wl.w, empty)
    A = orc.dequant(f0["a"], f0["aS"], f0["s_x"])
    W = orc.dequant(f0["wc"], f0["wS"], f0["s_w"])
    assert np.abs(f0["y"] - A @ W.T).max() <= 1e-12 * f0["absdot"].max()
    # and the main-loop codes do not depend on the selection
    sel, _ = orc.calibrate(wl.x_cal, wl.Kp)
    f1 = orc.dense_rac_forward(wl.x, wl.w, sel)
    for k in ("a", "aS", "wc", "wS"):
        assert np.array_equal(f0[k], f1[k])


# ------------------------------------------------------------------ calibration / selection
def test_r1_selects_every_channel(orc):
    wl = syn.dense_tiny()
    sel, _ = orc.calibrate(wl.x_cal, wl.K)
    assert np.array_equal(sel, np.arange(wl.K))


def test_selection_matches_sequential_python(orc):
    rng = np.random.default_rng(6)
    T, K, Kp = 12, 64, 32
    x = syn.normal_bf16(7, 3, T, K, 1.0, np.exp(rng.standard_normal(K)))
    x[:, 5] = x[:, 6]  # identical channels -> equal errors, tie broken by index
    sel, err = orc.calibrate(x, Kp)
    s_g = orc.global_scale(orc.amax_bf16(x))
    _, _, dq = orc.quantize_f32(syn.bf16_to_f32(x), s_g)
    r = (syn.bf16_to_f32(x) - dq).astype(np.float32)
    e = []
    for k in range(K):
        acc = 0.0
        for t in range(T):
            acc += float(r[t, k]) * float(r[t, k])
        e.append(acc)
    assert np.array_equal(np.array(e), err)
    order = sorted(range(K), key=lambda k: (-e[k], k))
    assert sel.tolist() == sorted(order[:Kp])


def test_outlier_channels_are_selected(orc):
    wl = syn.dense_tiny()
    sel, _ = orc.calibrate(wl.x_cal, wl.Kp)
    for k in syn.outlier_channels(0, wl.K):
        assert k in sel


def test_compensation_never_increases_error_on_calibration_data(orc):
    """r > 0 lowers mean |Y - Y_bf16| relative to r = 0 on the calibration batch."""
    wl = syn.dense_tiny()
    xf = syn.bf16_to_f32(wl.x_cal).astype(np.float64)
    wf = syn.bf16_to_f32(wl.w).astype(np.float64)
    y_ref = xf @ wf.T
    errs = []
    for r in (0.0, 0.25, 0.5, 1.0):
        Kp = syn.kp_from_ratio(wl.K, r)
        sel, _ = orc.calibrate(wl.x_cal, Kp)
        f = orc.dense_rac_forward(wl.x_cal, wl.w, sel)
        errs.append(np.abs(f["y"] - y_ref).mean())
    assert all(e <= errs[0] for e in errs[1:]), errs
    assert all(b <= a for a, b in zip(errs, errs[1:])), errs  # monotone in r on this batch


@pytest.mark.slow
def test_compensation_never_increases_error_on_moe_prefill_calibration_data(orc):
    """The MoE prefill block (4096 tokens, hidden 2048, 128 experts, top-8, intermediate 768) on its
    own calibration data: mean |Y - Y_bf16| over r in {0, 0.25, 0.5, 1} never rises (r = 0 is
    plain W4A4).  Y is the whole block through the oracle: quantise X (+ residual), gate_up,
    SwiGLU, quantise h (+ residual), down; Y_bf16 the binary64 product of the bf16 inputs.  The
    rows are every calibration pair of six experts; the channel lists are calibrated on the whole
    calibration batch (gate_up on X_cal, down on the pooled h_cal) as the rollout does."""
    wl = syn.moe_prefill()
    h_cal = syn.moe_down_calibration_batch(wl)
    off = syn.moe_down_calibration_offsets(wl)
    T = wl.x_cal.shape[0]
    topk = syn.route_topk(wl.seed, T, wl.E, wl.topk_ids.shape[1], stream=syn.STREAM_ROUTER_CAL)
    pt, pe, _ = syn.sort_pairs(topk, wl.E)
    experts = [0, 17, 42, 64, 101, 127]
    f64 = lambda a: syn.bf16_to_f32(a).astype(np.float64)
    xf = f64(wl.x_cal)
    s_x = orc.global_scale(orc.amax_bf16(wl.x_cal))
    rows = {e: pt[off[e]:off[e + 1]] for e in experts}
    y_ref = {}
    for e in experts:
        gu = xf[rows[e]] @ f64(wl.gate_up_expert(e)).T
        h = gu[:, :wl.I] / (1.0 + np.exp(-gu[:, :wl.I])) * gu[:, wl.I:]
        y_ref[e] = h @ f64(wl.down_expert(e)).T
    errs = []
    for r in (0.0, 0.25, 0.5, 1.0):
        Kp_gu, Kp_dn = syn.kp_from_ratio(wl.H, r), syn.kp_from_ratio(wl.I, r)
        sel_gu = orc.calibrate(wl.x_cal, Kp_gu)[0] if Kp_gu else np.zeros(0, np.int32)
        sel_dn = orc.calibrate(h_cal, Kp_dn)[0] if Kp_dn else np.zeros(0, np.int32)
        hs = {}
        for e in experts:
            ac, aS, rc, rS, _ = orc.act_quant_rac(wl.x_cal[rows[e]], s_x, sel_gu)
            wgu = wl.gate_up_expert(e)
            s_w = orc.global_scale(orc.amax_bf16(wgu))
            gu, _ = orc.gemm_rac(ac, aS, rc, rS, *orc.weight_pack(wgu, s_w, sel_gu), s_x, s_w)
            hs[e] = orc.swiglu(orc.f64_to_bf16_array(gu))[0]
        s_h = orc.global_scale(orc.amax_bf16(np.concatenate([hs[e] for e in experts])))
        tot, n = 0.0, 0
        for e in experts:
            hc, hS, hrc, hrS, _ = orc.act_quant_rac(hs[e], s_h, sel_dn)
            wdn = wl.down_expert(e)
            s_w = orc.global_scale(orc.amax_bf16(wdn))
            y, _ = orc.gemm_rac(hc, hS, hrc, hrS, *orc.weight_pack(wdn, s_w, sel_dn), s_h, s_w)
            tot += float(np.abs(y - y_ref[e]).sum())
            n += y.size
        errs.append(tot / n)
    print('mean |Y - Y_bf16| at r = 0, 0.25, 0.5, 1:', errs)
    assert all(e <= errs[0] for e in errs[1:]), errs
    assert all(b <= a for a, b in zip(errs, errs[1:])), errs


def test_compensation_shrinks_activation_error(orc):
    """Against X_bf16 @ DQ(Q(W))^T (weight error removed), the residual pass over all channels
    removes most of the activation quantisation error."""
    wl = syn.dense_tiny()
    xf = syn.bf16_to_f32(wl.x_cal).astype(np.float64)
    errs = []
    for r in (0.0, 1.0):
        Kp = syn.kp_from_ratio(wl.K, r)
        sel, _ = orc.calibrate(wl.x_cal, Kp)
        f = orc.dense_rac_forward(wl.x_cal, wl.w, sel)
        Wq = orc.dequant(f["wc"], f["wS"], f["s_w"])
        errs.append(np.abs(f["y"] - xf @ Wq.T).mean())
    assert errs[1] < 0.25 * errs[0], errs


# ------------------------------------------------------------------ weights / trainer fake-quant
def test_shared_weight_path_is_bit_identical(orc):
    """The packed weights dequantise to exactly the trainer's fake-quantised weights."""
    w = syn.normal_bf16(0, 2, 64, 256, 0.02)
    s_w = orc.global_scale(orc.amax_bf16(w))
    sel = np.arange(64, dtype=np.int32)
    wc, wS, _, _ = orc.weight_pack(w, s_w, sel)
    qdq, s2 = orc.weight_qdq(w)
    assert float(s2) == float(s_w)
    e = np.array(E2M1_GRID, np.float32)[wc & 7] * np.where(wc & 8, np.float32(-1), np.float32(1))
    d = (np.array(E4M3_POS, np.float32)[wS] * np.float32(s_w)).astype(np.float32)
    dq32 = (e * np.repeat(d, 16, axis=1)).astype(np.float32)
    torch = pytest.importorskip("torch")
    ref = torch.from_numpy(dq32).to(torch.bfloat16).view(torch.int16).numpy().astype(np.uint16)
    assert np.array_equal(qdq, ref)


def test_weight_sel_is_raw_columns(orc):
    w = syn.normal_bf16(0, 2, 32, 128, 0.02)
    s_w = orc.global_scale(orc.amax_bf16(w))
    sel = np.array(sorted(np.random.default_rng(7).choice(128, 64, replace=False)), np.int32)
    _, _, sc, sS = orc.weight_pack(w, s_w, sel)
    c2, S2, _ = orc.quantize_f32(syn.bf16_to_f32(w)[:, sel], s_w)
    assert np.array_equal(sc, c2) and np.array_equal(sS, S2)


# ------------------------------------------------------------------ SwiGLU
def test_swiglu_closed_form(orc):
    g = np.array([0.0, 1.0, -1.0, 4.0, -20.0, 0.5], np.float32)
    u = np.array([3.0, 2.0, 2.0, -0.5, 1.0, 1.0], np.float32)
    gu = np.concatenate([g, u]).reshape(1, -1)
    gub = (gu.view(np.uint32) >> 16).astype(np.uint16)
    h, hx = orc.swiglu(gub)
    for i in range(6):
        ref = float(g[i]) / (1 + math.exp(-float(g[i]))) * float(u[i])
        assert abs(hx[0, i] - ref) <= 1e-15 * max(1.0, abs(ref))
        assert h[0, i] == orc.f64_to_bf16(ref)
    assert hx[0, 0] == 0.0


# ------------------------------------------------------------------------------------------ MoE block
def test_route_topk_matches_stable_sort(orc):
    """Top-k of the logits, ties to the lower expert: a stable sort of the negated logits."""
    rng = np.random.default_rng(3)
    logits = rng.integers(-3, 4, (128, 32)).astype(np.float32)  # many exact ties
    for k in (1, 2, 8):
        ids, _ = orc.route_topk(logits, k)
        ref = np.argsort(-logits, axis=1, kind="stable")[:, :k]
        assert np.array_equal(ids, ref)


def test_route_weights_closed_forms(orc):
    rng = np.random.default_rng(4)
    logits = rng.standard_normal((64, 40)).astype(np.float32)
    ids, w = orc.route_topk(logits, 1)
    assert np.all(w == 1.0)
    ids, w = orc.route_topk(logits, 8)
    assert np.allclose(w.sum(axis=1), 1.0, atol=1e-6)
    assert np.all(np.diff(w, axis=1) <= 0)  # best first
    chosen = np.take_along_axis(logits.astype(np.float64), ids.astype(np.int64), axis=1)
    ratio = w[:, 1:].astype(np.float64) / w[:, :1]
    assert np.allclose(ratio, np.exp(chosen[:, 1:] - chosen[:, :1]), rtol=1e-6)
    # two equal best logits share the weight exactly
    two = np.array([[0.0, 1.5, 1.5, -2.0]], np.float32)
    ids, w = orc.route_topk(two, 2)
    assert ids.tolist() == [[1, 2]] and w.tolist() == [[0.5, 0.5]]


def test_dispatch_plan_brute_force(orc):
    rng = np.random.default_rng(5)
    T, E, k = 50, 9, 3
    ids = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
    ids[:, 0] = np.where(np.arange(T) % 4 == 0, 2, ids[:, 0])  # a busy expert
    ids[ids == 7] = 8                                           # an empty one (may duplicate: fix below)
    for t in range(T):
        if len(set(ids[t].tolist())) < k:
            ids[t] = np.array([e for e in [0, 1, 3, 4, 5, 6] if e not in ids[t]][:k], np.int32)
    for pad in (1, 16, 128):
        off, row = orc.dispatch_plan(ids, E, pad)
        pairs = sorted((int(ids[t, j]), t, j) for t in range(T) for j in range(k))
        counts = [sum(1 for p in pairs if p[0] == e) for e in range(E)]
        start = [0]
        for c in counts:
            start.append(start[-1] + -(-c // pad) * pad)
        assert off.tolist() == start
        seen = {}
        for e, t, j in pairs:
            r = start[e] + seen.get(e, 0)
            seen[e] = seen.get(e, 0) + 1
            assert row[t, j] == r
        assert counts[7] == 0 and off[8] == off[7]


def test_combine_reduces_to_gather_and_is_linear(orc):
    rng = np.random.default_rng(6)
    R, H, T, k = 40, 48, 10, 3
    y = syn._f32_to_bf16_bits(rng.standard_normal((R, H)).astype(np.float32))
    row = np.stack([rng.permutation(R)[:k] for _ in range(T)]).astype(np.int64)
    onehot = np.zeros((T, k), np.float32)
    onehot[:, 1] = 1.0
    out = orc.combine(y, row, onehot)
    assert np.array_equal(out, syn.bf16_to_f32(y[row[:, 1]]).astype(np.float64))
    # dyadic weights: w1 + w2 is exact in binary32, so linearity holds to binary64 rounding
    w1 = (rng.integers(0, 256, (T, k)) / 256.0).astype(np.float32)
    w2 = (rng.integers(0, 256, (T, k)) / 256.0).astype(np.float32)
    a, b, c = orc.combine(y, row, w1), orc.combine(y, row, w2), orc.combine(y, row, w1 + w2)
    ref = np.einsum("tj,tjh->th", (w1 + w2).astype(np.float64), syn.bf16_to_f32(y[row]).astype(np.float64))
    assert np.allclose(c, a + b, rtol=1e-12, atol=1e-12) and np.allclose(c, ref, rtol=1e-12, atol=1e-12)


# ------------------------------------------------------------------------------------------ RAC variant
def test_masked_residual_empty_selection_is_plain_w4a4(orc):
    """Masked full-K variant: no selected channel -> zero residual codes and the plain W4A4 GEMM."""
    wl = syn.dense_tiny()
    s_x = orc.global_scale(orc.amax_bf16(wl.x))
    c, S, mc, mS = orc.act_quant_masked(wl.x, s_x, np.zeros(0, np.int32))
    assert not mc.any() and not mS.any()
    y, _ = orc.masked_rac_forward(wl.x, wl.w, np.zeros(0, np.int32))
    y0 = orc.dense_rac_forward(wl.x, wl.w, np.zeros(0, np.int32))["y"]
    assert np.array_equal(y, y0)


def test_masked_residual_matches_compact_on_aligned_and_full_selections(orc):
    """When the selection is whole aligned 16-blocks, every masked residual block is the compact
    residual block of the same channels (same 16 values, same order); when it is every channel
    the two layouts coincide.  Off the selection the masked residual is exactly zero."""
    wl = syn.dense_tiny()
    s_x = orc.global_scale(orc.amax_bf16(wl.x))
    K = wl.x.shape[1]
    sel = np.concatenate([np.arange(32, 64), np.arange(160, 176)]).astype(np.int32)
    c, S, mc, mS = orc.act_quant_masked(wl.x, s_x, sel)
    c2, S2, rc, rS, _ = orc.act_quant_rac(wl.x, s_x, sel)
    assert np.array_equal(c, c2) and np.array_equal(S, S2)  # the main pass is unchanged
    assert np.array_equal(mc[:, 32:64], rc[:, 0:32]) and np.array_equal(mS[:, 2:4], rS[:, 0:2])
    assert np.array_equal(mc[:, 160:176], rc[:, 32:48]) and np.array_equal(mS[:, 10], rS[:, 2])
    off = np.ones(K, bool)
    off[sel] = False
    assert not mc[:, off].any()
    full = np.arange(K, dtype=np.int32)
    _, _, mcf, mSf = orc.act_quant_masked(wl.x, s_x, full)
    _, _, rcf, rSf, _ = orc.act_quant_rac(wl.x, s_x, full)
    assert np.array_equal(mcf, rcf) and np.array_equal(mSf, rSf)


def test_masked_gemm_matches_dequantized_float_matmul(orc):
    """Y = DQ(Q(X)) DQ(Q(W))^T + DQ(Q(M)) DQ(Q(W))^T with the masked residual (float64 reference)."""
    wl = syn.dense_tiny()
    sel, _ = orc.calibrate(wl.x_cal, wl.Kp)
    s_x = orc.global_scale(orc.amax_bf16(wl.x))
    s_w = orc.global_scale(orc.amax_bf16(wl.w))
    c, S, mc, mS = orc.act_quant_masked(wl.x, s_x, sel)
    wc, wS, _, _ = orc.weight_pack(wl.w, s_w, np.zeros(0, np.int32))
    ref = (orc.dequant(c, S, s_x) + orc.dequant(mc, mS, s_x)) @ orc.dequant(wc, wS, s_w).T
    y, ad = orc.masked_rac_forward(wl.x, wl.w, sel)
    assert np.abs(y - ref).max() <= 1e-12 * ad.max()


def test_masked_residual_reduces_error_on_calibration_data(orc):
    """Like the compact residual, the masked residual lowers the mean error against the exact
    bf16 product on the calibration batch."""
    wl = syn.dense_tiny()
    sel, _ = orc.calibrate(wl.x_cal, wl.Kp)
    xf = syn.bf16_to_f32(wl.x_cal).astype(np.float64)
    wf = syn.bf16_to_f32(wl.w).astype(np.float64)
    exact = xf @ wf.T
    y_plain = orc.dense_rac_forward(wl.x_cal, wl.w, np.zeros(0, np.int32))["y"]
    y_mask, _ = orc.masked_rac_forward(wl.x_cal, wl.w, sel)
    assert np.mean(np.abs(y_mask - exact)) < np.mean(np.abs(y_plain - exact))


# ---- per-expert channel lists (a RAC variant the pages leave open: one list per expert) ----

def _grouped_batch(seed=11, T=30, K=128, offsets=(0, 7, 7, 19, 30)):
    rng = np.random.default_rng(seed)
    x = syn.normal_bf16(seed, 3, T, K, 1.0, np.exp(rng.standard_normal(K)))
    return x, np.array(offsets, np.int64)


def test_grouped_selection_single_group_equals_shared(orc):
    x, _ = _grouped_batch()
    sel, err = orc.calibrate(x, 64)
    sg, eg = orc.calibrate_grouped(x, np.array([0, x.shape[0]]), 64)
    assert np.array_equal(sg[0], sel) and np.array_equal(eg[0], err)


def test_grouped_selection_matches_sequential_python(orc):
    """e_k of group g sums only rows [off[g], off[g+1]) of the residual of the pooled batch
    (quantised once with the batch's own s_g), t ascending; ties go to the lower channel."""
    x, off = _grouped_batch()
    x[:, 9] = x[:, 10]  # equal errors in every group: the tie goes to channel 9
    Kp = 32
    sel, err = orc.calibrate_grouped(x, off, Kp)
    s_g = orc.global_scale(orc.amax_bf16(x))
    _, _, dq = orc.quantize_f32(syn.bf16_to_f32(x), s_g)
    r = (syn.bf16_to_f32(x) - dq).astype(np.float32)
    K = x.shape[1]
    for g in range(off.size - 1):
        e = []
        for k in range(K):
            acc = 0.0
            for t in range(int(off[g]), int(off[g + 1])):
                acc += float(r[t, k]) * float(r[t, k])
            e.append(acc)
        assert np.array_equal(np.array(e), err[g]), g
        order = sorted(range(K), key=lambda k: (-e[k], k))
        assert sel[g].tolist() == sorted(order[:Kp]), g


def test_grouped_selection_empty_group_takes_lowest_channels(orc):
    x, off = _grouped_batch()  # group 1 is empty
    sel, err = orc.calibrate_grouped(x, off, 32)
    assert np.all(err[1] == 0.0) and sel[1].tolist() == list(range(32))


def test_grouped_selection_follows_each_groups_outliers(orc):
    """Channels scaled x20 in one group's rows only: a x20 channel sets its 16-block's scale, so
    the largest residuals sit in that block (its other channels are flushed towards zero).  Each
    group's list lies inside its own hot blocks and avoids the other group's."""
    T, K = 40, 128
    x = syn.normal_bf16(5, 3, T, K, 1.0)
    xf = syn.bf16_to_f32(x).astype(np.float64)
    hot = {0: [3, 70], 1: [40, 101]}
    off = np.array([0, 20, 40])
    for g, chans in hot.items():
        for c in chans:
            xf[off[g]:off[g + 1], c] *= 20.0
    x = orc.f64_to_bf16_array(xf)
    sel, _ = orc.calibrate_grouped(x, off, 16)
    for g, chans in hot.items():
        own = {c // 16 for c in chans}
        other = {c // 16 for c in hot[1 - g]}
        blocks = {int(c) // 16 for c in sel[g]}
        assert blocks <= own and not (blocks & other), (g, sel[g])


def test_grouped_selection_drops_no_more_residual_energy_than_shared(orc):
    """For every group, the residual energy left outside its own list is at most what the shared
    list leaves outside (the group's list takes the group's Kp largest e_k)."""
    wl = syn.dense_tiny()
    x = wl.x_cal
    off = np.array([0, 16, 40, x.shape[0]])
    Kp = wl.Kp
    sel_g, err_g = orc.calibrate_grouped(x, off, Kp)
    sel_s, _ = orc.calibrate(x, Kp)
    for g in range(off.size - 1):
        mask_g = np.ones(x.shape[1], bool)
        mask_g[sel_g[g]] = False
        mask_s = np.ones(x.shape[1], bool)
        mask_s[sel_s] = False
        assert err_g[g][mask_g].sum() <= err_g[g][mask_s].sum()


def test_grouped_residual_rows_follow_their_group(orc):
    x, _ = _grouped_batch(T=12, K=128)
    s_g = orc.global_scale(orc.amax_bf16(x))
    rng = np.random.default_rng(3)
    sel = np.stack([np.sort(rng.choice(128, 64, replace=False)) for _ in range(3)]).astype(np.int32)
    rg = np.array([2, 0, -1, 1, 1, 0, 2, -1, 0, 0, 1, 2])
    codes, S, rc, rS, rr = orc.act_quant_rac_grouped(x, s_g, sel, rg)
    c0, S0, _, _, _ = orc.act_quant_rac(x, s_g, sel[0])
    assert np.array_equal(codes, c0) and np.array_equal(S, S0)  # the main pass ignores the lists
    xf = syn.bf16_to_f32(x)
    _, _, dq = orc.quantize_f32(xf, s_g)
    for t in range(x.shape[0]):
        if rg[t] < 0:
            assert not rc[t].any() and not rS[t].any() and not rr[t].any()
            continue
        r = (xf[t] - dq[t]).astype(np.float32)[sel[rg[t]]]
        assert np.array_equal(rr[t], r), t
        c2, S2, _ = orc.quantize_f32(r[None, :], s_g)
        assert np.array_equal(rc[t], c2[0]) and np.array_equal(rS[t], S2[0]), t
    # one list for every group reduces to the shared residual
    same = np.stack([sel[1]] * 3)
    _, _, rc1, rS1, _ = orc.act_quant_rac_grouped(x, s_g, same, np.abs(rg))
    _, _, rc2, rS2, _ = orc.act_quant_rac(x, s_g, sel[1])
    assert np.array_equal(rc1, rc2) and np.array_equal(rS1, rS2)


def test_grouped_weight_sel_is_each_experts_raw_columns(orc):
    E, N, K = 3, 32, 128
    w = np.stack([syn.normal_bf16(e, 2, N, K, 0.02) for e in range(E)])
    s_w = np.array([orc.global_scale(orc.amax_bf16(w[e])) for e in range(E)], np.float32)
    rng = np.random.default_rng(8)
    sel = np.stack([np.sort(rng.choice(K, 64, replace=False)) for _ in range(E)]).astype(np.int32)
    codes, S, sc, sS = orc.weight_pack_grouped(w, s_w, sel)
    for e in range(E):
        c2, S2, _ = orc.quantize_f32(syn.bf16_to_f32(w[e])[:, sel[e]], s_w[e])
        assert np.array_equal(sc[e], c2) and np.array_equal(sS[e], S2)
        c3, S3, _ = orc.quantize_f32(syn.bf16_to_f32(w[e]), s_w[e])
        assert np.array_equal(codes[e], c3) and np.array_equal(S[e], S3)


def test_own_scale_residual_largest_block_scale_is_448(orc):
    """With its own tensor scale s_r = amax(R_sel) / 2688 the block holding the residual's amax gets
    the largest finite E4M3 scale (448, code 0x7E) and no block scale is larger; with the shared
    scale of X the residual's scales stay far below it.  A mix-up of the two scales fails here."""
    wl = syn.dense_tiny()
    sel, _ = orc.calibrate(wl.x_cal, wl.Kp)
    s_x = orc.global_scale(orc.amax_bf16(wl.x))
    _, _, rc_sh, rS_sh, resid = orc.act_quant_rac(wl.x, s_x, sel)
    codes, S, rc, rS, s_r = orc.act_quant_rac_own(wl.x, s_x, sel)
    assert s_r == orc.global_scale(np.float32(np.abs(resid).max()))
    assert rS.max() == 0x7E and S.max() == 0x7E
    assert rS_sh.max() < 0x70
    # main codes do not depend on the residual's scale
    c2, S2, _, _, _ = orc.act_quant_rac(wl.x, s_x, sel)
    assert np.array_equal(codes, c2) and np.array_equal(S, S2)


def test_own_scale_residual_is_scale_equivariant(orc):
    """x -> 2^k x (exact in bf16) leaves every code and block scale unchanged and multiplies s_x and
    s_r by 2^k."""
    wl = syn.dense_tiny()
    sel, _ = orc.calibrate(wl.x_cal, wl.Kp)
    x = wl.x
    x8 = (syn.bf16_to_f32(x) * np.float32(8.0)).astype(np.float32).view(np.uint32) >> 16
    x8 = x8.astype(np.uint16)
    s_x = orc.global_scale(orc.amax_bf16(x))
    s_x8 = orc.global_scale(orc.amax_bf16(x8))
    assert s_x8 == np.float32(8.0) * s_x
    a = orc.act_quant_rac_own(x, s_x, sel)
    b = orc.act_quant_rac_own(x8, s_x8, sel)
    for u, v in zip(a[:4], b[:4]):
        assert np.array_equal(u, v)
    assert b[4] == np.float32(8.0) * a[4]


def test_own_scale_gemm_is_the_sum_of_both_scaled_products(orc):
    """gemm_rac_own equals the float64 product of the dequantised operands, each residual factor
    taken with its own scale (s_r for R_sel, s_w for W_sel); with s_r = s_x it is the shared-scale
    GEMM; with no channels it is plain W4A4."""
    wl = syn.dense_tiny()
    sel, _ = orc.calibrate(wl.x_cal, wl.Kp)
    s_x = orc.global_scale(orc.amax_bf16(wl.x))
    s_w = orc.global_scale(orc.amax_bf16(wl.w))
    codes, S, rc, rS, s_r = orc.act_quant_rac_own(wl.x, s_x, sel)
    wc, wS, wsc, wsS = orc.weight_pack(wl.w, s_w, sel)
    y, _ = orc.gemm_rac_own(codes, S, rc, rS, wc, wS, wsc, wsS, s_x, s_r, s_w)
    ref = orc.dequant(codes, S, s_x) @ orc.dequant(wc, wS, s_w).T + \
        orc.dequant(rc, rS, s_r) @ orc.dequant(wsc, wsS, s_w).T
    assert np.allclose(y, ref, rtol=1e-12, atol=1e-12)
    _, _, rc2, rS2, _ = orc.act_quant_rac_own(wl.x, s_x, sel, s_r=s_x)
    _, _, rc3, rS3, _ = orc.act_quant_rac(wl.x, s_x, sel)
    assert np.array_equal(rc2, rc3) and np.array_equal(rS2, rS3)
    y_sh, _ = orc.gemm_rac_own(codes, S, rc3, rS3, wc, wS, wsc, wsS, s_x, s_x, s_w)
    y_ref, ad = orc.gemm_rac(codes, S, rc3, rS3, wc, wS, wsc, wsS, s_x, s_w)
    assert np.all(np.abs(y_sh - y_ref) <= 1e-13 * ad)  # two binary64 sums instead of one
    y0, _ = orc.gemm_rac_own(codes, S, None, None, wc, wS, None, None, s_x, s_r, s_w)
    y0_ref, _ = orc.gemm_rac(codes, S, None, None, wc, wS, None, None, s_x, s_w)
    assert np.array_equal(y0, y0_ref)


def test_own_scale_wins_where_shared_residual_scales_are_subnormal(orc):
    """A few very large channels raise s_x so far that the other channels' residual block scales
    under s_x fall into the E4M3 subnormals (or to zero); quantised with its own scale the
    residual then loses far less (the case the variant is for)."""
    K = 256
    x = syn.normal_bf16(5, 1, 64, K, 1.0, np.where(np.arange(K) < 4, 3.0e5, 1.0))
    sel = np.arange(64, 128, dtype=np.int32)  # ordinary channels only
    s_x = orc.global_scale(orc.amax_bf16(x))
    _, _, rc, rS, resid = orc.act_quant_rac(x, s_x, sel)
    assert np.all(rS < 8)                        # subnormal (or zero) residual block scales under s_x
    _, _, rco, rSo, s_r = orc.act_quant_rac_own(x, s_x, sel)
    e_sh = np.linalg.norm(resid - orc.dequant(rc, rS, s_x))
    e_own = np.linalg.norm(resid - orc.dequant(rco, rSo, s_r))
    assert e_own < 0.5 * e_sh


def test_own_scale_residual_changes_little_on_the_workload_inputs(orc):
    """The variant that quantises R_sel with its own tensor scale (s_r = amax(R_sel) / 2688, two
    accumulators) would change the activation error only where shared-scale residual block scales
    fall into the E4M3 subnormals; on inputs with the MoE prefill statistics none do, and the
    activation error moves by under 0.1 %."""
    wl = syn.moe_block(T=256, H=2048, E=16, topk=8, I=768, T_cal=256)
    sel, _ = orc.calibrate(wl.x_cal, 1024)
    x = wl.x
    s_x = orc.global_scale(orc.amax_bf16(x))
    codes, S, rc, rS, resid = orc.act_quant_rac(x, s_x, sel)
    assert not np.any((rS > 0) & (rS < 8))  # no subnormal residual block scale
    _, _, dq_x = orc.quantize_f32(syn.bf16_to_f32(x), s_x)
    _, _, dq_shared = orc.quantize_f32(resid, s_x)
    s_r = orc.global_scale(np.float32(np.abs(resid).max()))
    _, _, dq_own = orc.quantize_f32(resid, s_r)
    xf = syn.bf16_to_f32(x).astype(np.float64)
    unsel = np.ones(x.shape[1], bool)
    unsel[sel] = False
    main_err = np.linalg.norm((xf - dq_x)[:, unsel]) ** 2
    e_shared = np.sqrt(main_err + np.linalg.norm(resid.astype(np.float64) - dq_shared) ** 2)
    e_own = np.sqrt(main_err + np.linalg.norm(resid.astype(np.float64) - dq_own) ** 2)
    assert abs(e_own - e_shared) <= 1e-3 * e_shared
    assert e_shared < 0.6 * np.linalg.norm(xf - dq_x)  # the shared-scale residual pass does work
