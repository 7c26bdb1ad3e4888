"""CPU oracle for the NVFP4 W4A4 + RAC path (TEST INFRASTRUCTURE ONLY).

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline / reference leg of
``bench.py`` may import this package.  The product path (the CUDA library and its
binding) never loads it, and it never loads the product path: the two share no
code.  All arithmetic lives in ``nvfp4_oracle.c``; this module compiles it with
gcc (binary32 with round-to-nearest, no fast-math, no FMA contraction) and
marshals numpy arrays in and out.

Layouts here are logical: one E2M1 code per byte, one E4M3 scale code per
16-element block in row-major ``[rows, L/16]`` order, bf16 values as uint16 bit
patterns.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "nvfp4_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle next to its source."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-ffp-contract=off",
                               "-fno-fast-math", "-std=c11", _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _get():
    global _lib
    if _lib is not None:
        return _lib
    lib = ctypes.CDLL(build())
    vp, i64, i32, f32, f64 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_float, ctypes.c_double
    sigs = {
        "orc_bf16_to_f32": ([ctypes.c_uint16], f32),
        "orc_f64_to_bf16": ([f64], ctypes.c_uint16),
        "orc_f32_to_bf16": ([f32], ctypes.c_uint16),
        "orc_e2m1_decode": ([ctypes.c_int], f64),
        "orc_e2m1_encode": ([f32], ctypes.c_int),
        "orc_e4m3_decode": ([ctypes.c_int], f64),
        "orc_e4m3_encode": ([f32], ctypes.c_int),
        "orc_amax_bf16": ([vp, i64, i64, i64], f32),
        "orc_amax_f32": ([vp, i64], f32),
        "orc_global_scale": ([f32], f32),
        "orc_quantize_f32": ([vp, i64, i64, f32, vp, vp, vp], None),
        "orc_act_quant_rac": ([vp, i64, i64, i64, f32, vp, i32, vp, vp, vp, vp, vp], None),
        "orc_weight_pack": ([vp, i64, i64, f32, vp, i32, vp, vp, vp, vp], None),
        "orc_weight_qdq": ([vp, i64, f32, vp], None),
        "orc_gemm_rac": ([vp, vp, vp, vp, i64, i32, vp, vp, vp, vp, i64, f64, f64, vp, i64, vp, vp], None),
        "orc_calibrate": ([vp, i64, i64, i32, vp, vp], None),
        "orc_calibrate_grouped": ([vp, i64, i64, vp, i32, i32, vp, vp], None),
        "orc_swiglu": ([vp, i64, i64, vp, vp], None),
        "orc_e2m1_encode_array": ([vp, i64, vp], None),
        "orc_e4m3_encode_array": ([vp, i64, vp], None),
        "orc_f64_to_bf16_array": ([vp, i64, vp], None),
        "orc_num_threads": ([], ctypes.c_int),
        "orc_act_quant_masked": ([vp, i64, i64, i64, f32, vp, i32, vp, vp, vp, vp], None),
        "orc_route_topk": ([vp, i64, i32, i32, vp, vp], None),
        "orc_dispatch_plan": ([vp, i64, i32, i32, i32, vp, vp], None),
        "orc_combine": ([vp, i64, vp, vp, i64, i32, i64, vp], None),
        "orc_mx8_exponent": ([f32], ctypes.c_int),
        "orc_e4m3_encode_signed": ([f32], ctypes.c_int),
        "orc_e4m3_decode_signed": ([ctypes.c_int], f64),
        "orc_mx8_quantize": ([vp, i64, i64, i64, vp, vp], None),
        "orc_mx8_gemm": ([vp, vp, vp, vp, i64, i64, i64, vp, vp], None),
    }
    for name, (args, res) in sigs.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = res
    _lib = lib
    return lib


def _p(a: np.ndarray | None):
    return None if a is None else a.ctypes.data


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def num_threads() -> int:
    return int(_get().orc_num_threads())


# -------------------------------------------------------------------------- codecs
def e2m1_decode(code: int) -> float:
    return float(_get().orc_e2m1_decode(int(code)))


def e2m1_encode(v: float) -> int:
    return int(_get().orc_e2m1_encode(float(v)))


def e4m3_decode(code: int) -> float:
    return float(_get().orc_e4m3_decode(int(code)))


def e4m3_encode(raw: float) -> int:
    return int(_get().orc_e4m3_encode(float(raw)))


def e2m1_encode_array(v: np.ndarray) -> np.ndarray:
    v = _c(v, np.float32).reshape(-1)
    out = np.empty(v.size, dtype=np.uint8)
    _get().orc_e2m1_encode_array(_p(v), v.size, _p(out))
    return out


def e4m3_encode_array(v: np.ndarray) -> np.ndarray:
    v = _c(v, np.float32).reshape(-1)
    out = np.empty(v.size, dtype=np.uint8)
    _get().orc_e4m3_encode_array(_p(v), v.size, _p(out))
    return out


def f64_to_bf16(d: float) -> int:
    return int(_get().orc_f64_to_bf16(float(d)))


def f64_to_bf16_array(v: np.ndarray) -> np.ndarray:
    v = _c(v, np.float64)
    out = np.empty(v.shape, dtype=np.uint16)
    _get().orc_f64_to_bf16_array(_p(v), v.size, _p(out))
    return out


def bf16_to_f32(b: int) -> float:
    return float(_get().orc_bf16_to_f32(int(b)))


# -------------------------------------------------------------------------- scales
def amax_bf16(x: np.ndarray) -> np.float32:
    x = _c(x, np.uint16)
    rows, cols = x.shape
    return np.float32(_get().orc_amax_bf16(_p(x), rows, cols, cols))


def global_scale(amax: float) -> np.float32:
    return np.float32(_get().orc_global_scale(np.float32(amax)))


# -------------------------------------------------------------------------- quantisation
def quantize_f32(t: np.ndarray, s_g: float):
    """Quantise float32 rows [rows, L] with per-tensor scale s_g -> (codes, S, dq)."""
    t = _c(t, np.float32)
    rows, L = t.shape
    codes = np.empty((rows, L), np.uint8)
    S = np.empty((rows, L // 16), np.uint8)
    dq = np.empty((rows, L), np.float32)
    _get().orc_quantize_f32(_p(t), rows, L, np.float32(s_g), _p(codes), _p(S), _p(dq))
    return codes, S, dq


def act_quant_rac(x: np.ndarray, s_g: float, sel: np.ndarray):
    """bf16 x [rows, K] -> (codes [rows,K], S [rows,K/16], rcodes [rows,Kp], rS [rows,Kp/16], resid [rows,Kp])."""
    x = _c(x, np.uint16)
    rows, K = x.shape
    sel = _c(sel, np.int32)
    Kp = sel.size
    codes = np.empty((rows, K), np.uint8)
    S = np.empty((rows, K // 16), np.uint8)
    rcodes = np.empty((rows, Kp), np.uint8)
    rS = np.empty((rows, Kp // 16), np.uint8)
    resid = np.empty((rows, Kp), np.float32)
    _get().orc_act_quant_rac(_p(x), rows, K, K, np.float32(s_g), _p(sel), Kp, _p(codes), _p(S), _p(rcodes),
                             _p(rS), _p(resid))
    return codes, S, rcodes, rS, resid


def act_quant_rac_own(x: np.ndarray, s_g: float, sel: np.ndarray, s_r: float | None = None):
    """RAC variant with the residual's own tensor scale: the main pass and R_sel exactly as in
    act_quant_rac, then R_sel quantised with s_r = RN(amax(R_sel) / 2688) (amax over every row of
    the tensor) instead of s_g.  s_r may be given (an amax taken over a larger batch).
    -> (codes, S, rcodes, rS, s_r)."""
    codes, S, _, _, resid = act_quant_rac(x, s_g, sel)
    if resid.size == 0:
        rows = resid.shape[0]
        return codes, S, np.zeros((rows, 0), np.uint8), np.zeros((rows, 0), np.uint8), np.float32(0.0)
    if s_r is None:
        s_r = global_scale(amax_f32(resid))
    rcodes, rS, _ = quantize_f32(resid, s_r)
    return codes, S, rcodes, rS, np.float32(s_r)


def gemm_rac_own(a, aS, r, rS, w, wS, ws, wsS, s_a: float, s_r: float, s_w: float, rows=None):
    """The two-accumulator form of the RAC GEMM: y = s_a s_w (Q(X) Q(W)^T) + s_r s_w (Q(R_sel)
    Q(W_sel)^T), each product exact (gemm_rac with no residual), scaled and summed in binary64.
    -> (y float64, absdot of both products)."""
    y1, ad1 = gemm_rac(a, aS, None, None, w, wS, None, None, s_a, s_w, rows=rows)
    if r is None or r.size == 0:
        return y1, ad1
    y2, ad2 = gemm_rac(r, rS, None, None, ws, wsS, None, None, s_r, s_w, rows=rows)
    return y1 + y2, ad1 + ad2


def amax_f32(t: np.ndarray) -> np.float32:
    t = _c(t, np.float32).reshape(-1)
    return np.float32(_get().orc_amax_f32(_p(t), t.size))


def act_quant_masked(x: np.ndarray, s_g: float, sel: np.ndarray):
    """RAC variant with the residual kept at its channels (zero off sel) and quantised along K:
    bf16 x [rows, K] -> (codes [rows,K], S [rows,K/16], mcodes [rows,K], mS [rows,K/16])."""
    x = _c(x, np.uint16)
    rows, K = x.shape
    sel = _c(sel, np.int32)
    codes = np.empty((rows, K), np.uint8)
    S = np.empty((rows, K // 16), np.uint8)
    mcodes = np.empty((rows, K), np.uint8)
    mS = np.empty((rows, K // 16), np.uint8)
    _get().orc_act_quant_masked(_p(x), rows, K, K, np.float32(s_g), _p(sel), sel.size, _p(codes), _p(S),
                                _p(mcodes), _p(mS))
    return codes, S, mcodes, mS


def masked_rac_forward(x: np.ndarray, w: np.ndarray, sel: np.ndarray):
    """Y = s_x s_w (Q(X) Q(W)^T + Q(M) Q(W)^T) for the masked full-K variant -> (y float64, absdot)."""
    s_x = global_scale(amax_bf16(x))
    s_w = global_scale(amax_bf16(w))
    codes, S, mcodes, mS = act_quant_masked(x, s_x, sel)
    wc, wS, _, _ = weight_pack(w, s_w, np.zeros(0, np.int32))
    return gemm_rac(codes, S, mcodes, mS, wc, wS, wc, wS, s_x, s_w)


def weight_pack(w: np.ndarray, s_gw: float, sel: np.ndarray):
    """bf16 w [N, K] -> (codes, S, sel codes [N,Kp], sel S [N,Kp/16]) with one per-tensor scale s_gw."""
    w = _c(w, np.uint16)
    N, K = w.shape
    sel = _c(sel, np.int32)
    Kp = sel.size
    codes = np.empty((N, K), np.uint8)
    S = np.empty((N, K // 16), np.uint8)
    sc = np.empty((N, Kp), np.uint8)
    sS = np.empty((N, Kp // 16), np.uint8)
    _get().orc_weight_pack(_p(w), N, K, np.float32(s_gw), _p(sel), Kp, _p(codes), _p(S), _p(sc), _p(sS))
    return codes, S, sc, sS


def weight_qdq(w: np.ndarray, s_g: float | None = None):
    """Trainer fake-quant of one tensor -> (bf16 out, s_g)."""
    w = _c(w, np.uint16)
    if s_g is None:
        s_g = global_scale(amax_bf16(w.reshape(1, -1)))
    out = np.empty_like(w)
    _get().orc_weight_qdq(_p(w), w.size, np.float32(s_g), _p(out))
    return out, np.float32(s_g)


def gemm_rac(a, aS, r, rS, w, wS, ws, wsS, s_a: float, s_w: float, rows=None):
    """Exact W4A4 + residual GEMM on logical codes.  Returns (y [n_rows, N] float64, absdot)."""
    a, aS, w, wS = _c(a, np.uint8), _c(aS, np.uint8), _c(w, np.uint8), _c(wS, np.uint8)
    M, K = a.shape
    N = w.shape[0]
    assert w.shape[1] == K
    if r is None or r.size == 0:
        Kp = 0
        r = np.zeros((M, 0), np.uint8)
        rS = np.zeros((M, 0), np.uint8)
        ws = np.zeros((N, 0), np.uint8)
        wsS = np.zeros((N, 0), np.uint8)
    r, rS, ws, wsS = _c(r, np.uint8), _c(rS, np.uint8), _c(ws, np.uint8), _c(wsS, np.uint8)
    Kp = r.shape[1]
    rows = np.arange(M, dtype=np.int64) if rows is None else _c(rows, np.int64)
    y = np.empty((rows.size, N), np.float64)
    ad = np.empty((rows.size, N), np.float64)
    _get().orc_gemm_rac(_p(a), _p(aS), _p(r), _p(rS), K, Kp, _p(w), _p(wS), _p(ws), _p(wsS), N, float(s_a),
                        float(s_w), _p(rows), rows.size, _p(y), _p(ad))
    return y, ad


def calibrate(x_cal: np.ndarray, Kp: int):
    """RAC channel selection -> (sel ascending int32 [Kp], per-channel error float64 [K])."""
    x = _c(x_cal, np.uint16)
    T, K = x.shape
    sel = np.empty(Kp, np.int32)
    err = np.empty(K, np.float64)
    _get().orc_calibrate(_p(x), T, K, int(Kp), _p(sel), _p(err))
    return sel, err


def calibrate_grouped(x_cal: np.ndarray, offsets: np.ndarray, Kp: int):
    """Per-expert RAC selection: rows [offsets[g], offsets[g+1]) of the calibration batch form
    group g; the batch is quantised once with its own s_g and each group keeps the Kp channels with
    the largest error over its own rows -> (sel int32 [G, Kp] ascending per row, err float64 [G, K])."""
    x = _c(x_cal, np.uint16)
    T, K = x.shape
    off = _c(offsets, np.int64)
    G = off.size - 1
    assert G >= 1 and off[0] == 0 and off[-1] == T and np.all(np.diff(off) >= 0)
    sel = np.empty((G, Kp), np.int32)
    err = np.empty((G, K), np.float64)
    _get().orc_calibrate_grouped(_p(x), T, K, _p(off), G, int(Kp), _p(sel), _p(err))
    return sel, err


def act_quant_rac_grouped(x: np.ndarray, s_g: float, sel: np.ndarray, row_group: np.ndarray):
    """act_quant_rac with one channel list per group: row t uses sel[row_group[t]] (all rows share
    s_g); a row with row_group < 0 gets an all-zero residual (codes 0, scales 0)."""
    x = _c(x, np.uint16)
    sel = _c(sel, np.int32)
    rows, K = x.shape
    G, Kp = sel.shape
    rg = np.asarray(row_group, np.int64)
    codes, S, _, _, _ = act_quant_rac(x, s_g, np.zeros(0, np.int32))
    rcodes = np.zeros((rows, Kp), np.uint8)
    rS = np.zeros((rows, Kp // 16), np.uint8)
    resid = np.zeros((rows, Kp), np.float32)
    for g in range(G):
        idx = np.nonzero(rg == g)[0]
        if idx.size == 0:
            continue
        _, _, rc, rs, rr = act_quant_rac(x[idx], s_g, sel[g])
        rcodes[idx], rS[idx], resid[idx] = rc, rs, rr
    return codes, S, rcodes, rS, resid


def weight_pack_grouped(w: np.ndarray, s_gw: np.ndarray, sel: np.ndarray):
    """weight_pack of E expert matrices w [E, N, K], expert e with its own s_gw[e] and channel
    list sel[e] -> (codes [E,N,K], S, sel codes [E,N,Kp], sel S)."""
    outs = [weight_pack(w[e], float(s_gw[e]), sel[e]) for e in range(w.shape[0])]
    return tuple(np.stack([o[i] for o in outs]) for i in range(4))


def route_topk(logits: np.ndarray, k: int):
    """Router: float32 logits [T, E] -> (expert ids int32 [T, k], best first; weights float32 [T, k])."""
    lg = _c(logits, np.float32)
    T, E = lg.shape
    ids = np.empty((T, k), np.int32)
    w = np.empty((T, k), np.float32)
    _get().orc_route_topk(_p(lg), T, E, int(k), _p(ids), _p(w))
    return ids, w


def dispatch_plan(ids: np.ndarray, E: int, pad: int):
    """Expert-grouped layout of the (token, expert) pairs -> (offsets int64 [E+1], row int64 [T, k])."""
    ids = _c(ids, np.int32)
    T, k = ids.shape
    off = np.empty(E + 1, np.int64)
    row = np.empty((T, k), np.int64)
    _get().orc_dispatch_plan(_p(ids), T, int(k), int(E), int(pad), _p(off), _p(row))
    return off, row


def combine(y: np.ndarray, row: np.ndarray, w: np.ndarray):
    """out[t] = sum_j w[t, j] * y[row[t, j]] in binary64; y bf16 bits [R, H] -> float64 [T, H]."""
    y = _c(y, np.uint16)
    row = _c(row, np.int64)
    w = _c(w, np.float32)
    T, k = row.shape
    H = y.shape[1]
    out = np.empty((T, H), np.float64)
    _get().orc_combine(_p(y), H, _p(row), _p(w), T, int(k), H, _p(out))
    return out


def swiglu(gu: np.ndarray):
    """bf16 gate_up [rows, 2I] (gate first) -> (h bf16 [rows, I], h exact float64)."""
    gu = _c(gu, np.uint16)
    rows, two_i = gu.shape
    I = two_i // 2
    h = np.empty((rows, I), np.uint16)
    hx = np.empty((rows, I), np.float64)
    _get().orc_swiglu(_p(gu), rows, I, _p(h), _p(hx))
    return h, hx


# -------------------------------------------------------------------------- composite helpers
def dequant(codes: np.ndarray, S: np.ndarray, s_g: float) -> np.ndarray:
    """binary64 value of logical codes: e(q) * S(block) * s_g (exact products of small dyadics and s_g)."""
    mag = np.array([0, .5, 1, 1.5, 2, 3, 4, 6], np.float64)
    e = mag[codes & 7] * np.where(codes & 8, -1.0, 1.0)
    svals = np.array([e4m3_decode(c) if c != 0x7F and c != 0xFF else np.nan for c in range(256)])
    s = np.repeat(svals[S], 16, axis=-1)
    return e * s * float(s_g)


def dense_rac_forward(x: np.ndarray, w: np.ndarray, sel: np.ndarray, rows=None):
    """Full oracle of the dense W4A4 + RAC linear: quantise X (own s_g) with residual on sel,
    pack W (own s_gw), exact GEMM.  Returns dict with all intermediates and y (float64)."""
    s_x = global_scale(amax_bf16(x))
    a, aS, r, rS, resid = act_quant_rac(x, s_x, sel)
    s_w = global_scale(amax_bf16(w))
    wc, wS, wsc, wsS = weight_pack(w, s_w, sel)
    y, ad = gemm_rac(a, aS, r, rS, wc, wS, wsc, wsS, s_x, s_w, rows=rows)
    return dict(s_x=s_x, a=a, aS=aS, r=r, rS=rS, resid=resid, s_w=s_w, wc=wc, wS=wS, wsc=wsc, wsS=wsS, y=y,
                absdot=ad)


# ---- FP8 comparison format: E4M3 elements, one power-of-two scale per 32 elements along K ----
def mx8_exponent(b: float) -> int:
    """Smallest X in [-127, 127] with 448 * 2^X >= b."""
    return int(_get().orc_mx8_exponent(np.float32(b)))


def e4m3_encode_signed(v: float) -> int:
    return int(_get().orc_e4m3_encode_signed(np.float32(v)))


def e4m3_decode_signed(code: int) -> float:
    return float(_get().orc_e4m3_decode_signed(int(code)))


def mx8_quantize(x: np.ndarray):
    """bf16 x [rows, K] (K % 32 == 0) -> (codes uint8 [rows, K], E8M0 scale codes uint8 [rows, K/32])."""
    x = _c(x, np.uint16)
    rows, K = x.shape
    codes = np.empty((rows, K), np.uint8)
    S = np.empty((rows, K // 32), np.uint8)
    _get().orc_mx8_quantize(_p(x), rows, K, K, _p(codes), _p(S))
    return codes, S


def mx8_dequant(codes: np.ndarray, S: np.ndarray) -> np.ndarray:
    """Values of MXFP8 codes as float64 [rows, K]."""
    table = np.array([e4m3_decode_signed(c) for c in range(256)])
    rows, K = codes.shape
    scale = np.ldexp(1.0, S.astype(np.int64) - 127)
    return table[codes] * np.repeat(scale, 32, axis=1).reshape(rows, K)


def mx8_gemm(ac, aS, wc, wS):
    """y = A W^T over MXFP8 operands (block sums exact, added in binary64) -> (y, absdot)."""
    ac, aS, wc, wS = (_c(v, np.uint8) for v in (ac, aS, wc, wS))
    rows, K = ac.shape
    N = wc.shape[0]
    y = np.empty((rows, N), np.float64)
    ad = np.empty((rows, N), np.float64)
    _get().orc_mx8_gemm(_p(ac), _p(aS), _p(wc), _p(wS), rows, N, K, _p(y), _p(ad))
    return y, ad
