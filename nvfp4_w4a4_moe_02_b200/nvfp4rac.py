"""Python binding of the C-ABI library ``libnvfp4rac.so`` (ctypes).

Argument marshalling only: every step of the NVFP4 W4A4 + RAC path runs in the CUDA
kernels behind the C ABI (declared in ``include/nvfp4rac.h``).  PyTorch provides device
memory and the current stream.  If the compiled library is missing, loading it raises: there
is no fallback implementation.

Call names match the C ABI: ``nvfp4_quantize``, ``rac_calibrate``, ``pack_weights``,
``w4a4_rac_gemm``, ``grouped_w4a4_rac_moe``, ``weight_qdq``.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libnvfp4rac.so")

OK = 0
STATUS_NAMES = {0: "OK", 1: "ERR_INVALID_ARG", 2: "ERR_UNSUPPORTED_SHAPE", 3: "ERR_ALIGNMENT", 4: "ERR_RANGE",
                5: "ERR_CUDA", 6: "ERR_TIMEOUT"}
OUT_F32, OUT_BF16 = 0, 1
RAC_OWN_RES_SCALE = 1  # the residual's own tensor scale (quantise and GEMM *_ex calls)
EPI_NONE, EPI_SWIGLU_AMAX = 0, 1


class NVFP4Error(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {msg}")
        self.status = status


class CTensor(ctypes.Structure):
    _fields_ = [("codes", ctypes.c_void_p), ("sf", ctypes.c_void_p), ("s_g", ctypes.c_void_p),
                ("slabs", ctypes.c_int64), ("rows", ctypes.c_int64), ("rows_padded", ctypes.c_int64),
                ("cols", ctypes.c_int64), ("sf_layout", ctypes.c_int32)]


_lib = None


def load() -> ctypes.CDLL:
    """Load the CUDA library (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m nvfp4_w4a4_moe_02_b200.build_lib`")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i64, i32, sz, u64 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_size_t, ctypes.c_uint64
    tp = ctypes.POINTER(CTensor)
    sigs = {
        "nvfp4_version": ([], i32),
        "nvfp4_status_string": ([ctypes.c_int], ctypes.c_char_p),
        "nvfp4_last_error_string": ([], ctypes.c_char_p),
        "nvfp4_codes_bytes": ([i64, i64], sz),
        "nvfp4_sf_bytes": ([i64, i64], sz),
        "nvfp4_sf_bytes_layout": ([i64, i64, i32], sz),
        "nvfp4_kp_from_ratio": ([i64, ctypes.c_double], i32),
        "nvfp4_set_wait_limit_ns": ([u64], None),
        "nvfp4_set_gemm_tile_n": ([i32], None),
        "nvfp4_set_act_tile": ([i32, i32], None),
        "nvfp4_set_gemm_pairs": ([i32], None),
        "nvfp4_set_qdq_one_pass": ([i32], None),
        "nvfp4_quantize_workspace_size": ([i64, i64], sz),
        "nvfp4_quantize": ([vp, i64, i64, i64, vp, i64, vp, i32, vp, tp, tp, vp, sz, vp, vp], ctypes.c_int),
        "nvfp4_quantize_scatter": ([vp, i64, i64, i64, vp, i32, vp, i32, vp, tp, tp, vp, sz, vp, vp], ctypes.c_int),
        "nvfp4_quantize_ex": ([vp, i64, i64, i64, vp, i64, vp, i32, vp, tp, tp, vp, sz, vp, vp, ctypes.c_uint32],
                              ctypes.c_int),
        "nvfp4_quantize_scatter_ex": ([vp, i64, i64, i64, vp, i32, vp, i32, vp, tp, tp, vp, sz, vp, vp,
                                       ctypes.c_uint32], ctypes.c_int),
        "nvfp4_quantize_segments_ex": ([vp, i64, i64, i64, vp, vp, i32, vp, i32, vp, tp, tp, vp, sz, vp, vp,
                                        ctypes.c_uint32], ctypes.c_int),
        "w4a4_rac_gemm_ex": ([tp, tp, tp, tp, i64, i64, i64, i32, ctypes.c_int, vp, i64, vp, vp, ctypes.c_uint32],
                             ctypes.c_int),
        "grouped_w4a4_rac_moe_ex": ([tp, tp, vp, vp, i32, tp, tp, i64, i64, i32, ctypes.c_int, ctypes.c_int, vp, i64,
                                     vp, vp, vp, ctypes.c_uint32], ctypes.c_int),
        "nvfp4_quantize_segments": ([vp, i64, i64, i64, vp, vp, i32, vp, i32, vp, tp, tp, vp, sz, vp, vp],
                                    ctypes.c_int),
        "nvfp4_quantize_grouped_sel": ([vp, i64, i64, i64, vp, i64, vp, i32, vp, i32, vp, tp, tp, vp, sz, vp, vp],
                                       ctypes.c_int),
        "rac_calibrate_workspace_size": ([i64, i64], sz),
        "rac_calibrate": ([vp, i64, i64, i32, vp, vp, vp, sz, vp, vp], ctypes.c_int),
        "rac_calibrate_grouped_workspace_size": ([i64, i64, i32], sz),
        "rac_calibrate_grouped": ([vp, i64, i64, vp, i32, i32, vp, vp, vp, sz, vp, vp], ctypes.c_int),
        "pack_weights_workspace_size": ([i64, i64, i64], sz),
        "pack_weights": ([vp, i64, i64, i64, vp, i32, i32, tp, tp, vp, sz, vp, vp], ctypes.c_int),
        "pack_weights_grouped_sel": ([vp, i64, i64, i64, vp, i32, i32, tp, tp, vp, sz, vp, vp], ctypes.c_int),
        "moe_row_groups": ([vp, i32, i64, vp, vp], ctypes.c_int),
        "w4a4_rac_gemm": ([tp, tp, tp, tp, i64, i64, i64, i32, ctypes.c_int, vp, i64, vp, vp], ctypes.c_int),
        "grouped_w4a4_rac_moe": ([tp, tp, vp, vp, i32, tp, tp, i64, i64, i32, ctypes.c_int, ctypes.c_int, vp, i64,
                                  vp, vp, vp], ctypes.c_int),
        "grouped_w4a4_rac_moe_segments": ([tp, tp, vp, vp, vp, i32, tp, tp, i64, i64, i32, ctypes.c_int,
                                           ctypes.c_int, vp, i64, vp, vp, vp], ctypes.c_int),
        "nvfp4_amax": ([vp, i64, i64, i64, vp, vp, sz, vp, vp], ctypes.c_int),
        "grouped_w4a4_rac_moe_decode": ([tp, tp, vp, vp, i32, i32, tp, tp, i64, i64, i32, ctypes.c_int, ctypes.c_int,
                                         vp, i64, vp, vp, vp], ctypes.c_int),
        "moe_route_topk": ([vp, i64, i32, i32, vp, vp, vp, vp], ctypes.c_int),
        "moe_rows_capacity": ([i64, i32, i32, i32], i64),
        "moe_dispatch_workspace_size": ([i32], sz),
        "moe_dispatch_plan": ([vp, i64, i32, i32, i32, i64, vp, vp, vp, vp, vp, i32, vp, sz, vp, vp], ctypes.c_int),
        "moe_combine": ([vp, i64, i64, vp, vp, i64, i32, i64, vp, i64, vp, vp], ctypes.c_int),
        "moe_row_pairs": ([vp, i64, i32, i64, vp, vp, vp], ctypes.c_int),
        "grouped_w4a4_rac_moe_combine": ([tp, tp, vp, vp, i32, tp, tp, i64, i64, i32, vp, vp, i64, i32, vp, vp, i64,
                                          vp, vp], ctypes.c_int),
        "weight_qdq_workspace_size": ([i64, i64], sz),
        "weight_qdq": ([vp, i64, i64, vp, vp, vp, sz, vp, vp], ctypes.c_int),
        "weight_qdq_backward": ([vp, i64, vp, vp, vp], ctypes.c_int),
        "nvfp4_unpack_logical": ([tp, i64, vp, vp, vp], ctypes.c_int),
        "nvfp4_encode_e2m1": ([vp, i64, vp, vp], ctypes.c_int),
        "nvfp4_encode_e4m3": ([vp, i64, vp, vp], ctypes.c_int),
        "nvfp4_selftest_wait_timeout": ([u64, vp, vp], ctypes.c_int),
    }
    for name, (args, res) in sigs.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = res
    _lib = lib
    return lib


def _check(status: int):
    if status != OK:
        raise NVFP4Error(status, load().nvfp4_last_error_string().decode())


def _stream(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _ptr(t):
    return None if t is None else t.data_ptr()


def _u16(x: torch.Tensor) -> torch.Tensor:
    assert x.is_cuda and x.dtype in (torch.bfloat16, torch.int16, torch.uint16), x.dtype
    return x


def round_up(v: int, a: int) -> int:
    return (v + a - 1) // a * a


SF_ATOM128, SF_SLAB16 = 0, 1


def sf_bytes(rows_padded: int, cols: int, sf_layout: int = SF_ATOM128) -> int:
    """Scale-atom bytes of one rows_padded x cols matrix (same rule as nvfp4_sf_bytes_layout)."""
    if sf_layout == SF_SLAB16:
        return rows_padded // 16 * (cols // 64) * 512
    return rows_padded * cols // 16


@dataclass
class Packed:
    """Caller-side owner of one packed NVFP4 tensor (device buffers allocated by torch)."""
    codes: torch.Tensor   # uint8 [slabs * rows_padded * cols/2]
    sf: torch.Tensor      # uint8 [slabs * sf_bytes(rows_padded, cols, sf_layout)]
    s_g: torch.Tensor     # float32 [slabs]
    slabs: int
    rows: int
    rows_padded: int
    cols: int
    sf_layout: int = SF_ATOM128

    @staticmethod
    def empty(rows: int, cols: int, slabs: int = 1, rows_padded: int | None = None, device="cuda",
              zero: bool = False, sf_layout: int = SF_ATOM128) -> "Packed":
        group = 16 if sf_layout == SF_SLAB16 else 128
        rp = round_up(max(rows, 1), group) if rows_padded is None else rows_padded
        alloc = torch.zeros if zero else torch.empty
        codes = alloc(slabs * rp * cols // 2, dtype=torch.uint8, device=device)
        sf = alloc(slabs * sf_bytes(rp, cols, sf_layout), dtype=torch.uint8, device=device)
        s_g = torch.empty(slabs, dtype=torch.float32, device=device)
        return Packed(codes, sf, s_g, slabs, rows, rp, cols, sf_layout)

    def c(self) -> CTensor:
        return CTensor(self.codes.data_ptr(), self.sf.data_ptr(), self.s_g.data_ptr(), self.slabs, self.rows,
                       self.rows_padded, self.cols, self.sf_layout)

    def prefix(self, rows_padded: int) -> "Packed":
        """View of the first rows_padded rows (a multiple of the scale layout's row group) of a
        single-slab tensor, sharing storage."""
        group = 16 if self.sf_layout == SF_SLAB16 else 128
        assert self.slabs == 1 and rows_padded % group == 0 and rows_padded <= self.rows_padded
        return Packed(self.codes[:rows_padded * self.cols // 2], self.sf[:sf_bytes(rows_padded, self.cols, self.sf_layout)],
                      self.s_g, 1, min(self.rows, rows_padded), rows_padded, self.cols, self.sf_layout)

    def slab(self, e: int) -> "Packed":
        """View of slab e alone (slabs = 1), sharing storage (e.g. to pack one expert at a time)."""
        cb = self.rows_padded * self.cols // 2
        sb = sf_bytes(self.rows_padded, self.cols, self.sf_layout)
        return Packed(self.codes[e * cb:(e + 1) * cb], self.sf[e * sb:(e + 1) * sb], self.s_g[e:e + 1], 1,
                      self.rows, self.rows_padded, self.cols, self.sf_layout)


class Workspace:
    """Grow-only device scratch buffer handed to calls that need one."""

    def __init__(self, device="cuda"):
        self.buf = torch.empty(0, dtype=torch.uint8, device=device)

    def get(self, nbytes: int) -> torch.Tensor:
        if self.buf.numel() < nbytes:
            self.buf = torch.empty(round_up(max(nbytes, 1), 1 << 20), dtype=torch.uint8, device=self.buf.device)
        return self.buf


_ws: dict = {}


def _workspace(device) -> Workspace:
    key = str(device)
    if key not in _ws:
        _ws[key] = Workspace(device)
    return _ws[key]


def new_status(device="cuda") -> torch.Tensor:
    return torch.zeros(1, dtype=torch.int32, device=device)


def check_status(status: torch.Tensor):
    """Raise if a device-side error was recorded (synchronises)."""
    v = int(status.item())
    if v != OK:
        raise NVFP4Error(v, "device-side error")


def kp_from_ratio(K: int, r: float) -> int:
    return int(load().nvfp4_kp_from_ratio(K, r))


def set_wait_limit_ns(ns: int):
    load().nvfp4_set_wait_limit_ns(ns)


def set_gemm_tile_n(n: int):
    """Force the GEMM N-tile (128 or 256); 0 restores the automatic choice."""
    load().nvfp4_set_gemm_tile_n(n)


def set_gemm_pairs(on: bool):
    """Run the GEMMs with N % 256 == 0 on CTA pairs or on single SMs (default)."""
    load().nvfp4_set_gemm_pairs(1 if on else 0)


def set_qdq_one_pass(on: bool):
    """weight_qdq in one pass over HBM (default, tensors of up to 4M elements) or in two."""
    load().nvfp4_set_qdq_one_pass(1 if on else 0)


def set_act_tile(rows: int, warps: int):
    """Force the activation quantiser's rows per tile and consumer warps; 0, 0 restores the
    automatic choice."""
    load().nvfp4_set_act_tile(rows, warps)


# ------------------------------------------------------------------------------------- calls
def nvfp4_quantize(x: torch.Tensor, sel: torch.Tensor | None = None, row_gather: torch.Tensor | None = None,
                   M_out: int | None = None, rows_padded: int | None = None, amax_in: torch.Tensor | None = None,
                   out: Packed | None = None, out_res: Packed | None = None, status: torch.Tensor | None = None,
                   stream=None, masked: bool = False, row_group: torch.Tensor | None = None, own_scale: bool = False):
    """Online activation quantisation with the residual pass on ``sel`` -> (Packed, Packed | None).

    masked=True selects the masked full-K residual variant (residual at its channel, zero off
    ``sel``, K wide): pair it with the main packed weight as w_sel in w4a4_rac_gemm.
    A 2-D ``sel`` [G, Kp] is one channel list per group (the per-expert variant): output row o
    uses list ``row_group[o]`` (int32 [rows_padded]; < 0 gives a zero residual row)."""
    lib = load()
    _u16(x)
    M, K = x.shape
    ldx = x.stride(0)
    assert x.stride(1) == 1
    grouped = sel is not None and sel.dim() == 2
    Kp = 0 if sel is None else int(sel.shape[-1])
    if M_out is None:
        M_out = M if row_gather is None else int(row_gather.numel())
    if out is None:
        out = Packed.empty(M_out, K, rows_padded=rows_padded, device=x.device)
    if Kp > 0 and out_res is None:
        out_res = Packed.empty(M_out, K if masked else Kp, rows_padded=out.rows_padded, device=x.device)
    ws_bytes = lib.nvfp4_quantize_workspace_size(M, K)
    ws = _workspace(x.device).get(ws_bytes)
    st = status if status is not None else new_status(x.device)
    q = out.c()
    qr = out_res.c() if Kp > 0 else None
    if grouped:
        assert not masked and row_group is not None and row_group.dtype == torch.int32
        assert sel.dtype == torch.int32 and sel.is_contiguous() and row_group.numel() >= out.rows_padded
        _check(lib.nvfp4_quantize_grouped_sel(x.data_ptr(), M, K, ldx, _ptr(row_gather), M_out, row_group.data_ptr(),
                                              int(sel.shape[0]), sel.data_ptr(), Kp, _ptr(amax_in), ctypes.byref(q),
                                              ctypes.byref(qr), ws.data_ptr(), ws.numel(), st.data_ptr(),
                                              _stream(stream)))
        return out, out_res
    _check(lib.nvfp4_quantize_ex(x.data_ptr(), M, K, ldx, _ptr(row_gather), M_out, _ptr(sel), Kp, _ptr(amax_in),
                                 ctypes.byref(q), ctypes.byref(qr) if qr is not None else None, ws.data_ptr(),
                                 ws.numel(), st.data_ptr(), _stream(stream), RAC_OWN_RES_SCALE if own_scale else 0))
    return out, (out_res if Kp > 0 else None)


def nvfp4_quantize_scatter(x: torch.Tensor, row_scatter: torch.Tensor, rows_padded: int,
                           sel: torch.Tensor | None = None, amax_in: torch.Tensor | None = None,
                           out: Packed | None = None, out_res: Packed | None = None,
                           status: torch.Tensor | None = None, stream=None, sf_layout: int = SF_ATOM128,
                           own_scale: bool = False):
    """Quantise each row of x once and write it to the rows row_scatter[m, :] of the outputs.

    row_scatter: int32 [M, fanout] (-1 = unused).  Rows no entry names are left untouched, so
    freshly created outputs are zero-filled.  sf_layout picks the scale order of outputs created
    here (SF_SLAB16 for the decode GEMM).  Returns (Packed, Packed | None)."""
    lib = load()
    _u16(x)
    M, K = x.shape
    assert x.stride(1) == 1 and row_scatter.dtype == torch.int32 and row_scatter.is_contiguous()
    fanout = row_scatter.shape[1]
    Kp = 0 if sel is None else int(sel.numel())
    if out is None:
        out = Packed.empty(rows_padded, K, rows_padded=rows_padded, device=x.device, zero=True, sf_layout=sf_layout)
    if Kp > 0 and out_res is None:
        out_res = Packed.empty(rows_padded, Kp, rows_padded=rows_padded, device=x.device, zero=True,
                               sf_layout=sf_layout)
    ws = _workspace(x.device).get(lib.nvfp4_quantize_workspace_size(M, K))
    st = status if status is not None else new_status(x.device)
    q = out.c()
    qr = out_res.c() if Kp > 0 else None
    _check(lib.nvfp4_quantize_scatter_ex(x.data_ptr(), M, K, x.stride(0), row_scatter.data_ptr(), fanout, _ptr(sel),
                                         Kp, _ptr(amax_in), ctypes.byref(q),
                                         ctypes.byref(qr) if qr is not None else None, ws.data_ptr(), ws.numel(),
                                         st.data_ptr(), _stream(stream), RAC_OWN_RES_SCALE if own_scale else 0))
    return out, (out_res if Kp > 0 else None)


def nvfp4_quantize_segments(x: torch.Tensor, expert_offsets: torch.Tensor, expert_rows: torch.Tensor,
                            sel: torch.Tensor | None = None, amax_in: torch.Tensor | None = None,
                            out: Packed | None = None, out_res: Packed | None = None,
                            status: torch.Tensor | None = None, stream=None, own_scale: bool = False):
    """Quantise only the token rows of an expert-grouped layout: rows
    [expert_offsets[e], expert_offsets[e] + expert_rows[e]) of x (device int32 [E] each) into the
    same rows of the outputs; other output rows are left as they are.  Returns (Packed, Packed | None)."""
    lib = load()
    _u16(x)
    M, K = x.shape
    assert x.stride(1) == 1
    assert expert_offsets.dtype == torch.int32 and expert_rows.dtype == torch.int32
    E = int(expert_rows.numel())
    Kp = 0 if sel is None else int(sel.numel())
    if out is None:
        out = Packed.empty(M, K, device=x.device, zero=True)
    if Kp > 0 and out_res is None:
        out_res = Packed.empty(M, Kp, rows_padded=out.rows_padded, device=x.device, zero=True)
    ws = _workspace(x.device).get(lib.nvfp4_quantize_workspace_size(M, K))
    st = status if status is not None else new_status(x.device)
    q = out.c()
    qr = out_res.c() if Kp > 0 else None
    _check(lib.nvfp4_quantize_segments_ex(x.data_ptr(), M, K, x.stride(0), expert_offsets.data_ptr(),
                                          expert_rows.data_ptr(), E, _ptr(sel), Kp, _ptr(amax_in), ctypes.byref(q),
                                          ctypes.byref(qr) if qr is not None else None, ws.data_ptr(), ws.numel(),
                                          st.data_ptr(), _stream(stream), RAC_OWN_RES_SCALE if own_scale else 0))
    return out, (out_res if Kp > 0 else None)


def rac_calibrate(x_cal: torch.Tensor, Kp: int, want_err: bool = False, status: torch.Tensor | None = None,
                  stream=None):
    """Select the Kp highest-error channels of a calibration batch -> (sel int32 [Kp], err float64 [K] | None)."""
    lib = load()
    _u16(x_cal)
    T, K = x_cal.shape
    assert x_cal.is_contiguous()
    sel = torch.empty(Kp, dtype=torch.int32, device=x_cal.device)
    err = torch.empty(K, dtype=torch.float64, device=x_cal.device) if want_err else None
    ws = _workspace(x_cal.device).get(lib.rac_calibrate_workspace_size(T, K))
    st = status if status is not None else new_status(x_cal.device)
    _check(lib.rac_calibrate(x_cal.data_ptr(), T, K, Kp, sel.data_ptr(), _ptr(err), ws.data_ptr(), ws.numel(),
                             st.data_ptr(), _stream(stream)))
    return sel, err


def rac_calibrate_grouped(x_cal: torch.Tensor, offsets: torch.Tensor, Kp: int, want_err: bool = False,
                          status: torch.Tensor | None = None, stream=None):
    """One channel list per group of calibration rows (group g = rows [offsets[g], offsets[g+1]),
    int32 device tensor [G + 1]) -> (sel int32 [G, Kp], err float64 [G, K] | None)."""
    lib = load()
    _u16(x_cal)
    T, K = x_cal.shape
    assert x_cal.is_contiguous() and offsets.dtype == torch.int32 and offsets.is_cuda
    G = int(offsets.numel()) - 1
    sel = torch.empty(G, Kp, dtype=torch.int32, device=x_cal.device)
    err = torch.empty(G, K, dtype=torch.float64, device=x_cal.device) if want_err else None
    ws = _workspace(x_cal.device).get(lib.rac_calibrate_grouped_workspace_size(T, K, G))
    st = status if status is not None else new_status(x_cal.device)
    _check(lib.rac_calibrate_grouped(x_cal.data_ptr(), T, K, offsets.data_ptr(), G, Kp, sel.data_ptr(), _ptr(err),
                                     ws.data_ptr(), ws.numel(), st.data_ptr(), _stream(stream)))
    return sel, err


def moe_row_groups(expert_offsets: torch.Tensor, E: int, rows: int, out: torch.Tensor | None = None, stream=None):
    """Expert of every row of an expert-grouped layout (-1 past the last segment) -> int32 [rows]."""
    lib = load()
    if out is None:
        out = torch.empty(max(rows, 1), dtype=torch.int32, device=expert_offsets.device)
    _check(lib.moe_row_groups(expert_offsets.data_ptr(), E, rows, out.data_ptr(), _stream(stream)))
    return out


def pack_weights(w: torch.Tensor, sel: torch.Tensor | None = None, gate_up_interleave: bool = False,
                 out: Packed | None = None, out_sel: Packed | None = None, status: torch.Tensor | None = None,
                 stream=None):
    """Rollout weight pack: Q(W) and Q(W[:, sel]) with one scale per slab -> (Packed, Packed | None).

    A 2-D ``sel`` [E, Kp] is one channel list per expert (W_sel of expert e = W_e[:, sel[e]])."""
    lib = load()
    _u16(w)
    if w.dim() == 2:
        w = w.unsqueeze(0)
    E, N, K = w.shape
    assert w.is_contiguous()
    grouped = sel is not None and sel.dim() == 2
    if grouped:
        assert sel.shape[0] == E and sel.dtype == torch.int32 and sel.is_contiguous()
    Kp = 0 if sel is None else int(sel.shape[-1])
    if out is None:
        out = Packed.empty(N, K, slabs=E, rows_padded=N, device=w.device)
    if Kp > 0 and out_sel is None:
        out_sel = Packed.empty(N, Kp, slabs=E, rows_padded=N, device=w.device)
    ws = _workspace(w.device).get(lib.pack_weights_workspace_size(E, N, K))
    st = status if status is not None else new_status(w.device)
    q = out.c()
    qs = out_sel.c() if Kp > 0 else None
    fn = lib.pack_weights_grouped_sel if grouped else lib.pack_weights
    _check(fn(w.data_ptr(), E, N, K, _ptr(sel), Kp, int(gate_up_interleave), ctypes.byref(q),
              ctypes.byref(qs) if qs is not None else None, ws.data_ptr(), ws.numel(), st.data_ptr(), _stream(stream)))
    return out, (out_sel if Kp > 0 else None)


def w4a4_rac_gemm(a: Packed, a_res: Packed | None, w: Packed, w_sel: Packed | None, M: int,
                  out_dtype=torch.bfloat16, y: torch.Tensor | None = None, status: torch.Tensor | None = None,
                  stream=None, own_scale: bool = False) -> torch.Tensor:
    """Dense Y = s_a s_w (Q(X)Q(W)^T + Q(R_sel)Q(W_sel)^T) -> y [M, N]."""
    lib = load()
    N, K = w.rows, w.cols
    Kp = 0 if a_res is None else a_res.cols
    if y is None:
        y = torch.empty(M, N, dtype=out_dtype, device=a.codes.device)
    od = OUT_BF16 if y.dtype == torch.bfloat16 else OUT_F32
    st = status if status is not None else new_status(a.codes.device)
    ca, cw = a.c(), w.c()
    car = a_res.c() if Kp > 0 else None
    cws = w_sel.c() if Kp > 0 else None
    _check(lib.w4a4_rac_gemm_ex(ctypes.byref(ca), ctypes.byref(car) if car else None, ctypes.byref(cw),
                                ctypes.byref(cws) if cws else None, M, N, K, Kp, od, y.data_ptr(), y.stride(0),
                                st.data_ptr(), _stream(stream), RAC_OWN_RES_SCALE if own_scale else 0))
    return y


def grouped_w4a4_rac_moe(a: Packed, a_res: Packed | None, expert_offsets: torch.Tensor, w: Packed,
                         w_sel: Packed | None, swiglu: bool = False, out_dtype=torch.bfloat16,
                         y: torch.Tensor | None = None, amax_out: torch.Tensor | None = None,
                         status: torch.Tensor | None = None, stream=None, expert_rows: torch.Tensor | None = None,
                         own_scale: bool = False):
    """Grouped GEMM over expert segments -> y (rows a.rows_padded) [and amax of the SwiGLU output].

    expert_rows (optional device int32 [E]): token rows per segment; 32-row output boxes of padding
    only are then left unwritten."""
    lib = load()
    E = w.slabs
    N, K = w.rows, w.cols
    Kp = 0 if a_res is None else a_res.cols
    ycols = N // 2 if swiglu else N
    if y is None:
        y = torch.empty(a.rows_padded, ycols, dtype=torch.bfloat16 if swiglu else out_dtype, device=a.codes.device)
    if swiglu and amax_out is None:
        amax_out = torch.empty(1, dtype=torch.float32, device=a.codes.device)
    od = OUT_BF16 if y.dtype == torch.bfloat16 else OUT_F32
    st = status if status is not None else new_status(a.codes.device)
    ca, cw = a.c(), w.c()
    car = a_res.c() if Kp > 0 else None
    cws = w_sel.c() if Kp > 0 else None
    _check(lib.grouped_w4a4_rac_moe_ex(ctypes.byref(ca), ctypes.byref(car) if car else None,
                                       expert_offsets.data_ptr(), _ptr(expert_rows), E, ctypes.byref(cw),
                                       ctypes.byref(cws) if cws else None, N, K, Kp,
                                       EPI_SWIGLU_AMAX if swiglu else EPI_NONE, od, y.data_ptr(), y.stride(0),
                                       _ptr(amax_out), st.data_ptr(), _stream(stream),
                                       RAC_OWN_RES_SCALE if own_scale else 0))
    return (y, amax_out) if swiglu else y


def grouped_w4a4_rac_moe_segments(a: Packed, a_res: Packed | None, seg_offsets: torch.Tensor,
                                  seg_rows: torch.Tensor | None, seg_expert: torch.Tensor, w: Packed,
                                  w_sel: Packed | None, swiglu: bool = False, out_dtype=torch.bfloat16,
                                  y: torch.Tensor | None = None, amax_out: torch.Tensor | None = None,
                                  status: torch.Tensor | None = None, stream=None):
    """Grouped GEMM over row segments [seg_offsets[i], seg_offsets[i+1]) with weight slab
    seg_expert[i] (device int32 tensors) -> y [and the amax of the SwiGLU output]."""
    lib = load()
    N, K = w.rows, w.cols
    Kp = 0 if a_res is None else a_res.cols
    n_seg = int(seg_expert.numel())
    assert seg_offsets.dtype == torch.int32 and seg_expert.dtype == torch.int32 and seg_offsets.numel() >= n_seg + 1
    ycols = N // 2 if swiglu else N
    if y is None:
        y = torch.empty(a.rows_padded, ycols, dtype=torch.bfloat16 if swiglu else out_dtype, device=a.codes.device)
    if swiglu and amax_out is None:
        amax_out = torch.empty(1, dtype=torch.float32, device=a.codes.device)
    od = OUT_BF16 if y.dtype == torch.bfloat16 else OUT_F32
    st = status if status is not None else new_status(a.codes.device)
    ca, cw = a.c(), w.c()
    car = a_res.c() if Kp > 0 else None
    cws = w_sel.c() if Kp > 0 else None
    _check(lib.grouped_w4a4_rac_moe_segments(ctypes.byref(ca), ctypes.byref(car) if car else None,
                                             seg_offsets.data_ptr(), _ptr(seg_rows), seg_expert.data_ptr(), n_seg,
                                             ctypes.byref(cw), ctypes.byref(cws) if cws else None, N, K, Kp,
                                             EPI_SWIGLU_AMAX if swiglu else EPI_NONE, od, y.data_ptr(), y.stride(0),
                                             _ptr(amax_out), st.data_ptr(), _stream(stream)))
    return (y, amax_out) if swiglu else y


def nvfp4_amax(x: torch.Tensor, out: torch.Tensor | None = None, status: torch.Tensor | None = None, stream=None):
    """max |x| of a bf16 matrix into a device float32 [1]."""
    lib = load()
    _u16(x)
    M, K = x.shape
    assert x.stride(1) == 1
    out = torch.empty(1, dtype=torch.float32, device=x.device) if out is None else out
    ws = _workspace(x.device).get(lib.nvfp4_quantize_workspace_size(M, K))
    st = status if status is not None else new_status(x.device)
    _check(lib.nvfp4_amax(x.data_ptr(), M, K, x.stride(0), out.data_ptr(), ws.data_ptr(), ws.numel(), st.data_ptr(),
                          _stream(stream)))
    return out


def grouped_w4a4_rac_moe_decode(a: Packed, a_res: Packed | None, slot_expert: torch.Tensor,
                                slot_count: torch.Tensor, w: Packed, w_sel: Packed | None, swiglu: bool = False,
                                out_dtype=torch.bfloat16, y: torch.Tensor | None = None,
                                amax_out: torch.Tensor | None = None, status: torch.Tensor | None = None,
                                stream=None):
    """Swap-AB decode GEMM over 16-token expert slabs -> y [16 * n_slots, N (or N/2)] [and amax of h].

    a / a_res are in the SF_SLAB16 layout; slot_expert / slot_count are device int32 [n_slots]."""
    lib = load()
    E = w.slabs
    N, K = w.rows, w.cols
    Kp = 0 if a_res is None else a_res.cols
    n_slots = int(slot_expert.numel())
    assert slot_expert.dtype == torch.int32 and slot_count.dtype == torch.int32
    ycols = N // 2 if swiglu else N
    if y is None:
        y = torch.empty(16 * n_slots, ycols, dtype=out_dtype, device=a.codes.device)
    if swiglu and amax_out is None:
        amax_out = torch.empty(1, dtype=torch.float32, device=a.codes.device)
    od = OUT_BF16 if y.dtype == torch.bfloat16 else OUT_F32
    st = status if status is not None else new_status(a.codes.device)
    ca, cw = a.c(), w.c()
    car = a_res.c() if Kp > 0 else None
    cws = w_sel.c() if Kp > 0 else None
    _check(lib.grouped_w4a4_rac_moe_decode(ctypes.byref(ca), ctypes.byref(car) if car else None,
                                           slot_expert.data_ptr(), slot_count.data_ptr(), n_slots, E,
                                           ctypes.byref(cw), ctypes.byref(cws) if cws else None, N, K, Kp,
                                           EPI_SWIGLU_AMAX if swiglu else EPI_NONE, od, y.data_ptr(), y.stride(0),
                                           _ptr(amax_out), st.data_ptr(), _stream(stream)))
    return (y, amax_out) if swiglu else y


def moe_route_topk(logits: torch.Tensor, k: int, ids: torch.Tensor | None = None, w: torch.Tensor | None = None,
                   status: torch.Tensor | None = None, stream=None):
    """Router top-k: float32 logits [T, E] -> (ids int32 [T, k], weights float32 [T, k])."""
    lib = load()
    assert logits.is_cuda and logits.dtype == torch.float32 and logits.is_contiguous()
    T, E = logits.shape
    ids = torch.empty(T, k, dtype=torch.int32, device=logits.device) if ids is None else ids
    w = torch.empty(T, k, dtype=torch.float32, device=logits.device) if w is None else w
    st = status if status is not None else new_status(logits.device)
    _check(lib.moe_route_topk(logits.data_ptr(), T, E, k, ids.data_ptr(), w.data_ptr(), st.data_ptr(),
                              _stream(stream)))
    return ids, w


def moe_rows_capacity(T: int, k: int, E: int, pad: int) -> int:
    return int(load().moe_rows_capacity(T, k, E, pad))


def moe_dispatch_plan(ids: torch.Tensor, E: int, pad: int, rows_capacity: int | None = None,
                      n_slots: int | None = None, offsets: torch.Tensor | None = None,
                      row_scatter: torch.Tensor | None = None, slot_expert: torch.Tensor | None = None,
                      slot_count: torch.Tensor | None = None, status: torch.Tensor | None = None, stream=None,
                      expert_rows: torch.Tensor | None = None):
    """Expert-grouped layout of the pairs of ids [T, k] -> (offsets [E+1], row_scatter [T, k], slot_expert,
    slot_count); the slot tables (pad 16) only when n_slots is given."""
    lib = load()
    assert ids.dtype == torch.int32 and ids.is_contiguous()
    T, k = ids.shape
    dev = ids.device
    cap = moe_rows_capacity(T, k, E, pad) if rows_capacity is None else rows_capacity
    offsets = torch.empty(E + 1, dtype=torch.int32, device=dev) if offsets is None else offsets
    row_scatter = torch.empty(T, k, dtype=torch.int32, device=dev) if row_scatter is None else row_scatter
    if n_slots is not None:
        slot_expert = torch.empty(n_slots, dtype=torch.int32, device=dev) if slot_expert is None else slot_expert
        slot_count = torch.empty(n_slots, dtype=torch.int32, device=dev) if slot_count is None else slot_count
    ws = _workspace(dev).get(lib.moe_dispatch_workspace_size(E))
    st = status if status is not None else new_status(dev)
    _check(lib.moe_dispatch_plan(ids.data_ptr(), T, k, E, pad, cap, offsets.data_ptr(), row_scatter.data_ptr(),
                                 _ptr(expert_rows), _ptr(slot_expert), _ptr(slot_count), 0 if n_slots is None else n_slots,
                                 ws.data_ptr(), ws.numel(), st.data_ptr(), _stream(stream)))
    return offsets, row_scatter, slot_expert, slot_count


def moe_combine(y: torch.Tensor, row_scatter: torch.Tensor, w: torch.Tensor, out: torch.Tensor | None = None,
                status: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """out[t] = sum_j w[t, j] * y[row_scatter[t, j]] -> bf16 [T, H]."""
    lib = load()
    _u16(y)
    T, k = row_scatter.shape
    H = y.shape[1]
    out = torch.empty(T, H, dtype=torch.bfloat16, device=y.device) if out is None else out
    st = status if status is not None else new_status(y.device)
    _check(lib.moe_combine(y.data_ptr(), y.stride(0), y.shape[0], row_scatter.data_ptr(), w.data_ptr(), T, k, H,
                           out.data_ptr(), out.stride(0), st.data_ptr(), _stream(stream)))
    return out


def moe_row_pairs(row_scatter: torch.Tensor, rows: int, row_pair: torch.Tensor | None = None,
                  status: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """row_pair[r] = t * k + j for row_scatter[t, j] = r, -1 elsewhere (device int32 [rows])."""
    lib = load()
    T, k = row_scatter.shape
    assert row_scatter.dtype == torch.int32 and row_scatter.is_contiguous()
    if row_pair is None:
        row_pair = torch.empty(rows, dtype=torch.int32, device=row_scatter.device)
    st = status if status is not None else new_status(row_scatter.device)
    _check(lib.moe_row_pairs(row_scatter.data_ptr(), T, k, rows, row_pair.data_ptr(), st.data_ptr(),
                             _stream(stream)))
    return row_pair


def grouped_w4a4_rac_moe_combine(a: Packed, a_res: Packed | None, expert_offsets: torch.Tensor, w: Packed,
                                 w_sel: Packed | None, row_pair: torch.Tensor, topk_w: torch.Tensor,
                                 out: torch.Tensor | None = None, out32: torch.Tensor | None = None,
                                 status: torch.Tensor | None = None, stream=None,
                                 expert_rows: torch.Tensor | None = None) -> torch.Tensor:
    """Down projection with the weighted combine in the GEMM epilogue -> bf16 [T, N]."""
    lib = load()
    E = w.slabs
    N, K = w.rows, w.cols
    Kp = 0 if a_res is None else a_res.cols
    T, k = topk_w.shape
    dev = a.codes.device
    assert topk_w.dtype == torch.float32 and topk_w.is_contiguous() and row_pair.dtype == torch.int32
    if out is None:
        out = torch.empty(T, N, dtype=torch.bfloat16, device=dev)
    if out32 is None:
        out32 = torch.empty(T, N, dtype=torch.float32, device=dev)
    st = status if status is not None else new_status(dev)
    ca, cw = a.c(), w.c()
    car = a_res.c() if Kp > 0 else None
    cws = w_sel.c() if Kp > 0 else None
    _check(lib.grouped_w4a4_rac_moe_combine(ctypes.byref(ca), ctypes.byref(car) if car else None,
                                            expert_offsets.data_ptr(), _ptr(expert_rows), E, ctypes.byref(cw),
                                            ctypes.byref(cws) if cws else None, N, K, Kp, row_pair.data_ptr(),
                                            topk_w.data_ptr(), T, k, out32.data_ptr(), out.data_ptr(), out.stride(0),
                                            st.data_ptr(), _stream(stream)))
    return out


def weight_qdq(w: torch.Tensor, out: torch.Tensor | None = None, s_g: torch.Tensor | None = None,
               status: torch.Tensor | None = None, stream=None):
    """Trainer fake-quant bf16(DQ(Q(w))) per tensor; w is [n_tensors, elems] (or one tensor of any shape)."""
    lib = load()
    _u16(w)
    assert w.is_contiguous()
    n = w.shape[0] if w.dim() >= 2 else 1
    elems = w.numel() // n
    if out is None:
        out = torch.empty_like(w)
    if s_g is None:
        s_g = torch.empty(n, dtype=torch.float32, device=w.device)
    ws = _workspace(w.device).get(lib.weight_qdq_workspace_size(n, elems))
    st = status if status is not None else new_status(w.device)
    _check(lib.weight_qdq(w.data_ptr(), n, elems, out.data_ptr(), s_g.data_ptr(), ws.data_ptr(), ws.numel(),
                          st.data_ptr(), _stream(stream)))
    return out, s_g


def weight_qdq_backward(grad_fq: torch.Tensor, grad_w: torch.Tensor | None = None,
                        grad_acc: torch.Tensor | None = None, stream=None):
    """Straight-through gradient of the fake-quant: grad_w = grad_fq (bf16) and/or
    grad_acc += grad_fq (float32 master gradient)."""
    lib = load()
    _u16(grad_fq)
    assert grad_fq.is_contiguous()
    if grad_w is None and grad_acc is None:
        grad_w = torch.empty_like(grad_fq)
    if grad_acc is not None:
        assert grad_acc.dtype == torch.float32 and grad_acc.is_contiguous() and grad_acc.numel() == grad_fq.numel()
    _check(lib.weight_qdq_backward(grad_fq.data_ptr(), grad_fq.numel(), _ptr(grad_w), _ptr(grad_acc),
                                   _stream(stream)))
    return grad_w if grad_w is not None else grad_acc


class FakeQuantSTE(torch.autograd.Function):
    """W -> bf16(DQ(Q(W))) per tensor in the forward pass (weight_qdq), the straight-through
    gradient in the backward pass (weight_qdq_backward): the trainer side of the shared
    quantise-dequantise path."""

    @staticmethod
    def forward(ctx, w):
        out, _ = weight_qdq(w.contiguous())
        return out

    @staticmethod
    def backward(ctx, g):
        return weight_qdq_backward(g.contiguous())


def unpack_logical(p: Packed, slab: int = 0, stream=None):
    """Codes (uint8 [rows, cols], one per byte) and block scales (uint8 [rows, cols/16]) of one
    slab of a packed tensor, in logical order, made by the library's unpack kernel."""
    lib = load()
    codes = torch.empty(p.rows, p.cols, dtype=torch.uint8, device=p.codes.device)
    sf = torch.empty(p.rows, p.cols // 16, dtype=torch.uint8, device=p.codes.device)
    c = p.c()
    _check(lib.nvfp4_unpack_logical(ctypes.byref(c), slab, codes.data_ptr(), sf.data_ptr(), _stream(stream)))
    return codes, sf


def encode_e2m1(v: torch.Tensor, stream=None) -> torch.Tensor:
    out = torch.empty(v.numel(), dtype=torch.uint8, device=v.device)
    _check(load().nvfp4_encode_e2m1(v.data_ptr(), v.numel(), out.data_ptr(), _stream(stream)))
    return out


def encode_e4m3(v: torch.Tensor, stream=None) -> torch.Tensor:
    out = torch.empty(v.numel(), dtype=torch.uint8, device=v.device)
    _check(load().nvfp4_encode_e4m3(v.data_ptr(), v.numel(), out.data_ptr(), _stream(stream)))
    return out


def selftest_wait_timeout(limit_ns: int, status: torch.Tensor, stream=None):
    _check(load().nvfp4_selftest_wait_timeout(limit_ns, status.data_ptr(), _stream(stream)))
