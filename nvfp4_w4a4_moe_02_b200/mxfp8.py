"""Binding of the FP8 comparison path of the C ABI (``mxfp8_*`` and ``grouped_mxfp8_moe`` in
``include/nvfp4rac.h``): E4M3 codes with one power-of-two scale per 32 elements, the format the
NVFP4 + RAC path is timed against.  Argument marshalling only; every step runs in the library's
kernels."""
from __future__ import annotations

import ctypes
from dataclasses import dataclass

import torch

from . import nvfp4rac as R


class CMx8Tensor(ctypes.Structure):
    _fields_ = [("codes", ctypes.c_void_p), ("sf", ctypes.c_void_p), ("slabs", ctypes.c_int64),
                ("rows", ctypes.c_int64), ("rows_padded", ctypes.c_int64), ("cols", ctypes.c_int64)]


_SIGS_DONE = False


def load() -> ctypes.CDLL:
    global _SIGS_DONE
    lib = R.load()
    if not _SIGS_DONE:
        vp, i64, i32, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_size_t
        tp = ctypes.POINTER(CMx8Tensor)
        sigs = {
            "mxfp8_codes_bytes": ([i64, i64], sz),
            "mxfp8_sf_bytes": ([i64, i64], sz),
            "mxfp8_quantize": ([vp, i64, i64, i64, vp, i64, tp, vp, vp], ctypes.c_int),
            "mxfp8_quantize_scatter": ([vp, i64, i64, i64, vp, i32, tp, vp, vp], ctypes.c_int),
            "mxfp8_pack_weights": ([vp, i64, i64, i64, i32, tp, vp, vp], ctypes.c_int),
            "mxfp8_gemm": ([tp, tp, i64, i64, i64, ctypes.c_int, vp, i64, vp, vp], ctypes.c_int),
            "grouped_mxfp8_moe": ([tp, vp, vp, i32, tp, i64, i64, ctypes.c_int, ctypes.c_int, vp, i64, vp, vp, vp],
                                  ctypes.c_int),
        }
        for name, (args, res) in sigs.items():
            fn = getattr(lib, name)
            fn.argtypes = args
            fn.restype = res
        _SIGS_DONE = True
    return lib


@dataclass
class Mx8Packed:
    """Caller-side owner of one FP8 tensor: codes uint8 [slabs * rows_padded * cols], scale atoms
    uint8 [slabs * rows_padded * cols / 32]."""
    codes: torch.Tensor
    sf: torch.Tensor
    slabs: int
    rows: int
    rows_padded: int
    cols: int

    @staticmethod
    def empty(rows: int, cols: int, slabs: int = 1, rows_padded: int | None = None, device="cuda",
              zero: bool = False) -> "Mx8Packed":
        rp = R.round_up(max(rows, 1), 128) if rows_padded is None else rows_padded
        alloc = torch.zeros if zero else torch.empty
        return Mx8Packed(alloc(slabs * rp * cols, dtype=torch.uint8, device=device),
                         alloc(slabs * rp * cols // 32, dtype=torch.uint8, device=device), slabs, rows, rp, cols)

    def c(self) -> CMx8Tensor:
        return CMx8Tensor(self.codes.data_ptr(), self.sf.data_ptr(), self.slabs, self.rows, self.rows_padded,
                          self.cols)


def quantize(x: torch.Tensor, row_gather: torch.Tensor | None = None, M_out: int | None = None,
             rows_padded: int | None = None, out: Mx8Packed | None = None, status: torch.Tensor | None = None,
             stream=None) -> Mx8Packed:
    lib = load()
    M, K = x.shape
    assert x.stride(1) == 1 and x.dtype in (torch.bfloat16, torch.int16)
    if M_out is None:
        M_out = M if row_gather is None else int(row_gather.numel())
    if out is None:
        out = Mx8Packed.empty(M_out, K, rows_padded=rows_padded, device=x.device)
    st = status if status is not None else R.new_status(x.device)
    q = out.c()
    R._check(lib.mxfp8_quantize(x.data_ptr(), M, K, x.stride(0), R._ptr(row_gather), M_out, ctypes.byref(q),
                                st.data_ptr(), R._stream(stream)))
    return out


def quantize_scatter(x: torch.Tensor, row_scatter: torch.Tensor, rows_padded: int, out: Mx8Packed | None = None,
                     status: torch.Tensor | None = None, stream=None) -> Mx8Packed:
    """Each x row quantised once and written to rows row_scatter[m, :] (-1 = unused); rows no
    entry names keep their contents, so freshly created outputs are zero-filled."""
    lib = load()
    M, K = x.shape
    assert x.stride(1) == 1 and row_scatter.dtype == torch.int32 and row_scatter.is_contiguous()
    if out is None:
        out = Mx8Packed.empty(rows_padded, K, rows_padded=rows_padded, device=x.device, zero=True)
    st = status if status is not None else R.new_status(x.device)
    q = out.c()
    R._check(lib.mxfp8_quantize_scatter(x.data_ptr(), M, K, x.stride(0), row_scatter.data_ptr(), row_scatter.shape[1],
                                        ctypes.byref(q), st.data_ptr(), R._stream(stream)))
    return out


def pack_weights(w: torch.Tensor, gate_up_interleave: bool = False, out: Mx8Packed | None = None,
                 status: torch.Tensor | None = None, stream=None) -> Mx8Packed:
    lib = load()
    if w.dim() == 2:
        w = w.unsqueeze(0)
    E, N, K = w.shape
    assert w.is_contiguous()
    if out is None:
        out = Mx8Packed.empty(N, K, slabs=E, rows_padded=N, device=w.device)
    st = status if status is not None else R.new_status(w.device)
    q = out.c()
    R._check(lib.mxfp8_pack_weights(w.data_ptr(), E, N, K, int(gate_up_interleave), ctypes.byref(q), st.data_ptr(),
                                    R._stream(stream)))
    return out


def gemm(a: Mx8Packed, w: Mx8Packed, M: int, out_dtype=torch.bfloat16, y: torch.Tensor | None = None,
         status: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    lib = load()
    N, K = w.rows, w.cols
    if y is None:
        y = torch.empty(M, N, dtype=out_dtype, device=a.codes.device)
    st = status if status is not None else R.new_status(a.codes.device)
    ca, cw = a.c(), w.c()
    od = R.OUT_BF16 if y.dtype == torch.bfloat16 else R.OUT_F32
    R._check(lib.mxfp8_gemm(ctypes.byref(ca), ctypes.byref(cw), M, N, K, od, y.data_ptr(), y.stride(0),
                            st.data_ptr(), R._stream(stream)))
    return y


def grouped_moe(a: Mx8Packed, expert_offsets: torch.Tensor, w: Mx8Packed, swiglu: bool = False,
                out_dtype=torch.bfloat16, y: torch.Tensor | None = None, amax_out: torch.Tensor | None = None,
                status: torch.Tensor | None = None, stream=None, expert_rows: torch.Tensor | None = None):
    """Grouped FP8 GEMM over expert segments -> y (rows a.rows_padded; SwiGLU halves the columns)."""
    lib = load()
    E, N, K = w.slabs, w.rows, w.cols
    if y is None:
        y = torch.empty(a.rows_padded, N // 2 if swiglu else N, dtype=torch.bfloat16 if swiglu else out_dtype,
                        device=a.codes.device)
    st = status if status is not None else R.new_status(a.codes.device)
    ca, cw = a.c(), w.c()
    od = R.OUT_BF16 if y.dtype == torch.bfloat16 else R.OUT_F32
    R._check(lib.grouped_mxfp8_moe(ctypes.byref(ca), expert_offsets.data_ptr(), R._ptr(expert_rows), E,
                                   ctypes.byref(cw), N, K, R.EPI_SWIGLU_AMAX if swiglu else R.EPI_NONE, od, y.data_ptr(),
                                   y.stride(0), R._ptr(amax_out), st.data_ptr(), R._stream(stream)))
    return y
