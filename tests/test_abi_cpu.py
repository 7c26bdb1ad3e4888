"""CPU checks of the boundary: the C library loads, exports every declared entry point, and
rejects bad arguments on the host before touching a device.  Also pins the test-side layout
decoder against the storage definition written in the header."""
import ctypes
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "nvfp4rac.h")


@pytest.fixture(scope="module")
def lib():
    from nvfp4_w4a4_moe_02_b200 import build_lib, nvfp4rac

    build_lib.build()
    return nvfp4rac.load()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\*?\s+([A-Za-z_][A-Za-z0-9_]*)\s*\(", text, re.M)
    return sorted(set(n for n in names if n not in ("if", "return")))


def test_header_declares_the_hot_path_calls():
    names = declared_functions()
    for n in ("nvfp4_quantize", "rac_calibrate", "pack_weights", "w4a4_rac_gemm", "grouped_w4a4_rac_moe",
              "weight_qdq"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing


def test_status_strings_and_sizes(lib):
    assert lib.nvfp4_version() >= 100
    assert lib.nvfp4_status_string(0) == b"ok"
    assert lib.nvfp4_status_string(6) == b"device wait timed out"
    assert lib.nvfp4_codes_bytes(128, 256) == 128 * 128
    assert lib.nvfp4_sf_bytes(128, 256) == 128 * 16
    assert lib.nvfp4_kp_from_ratio(4096, 0.5) == 2048
    assert lib.nvfp4_kp_from_ratio(768, 0.5) == 384
    assert lib.nvfp4_kp_from_ratio(768, 0.25) == 192
    assert lib.nvfp4_kp_from_ratio(256, 0.0) == 0
    assert lib.nvfp4_kp_from_ratio(256, 1.0) == 256


def test_host_side_rejections(lib):
    from nvfp4_w4a4_moe_02_b200.nvfp4rac import CTensor

    t = CTensor(16, 16, 16, 1, 64, 128, 100)  # fake non-null pointers, never dereferenced
    # K not a multiple of 64
    st = lib.nvfp4_quantize(16, 64, 100, 104, None, 64, None, 0, None, ctypes.byref(t), None, 16, 1024, None, None)
    assert st == 2 and b"K" in lib.nvfp4_last_error_string()
    # misaligned x
    t.cols = 128
    st = lib.nvfp4_quantize(18, 64, 128, 128, None, 64, None, 0, None, ctypes.byref(t), None, 16, 1024, None, None)
    assert st == 3
    # Kp not a multiple of 64
    st = lib.nvfp4_quantize(16, 64, 128, 128, None, 64, 16, 32, None, ctypes.byref(t), ctypes.byref(t), 16, 1024,
                            None, None)
    assert st == 2
    # rows_padded not a multiple of 128
    t2 = CTensor(16, 16, 16, 1, 64, 100, 128)
    st = lib.nvfp4_quantize(16, 64, 128, 128, None, 64, None, 0, None, ctypes.byref(t2), None, 16, 1024, None, None)
    assert st == 2
    # GEMM: N not a multiple of 128
    a = CTensor(16, 16, 16, 1, 64, 128, 128)
    w = CTensor(16, 16, 16, 1, 96, 96, 128)
    st = lib.w4a4_rac_gemm(ctypes.byref(a), None, ctypes.byref(w), None, 64, 96, 128, 0, 0, 16, 96, None, None)
    assert st == 2
    # grouped: SwiGLU needs bf16 output
    st = lib.grouped_w4a4_rac_moe(ctypes.byref(a), None, 16, None, 1, ctypes.byref(w), None, 128, 128, 0, 1, 0, 16,
                                  64, 16, None, None)
    assert st == 1
    # weight_qdq: elems not a multiple of 16
    st = lib.weight_qdq(16, 1, 100, 16, None, 16, 1 << 20, None, None)
    assert st == 2
    # calibration: Kp > K
    st = lib.rac_calibrate(16, 64, 128, 256, 16, None, 16, 1 << 30, None, None)
    assert st == 2
    # null status pointer is rejected by the self-test entry
    assert lib.nvfp4_selftest_wait_timeout(1000, None, None) == 1
    # dispatch plan: k above 128 (the rank kernel keeps a pair's slot in seven bits)
    ws = lib.moe_dispatch_workspace_size(8)
    st = lib.moe_dispatch_plan(16, 4, 129, 8, 128, 4096, 16, 16, None, None, None, 0, 16, ws, None, None)
    assert st == 2 and b"128" in lib.nvfp4_last_error_string()


def test_noalloc_host_side_rejections(lib):
    """weight_qdq_noalloc checks its arguments and its scratch limit on the host, before any CUDA
    call, and a good call after a rejected one leaves no stale error text."""
    fn = lib.weight_qdq_noalloc
    vp, i64 = ctypes.c_void_p, ctypes.c_int64
    fn.argtypes = [vp, i64, i64, vp, vp, vp, vp]
    fn.restype = ctypes.c_int
    # NULL input or output
    assert fn(None, 1, 16, 16, None, None, None) == 1
    assert fn(16, 1, 16, None, None, None, None) == 1
    # elements per tensor not a multiple of 16, no tensors
    assert fn(16, 1, 24, 16, None, None, None) == 2
    assert fn(16, 0, 16, 16, None, None, None) == 2
    # misaligned input
    assert fn(18, 1, 16, 16, None, None, None) == 3
    # the fixed scratch holds one amax partial per tensor from 512 tensors on: 4097 is too many
    assert fn(16, 4097, 16, 16, None, None, None) == 2
    assert b"4096" in lib.nvfp4_last_error_string()
    # a later call does not keep that text: without a GPU it stops at the device lookup and
    # reports that instead
    assert fn(16, 4096, 16, 16, None, None, None) == 5
    assert b"4096" not in lib.nvfp4_last_error_string()


def test_decode_and_layout_rejections(lib):
    from nvfp4_w4a4_moe_02_b200.nvfp4rac import SF_SLAB16, CTensor

    assert lib.nvfp4_sf_bytes_layout(128, 256, 0) == 128 * 16
    assert lib.nvfp4_sf_bytes_layout(48, 256, SF_SLAB16) == 3 * 4 * 512
    w = CTensor(16, 16, 16, 4, 256, 256, 128)
    a16 = CTensor(16, 16, 16, 1, 32, 32, 128, SF_SLAB16)
    a128 = CTensor(16, 16, 16, 1, 128, 128, 128)
    args = lambda a, n_slots=2, N=256, ep=0: (ctypes.byref(a), None, 16, 16, n_slots, 4, ctypes.byref(w), None, N, 128,
                                              0, ep, 0, 16, N, None, None, None)
    # the decode GEMM takes slab-layout activations only
    assert lib.grouped_w4a4_rac_moe_decode(*args(a128)) == 2
    assert b"sf_layout" in lib.nvfp4_last_error_string()
    # more slots than rows
    assert lib.grouped_w4a4_rac_moe_decode(*args(a16, n_slots=3)) == 2
    # N not a multiple of 128
    assert lib.grouped_w4a4_rac_moe_decode(*args(a16, N=192)) == 2
    # SwiGLU without amax_out
    assert lib.grouped_w4a4_rac_moe_decode(*args(a16, ep=1)) == 1
    # missing slot tables
    st = lib.grouped_w4a4_rac_moe_decode(ctypes.byref(a16), None, None, 16, 2, 4, ctypes.byref(w), None, 256, 128, 0,
                                         0, 0, 16, 256, None, None, None)
    assert st == 1
    # an unknown layout value, and prefill GEMMs refuse slab-layout operands
    bad = CTensor(16, 16, 16, 1, 32, 32, 128, 7)
    st = lib.nvfp4_quantize(16, 32, 128, 128, None, 32, None, 0, None, ctypes.byref(bad), None, 16, 1024, None, None)
    assert st == 1
    w1 = CTensor(16, 16, 16, 1, 256, 256, 128)
    st = lib.w4a4_rac_gemm(ctypes.byref(a16), None, ctypes.byref(w1), None, 32, 256, 128, 0, 0, 16, 256, None, None)
    assert st == 2
    # q and q_res must share the layout
    r128 = CTensor(16, 16, 16, 1, 32, 128, 64)
    st = lib.nvfp4_quantize(16, 32, 128, 128, None, 32, 16, 64, None, ctypes.byref(a16), ctypes.byref(r128), 16, 1024,
                            None, None)
    assert st == 2


def test_grouped_sel_rejections(lib):
    """Per-expert channel lists: argument checks on the host, before any device work."""
    from nvfp4_w4a4_moe_02_b200.nvfp4rac import CTensor

    q = CTensor(16, 16, 16, 1, 64, 128, 128)
    qr = CTensor(16, 16, 16, 1, 64, 128, 64)
    qm = CTensor(16, 16, 16, 1, 64, 128, 128)  # K wide: the masked variant's residual

    def quant(row_group=16, groups=2, sel=16, res=qr):
        return lib.nvfp4_quantize_grouped_sel(16, 64, 128, 128, None, 64, row_group, groups, sel, 64, None,
                                              ctypes.byref(q), ctypes.byref(res), 16, 1024, None, None)

    assert quant(groups=0) == 2
    assert quant(sel=None) == 1
    assert quant(res=qm) == 2 and b"compact" in lib.nvfp4_last_error_string()
    assert quant(row_group=None) == 1
    assert quant(sel=24) == 3
    # calibration: offsets required, group count in range
    assert lib.rac_calibrate_grouped(16, 64, 128, None, 2, 64, 16, None, 16, 1 << 30, None, None) == 1
    assert lib.rac_calibrate_grouped(16, 64, 128, 16, 0, 64, 16, None, 16, 1 << 30, None, None) == 2
    assert lib.rac_calibrate_grouped_workspace_size(64, 128, 3) > lib.rac_calibrate_workspace_size(64, 128)
    # pack: per-expert lists must be 16-byte aligned
    w_q = CTensor(16, 16, 16, 2, 128, 128, 128)
    w_s = CTensor(16, 16, 16, 2, 128, 128, 64)
    st = lib.pack_weights_grouped_sel(16, 2, 128, 128, 24, 64, 0, ctypes.byref(w_q), ctypes.byref(w_s), 16, 1 << 20,
                                      None, None)
    assert st == 3
    # row groups: nothing to do for zero rows; E must be positive; buffers must be given
    assert lib.moe_row_groups(None, 4, 0, None, None) == 0
    assert lib.moe_row_groups(16, 0, 8, 16, None) == 2
    assert lib.moe_row_groups(None, 4, 8, 16, None) == 1


def test_fp8_path_rejections(lib):
    """The FP8 comparison entry points check shapes on the host, before any device work."""
    from nvfp4_w4a4_moe_02_b200.mxfp8 import CMx8Tensor, load

    load()
    assert lib.mxfp8_codes_bytes(128, 256) == 128 * 256 and lib.mxfp8_sf_bytes(128, 256) == 128 * 8
    q = CMx8Tensor(16, 16, 1, 64, 128, 192)
    # K must be a multiple of 128
    assert lib.mxfp8_quantize(16, 64, 192, 192, None, 64, ctypes.byref(q), None, None) == 2
    q.cols = 256
    assert lib.mxfp8_quantize(16, 64, 256, 256, None, 32, ctypes.byref(q), None, None) == 2  # M_out != M
    assert lib.mxfp8_quantize_scatter(16, 64, 256, 256, 16, 33, ctypes.byref(q), None, None) == 2  # fanout > 32
    assert lib.mxfp8_quantize(24, 64, 256, 256, None, 64, ctypes.byref(q), None, None) == 3  # misaligned x
    w = CMx8Tensor(16, 16, 2, 96, 96, 256)
    assert lib.mxfp8_pack_weights(16, 2, 96, 256, 0, ctypes.byref(w), None, None) == 2  # N % 128
    a = CMx8Tensor(16, 16, 1, 128, 128, 256)
    w1 = CMx8Tensor(16, 16, 1, 128, 128, 256)
    # SwiGLU writes bf16 only; N % 128
    assert lib.grouped_mxfp8_moe(ctypes.byref(a), 16, None, 1, ctypes.byref(w1), 128, 256, 1, 0, 16, 64, None, None,
                                 None) == 1
    assert lib.mxfp8_gemm(ctypes.byref(a), ctypes.byref(w1), 128, 96, 256, 0, 16, 96, None, None) == 2


def test_decode_slots_host_logic():
    from nvfp4_layout import decode_slots

    counts = [0, 3, 16, 17, 0, 1, 40]
    se, sc, rows = decode_slots(counts)
    assert se.tolist() == [1, 2, 3, 3, 5, 6, 6, 6]
    assert sc.tolist() == [3, 16, 16, 1, 1, 16, 16, 8]
    assert rows.size == sum(counts) and len(set(rows.tolist())) == rows.size
    # pairs of expert e land in its own slabs, in order
    start = 0
    for e, c in enumerate(counts):
        r = rows[start:start + c]
        assert all(se[x // 16] == e for x in r)
        assert all(x % 16 < sc[x // 16] for x in r)
        start += c
    assert decode_slots([0, 0])[0].size == 0


def test_layout_decoder_matches_storage_definition():
    from nvfp4_layout import pack_codes, pack_sf, unpack_codes, unpack_sf

    rng = np.random.default_rng(0)
    rows_p, cols = 256, 192
    S = rng.integers(0, 0x7F, (rows_p, cols // 16), dtype=np.uint8)
    flat = pack_sf(S, rows_p)
    # spot values written straight from the header formula
    for r, c in [(0, 0), (1, 0), (31, 3), (32, 0), (127, 11), (128, 5), (255, 11), (77, 6)]:
        atom = (r // 128) * (cols // 64) + c // 4
        off = atom * 512 + (r % 128 % 32) * 16 + (r % 128 // 32) * 4 + c % 4
        assert flat[off] == S[r, c]
    assert np.array_equal(unpack_sf(flat, rows_p, rows_p, cols), S)
    # 16-row slab layout: slab r // 16 owns atom (r // 16, c // 4); row r at byte (r % 16)*16 + c % 4
    from nvfp4_layout import sf_index_slab16

    idx = sf_index_slab16(48, cols)
    for r, c in [(0, 0), (15, 3), (16, 0), (17, 5), (47, 11)]:
        assert idx[r, c] == ((r // 16) * (cols // 64) + c // 4) * 512 + (r % 16) * 16 + c % 4
    assert len(set(idx.reshape(-1).tolist())) == idx.size
    assert np.array_equal(unpack_sf(np.arange(3 * 3 * 512) % 251, 48, 48, cols, slab16=True),
                          (np.arange(3 * 3 * 512) % 251)[idx])
    C = rng.integers(0, 16, (rows_p, cols), dtype=np.uint8)
    b = pack_codes(C)
    assert b[0] == C[0, 0] | (C[0, 1] << 4)
    assert np.array_equal(unpack_codes(b, rows_p, rows_p, cols), C)
