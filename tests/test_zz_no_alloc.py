"""GPU test of weight_qdq_noalloc, the allocation-free trainer fake-quant entry point.

It serves callers that cannot call cudaMalloc (a framework that owns device memory through
its own allocator, a latency-bound loop that cannot take cudaMalloc's implicit
synchronisation, a plain C host program with no allocator).  The test calls it through the C
ABI and compares it with weight_qdq (the workspace-taking entry point) on two calls in a row,
bit for bit, as the parity tests of weight_qdq do; it also checks the size limit.  The file is
named so that pytest collects it last.
"""
import ctypes

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


def _noalloc_fn(lib):
    fn = lib.weight_qdq_noalloc
    vp, i64 = ctypes.c_void_p, ctypes.c_int64
    fn.argtypes = [vp, i64, i64, vp, vp, vp, vp]
    fn.restype = ctypes.c_int
    return fn


def test_weight_qdq_noalloc_matches_weight_qdq():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from nvfp4_w4a4_moe_02_b200 import nvfp4rac as R
    from nvfp4_w4a4_moe_02_b200 import synthetic as syn

    lib = R.load()
    fn = _noalloc_fn(lib)
    dev = torch.device("cuda:0")
    stream = torch.cuda.current_stream().cuda_stream
    # two calls in a row, the second with fewer tensors and different data, so that scales
    # left in the shared scratch by the first call cannot stand in for the second's
    for call, (n, elems, seed) in enumerate([(6, 4096 + 48, 1), (3, 2048, 2)]):
        w_np = syn.normal_bf16(seed, 9, n, elems, 0.02)
        w_np[call, :64] = syn.normal_bf16(seed, 10, 1, 64, 0.64)[0]  # a few larger weights in one tensor
        w = torch.from_numpy(w_np.view(np.int16)).to(dev).view(torch.bfloat16)
        ref, s_ref = R.weight_qdq(w)
        out = torch.empty_like(w)
        s_g = torch.empty(n, dtype=torch.float32, device=dev)
        st = R.new_status(dev)
        rc = fn(w.data_ptr(), n, elems, out.data_ptr(), s_g.data_ptr(), st.data_ptr(), stream)
        assert rc == 0, lib.nvfp4_last_error_string()
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        assert torch.equal(out.view(torch.int16), ref.view(torch.int16)), f"call {call}: outputs differ"
        assert torch.equal(s_g, s_ref), f"call {call}: scales differ"


def test_weight_qdq_noalloc_rejects_oversize():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from nvfp4_w4a4_moe_02_b200 import nvfp4rac as R
    from nvfp4_w4a4_moe_02_b200 import synthetic as syn

    lib = R.load()
    fn = _noalloc_fn(lib)
    dev = torch.device("cuda:0")
    w = torch.zeros(4097, 16, dtype=torch.bfloat16, device=dev)
    out = torch.empty_like(w)
    stream = torch.cuda.current_stream().cuda_stream
    rc = fn(w.data_ptr(), 4097, 16, out.data_ptr(), None, None, stream)
    assert rc == 2
    assert b"4096" in lib.nvfp4_last_error_string()
    # the largest accepted call (4096 tensors) right after the rejected one: it succeeds, leaves
    # no stale error text, and matches weight_qdq
    w = torch.from_numpy(syn.normal_bf16(3, 9, 4096, 16, 0.02).view(np.int16)).to(dev).view(torch.bfloat16)
    ref, s_ref = R.weight_qdq(w)
    out = torch.empty_like(w)
    s_g = torch.empty(4096, dtype=torch.float32, device=dev)
    st = R.new_status(dev)
    rc = fn(w.data_ptr(), 4096, 16, out.data_ptr(), s_g.data_ptr(), st.data_ptr(), stream)
    assert rc == 0 and lib.nvfp4_last_error_string() == b""
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert torch.equal(out.view(torch.int16), ref.view(torch.int16)) and torch.equal(s_g, s_ref)
