"""The bench's whole-layer step (router, plan, quantise, GEMMs, combine) on small MoE blocks, run
the way bench.py runs it: prefill with the combine kernel and with the combine in the down GEMM's
epilogue (the two must agree within the combine's summation-order bound), and decode."""
import numpy as np
import pytest
import torch

import bench
from nvfp4_w4a4_moe_02_b200 import nvfp4rac as R
from nvfp4_w4a4_moe_02_b200 import synthetic as syn

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    R.load()
    return torch.device("cuda:0")


def bf16_f64(t):
    return t.float().double().cpu().numpy()


def test_prefill_layer_step_with_and_without_fused_combine(dev):
    wl = syn.moe_block(0, 0.5, T=256, H=512, E=8, topk=2, I=256, T_cal=128)
    inner = bench.MoEStep(wl, syn.moe_down_calibration_batch(wl), dev)
    packed = (inner.pgu, inner.pgus, inner.pdn, inner.pdns)
    plain = bench.MoEBlockStep(wl, packed, inner.sel_gu, inner.sel_dn, False, dev)
    fused = bench.MoEBlockStep(wl, packed, inner.sel_gu, inner.sel_dn, False, dev, fused_combine=True)
    assert fused.fused_combine and not plain.fused_combine
    y0 = plain.run().clone()
    y1 = fused.run().clone()
    torch.cuda.synchronize()
    R.check_status(plain.status)
    R.check_status(fused.status)
    # bound: both sums are within k 2^-23 sum_j |w_j y_j| of the exact one before the bf16 rounding
    rows, w = plain.rows.cpu().numpy(), plain.w.cpu().numpy()
    ye = np.abs(bf16_f64(plain.ye))
    absdot = np.einsum("tk,tkh->th", np.abs(w).astype(np.float64), ye[rows])
    a, b = bf16_f64(y0), bf16_f64(y1)
    ulp = np.exp2(np.floor(np.log2(np.maximum(np.maximum(np.abs(a), np.abs(b)), 1e-30))) - 7)
    k = rows.shape[1]
    assert np.all(np.abs(a - b) <= 2 * k * 2.0 ** -23 * absdot + 2 * ulp)
    assert np.isfinite(a).all() and np.abs(a).max() > 0


def test_step_replayed_from_a_cuda_graph_gives_the_same_outputs(dev):
    """The bench times the step's C-ABI calls replayed from one CUDA graph: the replay computes the
    same rows as the calls themselves, bit for bit (prefill block and whole layer)."""
    wl = syn.moe_block(0, 0.5, T=256, H=512, E=8, topk=2, I=256, T_cal=128)
    step = bench.MoEStep(wl, syn.moe_down_calibration_batch(wl), dev)
    layer = bench.MoEBlockStep(wl, (step.pgu, step.pgus, step.pdn, step.pdns), step.sel_gu, step.sel_dn, False, dev)
    pair_rows = torch.from_numpy(step.pair_rows).to(dev)
    for s in (step, layer):
        s.run()
        torch.cuda.synchronize()
        # rows that hold pairs (padding rows of the expert-sorted buffers are never written)
        hr = pair_rows if s is step else s.rows.reshape(-1).long()
        yr = pair_rows if s is step else torch.arange(s.y.shape[0], device=dev)
        ref = s.y[yr].clone()
        href = s.h[hr].clone()
        s.y.zero_()
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            s.run()
        torch.cuda.current_stream().wait_stream(side)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            s.run()
        s.y.zero_()
        s.h.zero_()
        g.replay()
        g.replay()
        torch.cuda.synchronize()
        R.check_status(s.status)
        assert torch.equal(s.y[yr], ref) and torch.equal(s.h[hr], href)
        del g
    # the layer's output buffer argument (the pipelined end-to-end loop): same rows elsewhere
    out = torch.empty_like(layer.y)
    layer.run(out=out)
    torch.cuda.synchronize()
    assert torch.equal(out, ref)


def test_decode_layer_step_runs(dev):
    wl = syn.moe_block(0, 0.5, T=16, H=512, E=16, topk=4, I=256, T_cal=128, materialize_weights=False)
    inner = bench.DecodeStep(wl, dev)
    step = bench.MoEBlockStep(wl, (inner.pgu, inner.pgus, inner.pdn, inner.pdns), inner.sel_gu, inner.sel_dn, True,
                              dev)
    y = step.run()
    torch.cuda.synchronize()
    R.check_status(step.status)
    a = bf16_f64(y)
    assert np.isfinite(a).all() and np.abs(a).max() > 0
