"""The CTA-pair form of the W4A4 + RAC GEMM (one 256 x 256 tile over the two SMs of a cluster)
against the oracle: dense shapes with a ragged last pair, the grouped MoE block with segments of
an odd number of 128-row blocks (the follower's half runs past the segment and must store
nothing), the SwiGLU epilogue, the expert_rows box skipping, and the two full-size prefill
configurations on whole m-blocks spread over the tile order."""
import numpy as np
import pytest
import torch

from nvfp4_w4a4_moe_02_b200 import nvfp4rac as R
from nvfp4_w4a4_moe_02_b200 import synthetic as syn
import test_gpu_parity as P

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    R.load()
    R.set_gemm_pairs(True)
    yield torch.device("cuda:0")
    R.set_gemm_pairs(False)


@pytest.mark.parametrize("M,N,K,Kp", [(300, 512, 768, 384), (520, 256, 1024, 1024), (128, 768, 320, 64),
                                      (1000, 1024, 2048, 0)])
def test_pair_gemm_dense_matches_oracle(dev, orc, M, N, K, Kp):
    rng = np.random.default_rng(M + N + K)
    cs = np.exp(rng.standard_normal(K))
    x = syn.normal_bf16(12, 1, M, K, 1.0, cs)
    w = syn.normal_bf16(12, 2, N, K, 0.02)
    x_cal = syn.normal_bf16(12, 3, 128, K, 1.0, cs)
    P.run_dense(dev, orc, x, w, x_cal, Kp, torch.float32)
    P.run_dense(dev, orc, x, w, x_cal, Kp, torch.bfloat16)


def test_pair_gemm_moe_small_ragged(dev, orc):
    P.test_moe_small_ragged(dev, orc)


def test_pair_gemm_expert_rows_skips_padding_boxes(dev, orc):
    P.test_grouped_expert_rows_skips_padding_boxes(dev, orc)


def test_pair_gemm_dense_prefill_whole_blocks(dev, orc):
    P.test_gemm_dense_prefill_sampled(dev, orc)


def test_pair_gemm_moe_prefill_whole_blocks(dev, orc):
    P.test_moe_prefill_full_sampled(dev, orc)


def test_pair_and_single_sm_agree(dev, orc):
    """The same operands through both forms: every output within the GEMM tolerance of each
    other (the exact product of the quantised operands is the same)."""
    M, N, K, Kp = 640, 768, 1024, 512
    x = syn.normal_bf16(31, 1, M, K, 1.0, syn.outlier_colscale(31, K))
    w = syn.normal_bf16(31, 2, N, K, 0.02)
    sel = torch.from_numpy(np.sort(np.random.default_rng(31).choice(K, Kp, replace=False)).astype(np.int32)).to(dev)
    st = R.new_status(dev)
    q, qr = R.nvfp4_quantize(P.to_dev(x, dev), sel, status=st)
    wq, wsq = R.pack_weights(P.to_dev(w, dev), sel, status=st)
    y2 = R.w4a4_rac_gemm(q, qr, wq, wsq, M, out_dtype=torch.float32, status=st)
    R.set_gemm_pairs(False)
    try:
        y1 = R.w4a4_rac_gemm(q, qr, wq, wsq, M, out_dtype=torch.float32, status=st)
    finally:
        R.set_gemm_pairs(True)
    torch.cuda.synchronize()
    R.check_status(st)
    f = orc.dense_rac_forward(x, w, sel.cpu().numpy(), rows=np.arange(M))
    tol = 2e-3 * f["absdot"] + 2e-6
    assert (np.abs(y1.cpu().numpy().astype(np.float64) - y2.cpu().numpy()) <= tol).all()
