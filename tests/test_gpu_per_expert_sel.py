"""Per-expert channel lists (a RAC variant the pages leave open) on a B200, through the C ABI:
grouped activation quantisation, grouped weight pack, grouped calibration and the row -> expert
map, each bit-exact against the oracle; malformed lists are reported in the device status."""
import numpy as np
import pytest
import torch

from nvfp4_w4a4_moe_02_b200 import nvfp4rac as R
from nvfp4_w4a4_moe_02_b200 import synthetic as syn
from test_gpu_parity import logical, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    R.load()
    return torch.device("cuda:0")


def random_lists(seed: int, G: int, K: int, Kp: int) -> np.ndarray:
    rng = np.random.default_rng(seed)
    return np.stack([np.sort(rng.choice(K, Kp, replace=False)) for _ in range(G)]).astype(np.int32)


def row_groups_ref(off: np.ndarray, rows: int) -> np.ndarray:
    g = np.full(rows, -1, np.int32)
    if off[-1] < 0:
        return g
    for e in range(off.size - 1):
        g[off[e]:off[e + 1]] = e
    return g


@pytest.mark.parametrize("off", [[0, 128, 128, 384, 512, 896], [0, 16, 16, 16, 48, 64], [0, 0, 0, 0, 0, 0],
                                 [0, 128, 256, 256, 384, -1]])
def test_row_groups_match_offsets(dev, off):
    off = np.array(off, np.int32)
    rows = 1000
    got = R.moe_row_groups(torch.from_numpy(off).to(dev), off.size - 1, rows)
    torch.cuda.synchronize()
    assert np.array_equal(got.cpu().numpy(), row_groups_ref(off.astype(np.int64), rows))


# rows < 2 * SMs * 8 run one CTA per row; more rows run one warp per row: both kernels are covered
@pytest.mark.parametrize("rows,K,Kp,G", [(40, 256, 64, 3), (300, 768, 384, 5), (4100, 768, 384, 7),
                                         (2200, 2048, 1024, 4)])
def test_grouped_quantize_matches_oracle(dev, orc, rows, K, Kp, G):
    rng = np.random.default_rng(rows)
    x = syn.normal_bf16(rows, 1, rows, K, 1.0, np.exp(rng.standard_normal(K)))
    sel = random_lists(K + G, G, K, Kp)
    rows_padded = (rows + 127) // 128 * 128 + 128
    rg = rng.integers(-1, G, rows_padded).astype(np.int32)
    st = R.new_status(dev)
    q, qr = R.nvfp4_quantize(to_dev(x, dev), torch.from_numpy(sel).to(dev), rows_padded=rows_padded, status=st,
                             row_group=torch.from_numpy(rg).to(dev))
    torch.cuda.synchronize()
    R.check_status(st)
    s_ref = orc.global_scale(orc.amax_bf16(x))
    assert q.s_g.item() == float(s_ref) and qr.s_g.item() == float(s_ref)
    codes, S, rcodes, rS, _ = orc.act_quant_rac_grouped(x, s_ref, sel, rg[:rows])
    gc, gS = logical(q)
    assert np.array_equal(gS, S) and np.array_equal(gc, codes)
    grc, grS = logical(qr)
    assert np.array_equal(grS, rS), np.argwhere(grS != rS)[:5]
    assert np.array_equal(grc, rcodes), np.argwhere(grc != rcodes)[:5]
    # rows past M are zero in both tensors whatever their group
    fc, fS = logical(qr, rows=rows_padded)
    assert not fc[rows:].any() and not fS[rows:].any()


@pytest.mark.parametrize("interleave", [False, True])
def test_grouped_pack_matches_oracle(dev, orc, interleave):
    E, N, K, Kp = 3, 256, 512, 256
    w = syn.normal_bf16(4, 2, E * N, K, 0.02).reshape(E, N, K)
    sel = random_lists(5, E, K, Kp)
    wq, wsq = R.pack_weights(to_dev(w, dev), torch.from_numpy(sel).to(dev), gate_up_interleave=interleave)
    torch.cuda.synchronize()
    for e in range(E):
        s_ref = orc.global_scale(orc.amax_bf16(w[e]))
        assert wq.s_g[e].item() == float(s_ref) and wsq.s_g[e].item() == float(s_ref)
        we = w[e]
        if interleave:
            p = np.arange(N)
            q, j = p // 128, p % 128
            we = we[np.where(j < 64, q * 64 + j, N // 2 + q * 64 + j - 64)]
        c, S, sc, sS = orc.weight_pack(we, s_ref, sel[e])
        gc, gS = logical(wq, e)
        gsc, gsS = logical(wsq, e)
        assert np.array_equal(gc, c) and np.array_equal(gS, S)
        assert np.array_equal(gsc, sc) and np.array_equal(gsS, sS)


@pytest.mark.parametrize("T,K,Kp,off", [(96, 256, 128, [0, 30, 30, 96]), (1500, 768, 384, [0, 700, 701, 1200, 1500]),
                                        (64, 320, 64, [0, 64])])
def test_grouped_calibrate_matches_oracle(dev, orc, T, K, Kp, off):
    rng = np.random.default_rng(T)
    x = syn.normal_bf16(9, 3, T, K, 1.0, np.exp(rng.standard_normal(K)))
    off = np.array(off, np.int64)
    sel_ref, err_ref = orc.calibrate_grouped(x, off, Kp)
    st = R.new_status(dev)
    sel, err = R.rac_calibrate_grouped(to_dev(x, dev), torch.from_numpy(off.astype(np.int32)).to(dev), Kp,
                                       want_err=True, status=st)
    torch.cuda.synchronize()
    R.check_status(st)
    assert np.array_equal(err.cpu().numpy(), err_ref)
    assert np.array_equal(sel.cpu().numpy(), sel_ref)


def test_malformed_lists_and_groups_are_reported(dev):
    """A list that is not ascending, a group index past the last list and offsets outside
    [0, T] each end in NVFP4_ERR_INVALID_ARG in the status; every access stays in bounds."""
    K, Kp, rows = 256, 64, 256
    x = to_dev(syn.normal_bf16(2, 1, rows, K, 1.0), dev)
    sel = random_lists(1, 2, K, Kp)
    bad = sel.copy()
    bad[1, 10], bad[1, 11] = bad[1, 11], bad[1, 10]
    rg = torch.zeros(rows, dtype=torch.int32, device=dev)
    rg[5] = 1
    st = R.new_status(dev)
    R.nvfp4_quantize(x, torch.from_numpy(bad).to(dev), status=st, row_group=rg)
    torch.cuda.synchronize()
    assert st.item() == 1  # NVFP4_ERR_INVALID_ARG
    rg[5] = 2  # only lists 0 and 1 exist
    st = R.new_status(dev)
    R.nvfp4_quantize(x, torch.from_numpy(sel).to(dev), status=st, row_group=rg)
    torch.cuda.synchronize()
    assert st.item() == 1  # NVFP4_ERR_INVALID_ARG
    st = R.new_status(dev)
    R.rac_calibrate_grouped(x, torch.tensor([0, 300], dtype=torch.int32, device=dev), Kp, status=st)
    torch.cuda.synchronize()
    assert st.item() == 1  # NVFP4_ERR_INVALID_ARG
