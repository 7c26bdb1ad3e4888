"""Host-side layout helpers and input builders, checked on the CPU against their definitions:
the expert-sorted padded layout (gather / scatter maps), and the per-expert grouping of the down
projection's calibration rows."""
import numpy as np

from nvfp4_w4a4_moe_02_b200 import nvfp4rac as R
import nvfp4_layout as L
from nvfp4_w4a4_moe_02_b200 import synthetic as syn


def test_gather_and_scatter_maps_describe_the_same_padded_layout():
    rng = np.random.default_rng(4)
    T, E, k = 50, 6, 2
    ids = np.stack([rng.choice(E, k, replace=False) for _ in range(T)])
    ids[ids == 5] = 4  # expert 5 gets nothing
    ids[:, 1] = np.where(ids[:, 1] == ids[:, 0], (ids[:, 0] + 1) % 5, ids[:, 1])
    pt, pe, counts = syn.sort_pairs(ids, E)
    g, off, pair_rows = L.gather_map(pt, counts)
    assert off[0] == 0 and np.all(np.diff(off) % 128 == 0) and counts[5] == 0 and off[6] == off[5]
    for e in range(E):  # each expert's pairs fill the head of its 128-padded segment, in order
        rows = pair_rows[pe == e]
        assert np.array_equal(rows, off[e] + np.arange(counts[e]))
        assert np.all(g[off[e] + counts[e]:off[e + 1]] == -1)
    assert np.array_equal(g[pair_rows], pt)
    sm = L.scatter_map(pt, pair_rows, T, k)
    for t in range(T):  # a token's scatter rows are exactly the rows whose gather source is t
        assert sorted(sm[t][sm[t] >= 0].tolist()) == sorted(np.nonzero(g == t)[0].tolist())


def test_decode_slots_cover_each_expert_in_16_row_slabs():
    counts = np.array([0, 17, 3, 0, 16, 33])
    se, sc, pr = L.decode_slots(counts)
    assert se.tolist() == [1, 1, 2, 4, 5, 5, 5] and sc.tolist() == [16, 1, 3, 16, 16, 16, 1]
    assert pr.size == counts.sum() and len(set(pr.tolist())) == pr.size
    assert np.all(pr // 16 < se.size) and np.all(pr % 16 < sc[pr // 16])


def test_down_calibration_offsets_line_up_with_the_calibration_rows():
    """Group e of the calibration batch holds exactly the (token, expert e) pairs of the
    calibration routing: its rows are silu(g) * u of expert e's own weights."""
    wl = syn.moe_block(T=32, H=256, E=4, topk=2, I=128, T_cal=24)
    h_cal = syn.moe_down_calibration_batch(wl)
    off = syn.moe_down_calibration_offsets(wl)
    assert off[0] == 0 and off[-1] == h_cal.shape[0] and np.all(np.diff(off) >= 0)
    topk = syn.route_topk(wl.seed, wl.x_cal.shape[0], wl.E, 2, stream=syn.STREAM_ROUTER_CAL)
    pt, pe, _ = syn.sort_pairs(topk, wl.E)
    xf = syn.bf16_to_f32(wl.x_cal).astype(np.float64)
    for e in range(wl.E):
        idx = np.arange(off[e], off[e + 1])
        assert np.all(pe[idx] == e)
        if idx.size == 0:
            continue
        w = syn.bf16_to_f32(wl.gate_up_expert(e)).astype(np.float64)
        gu = xf[pt[idx[0]]] @ w.T
        h = gu[:wl.I] / (1.0 + np.exp(-gu[:wl.I])) * gu[wl.I:]
        got = syn.bf16_to_f32(h_cal[idx[0]]).astype(np.float64)
        assert np.allclose(got, h, rtol=2 ** -7, atol=1e-30), e
