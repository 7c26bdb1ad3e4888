"""The MoE block around the expert GEMMs on the device (router top-k, dispatch plan, combine),
through the C ABI, against the CPU oracle.

Bit-exact: expert ids, segment offsets, pair rows, slot tables, and the GEMM outputs of a
pipeline driven by the device plan against the same pipeline driven by a host-built layout.
Router weights: binary32 exp / sum against the oracle's binary64, relative 1e-5.  Combine:
|out - ref| <= k * 2^-23 * sum_j |w_j y_j| + one bf16 ulp of ref.
"""
import numpy as np
import pytest
import torch

from nvfp4_w4a4_moe_02_b200 import nvfp4rac as R
import nvfp4_layout as L
from nvfp4_w4a4_moe_02_b200 import synthetic as syn
from test_gpu_parity import bf16_bits, bf16_ulp, decode_pipeline, moe_pipeline, pack_host_weights, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    R.load()
    return torch.device("cuda:0")


def router_logits(T, E, seed=0):
    return syn.normal_f64(seed, syn.STREAM_ROUTER, T * E).reshape(T, E).astype(np.float32)


@pytest.mark.parametrize("T,E,k", [(4096, 128, 8), (64, 256, 8), (37, 1024, 32), (5, 3, 1), (300, 40, 6),
                                   (99, 500, 8)])
def test_route_topk_matches_oracle(dev, orc, T, E, k):
    logits = router_logits(T, E)
    st = R.new_status(dev)
    ids, w = R.moe_route_topk(torch.from_numpy(logits).to(dev), k, status=st)
    torch.cuda.synchronize()
    R.check_status(st)
    ids_ref, w_ref = orc.route_topk(logits, k)
    assert np.array_equal(ids.cpu().numpy(), ids_ref)
    assert np.allclose(w.cpu().numpy(), w_ref, rtol=1e-5, atol=0)


def test_route_topk_ties_go_to_the_lower_expert(dev, orc):
    logits = np.random.default_rng(1).integers(-2, 3, (300, 64)).astype(np.float32)
    ids, w = R.moe_route_topk(torch.from_numpy(logits).to(dev), 8)
    ids_ref, w_ref = orc.route_topk(logits, 8)
    assert np.array_equal(ids.cpu().numpy(), ids_ref)
    assert np.allclose(w.cpu().numpy(), w_ref, rtol=1e-5, atol=0)


def test_route_rejects_non_finite_logits(dev):
    logits = torch.zeros(4, 16, device=dev)
    logits[2, 5] = float("inf")
    st = R.new_status(dev)
    R.moe_route_topk(logits, 2, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 4


@pytest.mark.parametrize("T,E,k,pad", [(4096, 128, 8, 128), (4096, 128, 8, 16), (9000, 64, 4, 128), (300, 12, 3, 16),
                                       (50, 160, 128, 128)])
def test_dispatch_plan_matches_oracle(dev, orc, T, E, k, pad):
    """Offsets, pair rows and slot tables bit for bit; 9000 tokens span more than one chunk of
    the rank kernel (4096 tokens)."""
    ids_ref, _ = orc.route_topk(router_logits(T, E, seed=3), k)
    # make one expert empty and one very busy
    ids_ref = np.where(ids_ref == 5, 6, ids_ref)
    ids_ref[:, 0] = np.where(np.arange(T) % 2 == 0, 7, ids_ref[:, 0])
    for t in range(T):  # keep each token's experts distinct
        row = ids_ref[t]
        if len(set(row.tolist())) < k:
            free = [e for e in range(E) if e not in row and e != 5]
            seen = set()
            for j in range(k):
                if row[j] in seen:
                    row[j] = free.pop(0)
                seen.add(int(row[j]))
    off_ref, rows_ref = orc.dispatch_plan(ids_ref, E, pad)
    n_slots = R.moe_rows_capacity(T, k, E, 16) // 16 if pad == 16 else None
    st = R.new_status(dev)
    off, rows, se, sc = R.moe_dispatch_plan(torch.from_numpy(ids_ref).to(dev), E, pad, n_slots=n_slots, status=st)
    torch.cuda.synchronize()
    R.check_status(st)
    assert np.array_equal(off.cpu().numpy(), off_ref)
    assert np.array_equal(rows.cpu().numpy(), rows_ref)
    if pad == 16:
        counts = np.bincount(ids_ref.reshape(-1), minlength=E)
        se_ref, sc_ref, _ = L.decode_slots(counts)
        se_g, sc_g = se.cpu().numpy(), sc.cpu().numpy()
        assert np.array_equal(se_g[:se_ref.size], se_ref) and np.array_equal(sc_g[:sc_ref.size], sc_ref)
        assert np.all(se_g[se_ref.size:] == -1) and np.all(sc_g[se_ref.size:] == 0)


def test_dispatch_plan_capacity_overflow_is_reported(dev):
    ids = torch.zeros(64, 1, dtype=torch.int32, device=dev)  # 64 pairs on expert 0: 128 rows needed
    st = R.new_status(dev)
    off, rows, _, _ = R.moe_dispatch_plan(ids, 4, 128, rows_capacity=0, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 1
    assert int(off[4].item()) == -1 and bool((rows == -1).all())


def test_combine_matches_oracle(dev, orc):
    rng = np.random.default_rng(2)
    T, k, R_, H = 300, 8, 2500, 2048
    y = syn._f32_to_bf16_bits(rng.standard_normal((R_, H)).astype(np.float32))
    rows = np.stack([rng.permutation(R_)[:k] for _ in range(T)]).astype(np.int32)
    rows[7, 3] = -1  # an unrouted pair
    w = rng.random((T, k)).astype(np.float32)
    st = R.new_status(dev)
    out = R.moe_combine(to_dev(y, dev), torch.from_numpy(rows).to(dev), torch.from_numpy(w).to(dev), status=st)
    torch.cuda.synchronize()
    R.check_status(st)
    w_used = np.where(rows >= 0, w, 0.0).astype(np.float32)
    ref = orc.combine(y, np.maximum(rows, 0).astype(np.int64), w_used)
    absdot = orc.combine(syn._f32_to_bf16_bits(np.abs(syn.bf16_to_f32(y))), np.maximum(rows, 0).astype(np.int64),
                         w_used)
    got = syn.bf16_to_f32(bf16_bits(out)).astype(np.float64)
    tol = k * 2.0 ** -23 * absdot + bf16_ulp(ref)
    bad = np.argwhere(np.abs(got - ref) > tol)
    assert bad.size == 0, (bad[:5], got[tuple(bad[0])], ref[tuple(bad[0])])


def test_prefill_pipeline_with_device_plan(dev, orc):
    """Grouped prefill driven by the device plan gives the host-layout pipeline's rows bit for bit."""
    wl = syn.moe_block(T=200, H=512, E=8, topk=2, I=128, T_cal=64)
    sel_gu, _ = orc.calibrate(wl.x_cal, wl.Kp_gu)
    sel_dn, _ = orc.calibrate(syn.moe_down_calibration_batch(wl), wl.Kp_dn)
    host = moe_pipeline(dev, wl, sel_gu, sel_dn)
    st = R.new_status(dev)
    T, k = wl.topk_ids.shape
    ids = torch.from_numpy(wl.topk_ids.astype(np.int32)).to(dev)
    cap = R.moe_rows_capacity(T, k, wl.E, 128)
    off, rows, _, _ = R.moe_dispatch_plan(ids, wl.E, 128, rows_capacity=cap, status=st)
    seld_gu, seld_dn = torch.from_numpy(sel_gu).to(dev), torch.from_numpy(sel_dn).to(dev)
    a = R.Packed.empty(cap, wl.H, rows_padded=cap, device=dev, zero=True)
    ar = R.Packed.empty(cap, wl.Kp_gu, rows_padded=cap, device=dev, zero=True)
    R.nvfp4_quantize_scatter(to_dev(wl.x, dev), rows, cap, seld_gu, out=a, out_res=ar, status=st)
    pgu, pgus = R.pack_weights(to_dev(wl.wgu, dev), seld_gu, gate_up_interleave=True, status=st)
    pdn, pdns = R.pack_weights(to_dev(wl.wdn, dev), seld_dn, status=st)
    h, amax = R.grouped_w4a4_rac_moe(a, ar, off, pgu, pgus, swiglu=True, status=st)
    hq, hqr = R.nvfp4_quantize(h, seld_dn, amax_in=amax, status=st)
    y = R.grouped_w4a4_rac_moe(hq, hqr, off, pdn, pdns, status=st)
    torch.cuda.synchronize()
    R.check_status(st)
    rows_np = rows.cpu().numpy()
    # the device plan is the host layout: pair i of the (expert, token) order sits at pair_rows[i]
    pos = {(int(t), int(e)): j for t in range(T) for j, e in enumerate(wl.topk_ids[t])}
    dev_rows = np.array([rows_np[t, pos[(int(t), int(e))]] for t, e in zip(wl.pair_token, wl.pair_expert)])
    assert np.array_equal(dev_rows, host["pair_rows"])
    assert amax.item() == host["amax_h"].item()
    hr = torch.from_numpy(dev_rows).to(dev)
    assert torch.equal(h[hr], host["h"][hr]) and torch.equal(y[hr], host["y"][hr])
    # combine of the expert outputs against the oracle
    _, w_np = orc.route_topk(router_logits(T, wl.E), k)  # any weights in [0, 1]
    out = R.moe_combine(y, rows, torch.from_numpy(w_np).to(dev), status=st)
    torch.cuda.synchronize()
    ref = orc.combine(bf16_bits(y), rows_np.astype(np.int64), w_np)
    got = syn.bf16_to_f32(bf16_bits(out)).astype(np.float64)
    absdot = orc.combine(syn._f32_to_bf16_bits(np.abs(syn.bf16_to_f32(bf16_bits(y)))), rows_np.astype(np.int64),
                         w_np)
    assert np.all(np.abs(got - ref) <= k * 2.0 ** -23 * absdot + bf16_ulp(ref))


@pytest.mark.parametrize("with_rows", [True, False])
def test_down_projection_with_fused_combine(dev, orc, with_rows):
    """grouped_w4a4_rac_moe_combine (the weighted combine in the down GEMM's epilogue) against the
    oracle's combine of the unfused down projection's rows, and moe_row_pairs against the
    inverse of the plan's row map; both tile widths of the down GEMM (N = 512 and 384)."""
    for H in (512, 384):
        wl = syn.moe_block(T=300, H=H, E=8, topk=3, I=256, T_cal=64)
        sel_dn, _ = orc.calibrate(syn.moe_down_calibration_batch(wl), wl.Kp_dn)
        st = R.new_status(dev)
        T, k = wl.topk_ids.shape
        ids = torch.from_numpy(wl.topk_ids.astype(np.int32)).to(dev)
        cap = R.moe_rows_capacity(T, k, wl.E, 128)
        off, rows, _, _ = R.moe_dispatch_plan(ids, wl.E, 128, rows_capacity=cap, status=st)
        er = torch.empty(wl.E, dtype=torch.int32, device=dev)
        R.moe_dispatch_plan(ids, wl.E, 128, rows_capacity=cap, offsets=off, row_scatter=rows, expert_rows=er,
                            status=st)
        # h: any bf16 rows in the padded expert-grouped order
        h_np = syn.normal_bf16(7, 3, cap, wl.I, 1.0)
        seld = torch.from_numpy(sel_dn).to(dev)
        hq, hqr = R.nvfp4_quantize(to_dev(h_np, dev), seld, status=st)
        pdn, pdns = R.pack_weights(to_dev(wl.wdn, dev), seld, status=st)
        _, w_np = orc.route_topk(router_logits(T, wl.E, seed=3), k)
        wd = torch.from_numpy(w_np).to(dev)
        pairs = R.moe_row_pairs(rows, cap, status=st)
        kw = {"expert_rows": er} if with_rows else {}
        y = R.grouped_w4a4_rac_moe(hq, hqr, off, pdn, pdns, status=st, **kw)
        out = R.grouped_w4a4_rac_moe_combine(hq, hqr, off, pdn, pdns, pairs, wd, status=st, **kw)
        torch.cuda.synchronize()
        R.check_status(st)
        rows_np, pairs_np = rows.cpu().numpy(), pairs.cpu().numpy()
        inv = np.full(cap, -1, np.int64)
        inv[rows_np.reshape(-1)] = np.arange(T * k)
        assert np.array_equal(pairs_np, inv)
        yb = bf16_bits(y)
        ref = orc.combine(yb, rows_np.astype(np.int64), w_np)
        absdot = orc.combine(syn._f32_to_bf16_bits(np.abs(syn.bf16_to_f32(yb))), rows_np.astype(np.int64), w_np)
        got = syn.bf16_to_f32(bf16_bits(out)).astype(np.float64)
        tol = k * 2.0 ** -23 * absdot + bf16_ulp(ref)
        bad = np.argwhere(np.abs(got - ref) > tol)
        assert bad.size == 0, (H, bad[:5])


def test_row_pairs_rejects_rows_past_the_buffer(dev):
    rows = torch.tensor([[0, 5], [-1, 9]], dtype=torch.int32, device=dev)
    st = R.new_status(dev)
    pairs = R.moe_row_pairs(rows, 8, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 1
    assert pairs.cpu().numpy().tolist() == [0, -1, -1, -1, -1, 1, -1, -1]


def test_decode_pipeline_with_device_slot_tables(dev, orc):
    """Decode driven by device slot tables (worst-case slot count, unused slots skipped) gives the
    host-slot pipeline's rows bit for bit."""
    from test_gpu_parity import skewed_decode_workload

    wl = skewed_decode_workload()
    sel_gu, _ = orc.calibrate(wl.x_cal, wl.Kp_gu)
    sel_dn, _ = orc.calibrate(syn.moe_down_calibration_batch(wl), wl.Kp_dn)
    packed = pack_host_weights(dev, wl, sel_gu, sel_dn)
    host = decode_pipeline(dev, wl, sel_gu, sel_dn, packed)
    st = R.new_status(dev)
    T, k = wl.topk_ids.shape
    cap = R.moe_rows_capacity(T, k, wl.E, 16)
    n_slots = cap // 16
    off, rows, se, sc = R.moe_dispatch_plan(torch.from_numpy(wl.topk_ids.astype(np.int32)).to(dev), wl.E, 16,
                                            rows_capacity=cap, n_slots=n_slots, status=st)
    seld_gu, seld_dn = torch.from_numpy(sel_gu).to(dev), torch.from_numpy(sel_dn).to(dev)
    S16 = R.SF_SLAB16
    a = R.Packed.empty(cap, wl.H, rows_padded=cap, device=dev, zero=True, sf_layout=S16)
    ar = R.Packed.empty(cap, wl.Kp_gu, rows_padded=cap, device=dev, zero=True, sf_layout=S16)
    R.nvfp4_quantize_scatter(to_dev(wl.x, dev), rows, cap, seld_gu, out=a, out_res=ar, status=st)
    pgu, pgus, pdn, pdns = packed
    h = torch.zeros(cap, wl.I, dtype=torch.bfloat16, device=dev)
    _, amax = R.grouped_w4a4_rac_moe_decode(a, ar, se, sc, pgu, pgus, swiglu=True, y=h, status=st)
    hq = R.Packed.empty(cap, wl.I, rows_padded=cap, device=dev, sf_layout=S16)
    hqr = R.Packed.empty(cap, wl.Kp_dn, rows_padded=cap, device=dev, sf_layout=S16)
    R.nvfp4_quantize(h, seld_dn, amax_in=amax, out=hq, out_res=hqr, status=st)
    y = R.grouped_w4a4_rac_moe_decode(hq, hqr, se, sc, pdn, pdns, status=st)
    torch.cuda.synchronize()
    R.check_status(st)
    used = int(off[wl.E].item()) // 16
    assert used == host["slot_expert"].size and used < n_slots
    rows_np = rows.cpu().numpy()
    pos = {(int(t), int(e)): j for t in range(T) for j, e in enumerate(wl.topk_ids[t])}
    dev_rows = np.array([rows_np[t, pos[(int(t), int(e))]] for t, e in zip(wl.pair_token, wl.pair_expert)])
    assert np.array_equal(dev_rows, host["pair_rows"])
    assert amax.item() == host["amax_h"].item()
    hr = torch.from_numpy(dev_rows).to(dev)
    assert torch.equal(h[hr], host["h"][hr]) and torch.equal(y[hr], host["y"][hr])
