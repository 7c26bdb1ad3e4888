"""Expert parallelism over two gloo ranks on CPU (the multi-GPU exchange is not run on hardware
here: one GPU per run).

Each rank holds half of the tokens and half of the experts.  The data movement is the product's
(nvfp4_w4a4_moe_02_b200.ep: count exchange, all-to-all of the packed NVFP4 rows, global amax
reductions, the reverse all-to-all); the arithmetic on each rank is the oracle's (quantisation,
gate_up, SwiGLU, down, combine), in place of the GPU kernels.  The result on every rank must be
bit-identical to the single-rank pipeline over the whole batch, and the rows each rank receives
must be exactly the single-rank layout's rows of its experts."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HERE = os.path.dirname(os.path.abspath(__file__))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _workload():
    from nvfp4_w4a4_moe_02_b200 import synthetic as syn

    return syn.moe_block(T=96, H=256, E=8, topk=3, I=128, T_cal=64)


def _single_rank(orc, wl, sel_gu, sel_dn):
    """The oracle pipeline over the whole batch on one rank: (out [T, H] float64, plan, codes)."""
    s_x = orc.global_scale(orc.amax_bf16(wl.x))
    off, row = orc.dispatch_plan(wl.topk_ids, wl.E, 128)
    T, k = wl.topk_ids.shape
    ac, aS, rc, rS, _ = orc.act_quant_rac(wl.x, s_x, sel_gu)
    rows = int(off[-1])
    codes = np.zeros((rows, wl.H), np.uint8)
    for t in range(T):
        for j in range(k):
            codes[row[t, j]] = ac[t]
    h = np.zeros((rows, wl.I), np.uint16)
    for e in range(wl.E):
        r = [(t, j) for t in range(T) for j in range(k) if wl.topk_ids[t, j] == e]
        if not r:
            continue
        toks = np.array([t for t, _ in r])
        wgu = wl.gate_up_expert(e)
        s_w = orc.global_scale(orc.amax_bf16(wgu))
        gu, _ = orc.gemm_rac(ac[toks], aS[toks], rc[toks], rS[toks], *orc.weight_pack(wgu, s_w, sel_gu), s_x, s_w)
        h[[row[t, j] for t, j in r]] = orc.swiglu(orc.f64_to_bf16_array(gu))[0]
    used = np.zeros(rows, bool)
    used[row.reshape(-1)] = True
    s_h = orc.global_scale(orc.amax_bf16(h[used]))
    y = np.zeros((rows, wl.H), np.uint16)
    for e in range(wl.E):
        rr = np.arange(off[e], off[e + 1])
        rr = rr[used[rr]]
        if rr.size == 0:
            continue
        hc, hS, hrc, hrS, _ = orc.act_quant_rac(h[rr], s_h, sel_dn)
        wdn = wl.down_expert(e)
        s_w = orc.global_scale(orc.amax_bf16(wdn))
        yy, _ = orc.gemm_rac(hc, hS, hrc, hrS, *orc.weight_pack(wdn, s_w, sel_dn), s_h, s_w)
        y[rr] = orc.f64_to_bf16_array(yy)
    w = np.full(wl.topk_ids.shape, 0.25, np.float32)
    return orc.combine(y, row, w), off, row, codes


def _worker(rank, ws, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    sys.path.insert(0, HERE)
    import datetime

    import oracle as orc
    from nvfp4_layout import pack_codes, pack_sf, unpack_codes, unpack_sf
    from nvfp4_w4a4_moe_02_b200 import synthetic as syn
    from nvfp4_w4a4_moe_02_b200.ep import ExpertParallel

    dist.init_process_group("gloo", rank=rank, world_size=ws, timeout=datetime.timedelta(seconds=120))
    try:
        orc.build()
        wl = _workload()
        sel_gu = orc.calibrate(wl.x_cal, wl.Kp_gu)[0]
        sel_dn = orc.calibrate(syn.moe_down_calibration_batch(wl), wl.Kp_dn)[0]
        out_ref, off_ref, row_ref, codes_ref = _single_rank(orc, wl, sel_gu, sel_dn)

        ep = ExpertParallel(wl.E)
        T = wl.x.shape[0] // ws
        x = wl.x[rank * T:(rank + 1) * T]
        ids = wl.topk_ids[rank * T:(rank + 1) * T]
        k = ids.shape[1]
        H, I, El = wl.H, wl.I, ep.E_local
        # the send layout: the dispatch plan over all E experts of this rank's tokens
        off, row = orc.dispatch_plan(ids, wl.E, 128)
        counts = np.bincount(ids.reshape(-1), minlength=wl.E).astype(np.int32)
        amax = torch.tensor([float(orc.amax_bf16(x))], dtype=torch.float32)
        s_x = orc.global_scale(float(ep.global_amax(amax)[0]))
        ac, aS, rc, rS, _ = orc.act_quant_rac(x, s_x, sel_gu)
        rows = int(off[-1])
        send = {n: np.zeros((rows, c), np.uint8) for n, c in (("c", H), ("s", H // 16), ("rc", len(sel_gu)),
                                                                ("rs", len(sel_gu) // 16))}
        for t in range(T):
            for j in range(k):
                send["c"][row[t, j]], send["s"][row[t, j]] = ac[t], aS[t]
                send["rc"][row[t, j]], send["rs"][row[t, j]] = rc[t], rS[t]
        to_t = lambda a: torch.from_numpy(np.ascontiguousarray(a))
        send_rows = ep.send_rows(torch.from_numpy(off.astype(np.int32)))
        recv_counts = ep.exchange_counts(torch.from_numpy(counts))
        seg_off, seg_rows, seg_expert, recv_rows = ep.recv_segments(recv_counts)
        got = {}
        for main, sc, cols in (("c", "s", H), ("rc", "rs", len(sel_gu))):
            codes_b, sf_b = ep.exchange_packed(to_t(pack_codes(send[main])), to_t(pack_sf(send[sc], rows)), cols,
                                               send_rows, recv_rows)
            n = sum(recv_rows)
            got[main] = unpack_codes(codes_b.numpy(), n, n, cols)
            got[sc] = unpack_sf(sf_b.numpy(), n, n, cols)
        # the rows received for local expert e from source s are the single-rank rows of expert
        # r E/P + e taken by source s's tokens, in token order
        so = seg_off.numpy()
        for si in range(ws * El):
            s, e = divmod(si, El)
            ge = rank * El + e
            ref_rows = [row_ref[t, j] for t in range(s * T, (s + 1) * T) for j in range(k) if wl.topk_ids[t, j] == ge]
            n = int(seg_rows[si])
            assert n == len(ref_rows)
            assert np.array_equal(got["c"][so[si]:so[si] + n], codes_ref[ref_rows])
        # the local experts on the received segments (oracle arithmetic)
        n = sum(recv_rows)
        h = np.zeros((n, I), np.uint16)
        hmask = np.zeros(n, bool)
        for si in range(ws * El):
            e = int(seg_expert[si])
            rr = np.arange(so[si], so[si] + int(seg_rows[si]))
            if rr.size == 0:
                continue
            wgu = wl.gate_up_expert(rank * El + e)
            s_w = orc.global_scale(orc.amax_bf16(wgu))
            gu, _ = orc.gemm_rac(got["c"][rr], got["s"][rr], got["rc"][rr], got["rs"][rr],
                                 *orc.weight_pack(wgu, s_w, sel_gu), s_x, s_w)
            h[rr] = orc.swiglu(orc.f64_to_bf16_array(gu))[0]
            hmask[rr] = True
        amax_h = torch.tensor([float(orc.amax_bf16(h[hmask])) if hmask.any() else 0.0], dtype=torch.float32)
        s_h = orc.global_scale(float(ep.global_amax(amax_h)[0]))
        y = np.zeros((n, H), np.uint16)
        for si in range(ws * El):
            e = int(seg_expert[si])
            rr = np.arange(so[si], so[si] + int(seg_rows[si]))
            if rr.size == 0:
                continue
            hc, hS, hrc, hrS, _ = orc.act_quant_rac(h[rr], s_h, sel_dn)
            wdn = wl.down_expert(rank * El + e)
            s_w = orc.global_scale(orc.amax_bf16(wdn))
            yy, _ = orc.gemm_rac(hc, hS, hrc, hrS, *orc.weight_pack(wdn, s_w, sel_dn), s_h, s_w)
            y[rr] = orc.f64_to_bf16_array(yy)
        back = ep.exchange_rows(torch.from_numpy(y.view(np.uint8).reshape(n, 2 * H)), recv_rows, send_rows)
        out = orc.combine(back.numpy().view(np.uint16).reshape(-1, H), row, np.full(ids.shape, 0.25, np.float32))
        q.put((rank, bool(np.array_equal(out, out_ref[rank * T:(rank + 1) * T])), send_rows, recv_rows))
    except Exception as exc:  # report instead of hanging the other rank's queue read
        q.put((rank, repr(exc), None, None))
        raise
    finally:
        dist.destroy_process_group()


def test_two_rank_expert_parallel_matches_one_rank():
    ws, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, ws, port, q)) for r in range(ws)]
    for p in procs:
        p.start()
    results = sorted(q.get(timeout=300) for _ in range(ws))
    for p in procs:
        p.join(timeout=60)
    for rank, ok, send_rows, recv_rows in results:
        assert ok is True, (rank, ok)
        assert all(r % 128 == 0 for r in send_rows + recv_rows)
    # what rank 0 sends to rank 1 is what rank 1 receives from rank 0
    assert results[0][2][1] == results[1][3][0] and results[1][2][0] == results[0][3][1]
    for p in procs:
        assert p.exitcode == 0


def test_layout_helpers_on_one_rank():
    """recv_segments pads each (source, expert) segment to 128 rows in source-major order."""
    sys.path.insert(0, ROOT)
    from nvfp4_w4a4_moe_02_b200.ep import ExpertParallel

    ep = ExpertParallel.__new__(ExpertParallel)
    ep.P, ep.E_local, ep.pad, ep.E = 2, 3, 128, 6
    off, rows, expert, per_source = ep.recv_segments(torch.tensor([[5, 0, 130], [128, 1, 0]], dtype=torch.int32))
    assert off.tolist() == [0, 128, 128, 384, 512, 640, 640]
    assert rows.tolist() == [5, 0, 130, 128, 1, 0]
    assert expert.tolist() == [0, 1, 2, 0, 1, 2]
    assert per_source == [384, 256]
    assert ep.send_rows.__doc__ and [ExpertParallel.owner(ep, e) for e in range(6)] == [0, 0, 0, 1, 1, 1]
