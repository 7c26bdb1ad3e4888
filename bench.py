"""Benchmark of the NVFP4 W4A4 + RAC hot path on B200.

Default workload (moe_prefill), the MoE prefill expert block, one step = the rollout hot path
over one batch with weights already packed (packing runs once per trainer -> rollout sync):
    per-tensor amax of X -> quantise X (+ residual on the calibrated channels) scattered into
    expert-sorted, 128-padded rows -> grouped gate_up GEMM (W4A4 + RAC) with the SwiGLU + amax
    epilogue -> quantise h (+ residual) -> grouped down GEMM (W4A4 + RAC).
    4096 tokens, hidden 2048, 128 experts, top-8 of softmax(N(0,1) logits), gate_up
    128 x (1536 x 2048), down 128 x (2048 x 768), r = 0.5; synthetic seeded inputs.
Other workloads (--workload): dense (8192 x 4096 x 4096 projection), moe_decode (64 tokens,
hidden 7168, 256 experts, swap-AB decode GEMMs), moe_prefill_layer / moe_decode_layer (the
same with the device router, dispatch plan and combine: no host work per step), qdq /
qdq_single (trainer fake-quant of 2^31 weights), sweep (r in {0, 0.25, 0.5, 1}, the masked and per-expert
variants, and the same block on the FP8 comparison format).

Metric: effective TFLOP/s of the step's GEMMs, 2*rows*N*(K + K') summed over the GEMMs (the
residual loop counted, as it is part of the method), over the measured step time; GB/s for
the fake-quant workloads.  Also reported: act-quant GB/s, per-kernel times and the roofline of
the dominant kernel.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload W] [--impl reference]
Under torchrun every rank runs its own replica (weak scaling, no data-path collective);
rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
FP4_OVER_BF16 = 4.0  # nominal dense FP4 / BF16 tensor ratio (9 / 2.25 PFLOP/s)
METRIC = "W4A4+RAC MoE GEMM effective TFLOPS & % FP4 peak; act-quant GB/s"


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return PEAKS_FALLBACK, "fallback"


def max_over_ranks(value: float, ws: int, device) -> float:
    """The largest per-rank value (a step time): every rank takes part, every rank gets it."""
    if ws <= 1:
        return value
    import torch
    import torch.distributed as dist

    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(work_per_rank: float, ws: int, t_ms_max: float, scale: float) -> float:
    """Weak scaling: every rank does work_per_rank in t_ms_max (the slowest rank's time)."""
    return ws * work_per_rank / (t_ms_max * 1e-3) / scale


def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


# ------------------------------------------------------------------------------------------ workload
def build_inputs(seed=0, experts=None):
    from nvfp4_w4a4_moe_02_b200 import synthetic as syn

    wl = syn.moe_prefill(seed=seed) if experts is None else \
        syn.moe_block(seed, 0.5, T=4096, H=2048, E=experts, topk=8, I=768)
    h_cal = syn.moe_down_calibration_batch(wl)
    return wl, h_cal


def flops_of(wl, Kp_gu, Kp_dn):
    P = int(wl.pair_token.size)
    gu = 2.0 * P * (2 * wl.I) * (wl.H + Kp_gu)
    dn = 2.0 * P * wl.H * (wl.I + Kp_dn)
    return gu, dn


def quant_bytes(rows, K, Kp):
    # bf16 read once + codes and scales of X and R_sel
    return rows * (2.0 * K + 0.5625 * (K + Kp))


def device_layout(R, wl, dev, pad, status, decode=False):
    """The workload's expert-grouped layout made on the device by moe_dispatch_plan (segments padded
    to `pad` rows; 16-row slot tables for decode).  Returns a dict of device tensors and, for the
    error sampling and the configuration record, the host copies it needs."""
    import torch

    T, k = wl.topk_ids.shape
    ids = torch.from_numpy(np.ascontiguousarray(wl.topk_ids, dtype=np.int32)).to(dev)
    cap = R.moe_rows_capacity(T, k, wl.E, pad)
    n_slots = cap // 16 if decode else None
    off, rs, se, sc = R.moe_dispatch_plan(ids, wl.E, pad, rows_capacity=cap, n_slots=n_slots, status=status,
                                          expert_rows=(er := torch.empty(wl.E, dtype=torch.int32, device=dev)))
    torch.cuda.synchronize()
    R.check_status(status)
    rows_scatter = rs.cpu().numpy()
    # the row of every (expert, token)-sorted pair, for sampling rows of the outputs
    e_flat = wl.topk_ids.reshape(-1)
    t_flat = np.repeat(np.arange(T), k)
    order = np.lexsort((t_flat, e_flat))
    assert np.array_equal(t_flat[order], wl.pair_token) and np.array_equal(e_flat[order], wl.pair_expert)
    out = dict(offsets=off, row_scatter=rs, expert_rows=er, cap=cap, rows_used=int(off[-1].item()),
               pair_rows=rows_scatter.reshape(-1)[order].astype(np.int64))
    if decode:
        out.update(slot_expert=se, slot_count=sc, n_slots=n_slots, slots_used=int((sc > 0).sum().item()),
                   slot_first_row=torch.arange(n_slots, dtype=torch.int32, device=dev) * 16)
    return out


class MoEStep:
    """Device-resident state of one replica and the step itself (C-ABI calls only)."""

    def __init__(self, wl, h_cal, dev, masked=False, h_cal_offsets=None, own_scale=False):
        """h_cal_offsets (int64 [E + 1], rows of h_cal per expert) selects the per-expert variant:
        one down-projection channel list per expert, calibrated on that expert's rows.  own_scale
        selects the variant with the residual's own tensor scale (two accumulators)."""
        import torch

        from nvfp4_w4a4_moe_02_b200 import nvfp4rac as R

        self.R, self.torch, self.dev, self.wl, self.masked = R, torch, dev, wl, masked
        self.own = own_scale
        to = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to(dev).view(torch.bfloat16)
        self.status = R.new_status(dev)
        # offline: channel selection on the calibration batches, weight pack
        self.sel_gu, _ = R.rac_calibrate(to(wl.x_cal), wl.Kp_gu, status=self.status)
        if h_cal_offsets is None:
            self.sel_dn, _ = R.rac_calibrate(to(h_cal), wl.Kp_dn, status=self.status)
        else:
            offd = torch.from_numpy(np.asarray(h_cal_offsets, np.int32)).to(dev)
            self.sel_dn, _ = R.rac_calibrate_grouped(to(h_cal), offd, wl.Kp_dn, status=self.status)
        if masked:
            # masked full-K residual variant: the residual pass reuses the main packed weights
            self.pgu, _ = R.pack_weights(to(wl.wgu), None, gate_up_interleave=True, status=self.status)
            self.pdn, _ = R.pack_weights(to(wl.wdn), None, status=self.status)
            self.pgus, self.pdns = self.pgu, self.pdn
        else:
            self.pgu, self.pgus = R.pack_weights(to(wl.wgu), self.sel_gu, gate_up_interleave=True,
                                                 status=self.status)
            self.pdn, self.pdns = R.pack_weights(to(wl.wdn), self.sel_dn, status=self.status)
        # expert-grouped layout of the routed pairs, made on the device (routing is fixed for the
        # run, so the plan is made once; the *_layer workloads make it every step)
        lay = device_layout(R, wl, dev, 128, self.status)
        self.pair_rows = lay["pair_rows"]
        self.rows_padded = lay["rows_used"]
        self.scatter, self.offsets, self.expert_rows = lay["row_scatter"], lay["offsets"], lay["expert_rows"]
        cap = lay["cap"]
        # per-expert lists: each expert-sorted row of h takes its expert's list
        self.row_group = R.moe_row_groups(self.offsets, wl.E, cap) if h_cal_offsets is not None else None
        self.x = to(wl.x)
        # preallocated outputs (the step allocates nothing), sized for the worst-case layout;
        # padding rows of the expert-grouped activations are never written: zero them once
        P = R.Packed
        self.a = P.empty(cap, wl.H, rows_padded=cap, device=dev, zero=True)
        self.ar = P.empty(cap, wl.H if masked else wl.Kp_gu, rows_padded=cap, device=dev, zero=True)
        self.h = torch.zeros(cap, wl.I, dtype=torch.bfloat16, device=dev)
        self.amax_h = torch.zeros(1, dtype=torch.float32, device=dev)
        self.hq = P.empty(cap, wl.I, rows_padded=cap, device=dev, zero=True)
        self.hqr = P.empty(cap, wl.I if masked else wl.Kp_dn, rows_padded=cap, device=dev, zero=True)
        self.y = torch.empty(cap, wl.H, dtype=torch.bfloat16, device=dev)
        # the variants quantise h with the row quantiser over the used rows (views of the same storage)
        self.h_used = self.h[:self.rows_padded]
        self.hq_used, self.hqr_used = self.hq.prefix(self.rows_padded), self.hqr.prefix(self.rows_padded)
        self.row_group_used = self.row_group[:self.rows_padded] if self.row_group is not None else None
        torch.cuda.synchronize()
        R.check_status(self.status)
        torch.cuda.empty_cache()  # drop the bf16 weight staging buffers

    def run(self, x=None, events=None):
        R = self.R
        x = self.x if x is None else x
        ev = events or {}
        if "q0" in ev:
            ev["q0"].record()
        R.nvfp4_quantize_scatter(x, self.scatter, self.rows_padded, self.sel_gu, out=self.a, out_res=self.ar,
                                 status=self.status, own_scale=self.own)
        if "g0" in ev:
            ev["g0"].record()
        R.grouped_w4a4_rac_moe(self.a, self.ar, self.offsets, self.pgu, self.pgus, swiglu=True, y=self.h,
                               amax_out=self.amax_h, status=self.status, expert_rows=self.expert_rows,
                               own_scale=self.own)
        if "q1" in ev:
            ev["q1"].record()
        if self.masked or self.row_group is not None:
            R.nvfp4_quantize(self.h_used, self.sel_dn, amax_in=self.amax_h, out=self.hq_used, out_res=self.hqr_used,
                             status=self.status, masked=self.masked, row_group=self.row_group_used)
        else:
            # the token rows of each expert segment only
            R.nvfp4_quantize_segments(self.h, self.offsets, self.expert_rows, self.sel_dn, amax_in=self.amax_h,
                                      out=self.hq, out_res=self.hqr, status=self.status, own_scale=self.own)
        if "d0" in ev:
            ev["d0"].record()
        R.grouped_w4a4_rac_moe(self.hq, self.hqr, self.offsets, self.pdn, self.pdns, y=self.y, status=self.status,
                               expert_rows=self.expert_rows, own_scale=self.own)
        if "end" in ev:
            ev["end"].record()
        return self.y

    KERNELS_PER_STEP = 5  # amax, quantise X, gate_up GEMM, quantise h, down GEMM


class Mx8MoEStep:
    """The same MoE expert block on the FP8 comparison format (E4M3, one power-of-two scale per
    32 elements; C-ABI calls only): quantise-scatter X, grouped gate_up with SwiGLU, quantise h,
    grouped down.  No calibration, no residual, no tensor scales."""

    KERNELS_PER_STEP = 4  # quantise X, gate_up GEMM, quantise h, down GEMM

    def __init__(self, wl, dev):
        import torch

        from nvfp4_w4a4_moe_02_b200 import mxfp8 as F
        from nvfp4_w4a4_moe_02_b200 import nvfp4rac as R

        self.F, self.R, self.wl = F, R, wl
        to = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to(dev).view(torch.bfloat16)
        self.status = R.new_status(dev)
        self.wgu = F.pack_weights(to(wl.wgu), gate_up_interleave=True, status=self.status)
        self.wdn = F.pack_weights(to(wl.wdn), status=self.status)
        lay = device_layout(R, wl, dev, 128, self.status)
        self.pair_rows = lay["pair_rows"]
        self.rows_padded = lay["rows_used"]
        self.scatter, self.offsets, self.expert_rows = lay["row_scatter"], lay["offsets"], lay["expert_rows"]
        self.x = to(wl.x)
        # padding rows are never written: the activations and h start zeroed and stay so
        rp = self.rows_padded
        self.a = F.Mx8Packed.empty(rp, wl.H, rows_padded=rp, device=dev, zero=True)
        self.h = torch.zeros(rp, wl.I, dtype=torch.bfloat16, device=dev)
        self.hq = F.Mx8Packed.empty(rp, wl.I, device=dev)
        self.y = torch.empty(rp, wl.H, dtype=torch.bfloat16, device=dev)
        torch.cuda.synchronize()
        R.check_status(self.status)
        torch.cuda.empty_cache()

    def run(self, x=None, events=None):
        F = self.F
        ev = events or {}
        if "q0" in ev:
            ev["q0"].record()
        F.quantize_scatter(self.x if x is None else x, self.scatter, self.rows_padded, out=self.a, status=self.status)
        if "g0" in ev:
            ev["g0"].record()
        F.grouped_moe(self.a, self.offsets, self.wgu, swiglu=True, y=self.h, status=self.status,
                      expert_rows=self.expert_rows)
        if "q1" in ev:
            ev["q1"].record()
        F.quantize(self.h, out=self.hq, status=self.status)
        if "d0" in ev:
            ev["d0"].record()
        F.grouped_moe(self.hq, self.offsets, self.wdn, y=self.y, status=self.status, expert_rows=self.expert_rows)
        if "end" in ev:
            ev["end"].record()
        return self.y


class DenseStep:
    """Dense prefill projection: quantise X (+ residual) and the W4A4 + RAC GEMM, W pre-packed."""

    KERNELS_PER_STEP = 3  # amax, quantise X, GEMM

    def __init__(self, wl, dev):
        import torch

        from nvfp4_w4a4_moe_02_b200 import nvfp4rac as R

        self.R, self.torch, self.wl = R, torch, wl
        to = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to(dev).view(torch.bfloat16)
        self.status = R.new_status(dev)
        self.sel, _ = R.rac_calibrate(to(wl.x_cal), wl.Kp, status=self.status)
        self.w, self.ws = R.pack_weights(to(wl.w), self.sel, status=self.status)
        self.x = to(wl.x)
        self.a = R.Packed.empty(wl.M, wl.K, device=dev)
        self.ar = R.Packed.empty(wl.M, wl.Kp, rows_padded=self.a.rows_padded, device=dev)
        self.y = torch.empty(wl.M, wl.N, dtype=torch.bfloat16, device=dev)
        torch.cuda.synchronize()
        R.check_status(self.status)
        torch.cuda.empty_cache()

    def run(self, x=None, events=None):
        R = self.R
        ev = events or {}
        if "q0" in ev:
            ev["q0"].record()
        R.nvfp4_quantize(self.x if x is None else x, self.sel, out=self.a, out_res=self.ar, status=self.status)
        if "g0" in ev:
            ev["g0"].record()
        R.w4a4_rac_gemm(self.a, self.ar, self.w, self.ws, self.wl.M, y=self.y, status=self.status)
        if "end" in ev:
            ev["end"].record()
        return self.y


class DecodeStep:
    """MoE decode step: 64 tokens routed top-8 over 256 experts; each expert's tokens gathered into
    16-token slabs; swap-AB decode GEMMs stream the touched experts' packed weights."""

    KERNELS_PER_STEP = 5  # amax, quantise X, decode gate_up, quantise h, decode down

    def __init__(self, wl, dev):
        import torch

        from nvfp4_w4a4_moe_02_b200 import nvfp4rac as R
        from nvfp4_w4a4_moe_02_b200 import synthetic as syn

        self.R, self.torch, self.wl = R, torch, wl
        to = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to(dev).view(torch.bfloat16)
        self.status = R.new_status(dev)
        # offline: channel selection, then the pack of every expert (weights made on the device)
        self.sel_gu, _ = R.rac_calibrate(to(wl.x_cal), wl.Kp_gu, status=self.status)
        h_cal = syn.moe_down_calibration_batch_torch(wl, dev)
        self.sel_dn, _ = R.rac_calibrate(to(h_cal), wl.Kp_dn, status=self.status)
        N_gu = 2 * wl.I
        P = R.Packed
        self.pgu = P.empty(N_gu, wl.H, slabs=wl.E, rows_padded=N_gu, device=dev)
        self.pgus = P.empty(N_gu, wl.Kp_gu, slabs=wl.E, rows_padded=N_gu, device=dev)
        self.pdn = P.empty(wl.H, wl.I, slabs=wl.E, rows_padded=wl.H, device=dev)
        self.pdns = P.empty(wl.H, wl.Kp_dn, slabs=wl.E, rows_padded=wl.H, device=dev)
        wbuf = torch.empty(N_gu, wl.H, dtype=torch.bfloat16, device=dev)
        dbuf = torch.empty(wl.H, wl.I, dtype=torch.bfloat16, device=dev)
        for e in range(wl.E):
            R.pack_weights(wl.gate_up_expert_torch(e, dev, out=wbuf), self.sel_gu, gate_up_interleave=True,
                           out=self.pgu.slab(e), out_sel=self.pgus.slab(e), status=self.status)
            R.pack_weights(wl.down_expert_torch(e, dev, out=dbuf), self.sel_dn, out=self.pdn.slab(e),
                           out_sel=self.pdns.slab(e), status=self.status)
        del wbuf, dbuf
        # 16-token expert slabs from the device plan (worst-case slot table; the decode GEMM skips
        # the unused slots, the h quantiser takes the used rows of each slot only)
        lay = device_layout(R, wl, dev, 16, self.status, decode=True)
        self.n_slots = lay["n_slots"]
        self.slots_used = lay["slots_used"]
        self.rows = 16 * self.n_slots
        self.slot_expert, self.slot_count = lay["slot_expert"], lay["slot_count"]
        self.slot_first_row = lay["slot_first_row"]
        self.scatter = lay["row_scatter"]
        self.pair_rows = lay["pair_rows"]
        self.x = to(wl.x)
        S16 = R.SF_SLAB16
        # rows of a slab past its count are never named by the scatter map: zero them once
        self.a = P.empty(self.rows, wl.H, rows_padded=self.rows, device=dev, zero=True, sf_layout=S16)
        self.ar = P.empty(self.rows, wl.Kp_gu, rows_padded=self.rows, device=dev, zero=True, sf_layout=S16)
        self.h = torch.zeros(self.rows, wl.I, dtype=torch.bfloat16, device=dev)
        self.amax_h = torch.zeros(1, dtype=torch.float32, device=dev)
        self.hq = P.empty(self.rows, wl.I, rows_padded=self.rows, device=dev, sf_layout=S16, zero=True)
        self.hqr = P.empty(self.rows, wl.Kp_dn, rows_padded=self.rows, device=dev, sf_layout=S16, zero=True)
        self.y = torch.empty(self.rows, wl.H, dtype=torch.bfloat16, device=dev)
        torch.cuda.synchronize()
        R.check_status(self.status)
        torch.cuda.empty_cache()

    def run(self, x=None, events=None):
        R = self.R
        ev = events or {}
        if "q0" in ev:
            ev["q0"].record()
        R.nvfp4_quantize_scatter(self.x if x is None else x, self.scatter, self.rows, self.sel_gu, out=self.a,
                                 out_res=self.ar, status=self.status)
        if "g0" in ev:
            ev["g0"].record()
        R.grouped_w4a4_rac_moe_decode(self.a, self.ar, self.slot_expert, self.slot_count, self.pgu, self.pgus,
                                      swiglu=True, y=self.h, amax_out=self.amax_h, status=self.status)
        if "q1" in ev:
            ev["q1"].record()
        # the token rows of each slot only (slot s: rows 16 s .. 16 s + slot_count[s] - 1)
        R.nvfp4_quantize_segments(self.h, self.slot_first_row, self.slot_count, self.sel_dn, amax_in=self.amax_h,
                                  out=self.hq, out_res=self.hqr, status=self.status)
        if "d0" in ev:
            ev["d0"].record()
        R.grouped_w4a4_rac_moe_decode(self.hq, self.hqr, self.slot_expert, self.slot_count, self.pdn, self.pdns,
                                      y=self.y, status=self.status)
        if "end" in ev:
            ev["end"].record()
        return self.y


class MoEBlockStep:
    """A whole MoE layer on the device, nothing on the host per step: router top-k of the logits,
    dispatch plan, quantise-scatter of X, gate_up (SwiGLU + amax), quantise h, down, weighted
    combine into [T, H].  Prefill uses 128-row expert segments and the grouped GEMM; decode uses
    16-token slabs (worst-case slot count, unused slots skipped) and the swap-AB GEMM."""

    # router, count, offsets, rank, amax, quantise X, gate_up, quantise h, down, combine; prefill with
    # the combine in the down GEMM's epilogue: + row pairs, the combine kernel becomes the bf16 finalise
    KERNELS_PER_STEP = 10

    def __init__(self, wl, packed, sel_gu, sel_dn, decode, dev, fused_combine=False):
        import torch

        from nvfp4_w4a4_moe_02_b200 import nvfp4rac as R
        from nvfp4_w4a4_moe_02_b200 import synthetic as syn

        self.R, self.torch, self.wl, self.decode = R, torch, wl, decode
        self.status = R.new_status(dev)
        self.sel_gu, self.sel_dn = sel_gu, sel_dn
        self.pgu, self.pgus, self.pdn, self.pdns = packed
        T, k = wl.topk_ids.shape
        self.T, self.k = T, k
        self.pad = 16 if decode else 128
        self.cap = R.moe_rows_capacity(T, k, wl.E, self.pad)
        self.n_slots = self.cap // 16 if decode else None
        self.logits_np = syn.normal_f64(wl.seed, syn.STREAM_ROUTER, T * wl.E).reshape(T, wl.E).astype(np.float32)
        self.logits = torch.from_numpy(self.logits_np).to(dev)
        self.x = torch.from_numpy(np.ascontiguousarray(wl.x).view(np.int16)).to(dev).view(torch.bfloat16)
        P = R.Packed
        lay = R.SF_SLAB16 if decode else R.SF_ATOM128
        self.ids = torch.empty(T, k, dtype=torch.int32, device=dev)
        self.w = torch.empty(T, k, dtype=torch.float32, device=dev)
        self.off = torch.empty(wl.E + 1, dtype=torch.int32, device=dev)
        self.rows = torch.empty(T, k, dtype=torch.int32, device=dev)
        self.expert_rows = torch.empty(wl.E, dtype=torch.int32, device=dev)
        self.se = torch.empty(self.n_slots, dtype=torch.int32, device=dev) if decode else None
        self.sc = torch.empty(self.n_slots, dtype=torch.int32, device=dev) if decode else None
        self.a = P.empty(self.cap, wl.H, rows_padded=self.cap, device=dev, zero=True, sf_layout=lay)
        self.ar = P.empty(self.cap, wl.Kp_gu, rows_padded=self.cap, device=dev, zero=True, sf_layout=lay)
        self.h = torch.zeros(self.cap, wl.I, dtype=torch.bfloat16, device=dev)
        self.amax_h = torch.zeros(1, dtype=torch.float32, device=dev)
        self.hq = P.empty(self.cap, wl.I, rows_padded=self.cap, device=dev, sf_layout=lay, zero=True)
        self.hqr = P.empty(self.cap, wl.Kp_dn, rows_padded=self.cap, device=dev, sf_layout=lay, zero=True)
        self.slot_first_row = torch.arange(self.n_slots, dtype=torch.int32, device=dev) * 16 if decode else None
        # the combine in the down GEMM's epilogue (atomic binary32 adds) measured slower than the
        # bf16 rows + combine kernel on the prefill block; kept as an option
        self.fused_combine = fused_combine and not decode
        self.kernels_per_step = self.KERNELS_PER_STEP + (1 if self.fused_combine else 0)
        if self.fused_combine:
            self.row_pair = torch.empty(self.cap, dtype=torch.int32, device=dev)
            self.y32 = torch.empty(T, wl.H, dtype=torch.float32, device=dev)
        else:
            self.ye = torch.zeros(self.cap, wl.H, dtype=torch.bfloat16, device=dev)
        self.y = torch.empty(T, wl.H, dtype=torch.bfloat16, device=dev)
        torch.cuda.synchronize()

    # run() takes an output buffer: the end-to-end loop pipelines steps over two of them
    takes_out = True

    def run(self, x=None, logits=None, events=None, out=None):
        R = self.R
        ev = events or {}
        y_out = self.y if out is None else out
        if "r0" in ev:
            ev["r0"].record()
        R.moe_route_topk(self.logits if logits is None else logits, self.k, ids=self.ids, w=self.w,
                         status=self.status)
        R.moe_dispatch_plan(self.ids, self.wl.E, self.pad, rows_capacity=self.cap, n_slots=self.n_slots,
                            offsets=self.off, row_scatter=self.rows, slot_expert=self.se, slot_count=self.sc,
                            status=self.status, expert_rows=self.expert_rows)
        if self.fused_combine:
            R.moe_row_pairs(self.rows, self.cap, row_pair=self.row_pair, status=self.status)
        if "q0" in ev:
            ev["q0"].record()
        R.nvfp4_quantize_scatter(self.x if x is None else x, self.rows, self.cap, self.sel_gu, out=self.a,
                                 out_res=self.ar, status=self.status)
        if "g0" in ev:
            ev["g0"].record()
        if self.decode:
            R.grouped_w4a4_rac_moe_decode(self.a, self.ar, self.se, self.sc, self.pgu, self.pgus, swiglu=True,
                                          y=self.h, amax_out=self.amax_h, status=self.status)
        else:
            R.grouped_w4a4_rac_moe(self.a, self.ar, self.off, self.pgu, self.pgus, swiglu=True, y=self.h,
                                   amax_out=self.amax_h, status=self.status, expert_rows=self.expert_rows)
        if "q1" in ev:
            ev["q1"].record()
        # the token rows only: each expert segment's (prefill) or each slot's (decode)
        seg_first, seg_rows = (self.slot_first_row, self.sc) if self.decode else (self.off, self.expert_rows)
        R.nvfp4_quantize_segments(self.h, seg_first, seg_rows, self.sel_dn, amax_in=self.amax_h, out=self.hq,
                                  out_res=self.hqr, status=self.status)
        if "d0" in ev:
            ev["d0"].record()
        if self.fused_combine:
            # down projection with the weighted combine in its epilogue, then the bf16 rows
            R.grouped_w4a4_rac_moe_combine(self.hq, self.hqr, self.off, self.pdn, self.pdns, self.row_pair, self.w,
                                           out=y_out, out32=self.y32, status=self.status,
                                           expert_rows=self.expert_rows)
            if "c0" in ev:
                ev["c0"].record()
        else:
            if self.decode:
                R.grouped_w4a4_rac_moe_decode(self.hq, self.hqr, self.se, self.sc, self.pdn, self.pdns, y=self.ye,
                                              status=self.status)
            else:
                R.grouped_w4a4_rac_moe(self.hq, self.hqr, self.off, self.pdn, self.pdns, y=self.ye,
                                       status=self.status, expert_rows=self.expert_rows)
            if "c0" in ev:
                ev["c0"].record()
            R.moe_combine(self.ye, self.rows, self.w, out=y_out, status=self.status)
        if "end" in ev:
            ev["end"].record()
        return y_out


class QdqStep:
    """Trainer-side fake quantisation of a set of weight tensors: one weight_qdq call."""

    def __init__(self, w_np, dev):
        import torch

        from nvfp4_w4a4_moe_02_b200 import nvfp4rac as R

        self.R, self.torch = R, torch
        self.status = R.new_status(dev)
        self.n_tensors, self.elems = w_np.shape
        self.x = torch.from_numpy(w_np.view(np.int16)).to(dev).view(torch.bfloat16)
        self.y = torch.empty_like(self.x)
        self.s_g = torch.empty(self.n_tensors, dtype=torch.float32, device=dev)
        # tensors of up to 4M elements: one kernel (the one-pass form); larger: amax, then qdq
        self.kernels_per_step = 1 if self.elems <= (4 << 20) else 2

    def run(self, x=None, events=None):
        ev = events or {}
        if "q0" in ev:
            ev["q0"].record()
        self.R.weight_qdq(self.x if x is None else x, out=self.y, s_g=self.s_g, status=self.status)
        if "end" in ev:
            ev["end"].record()
        return self.y


# ------------------------------------------------------------------------------------------ clocks
class ClockSampler:
    """nvidia-smi clock / throttle-reason samples every 50 ms; samples are kept for the wall-clock
    window of the timed region (if the region is shorter than the sampling period, the samples
    closest to it are used)."""
    FIELDS = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = os.path.join("/tmp", f"bench_clocks_{os.getpid()}.csv")

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "50"],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def wait_first_sample(self, timeout=5.0):
        t0 = time.time()
        while self.proc is not None and time.time() - t0 < timeout:
            if os.path.exists(self.path) and os.path.getsize(self.path) > 0:
                return
            time.sleep(0.05)

    def stop(self, t0=None, t1=None):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.1)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        import datetime

        rows = []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                ts = datetime.datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                rows.append((ts, float(parts[1]), float(parts[2]), parts[5:9]))
            except ValueError:
                continue
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        if t0 is not None:
            inside = [r for r in rows if t0 - 0.05 <= r[0] <= t1 + 0.05]
            if not inside:  # region shorter than the sampling period: the nearest samples
                inside = sorted(rows, key=lambda r: min(abs(r[0] - t0), abs(r[0] - t1)))[:2]
            rows = inside
        reasons = sorted({n for r in rows for n, v in zip(names, r[3]) if v.lower() == "active"})
        return {"sm_mhz": float(np.median([r[1] for r in rows])), "sm_max_mhz": max(r[2] for r in rows),
                "reasons": reasons, "samples": len(rows)}


# ------------------------------------------------------------------------------------------ CPU oracle leg
def oracle_pack(wl, sel_gu, sel_dn, experts):
    """The oracle's packed weights of the given experts (the rollout's once-per-sync weight pack,
    kept out of the timed step like the GPU path's)."""
    import oracle as orc

    packed = {}
    for e in experts:
        e = int(e)
        wgu, wdn = wl.gate_up_expert(e), wl.down_expert(e)
        s_gu = orc.global_scale(orc.amax_bf16(wgu))
        s_dn = orc.global_scale(orc.amax_bf16(wdn))
        packed[e] = (s_gu, orc.weight_pack(wgu, s_gu, sel_gu), s_dn, orc.weight_pack(wdn, s_dn, sel_dn))
    return packed


def sample_pairs(wl, n_pairs, seed):
    rng = np.random.default_rng(seed)
    return np.sort(rng.choice(wl.pair_token.size, n_pairs, replace=False))


def oracle_sample(wl, sel_gu, sel_dn, n_pairs, seed=0, packed=None):
    """The oracle on a bounded sample of the step: n_pairs (token, expert) rows through quantise,
    gate_up, SwiGLU, quantise, down, with the experts' weights packed beforehand (outside the
    timing, as on the GPU).  Returns (seconds, flops of the sample)."""
    import oracle as orc

    pairs = sample_pairs(wl, n_pairs, seed)
    if packed is None:
        packed = oracle_pack(wl, sel_gu, sel_dn, np.unique(wl.pair_expert[pairs]))
    t0 = time.perf_counter()
    s_x = orc.global_scale(orc.amax_bf16(wl.x))
    h_rows, exps = [], []
    for e in np.unique(wl.pair_expert[pairs]):
        idx = pairs[wl.pair_expert[pairs] == e]
        xa = wl.x[wl.pair_token[idx]]
        ac, aS, rc, rS, _ = orc.act_quant_rac(xa, s_x, sel_gu)
        s_w, (wc, wS, wsc, wsS), _, _ = packed[int(e)]
        gu, _ = orc.gemm_rac(ac, aS, rc, rS, wc, wS, wsc, wsS, s_x, s_w)
        gu_b = orc.f64_to_bf16_array(gu)
        h, _ = orc.swiglu(gu_b)
        h_rows.append(h)
        exps.append((e, h.shape[0]))
    hh = np.concatenate(h_rows)
    s_h = orc.global_scale(orc.amax_bf16(hh))
    start = 0
    for e, n in exps:
        hc, hS, hrc, hrS, _ = orc.act_quant_rac(hh[start:start + n], s_h, sel_dn)
        _, _, s_w, (dc, dS, dsc, dsS) = packed[int(e)]
        orc.gemm_rac(hc, hS, hrc, hrS, dc, dS, dsc, dsS, s_h, s_w)
        start += n
    dt = time.perf_counter() - t0
    gu_f, dn_f = flops_of(wl, len(sel_gu), len(sel_dn))
    frac = n_pairs / wl.pair_token.size
    return dt, (gu_f + dn_f) * frac


def run_reference(args):
    """The reference arm: the CPU oracle as it stands, on the same metric and workload."""
    ws, rank, local = dist_env()
    if rank != 0:
        return 0
    import oracle as orc

    orc.build()
    wl, h_cal = build_inputs()
    sel_gu, _ = orc.calibrate(wl.x_cal, wl.Kp_gu)
    sel_dn, _ = orc.calibrate(h_cal, wl.Kp_dn)
    n_pairs = args.ref_pairs
    # the weight pack happens once per trainer -> rollout sync, outside the steps (as on the GPU)
    packed = oracle_pack(wl, sel_gu, sel_dn, np.unique(np.concatenate(
        [wl.pair_expert[sample_pairs(wl, n, i)] for i, n in [(0, max(8, n_pairs // 8))] +
         [(i, n_pairs) for i in range(args.steps)]])))
    for _ in range(args.warmup):
        oracle_sample(wl, sel_gu, sel_dn, max(8, n_pairs // 8), packed=packed)
    times, flops = [], 0.0
    for i in range(args.steps):
        dt, f = oracle_sample(wl, sel_gu, sel_dn, n_pairs, seed=i, packed=packed)
        times.append(dt)
        flops += f
    total = sum(times)
    value = flops / total / 1e12
    cores = orc.num_threads()
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int64-exact GEMM, f32 quant",
            "data": "synthetic (seeded)",
            "config": {"workload": wl.name + f"_r{wl.r}", "sample_pairs_per_step": n_pairs},
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                             "sample": f"{n_pairs} of {wl.pair_token.size} (token, expert) rows per step, "
                                       "weights packed before the timed steps"},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------------------------------ main
def spec_moe(dev, args, peaks):
    wl, h_cal = build_inputs(experts=args.experts)
    step = MoEStep(wl, h_cal, dev)
    gu_f, dn_f = flops_of(wl, wl.Kp_gu, wl.Kp_dn)
    P = int(wl.pair_token.size)
    gu_bytes = (wl.E * 2 * wl.I * (wl.H + wl.Kp_gu) * 0.5625 + P * (wl.H + wl.Kp_gu) * 0.5625 + P * wl.I * 2.0)

    def cpu_leg():
        import oracle as orc

        orc.build()
        sg, sd = step.sel_gu.cpu().numpy(), step.sel_dn.cpu().numpy()
        packed = oracle_pack(wl, sg, sd, np.unique(wl.pair_expert[sample_pairs(wl, args.cpu_pairs, 0)]))
        dt, f = oracle_sample(wl, sg, sd, args.cpu_pairs, packed=packed)
        return {"value": f / dt / 1e12, "unit": "TFLOP/s", "cores": orc.num_threads(), "kind": "oracle",
                "sample": f"{args.cpu_pairs} of {P} (token, expert) rows of one step, weights packed beforehand "
                          f"(outside the timing), {dt:.1f} s"}

    # end to end: the whole layer through the public API (router top-k of the logits, dispatch
    # plan, quantise, both GEMMs, weighted combine into [T, H]) with X and the logits copied in
    # and the [T, H] output copied out every step
    e2e_step = MoEBlockStep(wl, (step.pgu, step.pgus, step.pdn, step.pdns), step.sel_gu, step.sel_dn, False, dev)

    return dict(
        step=step, x_np=wl.x, flops=gu_f + dn_f, events=["q0", "g0", "q1", "d0", "end"],
        e2e_step=e2e_step, e2e_extra_h2d={"logits": e2e_step.logits_np},
        segments={"quant_x": ("q0", "g0"), "gate_up": ("g0", "q1"), "quant_h": ("q1", "d0"), "down": ("d0", "end")},
        dominant=("gate_up", gu_f, gu_bytes, "grouped gate_up W4A4+RAC GEMM (SwiGLU epilogue)"),
        # DRAM bytes read + written by one gate_up launch at this workload (one-pass ncu capture of
        # dram__bytes_read.sum + dram__bytes_write.sum of the kernel as it is: 410.4 + 46.6 MB)
        traffic=456994304.0,
        quant={"x": ("quant_x", int(wl.x.nbytes) + P * 0.5625 * (wl.H + wl.Kp_gu)),  # X read once, 8 copies out
               "h": ("quant_h", quant_bytes(P, wl.I, wl.Kp_dn))},
        config={"workload": wl.name + f"_r{wl.r}", "tokens": int(wl.x.shape[0]), "pairs": P, "experts": wl.E,
                "hidden": wl.H, "intermediate": wl.I, "Kp_gate_up": wl.Kp_gu, "Kp_down": wl.Kp_dn,
                "rows_padded": step.rows_padded},
        cpu=cpu_leg, kernels_per_step=MoEStep.KERNELS_PER_STEP)


def oracle_sample_fp8(wl, n_pairs, seed=0):
    """The oracle on a bounded sample of the FP8 comparison step: n_pairs (token, expert) rows
    through FP8 quantise, gate_up, SwiGLU, FP8 quantise, down.  Returns (seconds, flops)."""
    import oracle as orc

    rng = np.random.default_rng(seed)
    pairs = np.sort(rng.choice(wl.pair_token.size, n_pairs, replace=False))
    t0 = time.perf_counter()
    for e in np.unique(wl.pair_expert[pairs]):
        idx = pairs[wl.pair_expert[pairs] == e]
        ac, aS = orc.mx8_quantize(wl.x[wl.pair_token[idx]])
        wc, wS = orc.mx8_quantize(wl.gate_up_expert(int(e)))
        gu, _ = orc.mx8_gemm(ac, aS, wc, wS)
        h, _ = orc.swiglu(orc.f64_to_bf16_array(gu))
        hc, hS = orc.mx8_quantize(h)
        dc, dS = orc.mx8_quantize(wl.down_expert(int(e)))
        orc.mx8_gemm(hc, hS, dc, dS)
    dt = time.perf_counter() - t0
    return dt, sum(flops_of(wl, 0, 0)) * n_pairs / wl.pair_token.size


def spec_fp8_moe(dev, args, peaks):
    """The MoE prefill block on the FP8 comparison format (E4M3, power-of-two scale per 32)."""
    wl, _ = build_inputs(experts=args.experts)
    step = Mx8MoEStep(wl, dev)
    gu_f, dn_f = flops_of(wl, 0, 0)
    P = int(wl.pair_token.size)
    b8 = 1.0 + 1.0 / 32  # bytes per FP8 element with its scale
    gu_bytes = wl.E * 2 * wl.I * wl.H * b8 + P * wl.H * b8 + P * wl.I * 2.0

    def cpu_leg():
        import oracle as orc

        orc.build()
        dt, f = oracle_sample_fp8(wl, args.cpu_pairs)
        return {"value": f / dt / 1e12, "unit": "TFLOP/s", "cores": orc.num_threads(), "kind": "oracle",
                "sample": f"{args.cpu_pairs} of {P} (token, expert) rows of one step, {dt:.1f} s"}

    return dict(
        step=step, x_np=wl.x, flops=gu_f + dn_f, events=["q0", "g0", "q1", "d0", "end"],
        segments={"quant_x": ("q0", "g0"), "gate_up": ("g0", "q1"), "quant_h": ("q1", "d0"), "down": ("d0", "end")},
        dominant=("gate_up", gu_f, gu_bytes, "grouped gate_up FP8 GEMM (SwiGLU epilogue)"),
        traffic=None,
        quant={"x": ("quant_x", int(wl.x.nbytes) + P * b8 * wl.H), "h": ("quant_h", P * (2.0 + b8) * wl.I)},
        config={"workload": wl.name.replace(f"_r{wl.r}", "") + "_fp8_e4m3_pow2_per32", "tokens": int(wl.x.shape[0]),
                "pairs": P, "experts": wl.E, "hidden": wl.H, "intermediate": wl.I, "rows_padded": step.rows_padded},
        cpu=cpu_leg, kernels_per_step=Mx8MoEStep.KERNELS_PER_STEP,
        dtype="fp8 (e4m3 x e4m3, e8m0 power-of-two scale per 32) -> f32 accumulate")


def spec_dense(dev, args, peaks):
    from nvfp4_w4a4_moe_02_b200 import synthetic as syn

    wl = syn.dense_prefill()
    step = DenseStep(wl, dev)
    flops = 2.0 * wl.M * wl.N * (wl.K + wl.Kp)
    gbytes = 0.5625 * (wl.M + wl.N) * (wl.K + wl.Kp) + 2.0 * wl.M * wl.N

    def cpu_leg():
        import oracle as orc

        orc.build()
        rows = np.arange(0, wl.M, wl.M // max(1, args.cpu_rows))[:args.cpu_rows]
        t0 = time.perf_counter()
        orc.dense_rac_forward(wl.x, wl.w, step.sel.cpu().numpy(), rows=rows)
        dt = time.perf_counter() - t0
        f = 2.0 * rows.size * wl.N * (wl.K + wl.Kp)
        return {"value": f / dt / 1e12, "unit": "TFLOP/s", "cores": orc.num_threads(), "kind": "oracle",
                "sample": f"{rows.size} of {wl.M} output rows (full quantisation of X and W included), {dt:.1f} s"}

    return dict(
        step=step, x_np=wl.x, flops=flops, events=["q0", "g0", "end"],
        segments={"quant_x": ("q0", "g0"), "gemm": ("g0", "end")},
        dominant=("gemm", flops, gbytes, "dense W4A4+RAC GEMM"),
        quant={"x": ("quant_x", quant_bytes(wl.M, wl.K, wl.Kp))},
        config={"workload": wl.name + f"_r{wl.r}", "M": wl.M, "N": wl.N, "K": wl.K, "Kp": wl.Kp},
        cpu=cpu_leg, kernels_per_step=DenseStep.KERNELS_PER_STEP)


def spec_decode(dev, args, peaks):
    from nvfp4_w4a4_moe_02_b200 import synthetic as syn

    wl = syn.moe_decode() if args.experts is None else \
        syn.moe_block(0, 0.5, T=64, H=7168, E=args.experts, topk=8, I=2048, materialize_weights=False)
    step = DecodeStep(wl, dev)
    gu_f, dn_f = flops_of(wl, wl.Kp_gu, wl.Kp_dn)
    P = int(wl.pair_token.size)
    touched = int((wl.counts > 0).sum())
    # algorithmic bytes: each touched expert's packed W + W_sel once, the slab activations once,
    # the output once
    gu_w = touched * 2 * wl.I * (wl.H + wl.Kp_gu) * 0.5625
    dn_w = touched * wl.H * (wl.I + wl.Kp_dn) * 0.5625
    gu_bytes = gu_w + step.rows * (wl.H + wl.Kp_gu) * 0.5625 + step.rows * wl.I * 2.0
    dn_bytes = dn_w + step.rows * (wl.I + wl.Kp_dn) * 0.5625 + step.rows * wl.H * 2.0
    n_cpu = max(2, args.cpu_pairs // 32)

    def cpu_leg():
        import oracle as orc

        orc.build()
        dt, f = oracle_sample(wl, step.sel_gu.cpu().numpy(), step.sel_dn.cpu().numpy(), n_cpu)
        return {"value": f / dt / 1e12, "unit": "TFLOP/s", "cores": orc.num_threads(), "kind": "oracle",
                "sample": f"{n_cpu} of {P} (token, expert) rows of one step (their experts' weights packed by the "
                          f"oracle), {dt:.1f} s"}

    return dict(
        step=step, x_np=wl.x, flops=gu_f + dn_f, events=["q0", "g0", "q1", "d0", "end"],
        segments={"quant_x": ("q0", "g0"), "gate_up": ("g0", "q1"), "quant_h": ("q1", "d0"), "down": ("d0", "end")},
        dominant=("gate_up", gu_f, gu_bytes, "decode gate_up W4A4+RAC GEMM (swap-AB, SwiGLU epilogue)"),
        quant={"x": ("quant_x", int(wl.x.nbytes) + P * 0.5625 * (wl.H + wl.Kp_gu)),
               "h": ("quant_h", quant_bytes(step.rows, wl.I, wl.Kp_dn))},
        extra_gbs={"gate_up": ("gate_up", gu_bytes), "down": ("down", dn_bytes),
                   "weights_step": (None, gu_w + dn_w)},
        config={"workload": wl.name + f"_r{wl.r}", "tokens": int(wl.x.shape[0]), "pairs": P, "experts": wl.E,
                "touched_experts": touched, "slabs": step.slots_used, "slot_table": step.n_slots, "hidden": wl.H,
                "intermediate": wl.I,
                "Kp_gate_up": wl.Kp_gu, "Kp_down": wl.Kp_dn, "weight_bytes_touched": gu_w + dn_w},
        cpu=cpu_leg, kernels_per_step=DecodeStep.KERNELS_PER_STEP)


def _spec_block(dev, args, decode):
    if decode:
        from nvfp4_w4a4_moe_02_b200 import synthetic as syn

        wl = syn.moe_decode() if args.experts is None else \
            syn.moe_block(0, 0.5, T=64, H=7168, E=args.experts, topk=8, I=2048, materialize_weights=False)
        inner = DecodeStep(wl, dev)
    else:
        wl, h_cal = build_inputs(experts=args.experts)
        inner = MoEStep(wl, h_cal, dev)
    step = MoEBlockStep(wl, (inner.pgu, inner.pgus, inner.pdn, inner.pdns), inner.sel_gu, inner.sel_dn, decode, dev,
                        fused_combine=bool(getattr(args, "fused_combine", False)))
    # the device router must reproduce the workload's routing (same logits, same reading)
    step.run()
    import torch

    torch.cuda.synchronize()
    step.R.check_status(step.status)
    gu_f, dn_f = flops_of(wl, wl.Kp_gu, wl.Kp_dn)
    T = wl.x.shape[0]
    P = int(wl.pair_token.size)
    n_w = int((wl.counts > 0).sum()) if decode else wl.E  # experts whose weights the step reads
    rows = step.cap if decode else P
    gu_bytes = n_w * 2 * wl.I * (wl.H + wl.Kp_gu) * 0.5625 + rows * (wl.H + wl.Kp_gu) * 0.5625 + rows * wl.I * 2.0
    name = wl.name + f"_r{wl.r}_layer"
    return dict(
        step=step, x_np=wl.x, extra_h2d={"logits": step.logits_np}, flops=gu_f + dn_f,
        events=["r0", "q0", "g0", "q1", "d0", "c0", "end"],
        segments={"route_plan": ("r0", "q0"), "quant_x": ("q0", "g0"), "gate_up": ("g0", "q1"),
                  "quant_h": ("q1", "d0"), "down": ("d0", "c0"), "combine": ("c0", "end")},
        dominant=("gate_up", gu_f, gu_bytes, "gate_up W4A4+RAC GEMM of the layer (SwiGLU epilogue)"),
        quant={}, config={"workload": name, "tokens": T, "experts": wl.E, "hidden": wl.H, "intermediate": wl.I,
                          "plan": "device (router top-k, dispatch plan); combine into [T, H]",
                          "combine": "in the down GEMM's epilogue" if step.fused_combine else "combine kernel",
                          "rows_capacity": step.cap},
        cpu=lambda: None, kernels_per_step=step.kernels_per_step)


def spec_block_prefill(dev, args, peaks):
    return _spec_block(dev, args, False)


def spec_block_decode(dev, args, peaks):
    return _spec_block(dev, args, True)


def _spec_qdq(dev, args, n_tensors, elems=1 << 31):
    from nvfp4_w4a4_moe_02_b200 import synthetic as syn

    w = syn.trainer_weights(n_tensors=n_tensors, elems=elems)
    step = QdqStep(w, dev)
    n = w.size
    label = f"weight_qdq_{n_tensors}x{w.shape[1]}"

    def cpu_leg():
        import oracle as orc

        orc.build()
        k = max(1, min(n_tensors, 64))
        rows = w.reshape(n_tensors, -1)[:k] if n_tensors > 1 else w.reshape(-1)[:k << 21].reshape(1, -1)
        t0 = time.perf_counter()
        for r in rows:
            orc.weight_qdq(r)  # amax of the tensor, then the fake-quant
        dt = time.perf_counter() - t0
        return {"value": 4.0 * rows.size / dt / 1e9, "unit": "GB/s", "cores": orc.num_threads(), "kind": "oracle",
                "sample": f"{rows.shape[0]} tensors of {rows.shape[1]} elements (amax + QDQ), {dt:.1f} s"}

    # a tensor that fits on chip is read once and written once (4 B per element); one larger than
    # L2 must be read twice, since its scale depends on every element before any can be quantised
    fits = step.kernels_per_step == 1
    d_bytes = (4.0 if fits else 6.0) * n
    d_label = ("weight_qdq (amax + fake-quant in one pass, 4 B/element algorithmic: one read, one write)" if fits
               else "weight_qdq (amax pass + fake-quant pass, 6 B/element algorithmic: two reads, one write)")
    return dict(
        step=step, x_np=w, flops=0.0, work=4.0 * n, unit="GB/s", dtype="bf16 -> nvfp4 -> bf16 (f32 arithmetic)",
        events=["q0", "end"], segments={"qdq": ("q0", "end")},
        dominant=("qdq", 0.0, d_bytes, d_label), quant={},
        config={"workload": label, "tensors": n_tensors, "elements": int(n), "distribution": "N(0, 0.02)"},
        cpu=cpu_leg, kernels_per_step=step.kernels_per_step)


def spec_qdq(dev, args, peaks):
    # tensors of 1024 x 2048 elements (1024 of them: 2^31 elements)
    return _spec_qdq(dev, args, args.qdq_tensors, args.qdq_tensors << 21)


def spec_qdq_single(dev, args, peaks):
    return _spec_qdq(dev, args, 1)


SPECS = {"moe_prefill": spec_moe, "fp8_moe_prefill": spec_fp8_moe, "dense": spec_dense, "moe_decode": spec_decode,
         "qdq": spec_qdq,
         "qdq_single": spec_qdq_single, "moe_prefill_layer": spec_block_prefill,
         "moe_decode_layer": spec_block_decode}


def at_r(rows, r):
    return next(x for x in rows if x["r"] == r)


def run_sweep(args):
    """RAC ratio sweep on the MoE prefill shapes: r in {0, 0.25, 0.5, 1}; per r the step's
    TFLOP/s and the error of h (SwiGLU output) and y (down output) against the binary64 product
    of the bf16 inputs on sampled (token, expert) rows."""
    import dataclasses

    import torch

    from nvfp4_w4a4_moe_02_b200 import nvfp4rac as R
    from nvfp4_w4a4_moe_02_b200 import synthetic as syn

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    R.load()
    base, h_cal = build_inputs(experts=args.experts)
    rng = np.random.default_rng(0)
    P = int(base.pair_token.size)
    sample = np.sort(rng.choice(P, 256, replace=False))
    I = base.I
    # binary64 reference of the sampled rows from the bf16 inputs
    f64 = lambda a: syn.bf16_to_f32(a).astype(np.float64)
    h_ref, y_ref = [], []
    for i in sample:
        e, t = int(base.pair_expert[i]), int(base.pair_token[i])
        gu = f64(base.x[t]) @ f64(base.wgu[e]).T
        h = gu[:I] / (1.0 + np.exp(-gu[:I])) * gu[I:]
        h_ref.append(h)
        y_ref.append(h @ f64(base.wdn[e]).T)
    h_ref, y_ref = np.array(h_ref), np.array(y_ref)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    err = lambda a, b: (float(np.linalg.norm(a - b) / np.linalg.norm(b)), float(np.mean(np.abs(a - b))))

    def measure(step):
        """mean step time (ms) and the errors of h and y on the sampled rows"""
        for _ in range(max(3, args.warmup)):
            flush.zero_()
            step.run()
        evs = [{n: torch.cuda.Event(enable_timing=True) for n in ("q0", "g0", "q1", "d0", "end")}
               for _ in range(args.steps)]
        for i in range(args.steps):
            flush.zero_()
            step.run(events=evs[i])
        torch.cuda.synchronize()
        R.check_status(step.status)
        ms = float(np.mean([e["q0"].elapsed_time(e["end"]) for e in evs]))
        seg = {"quant_x": ("q0", "g0"), "gate_up": ("g0", "q1"), "quant_h": ("q1", "d0"), "down": ("d0", "end")}
        kernel_ms = {k: float(np.mean([e[a].elapsed_time(e[b]) for e in evs])) for k, (a, b) in seg.items()}
        prow = torch.from_numpy(step.pair_rows[sample]).to(dev)
        (hf, hm), (yf, ym) = err(step.h[prow].double().cpu().numpy(), h_ref), err(step.y[prow].double().cpu().numpy(),
                                                                                  y_ref)
        return ms, {"h_rel_fro": hf, "h_mean_abs": hm, "y_rel_fro": yf, "y_mean_abs": ym, "kernel_ms": kernel_ms}

    rows = []
    for r in (0.0, 0.25, 0.5, 1.0):
        wl = dataclasses.replace(base, r=r, Kp_gu=syn.kp_from_ratio(base.H, r), Kp_dn=syn.kp_from_ratio(base.I, r))
        step = MoEStep(wl, h_cal, dev)
        ms, e = measure(step)
        gu_f, dn_f = flops_of(wl, wl.Kp_gu, wl.Kp_dn)
        plain_f = sum(flops_of(wl, 0, 0))
        rows.append({"r": r, "Kp_gate_up": wl.Kp_gu, "Kp_down": wl.Kp_dn, "ms_per_step": ms,
                     "tflops": (gu_f + dn_f) / (ms * 1e-3) / 1e12,
                     "tflops_plain_w4a4_equivalent": plain_f / (ms * 1e-3) / 1e12, **e})
        del step
        torch.cuda.empty_cache()
    wl = dataclasses.replace(base, r=0.5, Kp_gu=syn.kp_from_ratio(base.H, 0.5), Kp_dn=syn.kp_from_ratio(base.I, 0.5))
    plain_f = sum(flops_of(wl, 0, 0))
    # the masked full-K residual variant at r = 0.5 (residual over all K, main weights reused)
    step = MoEStep(wl, h_cal, dev, masked=True)
    ms, e = measure(step)
    f_full = sum(flops_of(wl, wl.H, wl.I))  # both residual loops run over all K
    masked_row = {"variant": "masked_full_k_residual", "r": 0.5, "ms_per_step": ms,
                  "tflops": f_full / (ms * 1e-3) / 1e12, "tflops_plain_w4a4_equivalent": plain_f / (ms * 1e-3) / 1e12,
                  **e, "weight_bytes_per_elem": 0.5625}
    del step
    torch.cuda.empty_cache()
    # per-expert channel lists for the down projection at r = 0.5 (gate_up keeps the shared list:
    # each token's X residual is quantised once for all its experts)
    step = MoEStep(wl, h_cal, dev, h_cal_offsets=syn.moe_down_calibration_offsets(base))
    ms, e = measure(step)
    per_expert_row = {"variant": "per_expert_down_lists", "r": 0.5, "ms_per_step": ms,
                      "tflops": sum(flops_of(wl, wl.Kp_gu, wl.Kp_dn)) / (ms * 1e-3) / 1e12,
                      "tflops_plain_w4a4_equivalent": plain_f / (ms * 1e-3) / 1e12, **e}
    del step
    torch.cuda.empty_cache()
    # the residual with its own tensor scale (two accumulators) at r = 0.5
    step = MoEStep(wl, h_cal, dev, own_scale=True)
    ms, e = measure(step)
    own_row = {"variant": "own_scale_residual", "r": 0.5, "ms_per_step": ms,
               "tflops": sum(flops_of(wl, wl.Kp_gu, wl.Kp_dn)) / (ms * 1e-3) / 1e12,
               "tflops_plain_w4a4_equivalent": plain_f / (ms * 1e-3) / 1e12, **e}
    del step
    torch.cuda.empty_cache()
    # the FP8 comparison format on the same block (E4M3, power-of-two scale per 32 elements)
    step = Mx8MoEStep(base, dev)
    ms, e = measure(step)
    fp8_row = {"variant": "fp8_e4m3_pow2_scale_per_32", "ms_per_step": ms,
               "tflops": plain_f / (ms * 1e-3) / 1e12, **e, "weight_bytes_per_elem": 1.0 + 1.0 / 32,
               "nvfp4_rac_r0.5_speedup": ms / at_r(rows, 0.5)["ms_per_step"]}
    del step
    torch.cuda.empty_cache()
    mono = all(rows[i + 1]["y_mean_abs"] <= rows[i]["y_mean_abs"] for i in range(len(rows) - 1))
    at = {x["r"]: x for x in rows}
    line = {"metric": METRIC, "value": at[0.5]["tflops"], "unit": "TFLOP/s", "n_gpus": 1, "steps": args.steps,
            "warmup": max(3, args.warmup), "ms_per_step": at[0.5]["ms_per_step"], "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None,
            "dtype": "nvfp4 (e2m1 x e2m1, ue4m3 block scales) -> f32 accumulate",
            "data": "synthetic (seeded counter-based generator)",
            "config": {"workload": base.name + "_r_sweep", "r": [x["r"] for x in rows],
                       "error_reference": "binary64 product of the bf16 inputs (gate_up, silu(g)*u, down) on 256 "
                                          "sampled (token, expert) rows",
                       "l2": "flushed between timed steps (256 MiB write outside the per-step events)"},
            "sweep": rows, "masked_variant": masked_row, "per_expert_variant": per_expert_row,
            "own_scale_variant": own_row,
            "fp8_comparison": fp8_row, "y_error_non_increasing_in_r": mono, "e2e": None,
            "gpu_launches": MoEStep.KERNELS_PER_STEP * args.steps * (len(rows) + 3) + 2 * args.steps +
            Mx8MoEStep.KERNELS_PER_STEP * args.steps}
    print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="nvfp4rac", choices=["nvfp4rac", "reference"])
    ap.add_argument("--workload", default="moe_prefill", choices=sorted(SPECS) + ["sweep"])
    ap.add_argument("--ref-pairs", type=int, default=256)
    ap.add_argument("--cpu-pairs", type=int, default=256)
    ap.add_argument("--cpu-rows", type=int, default=16)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--gemm-pairs", type=int, default=None, choices=[0, 1],
                    help="GEMMs on CTA pairs (1) or single SMs (0); default: the library's choice")
    ap.add_argument("--qdq-tensors", type=int, default=1024,
                    help="qdq workload: number of 1024 x 2048 tensors (1024 = 2^31 elements; fewer for profiler captures)")
    ap.add_argument("--fused-combine", action="store_true",
                    help="layer workloads (prefill): the weighted combine in the down GEMM's epilogue")
    ap.add_argument("--no-graph", action="store_true",
                    help="time the step's API calls directly instead of replaying them from a CUDA graph")
    ap.add_argument("--experts", type=int, default=None,
                    help="MoE workloads: expert count override (smaller device footprint for profiler captures)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args)
    if args.workload == "sweep":
        return run_sweep(args)

    import torch

    ws, rank, local = dist_env()
    if ws > 1:
        import datetime

        import torch.distributed as dist

        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)

    from nvfp4_w4a4_moe_02_b200 import nvfp4rac as R

    R.load()
    if args.gemm_pairs is not None:
        R.set_gemm_pairs(bool(args.gemm_pairs))
    peaks, peak_kind = load_peaks()
    sp = SPECS[args.workload](dev, args, peaks)
    step = sp["step"]
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    def barrier():
        if ws > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize()

    clocks = ClockSampler(local)
    clocks.start()
    # warm-up (also gives the clock sampler time to start)
    for _ in range(args.warmup):
        flush.zero_()
        step.run()
    torch.cuda.synchronize()
    clocks.wait_first_sample()
    R.check_status(step.status)

    # the step's launches captured once into a CUDA graph (same buffers every step), so the
    # host's per-call work (argument checks, tensor-map encoding) is off the device's timeline
    graph = None
    if not args.no_graph:
        try:
            side = torch.cuda.Stream()
            side.wait_stream(torch.cuda.current_stream())
            with torch.cuda.stream(side):
                step.run()
            torch.cuda.current_stream().wait_stream(side)
            torch.cuda.synchronize()
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph):
                step.run()
            torch.cuda.synchronize()
            for _ in range(args.warmup):
                flush.zero_()
                graph.replay()
            torch.cuda.synchronize()
            R.check_status(step.status)
        except Exception as ex:  # capture not possible for this step: plain launches
            print(f"# CUDA graph capture failed ({str(ex)[:120]}); timing plain launches", file=sys.stderr)
            graph = None
            torch.cuda.synchronize()

    # timed region: K steps with events at the step boundaries only (an event between two
    # kernels holds the second until the first has drained: about 8 us per MoE step); L2 flushed
    # between steps (outside the per-step events)
    first, last = sp["events"][0], sp["events"][-1]
    evs_step = [{n: torch.cuda.Event(enable_timing=True) for n in (first, last)} for _ in range(args.steps)]
    barrier()
    t_wall0 = time.time()
    for i in range(args.steps):
        flush.zero_()
        if graph is not None:
            evs_step[i][first].record()
            graph.replay()
            evs_step[i][last].record()
        else:
            step.run(events=evs_step[i])
    barrier()
    t_wall1 = time.time()
    clk = clocks.stop(t_wall0, t_wall1)
    R.check_status(step.status)
    # per-kernel times (kernel_ms, the roofline's kernel duration): K further steps, right after
    # the timed region, with events between the kernels
    evs = [{n: torch.cuda.Event(enable_timing=True) for n in sp["events"]} for _ in range(args.steps)]
    for i in range(args.steps):
        flush.zero_()
        step.run(events=evs[i])
    torch.cuda.synchronize()
    R.check_status(step.status)
    per = {k: [e[a].elapsed_time(e[b]) for e in evs] for k, (a, b) in sp["segments"].items()}
    t_step_ms = float(np.sum([e[first].elapsed_time(e[last]) for e in evs_step])) / args.steps
    t_step_ms = max_over_ranks(t_step_ms, ws, dev)
    unit = sp.get("unit", "TFLOP/s")
    work = sp.get("work", sp["flops"])
    scale = 1e12 if unit == "TFLOP/s" else 1e9
    value = whole_job_rate(work, ws, t_step_ms, scale)

    # roofline of the dominant kernel: algorithmic bytes / flops over its event-timed duration
    k_ms = {k: float(np.mean(v)) for k, v in per.items()}
    seg, d_flops, d_bytes, d_label = sp["dominant"]
    fp4_peak = peaks["bf16_tflops"] * FP4_OVER_BF16
    if d_bytes / (peaks["hbm_gbs"] * 1e9) >= d_flops / (fp4_peak * 1e12):
        achieved = d_bytes / (k_ms[seg] * 1e-3) / 1e9
        roof = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": achieved / peaks["hbm_gbs"], "traffic": None}
    else:
        achieved = d_flops / (k_ms[seg] * 1e-3) / 1e12
        roof = {"bound": "tensor", "achieved": achieved, "peak": fp4_peak, "unit": "TFLOP/s",
                "frac": achieved / fp4_peak, "traffic": None}
    # DRAM traffic of the dominant kernel from the committed ncu capture of this workload (None
    # when no capture of the current kernel exists)
    roof["traffic"] = sp.get("traffic")
    roof["kernel"] = d_label
    roof["algorithmic"] = {"bytes": d_bytes, "flops": d_flops}
    roof["peak_source"] = (f"{peak_kind}: HBM = copy bandwidth, FP4 = bf16 burst x {FP4_OVER_BF16:g} (nominal ratio)"
                           if peak_kind == "measured" else "recipe fallback")

    # end-to-end through the public API with host buffers: H2D of the inputs, D2H of the result
    # every step (for the MoE block: the whole layer, [T, H] out)
    e2e_step = sp.get("e2e_step", step)
    e2e_h2d = sp.get("e2e_extra_h2d", sp.get("extra_h2d", {}))
    x_np = sp["x_np"]
    x_host = torch.from_numpy(x_np.view(np.int16)).pin_memory()
    y_host = torch.empty(e2e_step.y.shape, dtype=torch.bfloat16).pin_memory()
    x_dev = torch.empty(x_np.shape, dtype=torch.bfloat16, device=dev)
    extra_host = {k: torch.from_numpy(v).pin_memory() for k, v in e2e_h2d.items()}
    extra_dev = {k: torch.empty_like(v, device=dev) for k, v in extra_host.items()}
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n_e2e = max(3, args.steps // 4)
    e2e_ms = 0.0
    pipelined = getattr(e2e_step, "takes_out", False)
    if pipelined:
        # steps pipelined over two buffer sets: step i's inputs go up on a copy stream while step
        # i - 1 computes and step i - 2's output comes down on a third stream.  Every step still
        # copies its inputs in and its [T, H] output out; the packed weights (larger than L2)
        # stream through L2 every step, so no flush runs between these steps.
        cur = torch.cuda.current_stream()
        s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
        xs = [x_dev, torch.empty_like(x_dev)]
        exs = [extra_dev, {k: torch.empty_like(v) for k, v in extra_dev.items()}]
        ys = [torch.empty_like(e2e_step.y), torch.empty_like(e2e_step.y)]
        yh = [y_host, torch.empty_like(y_host).pin_memory()]
        done_in = [torch.cuda.Event() for _ in range(n_e2e)]
        done_run = [torch.cuda.Event() for _ in range(n_e2e)]
        done_out = [torch.cuda.Event() for _ in range(n_e2e)]
        torch.cuda.synchronize()
        e0.record(s_in)
        for i in range(n_e2e):
            b = i % 2
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(done_run[i - 2])  # buffer set b read by step i - 2
                xs[b].view(torch.int16).copy_(x_host, non_blocking=True)
                for k, v in extra_host.items():
                    exs[b][k].copy_(v, non_blocking=True)
                done_in[i].record(s_in)
            cur.wait_event(done_in[i])
            if i >= 2:
                cur.wait_event(done_out[i - 2])  # output buffer b read back by step i - 2
            e2e_step.run(x=xs[b], out=ys[b], **exs[b])
            done_run[i].record(cur)
            with torch.cuda.stream(s_out):
                s_out.wait_event(done_run[i])
                yh[b].copy_(ys[b], non_blocking=True)
                done_out[i].record(s_out)
        e1.record(s_out)
        torch.cuda.synchronize()
        e2e_ms = e0.elapsed_time(e1) / n_e2e
    else:
        for _ in range(n_e2e):
            flush.zero_()
            e0.record()
            x_dev.view(torch.int16).copy_(x_host, non_blocking=True)
            for k, v in extra_host.items():
                extra_dev[k].copy_(v, non_blocking=True)
            y = e2e_step.run(x=x_dev, **extra_dev)
            y_host.copy_(y, non_blocking=True)
            e1.record()
            torch.cuda.synchronize()
            e2e_ms += e0.elapsed_time(e1)
        e2e_ms /= n_e2e
    e2e_ms = max_over_ranks(e2e_ms, ws, dev)
    R.check_status(e2e_step.status)
    e2e = {"value": whole_job_rate(work, ws, e2e_ms, scale), "unit": unit,
           "h2d_bytes_per_step": int(x_np.nbytes) + sum(int(v.nbytes) for v in e2e_h2d.values()),
           "d2h_bytes_per_step": int(y_host.numel() * 2),
           "call": "whole MoE layer (router, plan, quantise, GEMMs, combine into [T, H])" if "e2e_step" in sp
           else "the timed step",
           "schedule": ("steps pipelined on three streams (copy in / compute / copy out, two buffer sets); "
                        "no L2 flush: the packed weights, larger than L2, stream every step") if pipelined
           else "one step at a time, L2 flushed before each"}

    cpu = sp["cpu"]() if (rank == 0 and ws == 1 and not args.no_cpu_baseline) else None

    if rank == 0:
        config = dict(sp["config"])
        config["l2"] = "flushed between timed steps (256 MiB write outside the per-step events)"
        config["timing"] = ("ms_per_step: events at step boundaries only" +
                            (", the step's launches replayed from one CUDA graph" if graph is not None else "") +
                            "; kernel_ms and the roofline's kernel duration: the same number of steps right after, "
                            "launched through the API with events between the kernels")
        config["parallelism"] = f"replicas x{ws}"
        if args.gemm_pairs is not None:
            config["gemm_pairs"] = bool(args.gemm_pairs)
        line = {
            "metric": METRIC, "value": value, "unit": unit, "n_gpus": ws, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": t_step_ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None,
            "dtype": sp.get("dtype", "nvfp4 (e2m1 x e2m1, ue4m3 block scales) -> f32 accumulate"),
            "data": "synthetic (seeded counter-based generator)",
            "config": config,
            "fp4_peak_tflops": fp4_peak,
            "frac_fp4_peak": value / ws / fp4_peak if unit == "TFLOP/s" else None,
            "kernel_ms": k_ms,
            "act_quant_gbs": {k: b / (k_ms[s] * 1e-3) / 1e9 for k, (s, b) in sp["quant"].items()},
            "kernel_gbs": {k: b / ((k_ms[s] if s else t_step_ms) * 1e-3) / 1e9
                           for k, (s, b) in sp.get("extra_gbs", {}).items()},
            "roofline": roof,
            "cpu_baseline": cpu,
            "e2e": e2e,
            "gpu_launches": sp["kernels_per_step"] * args.steps,
            "clocks": clk,
        }
        print(json.dumps(line), flush=True)
    del graph  # released before the process group goes
    if ws > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
