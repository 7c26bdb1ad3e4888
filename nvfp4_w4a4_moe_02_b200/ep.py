"""Expert parallelism for the NVFP4 W4A4 + RAC MoE expert block (torch.distributed plumbing).

The QUADS abstract places the method in MoE rollouts; a rollout engine spreads the experts of a
layer over the GPUs of a node.  With P ranks, rank r owns experts [r E/P, (r+1) E/P) and its own
batch of tokens.  One layer step on rank r:

  1. router top-k of its tokens and the expert-grouped dispatch plan over all E experts, segments
     padded to 128 rows (moe_route_topk, moe_dispatch_plan): the rows of destination d are the
     contiguous block of experts [d E/P, (d+1) E/P);
  2. the tensor scale of X is the amax over every rank's tokens (one all-reduce of a float), so
     that each token is quantised exactly as on one GPU holding the whole batch;
  3. quantise X once per token and scatter its codes / scales / residual into its expert rows
     (nvfp4_quantize_scatter), i.e. straight into the send buffer;
  4. exchange the token counts per expert (all-to-all of E/P ints per rank) and the packed rows
     (all-to-all of codes, scales, residual codes, residual scales: one contiguous block per
     destination, 128-row aligned so that the scale atoms split cleanly);
  5. the received rows form P x E/P segments (source-major), each 128-padded: the grouped GEMMs
     take them with a segment -> local expert map; h's tensor scale is again a global amax;
  6. the expert outputs go back with the reverse all-to-all, and each rank combines its tokens'
     k rows (moe_combine) from its own send layout.

Only steps 2, 4 and 6 move data between ranks; everything else runs in the library's kernels.
The functions here take and return torch tensors on any device, so the same plumbing runs over
NCCL on GPUs and over gloo on CPU (where the tests drive it with the oracle's arithmetic).
"""
from __future__ import annotations

import torch
import torch.distributed as dist


class ExpertParallel:
    """Rank bookkeeping and the collectives of one expert-parallel group."""

    def __init__(self, E: int, group=None, pad: int = 128):
        self.group = group
        self.P = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        if E % self.P != 0:
            raise ValueError(f"E = {E} experts do not split evenly over {self.P} ranks")
        self.E = E
        self.E_local = E // self.P
        self.pad = pad

    # ----------------------------------------------------------------------------- layout
    def owner(self, expert: int) -> int:
        return expert // self.E_local

    def send_rows(self, offsets: torch.Tensor) -> list[int]:
        """Rows of the send buffer (the dispatch plan's padded layout) going to each rank: the
        block of experts [d E/P, (d+1) E/P).  Reads the offsets on the host (one sync)."""
        o = offsets.to("cpu", torch.int64)
        El = self.E_local
        return [int(o[(d + 1) * El] - o[d * El]) for d in range(self.P)]

    def exchange_counts(self, expert_rows: torch.Tensor) -> torch.Tensor:
        """Token rows per expert [E] of this rank -> token rows this rank receives from each
        source for each of its local experts, int32 [P, E/P]."""
        send = expert_rows.to(torch.int32).contiguous()
        recv = torch.empty(self.P * self.E_local, dtype=torch.int32, device=send.device)
        dist.all_to_all_single(recv, send, group=self.group)
        return recv.view(self.P, self.E_local)

    def recv_segments(self, recv_counts: torch.Tensor):
        """The received rows as P x E/P segments in source-major order, each padded to `pad` rows:
        (seg_offsets int32 [P E/P + 1], seg_rows int32 [P E/P] token rows, seg_expert int32
        [P E/P] local expert of each segment, rows received from each source [P])."""
        c = recv_counts.to(torch.int64)
        padded = (c + self.pad - 1) // self.pad * self.pad
        seg_off = torch.zeros(self.P * self.E_local + 1, dtype=torch.int64, device=c.device)
        seg_off[1:] = torch.cumsum(padded.reshape(-1), 0)
        seg_expert = torch.arange(self.E_local, dtype=torch.int32, device=c.device).repeat(self.P)
        per_source = [int(v) for v in padded.sum(1).cpu()]
        return seg_off.to(torch.int32), c.reshape(-1).to(torch.int32), seg_expert, per_source

    # ----------------------------------------------------------------------------- data movement
    def exchange_rows(self, send: torch.Tensor, send_rows: list[int], recv_rows: list[int]) -> torch.Tensor:
        """All-to-all of row blocks: send [sum(send_rows), ...] with block d going to rank d ->
        [sum(recv_rows), ...] with block s from rank s."""
        out = torch.empty((sum(recv_rows),) + tuple(send.shape[1:]), dtype=send.dtype, device=send.device)
        dist.all_to_all_single(out, send.contiguous(), output_split_sizes=recv_rows, input_split_sizes=send_rows,
                               group=self.group)
        return out

    def exchange_packed(self, codes: torch.Tensor, sf: torch.Tensor, cols: int, send_rows: list[int],
                        recv_rows: list[int]):
        """All-to-all of a packed NVFP4 matrix (codes [rows * cols/2] bytes, scale atoms
        [rows * cols/16] bytes, rows grouped in 128-row atom blocks): every block boundary is a
        multiple of 128 rows, so the atom bytes of each block are contiguous."""
        assert all(r % 128 == 0 for r in send_rows + recv_rows)
        n_send = sum(send_rows)
        c = codes[:n_send * cols // 2].view(n_send, cols // 2)
        s = sf[:n_send * cols // 16].view(n_send, cols // 16)
        return (self.exchange_rows(c, send_rows, recv_rows).view(-1),
                self.exchange_rows(s, send_rows, recv_rows).view(-1))

    def global_amax(self, amax: torch.Tensor) -> torch.Tensor:
        """In place: the largest amax over the ranks (so every rank quantises with the scale a
        single GPU holding the whole batch would use)."""
        dist.all_reduce(amax, op=dist.ReduceOp.MAX, group=self.group)
        return amax


class EPMoEBlock:
    """One expert-parallel MoE layer step through the C ABI on this rank's GPU (nothing on the
    host per step except the split sizes of the all-to-alls).

    Weights: this rank's E/P experts, packed (gate_up with the SwiGLU interleave); channel lists
    shared by all experts (sel_gu over the hidden channels, sel_dn over the intermediate ones)."""

    def __init__(self, ep: ExpertParallel, T: int, k: int, H: int, I: int, packed, sel_gu, sel_dn, device):
        from . import nvfp4rac as R

        self.R, self.ep, self.dev = R, ep, device
        self.T, self.k, self.H, self.I = T, k, H, I
        self.pgu, self.pgus, self.pdn, self.pdns = packed
        self.sel_gu, self.sel_dn = sel_gu, sel_dn
        self.status = R.new_status(device)
        self.cap = R.moe_rows_capacity(T, k, ep.E, 128)
        P = R.Packed
        self.ids = torch.empty(T, k, dtype=torch.int32, device=device)
        self.w = torch.empty(T, k, dtype=torch.float32, device=device)
        self.off = torch.empty(ep.E + 1, dtype=torch.int32, device=device)
        self.rows = torch.empty(T, k, dtype=torch.int32, device=device)
        self.expert_rows = torch.empty(ep.E, dtype=torch.int32, device=device)
        self.a = P.empty(self.cap, H, rows_padded=self.cap, device=device, zero=True)
        self.ar = P.empty(self.cap, len(sel_gu), rows_padded=self.cap, device=device, zero=True)
        self.amax_x = torch.zeros(1, dtype=torch.float32, device=device)
        self.amax_h = torch.zeros(1, dtype=torch.float32, device=device)
        self.y = torch.empty(T, H, dtype=torch.bfloat16, device=device)

    def run(self, x: torch.Tensor, logits: torch.Tensor) -> torch.Tensor:
        R, ep, st = self.R, self.ep, self.status
        # 1. routing and the send layout (all E experts, 128-row segments)
        R.moe_route_topk(logits, self.k, ids=self.ids, w=self.w, status=st)
        R.moe_dispatch_plan(self.ids, ep.E, 128, rows_capacity=self.cap, offsets=self.off, row_scatter=self.rows,
                            status=st, expert_rows=self.expert_rows)
        # 2. the global tensor scale of X
        R.nvfp4_amax(x, out=self.amax_x, status=st)
        ep.global_amax(self.amax_x)
        # 3. quantise once per token, scatter into the send rows
        R.nvfp4_quantize_scatter(x, self.rows, self.cap, self.sel_gu, amax_in=self.amax_x, out=self.a,
                                 out_res=self.ar, status=st)
        # 4. counts, then the packed rows
        send_rows = ep.send_rows(self.off)
        recv_counts = ep.exchange_counts(self.expert_rows)
        seg_off, seg_rows, seg_expert, recv_rows = ep.recv_segments(recv_counts)
        n_recv = sum(recv_rows)
        Kg = len(self.sel_gu)
        rc, rs = ep.exchange_packed(self.a.codes, self.a.sf, self.H, send_rows, recv_rows)
        rrc, rrs = ep.exchange_packed(self.ar.codes, self.ar.sf, Kg, send_rows, recv_rows)
        n_alloc = max(n_recv, 128)
        a_in = R.Packed(_fit(rc, n_alloc * self.H // 2), _fit(rs, n_alloc * self.H // 16), self.a.s_g, 1, n_alloc,
                        n_alloc, self.H)
        ar_in = R.Packed(_fit(rrc, n_alloc * Kg // 2), _fit(rrs, n_alloc * Kg // 16), self.a.s_g, 1, n_alloc,
                         n_alloc, Kg)
        # 5. the local experts over the received segments; h's scale is global too
        h = torch.zeros(n_alloc, self.I, dtype=torch.bfloat16, device=self.dev)
        R.grouped_w4a4_rac_moe_segments(a_in, ar_in, seg_off, seg_rows, seg_expert, self.pgu, self.pgus, swiglu=True,
                                        y=h, amax_out=self.amax_h, status=st)
        ep.global_amax(self.amax_h)
        Kd = len(self.sel_dn)
        hq = R.Packed.empty(n_alloc, self.I, rows_padded=n_alloc, device=self.dev, zero=True)
        hqr = R.Packed.empty(n_alloc, Kd, rows_padded=n_alloc, device=self.dev, zero=True)
        R.nvfp4_quantize_segments(h, seg_off, seg_rows, self.sel_dn, amax_in=self.amax_h, out=hq, out_res=hqr,
                                  status=st)
        ye = torch.zeros(n_alloc, self.H, dtype=torch.bfloat16, device=self.dev)
        R.grouped_w4a4_rac_moe_segments(hq, hqr, seg_off, seg_rows, seg_expert, self.pdn, self.pdns, y=ye, status=st)
        # 6. back to the token owners, combined into [T, H]
        back = ep.exchange_rows(ye[:n_recv], recv_rows, send_rows)
        R.moe_combine(back, self.rows, self.w, out=self.y, status=st)
        return self.y


def _fit(t: torch.Tensor, n: int) -> torch.Tensor:
    """t padded with zeros (or cut) to n elements."""
    if t.numel() >= n:
        return t[:n]
    out = torch.zeros(n, dtype=t.dtype, device=t.device)
    out[:t.numel()] = t
    return out
