"""Expert-parallel MoE layer over the GPUs of one node.

Rank r of R holds the routed experts [r E/R, (r+1) E/R) and the shared expert,
packed (flint_pack_nvfp4 / flint_pack_bf16) as E/R routed experts plus one
shared, so that with the local shape (E/R + 1 experts, top_k 1, no shared) the
shared expert is local id E/R. One layer step on a rank:

  1. route its tokens (flint_moe_route, replicated router weights);
  2. dispatch (flint_ep_dispatch): every (token, slot) pair to the rank that
     holds its expert, the shared-expert pair to the token's own rank, rows in
     destination order;
  3. exchange the per-rank row counts, then the rows, their local expert ids
     and gates (all-to-all with those splits);
  4. run the received rows through the local experts (flint_moe_forward_routed,
     each row scaled by its gate), bf16 rows out;
  5. return the rows to their home ranks (the reverse all-to-all);
  6. sum each token's rows plus the residual (flint_ep_combine).

Every arithmetic step runs in the library's kernels; this module sizes the
buffers and moves the rows. The exchange is `torch.distributed`'s
all_to_all_single (NCCL over NVLink between GPUs; the same calls run on gloo
for CPU tensors).
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import (FLINT_ERR_DEVICE_CHECK, FlintError, Shape, Weights, flint_ep_combine, flint_ep_dispatch,
               flint_moe_forward_routed, flint_moe_get_status, flint_moe_route, flint_moe_workspace_bytes,
               flint_moe_workspace_init)


class AllToAll:
    """Row exchange between the ranks of a process group."""

    def __init__(self, group=None):
        self.group = group

    def counts(self, send_counts: torch.Tensor) -> torch.Tensor:
        """send_counts[r] rows go to rank r; returns recv_counts[r] from rank r."""
        recv = torch.empty_like(send_counts)
        dist.all_to_all_single(recv, send_counts, group=self.group)
        return recv

    def rows(self, send: torch.Tensor, send_splits: list[int], recv_splits: list[int],
             out: torch.Tensor) -> torch.Tensor:
        """send: rows in destination-rank order, send_splits[r] of them for rank
        r; out receives recv_splits[r] rows from each rank r, in rank order."""
        dist.all_to_all_single(out, send, output_split_sizes=list(recv_splits), input_split_sizes=list(send_splits),
                               group=self.group)
        return out


def local_shape(shape: Shape, n_ranks: int) -> Shape:
    """The per-rank shape of the expert call: E/R routed + the shared expert as
    one more local expert, top_k 1, no separate shared expert."""
    if shape.n_experts % n_ranks:
        raise ValueError("n_experts must be a multiple of the number of ranks")
    return Shape(shape.d, shape.inter, shape.n_experts // n_ranks + shape.n_shared, 1, 0, shape.wdtype)


def packing_shape(shape: Shape, n_ranks: int) -> Shape:
    """The shape to pack one rank's experts with: E/R routed + the shared."""
    return Shape(shape.d, shape.inter, shape.n_experts // n_ranks, shape.top_k, shape.n_shared, shape.wdtype)


class ExpertParallelLayer:
    """One rank's share of an expert-parallel MoE layer; buffers for up to
    `max_tokens` tokens per rank are allocated once, here."""

    def __init__(self, shape: Shape, rank: int, n_ranks: int, local_weights: Weights, router_w: torch.Tensor,
                 max_tokens: int, device="cuda"):
        self.shape, self.rank, self.R = shape, rank, n_ranks
        self.lshape = local_shape(shape, n_ranks)
        self.weights = local_weights
        self.router_w = router_w
        self.max_tokens = max_tokens
        d, k, S = shape.d, shape.top_k, shape.n_shared
        self.slots = k + S
        P = max_tokens * self.slots
        # rows a rank can receive: every routed pair of every rank, plus its own
        # shared-expert pairs
        self.max_recv = n_ranks * max_tokens * k + max_tokens * S
        i32, f32, bf = torch.int32, torch.float32, torch.bfloat16
        self.ids = torch.empty((max_tokens, k), dtype=i32, device=device)
        self.gates = torch.empty((max_tokens, k), dtype=f32, device=device)
        self.route_ws = torch.empty(flint_moe_workspace_bytes(shape, max_tokens), dtype=torch.uint8, device=device)
        self.send_x = torch.empty((P, d), dtype=bf, device=device)
        self.send_ids = torch.empty(P, dtype=i32, device=device)
        self.send_gates = torch.empty(P, dtype=f32, device=device)
        self.send_token = torch.empty(P, dtype=i32, device=device)
        self.send_counts = torch.zeros(n_ranks, dtype=i32, device=device)
        self.pair_pos = torch.empty((max_tokens, self.slots), dtype=i32, device=device)
        self.recv_x = torch.empty((self.max_recv, d), dtype=bf, device=device)
        self.recv_ids = torch.empty(self.max_recv, dtype=i32, device=device)
        self.recv_gates = torch.empty(self.max_recv, dtype=f32, device=device)
        self.y = torch.empty((self.max_recv, d), dtype=bf, device=device)
        self.y_back = torch.empty((P, d), dtype=bf, device=device)
        self.expert_ws = torch.empty(flint_moe_workspace_bytes(self.lshape, self.max_recv), dtype=torch.uint8,
                                     device=device)
        self.status = torch.zeros(1, dtype=i32, device=device)
        flint_moe_workspace_init(self.route_ws)
        flint_moe_workspace_init(self.expert_ws)

    # --------------------------------------------------------------- phases
    def send(self, x: torch.Tensor, T: int) -> torch.Tensor:
        """Route and dispatch this rank's tokens; returns the device send counts."""
        if T > self.max_tokens:
            raise ValueError(f"{T} tokens > max_tokens {self.max_tokens}")
        s = self.shape
        flint_moe_route(x, T, self.router_w, s, self.ids, self.gates, self.route_ws)
        flint_ep_dispatch(self.ids, self.gates, T, s.top_k, s.n_shared, s.n_experts, self.R, self.rank, x, s.d,
                          self.send_x, self.send_ids, self.send_gates, self.send_token, self.send_counts,
                          self.pair_pos, self.status)
        return self.send_counts

    def experts(self, n_recv: int) -> torch.Tensor:
        """The received rows through the local experts (gate-scaled rows)."""
        if n_recv > self.max_recv:
            raise ValueError(f"{n_recv} received rows > {self.max_recv}")
        if n_recv:
            flint_moe_forward_routed(self.recv_x, n_recv, self.recv_ids, self.recv_gates, self.weights, self.lshape,
                                     None, self.y, self.expert_ws)
        return self.y[:n_recv]

    def finish(self, T: int, out: torch.Tensor, residual=None) -> torch.Tensor:
        flint_ep_combine(self.y_back, self.pair_pos, T, self.slots, self.shape.d, residual, out)
        return out

    def check(self) -> None:
        """Synchronises and raises FlintError if a kernel of the last steps
        recorded a failed check: an out-of-range id in the dispatch or the
        router (FLINT_DEVCHECK_* bits of this rank's status words), or a
        bounded wait that gave up in the expert call. Clears the flags."""
        flags = int(self.status.item())
        self.status.zero_()
        rc_r, f_r = flint_moe_get_status(self.route_ws)
        rc_e, f_e = flint_moe_get_status(self.expert_ws)
        flags |= f_r | f_e
        rc = rc_e or rc_r
        if flags or rc:
            raise FlintError(rc or FLINT_ERR_DEVICE_CHECK,
                             f"expert-parallel step on rank {self.rank}: device check flags {flags:#x}")

    # --------------------------------------------------------------- one step
    def forward(self, x: torch.Tensor, T: int, out: torch.Tensor, residual=None, exchange: AllToAll | None = None):
        ex = exchange or AllToAll()
        counts = self.send(x, T)
        recv_counts = ex.counts(counts)
        sc = counts.cpu().tolist()
        rc = recv_counts.cpu().tolist()
        n_sent, n_recv = sum(sc), sum(rc)
        if n_recv > self.max_recv:
            raise ValueError(f"{n_recv} received rows > {self.max_recv}")
        ex.rows(self.send_x[:n_sent], sc, rc, self.recv_x[:n_recv])
        ex.rows(self.send_ids[:n_sent], sc, rc, self.recv_ids[:n_recv])
        ex.rows(self.send_gates[:n_sent], sc, rc, self.recv_gates[:n_recv])
        self.experts(n_recv)
        ex.rows(self.y[:n_recv], rc, sc, self.y_back[:n_sent])
        return self.finish(T, out, residual)


def slice_rank_weights(full_f32: torch.Tensor, shape: Shape, rank: int, n_ranks: int) -> torch.Tensor:
    """fp32 weights [E+S][3][...] of the full layer -> those rank `rank`
    packs: its E/R routed experts, then the shared expert."""
    el = shape.n_experts // n_ranks
    parts = [full_f32[rank * el:(rank + 1) * el]]
    if shape.n_shared:
        parts.append(full_f32[shape.n_experts:shape.n_experts + shape.n_shared])
    return torch.cat(parts).contiguous()


__all__ = ["AllToAll", "ExpertParallelLayer", "local_shape", "packing_shape", "slice_rank_weights"]
