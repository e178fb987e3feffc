"""Expert-parallel routed MoE layer over a torch.distributed process group.

The routed layer of turbospark-runtime 0.3.0, src/families/qwen/moe_batch.rs
(encode_qwen_layer_moe_batched: routes grouped by expert, phase 1 and phase 2
over the expert union, the seeded rank-ordered sum) with its E experts spread
over the W ranks of a group: rank r holds the contiguous block of experts
[r * E/W, (r + 1) * E/W). Every rank routes its own token rows, then

1. ``begin``   -- router + top-k + pairs in expert order (moe_router_topk) and
                  the pairs' token rows in that order (moe_dispatch_rows): the
                  rows bound for each rank form one contiguous block;
2. exchange    -- all-to-all of the row blocks and their experts;
3. ``expert_work`` -- the owner runs its experts over the rows it received, in
                  arrival order (moe_experts_grouped: fp32 down outputs);
4. exchange    -- all-to-all of the down outputs back to the rows' ranks, in
                  the order they were sent;
5. ``finish``  -- the shared expert and its gate (when the layer has one) and
                  the seeded rank-ordered sum plus the residual add
                  (moe_combine).

The GPU work is the library's kernels (``GpuOps``); the exchanges are
``torch.distributed.all_to_all_single`` (NCCL on GPUs). The number of rows each
rank sends to each other rank is read back to the host once per call (the
all-to-all split sizes). The result equals ``moe_layer`` on the same token rows
up to the fp32 summation order of the down projection's K splits.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Any, List, Optional, Sequence

import torch

from . import (FFN, MoePlan, QWeight, moe_combine, moe_dispatch_rows, moe_experts_grouped, moe_router_topk)


def owner_blocks(num_experts: int, world: int) -> int:
    """Experts per rank (rank r holds experts [r*n, (r+1)*n)); E must be a multiple of the world size."""
    if world < 1 or num_experts % world != 0:
        raise ValueError(f"{num_experts} experts cannot be split evenly over {world} ranks")
    return num_experts // world


def send_counts(offsets_host: Sequence[int], num_experts: int, world: int) -> List[int]:
    """Rows bound for each rank: the pairs of rank r's experts, one contiguous
    block of the expert-ordered slots (expert_offsets [E+1] on the host)."""
    n = owner_blocks(num_experts, world)
    return [int(offsets_host[(r + 1) * n]) - int(offsets_host[r * n]) for r in range(world)]


class GpuOps:
    """The layer's GPU work through the library (C ABI)."""

    def __init__(self, router: QWeight, local_experts: Sequence[FFN], num_experts: int, top_k: int, act: str,
                 rank: int, world: int, shared: Optional[FFN] = None, shared_gate: Optional[QWeight] = None):
        self.router, self.E, self.k, self.act = router, num_experts, top_k, act
        n = owner_blocks(num_experts, world)
        if len(local_experts) != n:
            raise ValueError(f"rank {rank} holds {len(local_experts)} experts, {n} expected")
        self.base = rank * n
        H = router.cols
        # The plan of this rank's block: its router rows are a slice of the
        # router (unused by moe_experts_grouped, which needs no routing).
        rows = router.q[self.base:self.base + n]
        self.plan = MoePlan(QWeight(router.format, n, H, rows), local_experts, 1, act)
        # The shared expert as a one-expert plan whose router row is the gate
        # vector: its logits are the gate logits, its expert output the seed's s.
        self.shared_plan = None
        self._zero_ids = {}   # row count -> int32 zeros: the shared plan's expert of every row
        if shared is not None:
            if shared_gate is None:
                raise ValueError("a shared expert needs its gate vector")
            self.shared_plan = MoePlan(shared_gate, [shared], 1, act)

    def route(self, x: torch.Tensor):
        M = x.shape[0]
        P = M * self.k
        perm = torch.empty(P, dtype=torch.int32, device=x.device)
        offsets = torch.empty(self.E + 1, dtype=torch.int32, device=x.device)
        idx, w = moe_router_topk(self.router, x, self.k, perm=perm, expert_offsets=offsets)
        return idx, w, perm, offsets

    def dispatch(self, x, idx, perm):
        return moe_dispatch_rows(x, idx, perm, self.k)

    def experts(self, rows, row_expert):
        return moe_experts_grouped(self.plan, rows, row_expert, self.base)

    def shared(self, x):
        if self.shared_plan is None:
            return None
        M = x.shape[0]
        z = torch.empty((M, 1), dtype=torch.float32, device=x.device)
        moe_router_topk(self.shared_plan.router, x, 1, logits_out=z)
        zeros = self._zero_ids.get(M)
        if zeros is None or zeros.device != x.device:
            zeros = self._zero_ids[M] = torch.zeros(M, dtype=torch.int32, device=x.device)
        s = moe_experts_grouped(self.shared_plan, x, zeros, 0)
        return s, z.reshape(M)

    def combine(self, d, perm, w, residual, shared_state):
        s, z = shared_state if shared_state is not None else (None, None)
        moe_combine(d, perm, w, residual, s, z)

    def close(self):
        self.plan.close()
        if self.shared_plan is not None:
            self.shared_plan.close()


@dataclass
class Pending:
    """What ``begin`` leaves for ``finish``: routing of this rank's tokens and
    the rows sent out (in the order their down outputs come back)."""
    w: Any
    perm: Any
    rows: Any
    experts: Any
    send: List[int]


class ExpertParallelMoE:
    """The routed MoE layer with this rank's block of experts.

    ``ops`` does the GPU work (``GpuOps``; tests may give a CPU stand-in with
    the same methods). ``group``: a torch.distributed process group, or None:
    then ``world`` ranks (1 by default: no exchange) whose exchanges the
    caller makes between ``begin``, ``expert_work`` and ``finish``."""

    def __init__(self, ops, num_experts: int, group=None, world: int = 1):
        self.ops, self.E, self.group = ops, num_experts, group
        if group is None:
            self.rank, self.world = 0, world
        else:
            import torch.distributed as dist
            self.rank, self.world = dist.get_rank(group), dist.get_world_size(group)
        owner_blocks(num_experts, self.world)

    # -- the three local steps ------------------------------------------------
    def begin(self, x: torch.Tensor) -> Pending:
        if x.shape[0] == 0:
            # No token rows here: nothing to send, but this rank still takes
            # every collective step (and holds experts for the others' rows).
            return Pending(None, None, x.new_empty((0,) + tuple(x.shape[1:])),
                           torch.empty(0, dtype=torch.int32, device=x.device), [0] * self.world)
        idx, w, perm, offsets = self.ops.route(x)
        rows, experts = self.ops.dispatch(x, idx, perm)
        # The split sizes of the all-to-all are read back to the host (a
        # synchronization); one rank keeps every row and needs none.
        send = [rows.shape[0]] if self.world == 1 else send_counts(offsets.cpu().tolist(), self.E, self.world)
        return Pending(w, perm, rows, experts, send)

    def expert_work(self, rows: torch.Tensor, experts: torch.Tensor):
        return self.ops.experts(rows, experts)

    def finish(self, p: Pending, d_back, x: torch.Tensor, residual: torch.Tensor) -> torch.Tensor:
        if residual.shape[0] == 0:
            return residual
        self.ops.combine(d_back, p.perm, p.w, residual, self.ops.shared(x))
        return residual

    # -- the whole layer, exchanges included ----------------------------------
    def forward(self, x: torch.Tensor, residual: torch.Tensor) -> torch.Tensor:
        p = self.begin(x)
        if self.group is None:
            if self.world != 1:
                raise ValueError("forward() exchanges rows through a process group; without one, call begin, "
                                 "expert_work and finish and exchange between them")
            return self.finish(p, self.expert_work(p.rows, p.experts), x, residual)
        import torch.distributed as dist
        recv = self.exchange_counts(p.send)
        # bf16 rows travel as int32 pairs (a type every backend can move)
        rows32 = p.rows.view(torch.int32)
        rows_in = rows32.new_empty((sum(recv),) + tuple(rows32.shape[1:]))
        exp_in = p.experts.new_empty(sum(recv))
        dist.all_to_all_single(rows_in, rows32, recv, p.send, group=self.group)
        dist.all_to_all_single(exp_in, p.experts, recv, p.send, group=self.group)
        d_in = self.expert_work(rows_in.view(p.rows.dtype), exp_in)
        d_back = d_in.new_empty((sum(p.send),) + tuple(d_in.shape[1:]))
        dist.all_to_all_single(d_back, d_in, p.send, recv, group=self.group)
        return self.finish(p, d_back, x, residual)

    def exchange_counts(self, send: List[int]) -> List[int]:
        """How many rows each rank sends to this one (one small all-to-all)."""
        import torch.distributed as dist
        dev = torch.device("cuda", torch.cuda.current_device()) if dist.get_backend(self.group) == "nccl" \
            else torch.device("cpu")
        out_t = torch.tensor(send, dtype=torch.int64, device=dev)
        in_t = torch.empty_like(out_t)
        dist.all_to_all_single(in_t, out_t, group=self.group)
        return [int(v) for v in in_t.cpu().tolist()]
