"""The per-rank step of a real D-GPU ZeRO group with the data movement done by
collectives (NCCL between GPUs, on one node or across nodes).

"7.10 — Fully-sharded data parallel (FSDP / ZeRO-3)", §4: the all-reduce of
the gradients becomes a reduce-scatter, after which rank r holds the summed
gradient of its partition P_r only; §3 and §5.1: after the update, the bf16
parameters are all-gathered.  "Building GPT from Scratch — Part 8",
"AllGather vs AllReduce": rank r receives the r-th slice of every rank's
gradient.

The collectives here move bytes only; the arithmetic stays in libzero3.so's
fused kernel, in the fixed rank order, so rank r's result equals the
single-GPU simulation's for P_r bit for bit (a library reduce-scatter sums in
an order of its own):

    1. all-to-all of the bf16 gradient: chunk j of rank d's buffer (its slice
       P_j) goes to rank j, so rank r receives P_r of every rank's gradient,
       back to back in rank order -- the reduce-scatter's data movement;
    2. the fused kernel on those D slices (the owned layout): the reduction in
       rank order, AdamW on the local fp32 state, the cast to the bf16 shard;
    3. all-gather of the bf16 shards into the flat block.

Compared with the peer-memory step (peer.py), this one needs no IPC mapping,
so it also runs between nodes, at the cost of the D x S receive buffer that
the peer step's direct loads avoid.  The collectives run on the caller's
current stream with the kernel, in stream order; nothing waits on the host.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import zero3 as z3


class CollectiveZero3Step:
    """Rank r's optimiser step in a D-rank process group (D = the group's size).

    grad:      this rank's full bf16 gradient of the block (N_pad elements).
    master, exp_avg, exp_avg_sq: this rank's fp32 state for P_r (S elements).
    work_bf16: this rank's bf16 working shard (S elements).
    flat:      this rank's gathered block (N_pad elements), written every step.
    """

    def __init__(self, plan: "z3.Plan", grad: torch.Tensor, master: torch.Tensor, exp_avg: torch.Tensor,
                 exp_avg_sq: torch.Tensor, work_bf16: torch.Tensor, flat: torch.Tensor, group=None,
                 reduce_dtype: int = z3.Z3_REDUCE_FP32, kernels=z3):
        self.group = group
        self.rank = dist.get_rank(group)
        D = dist.get_world_size(group)
        if plan.D != D:
            raise ValueError(f"the plan is for D = {plan.D} ranks, the group has {D}")
        S = plan.S
        for name, t, n in (("grad", grad, plan.N_pad), ("flat", flat, plan.N_pad), ("work_bf16", work_bf16, S)):
            if t.dtype != torch.bfloat16 or t.numel() != n or not t.is_contiguous():
                raise ValueError(f"{name} must be a contiguous bf16 tensor of {n} elements")
        self.plan, self.reduce_dtype, self.k = plan, reduce_dtype, kernels
        self.grad, self.master, self.exp_avg, self.exp_avg_sq = grad, master, exp_avg, exp_avg_sq
        self.work, self.flat = work_bf16, flat
        # P_r of every rank's gradient, back to back in rank order
        self.recv = torch.empty(D * S, dtype=torch.bfloat16, device=grad.device)
        self.slices = [self.recv[d * S:(d + 1) * S] for d in range(D)]

    def step(self, hp: "z3.AdamW") -> None:
        k = self.k
        dist.all_to_all_single(self.recv, self.grad, group=self.group)
        k.zero3_reduce_adamw(self.plan, self.rank, self.slices, self.master, self.exp_avg, self.exp_avg_sq,
                             self.work, hp, contrib_layout=k.Z3_CONTRIB_OWNED, reduce_dtype=self.reduce_dtype)
        dist.all_gather_into_tensor(self.flat, self.work, group=self.group)
