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

CollectiveHybridStep is HYBRID_SHARD across nodes on the same pattern: the
node's all-to-all, the node sum (zero3_node_sum), an all-gather of the node
sums among the replicas, the fold with AdamW (zero3_fold_adamw) and the node's
all-gather -- the two-level reduction of zero3_reduce_adamw_hybrid, split where
the node sums have to cross between machines.
"""
from __future__ import annotations

from typing import Optional

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

    def step(self, hp: "z3.AdamW", mark=None, marks: Optional[list] = None) -> None:
        """One step.  With mark (a callable returning a time mark, e.g. a CUDA
        event recorded on the current stream) and marks (a list), the four marks
        around the all-to-all, the fused kernel and the all-gather are appended to
        marks as one tuple."""
        k = self.k
        m0 = mark() if mark else None
        dist.all_to_all_single(self.recv, self.grad, group=self.group)
        m1 = mark() if mark else None
        k.zero3_reduce_adamw(self.plan, self.rank, self.slices, self.master, self.exp_avg, self.exp_avg_sq,
                             self.work, hp, contrib_layout=k.Z3_CONTRIB_OWNED, reduce_dtype=self.reduce_dtype)
        m2 = mark() if mark else None
        dist.all_gather_into_tensor(self.flat, self.work, group=self.group)
        if mark:
            marks.append((m0, m1, m2, mark()))


def hybrid_groups(n_nodes: int, D: int, world_group=None):
    """The process groups of HYBRID_SHARD over n_nodes nodes of D ranks, global
    rank k*D + d being local rank d of node k: every node's group of D ranks,
    and every local rank's group of its n_nodes replicas.  Every rank calls
    this, in the same order (group creation is collective).  Returns this
    rank's (node group, replica group); group ranks are in ascending global
    order, so a node group's rank is the local rank d and a replica group's
    rank is the node k."""
    rank = dist.get_rank(world_group)
    if dist.get_world_size(world_group) != n_nodes * D:
        raise ValueError(f"the world has {dist.get_world_size(world_group)} ranks, not {n_nodes} x {D}")
    node_group = replica_group = None
    for k in range(n_nodes):
        g = dist.new_group([k * D + d for d in range(D)])
        if rank // D == k:
            node_group = g
    for d in range(D):
        g = dist.new_group([k * D + d for k in range(n_nodes)])
        if rank % D == d:
            replica_group = g
    return node_group, replica_group


class CollectiveHybridStep:
    """Local rank d's optimiser step on node k in HYBRID_SHARD over R nodes of D
    ranks ("Building GPT from Scratch — Part 8", "HYBRID_SHARD: The Multi-Node
    Strategy": sharded D ways inside a node, replicated across the nodes).

        1. all-to-all inside the node: rank d receives P_d of its node's D
           gradients, in local rank order;
        2. zero3_node_sum: the node's rank-ordered sum for P_d (fp32, or bf16
           with the bf16 reduce);
        3. all-gather of the node sums across the R replicas of rank d, in node
           order -- the only bytes that leave the node: S sums per rank;
        4. zero3_fold_adamw: the node sums folded in node order, 1/(R*D),
           AdamW on the local fp32 state, the cast to the bf16 shard (every
           replica computes the same bits, so the replicas stay identical);
        5. all-gather of the bf16 shards inside the node into the flat block.

    grad: this rank's full bf16 gradient (N_pad); master, exp_avg, exp_avg_sq:
    fp32 state of P_d (S); work_bf16: the bf16 shard (S); flat: the gathered
    block (N_pad).  node_group and replica_group as hybrid_groups returns them.
    """

    def __init__(self, plan: "z3.Plan", n_nodes: int, grad: torch.Tensor, master: torch.Tensor,
                 exp_avg: torch.Tensor, exp_avg_sq: torch.Tensor, work_bf16: torch.Tensor, flat: torch.Tensor,
                 node_group, replica_group, reduce_dtype: int = z3.Z3_REDUCE_FP32, kernels=z3):
        D, S = plan.D, plan.S
        if dist.get_world_size(node_group) != D or dist.get_world_size(replica_group) != n_nodes:
            raise ValueError(f"need node groups of D = {D} ranks and replica groups of {n_nodes} ranks")
        for name, t, n in (("grad", grad, plan.N_pad), ("flat", flat, plan.N_pad), ("work_bf16", work_bf16, S)):
            if t.dtype != torch.bfloat16 or t.numel() != n or not t.is_contiguous():
                raise ValueError(f"{name} must be a contiguous bf16 tensor of {n} elements")
        self.plan, self.R, self.reduce_dtype, self.k = plan, n_nodes, reduce_dtype, kernels
        self.node_group, self.replica_group = node_group, replica_group
        self.d = dist.get_rank(node_group)
        self.grad, self.master, self.exp_avg, self.exp_avg_sq = grad, master, exp_avg, exp_avg_sq
        self.work, self.flat = work_bf16, flat
        dev = grad.device
        sum_dtype = torch.float32 if reduce_dtype == z3.Z3_REDUCE_FP32 else torch.bfloat16
        self.recv = torch.empty(D * S, dtype=torch.bfloat16, device=dev)
        self.slices = [self.recv[r * S:(r + 1) * S] for r in range(D)]
        self.node_sum = torch.empty(S, dtype=sum_dtype, device=dev)
        self.all_sums = torch.empty(n_nodes * S, dtype=sum_dtype, device=dev)
        self.sums = [self.all_sums[k * S:(k + 1) * S] for k in range(n_nodes)]

    def step(self, hp: "z3.AdamW") -> None:
        k = self.k
        dist.all_to_all_single(self.recv, self.grad, group=self.node_group)
        k.zero3_node_sum(self.plan, self.d, self.slices, self.node_sum, contrib_layout=k.Z3_CONTRIB_OWNED,
                         reduce_dtype=self.reduce_dtype)
        dist.all_gather_into_tensor(self.all_sums, self.node_sum, group=self.replica_group)
        k.zero3_fold_adamw(self.plan, self.d, self.sums, self.master, self.exp_avg, self.exp_avg_sq, self.work, hp,
                           reduce_dtype=self.reduce_dtype)
        dist.all_gather_into_tensor(self.flat, self.work, group=self.node_group)
