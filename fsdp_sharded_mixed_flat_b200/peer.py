"""The per-rank step of a real D-GPU ZeRO group on one node, over NVLink.

One process per GPU, ranks 0..D-1 of a torch.distributed group.  Each rank
shares its full bf16 gradient buffer (and its bf16 working shard, or its
gathered block) with every other rank through CUDA IPC, so the library's
kernels can address the peers' memory with plain loads and stores:

  ZeRO-3 ("7.10 — Fully-sharded data parallel (FSDP / ZeRO-3)", §5.1; "Building
  GPT from Scratch — Part 8", "AllGather vs AllReduce"):
    1. every rank's gradient is complete (stream synchronised, then a barrier);
    2. the fused kernel on rank r reads slice P_r of every rank's gradient in
       rank order 0..D-1 through the peer mappings (the reduce-scatter's data
       movement as P2P loads over NVLink), reduces, runs AdamW on the local
       fp32 state and writes the local bf16 shard;
    3. every rank's shard is updated (synchronise, barrier);
    4. the gather kernel pulls all D shards into the local gathered block
       (the all-gather as P2P loads).
  ZeRO-1 / ZeRO-2 (§3, §4): step 2's kernel also stores the new shard into
  every rank's gathered block (P2P stores; at most Z3_GATHER_MAX ranks), and a
  final barrier replaces steps 3-4.

The mappings come from libzero3's IPC entry points, which map each peer
allocation into the address space of the importing rank's own device with peer
access enabled, so the kernels launched there can address it.  Every wait is a
host-side stream synchronisation followed by a group barrier, so no kernel ever
waits on another rank; the barriers take the process group's timeout.  The kernels reach the peers' memory with plain loads and stores only (no
TMA), and no library kernel is ever handed a peer's memory: only libzero3.so's
own kernels touch the mappings.
"""
from __future__ import annotations

from typing import Callable, List, Optional

import torch
import torch.distributed as dist

from . import zero3 as z3


class PeerGroup:
    """The ranks of a process group, with CUDA IPC sharing of device tensors.

    By default a rank exports the allocation holding its tensor through
    libzero3 (zero3_ipc_export) and every other rank maps it into the address
    space of ITS OWN device (zero3_ipc_import, peer access to the owning GPU
    enabled as needed), the device its kernels launch on; the mapped view
    aliases the other rank's memory.  share_fn / open_fn replace the exchange
    (host tests use stand-ins)."""

    def __init__(self, group=None, share_fn: Optional[Callable] = None, open_fn: Optional[Callable] = None,
                 sync_fn: Optional[Callable] = None):
        self.group = group
        self.rank = dist.get_rank(group)
        self.size = dist.get_world_size(group)
        self._sync = sync_fn or (lambda device: torch.cuda.current_stream(device).synchronize())
        self._device = None
        self._mappings: List[int] = []
        if share_fn is None or open_fn is None:
            share_fn, open_fn = self._export, self._import
        self._share, self._open = share_fn, open_fn

    @staticmethod
    def _export(t: torch.Tensor):
        handle, offset, size = z3.zero3_ipc_export(t)
        return handle, offset, size, t.numel(), str(t.dtype).replace("torch.", "")

    def _import(self, shared) -> torch.Tensor:
        handle, offset, size, numel, dtype = shared
        view, base = z3.zero3_ipc_import(handle, offset, size, numel, getattr(torch, dtype), self._device)
        self._mappings.append(base)
        return view

    def share(self, t: torch.Tensor) -> List[torch.Tensor]:
        """Every rank's tensor `t`, in rank order: this rank's own, the others
        mapped into this process for the device `t` lives on."""
        if self.size == 1:
            return [t]                              # nobody to share with
        handles = [None] * self.size
        dist.all_gather_object(handles, self._share(t), group=self.group)
        self._device = t.get_device() if t.is_cuda else None
        return [t if k == self.rank else self._open(h) for k, h in enumerate(handles)]

    def close(self) -> None:
        """Release this rank's mappings of the other ranks' memory.  Call it once
        every kernel that reads or writes them has finished (after a fence)."""
        while self._mappings:
            z3.zero3_ipc_close(self._mappings.pop(), self._device)

    def fence(self, device) -> None:
        """Everything this rank enqueued on its current stream has finished, and so
        has every other rank's (a stream synchronisation, then a group barrier)."""
        self._sync(device)
        dist.barrier(group=self.group)


class PeerZero3Step:
    """Rank r's optimiser step in a D-GPU group (D = the group's size).

    grad:      this rank's full bf16 gradient of the block (N_pad elements).
    master, exp_avg, exp_avg_sq: this rank's fp32 state for P_r (S elements).
    work_bf16: this rank's bf16 working shard (S elements).
    flat:      this rank's gathered block (N_pad elements).
    stage:     3 (gather pulled after the update) or 1/2 (pushed by the kernel).
    """

    def __init__(self, peers: PeerGroup, plan: "z3.Plan", grad: torch.Tensor, master: torch.Tensor,
                 exp_avg: torch.Tensor, exp_avg_sq: torch.Tensor, work_bf16: torch.Tensor, flat: torch.Tensor,
                 stage: int = 3, reduce_dtype: int = z3.Z3_REDUCE_FP32, kernels=z3):
        if plan.D != peers.size:
            raise ValueError(f"the plan is for D = {plan.D} ranks, the group has {peers.size}")
        if stage != 3 and peers.size > z3.Z3_GATHER_MAX:
            raise ValueError(f"the fused all-gather writes at most {z3.Z3_GATHER_MAX} gathered blocks")
        self.peers, self.plan, self.stage, self.reduce_dtype, self.k = peers, plan, stage, reduce_dtype, kernels
        self.rank = peers.rank
        self.device = grad.device
        self.master, self.exp_avg, self.exp_avg_sq, self.work, self.flat = master, exp_avg, exp_avg_sq, work_bf16, flat
        self.grads = peers.share(grad)                      # D gradient buffers, rank order
        if stage == 3:
            self.shards = peers.share(work_bf16)            # D bf16 shards, rank order
        else:
            self.flats = peers.share(flat)                  # D gathered blocks, rank order

    def step(self, hp: "z3.AdamW", mark=None, marks: Optional[list] = None) -> None:
        """One step.  With mark (a callable returning a time mark, e.g. a CUDA event
        recorded on the current stream) and marks (a list), the marks around the
        fences and kernels are appended to marks as one tuple: (before the first
        fence, after it, after the fused kernel, after the second fence, after the
        gather) at stage 3; (before the first fence, after it, after the fused
        kernel, after the last fence) otherwise."""
        k = self.k
        t = [mark()] if mark else None
        self.peers.fence(self.device)                       # every rank's gradient is complete
        if t is not None:
            t.append(mark())
        if self.stage == 3:
            k.zero3_reduce_adamw(self.plan, self.rank, self.grads, self.master, self.exp_avg, self.exp_avg_sq,
                                 self.work, hp, contrib_layout=k.Z3_CONTRIB_FULL, reduce_dtype=self.reduce_dtype)
            if t is not None:
                t.append(mark())
            self.peers.fence(self.device)                   # every rank's shard is updated
            if t is not None:
                t.append(mark())
            k.zero3_gather_block(self.plan, self.shards, self.flat, None)
        else:
            k.zero3_reduce_adamw_gather(self.plan, self.rank, self.grads, self.master, self.exp_avg,
                                        self.exp_avg_sq, self.work, self.flats, hp,
                                        contrib_layout=k.Z3_CONTRIB_FULL, reduce_dtype=self.reduce_dtype)
            if t is not None:
                t.append(mark())
            self.peers.fence(self.device)                   # every rank's pushes have landed
        if t is not None:
            t.append(mark())
            marks.append(tuple(t))
