"""Layer-streamed optimiser step of one rank's resident ZeRO-3 shard.

"7.10 — Fully-sharded data parallel (FSDP / ZeRO-3)", §5.1: the backward pass
visits blocks from last to first and reduce-scatters each block's gradients as
it finishes, so a rank's owned gradient slices arrive one block at a time;
§5.2: at most two block-sized transient buffers are live; §5.4: the transfer
of the next block overlaps the work on the current one.

`LayerStreamer` keeps one rank's owned fp32 master / m / v and bf16 working
shard for L blocks resident in HBM (L x S elements each), and for blocks
L-1 .. 0 in turn: a copy stream fills one of two transient buffers with the
block's D owned contributions (what the reduce-scatter delivers), and the
compute stream runs the fused reduce + AdamW + cast kernel (owned layout) on
that buffer while the other buffer is being filled.  Events order the two
streams; no host synchronisation happens inside a step.  All arithmetic runs in
libzero3.so; torch provides the streams, events and device copies.
"""
from __future__ import annotations

from typing import Callable, Optional, Sequence

import torch

from . import zero3 as z3


class LayerStreamer:
    def __init__(self, plan: "z3.Plan", n_layers: int, rank: int, master: torch.Tensor,
                 exp_avg: torch.Tensor, exp_avg_sq: torch.Tensor, work_bf16: torch.Tensor,
                 reduce_dtype: int = z3.Z3_REDUCE_FP32, compute_priority: int = 0):
        """compute_priority: CUDA stream priority of the compute stream (0 is the
        default, negative is higher).  A higher priority than the copy stream's lets
        the block scheduler start the fused kernel's blocks first and run the
        arrival of the next block's bytes in the SMs it leaves free."""
        S, D = plan.S, plan.D
        for name, t in (("master", master), ("exp_avg", exp_avg), ("exp_avg_sq", exp_avg_sq),
                        ("work_bf16", work_bf16)):
            if t.numel() < n_layers * S:
                raise ValueError(f"{name} must hold n_layers * S = {n_layers * S} elements")
        if not 0 <= rank < D:
            raise ValueError("rank out of range")
        self.plan, self.L, self.rank, self.reduce_dtype = plan, n_layers, rank, reduce_dtype
        self.master, self.exp_avg, self.exp_avg_sq, self.work = master, exp_avg, exp_avg_sq, work_bf16
        dev = master.device
        self.device = dev
        # two transient buffers, each the D owned contributions of one block, back to back
        self.buf = [torch.empty(D * S, dtype=torch.bfloat16, device=dev) for _ in range(2)]
        self.compute = torch.cuda.Stream(dev, priority=compute_priority)
        self.copy = torch.cuda.Stream(dev)
        self.filled = [torch.cuda.Event() for _ in range(2)]
        self.free = [torch.cuda.Event() for _ in range(2)]

    def layer_views(self, layer: int):
        S = self.plan.S
        sl = slice(layer * S, (layer + 1) * S)
        return self.master[sl], self.exp_avg[sl], self.exp_avg_sq[sl], self.work[sl]

    def contributions(self, b: int):
        S = self.plan.S
        return [self.buf[b][d * S:(d + 1) * S] for d in range(self.plan.D)]

    def step(self, source: Optional[Callable[[int], torch.Tensor]], hp: "z3.AdamW",
             k1_events: Optional[Sequence] = None, copy_in: bool = True,
             fill: Optional[Callable[[int, torch.Tensor], None]] = None) -> None:
        """One optimiser step over every block, last to first.

        source(layer) gives the tensor to copy in for that block: D * S bf16, the D
        owned contributions back to back, on the device or in pinned host memory.
        k1_events, if given, is a list of L (start, end) CUDA event pairs recorded
        around each fused-kernel launch on the compute stream.  With copy_in=False
        the kernel reads each block's contributions where source(layer) holds them
        (a device tensor that stays valid for the step) and nothing is copied.
        With fill given, fill(layer, buffer) writes the block's contributions into
        the transient buffer on the copy stream instead of a copy from source."""
        caller = torch.cuda.current_stream(self.device)
        self.copy.wait_stream(caller)
        self.compute.wait_stream(caller)
        S, D = self.plan.S, self.plan.D
        for i, layer in enumerate(range(self.L - 1, -1, -1)):
            b = i & 1
            if not copy_in:
                src = source(layer)
                contribs = [src[d * S:(d + 1) * S] for d in range(D)]
                p, m, v, w = self.layer_views(layer)
                if k1_events is not None:
                    k1_events[i][0].record(self.compute)
                z3.zero3_reduce_adamw(self.plan, self.rank, contribs, p, m, v, w, hp,
                                      contrib_layout=z3.Z3_CONTRIB_OWNED, reduce_dtype=self.reduce_dtype,
                                      stream=self.compute)
                if k1_events is not None:
                    k1_events[i][1].record(self.compute)
                continue
            with torch.cuda.stream(self.copy):
                self.copy.wait_event(self.free[b])          # the kernel two blocks back is done with it
                if fill is not None:
                    fill(layer, self.buf[b])
                else:
                    src = source(layer)
                    self.buf[b].copy_(src, non_blocking=True)
                    if src.is_cuda:
                        src.record_stream(self.copy)
                self.filled[b].record(self.copy)
            self.compute.wait_event(self.filled[b])
            p, m, v, w = self.layer_views(layer)
            if k1_events is not None:
                k1_events[i][0].record(self.compute)
            z3.zero3_reduce_adamw(self.plan, self.rank, self.contributions(b), p, m, v, w, hp,
                                  contrib_layout=z3.Z3_CONTRIB_OWNED, reduce_dtype=self.reduce_dtype,
                                  stream=self.compute)
            if k1_events is not None:
                k1_events[i][1].record(self.compute)
            self.free[b].record(self.compute)
        caller.wait_stream(self.compute)
        caller.wait_stream(self.copy)
