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
streams; no host synchronisation happens inside a step.

`PrefetchSweep` is the other side of the same sweep: before block l runs, its
D shards are all-gathered into one of two transient gathered buffers, and the
gather of block l-1 is issued on a side stream while block l is used and its
partition updated (the prefetch of §5.4 within the two buffers of §5.2).

All arithmetic runs in libzero3.so; torch provides the streams, events and
device copies.
"""
from __future__ import annotations

from typing import Callable, Optional, Sequence

import torch

from . import zero3 as z3


class LayerStreamer:
    def __init__(self, plan: "z3.Plan", n_layers: int, rank: int, master: torch.Tensor,
                 exp_avg: torch.Tensor, exp_avg_sq: torch.Tensor, work_bf16: torch.Tensor,
                 reduce_dtype: int = z3.Z3_REDUCE_FP32):
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
        self.compute = torch.cuda.Stream(dev)
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


class PrefetchSweep:
    """One rank's backward sweep over L blocks with the next block's all-gather
    prefetched into one of two transient buffers.

    "7.10 — Fully-sharded data parallel (FSDP / ZeRO-3)", §5.1: in the backward
    pass each block, last to first, is gathered whole (full_params =
    all_gather of the D shards), used, then freed, and its gradients are
    reduce-scattered to the owners, which update their partition; §5.2: two
    block-sized transient buffers are live at most (one in use, one being
    filled); §5.4 and "Building GPT from Scratch — Part 8", "Prefetching:
    Hiding the Cost": the all-gather of the next block is issued while the
    current block computes.

    For blocks l = L-1 .. 0 (step i):
      gather stream   waits until buffer (i+1) mod 2 is released by the block
                      that used it two steps back, then gathers block l-1's D
                      shards into it (zero3_gather_block) -- issued before
                      block l's work, so it overlaps it;
      main stream     waits for block l's gather, runs consume(l, buffer) (the
                      block's use of its gathered weights, e.g. its backward
                      compute; optional), releases the buffer, then the fused
                      reduce + AdamW + cast of this rank's partition of block
                      l (owned layout), whose new bf16 shard is block l's
                      shards[l][rank].
    Events order the two streams; the host never waits inside a sweep.  With
    prefetch=False every gather runs on the main stream right before its
    block (the serial order, for comparison).

    shards[l]  the D bf16 shards (S elements each) of block l: the rank's own
               and, in this one-GPU simulation, the other ranks' (on D GPUs
               they would be the peers' shards, read over peer memory).
    master, exp_avg, exp_avg_sq  fp32, L x S: this rank's state, block by block.
    """

    def __init__(self, plan: "z3.Plan", shards: Sequence[Sequence[torch.Tensor]], rank: int, master: torch.Tensor,
                 exp_avg: torch.Tensor, exp_avg_sq: torch.Tensor, reduce_dtype: int = z3.Z3_REDUCE_FP32):
        S, D, L = plan.S, plan.D, len(shards)
        if not 0 <= rank < D:
            raise ValueError("rank out of range")
        if any(len(s) != D for s in shards):
            raise ValueError(f"every block needs its {D} shards")
        for name, t in (("master", master), ("exp_avg", exp_avg), ("exp_avg_sq", exp_avg_sq)):
            if t.numel() < L * S:
                raise ValueError(f"{name} must hold L * S = {L * S} elements")
        self.plan, self.shards, self.rank, self.L, self.reduce_dtype = plan, shards, rank, L, reduce_dtype
        self.master, self.exp_avg, self.exp_avg_sq = master, exp_avg, exp_avg_sq
        dev = master.device
        self.device = dev
        # exactly two transient gathered blocks, as the memory ledger counts them
        self.gathered = [torch.empty(plan.N_pad, dtype=torch.bfloat16, device=dev) for _ in range(2)]
        self.transient_bytes = sum(g.numel() * g.element_size() for g in self.gathered)
        if self.transient_bytes != z3.zero3_transient_bytes(plan.N_pad, 2):
            raise AssertionError("the transient buffers differ from the ledger's two gathered blocks")
        self.side = torch.cuda.Stream(dev)
        self.ready = [torch.cuda.Event() for _ in range(2)]
        self.free = [torch.cuda.Event() for _ in range(2)]

    def state_views(self, layer: int):
        S = self.plan.S
        sl = slice(layer * S, (layer + 1) * S)
        return self.master[sl], self.exp_avg[sl], self.exp_avg_sq[sl]

    def step(self, contributions: Callable[[int], Sequence[torch.Tensor]], hp: "z3.AdamW",
             consume: Optional[Callable[[int, torch.Tensor], None]] = None, prefetch: bool = True,
             events: Optional[dict] = None) -> None:
        """One sweep.  contributions(l): the D owned bf16 contributions of block l
        (S elements each, what the reduce-scatter delivers to this rank).  events,
        if given, maps "gather" and "k1" to lists that receive (start, end) CUDA
        event pairs recorded around every gather and fused-kernel launch."""
        main = torch.cuda.current_stream(self.device)
        self.side.wait_stream(main)
        order = list(range(self.L - 1, -1, -1))

        def timed(kind, stream, fn):
            if events is None:
                fn()
                return
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fn()
            b.record(stream)
            events.setdefault(kind, []).append((a, b))

        def gather(i, stream):
            layer, b = order[i], i & 1
            timed("gather", stream, lambda: z3.zero3_gather_block(self.plan, self.shards[layer], self.gathered[b],
                                                                  stream=stream))

        def prefetch_gather(i):
            b = i & 1
            self.side.wait_event(self.free[b])          # released by the block two steps back
            gather(i, self.side)
            self.ready[b].record(self.side)

        if prefetch:
            prefetch_gather(0)
        for i, layer in enumerate(order):
            b = i & 1
            if prefetch:
                if i + 1 < self.L:
                    prefetch_gather(i + 1)              # block l-1, into the other buffer
                main.wait_event(self.ready[b])
            else:
                gather(i, main)
            if consume is not None:
                consume(layer, self.gathered[b])
            self.free[b].record(main)
            p, m, v = self.state_views(layer)
            timed("k1", main, lambda: z3.zero3_reduce_adamw(
                self.plan, self.rank, contributions(layer), p, m, v, self.shards[layer][self.rank], hp,
                contrib_layout=z3.Z3_CONTRIB_OWNED, reduce_dtype=self.reduce_dtype, stream=main))
        main.wait_stream(self.side)
