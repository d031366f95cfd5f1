"""One block's optimiser step as a CUDA graph, replayed step after step.

The step-dependent AdamW scalars are the only thing that changes between
steps; the fused kernel reads them from a 32-byte device buffer
(zero3_reduce_adamw_dev), so the launches are captured once:

    ZeRO-3  (stage 3): fused reduce + AdamW + cast, then the gather of the shards
                       into the flat block;
    ZeRO-1/2 (stage 1, 2): the fused kernel writing the gathered block directly.

Each step the host forms the scalars (zero3_step_scalars) in a slot of a ring
of pinned host buffers, enqueues their copy into the device buffer and replays
the graph, both on the caller's stream, so the host never waits for the GPU
unless it has run a whole ring ahead.  All arithmetic runs in libzero3.so;
torch provides the graph, streams, events and copies.
"""
from __future__ import annotations

from typing import Optional, Sequence

import torch

from . import zero3 as z3

RING = 64


class GraphedStep:
    def __init__(self, plan: "z3.Plan", contribs: Sequence[torch.Tensor], master: torch.Tensor,
                 exp_avg: torch.Tensor, exp_avg_sq: torch.Tensor, work_bf16: Optional[torch.Tensor],
                 flat: Optional[torch.Tensor], stage: int = 3, reduce_dtype: int = z3.Z3_REDUCE_FP32):
        if stage == 3 and (work_bf16 is None or flat is None):
            raise ValueError("the ZeRO-3 step needs the bf16 shards (work_bf16) and the flat block")
        if stage != 3 and flat is None:
            raise ValueError("the ZeRO-1/2 step needs the gathered block (flat)")
        dev = master.device
        self.device, self.plan, self.stage = dev, plan, stage
        self.scalars = torch.zeros(z3.Z3_SCALARS, dtype=torch.float32, device=dev)
        self.pinned = torch.zeros((RING, z3.Z3_SCALARS), dtype=torch.float32, pin_memory=True)
        self.copied = [None] * RING
        self.i = 0
        S, D = plan.S, plan.D
        shards = None if work_bf16 is None else [work_bf16[r * S:(r + 1) * S] for r in range(D)]

        def launches(stream):
            if stage == 3:
                z3.zero3_reduce_adamw_dev(plan, -1, contribs, master, exp_avg, exp_avg_sq, work_bf16, [],
                                          self.scalars, reduce_dtype=reduce_dtype, stream=stream)
                z3.zero3_gather_block(plan, shards, flat, None, stream=stream)
            else:
                z3.zero3_reduce_adamw_dev(plan, -1, contribs, master, exp_avg, exp_avg_sq, work_bf16, [flat],
                                          self.scalars, reduce_dtype=reduce_dtype, stream=stream)

        self._warm_up(plan, stage, reduce_dtype)
        side = torch.cuda.Stream(dev)
        side.wait_stream(torch.cuda.current_stream(dev))
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph, stream=side):
            launches(side)
        torch.cuda.current_stream(dev).wait_stream(side)

    def _warm_up(self, plan, stage, reduce_dtype):
        """Run the same kernels once on a small scratch block, through both the
        16-byte vector path and the scalar path (buffers one element off), so that
        whichever kernel the graph captures is loaded before capture; the real
        state is not touched."""
        dev = self.device
        D = plan.D
        tiny = z3.zero3_plan([(D * plan.align_elems,)], D, plan.align_elems)
        n = tiny.N_pad
        sc = torch.zeros(z3.Z3_SCALARS, dtype=torch.float32, device=dev)
        sc.copy_(torch.tensor(z3.zero3_step_scalars(z3.adamw(step=1)), dtype=torch.float32))
        for skew in (0, 1):
            def buf(dtype):
                return torch.zeros(n + skew, dtype=dtype, device=dev)[skew:]
            c = [buf(torch.bfloat16) for _ in range(D)]
            p, m, v = buf(torch.float32), buf(torch.float32), buf(torch.float32)
            w, f = buf(torch.bfloat16), buf(torch.bfloat16)
            if stage == 3:
                z3.zero3_reduce_adamw_dev(tiny, -1, c, p, m, v, w, [], sc, reduce_dtype=reduce_dtype)
                z3.zero3_gather_block(tiny, [w[r * tiny.S:(r + 1) * tiny.S] for r in range(D)], f, None)
            else:
                z3.zero3_reduce_adamw_dev(tiny, -1, c, p, m, v, None, [f], sc, reduce_dtype=reduce_dtype)
        torch.cuda.synchronize(dev)

    def step(self, hp: "z3.AdamW") -> None:
        """Enqueue one step with hyper-parameters hp on the current stream."""
        stream = torch.cuda.current_stream(self.device)
        k = self.i % RING
        self.i += 1
        if self.copied[k] is not None:
            self.copied[k].synchronize()        # the slot's previous copy has been read
        z3.zero3_step_scalars(hp, self.pinned[k].data_ptr())
        self.scalars.copy_(self.pinned[k], non_blocking=True)
        ev = self.copied[k] or torch.cuda.Event()
        ev.record(stream)
        self.copied[k] = ev
        self.graph.replay()
