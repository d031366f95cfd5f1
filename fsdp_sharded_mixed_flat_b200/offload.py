"""The CPU-offload placement of the optimiser state, streamed through the GPU.

"7.10 — Fully-sharded data parallel (FSDP / ZeRO-3)", §8 (the CPU-offload
variant): the Adam state moves to CPU memory, freeing 12N/D bytes of GPU
memory per device, at the cost of PCIe traffic every step.

Here the state (fp32 master, m, v) lives in page-locked host memory and the
arithmetic stays on the GPU: each step walks the rank partitions P_0..P_{D-1};
for each, a copy-in stream brings the partition's master / m / v into one of
`n_stage` device staging buffers, the compute stream runs the fused reduce +
AdamW + cast kernel on it (rank r, full contribution layout, bf16 output into
the device-resident working shard), and a copy-out stream writes the updated
state back.  The copy engines drive both PCIe directions while the kernel runs.
All arithmetic runs in libzero3.so; torch provides streams, events and copies.

(The kernel can also read and write mapped host memory directly; staging moves
the state in bulk copies, which reach a much larger share of PCIe bandwidth
than the kernel's 16-byte accesses.)
"""
from __future__ import annotations

from typing import Optional, Sequence

import torch

from . import zero3 as z3


class OffloadedState:
    def __init__(self, plan: "z3.Plan", master: torch.Tensor, exp_avg: torch.Tensor, exp_avg_sq: torch.Tensor,
                 work_bf16: torch.Tensor, device, n_stage: int = 3, reduce_dtype: int = z3.Z3_REDUCE_FP32):
        S, N_pad = plan.S, plan.N_pad
        for name, t in (("master", master), ("exp_avg", exp_avg), ("exp_avg_sq", exp_avg_sq)):
            if t.device.type != "cpu" or not t.is_pinned() or t.dtype != torch.float32 or t.numel() < N_pad:
                raise ValueError(f"{name} must be a pinned host float32 tensor of N_pad elements")
        if work_bf16.device.type != "cuda" or work_bf16.numel() < N_pad:
            raise ValueError("work_bf16 must be a device bf16 tensor of N_pad elements")
        self.plan, self.reduce_dtype = plan, reduce_dtype
        self.host = (master, exp_avg, exp_avg_sq)
        self.work = work_bf16
        self.device = torch.device(device)
        self.stage = [torch.empty((3, S), dtype=torch.float32, device=self.device) for _ in range(n_stage)]
        self.copy_in = torch.cuda.Stream(self.device)
        self.compute = torch.cuda.Stream(self.device)
        self.copy_out = torch.cuda.Stream(self.device)
        self.loaded = [torch.cuda.Event() for _ in range(n_stage)]
        self.updated = [torch.cuda.Event() for _ in range(n_stage)]
        self.stored = [torch.cuda.Event() for _ in range(n_stage)]

    def step(self, contribs: Sequence[torch.Tensor], hp: "z3.AdamW",
             k1_events: Optional[Sequence] = None) -> None:
        """One optimiser step over every partition.  contribs: the D device bf16
        contributions in the full layout.  k1_events, if given, holds D (start, end)
        event pairs recorded around the kernels on the compute stream."""
        plan, S = self.plan, self.plan.S
        caller = torch.cuda.current_stream(self.device)
        for s in (self.copy_in, self.compute, self.copy_out):
            s.wait_stream(caller)
        n = len(self.stage)
        for r in range(plan.D):
            b = r % n
            sl = slice(r * S, (r + 1) * S)
            buf = self.stage[b]
            with torch.cuda.stream(self.copy_in):
                self.copy_in.wait_event(self.stored[b])     # the buffer's previous state is back on the host
                for k in range(3):
                    buf[k].copy_(self.host[k][sl], non_blocking=True)
                self.loaded[b].record(self.copy_in)
            self.compute.wait_event(self.loaded[b])
            if k1_events is not None:
                k1_events[r][0].record(self.compute)
            z3.zero3_reduce_adamw(plan, r, contribs, buf[0], buf[1], buf[2], self.work[sl], hp,
                                  contrib_layout=z3.Z3_CONTRIB_FULL, reduce_dtype=self.reduce_dtype,
                                  stream=self.compute)
            if k1_events is not None:
                k1_events[r][1].record(self.compute)
            self.updated[b].record(self.compute)
            with torch.cuda.stream(self.copy_out):
                self.copy_out.wait_event(self.updated[b])
                for k in range(3):
                    self.host[k][sl].copy_(buf[k], non_blocking=True)
                self.stored[b].record(self.copy_out)
        caller.wait_stream(self.compute)
        caller.wait_stream(self.copy_out)
