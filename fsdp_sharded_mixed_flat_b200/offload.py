"""The CPU-offload variant of the step: the optimiser state in host memory.

"7.10 — Fully-sharded data parallel (FSDP / ZeRO-3)", §8 (the CPU-offload
variant): the Adam state moves to CPU memory, freeing 12N/D bytes of GPU
memory per device, at the cost of PCIe traffic every step.  Two placements of
the arithmetic are built here; both give the fused kernel's results bit for
bit.

HostAdamWOffload is the page's own design: the GPU reduces the owned gradient
shard, the shard goes down over PCIe, AdamW runs on the host (libzero3's host
threads), and the new bf16 weights come back up -- 6 bytes per parameter
crossing PCIe per step with the fp32 reduce, 4 with the bf16 reduce.

OffloadedState keeps the arithmetic on the GPU instead: each step walks the
rank partitions P_0..P_{D-1}; for each, a copy-in stream brings the
partition's master / m / v into one of `n_stage` device staging buffers, the
compute stream runs the fused reduce + AdamW + cast kernel on it (rank r, full
contribution layout, bf16 output into the device-resident working shard), and
a copy-out stream writes the updated state back -- 24 bytes per parameter
crossing PCIe, with the copy engines driving both directions while the kernel
runs.  (The kernel can also read and write mapped host memory directly;
staging moves the state in bulk copies, which reach a much larger share of
PCIe bandwidth than the kernel's 16-byte accesses.)

All arithmetic runs in libzero3.so; torch provides streams, events and copies.
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


class HostAdamWOffload:
    """The CPU-offload variant as "7.10 — Fully-sharded data parallel (FSDP /
    ZeRO-3)", §8 describes it: the Adam state (fp32 master, m, v) lives in
    page-locked host memory and the optimiser runs on the host; every step
    sends the averaged gradient down and pulls the updated bf16 weights back
    over PCIe -- 4 bytes per parameter down (2 with the bf16 reduce) and 2 up,
    against the 12 bytes of state each way that OffloadedState moves.

    Per step, unit by unit (each partition P_0 .. P_{D-1} cut into `chunks`
    consecutive pieces), pipelined:
      compute stream  zero3_reduce_scatter of the unit -> one of `n_stage`
                      device staging buffers (the unit's averaged gradient);
      copy-down       the staging buffer -> the unit's slot of a pinned host
                      gradient buffer;
      host            waits for that copy only, then zero3_host_adamw on the
                      unit (libzero3's host threads: same operations, same bits
                      as the GPU kernels) writing its bf16 weights to a pinned
                      host buffer;
      copy-up         the unit's bf16 weights -> the device working shard.
    The GPU reduces and copies the next units down while the host updates this
    one, and this unit's weights go up while the host updates the next.  Smaller
    units start the host sooner and leave a shorter copy up at the end.  A unit
    of rank r's partition is reduced as a plan of its own (D ranks of the
    unit's length, the contributions in the owned layout at the unit's offset),
    so the arithmetic is the partition's, element for element.  The step
    returns once the last host update has run; the caller's stream is ordered
    after the last copy up, so kernels it enqueues next see every new weight.
    """

    def __init__(self, plan: "z3.Plan", master: torch.Tensor, exp_avg: torch.Tensor, exp_avg_sq: torch.Tensor,
                 work_bf16: torch.Tensor, device, n_stage: int = 3, reduce_dtype: int = z3.Z3_REDUCE_FP32,
                 n_threads: int = 0, chunks: int = 1):
        S, N_pad = plan.S, plan.N_pad
        for name, t in (("master", master), ("exp_avg", exp_avg), ("exp_avg_sq", exp_avg_sq)):
            if t.device.type != "cpu" or t.dtype != torch.float32 or t.numel() < N_pad or not t.is_contiguous():
                raise ValueError(f"{name} must be a contiguous host float32 tensor of N_pad elements")
        if work_bf16.device.type != "cuda" or work_bf16.numel() < N_pad:
            raise ValueError("work_bf16 must be a device bf16 tensor of N_pad elements")
        if n_stage < 1 or chunks < 1:
            raise ValueError("n_stage and chunks must be >= 1")
        self.plan, self.reduce_dtype, self.n_threads = plan, reduce_dtype, n_threads
        self.host = (master, exp_avg, exp_avg_sq)
        self.work = work_bf16
        self.device = torch.device(device)
        # units: (rank, first element within the partition, length); cuts on 128-element
        # boundaries keep every unit's vectors 16-byte aligned
        step = max(128, -(-(-(-S // chunks)) // 128) * 128)
        self.units = [(r, c0, min(step, S - c0)) for r in range(plan.D) for c0 in range(0, S, step)]
        self._plans = {}
        gdt = torch.float32 if reduce_dtype == z3.Z3_REDUCE_FP32 else torch.bfloat16
        self.grad_host = torch.empty(N_pad, dtype=gdt, pin_memory=True)
        self.work_host = torch.empty(N_pad, dtype=torch.bfloat16, pin_memory=True)
        self.stage = [torch.empty(min(step, max(S, 1)), dtype=gdt, device=self.device) for _ in range(n_stage)]
        self.compute = torch.cuda.Stream(self.device)
        self.down = torch.cuda.Stream(self.device)
        self.up = torch.cuda.Stream(self.device)
        self.reduced = [torch.cuda.Event() for _ in range(n_stage)]
        self.staged_free = [torch.cuda.Event() for _ in range(n_stage)]
        self.arrived = [torch.cuda.Event() for _ in self.units]      # the unit's gradient is on the host
        self.bytes_down = N_pad * self.grad_host.element_size()
        self.bytes_up = N_pad * 2

    def _unit_plan(self, length: int) -> "z3.Plan":
        if length not in self._plans:
            self._plans[length] = z3.zero3_plan([(length * self.plan.D,)], self.plan.D, 1)
        return self._plans[length]

    def _reduce_and_send(self, contribs, u: int, k_events) -> None:
        r, c0, n = self.units[u]
        lo = r * self.plan.S + c0
        b = u % len(self.stage)
        self.compute.wait_event(self.staged_free[b])   # the staging buffer's previous copy down is done
        if k_events is not None:
            k_events[u][0].record(self.compute)
        z3.zero3_reduce_scatter(self._unit_plan(n), 0, [c[lo:lo + n] for c in contribs], self.stage[b],
                                contrib_layout=z3.Z3_CONTRIB_OWNED, reduce_dtype=self.reduce_dtype,
                                stream=self.compute)
        if k_events is not None:
            k_events[u][1].record(self.compute)
        self.reduced[b].record(self.compute)
        with torch.cuda.stream(self.down):
            self.down.wait_event(self.reduced[b])
            self.grad_host[lo:lo + n].copy_(self.stage[b][:n], non_blocking=True)
            self.staged_free[b].record(self.down)
            self.arrived[u].record(self.down)

    def step(self, contribs: Sequence[torch.Tensor], hp: "z3.AdamW", k_events: Optional[Sequence] = None,
             host_seconds: Optional[list] = None) -> None:
        """One optimiser step over every partition.  contribs: the D device bf16
        contributions in the full layout.  k_events, if given, holds one (start,
        end) event pair per unit (len(self.units)), recorded around the reduce
        kernels; host_seconds, if given, receives the wall time of each unit's
        host update."""
        import time
        if len(contribs) != self.plan.D:
            raise ValueError(f"need {self.plan.D} contributions")
        caller = torch.cuda.current_stream(self.device)
        for s in (self.compute, self.down, self.up):
            s.wait_stream(caller)
        n = len(self.stage)
        U = len(self.units)
        for u in range(min(n, U)):
            self._reduce_and_send(contribs, u, k_events)
        master, exp_avg, exp_avg_sq = self.host
        for u in range(U):
            self.arrived[u].synchronize()                # only this unit's copy down
            if u + n < U:
                self._reduce_and_send(contribs, u + n, k_events)
            r, c0, length = self.units[u]
            sl = slice(r * self.plan.S + c0, r * self.plan.S + c0 + length)
            t0 = time.perf_counter()
            z3.zero3_host_adamw(self.grad_host[sl], master[sl], exp_avg[sl], exp_avg_sq[sl], self.work_host[sl], hp,
                                n_threads=self.n_threads)
            if host_seconds is not None:
                host_seconds.append(time.perf_counter() - t0)
            with torch.cuda.stream(self.up):
                self.work[sl].copy_(self.work_host[sl], non_blocking=True)
        caller.wait_stream(self.up)
        caller.wait_stream(self.compute)
        caller.wait_stream(self.down)
