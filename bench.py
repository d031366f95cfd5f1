"""Benchmark of one ZeRO-3 per-rank step on B200: the fused reduce-scatter
reduction + AdamW + bf16 cast over every owned partition of a LLaMA-7B decoder
block at D = 8 simulated ranks, then the all-gather of the 8 bf16 shards into
the flat block (with zero-copy per-tensor views) and the host-side plan and
memory ledger.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--D D] [--reduce-dtype fp32|bf16] [--stage 1|2|3]
                    [--graph] [--offload [state|host]] [--unflatten-copy] [--refill copy|fill|memset] [--drift]

One process per GPU (torchrun for N > 1).  With N = 1 the block's D ranks are
simulated on the one GPU.  With N > 1 the block is sharded over the N GPUs
(D = N, strong scaling: one block per step in all): the fused kernel on each
rank reads its partition of every rank's gradient through CUDA IPC mappings
with plain loads over NVLink (the reduce-scatter's data movement inside the
optimiser kernel) and updates the rank's state and bf16 shard, and the gather
kernel reads every rank's shard into the local block.  The line then also
times the same step with an NCCL all-to-all and all-gather around the fused
kernel (`baseline_nccl`; --transport nccl makes that form the headline).
--replicas runs N independent single-GPU replicas instead.  Rank 0 prints one
JSON line.

Timing: W untimed warm-up steps, then K steps between a barrier plus
cudaDeviceSynchronize on each side, timed with CUDA events on the launching
stream, max over ranks.  Each step streams about 9.3 GB through HBM, far more
than the 126 MB L2, so no flush is needed between steps.  The fused kernel is
also timed launch by launch with its own events for the roofline figure.

Workloads (--workload): llama7b_d8 (default), llama7b_d32, llama7b_policy (with
--D), llama7b_hybrid (HYBRID_SHARD, 4 nodes of 8), llama70b_shard (one rank's
80-layer shard, streamed), tiny_gpt, and the small profiling slices
profile_d8 and profile_hybrid.

Besides the throughput, the line carries the roofline of the fused kernel, the
SM clocks seen during the timed region, an end-to-end figure through the public
API from pinned host buffers, the memory ledger, and (N = 1, rank 0) the CPU
baseline: the oracle timed on one host core on a bounded sample, with our path
checked against it on that same sample (parity_vs_oracle).

--impl reference times the oracle (plain single-threaded C) on the host on a
bounded sample of the same workload; it is a deliberately slow baseline.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "owned params/s for fused reduce+AdamW+cast; achieved HBM GB/s vs ~8 TB/s"
UNIT = "owned params/s"
NVLINK_GBS = 770.0   # measured B200 peer copy over NVLink 5, per direction per GPU (900 GB/s nominal)
# committed ncu summaries of the fused kernel, by workload (fp32 reduce), with its DRAM traffic
PROFILE_K1 = {"llama7b_d8": os.path.join(ROOT, "profiles", "k_reduce_adamw_vec_llama7b_d8.md"),
              "llama7b_hybrid": os.path.join(ROOT, "profiles", "k_reduce_adamw_vec_hybrid_llama7b_4x8.md")}
# the sources whose code makes up the fused kernel
K1_SOURCES = [os.path.join(ROOT, "fsdp_sharded_mixed_flat_b200", "csrc", f)
              for f in ("reduce_adamw.cu", "step_common.cuh", "adamw_scalars.h")]
SLOW_REASONS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown")


# How the 70B shard's per-layer contributions arrive in a transient buffer (the
# reduce-scatter's delivery, simulated on one GPU).
# Measured on B200 for the 80-layer step: copy 93.8 ms, fill 85.9 ms (torch's
# bf16 fill kernel writes at about 3.9 TB/s), memset 70.0 ms (the CUDA driver's
# memset writes at about 6.8 TB/s).
ARRIVALS = {
    "copy": "device-to-device copy from a pool on the copy stream (read + write)",
    "fill": "write-only fill of the transient buffer by torch's fill kernel on the copy stream",
    "memset": "write-only cudaMemsetAsync of the transient buffer on the copy stream, as a delivery over NVLink "
              "writes it",
}
DEFAULT_ARRIVAL = "memset"


def parse_args(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=400)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="llama7b_d8")
    ap.add_argument("--e2e-steps", type=int, default=12)
    ap.add_argument("--cpu-sample", type=int, default=1 << 24, help="elements of the oracle's sample")
    ap.add_argument("--cpu-steps", type=int, default=20,
                    help="most oracle steps in the CPU baseline; fewer when a step takes long (about 10 s in all)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--D", type=int, default=0, help="simulated ranks (default: the workload's)")
    ap.add_argument("--reduce-dtype", choices=["fp32", "bf16"], default="fp32")
    ap.add_argument("--offload", nargs="?", const="state", default=None, choices=["state", "host"],
                    help="fp32 master / m / v in page-locked host memory: 'state' streams it through the GPU, "
                         "which keeps the arithmetic (24 B per param over PCIe); 'host' runs AdamW on the host, "
                         "with the averaged gradient down and the bf16 weights up (6 B per param, 4 in bf16)")
    ap.add_argument("--refill", choices=list(ARRIVALS), default=DEFAULT_ARRIVAL,
                    help="70B shard: how each layer's contributions arrive in the transient buffer: "
                         + "; ".join(f"{k}: {v}" for k, v in ARRIVALS.items()))
    ap.add_argument("--offload-chunks", type=int, default=1,
                    help="--offload host: pipeline units per rank partition")
    ap.add_argument("--replicas", action="store_true",
                    help="N > 1: run N independent single-GPU replicas (each simulating its own D ranks) instead "
                         "of the real D-GPU step with D = N")
    ap.add_argument("--transport", choices=["nccl", "peer"], default="peer",
                    help="N > 1: how the D-GPU step moves its bytes: the kernels' own plain loads of the peers' "
                         "memory through CUDA IPC mappings (the reduce-scatter fused into the optimiser kernel; "
                         "the default), or NCCL all-to-all and all-gather around the fused kernel (the baseline)")
    ap.add_argument("--no-nccl-baseline", action="store_true",
                    help="N > 1 with --transport peer: skip the NCCL form of the same step, which the line "
                         "otherwise times after the headline as `baseline_nccl`")
    ap.add_argument("--sweep-steps", type=int, default=10,
                    help="timed steps per configuration in the sweep of the target configurations")
    ap.add_argument("--no-sweep", action="store_true",
                    help="skip the sweep of the target configurations (one GPU only)")
    ap.add_argument("--graph", action="store_true",
                    help="capture the step's launches in a CUDA graph once and replay it every step")
    ap.add_argument("--unflatten-copy", action="store_true",
                    help="the gather also copies every tensor into its own buffer (straight from the shards)")
    ap.add_argument("--drift", action="store_true",
                    help="report the drift of the bf16-reduce path against the fp32-reduce path")
    ap.add_argument("--drift-elements", type=int, default=1 << 24)
    ap.add_argument("--nodes", type=int, default=0,
                    help="HYBRID_SHARD workload: number of nodes (default: the workload's)")
    ap.add_argument("--split", action="store_true",
                    help="HYBRID_SHARD workload: the node sums of every node, then their fold (two kernels, what "
                         "separate machines run) instead of the fused kernel")
    ap.add_argument("--stage", type=int, choices=[1, 2, 3], default=3,
                    help="3: ZeRO-3 step (fused reduce/AdamW/cast, then the gather of the shards); "
                         "1 or 2: the fused kernel also all-gathers into the replicated bf16 weights")
    return ap.parse_args(argv)


def host_info() -> dict:
    """The host the CPU baseline ran on: logical CPUs and the CPU model."""
    model = None
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return {"nproc": os.cpu_count(), "cpu_model": model}


def ledger(z3, N: int, N_pad: int, D: int, block_params: int) -> dict:
    """The memory ledger (bytes per device, per stage) for N real and N_pad padded
    parameters over D ranks, the transient bytes of two gathered blocks, and the
    bytes one device receives in the all-gathers of one pass over the blocks."""
    stages = {"ddp": 0, "zero1": 1, "zero2": 2, "zero3": 3}
    n_blocks = N_pad // block_params if block_params else 0
    return {"N": {k: z3.zero3_memory_bytes(N, D, v) for k, v in stages.items()},
            "N_pad": {k: z3.zero3_memory_bytes(N_pad, D, v) for k, v in stages.items()},
            "transient_2_blocks": z3.zero3_transient_bytes(block_params, 2),
            "allgather_per_pass": z3.zero3_allgather_bytes(block_params, n_blocks, D)}


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def code_sha256(paths) -> str:
    """sha256 of the code in the given C/CUDA sources, with // comments, trailing
    blanks and empty lines removed: a profile taken on some code stays matched
    to it through comment edits, and any change of code breaks the match."""
    lines = []
    for path in paths:
        for line in open(path, encoding="utf-8"):
            code = line.split("//", 1)[0].rstrip()
            if code:
                lines.append(code)
    return hashlib.sha256("\n".join(lines).encode()).hexdigest()


def profiled_traffic(workload: str):
    """DRAM bytes per launch from the committed ncu summary of the fused kernel on
    this workload, if that summary was taken on the kernel's current code; else None."""
    path = PROFILE_K1.get(workload)
    if path is None or not os.path.exists(path):
        return None
    text = open(path).read()
    sha = re.search(r"code_sha256:\s*([0-9a-f]{64})", text)
    tb = re.search(r"traffic_bytes_per_launch:\s*([0-9.eE+]+)", text)
    if not sha or not tb:
        return None
    return float(tb.group(1)) if sha.group(1) == code_sha256(K1_SOURCES) else None


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during the timed region."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_uuid: str | None):
        self.uuid = device_uuid
        self.proc = None
        self.lines: list[str] = []

    def start(self):
        cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "50"]
        if self.uuid:
            cmd += ["-i", self.uuid]
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.reader = threading.Thread(target=self._read, daemon=True)
        self.reader.start()
        time.sleep(0.3)

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.2)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, mx, reasons, power = [], [], set(), []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
                power.append(float(parts[2]))
            except ValueError:
                continue
            for n, val in zip(names, parts[4:8]):
                if val.lower().startswith("active"):
                    reasons.add(n)
        loaded = [s for s, p in zip(sm, power) if p > 300.0] or sm
        return {"sm_mhz": statistics.median(loaded) if loaded else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": sorted(reasons),
                "slowdown_seen": any(r in SLOW_REASONS for r in reasons),
                "samples": len(sm), "samples_under_load": len(loaded),
                "power_w_max": max(power) if power else None}


# ------------------------------------------------------------- distributed
def dist_env():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def aggregate(local_seconds: float, local_units: float, world: int, device=None):
    """(max seconds over ranks, total units over ranks): the whole-job figures."""
    if world == 1:
        return local_seconds, local_units
    import torch
    import torch.distributed as dist
    t = torch.tensor([local_seconds], dtype=torch.float64, device=device)
    u = torch.tensor([local_units], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    dist.all_reduce(u, op=dist.ReduceOp.SUM)
    return float(t.item()), float(u.item())


# --------------------------------------------------------------- the oracle
def oracle_workload(workload: str) -> str:
    """The workload whose elements the oracle samples (the 70B shard's are its layers')."""
    return "llama70b_layer" if workload == "llama70b_shard" else workload


def oracle_sample(workload: str, sample: int, steps: int, seed: int = 0, D: int = 0, reduce_dtype: int = 0,
                  keep: bool = False, nodes: int = 0):
    """Time the oracle over `steps` passes of a `sample`-element slice of the
    workload's owned elements (all D contributions, AdamW, cast).  Returns
    (owned params/s, seconds, description, kept), where kept holds the sample's
    inputs and the oracle's final state when `keep` is set (else None)."""
    import numpy as np

    import oracle
    import synth
    workload = oracle_workload(workload)
    w = synth.WORKLOADS[workload]
    D = D or w["D"]
    nodes = nodes or w.get("nodes", 1)
    n = min(sample, synth.block_numel(w["tensors"]))
    contribs = [synth.bf16_bits(synth.contribution(n, n, seed=seed, step=1, rank=d, sigma=w["sigma"],
                                                   dist=w["dist"], zero_frac=w.get("zero_frac", 0.0),
                                                   device="cpu")) for d in range(nodes * D)]
    p = synth.master_weights(n, n, seed=seed).numpy().copy()
    p0 = p.copy() if keep else None
    m, v, wk = np.zeros(n, np.float32), np.zeros(n, np.float32), np.zeros(n, np.uint16)
    oracle.lib()
    t0 = time.perf_counter()
    for t in range(1, steps + 1):
        if nodes > 1:
            oracle.reduce_adamw_hybrid(contribs, nodes, n, 0, p, m, v, wk, oracle.hp(step=t),
                                       layout=oracle.LAYOUT_OWNED, reduce_dtype=reduce_dtype)
        else:
            oracle.reduce_adamw(contribs, n, 0, p, m, v, wk, oracle.hp(step=t), layout=oracle.LAYOUT_OWNED,
                                reduce_dtype=reduce_dtype)
    dt = time.perf_counter() - t0
    shape = f"{nodes} nodes x D={D}" if nodes > 1 else f"D={D}"
    desc = (f"{workload}: first {n} owned elements x {steps} steps, {shape}, "
            f"{'bf16' if reduce_dtype else 'fp32'} reduce, one thread "
            f"(oracle/zero3_ref.c, single-threaded C)")
    kept = dict(contribs=contribs, p0=p0, p=p, m=m, v=v, wk=wk, n=n, D=D, nodes=nodes, steps=steps) if keep else None
    return n * steps / dt, dt, desc, kept


def sample_parity(z3, dev, kept: dict, reduce_dtype: int, split: bool = False) -> dict:
    """Our path, through the public API on the GPU, over the CPU baseline's own
    sample (the same contributions, master and steps, as rank 0's owned slice),
    compared element by element with the oracle's results.  split: the
    HYBRID_SHARD reduction as node sums and their fold, as the benchmark ran it."""
    import numpy as np
    import torch

    import synth
    n, D, nodes, steps = kept["n"], kept["D"], kept["nodes"], kept["steps"]
    plan = z3.zero3_plan([(n * D,)], D, 1)                     # S = n
    c = [synth.bits_to_bf16(x, dev) for x in kept["contribs"]]
    p = torch.from_numpy(kept["p0"]).to(dev)
    m, v = torch.zeros_like(p), torch.zeros_like(p)
    w = torch.zeros(n, dtype=torch.bfloat16, device=dev)
    sums = ([torch.empty(n, dtype=torch.float32 if reduce_dtype == 0 else torch.bfloat16, device=dev)
             for _ in range(nodes)] if split else None)
    for t in range(1, steps + 1):
        hp = z3.adamw(step=t)
        if split:
            for k in range(nodes):
                z3.zero3_node_sum(plan, 0, c[k * D:(k + 1) * D], sums[k], contrib_layout=z3.Z3_CONTRIB_OWNED,
                                  reduce_dtype=reduce_dtype)
            z3.zero3_fold_adamw(plan, 0, sums, p, m, v, w, hp, reduce_dtype=reduce_dtype)
        elif nodes > 1:
            z3.zero3_reduce_adamw_hybrid(plan, 0, nodes, c, p, m, v, w, hp, contrib_layout=z3.Z3_CONTRIB_OWNED,
                                         reduce_dtype=reduce_dtype)
        else:
            z3.zero3_reduce_adamw(plan, 0, c, p, m, v, w, hp, contrib_layout=z3.Z3_CONTRIB_OWNED,
                                  reduce_dtype=reduce_dtype)
    torch.cuda.synchronize(dev)

    def rel(got, ref):
        return float(np.max(np.abs(got.astype(np.float64) - ref) /
                            np.maximum(np.abs(ref.astype(np.float64)), np.finfo(np.float32).tiny)))

    def ulps(a, b):
        def ordered(x):
            x = x.astype(np.int32)
            return np.where(x & 0x8000, 0x8000 - (x & 0x7FFF), 0x8000 + (x & 0x7FFF))
        return int(np.max(np.abs(ordered(a) - ordered(b))))

    got = [t.cpu().numpy() for t in (p, m, v)]
    refs = [kept["p"], kept["m"], kept["v"]]
    gw = synth.bf16_bits(w)
    exact = all(np.array_equal(g.view(np.uint32), r.view(np.uint32)) for g, r in zip(got, refs)) and \
        np.array_equal(gw, kept["wk"])
    return {"elements": n, "steps": steps, "master_max_rel": rel(got[0], refs[0]),
            "exp_avg_max_rel": rel(got[1], refs[1]), "exp_avg_sq_max_rel": rel(got[2], refs[2]),
            "work_bf16_max_ulp": ulps(gw, kept["wk"]), "bit_exact": bool(exact)}


L2_NOTE = ("inputs larger than L2 (126 MB): every step streams the block's contributions and fp32 state "
           "through HBM, so no flush is needed between steps")


def contract_config(args, world: int, D: int, nodes: int, owned: int) -> dict:
    """The `config` both arms print (ours and the reference arm): the workload and
    the options that define the step, so that the two lines can be matched."""
    multi = world > 1 and not args.replicas
    if multi:
        par = (f"ZeRO-3 dp{world}: NCCL all-to-all of the gradients, fused reduce/AdamW/cast on each rank's "
               f"partition, NCCL all-gather of the bf16 shards" if args.transport == "nccl" else
               f"ZeRO-3 dp{world}: the kernels read every rank's gradient slice and shard through CUDA IPC "
               f"mappings (plain loads)")
    else:
        par = (f"replicas x{world}" if world > 1 else "one GPU") + \
            f", the block's {D if nodes == 1 else f'{nodes} x {D}'} ranks simulated on each GPU (no collective)"
    options = [o for o, on in (("graph", args.graph), ("unflatten_copy", args.unflatten_copy),
                               ("split", args.split)) if on]
    if args.offload:
        options.append(f"offload_{args.offload}")
    if args.workload == "llama70b_shard":
        options.append(f"arrival_{args.refill}")
    return {"workload": args.workload, "D": D, "nodes": nodes, "stage": args.stage,
            "reduce_dtype": args.reduce_dtype, "owned_params_per_step": owned, "options": options,
            "l2": L2_NOTE, "parallelism": par}


def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    import oracle
    import synth
    steps = max(1, args.steps)
    # each step is a bounded sample (2^20 elements) so that K steps stay within minutes
    sample = min(args.cpu_sample, 1 << 20)
    mode = 1 if args.reduce_dtype == "bf16" else 0
    multi = world > 1 and not args.replicas
    w = synth.WORKLOADS[oracle_workload(args.workload)]
    D = world if multi else (args.D or (8 if args.workload == "llama70b_shard" else w["D"]))
    nodes = 1 if multi else (args.nodes or w.get("nodes", 1))
    _, _, N_pad, S = oracle.plan([synth.numel(sh) for _, sh in w["tensors"]], D, synth.ALIGN)
    owned = w["layers"] * S if args.workload == "llama70b_shard" else N_pad
    if args.warmup > 0:
        oracle_sample(args.workload, min(sample, 1 << 16), 1, D=D, reduce_dtype=mode, nodes=nodes)
    value, secs, desc, _ = oracle_sample(args.workload, sample, steps, D=D, reduce_dtype=mode, nodes=nodes)
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": steps, "warmup": args.warmup, "ms_per_step": 1e3 * secs / steps,
            "higher_is_better": True, "scaling": "strong" if multi else "weak", "vs_baseline": None,
            "dtype": "f32", "data": "synthetic", "config": contract_config(args, world, D, nodes, owned),
            "sample_elements_per_step": sample,
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": 1, "kind": "oracle", "sample": desc,
                             "host": host_info()},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------- our path
class BlockRunner:
    """One block, every rank's partition in one launch: plan + ledger (host),
    fused reduce + AdamW + cast, gather into the flat block, zero-copy views.
    stage 1 or 2: one kernel does the reduce, AdamW, cast and the all-gather into
    the replicated bf16 weights (the flat block), with no separate shard."""

    def __init__(self, z3, synth, workload, D, reduce_dtype, seed, dev, stage=3, unflatten_copy=False,
                 graph=False, offload=False, split=False, nodes=0, offload_chunks=1):
        import torch
        w = synth.WORKLOADS[workload]
        self.z3, self.synth, self.w, self.D, self.mode = z3, synth, w, D, reduce_dtype
        self.device = dev
        self.shapes = [s for _, s in w["tensors"]]
        self.specs = z3.tensor_specs(self.shapes)       # the step's input: the block's tensor list
        plan = z3.zero3_plan(self.shapes, D, synth.ALIGN)
        self.N, self.N_pad, self.S = plan.N, plan.N_pad, plan.S
        # HYBRID_SHARD: `nodes` nodes of D ranks, contribution k*D + d from rank d of node k
        self.nodes = nodes or w.get("nodes", 1)
        if nodes and "nodes" not in w:
            raise SystemExit("--nodes needs a HYBRID_SHARD workload (llama7b_hybrid)")
        if self.nodes > 1 and (stage != 3 or graph or offload):
            raise SystemExit("the HYBRID_SHARD workload runs the plain ZeRO-3 block step")
        if split and self.nodes == 1:
            raise SystemExit("--split needs a HYBRID_SHARD workload (llama7b_hybrid)")
        # --split: the two-level reduction as the node sums of every node, then their fold
        # (what separate machines run), instead of the fused kernel
        self.split = split
        self.mid_events = []
        self.contribs = synth.contributions(self.nodes * D, self.N, self.N_pad, seed=seed, step=1,
                                            sigma=w["sigma"], dist=w["dist"], zero_frac=w.get("zero_frac", 0.0),
                                            device=dev)
        self.master = synth.master_weights(self.N, self.N_pad, seed=seed, device=dev)
        self.exp_avg, self.exp_avg_sq = torch.zeros_like(self.master), torch.zeros_like(self.master)
        self.offload = offload
        self.work = torch.zeros(self.N_pad, dtype=torch.bfloat16, device=dev)
        self.offloaded = None
        self.host_seconds = []
        if offload:
            # the optimiser state leaves the GPU: page-locked host memory
            from fsdp_sharded_mixed_flat_b200.offload import HostAdamWOffload, OffloadedState
            self.master, self.exp_avg, self.exp_avg_sq = (t.cpu().pin_memory() for t in
                                                          (self.master, self.exp_avg, self.exp_avg_sq))
            if offload == "host":
                self.offloaded = HostAdamWOffload(plan, self.master, self.exp_avg, self.exp_avg_sq, self.work, dev,
                                                  reduce_dtype=reduce_dtype, chunks=offload_chunks)
            else:
                self.offloaded = OffloadedState(plan, self.master, self.exp_avg, self.exp_avg_sq, self.work, dev,
                                                reduce_dtype=reduce_dtype)
        self.flat = torch.empty(self.N_pad, dtype=torch.bfloat16, device=dev)
        self.shards = [self.work[r * self.S:(r + 1) * self.S] for r in range(D)]
        self.stream = torch.cuda.current_stream(dev)
        self.step_no = 0
        self.stage = stage
        self.tensor_out = ([torch.empty(shape, dtype=torch.bfloat16, device=dev) for shape in self.shapes]
                           if unflatten_copy and stage == 3 else None)
        self.units_per_step = self.N_pad                       # owned params, all ranks
        self.ledger_args = (self.N, self.N_pad, D, self.N_pad)
        self.k1_launches_per_step = 1
        # stage 1/2: the bf16 goes to the block instead of the shard; same bytes
        self.k1_bytes_per_launch = (2 * self.nodes * D + 26) * self.N_pad
        self.step_bytes = self.k1_bytes_per_launch + (4 * self.N_pad if stage == 3 else 0) + \
            (4 * self.N if self.tensor_out is not None else 0)
        self.launches_per_step = (2 + (1 if self.tensor_out is not None else 0)) if stage == 3 else 1
        if split:
            esz = 4 if reduce_dtype == 0 else 2
            sum_dtype = torch.float32 if reduce_dtype == 0 else torch.bfloat16
            self.node_sums = [torch.empty(self.N_pad, dtype=sum_dtype, device=dev) for _ in range(self.nodes)]
            self.node_sum_bytes = self.nodes * (2 * D + esz) * self.N_pad      # all nodes' sums
            self.fold_bytes = (self.nodes * esz + 26) * self.N_pad
            self.k1_bytes_per_launch = self.node_sum_bytes + self.fold_bytes
            self.launches_per_step = self.nodes + 2
            self.step_bytes = self.k1_bytes_per_launch + 4 * self.N_pad
        ranks = f"{self.nodes} nodes x D={D}" if self.nodes > 1 else f"D={D}"
        self.k1_name = (f"k_reduce_adamw_vec<{'fp32' if reduce_dtype == 0 else 'bf16'}, {ranks}"
                        f"{', gather' if stage != 3 else ''}>")
        if split:
            self.k1_name = (f"{self.nodes} x k_node_sum_vec<D={D}> + k_fold_adamw_vec<R={self.nodes}> "
                            f"({'fp32' if reduce_dtype == 0 else 'bf16'}; the split HYBRID_SHARD reduction)")
        hybrid = (" (HYBRID_SHARD: each node's rank fold, then the node sums across %d nodes, then 1/%d%s)"
                  % (self.nodes, self.nodes * D, "; split: every node's sum written, then their fold"
                     if split else "") if self.nodes > 1 else "")
        what = ("fused reduce/AdamW/cast over all %d partitions%s + gather into the flat block%s" %
                (D, hybrid, " and into one buffer per tensor" if self.tensor_out is not None else "")
                if stage == 3
                else "one kernel: reduce/AdamW/cast over all %d partitions writing the replicated bf16 "
                     "weights in place of the gather (ZeRO-%d)" % (D, stage))
        self.graphed = None
        if graph:
            from fsdp_sharded_mixed_flat_b200.graph import GraphedStep
            self.graphed = GraphedStep(plan, self.contribs, self.master, self.exp_avg, self.exp_avg_sq,
                                       self.work if stage == 3 else None, self.flat, stage=stage,
                                       reduce_dtype=reduce_dtype)
            what += "; captured once in a CUDA graph and replayed (scalars from device memory)"
            # events around the replay time every kernel of the graph
            self.k1_bytes_per_launch = self.step_bytes
            self.k1_name = "CUDA graph of the step (%s)" % ("fused kernel + gather" if stage == 3 else "fused kernel")
        if offload == "state":
            what += ("; fp32 master/m/v in page-locked host memory, streamed partition by partition through "
                     "device staging buffers (copy-in, kernel, copy-out on three streams)")
            self.k1_name += " (rank-partition launches on staged state)"
            self.k1_launches_per_step = D
            self.k1_bytes_per_launch = (2 * D + 26) * self.S
            self.launches_per_step = D + 1
        elif offload == "host":
            gb = 4 if reduce_dtype == 0 else 2
            what += ("; fp32 master/m/v in page-locked host memory and AdamW on the host: per partition the "
                     "averaged gradient is reduced on the GPU, copied down, updated by libzero3's host threads, "
                     "and the bf16 weights copied up (pipelined over partitions)")
            self.k1_name = (f"k_node_sum_vec<{'fp32' if reduce_dtype == 0 else 'bf16'}, D={D}, scaled> "
                            "(the reduce-scatter's reduction alone, one launch per pipeline unit)")
            units = len(self.offloaded.units)
            self.k1_launches_per_step = units
            self.k1_bytes_per_launch = (2 * D + gb) * self.N_pad / units      # the mean unit
            self.launches_per_step = units + 1
            self.step_bytes = (2 * D + gb) * self.N_pad + 4 * self.N_pad
        self.desc = (f"{len(self.shapes)} tensors, N={self.N}, N_pad={self.N_pad}, S={self.S} per rank, D={D}, "
                     f"bf16 grads {w['dist']}(sigma={w['sigma']}), fp32 master N(0,0.02), AdamW lr=3e-4 "
                     f"b=(0.9,0.95) eps=1e-8 wd=0.1; step = plan + ledger + {what}")

    def hp(self):
        a = self.synth.ADAMW
        self.step_no += 1
        return self.z3.adamw(lr=a["lr"], beta1=a["beta1"], beta2=a["beta2"], eps=a["eps"],
                             weight_decay=a["weight_decay"], step=self.step_no)

    def step(self, k1_events=None, contribs=None, flat=None):
        z3 = self.z3
        contribs = self.contribs if contribs is None else contribs
        flat = self.flat if flat is None else flat
        # a1 + a2: host-side plan and ledger of the block (microseconds, overlapped with the GPU)
        pl = z3.Plan(self.shapes, self.D, self.synth.ALIGN, specs=self.specs)
        z3.zero3_memory_bytes(pl.N, self.D, self.stage)
        hp = self.hp()
        if self.graphed is not None and contribs is self.contribs and flat is self.flat:
            if k1_events is not None:
                k1_events[0][0].record(self.stream)
            self.graphed.step(hp)
            if k1_events is not None:
                k1_events[0][1].record(self.stream)
            return self.views(pl, flat)
        if k1_events is not None:
            k1_events[0][0].record(self.stream)
        if self.offloaded is not None:
            if self.offload == "host":
                self.offloaded.step(contribs, hp, k1_events, host_seconds=self.host_seconds)
            else:
                self.offloaded.step(contribs, hp, k1_events)
            z3.zero3_gather_block(pl, self.shards, flat, self.tensor_out, stream=self.stream)
            return self.views(pl, flat)
        if self.stage != 3:
            # ZeRO-1/2: the kernel writes each new bf16 weight into the replicated block
            z3.zero3_reduce_adamw_gather(pl, -1, contribs, self.master, self.exp_avg, self.exp_avg_sq, None,
                                         [flat], hp, reduce_dtype=self.mode, stream=self.stream)
            if k1_events is not None:
                k1_events[0][1].record(self.stream)
            return self.views(pl, flat)
        # a3 + a4: reduce-scatter reduction + AdamW + bf16 cast, every rank's partition in one launch
        if self.split:
            D = self.D
            for k in range(self.nodes):
                z3.zero3_node_sum(pl, -1, contribs[k * D:(k + 1) * D], self.node_sums[k], reduce_dtype=self.mode,
                                  stream=self.stream)
            if k1_events is not None:
                import torch
                mid = torch.cuda.Event(enable_timing=True)
                mid.record(self.stream)
                self.mid_events.append((k1_events[0][0], mid, k1_events[0][1]))
            z3.zero3_fold_adamw(pl, -1, self.node_sums, self.master, self.exp_avg, self.exp_avg_sq, self.work, hp,
                                reduce_dtype=self.mode, stream=self.stream)
        elif self.nodes > 1:
            z3.zero3_reduce_adamw_hybrid(pl, -1, self.nodes, contribs, self.master, self.exp_avg,
                                         self.exp_avg_sq, self.work, hp, reduce_dtype=self.mode, stream=self.stream)
        else:
            z3.zero3_reduce_adamw(pl, -1, contribs, self.master, self.exp_avg, self.exp_avg_sq, self.work, hp,
                                  reduce_dtype=self.mode, stream=self.stream)
        if k1_events is not None:
            k1_events[0][1].record(self.stream)
        # a5 + a6: all-gather of the D bf16 shards into the flat block; views are zero-copy
        z3.zero3_gather_block(pl, self.shards, flat, self.tensor_out, stream=self.stream)
        return self.views(pl, flat)

    def views(self, pl, flat):
        """a6: the zero-copy per-tensor views of the gathered block.  They alias the
        same buffer every step, so they are built once per buffer."""
        key = flat.data_ptr()
        cache = self.__dict__.setdefault("_views", {})
        if key not in cache:
            cache[key] = pl.views(flat)
        return cache[key]

    def e2e_setup(self):
        """Pinned host copies of the contributions and of the gathered block, and a
        second device set of both so that transfers of neighbouring steps overlap."""
        import torch
        dev = self.device
        self.host_c = [torch.empty(self.N_pad, dtype=torch.bfloat16, pin_memory=True) for _ in self.contribs]
        for h, c in zip(self.host_c, self.contribs):
            h.copy_(c)
        self.host_flat = torch.empty(self.N_pad, dtype=torch.bfloat16, pin_memory=True)
        self.dev_c = [self.contribs, [torch.empty_like(c) for c in self.contribs]]
        self.dev_flat = [self.flat, torch.empty_like(self.flat)]
        self.h2d_stream, self.d2h_stream = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        self.ev_in = [torch.cuda.Event() for _ in range(2)]     # contributions of set b arrived
        self.ev_used = [torch.cuda.Event() for _ in range(2)]   # step on set b finished reading / writing
        self.ev_out = [torch.cuda.Event() for _ in range(2)]    # gathered block b copied to the host
        self.e2e_i = 0
        return (sum(h.numel() * h.element_size() for h in self.host_c),
                self.host_flat.numel() * self.host_flat.element_size())

    def e2e_step(self):
        """One step through the public API from host buffers: H2D of the step's
        contributions (copy-in stream), the step (compute stream), D2H of its
        gathered block (copy-out stream).  Two device sets let the H2D of the next
        step and the D2H of the previous one overlap this step's kernels."""
        import torch
        b = self.e2e_i & 1
        self.e2e_i += 1
        with torch.cuda.stream(self.h2d_stream):
            self.h2d_stream.wait_event(self.ev_used[b])
            for h, c in zip(self.host_c, self.dev_c[b]):
                c.copy_(h, non_blocking=True)
            self.ev_in[b].record(self.h2d_stream)
        self.stream.wait_event(self.ev_in[b])
        self.stream.wait_event(self.ev_out[b])            # the host copy of this block's last use is done
        self.step(contribs=self.dev_c[b], flat=self.dev_flat[b])
        self.ev_used[b].record(self.stream)
        with torch.cuda.stream(self.d2h_stream):
            self.d2h_stream.wait_event(self.ev_used[b])
            self.host_flat.copy_(self.dev_flat[b], non_blocking=True)
            self.ev_out[b].record(self.d2h_stream)

    def e2e_drain(self):
        self.stream.wait_stream(self.h2d_stream)
        self.stream.wait_stream(self.d2h_stream)


class ShardRunner:
    """One rank's resident 70B shard (80 layers at D = 8): per step, the layers'
    owned contributions stream in last to first through two transient buffers
    (copy stream) while the fused kernel runs on the other buffer."""

    def __init__(self, z3, synth, workload, D, reduce_dtype, seed, dev, refill=DEFAULT_ARRIVAL):
        import torch
        from fsdp_sharded_mixed_flat_b200.stream import LayerStreamer
        w = synth.WORKLOADS["llama70b_layer"]
        self.z3, self.synth, self.w, self.D, self.mode = z3, synth, w, D, reduce_dtype
        self.L = w["layers"]
        plan = z3.zero3_plan([s for _, s in w["tensors"]], D, synth.ALIGN)
        self.plan, self.S = plan, plan.S
        S, L = self.S, self.L
        self.master = torch.empty(L * S, dtype=torch.float32, device=dev)
        for l in range(L):
            self.master[l * S:(l + 1) * S] = synth.master_weights(S, S, seed=seed * 100 + l, device=dev)
        self.exp_avg, self.exp_avg_sq = torch.zeros_like(self.master), torch.zeros_like(self.master)
        self.work = torch.zeros(L * S, dtype=torch.bfloat16, device=dev)
        # the refill source: two layers' worth of owned contributions (what the reduce-scatter delivers)
        self.pool = [torch.cat([synth.contribution(S, S, seed=seed, step=1, rank=d, sigma=w["sigma"], device=dev)
                                for d in range(D)]) for _ in range(2)]
        if refill not in ARRIVALS:
            raise SystemExit(f"unknown arrival {refill}")
        self.streamer = LayerStreamer(plan, L, 0, self.master, self.exp_avg, self.exp_avg_sq, self.work,
                                      reduce_dtype=reduce_dtype)
        self.stream = torch.cuda.current_stream(dev)
        self.step_no = 0
        self.units_per_step = L * S                            # owned params of this rank
        self.ledger_args = (L * plan.N, L * plan.N_pad, D, plan.N_pad)
        self.k1_launches_per_step = L
        self.k1_bytes_per_launch = (2 * D + 26) * S
        self.refill = refill
        self.refill_bytes = L * 2 * D * S * (2 if refill == "copy" else 1)   # copy: read + write
        self.step_bytes = L * self.k1_bytes_per_launch + self.refill_bytes
        self.launches_per_step = L
        self.k1_name = f"k_reduce_adamw_vec<{'fp32' if reduce_dtype == 0 else 'bf16'}, D={D}> (owned layout)"
        self.source = lambda l: self.pool[l & 1]
        # write-only refill: the transient buffer receives a value, as an NVLink delivery would write it
        self.fill = None
        if refill == "fill":
            self.fill = lambda l, buf: buf.fill_(1e-4 * (1 + (l & 7)))
        elif refill == "memset":
            from cuda.bindings import runtime as cudart

            def memset(l, buf):
                # bytes 0x38..0x3F: bf16 values 4.4e-5 .. 1.9, finite, a different one per layer
                err, = cudart.cudaMemsetAsync(buf.data_ptr(), 0x38 + (l & 7), buf.numel() * buf.element_size(),
                                              torch.cuda.current_stream(buf.device).cuda_stream)
                if err != cudart.cudaError_t.cudaSuccess:
                    raise RuntimeError(f"cudaMemsetAsync: {err}")
            self.fill = memset
        self.arrival_desc = f"{refill}: {ARRIVALS[refill]}"
        self.desc = (f"rank 0's resident shard of 80 LLaMA-70B-shaped layers ({len(w['tensors'])} tensors, "
                     f"855,654,400 params each), D={D}, S={S} per layer, {L * S} owned params "
                     f"({L * S * 14 / 1e9:.1f} GB of master+m+v+bf16); per step the 80 layers' owned bf16 "
                     f"contributions ({2 * D * S / 1e9:.2f} GB each) stream 79->0 through two transient buffers "
                     f"({ARRIVALS[refill]}) "
                     f"on a copy stream) while the fused kernel runs")

    def hp(self):
        a = self.synth.ADAMW
        self.step_no += 1
        return self.z3.adamw(lr=a["lr"], beta1=a["beta1"], beta2=a["beta2"], eps=a["eps"],
                             weight_decay=a["weight_decay"], step=self.step_no)

    def step(self, k1_events=None):
        self.streamer.step(self.source, self.hp(), k1_events, fill=self.fill)

    def step_in_place(self, k1_events=None):
        """The same 80 fused-kernel launches reading the pool in place: no refill traffic."""
        self.streamer.step(self.source, self.hp(), k1_events, copy_in=False)

    def e2e_setup(self):
        import torch
        self.host_pool = [torch.empty_like(p, device="cpu").pin_memory() for p in self.pool]
        for h, p in zip(self.host_pool, self.pool):
            h.copy_(p)
        self.host_out = torch.empty(self.S, dtype=torch.bfloat16, pin_memory=True)
        return self.L * self.host_pool[0].numel() * 2, self.S * 2

    def e2e_drain(self):
        pass

    def e2e_step(self):
        # contributions come from pinned host memory layer by layer; layer 0's bf16 shard goes back
        self.streamer.step(lambda l: self.host_pool[l & 1], self.hp())
        self.host_out.copy_(self.work[:self.S], non_blocking=True)


def mix_ceilings(dev, reps: int = 10) -> dict:
    """HBM bandwidth of plain torch kernels on this GPU, per read/write mix, best
    of `reps` launches timed with CUDA events on 1 GiB fp32 buffers (well beyond
    L2): write-only (fill), read-only (sum), copy (1 read : 1 write) and add (2
    reads : 1 write, the fused kernel's mix at D = 8).  Library kernels, so a
    kernel of ours can sit a little above them; they place its rate against the
    mix it moves."""
    import torch
    n = 1 << 28
    a = torch.rand(n, device=dev)
    b = torch.rand(n, device=dev)
    c = torch.empty(n, device=dev)
    ops = {"write_only_fill": (lambda: c.fill_(1.0), 4 * n),
           "read_only_sum": (lambda: a.sum(), 4 * n),
           "copy_1r_1w": (lambda: c.copy_(a), 8 * n),
           "add_2r_1w": (lambda: torch.add(a, b, out=c), 12 * n)}
    out = {}
    for name, (fn, nbytes) in ops.items():
        fn()
        best = None
        for _ in range(reps):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            torch.cuda.synchronize(dev)
            t = e0.elapsed_time(e1) / 1e3
            best = t if best is None else min(best, t)
        out[name] = nbytes / best / 1e9
    del a, b, c
    torch.cuda.empty_cache()
    return out


def time_runner(R, steps: int, warmup: int, dev, clocks=None, barrier=None, step=None):
    """W untimed warm-up steps, then `steps` steps timed with CUDA events on the
    runner's stream between synchronisations (and barriers, with several ranks);
    the fused kernel is timed launch by launch with its own events.  Returns
    (seconds of the timed steps, mean seconds per fused-kernel launch)."""
    import torch
    step = step or R.step
    for _ in range(warmup):
        step()
    torch.cuda.synchronize(dev)
    if clocks is not None:
        clocks.start()
    k1_ev = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(R.k1_launches_per_step)] for _ in range(steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if barrier is not None:
        barrier()
    torch.cuda.synchronize(dev)
    t0.record(R.stream)
    for i in range(steps):
        step(k1_ev[i])
    t1.record(R.stream)
    torch.cuda.synchronize(dev)
    if barrier is not None:
        barrier()
    secs = t0.elapsed_time(t1) / 1e3
    k1_ms = [a.elapsed_time(b) for step_ev in k1_ev for a, b in step_ev]
    return secs, statistics.mean(k1_ms) / 1e3


# The target configurations besides the headline: (key, workload, D).  Each is
# measured in both reduce dtypes by config_sweep.
SWEEP_BLOCKS = [("config1_llama7b_d8", "llama7b_d8", 8), ("config2_llama7b_d32", "llama7b_d32", 32),
                ("config3_policy_D2", "llama7b_policy", 2), ("config3_policy_D4", "llama7b_policy", 4),
                ("config3_policy_D8", "llama7b_policy", 8), ("config3_policy_D16", "llama7b_policy", 16)]
NOMINAL_HBM_GBS = 8000.0


def prefetch_sweep(z3, synth, dev, steps: int, L: int = 32, D: int = 8) -> dict:
    """The backward sweep of one rank over the L = 32 blocks of LLaMA-7B at D = 8
    with the next block's all-gather prefetched into one of two transient
    buffers (PrefetchSweep), timed against the same sweep with every gather
    serialised in front of its block.  Per block: the gather of the block's 8
    shards (4 B per element of the block) and the fused kernel on this rank's
    partition (42 B per owned element)."""
    import torch
    from fsdp_sharded_mixed_flat_b200.stream import PrefetchSweep
    w = synth.WORKLOADS["llama7b_d8"]
    plan = z3.zero3_plan([sh for _, sh in w["tensors"]], D, synth.ALIGN)
    S, N_pad = plan.S, plan.N_pad
    g = torch.Generator(device=dev).manual_seed(77)
    flat = torch.randn(L * N_pad, generator=g, device=dev).mul_(0.02).to(torch.bfloat16)   # every rank's shards
    shards = [[flat[l * N_pad + d * S:l * N_pad + (d + 1) * S] for d in range(D)] for l in range(L)]
    master = torch.randn(L * S, generator=g, device=dev).mul_(0.02)
    m, v = torch.zeros_like(master), torch.zeros_like(master)
    pool = torch.cat([synth.contribution(S, S, seed=77, step=1, rank=d, sigma=w["sigma"], device=dev)
                      for d in range(D)])
    contribs = [pool[d * S:(d + 1) * S] for d in range(D)]
    sweep = PrefetchSweep(plan, shards, 0, master, m, v)
    stream = torch.cuda.current_stream(dev)
    res = {}
    t = [0]

    def hp():
        t[0] += 1
        return z3.adamw(step=t[0], **synth.ADAMW)
    for prefetch in (True, False):
        sweep.step(lambda l: contribs, hp(), prefetch=prefetch)
        torch.cuda.synchronize(dev)
        ev = {}
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(steps):
            sweep.step(lambda l: contribs, hp(), prefetch=prefetch, events=ev)
        b.record(stream)
        torch.cuda.synchronize(dev)
        res[prefetch] = (a.elapsed_time(b) / 1e3 / steps,
                         statistics.mean(x.elapsed_time(y) for x, y in ev["gather"]) / 1e3,
                         statistics.mean(x.elapsed_time(y) for x, y in ev["k1"]) / 1e3)
    t_pre, g_pre, k_pre = res[True]
    t_ser, g_ser, k_ser = res[False]
    out = {"blocks": L, "D": D, "rank": 0, "transient_gathered_buffers": 2,
           "transient_bytes": sweep.transient_bytes,
           "ledger_transient_bytes_2_blocks": z3.zero3_transient_bytes(N_pad, 2),
           "sweep_ms_prefetch": 1e3 * t_pre, "sweep_ms_serial": 1e3 * t_ser,
           "gather_ms_serial": 1e3 * g_ser, "k1_ms_serial": 1e3 * k_ser,
           "sum_of_serial_kernels_ms": 1e3 * L * (g_ser + k_ser),
           "gather_gbs_serial": 4 * N_pad / g_ser / 1e9, "k1_gbs_serial": 42 * S / k_ser / 1e9,
           "gather_ms_overlapped": 1e3 * g_pre, "k1_ms_overlapped": 1e3 * k_pre,
           "hidden_fraction_of_gather": (t_ser - t_pre) / (L * g_ser),
           "owned_params_per_s_prefetch": L * S / t_pre,
           "sweep_hbm_gbs_prefetch": L * (4 * N_pad + 42 * S) / t_pre / 1e9,
           "note": "one GPU holds every rank's shards, so each gather reads HBM like the fused kernel does and "
                   "both are bound by the same HBM: the prefetch can only fill the gaps between launches. On D "
                   "GPUs the gather reads the peers' shards over NVLink, a separate resource, which is what the "
                   "prefetch hides"}
    del sweep, flat, shards, master, m, v, pool, contribs
    torch.cuda.empty_cache()
    return out


def config_sweep(z3, synth, dev, steps: int, warmup: int, hbm_peak: float, refill: str) -> dict:
    """Every target configuration on this GPU, with fewer steps than the headline:
    the fused kernel's own time, rate and fraction of peak, and the whole step's
    owned params/s (plan + fused kernel + gather for a block; the 80-layer
    streamed step for the 70B shard).  Target: the fused kernel at >= 80 % of
    nominal 8 TB/s, i.e. 6.4e12 / (2D + 26) owned params/s."""
    import torch
    out = {}

    def sweep_block(key, workload, D):
        entry = {}
        for name, mode in (("fp32", z3.Z3_REDUCE_FP32), ("bf16", z3.Z3_REDUCE_BF16)):
            R = BlockRunner(z3, synth, workload, D, mode, 2000, dev)
            secs, k1 = time_runner(R, steps, warmup, dev)
            gbs = R.k1_bytes_per_launch / k1 / 1e9
            target = 0.8 * NOMINAL_HBM_GBS * 1e9 / (2 * D + 26)
            entry[name] = {"k1_ms": 1e3 * k1, "k1_gbs": gbs, "k1_owned_params_per_s": R.units_per_step / k1,
                           "k1_frac": gbs / hbm_peak, "k1_frac_of_nominal_8000": gbs / NOMINAL_HBM_GBS,
                           "target_k1_owned_params_per_s": target,
                           "meets_80pct_of_nominal": R.units_per_step / k1 >= target,
                           "step_ms": 1e3 * secs / steps, "step_owned_params_per_s": R.units_per_step * steps / secs}
            del R
        entry.update(workload=workload, D=D, bytes_per_owned_param=2 * D + 26)
        out[key] = entry

    def sweep_shard():
        # config 4: one rank's 80-layer 70B shard, streamed through two transient buffers
        S4 = ShardRunner(z3, synth, "llama70b_shard", 8, z3.Z3_REDUCE_FP32, 2000, dev, refill=refill)
        shard_steps = max(2, steps // 5)
        secs, k1 = time_runner(S4, shard_steps, 1, dev)
        ip_secs, ip_k1 = time_runner(S4, shard_steps, 1, dev, step=S4.step_in_place)
        step_s = secs / shard_steps
        k1_bytes = S4.L * S4.k1_bytes_per_launch
        target = 0.8 * NOMINAL_HBM_GBS * 1e9 / 42
        out["config4_llama70b_shard"] = {
            "workload": "llama70b_shard", "D": 8, "layers": S4.L, "owned_params_per_step": S4.units_per_step,
            "streamed": {"arrival": S4.arrival_desc, "step_ms": 1e3 * step_s,
                         "step_owned_params_per_s": S4.units_per_step / step_s,
                         "k1_ms_per_layer": 1e3 * k1, "k1_gbs": S4.k1_bytes_per_launch / k1 / 1e9,
                         "k1_frac": S4.k1_bytes_per_launch / k1 / 1e9 / hbm_peak,
                         "step_hbm_gbs": (k1_bytes + S4.refill_bytes) / step_s / 1e9,
                         "arrival_bytes_per_step": S4.refill_bytes},
            "in_place": {"step_ms": 1e3 * ip_secs / shard_steps,
                         "step_owned_params_per_s": S4.units_per_step * shard_steps / ip_secs,
                         "k1_ms_per_layer": 1e3 * ip_k1, "k1_gbs": S4.k1_bytes_per_launch / ip_k1 / 1e9,
                         "k1_frac": S4.k1_bytes_per_launch / ip_k1 / 1e9 / hbm_peak,
                         "k1_owned_params_per_s": S4.S / ip_k1,
                         "meets_80pct_of_nominal": S4.S / ip_k1 >= target,
                         "note": "the same 80 fused-kernel launches reading the contributions where they lie: the "
                                 "kernel's own rate, without the arrival of the next layer's bytes"},
            "target_k1_owned_params_per_s": target, "steps": shard_steps}
        del S4

    def guarded(key, fn):
        # one entry's failure (say, memory taken by another process) is recorded, not raised:
        # the headline measured before the sweep stands
        try:
            fn()
        except Exception as e:   # noqa: BLE001
            out[key] = {"error": f"{type(e).__name__}: {e}"[:300]}
        if dev.type == "cuda":
            torch.cuda.synchronize(dev)
            torch.cuda.empty_cache()

    def sweep_step_variant(key, label, make, reps):
        """A whole block step of one of the NEXT rows: owned params/s and ms per step,
        with the fused kernel's own time and rate (or, offloaded, the PCIe figures)."""
        R = make()
        secs, k1 = time_runner(R, reps, 2, dev)
        entry = {"what": label, "step_ms": 1e3 * secs / reps, "step_owned_params_per_s": R.units_per_step * reps / secs,
                 "kernel": R.k1_name, "kernel_ms": 1e3 * k1, "kernel_gbs": R.k1_bytes_per_launch / k1 / 1e9,
                 "steps": reps}
        if getattr(R, "offload", None) == "host":
            host_s = R.host_seconds[-reps * len(R.offloaded.units):]
            entry.update(pcie_bytes_per_param=(R.offloaded.bytes_down + R.offloaded.bytes_up) / R.N_pad,
                         host_adamw_ms_per_step=1e3 * sum(host_s) / reps)
        elif getattr(R, "offload", None) == "state":
            entry.update(pcie_bytes_per_param=24)
        out.setdefault(key, {})[label] = entry
        del R

    for key, workload, D in SWEEP_BLOCKS:
        guarded(key, lambda key=key, workload=workload, D=D: sweep_block(key, workload, D))
    guarded("config4_llama70b_shard", sweep_shard)
    guarded("next2_prefetch_llama7b_L32_d8",
            lambda: out.__setitem__("next2_prefetch_llama7b_L32_d8",
                                    prefetch_sweep(z3, synth, dev, max(2, steps // 5))))
    # NEXT-3: the ZeRO-1/2 step (all-gather fused into the kernel), HYBRID_SHARD over 4 nodes of 8
    guarded("next3_zero12_llama7b_d8", lambda: sweep_step_variant(
        "next3_zero12_llama7b_d8", "fp32", lambda: BlockRunner(z3, synth, "llama7b_d8", 8, 0, 2000, dev, stage=2),
        steps))
    for name, mode in (("fp32", 0), ("bf16", 1)):
        guarded("next3_hybrid_llama7b_4x8", lambda name=name, mode=mode: sweep_step_variant(
            "next3_hybrid_llama7b_4x8", name, lambda: BlockRunner(z3, synth, "llama7b_hybrid", 8, mode, 2000, dev),
            steps))
    # NEXT-4: the CPU-offload step, AdamW on the host (the page's design) and the state
    # streamed through the GPU
    for place in ("host", "state"):
        guarded("next4_offload_llama7b_d8", lambda place=place: sweep_step_variant(
            "next4_offload_llama7b_d8", place,
            lambda: BlockRunner(z3, synth, "llama7b_d8", 8, 0, 2000, dev, offload=place), 3))
    # config 3's bf16-vs-fp32 drift over 100 steps (reported, not asserted)
    guarded("config3_drift", lambda: out.__setitem__("config3_drift", drift_measure(z3, synth, dev, 100, 1 << 24)))
    return out


class Clock:
    """Time marks: CUDA events recorded on the current stream, or the host clock
    when the step runs on the CPU (the host tests of the multi-rank path)."""

    def __init__(self, device):
        import torch
        self.torch, self.device, self.cuda = torch, device, device.type == "cuda"

    def mark(self):
        if self.cuda:
            e = self.torch.cuda.Event(enable_timing=True)
            e.record(self.torch.cuda.current_stream(self.device))
            return e
        return time.perf_counter()

    def seconds(self, a, b) -> float:
        return a.elapsed_time(b) / 1e3 if self.cuda else b - a

    def sync(self):
        if self.cuda:
            self.torch.cuda.synchronize(self.device)


class CollectiveRunner:
    """Rank r's share of the real D-GPU ZeRO-3 step, D = the world size, one
    process per GPU: this rank's full bf16 gradient of the block goes through an
    all-to-all (the reduce-scatter's data movement: rank r receives P_r of every
    rank's gradient, in rank order), the fused kernel reduces it in rank order and
    updates this rank's fp32 state and bf16 shard (owned layout), and an
    all-gather assembles the block ("7.10 — Fully-sharded data parallel", §4,
    §5.1).  With transport "peer" the kernels read the peers' gradients and
    shards through CUDA IPC mappings with plain loads instead (peer.py)."""

    def __init__(self, z3, synth, workload, world, rank, reduce_dtype, dev, kernels=None, transport="nccl",
                 peer_group=None, stage=3):
        import torch
        from fsdp_sharded_mixed_flat_b200.collective import CollectiveZero3Step
        w = synth.WORKLOADS[workload]
        self.shapes = [s for _, s in w["tensors"]]
        plan = z3.zero3_plan(self.shapes, world, synth.ALIGN)
        self.plan, self.D, self.rank, self.mode, self.device = plan, world, rank, reduce_dtype, dev
        N, N_pad, S = plan.N, plan.N_pad, plan.S
        self.N, self.N_pad, self.S = N, N_pad, S
        self.grad = synth.contribution(N, N_pad, seed=1000, step=1, rank=rank, sigma=w["sigma"], dist=w["dist"],
                                       zero_frac=w.get("zero_frac", 0.0), device=dev)
        self.master = synth.master_weights(N, N_pad, seed=1000, device=dev)[rank * S:(rank + 1) * S].clone()
        self.exp_avg, self.exp_avg_sq = torch.zeros_like(self.master), torch.zeros_like(self.master)
        self.work = torch.zeros(S, dtype=torch.bfloat16, device=dev)
        self.flat = torch.zeros(N_pad, dtype=torch.bfloat16, device=dev)
        self.transport, self.stage = transport, stage
        if transport == "peer":
            from fsdp_sharded_mixed_flat_b200.peer import PeerGroup, PeerZero3Step
            self.stepper = PeerZero3Step(peer_group or PeerGroup(), plan, self.grad, self.master, self.exp_avg,
                                         self.exp_avg_sq, self.work, self.flat, stage=stage,
                                         reduce_dtype=reduce_dtype, kernels=kernels or z3)
        else:
            self.stepper = CollectiveZero3Step(plan, self.grad, self.master, self.exp_avg, self.exp_avg_sq,
                                               self.work, self.flat, reduce_dtype=reduce_dtype, kernels=kernels or z3)
        self.z3, self.synth = z3, synth
        self.clock = Clock(dev)
        self.marks = []
        self.step_no = 0
        self.units_per_step = S                         # owned params of this rank
        self.k1_bytes_per_launch = (2 * world + 26) * S
        self.gather_bytes = 2 * N_pad * (world - 1) // world   # bytes this rank receives in the all-gather
        self.a2a_bytes = 2 * S * (world - 1)                     # gradient bytes it receives in the all-to-all

    def step(self, timed: bool = False):
        a = self.synth.ADAMW
        self.step_no += 1
        hp = self.z3.adamw(step=self.step_no, **a)
        self.stepper.step(hp, mark=self.clock.mark if timed else None, marks=self.marks)

    def close(self) -> None:
        """Once this rank's kernels are done, release its mappings of the other
        ranks' memory (peer form)."""
        self.clock.sync()
        if self.transport == "peer":
            self.stepper.peers.close()

    def phases(self) -> dict:
        """Mean seconds of each phase of the timed steps: the all-to-all, the fused
        kernel and the all-gather (NCCL); the two fences, the fused kernel reading
        the peers' gradients and the gather kernel reading their shards (peer,
        stage 3); the two fences around the one kernel that reads the peers'
        gradients and stores the new shard into every rank's block (peer, stages
        1 and 2)."""
        names = (("all_to_all", "reduce_adamw", "all_gather") if self.transport == "nccl" else
                 ("fence_before", "reduce_adamw", "fence_between", "gather") if self.stage == 3 else
                 ("fence_before", "reduce_adamw", "fence_between"))
        return {n: statistics.mean(self.clock.seconds(m[k], m[k + 1]) for m in self.marks)
                for k, n in enumerate(names)}


def time_collective_steps(R, steps: int, warmup: int, world: int, dev, barrier, clocks=None):
    """Warm-up, then `steps` timed steps bracketed by a barrier and a device
    synchronisation on both sides; (seconds of this rank, job seconds = the max
    over ranks, job units, clock record)."""
    for _ in range(warmup):
        R.step()
    R.clock.sync()
    barrier()
    if clocks is not None:
        clocks.start()
    t0 = R.clock.mark()
    R.marks.clear()
    for _ in range(steps):
        R.step(timed=True)
    t1 = R.clock.mark()
    R.clock.sync()
    barrier()
    clk = clocks.stop() if clocks is not None else None
    secs = R.clock.seconds(t0, t1)
    job_secs, job_units = aggregate(secs, float(R.units_per_step) * steps, world, dev if dev.type == "cuda" else None)
    return secs, job_secs, job_units, clk


def run_collective(args, rank: int, world: int, dev, z3, synth, kernels=None, clocks=None, barrier=None,
                   peer_group=None):
    """bench.py --gpus N, N > 1: the real D-GPU step with D = N, the block's
    ranks on N GPUs (strong scaling: one block's N_pad owned params per step in
    all, S = N_pad / N per rank).  The headline is the step as --transport sets
    it: by default the peer form, whose fused kernel reads every rank's gradient
    slice over the peer mappings (the reduce-scatter inside the optimiser
    kernel) and whose gather kernel reads every rank's shard; with it, the NCCL
    form of the same step is timed afterwards as `baseline_nccl`.  Returns (the
    JSON line, the headline's runner); only rank 0's line is printed."""
    import torch
    mode = z3.Z3_REDUCE_BF16 if args.reduce_dtype == "bf16" else z3.Z3_REDUCE_FP32
    peer = args.transport == "peer"
    unsupported = [o for o, on in (("--graph", args.graph), ("--unflatten-copy", args.unflatten_copy),
                                   ("--offload", bool(args.offload)), ("--split", args.split),
                                   ("--nodes", args.nodes > 1),
                                   (f"--workload {args.workload}",
                                    args.workload in ("llama7b_hybrid", "llama70b_shard", "profile_hybrid")))
                   if on]
    if unsupported:
        raise SystemExit(f"N > 1 runs the block step over the N GPUs; {', '.join(unsupported)} is measured on one "
                         f"GPU only (HYBRID_SHARD across GPUs is collective.CollectiveHybridStep)")
    if args.stage != 3 and not peer:
        raise SystemExit("--stage 1/2 with N > 1 is the peer form's fused kernel (--transport peer)")
    R = CollectiveRunner(z3, synth, args.workload, world, rank, mode, dev, kernels=kernels, transport=args.transport,
                         peer_group=peer_group, stage=args.stage)
    barrier = barrier or (lambda: torch.distributed.barrier())
    secs, job_secs, job_units, clk = time_collective_steps(R, args.steps, args.warmup, world, dev, barrier, clocks)
    ph = R.phases()

    # ---- end to end: this rank's gradient from pinned host memory, its new shard back
    pin = dev.type == "cuda"
    host_grad = R.grad.cpu().pin_memory() if pin else R.grad.clone()
    host_shard = torch.empty(R.S, dtype=torch.bfloat16, pin_memory=pin)
    e2e_steps = max(1, args.e2e_steps)
    barrier()
    e0 = R.clock.mark()
    for _ in range(e2e_steps):
        R.grad.copy_(host_grad, non_blocking=True)
        R.step()
        host_shard.copy_(R.work, non_blocking=True)
    e1 = R.clock.mark()
    R.clock.sync()
    barrier()
    e2e_secs, e2e_units = aggregate(R.clock.seconds(e0, e1), float(R.units_per_step) * e2e_steps, world,
                                    dev if dev.type == "cuda" else None)
    hbm_peak, peak_kind = measured_peaks()
    k1_s = ph["reduce_adamw"]
    k1_gbs = R.k1_bytes_per_launch / k1_s / 1e9
    step_s = secs / args.steps
    kname = f"k_reduce_adamw_vec<{'fp32' if mode == 0 else 'bf16'}, D={world}>"
    if peer:
        # the fused kernel pulls 2(D-1) bytes per owned element over NVLink and touches
        # 28 B of its own HBM (its gradient slice, the state); the link is the bound.
        # At stages 1 and 2 it also pushes 2(D-1) bytes per owned element out (the
        # new shard into every other rank's block).
        link_gbs = R.a2a_bytes / k1_s / 1e9
        fences = ph["fence_before"] + ph["fence_between"]
        if args.stage == 3:
            kdesc = " (full layout, peers' gradients through the IPC mappings)"
        else:
            kdesc = (" with the all-gather's stores fused (zero3_reduce_adamw_gather: peers' gradients read and "
                     "the new shard stored into every rank's block through the IPC mappings)")
        roofline = {"bound": "nvlink", "achieved": link_gbs, "peak": NVLINK_GBS, "unit": "GB/s",
                    "frac": link_gbs / NVLINK_GBS,
                    "peak_kind": "measured B200 peer copy over NVLink 5, per direction per GPU (900 nominal)",
                    "kernel": kname + kdesc, "nvlink_bytes_in_per_launch": R.a2a_bytes,
                    "hbm_algorithmic_gbs": k1_gbs, "traffic": None}
        collective = {"fence_ms": 1e3 * fences, "reduce_adamw_ms": 1e3 * k1_s,
                      "collective_share_of_step": fences / max(step_s, 1e-12),
                      "nvlink_bytes_in_per_rank": R.a2a_bytes + R.gather_bytes,
                      "note": "the reduce-scatter's data movement runs inside the fused kernel and the "
                              "all-gather's inside the gather kernel (stage 3) or the fused kernel's own "
                              "stores (stages 1 and 2); the fences are a stream synchronisation and a group "
                              "barrier"}
        if args.stage == 3:
            collective["gather_ms"] = 1e3 * ph["gather"]
    else:
        roofline = {"bound": "hbm", "achieved": k1_gbs, "peak": hbm_peak, "unit": "GB/s",
                    "frac": k1_gbs / hbm_peak, "peak_kind": peak_kind + " (HBM copy, MEASURED_PEAKS.json)",
                    "kernel": kname + " (owned layout)", "algorithmic_bytes_per_launch": R.k1_bytes_per_launch,
                    "traffic": None}
        collective = {"all_to_all_ms": 1e3 * ph["all_to_all"], "reduce_adamw_ms": 1e3 * k1_s,
                      "all_gather_ms": 1e3 * ph["all_gather"],
                      "collective_share_of_step": (ph["all_to_all"] + ph["all_gather"]) / max(step_s, 1e-12),
                      "all_to_all_bytes_in_per_rank": R.a2a_bytes, "all_gather_bytes_in_per_rank": R.gather_bytes}
    line = {
        "metric": METRIC, "value": job_units / job_secs, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": 1e3 * job_secs / args.steps, "higher_is_better": True,
        "scaling": "strong", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": contract_config(args, world, world, 1, R.N_pad),
        "workload_desc": (f"{args.workload}: one block of {R.N} params ({R.N_pad} padded) sharded over the {world} "
                          f"GPUs, S={R.S} owned per rank; bf16 gradients of every rank, fp32 master N(0,0.02), "
                          f"AdamW lr=3e-4 b=(0.9,0.95) eps=1e-8 wd=0.1; transport {args.transport}"),
        "per_rank_owned_params_per_s": R.units_per_step / step_s,
        "comm_nranks": world,
        "collective": collective,
        "kernels": {"reduce_adamw_ms": 1e3 * k1_s, "reduce_adamw_gbs": k1_gbs},
        "roofline": roofline,
        "clocks": clk,
        "e2e": {"value": e2e_units / e2e_secs, "unit": UNIT, "h2d_bytes_per_step": 2 * R.N_pad * world,
                "d2h_bytes_per_step": 2 * R.S * world, "steps": e2e_steps,
                "note": "bytes of all ranks: each copies its full gradient in and its new shard out"},
        "gpu_launches": args.steps * (2 if peer and args.stage == 3 else 1),
        "ledger_bytes_per_device": ledger(z3, R.N, R.N_pad, world, R.N_pad),
    }
    if peer and not args.no_nccl_baseline:
        B = CollectiveRunner(z3, synth, args.workload, world, rank, mode, dev, kernels=kernels, transport="nccl")
        _, b_secs, b_units, _ = time_collective_steps(B, args.steps, args.warmup, world, dev, barrier)
        bph = B.phases()
        B.close()
        line["baseline_nccl"] = {
            "value": b_units / b_secs, "unit": UNIT, "ms_per_step": 1e3 * b_secs / args.steps,
            "all_to_all_ms": 1e3 * bph["all_to_all"], "reduce_adamw_ms": 1e3 * bph["reduce_adamw"],
            "all_gather_ms": 1e3 * bph["all_gather"],
            "note": "the same step with NCCL all-to-all and all-gather around the fused kernel (owned layout)"}
        del B
    return line, R


def run_ours(args):
    import torch
    import torch.distributed as dist

    rank, world, local_rank = dist_env()
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)

    from fsdp_sharded_mixed_flat_b200 import build
    if rank == 0 or not os.path.exists(build.LIB):
        build.build()
    if world > 1:
        dist.barrier()
    import synth
    from fsdp_sharded_mixed_flat_b200 import zero3 as z3

    mode = z3.Z3_REDUCE_BF16 if args.reduce_dtype == "bf16" else z3.Z3_REDUCE_FP32
    if world > 1 and not args.replicas:
        props = torch.cuda.get_device_properties(dev)
        uuid = getattr(props, "uuid", None)
        line, R = run_collective(args, rank, world, dev, z3, synth,
                                 clocks=ClockSampler(f"GPU-{uuid}" if uuid is not None else None))
        if rank == 0:
            print(json.dumps(line), flush=True)
        R.close()
        del R
        dist.barrier()
        dist.destroy_process_group()
        return 0
    if args.graph and (args.unflatten_copy or args.workload == "llama70b_shard"):
        raise SystemExit("--graph covers the block step without --unflatten-copy")
    if args.offload and (args.graph or args.stage != 3 or args.workload == "llama70b_shard"):
        raise SystemExit("--offload covers the ZeRO-3 block step without --graph")
    seed = 1000 + rank  # every rank runs its own block
    if args.workload == "llama70b_shard":
        R = ShardRunner(z3, synth, args.workload, args.D or 8, mode, seed, dev, refill=args.refill)
    else:
        R = BlockRunner(z3, synth, args.workload, args.D or synth.WORKLOADS[args.workload]["D"], mode, seed, dev,
                        stage=args.stage, unflatten_copy=args.unflatten_copy, graph=args.graph,
                        offload=args.offload, split=args.split, nodes=args.nodes, offload_chunks=args.offload_chunks)
    stream = R.stream

    props = torch.cuda.get_device_properties(dev)
    uuid = getattr(props, "uuid", None)
    clocks = ClockSampler(f"GPU-{uuid}" if uuid is not None else None)
    secs, k1_avg_s = time_runner(R, args.steps, args.warmup, dev, clocks=clocks,
                                 barrier=dist.barrier if world > 1 else None)
    clk = clocks.stop()
    job_secs, job_units = aggregate(secs, float(R.units_per_step) * args.steps, world, dev)
    value = job_units / job_secs

    extra = {}
    if hasattr(R, "step_in_place"):
        # the fused kernel alone over the 80 layers, contributions read in place
        ev = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(R.k1_launches_per_step)] for _ in range(args.steps)]
        R.step_in_place()
        torch.cuda.synchronize(dev)
        a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a0.record(stream)
        for i in range(args.steps):
            R.step_in_place(ev[i])
        a1.record(stream)
        torch.cuda.synchronize(dev)
        ip_s = a0.elapsed_time(a1) / 1e3
        ip_k1 = statistics.mean([x.elapsed_time(y) for se in ev for x, y in se]) / 1e3
        extra["in_place"] = {"value": R.units_per_step * args.steps / ip_s, "unit": UNIT,
                             "ms_per_step": 1e3 * ip_s / args.steps, "reduce_adamw_ms": 1e3 * ip_k1,
                             "reduce_adamw_gbs": R.k1_bytes_per_launch / ip_k1 / 1e9,
                             "note": "no refill copy: every layer's kernel reads the contribution pool in place"}

    # ---- end to end through the public API with host buffers
    e2e_steps = max(1, args.e2e_steps)
    h2d, d2h = R.e2e_setup()
    for _ in range(2):
        R.e2e_step()
    R.e2e_drain()
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    if hasattr(R, "h2d_stream"):
        R.h2d_stream.wait_stream(stream)  # no transfer starts before the timed region does
    for _ in range(e2e_steps):
        R.e2e_step()
    R.e2e_drain()                     # the last step's host copy is inside the timed region
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_secs, e2e_units = aggregate(e0.elapsed_time(e1) / 1e3, float(R.units_per_step) * e2e_steps, world, dev)

    hbm_peak, peak_kind = measured_peaks()
    k1_gbs = R.k1_bytes_per_launch / k1_avg_s / 1e9
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": 1e3 * job_secs / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": contract_config(args, world, R.D, getattr(R, "nodes", 1), R.units_per_step),
        "workload_desc": f"{args.workload}: {R.desc}; each step streams {R.step_bytes / 1e9:.2f} GB",
        "step_hbm_gbs": R.step_bytes * args.steps * world / job_secs / 1e9,
        "kernels": {"reduce_adamw_ms": 1e3 * k1_avg_s, "reduce_adamw_gbs": k1_gbs,
                    "reduce_adamw_params_per_s": R.units_per_step / R.k1_launches_per_step / k1_avg_s,
                    "reduce_adamw_launches_per_step": R.k1_launches_per_step,
                    "rest_of_step_ms": max(0.0, 1e3 * secs / args.steps - 1e3 * k1_avg_s * R.k1_launches_per_step)},
        "roofline": {"bound": "hbm", "achieved": k1_gbs, "peak": hbm_peak, "unit": "GB/s",
                     "frac": k1_gbs / hbm_peak, "peak_kind": peak_kind + " (HBM copy, MEASURED_PEAKS.json)",
                     "frac_of_nominal_8000": k1_gbs / 8000.0, "kernel": R.k1_name,
                     "algorithmic_bytes_per_launch": R.k1_bytes_per_launch,
                     "traffic": (profiled_traffic(args.workload)
                                 if mode == 0 and args.stage == 3 and not args.graph and not args.split
                                 else None)},
        "clocks": clk,
        "e2e": {"value": e2e_units / e2e_secs, "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "steps": e2e_steps},
        "gpu_launches": R.launches_per_step * args.steps,
        "ledger_bytes_per_device": ledger(z3, *R.ledger_args),
    }
    if getattr(R, "split", False) and R.mid_events:
        ns = statistics.mean(a.elapsed_time(b) for a, b, _ in R.mid_events) / 1e3
        fo = statistics.mean(b.elapsed_time(c) for _, b, c in R.mid_events) / 1e3
        extra["split_hybrid"] = {"node_sums_ms": 1e3 * ns, "node_sums_gbs": R.node_sum_bytes / ns / 1e9,
                                 "fold_ms": 1e3 * fo, "fold_gbs": R.fold_bytes / fo / 1e9,
                                 "node_sum_bytes": R.node_sum_bytes, "fold_bytes": R.fold_bytes,
                                 "note": "every node's sum (R launches) on one GPU, then the fold: on separate "
                                         "machines each node runs one node sum and the fold"}
    line.update(extra)
    if getattr(R, "offload", None) == "state":
        # 12 B of state read and 12 B written per element cross PCIe; HBM carries the rest
        step_s = job_secs / args.steps
        line["offload"] = {"placement": "state streamed through the GPU, AdamW on the GPU",
                           "pcie_bytes_per_param": 24, "pcie_gbs_per_direction": 12 * R.N_pad / step_s / 1e9,
                           "note": "fp32 master/m/v (12 B per element) cross PCIe each way every step; the step "
                                   "is bound by PCIe, not HBM, so the hbm roofline fields describe the kernels "
                                   "on the staged device buffers only"}
        line["roofline"]["traffic"] = None
    elif getattr(R, "offload", None) == "host":
        step_s = job_secs / args.steps
        down = R.offloaded.bytes_down
        host_s = R.host_seconds[-args.steps * len(R.offloaded.units):]
        line["offload"] = {"placement": "AdamW on the host (the page's CPU-offload variant)",
                           "pipeline_units": len(R.offloaded.units),
                           "pcie_bytes_per_param": (down + R.offloaded.bytes_up) / R.N_pad,
                           "pcie_gbs_down": down / step_s / 1e9, "pcie_gbs_up": R.offloaded.bytes_up / step_s / 1e9,
                           "host_adamw_ms_per_step": 1e3 * sum(host_s) / args.steps,
                           "host_adamw_params_per_s": R.N_pad * args.steps / sum(host_s),
                           "host_threads": os.cpu_count(),
                           "note": "the averaged gradient (4 B, or 2 with the bf16 reduce) goes down and the bf16 "
                                   "weights (2 B) come up per param; the step is bound by the host's AdamW "
                                   "(30 B of host memory traffic per param), so the hbm roofline fields describe "
                                   "the GPU's reduce kernels only"}
        line["roofline"]["traffic"] = None
    if world == 1 and not args.no_sweep:
        # the K1 of the default workload reads 2 bytes per byte written (28 : 14 at D = 8)
        ceil = mix_ceilings(dev)
        line["roofline"]["mix_ceilings_torch_gbs"] = ceil
        line["roofline"]["frac_of_2r1w_ceiling"] = k1_gbs / ceil["add_2r_1w"]
    run_D, run_nodes, run_split = R.D, getattr(R, "nodes", 1), getattr(R, "split", False)
    if world == 1 and not args.no_sweep and args.workload == "llama7b_d8" and args.stage == 3 and \
            not (args.graph or args.offload or args.unflatten_copy):
        # every target configuration, on the same GPU after the headline (whose buffers are freed first)
        R.__dict__.clear()
        del R
        torch.cuda.empty_cache()
        sweep_clocks = ClockSampler(f"GPU-{uuid}" if uuid is not None else None)
        sweep_clocks.start()
        line["configs"] = config_sweep(z3, synth, dev, args.sweep_steps, max(3, min(args.warmup, 5)), hbm_peak,
                                       args.refill)
        line["configs"]["clocks"] = sweep_clocks.stop()
        line["configs"]["note"] = ("the fused kernel (K1) of every target configuration timed alone with CUDA events "
                                   "over %d steps after warm-up, both reduce dtypes; target: K1 at >= 80 %% of "
                                   "nominal 8 TB/s; k1_frac is of the measured copy peak" % args.sweep_steps)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        # calibrate on a small slice, then size the step count for about 10 s of oracle work
        nodes = run_nodes
        rate, _, _, _ = oracle_sample(args.workload, 1 << 16, 1, D=run_D, reduce_dtype=mode, nodes=nodes)
        n_cpu = min(args.cpu_sample, synth.block_numel(synth.WORKLOADS[oracle_workload(args.workload)]["tensors"]))
        cpu_steps = max(1, min(args.cpu_steps, round(10.0 * rate / max(1, n_cpu))))
        v, secs_cpu, desc, kept = oracle_sample(args.workload, args.cpu_sample, cpu_steps, D=run_D,
                                                reduce_dtype=mode, keep=True, nodes=nodes)
        line["cpu_baseline"] = {"value": v, "unit": UNIT, "cores": 1, "kind": "oracle", "sample": desc,
                                "host": host_info(),
                                "seconds": secs_cpu,
                                "parity_vs_oracle": sample_parity(z3, dev, kept, mode, split=run_split)}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def drift_measure(z3, synth, dev, steps: int, n: int) -> dict:
    """The policy sweep's drift: the same heavy-tailed contributions (Student-t nu=3,
    1% exact zeros, fresh every step) drive two copies of the same master, one
    reduced in bf16 and one in fp32, for `steps` steps at each D; how far the bf16
    path's master and bf16 weights end up from the fp32 path's.  The pages give no
    value for it: it is reported, not asserted."""
    import torch
    w = synth.WORKLOADS["llama7b_policy"]
    out = {"drift": {}, "steps": steps, "elements": n,
           "workload": "first %d elements of the LLaMA-7B block, Student-t nu=3 x %g, %g%% exact zeros, "
                       "fresh contributions every step" % (n, w["sigma"], 100 * w["zero_frac"])}
    for D in w["Ds"]:
        plan = z3.zero3_plan([(n,)], D, synth.ALIGN)
        N_pad = plan.N_pad
        p0 = synth.master_weights(n, N_pad, seed=11, device=dev)
        state = {mode: [p0.clone(), torch.zeros_like(p0), torch.zeros_like(p0),
                        torch.zeros(N_pad, dtype=torch.bfloat16, device=dev)] for mode in (0, 1)}
        for t in range(1, steps + 1):
            c = synth.contributions(D, n, N_pad, seed=11, step=t, sigma=w["sigma"], dist=w["dist"],
                                    zero_frac=w["zero_frac"], device=dev)
            for mode in (0, 1):
                z3.zero3_reduce_adamw(plan, -1, c, *state[mode], z3.adamw(step=t), reduce_dtype=mode)
        torch.cuda.synchronize(dev)
        pf, pb = state[0][0][:n].double(), state[1][0][:n].double()
        upd = (pf - p0[:n].double())
        diff = (pb - pf)
        rel = diff.abs() / pf.abs().clamp_min(1e-30)
        upd_rms = upd.pow(2).mean().sqrt()
        wf, wb = state[0][3][:n].view(torch.int16), state[1][3][:n].view(torch.int16)
        out["drift"][f"D={D}"] = {
            "master_median_rel": rel.median().item(),
            "max_abs_diff_over_update_rms": (diff.abs().max() / upd_rms).item(),
            "diff_rms_over_update_rms": (diff.pow(2).mean().sqrt() / upd_rms).item(),
            "bf16_weights_differing": (wf != wb).double().mean().item(),
        }
    return out


def run_drift(args):
    import torch

    import synth
    from fsdp_sharded_mixed_flat_b200 import build
    build.build()
    from fsdp_sharded_mixed_flat_b200 import zero3 as z3
    print(json.dumps(drift_measure(z3, synth, torch.device("cuda", 0), args.steps, args.drift_elements)), flush=True)
    return 0


def main():
    args = parse_args()
    if args.drift:
        return run_drift(args)
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
