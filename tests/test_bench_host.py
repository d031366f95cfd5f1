"""Host logic of the benchmark on CPU: the whole-job aggregation over ranks
(max of the per-rank times, sum of the units) on a world-size-2 gloo group,
the multi-GPU path (the D-GPU step with D = N) end to end on two gloo ranks
with the oracle standing in for the kernels, and the clock-sample parsing."""
import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    secs, units = bench.aggregate(1.0 + rank, 100.0 * (rank + 1), world)
    out[rank] = (secs, units)
    dist.barrier()
    dist.destroy_process_group()


def test_aggregate_two_ranks_gloo():
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        port = _free_port()
        procs = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(120)
            assert p.exitcode == 0
        assert out[0] == (2.0, 300.0) and out[1] == (2.0, 300.0)


def test_aggregate_single_rank_is_identity():
    assert bench.aggregate(1.5, 10.0, 1) == (1.5, 10.0)


def test_clock_sampler_parses_reasons():
    c = bench.ClockSampler(None)
    c.proc = type("P", (), {"terminate": lambda self: None, "wait": lambda self, timeout=None: 0})()
    c.lines = ["1965, 1965, 650.0, 0x0, Not Active, Not Active, Not Active, Not Active",
               "1800, 1965, 990.5, 0x4, Not Active, Not Active, Not Active, Active",
               "1810, 1965, 120.0, 0x0, Not Active, Not Active, Not Active, Not Active"]
    r = c.stop()
    assert r["sm_mhz"] == pytest.approx(1882.5) and r["sm_max_mhz"] == 1965.0
    assert r["reasons"] == ["sw_power_cap"] and r["samples"] == 3 and r["samples_under_load"] == 2
    assert r["slowdown_seen"] is False


def test_reference_arm_prints_one_contract_line():
    """`bench.py --impl reference` (the oracle on the host) prints one JSON line
    with the keys the benchmark contract asks for."""
    import json
    import subprocess
    import sys
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1", "--warmup", "0"],
                       cwd=bench.ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for k in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
              "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert k in d, k
    assert d["impl"] == "reference" and d["value"] > 0 and d["metric"] == bench.METRIC
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["cpu_baseline"]["kind"] == "oracle"
    assert d["cpu_baseline"]["cores"] == 1
    # the same config our arm prints for the default workload (7B block, D = 8, one GPU)
    assert d["config"] == bench.contract_config(bench.parse_args([]), 1, 8, 1, 202_383_360)


def _collective_worker(rank, world, port, mode, transport, stage, tmpdir, out):
    import numpy as np
    import torch

    import synth
    from fsdp_sharded_mixed_flat_b200 import zero3 as z3
    from test_collective_host import OracleKernels, file_peer_group
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    args = bench.parse_args(["--gpus", str(world), "--workload", "tiny_gpt", "--steps", "2", "--warmup", "1",
                             "--e2e-steps", "1", "--reduce-dtype", "bf16" if mode else "fp32",
                             "--transport", transport, "--stage", str(stage)])
    group = file_peer_group(tmpdir, rank) if transport == "peer" else None
    line, R = bench.run_collective(args, rank, world, torch.device("cpu"), z3, synth, kernels=OracleKernels(),
                                   barrier=dist.barrier, peer_group=group)
    out[rank] = (line, R.master.numpy().copy(), R.exp_avg.numpy().copy(), R.exp_avg_sq.numpy().copy(),
                 R.work.view(torch.int16).numpy().view(np.uint16).copy(),
                 R.flat.view(torch.int16).numpy().view(np.uint16).copy(), R.step_no)
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("transport,stage", [("peer", 3), ("peer", 2), ("nccl", 3)])
@pytest.mark.parametrize("mode", [0, 1], ids=["fp32", "bf16"])
def test_multi_gpu_path_end_to_end_on_two_gloo_ranks(mode, transport, stage, tmp_path):
    """bench.py's N > 1 path (run_collective: the D-GPU step, warm-up, timed
    steps, max-over-ranks aggregation, the end-to-end leg, the JSON line) on two
    gloo ranks, in both forms: the peer form over shared host mappings standing
    in for the IPC mappings (ZeRO-3, and the stage-2 step whose one kernel also
    stores the new shard into every rank's block; then also the NCCL form as the
    baseline), and the NCCL form with the collectives moving the real bytes.
    The oracle stands in for the kernels.  Every rank's state equals one oracle
    run over both ranks."""
    import numpy as np

    import oracle
    import synth
    world = 2
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        port = _free_port()
        procs = [ctx.Process(target=_collective_worker,
                             args=(r, world, port, mode, transport, stage, str(tmp_path), out))
                 for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(300)
            assert p.exitcode == 0
        res = dict(out)
    line = res[0][0]
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
              "vs_baseline", "dtype", "data", "config", "roofline", "e2e", "gpu_launches", "comm_nranks",
              "collective", "per_rank_owned_params_per_s"):
        assert k in line, k
    assert line["n_gpus"] == 2 and line["comm_nranks"] == 2 and line["scaling"] == "strong"
    assert line["config"]["D"] == 2 and line["value"] > 0 and line["e2e"]["value"] > 0
    assert line["metric"] == bench.METRIC and line["steps"] == 2 and line["warmup"] == 1
    if transport == "peer":
        assert line["roofline"]["bound"] == "nvlink" and line["gpu_launches"] == 2 * (2 if stage == 3 else 1)
        assert line["baseline_nccl"]["value"] > 0 and ("gather_ms" in line["collective"]) == (stage == 3)
    else:
        assert line["roofline"]["bound"] == "hbm" and line["gpu_launches"] == 2 and "baseline_nccl" not in line
    w = synth.WORKLOADS["tiny_gpt"]
    numels = [synth.numel(s) for _, s in w["tensors"]]
    _, N, N_pad, S = oracle.plan(numels, world, synth.ALIGN)
    assert line["config"]["owned_params_per_step"] == N_pad
    steps = res[0][6]
    assert steps == 1 + 2 + 1                          # warm-up, timed, end to end
    p = synth.master_weights(N, N_pad, seed=1000).numpy().copy()
    mm, vv, ww = np.zeros(N_pad, np.float32), np.zeros(N_pad, np.float32), np.zeros(N_pad, np.uint16)
    c = [synth.bf16_bits(synth.contribution(N, N_pad, seed=1000, step=1, rank=d, sigma=w["sigma"]))
         for d in range(world)]
    for t in range(1, steps + 1):
        oracle.reduce_adamw(c, S, -1, p, mm, vv, ww, oracle.hp(step=t), reduce_dtype=mode)
    for r in range(world):
        _, rp, rm, rv, rw, rflat, _ = res[r]
        sl = slice(r * S, (r + 1) * S)
        assert np.array_equal(rp.view(np.uint32), p[sl].view(np.uint32)), f"master rank {r}"
        assert np.array_equal(rm.view(np.uint32), mm[sl].view(np.uint32)), f"exp_avg rank {r}"
        assert np.array_equal(rv.view(np.uint32), vv[sl].view(np.uint32)), f"exp_avg_sq rank {r}"
        assert np.array_equal(rw, ww[sl]), f"work rank {r}"
        assert np.array_equal(rflat, ww), f"gathered block rank {r}"


def test_config_sweep_records_a_failing_entry_and_goes_on(monkeypatch):
    """The sweep after the headline: an entry that raises (e.g. memory taken by
    another process) is recorded as an error and the other entries still run."""
    import torch

    class FakeRunner:
        k1_bytes_per_launch, units_per_step, S, L = 42.0e9, 1.0e9, 1.0e8, 80
        refill_bytes, arrival_desc, k1_name = 1.0e9, "memset", "fake"

        def __init__(self, z3, synth, workload, D, *a, **k):
            if workload == "llama7b_d32":
                raise RuntimeError("CUDA out of memory (simulated)")
            self.offload, self.N_pad, self.host_seconds = k.get("offload"), 1.0e9, [0.01] * 64
            self.offloaded = type("O", (), {"units": [0] * 8, "bytes_down": 4.0e9, "bytes_up": 2.0e9})

        def step_in_place(self, *a):
            pass

    monkeypatch.setattr(bench, "BlockRunner", FakeRunner)
    monkeypatch.setattr(bench, "ShardRunner", FakeRunner)
    monkeypatch.setattr(bench, "time_runner", lambda R, steps, warmup, dev, step=None: (0.01 * steps, 0.006))
    monkeypatch.setattr(bench, "prefetch_sweep", lambda *a, **k: {"sweep_ms_prefetch": 1.0})
    monkeypatch.setattr(bench, "drift_measure", lambda *a, **k: {"drift": {}})
    z3 = type("Z3", (), {"Z3_REDUCE_FP32": 0, "Z3_REDUCE_BF16": 1})
    out = bench.config_sweep(z3, None, torch.device("cpu"), 10, 3, 6650.0, "memset")
    assert out["config2_llama7b_d32"] == {"error": "RuntimeError: CUDA out of memory (simulated)"}
    assert out["config1_llama7b_d8"]["fp32"]["k1_gbs"] == pytest.approx(7000.0)
    assert out["config1_llama7b_d8"]["fp32"]["meets_80pct_of_nominal"] is True
    assert set(out) == {k for k, _, _ in bench.SWEEP_BLOCKS} | {
        "config4_llama70b_shard", "next2_prefetch_llama7b_L32_d8", "next3_zero12_llama7b_d8",
        "next3_hybrid_llama7b_4x8", "next4_offload_llama7b_d8", "config3_drift"}
    assert out["config4_llama70b_shard"]["streamed"]["arrival"] == "memset"
    assert set(out["next3_hybrid_llama7b_4x8"]) == {"fp32", "bf16"}
    assert set(out["next4_offload_llama7b_d8"]) == {"host", "state"}
    assert out["next4_offload_llama7b_d8"]["state"]["pcie_bytes_per_param"] == 24
    assert out["next4_offload_llama7b_d8"]["host"]["pcie_bytes_per_param"] == pytest.approx(6.0)


def test_committed_k1_profiles_match_the_kernel_code():
    """The DRAM traffic the bench line reports comes from committed ncu profiles;
    they must have been taken on the kernel's current code."""
    for workload in ("llama7b_d8", "llama7b_hybrid"):
        assert bench.profiled_traffic(workload) is not None, workload


def test_code_hash_ignores_comments_only(tmp_path):
    a, b, c = tmp_path / "a.cu", tmp_path / "b.cu", tmp_path / "c.cu"
    a.write_text("// header\nint f(int x) {  // doubled\n    return 2 * x;\n}\n")
    b.write_text("// another header\n\nint f(int x) {\n    return 2 * x;   \n}\n// end\n")
    c.write_text("// header\nint f(int x) {\n    return 3 * x;\n}\n")
    assert bench.code_sha256([a]) == bench.code_sha256([b])
    assert bench.code_sha256([a]) != bench.code_sha256([c])


@pytest.mark.parametrize("flags", [["--graph"], ["--offload"], ["--nodes", "4"], ["--workload", "llama7b_hybrid"],
                                   ["--transport", "nccl", "--stage", "2"]])
def test_multi_gpu_path_refuses_what_it_does_not_measure(flags):
    """Options measured on one GPU only are refused at N > 1, before any collective,
    instead of being silently dropped."""
    import torch

    import synth
    from fsdp_sharded_mixed_flat_b200 import zero3 as z3
    args = bench.parse_args(["--gpus", "2"] + flags)
    with pytest.raises(SystemExit):
        bench.run_collective(args, 0, 2, torch.device("cpu"), z3, synth)
