"""Host logic of the benchmark on CPU: the whole-job aggregation over ranks
(max of the per-rank times, sum of the units) on a world-size-2 gloo group,
and the clock-sample parsing."""
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
