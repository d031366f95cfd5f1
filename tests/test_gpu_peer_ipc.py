"""The peer-memory step (fsdp_sharded_mixed_flat_b200/peer.py) through real CUDA
IPC mappings: two processes on one GPU, ranks of a gloo group, share their
gradient buffers and bf16 shards (ZeRO-3) or gathered blocks (ZeRO-1/2) with
torch's CUDA IPC, and run PeerZero3Step with the library's kernels, so each
rank's kernels read (and, at stage 2, write) the other process's memory through
the mapping.  No kernel waits on another rank: every wait is a stream
synchronisation followed by a gloo barrier.  Both ranks' state and gathered
block must equal one oracle run over both ranks, bit for bit."""
import os
import socket
from datetime import timedelta

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
import synth

pytestmark = pytest.mark.gpu

SHAPES = [(30000,), (77, 5), (4097,)]
SEED = 9


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _bits(t: torch.Tensor) -> np.ndarray:
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def test_ipc_export_reports_the_allocation_of_a_view():
    """Within one process (no mapping, no kernel): two views into one allocation
    export the same handle, offsets that differ by the views' distance, and an
    allocation size that holds both."""
    from fsdp_sharded_mixed_flat_b200 import build
    build.build()
    from fsdp_sharded_mixed_flat_b200 import zero3 as z3
    x = torch.zeros(1 << 20, dtype=torch.float32, device="cuda")
    h0, off0, size0 = z3.zero3_ipc_export(x)
    h1, off1, size1 = z3.zero3_ipc_export(x[12345:])
    assert len(h0) == z3.Z3_IPC_HANDLE_BYTES and h0 == h1 and size0 == size1
    assert off1 - off0 == 12345 * 4 and off0 >= 0 and off0 + x.numel() * 4 <= size0
    assert x.data_ptr() - off0 == x[12345:].data_ptr() - off1       # one allocation base


def _worker(rank, world, port, mode, stage, steps, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    torch.cuda.set_device(0)
    from fsdp_sharded_mixed_flat_b200 import zero3 as z3
    from fsdp_sharded_mixed_flat_b200.peer import PeerGroup, PeerZero3Step
    plan = z3.zero3_plan(SHAPES, world, 8)
    N, N_pad, S = plan.N, plan.N_pad, plan.S
    grad = torch.zeros(N_pad, dtype=torch.bfloat16, device="cuda")
    master = synth.master_weights(N, N_pad, seed=SEED, device="cuda")[rank * S:(rank + 1) * S].clone()
    m, v = torch.zeros_like(master), torch.zeros_like(master)
    work = torch.zeros(S, dtype=torch.bfloat16, device="cuda")
    flat = torch.zeros(N_pad, dtype=torch.bfloat16, device="cuda")
    step = PeerZero3Step(PeerGroup(), plan, grad, master, m, v, work, flat, stage=stage, reduce_dtype=mode)
    for t in range(1, steps + 1):
        grad.copy_(synth.contribution(N, N_pad, seed=SEED, step=t, rank=rank, sigma=1e-3, device="cuda"))
        step.step(z3.adamw(step=t))
    torch.cuda.synchronize()
    dist.barrier()                 # every rank's last writes into the others' memory have landed
    out[rank] = (master.cpu().numpy().copy(), m.cpu().numpy().copy(), v.cpu().numpy().copy(), _bits(work).copy(),
                 _bits(flat).copy())
    step.peers.close()             # unmap the other process's memory (this rank's kernels are done)
    del step
    torch.cuda.synchronize()
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("world,stage,mode", [(2, 3, 0), (2, 3, 1), (2, 2, 0), (2, 2, 1), (3, 3, 0), (3, 2, 1)])
def test_processes_share_through_cuda_ipc(world, stage, mode):
    """world ranks as processes on one GPU (3: the generic rank count's kernel)."""
    assert torch.cuda.is_available(), "the GPU tests need a CUDA device"
    from fsdp_sharded_mixed_flat_b200 import build
    build.build()
    steps = 3
    with mp.get_context("spawn").Manager() as manager:
        out = manager.dict()
        mp.spawn(_worker, args=(world, _free_port(), mode, stage, steps, out), nprocs=world, join=True)
        results = dict(out)
    _, N, N_pad, S = oracle.plan([int(np.prod(s)) for s in SHAPES], world, 8)
    # the same device generators as the ranks drew from
    p = synth.master_weights(N, N_pad, seed=SEED, device="cuda").cpu().numpy().copy()
    m, v, w = np.zeros(N_pad, np.float32), np.zeros(N_pad, np.float32), np.zeros(N_pad, np.uint16)
    for t in range(1, steps + 1):
        c = [synth.bf16_bits(synth.contribution(N, N_pad, seed=SEED, step=t, rank=d, sigma=1e-3, device="cuda"))
             for d in range(world)]
        oracle.reduce_adamw(c, S, -1, p, m, v, w, oracle.hp(step=t), reduce_dtype=mode)
    for r in range(world):
        rp, rm, rv, rw, rflat = results[r]
        sl = slice(r * S, (r + 1) * S)
        assert np.array_equal(rp.view(np.uint32), p[sl].view(np.uint32)), f"master rank {r}"
        assert np.array_equal(rm.view(np.uint32), m[sl].view(np.uint32)), f"exp_avg rank {r}"
        assert np.array_equal(rv.view(np.uint32), v[sl].view(np.uint32)), f"exp_avg_sq rank {r}"
        assert np.array_equal(rw, w[sl]), f"work rank {r}"
        assert np.array_equal(rflat, w), f"gathered block rank {r}"


def _bench_worker(rank, world, port, stage, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    torch.cuda.set_device(0)
    import bench
    from fsdp_sharded_mixed_flat_b200 import zero3 as z3
    args = bench.parse_args(["--gpus", str(world), "--workload", "tiny_gpt", "--steps", "2", "--warmup", "1",
                             "--e2e-steps", "1", "--transport", "peer", "--no-nccl-baseline",
                             "--stage", str(stage)])
    line, R = bench.run_collective(args, rank, world, torch.device("cuda", 0), z3, synth, barrier=dist.barrier)
    torch.cuda.synchronize()
    dist.barrier()
    out[rank] = (line, R.master.cpu().numpy().copy(), R.exp_avg.cpu().numpy().copy(),
                 R.exp_avg_sq.cpu().numpy().copy(), _bits(R.work).copy(), _bits(R.flat).copy(), R.step_no)
    R.close()
    del R
    torch.cuda.synchronize()
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("stage", [3, 2])
def test_bench_peer_path_in_two_processes_on_one_gpu(stage):
    """bench.py's N > 1 headline (run_collective, peer form; at stage 2 the one
    kernel that reads the peers' gradients and stores the new shard into every
    rank's block) with its real CUDA IPC mappings and kernels, two ranks as two
    processes on one GPU (the timings mean nothing here; the NCCL form, which
    needs a GPU per rank, is left out): the JSON line, and both ranks' state
    equal to one oracle run over both ranks."""
    assert torch.cuda.is_available(), "the GPU tests need a CUDA device"
    from fsdp_sharded_mixed_flat_b200 import build
    build.build()
    world = 2
    with mp.get_context("spawn").Manager() as manager:
        out = manager.dict()
        mp.spawn(_bench_worker, args=(world, _free_port(), stage, out), nprocs=world, join=True)
        res = dict(out)
    line = res[0][0]
    assert line["n_gpus"] == 2 and line["comm_nranks"] == 2 and line["value"] > 0 and line["e2e"]["value"] > 0
    assert line["roofline"]["bound"] == "nvlink" and line["gpu_launches"] == 2 * (2 if stage == 3 else 1)
    assert line["collective"]["reduce_adamw_ms"] > 0
    assert (line["collective"]["gather_ms"] > 0) if stage == 3 else ("gather_ms" not in line["collective"])
    assert "baseline_nccl" not in line
    w = synth.WORKLOADS["tiny_gpt"]
    _, N, N_pad, S = oracle.plan([synth.numel(s) for _, s in w["tensors"]], world, synth.ALIGN)
    steps = res[0][6]
    assert steps == 1 + 2 + 1                          # warm-up, timed, end to end
    p = synth.master_weights(N, N_pad, seed=1000, device="cuda").cpu().numpy().copy()
    m, v, wk = np.zeros(N_pad, np.float32), np.zeros(N_pad, np.float32), np.zeros(N_pad, np.uint16)
    c = [synth.bf16_bits(synth.contribution(N, N_pad, seed=1000, step=1, rank=d, sigma=w["sigma"],
                                            dist=w["dist"], zero_frac=w.get("zero_frac", 0.0), device="cuda"))
         for d in range(world)]
    for t in range(1, steps + 1):
        oracle.reduce_adamw(c, S, -1, p, m, v, wk, oracle.hp(step=t))
    for r in range(world):
        _, rp, rm, rv, rw, rflat, _ = res[r]
        sl = slice(r * S, (r + 1) * S)
        assert np.array_equal(rp.view(np.uint32), p[sl].view(np.uint32)), f"master rank {r}"
        assert np.array_equal(rm.view(np.uint32), m[sl].view(np.uint32)), f"exp_avg rank {r}"
        assert np.array_equal(rv.view(np.uint32), v[sl].view(np.uint32)), f"exp_avg_sq rank {r}"
        assert np.array_equal(rw, wk[sl]), f"work rank {r}"
        assert np.array_equal(rflat, wk), f"gathered block rank {r}"
