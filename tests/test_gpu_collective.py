"""The collective steps on one GPU: a one-rank NCCL group (the all-to-all and
all-gathers reduce to copies), with the real kernels, against the oracle --
ZeRO-3 with the fused kernel, HYBRID_SHARD with the node-sum and fold kernels.
Groups of several GPUs cannot run here (one GPU per run); the steps' data
movement with several ranks is tested on CPU with gloo in
test_collective_host.py."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist

import oracle
import synth
from parity_util import assert_bf16_parity, assert_f32_parity, checked_plan, f32_host, hp_for, oracle_hp

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def z3():
    assert torch.cuda.is_available(), "the GPU tests need a CUDA device"
    from fsdp_sharded_mixed_flat_b200 import build
    build.build()
    from fsdp_sharded_mixed_flat_b200 import zero3
    return zero3


@pytest.fixture()
def nccl_one_rank():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    from datetime import timedelta
    dist.init_process_group("nccl", rank=0, world_size=1, timeout=timedelta(seconds=60), device_id=dev)
    yield
    dist.destroy_process_group()


@pytest.mark.parametrize("mode", [0, 1], ids=["fp32", "bf16"])
def test_one_rank_nccl_group_matches_oracle(z3, nccl_one_rank, mode):
    from fsdp_sharded_mixed_flat_b200.collective import CollectiveZero3Step
    plan, ref = checked_plan(z3, [(50000,), (77, 3), (4097,)], 1, 128)
    N, N_pad, S = ref.N, ref.N_pad, ref.S
    grad = torch.zeros(N_pad, dtype=torch.bfloat16, device="cuda")
    p = synth.master_weights(N, N_pad, seed=31, device="cuda")
    m, v = torch.zeros_like(p), torch.zeros_like(p)
    w = torch.zeros(S, dtype=torch.bfloat16, device="cuda")
    flat = torch.zeros(N_pad, dtype=torch.bfloat16, device="cuda")
    step = CollectiveZero3Step(plan, grad, p, m, v, w, flat, reduce_dtype=mode)
    hp_, hm, hv, hw = f32_host(p).copy(), np.zeros(S, np.float32), np.zeros(S, np.float32), np.zeros(S, np.uint16)
    for t in range(1, 4):
        grad.copy_(synth.contribution(N, N_pad, seed=31, step=t, rank=0, sigma=1e-3, device="cuda"))
        step.step(z3.adamw(**hp_for(t)))
        oracle.reduce_adamw([synth.bf16_bits(grad)], S, 0, hp_, hm, hv, hw, oracle_hp(t), reduce_dtype=mode)
    torch.cuda.synchronize()
    assert_f32_parity(f32_host(p), hp_, "master")
    assert_f32_parity(f32_host(m), hm, "exp_avg")
    assert_f32_parity(f32_host(v), hv, "exp_avg_sq")
    assert_bf16_parity(synth.bf16_bits(w), hw, "work_bf16")
    assert np.array_equal(synth.bf16_bits(flat), hw)


@pytest.mark.parametrize("mode", [0, 1], ids=["fp32", "bf16"])
def test_one_rank_nccl_hybrid_step_matches_oracle(z3, nccl_one_rank, mode):
    """The HYBRID_SHARD collective step on a one-rank NCCL group (one node of one
    rank): node and replica groups, the node-sum and fold kernels, the gathers."""
    from fsdp_sharded_mixed_flat_b200.collective import CollectiveHybridStep, hybrid_groups
    node_group, replica_group = hybrid_groups(1, 1)
    plan, ref = checked_plan(z3, [(50000,), (77, 3), (4097,)], 1, 128)
    N, N_pad, S = ref.N, ref.N_pad, ref.S
    grad = torch.zeros(N_pad, dtype=torch.bfloat16, device="cuda")
    p = synth.master_weights(N, N_pad, seed=32, device="cuda")
    m, v = torch.zeros_like(p), torch.zeros_like(p)
    w = torch.zeros(S, dtype=torch.bfloat16, device="cuda")
    flat = torch.zeros(N_pad, dtype=torch.bfloat16, device="cuda")
    step = CollectiveHybridStep(plan, 1, grad, p, m, v, w, flat, node_group, replica_group, reduce_dtype=mode)
    hp_, hm, hv, hw = f32_host(p).copy(), np.zeros(S, np.float32), np.zeros(S, np.float32), np.zeros(S, np.uint16)
    for t in range(1, 4):
        grad.copy_(synth.contribution(N, N_pad, seed=32, step=t, rank=0, sigma=1e-3, device="cuda"))
        step.step(z3.adamw(**hp_for(t)))
        oracle.reduce_adamw_hybrid([synth.bf16_bits(grad)], 1, S, 0, hp_, hm, hv, hw, oracle_hp(t),
                                   reduce_dtype=mode)
    torch.cuda.synchronize()
    assert_f32_parity(f32_host(p), hp_, "master")
    assert_f32_parity(f32_host(m), hm, "exp_avg")
    assert_f32_parity(f32_host(v), hv, "exp_avg_sq")
    assert_bf16_parity(synth.bf16_bits(w), hw, "work_bf16")
    assert np.array_equal(synth.bf16_bits(flat), hw)


@pytest.mark.parametrize("transport", ["peer", "nccl"])
def test_bench_multi_gpu_path_on_a_one_rank_nccl_group(z3, nccl_one_rank, transport):
    """bench.py's N > 1 path (run_collective) on a one-rank NCCL group with the
    real kernels, in both forms (the peer form, then the NCCL form as its
    baseline; the NCCL form alone): CUDA-event timing of every phase, the
    end-to-end leg, the JSON line; the rank's state after every step equals the
    oracle's."""
    import bench
    args = bench.parse_args(["--workload", "tiny_gpt", "--steps", "3", "--warmup", "2", "--e2e-steps", "2",
                             "--transport", transport])
    line, R = bench.run_collective(args, 0, 1, torch.device("cuda", 0), z3, synth)
    assert line["n_gpus"] == 1 and line["comm_nranks"] == 1 and line["value"] > 0 and line["e2e"]["value"] > 0
    assert line["collective"]["reduce_adamw_ms"] > 0
    if transport == "peer":
        assert line["gpu_launches"] == 6 and line["collective"]["gather_ms"] > 0
        assert line["baseline_nccl"]["value"] > 0 and line["baseline_nccl"]["reduce_adamw_ms"] > 0
    else:
        assert line["gpu_launches"] == 3 and "baseline_nccl" not in line
    w = synth.WORKLOADS["tiny_gpt"]
    numels = [synth.numel(s) for _, s in w["tensors"]]
    _, N, N_pad, S = oracle.plan(numels, 1, synth.ALIGN)
    p = synth.master_weights(N, N_pad, seed=1000, device="cuda").cpu().numpy().copy()
    m, v, wk = np.zeros(N_pad, np.float32), np.zeros(N_pad, np.float32), np.zeros(N_pad, np.uint16)
    c = [synth.bf16_bits(synth.contribution(N, N_pad, seed=1000, step=1, rank=0, sigma=w["sigma"], device="cuda"))]
    for t in range(1, R.step_no + 1):
        oracle.reduce_adamw(c, S, -1, p, m, v, wk, oracle_hp(t))
    torch.cuda.synchronize()
    assert_f32_parity(f32_host(R.master), p, "master")
    assert_f32_parity(f32_host(R.exp_avg), m, "exp_avg")
    assert_f32_parity(f32_host(R.exp_avg_sq), v, "exp_avg_sq")
    assert_bf16_parity(synth.bf16_bits(R.work), wk, "work_bf16")
    assert np.array_equal(synth.bf16_bits(R.flat), wk)
