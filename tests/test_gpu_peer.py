"""The D-GPU step's code path on one GPU: a one-rank group (D = 1), its fences and
the real kernels, compared with the oracle.  (Groups
of several GPUs cannot run here: every run has one GPU; their host-side logic is
tested with gloo ranks in test_peer_host.py.)"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist

import oracle
import synth
from parity_util import assert_bf16_parity, assert_f32_parity, f32_host, hp_for, oracle_hp

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def z3():
    assert torch.cuda.is_available(), "the GPU tests need a CUDA device"
    from fsdp_sharded_mixed_flat_b200 import build
    build.build()
    from fsdp_sharded_mixed_flat_b200 import zero3
    return zero3


@pytest.fixture()
def one_rank_group():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=0, world_size=1)
    yield
    dist.destroy_process_group()


@pytest.mark.parametrize("stage", [3, 2])
def test_one_rank_group_matches_oracle(z3, one_rank_group, stage):
    from fsdp_sharded_mixed_flat_b200.peer import PeerGroup, PeerZero3Step
    plan = z3.zero3_plan([(5000,), (77, 3)], 1, 128)
    N, N_pad, S = plan.N, plan.N_pad, plan.S
    grad = torch.zeros(N_pad, dtype=torch.bfloat16, device="cuda")
    p = synth.master_weights(N, N_pad, seed=12, device="cuda")
    m, v = torch.zeros_like(p), torch.zeros_like(p)
    w = torch.zeros(S, dtype=torch.bfloat16, device="cuda")
    flat = torch.zeros(N_pad, dtype=torch.bfloat16, device="cuda")
    step = PeerZero3Step(PeerGroup(), plan, grad, p, m, v, w, flat, stage=stage)
    hp_, hm, hv, hw = f32_host(p).copy(), np.zeros(S, np.float32), np.zeros(S, np.float32), np.zeros(S, np.uint16)
    for t in range(1, 4):
        grad.copy_(synth.contribution(N, N_pad, seed=12, step=t, rank=0, sigma=1e-3, device="cuda"))
        step.step(z3.adamw(**hp_for(t)))
        oracle.reduce_adamw([synth.bf16_bits(grad)], S, 0, hp_, hm, hv, hw, oracle_hp(t))
    torch.cuda.synchronize()
    assert_f32_parity(f32_host(p), hp_, "master")
    assert_f32_parity(f32_host(m), hm, "exp_avg")
    assert_f32_parity(f32_host(v), hv, "exp_avg_sq")
    assert_bf16_parity(synth.bf16_bits(w), hw, "work_bf16")
    assert np.array_equal(synth.bf16_bits(flat), hw)
