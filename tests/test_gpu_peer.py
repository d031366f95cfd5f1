"""The D-GPU step's code path on one GPU, compared with the oracle: a one-rank
process group (D = 1) with its real fences, and D = 4 ranks emulated as host
threads that share one GPU (the buffers they hand each other stand in for the
IPC mappings of other GPUs' memory; every wait is a host barrier, so no kernel
waits on another).  Groups of several GPUs cannot run here: every run has one
GPU; their host-side logic is tested with gloo ranks in test_peer_host.py."""
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
    plan, ref = checked_plan(z3, [(5000,), (77, 3)], 1, 128)
    N, N_pad, S = ref.N, ref.N_pad, ref.S
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


class ThreadRanks:
    """D ranks emulated as host threads on one GPU, standing in for PeerGroup.

    share(t) hands every rank the D buffers that the ranks passed for the same
    role, in rank order (the k-th call on every rank is the same role), where a
    real group would hand out IPC mappings of the other GPUs' buffers.  fence()
    synchronises the device, then waits for every rank at a thread barrier.
    Every wait is on the host, with a timeout; no kernel waits on another."""

    def __init__(self, rank: int, table: dict, barrier):
        self.rank, self.size = rank, barrier.parties
        self._table, self._barrier, self._calls = table, barrier, 0

    def share(self, t):
        role = self._calls
        self._calls += 1
        self._table.setdefault(role, [None] * self.size)[self.rank] = t
        self._barrier.wait()
        return list(self._table[role])

    def fence(self, device):
        torch.cuda.synchronize(device)
        self._barrier.wait()


@pytest.mark.parametrize("stage,mode", [(3, 0), (3, 1), (2, 0), (1, 1)])
def test_four_ranks_emulated_by_threads_match_oracle(z3, stage, mode):
    """The D-GPU step's own code (PeerZero3Step) with D = 4 ranks: each rank's
    kernel reads slice P_r of every rank's gradient buffer in rank order, then
    the shards are gathered (stage 3) or pushed into every rank's block by the
    kernel (stages 1 and 2).  Every rank's state and gathered block must equal
    the oracle's."""
    import threading

    from fsdp_sharded_mixed_flat_b200.peer import PeerZero3Step
    D = 4
    plan, ref = checked_plan(z3, [(5000,), (77, 3), (4097,)], D, 128)
    N, N_pad, S = ref.N, ref.N_pad, ref.S
    p_full = synth.master_weights(N, N_pad, seed=21, device="cuda")
    grads = [torch.zeros(N_pad, dtype=torch.bfloat16, device="cuda") for _ in range(D)]
    state = [[p_full[r * S:(r + 1) * S].clone(), torch.zeros(S, device="cuda"), torch.zeros(S, device="cuda"),
              torch.zeros(S, dtype=torch.bfloat16, device="cuda")] for r in range(D)]
    flats = [torch.zeros(N_pad, dtype=torch.bfloat16, device="cuda") for _ in range(D)]
    table, barrier = {}, threading.Barrier(D, timeout=120)
    errors = []

    def rank_main(r):
        try:
            step = PeerZero3Step(ThreadRanks(r, table, barrier), plan, grads[r], *state[r], flats[r], stage=stage,
                                 reduce_dtype=mode)
            for t in range(1, 4):
                grads[r].copy_(synth.contribution(N, N_pad, seed=21, step=t, rank=r, sigma=1e-3, device="cuda"))
                step.step(z3.adamw(**hp_for(t)))
            step.peers.fence(step.device)
        except BaseException as e:      # noqa: BLE001  (re-raised on the main thread)
            errors.append(e)
            barrier.abort()

    threads = [threading.Thread(target=rank_main, args=(r,)) for r in range(D)]
    for th in threads:
        th.start()
    for th in threads:
        th.join(timeout=300)
    assert not errors, errors
    assert not any(th.is_alive() for th in threads)

    hp_, hm, hv, hw = f32_host(p_full).copy(), np.zeros(N_pad, np.float32), np.zeros(N_pad, np.float32), \
        np.zeros(N_pad, np.uint16)
    for t in range(1, 4):
        c = [synth.bf16_bits(synth.contribution(N, N_pad, seed=21, step=t, rank=r, sigma=1e-3, device="cuda"))
             for r in range(D)]
        oracle.reduce_adamw(c, S, -1, hp_, hm, hv, hw, oracle_hp(t), reduce_dtype=mode)
    torch.cuda.synchronize()
    for r in range(D):
        sl = slice(r * S, (r + 1) * S)
        what = f"stage {stage} mode {mode} rank {r}"
        assert_f32_parity(f32_host(state[r][0]), hp_[sl], "master " + what)
        assert_f32_parity(f32_host(state[r][1]), hm[sl], "exp_avg " + what)
        assert_f32_parity(f32_host(state[r][2]), hv[sl], "exp_avg_sq " + what)
        assert_bf16_parity(synth.bf16_bits(state[r][3]), hw[sl], "work_bf16 " + what)
        assert np.array_equal(synth.bf16_bits(flats[r]), hw), "gathered block " + what
