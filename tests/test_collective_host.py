"""The collective steps (fsdp_sharded_mixed_flat_b200/collective.py) on CPU:
gloo groups move the real bytes (all-to-all of the gradients, all-gathers of
the node sums and of the shards), and the oracle stands in for the kernels on
each rank.  ZeRO-3 over 2 and 4 ranks, and HYBRID_SHARD over 2 and 3 nodes of
2 ranks (node and replica subgroups): every rank's state and gathered block
must equal a single-process oracle run over all ranks, bit for bit."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
import synth

SHAPES = [(3000,), (77, 5), (4097,)]
SEED = 5


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _bits(t: torch.Tensor) -> np.ndarray:
    """A host bf16 tensor's storage as uint16 bit patterns (shared, not copied)."""
    return t.view(torch.int16).numpy().view(np.uint16)


class OracleKernels:
    """The kernels' entry points, computed by the oracle on host tensors."""
    Z3_CONTRIB_OWNED = oracle.LAYOUT_OWNED
    Z3_CONTRIB_FULL = oracle.LAYOUT_FULL

    @staticmethod
    def _hp(hp):
        return oracle.hp(hp.lr, hp.beta1, hp.beta2, hp.eps, hp.weight_decay, hp.step)

    def zero3_node_sum(self, plan, rank, contrib, node_sum, contrib_layout, reduce_dtype):
        vals = oracle.node_sum([_bits(c) for c in contrib], plan.S, rank, contrib_layout, reduce_dtype)
        node_sum.copy_(torch.from_numpy(vals).to(node_sum.dtype))      # exact: bf16 sums are bf16 values

    def zero3_fold_adamw(self, plan, rank, node_sums, master, exp_avg, exp_avg_sq, work, hp, reduce_dtype):
        oracle.fold_adamw([x.float().numpy() for x in node_sums], plan.D, master.numpy(), exp_avg.numpy(),
                          exp_avg_sq.numpy(), _bits(work), self._hp(hp), reduce_dtype=reduce_dtype)

    def zero3_reduce_adamw(self, plan, rank, contrib, master, exp_avg, exp_avg_sq, work, hp, contrib_layout,
                           reduce_dtype):
        assert contrib_layout in (oracle.LAYOUT_OWNED, oracle.LAYOUT_FULL)
        oracle.reduce_adamw([_bits(c) for c in contrib], plan.S, rank, master.numpy(), exp_avg.numpy(),
                            exp_avg_sq.numpy(), _bits(work),
                            oracle.hp(hp.lr, hp.beta1, hp.beta2, hp.eps, hp.weight_decay, hp.step),
                            layout=contrib_layout, reduce_dtype=reduce_dtype)

    def zero3_reduce_adamw_gather(self, plan, rank, contrib, master, exp_avg, exp_avg_sq, work, gathered, hp,
                                  contrib_layout, reduce_dtype):
        self.zero3_reduce_adamw(plan, rank, contrib, master, exp_avg, exp_avg_sq, work, hp, contrib_layout,
                                reduce_dtype)
        for g in gathered:                                  # the new shard into every rank's block
            _bits(g)[rank * plan.S:(rank + 1) * plan.S] = _bits(work)

    def zero3_gather_block(self, plan, shards, flat, tensor_out=None):
        assert tensor_out is None
        _bits(flat)[:] = oracle.all_gather([_bits(x) for x in shards], plan.S)


def file_peer_group(tmpdir: str, rank: int):
    """A PeerGroup whose "IPC" is a file every rank maps (host memory shared
    between the gloo processes): share() moves the tensor's storage into a
    fresh shared file mapping, so this rank's later writes are seen by every
    rank that opened it."""
    import itertools

    from fsdp_sharded_mixed_flat_b200.peer import PeerGroup
    count = itertools.count()

    def share(t):
        path = os.path.join(tmpdir, f"rank{rank}_{next(count)}")
        mapped = torch.from_file(path, shared=True, size=t.numel(), dtype=t.dtype)
        mapped.copy_(t)
        t.set_(mapped)
        return path, t.numel(), t.dtype

    def open_(handle):
        path, n, dtype = handle
        return torch.from_file(path, shared=True, size=n, dtype=dtype)

    return PeerGroup(share_fn=share, open_fn=open_, sync_fn=lambda device: None)


def _worker(rank, world, port, mode, steps, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    from fsdp_sharded_mixed_flat_b200 import zero3 as z3
    from fsdp_sharded_mixed_flat_b200.collective import CollectiveZero3Step
    plan = z3.zero3_plan(SHAPES, world, 8)
    N, N_pad, S = plan.N, plan.N_pad, plan.S
    p_full = synth.master_weights(N, N_pad, seed=SEED)
    grad = torch.zeros(N_pad, dtype=torch.bfloat16)
    master = p_full[rank * S:(rank + 1) * S].clone()
    m, v = torch.zeros(S), torch.zeros(S)
    work = torch.zeros(S, dtype=torch.bfloat16)
    flat = torch.zeros(N_pad, dtype=torch.bfloat16)
    step = CollectiveZero3Step(plan, grad, master, m, v, work, flat, reduce_dtype=mode, kernels=OracleKernels())
    for t in range(1, steps + 1):
        grad.copy_(synth.contribution(N, N_pad, seed=SEED, step=t, rank=rank, sigma=1e-3))
        step.step(z3.adamw(step=t))
    out[rank] = (master.numpy().copy(), m.numpy().copy(), v.numpy().copy(), _bits(work).copy(), _bits(flat).copy())
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("world,mode", [(2, 0), (4, 0), (4, 1)])
def test_collective_step_equals_one_oracle_run_over_all_ranks(world, mode):
    steps = 3
    with mp.get_context("spawn").Manager() as manager:
        out = manager.dict()
        mp.spawn(_worker, args=(world, _free_port(), mode, steps, out), nprocs=world, join=True)
        results = dict(out)
    offs, N, N_pad, S = oracle.plan([int(np.prod(s)) for s in SHAPES], world, 8)
    p = synth.master_weights(N, N_pad, seed=SEED).numpy().copy()
    m, v, w = np.zeros(N_pad, np.float32), np.zeros(N_pad, np.float32), np.zeros(N_pad, np.uint16)
    for t in range(1, steps + 1):
        c = [synth.bf16_bits(synth.contribution(N, N_pad, seed=SEED, step=t, rank=d, sigma=1e-3))
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


def test_collective_step_rejects_a_plan_for_another_group_size():
    port = _free_port()
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=0, world_size=1)
    try:
        from fsdp_sharded_mixed_flat_b200 import zero3 as z3
        from fsdp_sharded_mixed_flat_b200.collective import CollectiveZero3Step
        plan = z3.zero3_plan(SHAPES, 2, 8)
        bf = lambda n: torch.zeros(n, dtype=torch.bfloat16)   # noqa: E731
        with pytest.raises(ValueError, match="group has 1"):
            CollectiveZero3Step(plan, bf(plan.N_pad), torch.zeros(plan.S), torch.zeros(plan.S),
                                torch.zeros(plan.S), bf(plan.S), bf(plan.N_pad))
        plan1 = z3.zero3_plan(SHAPES, 1, 8)
        with pytest.raises(ValueError, match="flat"):
            CollectiveZero3Step(plan1, bf(plan1.N_pad), torch.zeros(plan1.S), torch.zeros(plan1.S),
                                torch.zeros(plan1.S), bf(plan1.S), bf(plan1.N_pad - 1))
    finally:
        dist.destroy_process_group()


def _hybrid_worker(rank, R, D, port, mode, steps, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=R * D)
    from fsdp_sharded_mixed_flat_b200 import zero3 as z3
    from fsdp_sharded_mixed_flat_b200.collective import CollectiveHybridStep, hybrid_groups
    node_group, replica_group = hybrid_groups(R, D)
    plan = z3.zero3_plan(SHAPES, D, 8)
    N, N_pad, S = plan.N, plan.N_pad, plan.S
    d = rank % D
    p_full = synth.master_weights(N, N_pad, seed=SEED)
    grad = torch.zeros(N_pad, dtype=torch.bfloat16)
    master = p_full[d * S:(d + 1) * S].clone()
    m, v = torch.zeros(S), torch.zeros(S)
    work = torch.zeros(S, dtype=torch.bfloat16)
    flat = torch.zeros(N_pad, dtype=torch.bfloat16)
    step = CollectiveHybridStep(plan, R, grad, master, m, v, work, flat, node_group, replica_group,
                                reduce_dtype=mode, kernels=OracleKernels())
    for t in range(1, steps + 1):
        grad.copy_(synth.contribution(N, N_pad, seed=SEED, step=t, rank=rank, sigma=1e-3))
        step.step(z3.adamw(step=t))
    out[rank] = (master.numpy().copy(), m.numpy().copy(), v.numpy().copy(), _bits(work).copy(), _bits(flat).copy())
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("R,D,mode", [(2, 2, 0), (2, 2, 1), (3, 2, 0)])
def test_collective_hybrid_step_equals_the_two_level_oracle(R, D, mode):
    """HYBRID_SHARD over R nodes of D gloo ranks: every rank equals one oracle
    run of the two-level reduction over all R*D ranks, bit for bit, and every
    replica of a local rank holds the same state."""
    steps = 3
    with mp.get_context("spawn").Manager() as manager:
        out = manager.dict()
        mp.spawn(_hybrid_worker, args=(R, D, _free_port(), mode, steps, out), nprocs=R * D, join=True)
        results = dict(out)
    offs, N, N_pad, S = oracle.plan([int(np.prod(s)) for s in SHAPES], D, 8)
    p = synth.master_weights(N, N_pad, seed=SEED).numpy().copy()
    m, v, w = np.zeros(N_pad, np.float32), np.zeros(N_pad, np.float32), np.zeros(N_pad, np.uint16)
    for t in range(1, steps + 1):
        c = [synth.bf16_bits(synth.contribution(N, N_pad, seed=SEED, step=t, rank=g, sigma=1e-3))
             for g in range(R * D)]
        oracle.reduce_adamw_hybrid(c, R, S, -1, p, m, v, w, oracle.hp(step=t), reduce_dtype=mode)
    for g in range(R * D):
        rp, rm, rv, rw, rflat = results[g]
        d = g % D
        sl = slice(d * S, (d + 1) * S)
        assert np.array_equal(rp.view(np.uint32), p[sl].view(np.uint32)), f"master rank {g}"
        assert np.array_equal(rm.view(np.uint32), m[sl].view(np.uint32)), f"exp_avg rank {g}"
        assert np.array_equal(rv.view(np.uint32), v[sl].view(np.uint32)), f"exp_avg_sq rank {g}"
        assert np.array_equal(rw, w[sl]), f"work rank {g}"
        assert np.array_equal(rflat, w), f"gathered block rank {g}"


def _failing_worker(rank, world, port, how, form, tmpdir, out):
    import time
    from datetime import timedelta
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=3))
    from fsdp_sharded_mixed_flat_b200 import zero3 as z3
    from fsdp_sharded_mixed_flat_b200.collective import CollectiveZero3Step
    plan = z3.zero3_plan(SHAPES, world, 8)
    N, N_pad, S = plan.N, plan.N_pad, plan.S
    grad = synth.contribution(N, N_pad, seed=SEED, step=1, rank=rank, sigma=1e-3)
    master = synth.master_weights(N, N_pad, seed=SEED)[rank * S:(rank + 1) * S].clone()
    m, v = torch.zeros(S), torch.zeros(S)
    work, flat = torch.zeros(S, dtype=torch.bfloat16), torch.zeros(N_pad, dtype=torch.bfloat16)
    if form == "peer":                               # the fused peer-memory step, fences = gloo barriers
        from fsdp_sharded_mixed_flat_b200.peer import PeerZero3Step
        step = PeerZero3Step(file_peer_group(tmpdir, rank), plan, grad, master, m, v, work, flat,
                             kernels=OracleKernels())
    else:
        step = CollectiveZero3Step(plan, grad, master, m, v, work, flat, kernels=OracleKernels())
    step.step(z3.adamw(step=1))                      # a whole step with every rank
    if rank == world - 1:                            # the failing rank leaves between steps
        if how == "stall":
            time.sleep(15)
        out[rank] = "left"
        os._exit(0)                                  # no goodbye to the group
    t0 = time.monotonic()
    try:
        step.step(z3.adamw(step=2))
        out[rank] = ("no error", time.monotonic() - t0)
    except Exception as e:                           # noqa: BLE001
        out[rank] = (type(e).__name__, time.monotonic() - t0)
    os._exit(0)


@pytest.mark.parametrize("form", ["nccl", "peer"])
@pytest.mark.parametrize("how", ["exit", "stall"])
def test_collective_step_surfaces_a_lost_rank_as_an_error(how, form, tmp_path):
    """A rank that exits, or stops answering, between steps: the surviving ranks'
    next step ends with an error from the process group (a closed connection, or
    its 3-second timeout), well before the lost rank would have come back; no rank
    waits forever.  Both forms of the step: collectives moving the bytes, and the
    peer-memory step whose fences are group barriers.  (Failure detection made on
    the host, with gloo ranks.)"""
    world = 3
    ctx = mp.get_context("spawn")
    with ctx.Manager() as manager:
        out = manager.dict()
        port = _free_port()
        procs = [ctx.Process(target=_failing_worker, args=(r, world, port, how, form, str(tmp_path), out))
                 for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(120)
            assert p.exitcode == 0, "a rank did not end"
        res = dict(out)
    assert res[world - 1] == "left"
    for r in range(world - 1):
        kind, secs = res[r]
        assert kind != "no error", f"rank {r} finished a step without the lost rank"
        assert secs < 14, f"rank {r} took {secs:.1f} s to notice"
