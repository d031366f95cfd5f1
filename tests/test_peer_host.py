"""Host-side logic of the D-GPU step (fsdp_sharded_mixed_flat_b200/peer.py) on
world-size-2 gloo groups, on CPU: the IPC exchange hands every rank all ranks'
buffers in rank order, and each step fences, launches and fences in the right
order with this rank's own arguments.  The IPC mapping and the kernels are
replaced by stand-ins that record what they are given."""
import os
import socket

import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


class FakePlan:
    def __init__(self, D):
        self.D = D


class FakeKernels:
    Z3_CONTRIB_FULL = 0

    def __init__(self, log):
        self.log = log

    def zero3_reduce_adamw(self, plan, rank, contrib, master, m, v, work, hp, contrib_layout, reduce_dtype):
        self.log.append(("reduce", rank, [int(c[0]) for c in contrib], int(master[0]), int(work[0]), hp))

    def zero3_reduce_adamw_gather(self, plan, rank, contrib, master, m, v, work, gathered, hp, contrib_layout,
                                  reduce_dtype):
        self.log.append(("fused", rank, [int(c[0]) for c in contrib], [int(g[0]) for g in gathered], hp))

    def zero3_gather_block(self, plan, shards, flat, tensor_out):
        self.log.append(("gather", [int(s[0]) for s in shards], int(flat[0])))


def _worker(rank, world, port, stage, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    from fsdp_sharded_mixed_flat_b200.peer import PeerGroup, PeerZero3Step
    log = []
    peers = PeerGroup(share_fn=lambda t: int(t[0]), open_fn=lambda v: torch.full((4,), v),
                      sync_fn=lambda device: log.append(("fence",)))
    tag = lambda base: torch.full((4,), base + rank)   # noqa: E731
    step = PeerZero3Step(peers, FakePlan(world), tag(100), tag(300), tag(400), tag(500), tag(200), tag(600),
                         stage=stage, kernels=FakeKernels(log))
    step.step("hp1")
    step.step("hp2")
    out[rank] = log
    dist.barrier()
    dist.destroy_process_group()


def _run(stage):
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        port = _free_port()
        procs = [ctx.Process(target=_worker, args=(r, 2, port, stage, out)) for r in range(2)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(120)
            assert p.exitcode == 0
        return dict(out)


def test_zero3_step_order_and_arguments():
    logs = _run(3)
    for rank in (0, 1):
        expect = []
        for hp in ("hp1", "hp2"):
            expect += [("fence",), ("reduce", rank, [100, 101], 300 + rank, 200 + rank, hp), ("fence",),
                       ("gather", [200, 201], 600 + rank)]
        assert logs[rank] == expect


def test_fused_zero12_step_order_and_arguments():
    logs = _run(2)
    for rank in (0, 1):
        expect = []
        for hp in ("hp1", "hp2"):
            expect += [("fence",), ("fused", rank, [100, 101], [600, 601], hp), ("fence",)]
        assert logs[rank] == expect
