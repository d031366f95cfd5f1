"""Host-side tests of the C ABI (no GPU needed): the library loads and exports
every entry point include/zero3.h declares, the planner and the memory ledger
agree with the oracle, and every argument error is reported before any device
work.  No call here reaches a CUDA API: each one either fails validation or
has nothing to do (an empty plan)."""
import ctypes as C
import os
import random
import re
import subprocess

import numpy as np
import pytest
import torch

import oracle
import synth
from fsdp_sharded_mixed_flat_b200 import build as pkg_build

pkg_build.build()
from fsdp_sharded_mixed_flat_b200 import zero3 as z3  # noqa: E402

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "zero3.h")


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"Z3_API\s+[\w\s\*]+?\b(zero3_\w+)\s*\(", text)))


def test_library_exports_every_declared_symbol():
    names = declared_symbols()
    assert names == sorted(["zero3_status_string", "zero3_plan", "zero3_plan_free", "zero3_plan_info",
                            "zero3_plan_tensor", "zero3_plan_rank", "zero3_memory_bytes",
                            "zero3_transient_bytes", "zero3_allgather_bytes", "zero3_reduce_adamw",
                            "zero3_reduce_adamw_hybrid", "zero3_node_sum", "zero3_fold_adamw",
                            "zero3_reduce_adamw_gather",
                            "zero3_step_scalars", "zero3_reduce_adamw_dev", "zero3_gather_block",
                            "zero3_reduce_scatter", "zero3_host_adamw", "zero3_ipc_export",
                            "zero3_ipc_import", "zero3_ipc_close"]), names
    out = subprocess.run(["nm", "-D", "--defined-only", z3.LIB_PATH], capture_output=True, text=True,
                         check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if line.strip()}
    for n in names:
        assert n in exported, n
        assert hasattr(z3.lib(), n)
    # nothing else of ours (and none of the static CUDA runtime) leaks out
    leaked = sorted(s for s in exported if s.startswith("cuda") or s.startswith("_ZN"))
    assert not leaked, leaked[:10]


def test_status_strings():
    for s in (0, -1, -2, -3, -4, -5):
        assert z3.status_string(s) and z3.status_string(s) != "unknown status"
    assert z3.status_string(-99) == "unknown status"


# ------------------------------------------------------------------ planner
def test_plan_matches_oracle_brute_force():
    rnd = random.Random(5)
    for _ in range(300):
        shapes = [tuple(rnd.randint(1, 9) for _ in range(rnd.randint(0, 4))) for _ in range(rnd.randint(0, 8))]
        D = rnd.randint(1, 64)
        A = rnd.choice([1, 2, 3, 8, 16, 128, 1000])
        p = z3.zero3_plan(shapes, D, A)
        numels = [int(np.prod(s)) if s else 1 for s in shapes]
        offs, N, N_pad, S = oracle.plan(numels, D, A)
        assert (p.N, p.N_pad, p.S, p.D, p.align_elems, p.n_tensors) == (N, N_pad, S, D, A, len(shapes))
        assert p.offsets == list(offs) and p.numels == numels
        for r in range(D):
            assert p.rank_range(r) == oracle.rank_range(N, S, r)


def test_plan_workloads_match_oracle():
    for name, w in synth.WORKLOADS.items():
        D = w["D"]
        p = z3.zero3_plan([s for _, s in w["tensors"]], D, synth.ALIGN)
        offs, N, N_pad, S = oracle.plan([synth.numel(s) for _, s in w["tensors"]], D, synth.ALIGN)
        assert (p.N, p.N_pad, p.S) == (N, N_pad, S) and p.offsets == list(offs)


def test_plan_errors():
    with pytest.raises(z3.Zero3Error) as e:
        z3.zero3_plan([(3,)], 0)
    assert e.value.status == z3.Z3_EINVAL
    for bad in [dict(D=65), dict(D=1, align_elems=0), dict(D=-1)]:
        with pytest.raises(z3.Zero3Error):
            z3.zero3_plan([(3,)], **bad)
    # shape product must equal numel
    spec = (z3.TensorSpec * 1)()
    spec[0].numel, spec[0].ndim = 7, 2
    spec[0].shape[0], spec[0].shape[1] = 2, 3
    h = C.c_void_p()
    assert z3.lib().zero3_plan(spec, 1, 2, 1, C.byref(h)) == z3.Z3_EINVAL
    spec[0].numel, spec[0].ndim = 6, 5
    assert z3.lib().zero3_plan(spec, 1, 2, 1, C.byref(h)) == z3.Z3_EINVAL
    spec[0].numel, spec[0].ndim = -1, 0
    assert z3.lib().zero3_plan(spec, 1, 2, 1, C.byref(h)) == z3.Z3_EINVAL
    assert z3.lib().zero3_plan(spec, 1, 2, 1, None) == z3.Z3_EINVAL
    # overflow: N itself beyond 2^62, and a padded size beyond 2^62 (2^62 - 1 = 3 mod 7)
    two = (z3.TensorSpec * 2)()
    for k in range(2):
        two[k].numel, two[k].ndim, two[k].shape[0] = 2 ** 61 + 1, 1, 2 ** 61 + 1
    assert z3.lib().zero3_plan(two, 2, 1, 1, C.byref(h)) == z3.Z3_EOVERFLOW
    spec[0].numel, spec[0].ndim = 2 ** 62 - 1, 1
    spec[0].shape[0] = 2 ** 62 - 1
    assert z3.lib().zero3_plan(spec, 1, 7, 1, C.byref(h)) == z3.Z3_EOVERFLOW
    assert z3.lib().zero3_plan(spec, 1, 3, 1, C.byref(h)) == z3.Z3_OK
    z3.lib().zero3_plan_free(h)
    p = z3.zero3_plan([(3,)], 2)
    with pytest.raises(z3.Zero3Error):
        z3.zero3_plan_tensor(p, 1)
    with pytest.raises(z3.Zero3Error):
        p.rank_range(2)


def test_plan_scalar_and_empty():
    p = z3.zero3_plan([(), (4,)], 2, 1)
    assert p.numels == [1, 4] and p.N == 5 and p.N_pad == 6 and p.S == 3
    e = z3.zero3_plan([], 4, 128)
    assert (e.N, e.N_pad, e.S) == (0, 0, 0)


# ------------------------------------------------------------------- ledger
def test_memory_bytes_matches_oracle():
    rnd = random.Random(9)
    cases = [(7_000_000_000, 32), (70_000_000_000, 8), (202_383_360, 8), (1, 1), (0, 5)]
    cases += [(rnd.randint(0, 10 ** 13), rnd.randint(1, 4096)) for _ in range(200)]
    for N, D in cases:
        for stage in range(4):
            got = z3.zero3_memory_bytes(N, D, stage)
            ref = oracle.memory_bytes(N, D, stage)
            # the ABI rounds each sharded term up to a whole byte; the oracle is real-valued
            assert ref - 1e-6 * max(1.0, ref) <= got <= ref + 1 + 1e-6 * max(1.0, ref), (N, D, stage)
            if (20 * N) % D == 0 and (12 * N) % D == 0 and (18 * N) % D == 0:
                assert got == round(ref)
    with pytest.raises(z3.Zero3Error):
        z3.zero3_memory_bytes(10, 2, 4)
    with pytest.raises(z3.Zero3Error):
        z3.zero3_memory_bytes(-1, 2, 3)
    with pytest.raises(z3.Zero3Error) as e:
        z3.zero3_memory_bytes(2 ** 62, 2, 0)
    assert e.value.status == z3.Z3_EOVERFLOW


def test_transient_bytes_matches_oracle():
    for block in (0, 1, 12 * 4096 * 4096, 855_654_400):
        for nb in (0, 1, 2):
            assert z3.zero3_transient_bytes(block, nb) == oracle.transient_bytes(block, nb)


def test_allgather_bytes_matches_oracle():
    """The ABI's integer all-gather volume is the oracle's, rounded up to a byte."""
    for block in (0, 1, 3, 12 * 4096 * 4096, 855_654_400, 100_000_000):
        for nb in (0, 1, 32, 80):
            for D in (1, 2, 3, 8, 32, 64):
                ref = oracle.allgather_bytes(2.0 * block, nb, D)
                got = z3.zero3_allgather_bytes(block, nb, D)
                exact_num = nb * 2 * block * (D - 1)          # the exact value is exact_num / D
                assert got == -(-exact_num // D), (block, nb, D)
                assert abs(got - ref) <= 1.0 + 1e-12 * ref
    # the page's figure: 32 blocks of 200 MB (100M bf16 parameters) at D = 32
    assert z3.zero3_allgather_bytes(100_000_000, 32, 32) == 6_200_000_000
    with pytest.raises(z3.Zero3Error) as e:
        z3.zero3_allgather_bytes(1, 1, 0)
    assert e.value.status == z3.Z3_EINVAL
    with pytest.raises(z3.Zero3Error) as e:
        z3.zero3_allgather_bytes(2 ** 62, 2, 2)
    assert e.value.status == z3.Z3_EOVERFLOW


# ------------------------------------------- argument errors, no device work
P16 = 0x10000  # fake, 16-byte aligned device addresses: never dereferenced here


def call_reduce(plan, rank=-1, contrib=None, layout=0, ptrs=None, mode=0, hp=None):
    D = plan.D
    if contrib is None:
        contrib = [P16 * (100 + d) for d in range(D)]
    arr = (C.c_void_p * max(1, D))(*contrib)
    ptrs = ptrs or [P16 * 1, P16 * 2, P16 * 3, P16 * 4]
    hp = hp or z3.adamw(step=1)
    return z3.lib().zero3_reduce_adamw(plan.handle, rank, arr, layout, *[C.c_void_p(x) for x in ptrs],
                                       mode, C.byref(hp), None)


def test_reduce_adamw_argument_errors():
    p = z3.zero3_plan([(1000,)], 4, 8)   # S = 256 elements = 1 KiB fp32
    E = z3.Z3_EINVAL
    assert call_reduce(p, rank=4) == E
    assert call_reduce(p, rank=-2) == E
    assert call_reduce(p, layout=1) == E                     # owned layout needs one rank
    assert call_reduce(p, layout=7, rank=0) == E
    assert call_reduce(p, mode=2) == E
    assert call_reduce(p, contrib=[P16, 0, P16 * 3, P16 * 4]) == E
    assert call_reduce(p, ptrs=[0, P16 * 2, P16 * 3, P16 * 4]) == E
    assert call_reduce(p, hp=z3.adamw(step=0)) == E
    assert call_reduce(p, hp=z3.adamw(beta1=1.0)) == E
    assert call_reduce(p, hp=z3.adamw(lr=float("nan"))) == E
    assert call_reduce(p, hp=z3.adamw(eps=float("inf"))) == E
    # eps = 0 would make a zero pad element compute 0/0; negative lr or decay are not AdamW
    assert call_reduce(p, hp=z3.adamw(eps=0.0)) == E
    assert call_reduce(p, hp=z3.adamw(eps=-1e-8)) == E
    assert call_reduce(p, hp=z3.adamw(lr=-1e-4)) == E
    assert call_reduce(p, hp=z3.adamw(weight_decay=-0.1)) == E
    assert z3.lib().zero3_reduce_adamw(None, 0, None, 0, None, None, None, None, 0, None, None) == E
    # misaligned: fp32 state off a 4-byte boundary, bf16 off a 2-byte boundary
    assert call_reduce(p, ptrs=[P16 + 2, P16 * 2, P16 * 3, P16 * 4]) == z3.Z3_EALIGN
    assert call_reduce(p, ptrs=[P16, P16 * 2, P16 * 3, P16 * 4 + 1]) == z3.Z3_EALIGN
    assert call_reduce(p, contrib=[P16 * 100 + 1] + [P16 * 101] * 3) == z3.Z3_EALIGN
    # overlapping outputs, and an output over a contribution it reads
    n_bytes = p.N_pad * 4
    assert call_reduce(p, ptrs=[P16 * 10, P16 * 10 + n_bytes - 4, P16 * 30, P16 * 40]) == E
    assert call_reduce(p, contrib=[P16 * 40] * 4, ptrs=[P16 * 10, P16 * 20, P16 * 30, P16 * 40]) == E
    # rank 1 reads contributions at [S, 2S): an output over that range is rejected
    S = p.S
    base = P16 * 1000
    assert call_reduce(p, rank=1, contrib=[base] * 4, ptrs=[base + 2 * S, P16 * 20, P16 * 30, P16 * 40]) == E


def call_hybrid(plan, n_nodes, contrib=None, rank=-1, ptrs=None, count=None):
    n = plan.D * n_nodes if count is None else count
    if contrib is None:
        contrib = [P16 * (100 + d) for d in range(n)]
    arr = (C.c_void_p * max(1, len(contrib)))(*contrib)
    ptrs = ptrs or [P16 * 1, P16 * 2, P16 * 3, P16 * 4]
    hp = z3.adamw(step=1)
    return z3.lib().zero3_reduce_adamw_hybrid(plan.handle, rank, n_nodes, arr, 0, *[C.c_void_p(x) for x in ptrs],
                                              0, C.byref(hp), None)


def test_reduce_adamw_hybrid_argument_errors():
    p = z3.zero3_plan([(1000,)], 4, 8)
    E = z3.Z3_EINVAL
    assert call_hybrid(p, 0, contrib=[P16 * 100] * 4) == E            # at least one node
    assert call_hybrid(p, -1, contrib=[P16 * 100] * 4) == E
    assert call_hybrid(p, 17) == E                                    # 17 * 4 ranks > Z3_D_MAX
    assert call_hybrid(p, 2, rank=4) == E
    c = [P16 * (100 + d) for d in range(8)]
    assert call_hybrid(p, 2, contrib=c[:5] + [0] + c[6:]) == E        # a NULL contribution on node 1
    assert call_hybrid(p, 2, contrib=c[:7] + [c[7] + 1]) == z3.Z3_EALIGN
    assert call_hybrid(p, 2, contrib=c[:6] + [P16 * 3] + c[7:]) == E  # exp_avg_sq over a node-1 contribution
    assert z3.lib().zero3_reduce_adamw_hybrid(p.handle, -1, 2, None, 0, None, None, None, None, 0, None,
                                              None) == E
    e = z3.zero3_plan([], 4, 8)
    assert call_hybrid(e, 16) == z3.Z3_OK                             # 64 contributions, empty plan
    assert call_hybrid(e, 1) == z3.Z3_OK


def test_reduce_scatter_argument_errors():
    p = z3.zero3_plan([(1000,)], 4, 8)
    L, E, A = z3.lib(), z3.Z3_EINVAL, z3.Z3_EALIGN
    c = [P16 * (100 + d) for d in range(4)]

    def rs(contrib=c, rank=-1, layout=0, mode=0, out=P16 * 50):
        arr = (C.c_void_p * 4)(*contrib)
        return L.zero3_reduce_scatter(p.handle, rank, arr, layout, mode, None if out is None else C.c_void_p(out),
                                      None)
    assert rs(out=None) == E
    assert rs(rank=4) == E
    assert rs(rank=-2) == E
    assert rs(layout=1) == E                             # owned layout needs one rank
    assert rs(mode=2) == E
    assert rs(contrib=c[:3] + [0]) == E
    assert rs(contrib=c[:3] + [c[3] + 1]) == A
    assert rs(out=P16 * 50 + 2) == A                      # fp32 gradient needs 4-byte alignment
    assert rs(out=c[1]) == E                              # over a contribution
    e = z3.zero3_plan([], 4, 8)
    assert L.zero3_reduce_scatter(e.handle, -1, (C.c_void_p * 4)(*c), 0, 1, C.c_void_p(P16 * 50), None) == z3.Z3_OK


def test_node_sum_and_fold_argument_errors():
    p = z3.zero3_plan([(1000,)], 4, 8)
    L, E, A = z3.lib(), z3.Z3_EINVAL, z3.Z3_EALIGN
    c = [P16 * (100 + d) for d in range(4)]

    def node_sum(contrib=c, rank=-1, layout=0, mode=0, out=P16 * 50):
        arr = (C.c_void_p * 4)(*contrib)
        return L.zero3_node_sum(p.handle, rank, arr, layout, mode, None if out is None else C.c_void_p(out), None)
    assert node_sum(out=None) == E
    assert node_sum(rank=4) == E
    assert node_sum(layout=1) == E                       # owned layout needs one rank
    assert node_sum(mode=2) == E
    assert node_sum(contrib=c[:3] + [0]) == E
    assert node_sum(contrib=c[:3] + [c[3] + 1]) == A
    assert node_sum(out=P16 * 50 + 2) == A                # fp32 sums need 4-byte alignment
    assert node_sum(out=c[2]) == E                        # over a contribution
    hp = z3.adamw(step=1)

    def fold(sums=(P16 * 200, P16 * 300), n_nodes=None, rank=-1, ptrs=None, mode=0, h=hp):
        arr = (C.c_void_p * max(1, len(sums)))(*sums)
        ptrs = ptrs or [P16 * 1, P16 * 2, P16 * 3, P16 * 4]
        return L.zero3_fold_adamw(p.handle, rank, len(sums) if n_nodes is None else n_nodes, arr,
                                  *[C.c_void_p(x) for x in ptrs], mode, None if h is None else C.byref(h), None)
    assert fold(n_nodes=0) == E
    assert fold(n_nodes=65) == E
    assert fold(rank=4) == E
    assert fold(mode=3) == E
    assert fold(h=None) == E
    assert fold(h=z3.adamw(step=0)) == E
    assert fold(sums=(P16 * 200, 0)) == E
    assert fold(sums=(P16 * 200, P16 * 300 + 2)) == A
    assert fold(ptrs=[P16 + 2, P16 * 2, P16 * 3, P16 * 4]) == A
    assert fold(ptrs=[P16 * 10, P16 * 10, P16 * 30, P16 * 40]) == E   # master = exp_avg
    assert fold(sums=(P16 * 200, P16 * 3)) == E                       # exp_avg_sq over a node sum
    e = z3.zero3_plan([], 4, 8)
    assert L.zero3_fold_adamw(e.handle, -1, 2, (C.c_void_p * 2)(P16 * 200, P16 * 300), C.c_void_p(P16),
                              C.c_void_p(P16 * 2), C.c_void_p(P16 * 3), C.c_void_p(P16 * 4), 0, C.byref(hp),
                              None) == z3.Z3_OK
    assert L.zero3_node_sum(e.handle, -1, (C.c_void_p * 4)(*c), 0, 0, C.c_void_p(P16 * 50), None) == z3.Z3_OK


def call_fused(plan, gathered, work=P16 * 4, rank=-1, n=None):
    D = plan.D
    arr = (C.c_void_p * D)(*[P16 * (100 + d) for d in range(D)])
    ga = (C.c_void_p * max(1, len(gathered)))(*gathered)
    hp = z3.adamw(step=1)
    return z3.lib().zero3_reduce_adamw_gather(plan.handle, rank, arr, 0, C.c_void_p(P16 * 1), C.c_void_p(P16 * 2),
                                              C.c_void_p(P16 * 3), None if work is None else C.c_void_p(work), ga,
                                              len(gathered) if n is None else n, 0, C.byref(hp), None)


def test_reduce_adamw_gather_argument_errors():
    p = z3.zero3_plan([(1000,)], 4, 8)
    E = z3.Z3_EINVAL
    far = P16 * 5000
    assert call_fused(p, [far], n=0) == E                         # at least one gathered block
    assert call_fused(p, [far] * 9) == E                          # at most Z3_GATHER_MAX
    assert call_fused(p, [far, 0]) == E                           # a NULL gathered block
    assert call_fused(p, [far + 1]) == z3.Z3_EALIGN
    assert call_fused(p, [far, far + 2]) == E                     # gathered blocks overlap
    assert call_fused(p, [P16 * 3]) == E                          # over exp_avg_sq
    assert call_fused(p, [P16 * 100]) == E                        # over a contribution
    e = z3.zero3_plan([], 4, 8)
    assert call_fused(e, [far], work=None) == z3.Z3_OK            # empty plan, work may be NULL


def test_step_scalars_match_the_oracle():
    """The scalars a graph-captured step reads equal the oracle's, bit for bit."""
    rnd = random.Random(17)
    cases = [dict(lr=3e-4, beta1=0.9, beta2=0.95, eps=1e-8, weight_decay=0.1, step=t) for t in (1, 2, 10, 1000)]
    cases += [dict(lr=rnd.uniform(1e-6, 1e-2), beta1=rnd.uniform(0, 0.999), beta2=rnd.uniform(0, 0.9999),
                   eps=10 ** rnd.uniform(-12, -4), weight_decay=rnd.uniform(0, 0.3), step=rnd.randint(1, 10 ** 6))
              for _ in range(200)]
    for c in cases:
        got = np.array(z3.zero3_step_scalars(z3.adamw(**c)), dtype=np.float32)
        ref = oracle.adamw_consts(oracle.hp(**c))
        assert np.array_equal(got.view(np.uint32), ref.view(np.uint32)), c
    with pytest.raises(z3.Zero3Error):
        z3.zero3_step_scalars(z3.adamw(step=0))
    with pytest.raises(z3.Zero3Error):
        z3.zero3_step_scalars(z3.adamw(beta2=1.0))
    for bad in (dict(eps=0.0), dict(eps=-1e-8), dict(lr=-3e-4), dict(weight_decay=-0.1)):
        with pytest.raises(z3.Zero3Error) as e:
            z3.zero3_step_scalars(z3.adamw(**bad))
        assert e.value.status == z3.Z3_EINVAL, bad
    # the edges that stay valid: no learning rate, no decay
    z3.zero3_step_scalars(z3.adamw(lr=0.0))
    z3.zero3_step_scalars(z3.adamw(weight_decay=0.0))


def test_reduce_adamw_dev_argument_errors():
    p = z3.zero3_plan([(1000,)], 4, 8)
    D = p.D
    arr = (C.c_void_p * D)(*[P16 * (100 + d) for d in range(D)])
    L = z3.lib()

    def call(scalars, work=P16 * 4, gathered=(), rank=-1):
        ga = (C.c_void_p * max(1, len(gathered)))(*gathered)
        return L.zero3_reduce_adamw_dev(p.handle, rank, arr, 0, C.c_void_p(P16), C.c_void_p(P16 * 2),
                                        C.c_void_p(P16 * 3), None if work is None else C.c_void_p(work),
                                        ga if gathered else None, len(gathered), 0,
                                        None if scalars is None else C.c_void_p(scalars), None)
    assert call(None) == z3.Z3_EINVAL
    assert call(P16 * 9000 + 4) == z3.Z3_EALIGN                # 16-byte alignment of the scalars
    assert call(P16 * 9000, work=None) == z3.Z3_EINVAL          # no shard and no gathered block
    assert call(P16 * 9000, gathered=[P16 * 5000] * 9) == z3.Z3_EINVAL
    assert call(P16 * 9000, rank=7) == z3.Z3_EINVAL
    assert call(P16 * 2 + 16) == z3.Z3_EINVAL                   # the scalars inside exp_avg
    e = z3.zero3_plan([], 4, 8)
    assert L.zero3_reduce_adamw_dev(e.handle, -1, arr, 0, C.c_void_p(P16), C.c_void_p(P16 * 2),
                                    C.c_void_p(P16 * 3), C.c_void_p(P16 * 4), None, 0, 0,
                                    C.c_void_p(P16 * 9000), None) == z3.Z3_OK


def test_reduce_adamw_empty_plan_is_a_no_op():
    p = z3.zero3_plan([], 4, 128)
    assert call_reduce(p) == z3.Z3_OK
    assert call_reduce(p, rank=2) == z3.Z3_OK


def call_gather(plan, shards=None, flat=P16 * 500, tensor_out=None):
    D = plan.D
    shards = shards if shards is not None else [P16 * (100 + 10 * r) for r in range(D)]
    sa = (C.c_void_p * max(1, D))(*shards)
    ta = None
    if tensor_out is not None:
        ta = (C.c_void_p * max(1, len(tensor_out)))(*tensor_out)
    return z3.lib().zero3_gather_block(plan.handle, sa, None if flat is None else C.c_void_p(flat), ta, None)


def test_gather_block_argument_errors():
    p = z3.zero3_plan([(64,), (64,)], 4, 8)
    E = z3.Z3_EINVAL
    assert call_gather(p, flat=None) == E
    assert call_gather(p, shards=[P16, 0, P16 * 3, P16 * 4]) == E
    assert call_gather(p, shards=[P16 + 1, P16 * 2, P16 * 3, P16 * 4]) == z3.Z3_EALIGN
    assert call_gather(p, flat=P16 * 500 + 1) == z3.Z3_EALIGN
    assert call_gather(p, flat=None, tensor_out=[P16 * 700 + 1, 0]) == z3.Z3_EALIGN
    S = p.S * 2                                                  # bytes per shard
    assert call_gather(p, flat=P16 * 100 - S) == E               # shard 0 where partition 1 lies
    assert call_gather(p, flat=P16 * 100 + 2) == E               # flat over shard 0, off its place
    # shard 0 sitting exactly in place (flat + 0*S) is accepted: see the GPU test
    assert call_gather(p, flat=None, tensor_out=[P16 * 700, P16 * 700 + 2]) == E   # tensors overlap
    assert call_gather(p, tensor_out=[P16 * 500, 0]) == E         # tensor over flat
    assert z3.lib().zero3_gather_block(None, None, None, None, None) == E


def test_gather_empty_plan_is_a_no_op():
    p = z3.zero3_plan([(0,)], 2, 8)
    assert call_gather(p) == z3.Z3_OK


def test_ipc_argument_errors():
    """The IPC entry points refuse NULL arguments, a negative offset and a base
    that is not one of their mappings, before any CUDA call."""
    L, E = z3.lib(), z3.Z3_EINVAL
    h = (C.c_char * z3.Z3_IPC_HANDLE_BYTES)()
    off, size = C.c_int64(), C.c_int64()
    ptr, base = C.c_void_p(), C.c_void_p()
    assert L.zero3_ipc_export(None, h, C.byref(off), C.byref(size)) == E
    assert L.zero3_ipc_export(P16, None, C.byref(off), C.byref(size)) == E
    assert L.zero3_ipc_export(P16, h, None, C.byref(size)) == E
    assert L.zero3_ipc_export(P16, h, C.byref(off), None) == E
    assert L.zero3_ipc_import(None, 0, C.byref(ptr), C.byref(base)) == E
    assert L.zero3_ipc_import(h, -1, C.byref(ptr), C.byref(base)) == E
    assert L.zero3_ipc_import(h, 0, None, C.byref(base)) == E
    assert L.zero3_ipc_import(h, 0, C.byref(ptr), None) == E
    assert L.zero3_ipc_close(None) == E
    assert L.zero3_ipc_close(P16 * 5) == E                       # never imported
    with pytest.raises(ValueError):                              # the binding checks the exporter's size
        z3.zero3_ipc_import(bytes(64), 4096, 4096, 1, torch.float32, 0)
