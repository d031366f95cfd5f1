"""Randomised GPU parity against the oracle over the whole argument space of the
fused kernel and the gather: D in 1..64, alignments 1..128, random tensor lists
(ragged tails, empty tensors), all ranks or one rank, both contribution layouts,
both reduce dtypes, misaligned buffers (scalar paths), 0..3 fused gathered blocks,
scalars as launch arguments or in device memory; the HYBRID_SHARD step over
random node counts (R * D up to 64); and its split form for separate machines
(each node's sum, then the fold).  Every case runs two steps and compares every
element; canary bands must stay intact."""
import random

import numpy as np
import pytest
import torch

import oracle
import synth
from parity_util import (Guarded, assert_bf16_parity, assert_f32_parity, checked_plan, f32_host, hp_for,
                         oracle_hp)

pytestmark = pytest.mark.gpu
SENTINEL = 0x7FAB


@pytest.fixture(scope="module")
def z3():
    assert torch.cuda.is_available(), "the GPU tests need a CUDA device"
    from fsdp_sharded_mixed_flat_b200 import build
    build.build()
    from fsdp_sharded_mixed_flat_b200 import zero3
    return zero3


def one_case(z3, rnd: random.Random, seed: int):
    D = rnd.choice([1, 2, 3, 4, 5, 7, 8, 9, 16, 17, 31, 32, 33, 64])
    A = rnd.choice([1, 2, 3, 8, 16, 128])
    shapes = [(rnd.randint(0, 3000),) if rnd.random() < 0.7 else (rnd.randint(1, 30), rnd.randint(1, 90))
              for _ in range(rnd.randint(1, 6))]
    plan, ref = checked_plan(z3, shapes, D, A)
    N, N_pad, S = ref.N, ref.N_pad, ref.S
    rank = -1 if rnd.random() < 0.5 else rnd.randrange(D)
    layout = z3.Z3_CONTRIB_OWNED if rank >= 0 and rnd.random() < 0.5 else z3.Z3_CONTRIB_FULL
    mode = rnd.choice([0, 1])
    ng = rnd.choice([0, 0, 1, 2, 3])
    use_dev = rnd.random() < 0.4
    with_work = ng == 0 or rnd.random() < 0.5
    skew = [rnd.choice([0, 0, 0, 1, 2]) for _ in range(6)]
    n = N_pad if rank < 0 else S
    desc = f"seed={seed} D={D} A={A} shapes={shapes} rank={rank} layout={layout} mode={mode} ng={ng} " \
           f"dev={use_dev} work={with_work} skew={skew}"
    p_full = synth.master_weights(N, N_pad, seed=seed, device="cuda")
    p0 = p_full if rank < 0 else p_full[rank * S:(rank + 1) * S]
    gp = Guarded(n, torch.float32, skew[0], fill=p0)
    gm = Guarded(n, torch.float32, skew[1], fill=torch.zeros(n, device="cuda"))
    gv = Guarded(n, torch.float32, skew[2], fill=torch.zeros(n, device="cuda"))
    gw = Guarded(n, torch.bfloat16, skew[3], fill=torch.zeros(n, device="cuda", dtype=torch.bfloat16)) \
        if with_work else None
    gg = []
    for k in range(ng):
        g = Guarded(N_pad, torch.bfloat16, skew[4] if k == 0 else 0)
        g.t.view(torch.int16).fill_(SENTINEL)
        gg.append(g)
    sc = torch.zeros(z3.Z3_SCALARS, dtype=torch.float32, device="cuda")
    hp_, hm, hv, hw = f32_host(p0).copy(), np.zeros(n, np.float32), np.zeros(n, np.float32), np.zeros(n, np.uint16)
    for t in (1, 2):
        contribs = synth.contributions(D, N, N_pad, seed=seed, step=t, sigma=1e-3,
                                       dist=rnd.choice(["normal", "student_t"]), zero_frac=0.02, device="cuda")
        if layout == z3.Z3_CONTRIB_OWNED:
            contribs = [c[rank * S:(rank + 1) * S].clone() for c in contribs]
        gc = [Guarded(c.numel(), torch.bfloat16, skew[5], fill=c) for c in contribs]
        hp = z3.adamw(**hp_for(t))
        work = None if gw is None else gw.t
        if use_dev:
            sc.copy_(torch.tensor(z3.zero3_step_scalars(hp), dtype=torch.float32))
            z3.zero3_reduce_adamw_dev(plan, rank, [g.t for g in gc], gp.t, gm.t, gv.t, work, [g.t for g in gg], sc,
                                      contrib_layout=layout, reduce_dtype=mode)
        elif ng:
            z3.zero3_reduce_adamw_gather(plan, rank, [g.t for g in gc], gp.t, gm.t, gv.t, work, [g.t for g in gg],
                                         hp, contrib_layout=layout, reduce_dtype=mode)
        else:
            z3.zero3_reduce_adamw(plan, rank, [g.t for g in gc], gp.t, gm.t, gv.t, work, hp,
                                  contrib_layout=layout, reduce_dtype=mode)
        oracle.reduce_adamw([synth.bf16_bits(c) for c in contribs], S, rank, hp_, hm, hv, hw, oracle_hp(t),
                            layout=layout, reduce_dtype=mode)
        torch.cuda.synchronize()
        assert_f32_parity(f32_host(gp.t), hp_, "master " + desc)
        assert_f32_parity(f32_host(gm.t), hm, "exp_avg " + desc)
        assert_f32_parity(f32_host(gv.t), hv, "exp_avg_sq " + desc)
        if gw is not None:
            assert_bf16_parity(synth.bf16_bits(gw.t), hw, "work " + desc)
        lo = 0 if rank < 0 else rank * S
        for g in gg:
            bits = synth.bf16_bits(g.t)
            assert_bf16_parity(bits[lo:lo + n], hw, "gathered " + desc)
            assert (np.concatenate([bits[:lo], bits[lo + n:]]) == SENTINEL).all(), "gathered outside " + desc
        for g in [gp, gm, gv, *([gw] if gw else []), *gg, *gc]:
            assert g.guards_intact(), "canary " + desc
    # the gather of the resulting shards, flat and per tensor, against the oracle
    if rank < 0 and gw is not None:
        shards = [gw.t[r * S:(r + 1) * S] for r in range(D)]
        flat = Guarded(N_pad, torch.bfloat16, skew[4])
        outs = [Guarded(k, torch.bfloat16, rnd.choice([0, 1, 3])) if k else None for k in ref.numels]
        z3.zero3_gather_block(plan, shards, flat.t, [None if o is None else o.t for o in outs])
        torch.cuda.synchronize()
        ref_flat = oracle.all_gather([hw[r * S:(r + 1) * S] for r in range(D)], S)
        assert np.array_equal(synth.bf16_bits(flat.t), ref_flat), "flat " + desc
        for o, r in zip(outs, oracle.unflatten(ref_flat, ref.offsets, ref.numels)):
            if o is not None:
                assert np.array_equal(synth.bf16_bits(o.t), r), "tensor " + desc
                assert o.guards_intact()
        assert flat.guards_intact()


@pytest.mark.parametrize("block", range(8))
def test_fuzz_against_oracle(z3, block):
    for k in range(25):
        seed = 1000 * block + k
        one_case(z3, random.Random(seed), seed)


def hybrid_case(z3, rnd: random.Random, seed: int):
    D = rnd.choice([1, 2, 3, 4, 5, 8, 16])
    R = rnd.randint(1, 64 // D)
    A = rnd.choice([1, 2, 8, 128])
    shapes = [(rnd.randint(0, 3000),) for _ in range(rnd.randint(1, 4))]
    plan, ref = checked_plan(z3, shapes, D, A)
    N, N_pad, S = ref.N, ref.N_pad, ref.S
    rank = -1 if rnd.random() < 0.5 else rnd.randrange(D)
    layout = z3.Z3_CONTRIB_OWNED if rank >= 0 and rnd.random() < 0.5 else z3.Z3_CONTRIB_FULL
    mode = rnd.choice([0, 1])
    skew = [rnd.choice([0, 0, 0, 1, 2]) for _ in range(5)]
    n = N_pad if rank < 0 else S
    desc = f"seed={seed} R={R} D={D} A={A} shapes={shapes} rank={rank} layout={layout} mode={mode} skew={skew}"
    p_full = synth.master_weights(N, N_pad, seed=seed, device="cuda")
    p0 = p_full if rank < 0 else p_full[rank * S:(rank + 1) * S]
    gp = Guarded(n, torch.float32, skew[0], fill=p0)
    gm = Guarded(n, torch.float32, skew[1], fill=torch.zeros(n, device="cuda"))
    gv = Guarded(n, torch.float32, skew[2], fill=torch.zeros(n, device="cuda"))
    gw = Guarded(n, torch.bfloat16, skew[3], fill=torch.zeros(n, device="cuda", dtype=torch.bfloat16))
    hp_, hm, hv, hw = f32_host(p0).copy(), np.zeros(n, np.float32), np.zeros(n, np.float32), np.zeros(n, np.uint16)
    for t in (1, 2):
        contribs = synth.contributions(R * D, N, N_pad, seed=seed, step=t, sigma=1e-3,
                                       dist=rnd.choice(["normal", "student_t"]), zero_frac=0.02, device="cuda")
        if layout == z3.Z3_CONTRIB_OWNED:
            contribs = [c[rank * S:(rank + 1) * S].clone() for c in contribs]
        gc = [Guarded(c.numel(), torch.bfloat16, skew[4], fill=c) for c in contribs]
        z3.zero3_reduce_adamw_hybrid(plan, rank, R, [g.t for g in gc], gp.t, gm.t, gv.t, gw.t,
                                     z3.adamw(**hp_for(t)), contrib_layout=layout, reduce_dtype=mode)
        oracle.reduce_adamw_hybrid([synth.bf16_bits(c) for c in contribs], R, S, rank, hp_, hm, hv, hw,
                                   oracle_hp(t), layout=layout, reduce_dtype=mode)
        torch.cuda.synchronize()
        assert_f32_parity(f32_host(gp.t), hp_, "master " + desc)
        assert_f32_parity(f32_host(gm.t), hm, "exp_avg " + desc)
        assert_f32_parity(f32_host(gv.t), hv, "exp_avg_sq " + desc)
        assert_bf16_parity(synth.bf16_bits(gw.t), hw, "work " + desc)
        for g in [gp, gm, gv, gw, *gc]:
            assert g.guards_intact(), "canary " + desc


@pytest.mark.parametrize("block", range(4))
def test_fuzz_hybrid_against_oracle(z3, block):
    for k in range(25):
        seed = 50_000 + 1000 * block + k
        hybrid_case(z3, random.Random(seed), seed)


def node_fold_case(z3, rnd: random.Random, seed: int):
    """HYBRID_SHARD across nodes: each node's sum (zero3_node_sum), then their
    fold (zero3_fold_adamw), against the oracle's two-level step."""
    D = rnd.choice([1, 2, 3, 4, 5, 8, 16, 32])
    R = rnd.randint(1, 8)
    A = rnd.choice([1, 2, 8, 128])
    shapes = [(rnd.randint(0, 3000),) for _ in range(rnd.randint(1, 4))]
    plan, ref = checked_plan(z3, shapes, D, A)
    N, N_pad, S = ref.N, ref.N_pad, ref.S
    rank = -1 if rnd.random() < 0.5 else rnd.randrange(D)
    layout = z3.Z3_CONTRIB_OWNED if rank >= 0 and rnd.random() < 0.5 else z3.Z3_CONTRIB_FULL
    mode = rnd.choice([0, 1])
    skew = [rnd.choice([0, 0, 0, 1]) for _ in range(4)]
    n = N_pad if rank < 0 else S
    desc = f"seed={seed} R={R} D={D} A={A} shapes={shapes} rank={rank} layout={layout} mode={mode} skew={skew}"
    dt = torch.float32 if mode == 0 else torch.bfloat16
    p_full = synth.master_weights(N, N_pad, seed=seed, device="cuda")
    p0 = p_full if rank < 0 else p_full[rank * S:(rank + 1) * S]
    gp = Guarded(n, torch.float32, skew[0], fill=p0)
    gm = Guarded(n, torch.float32, 0, fill=torch.zeros(n, device="cuda"))
    gv = Guarded(n, torch.float32, 0, fill=torch.zeros(n, device="cuda"))
    gw = Guarded(n, torch.bfloat16, skew[1], fill=torch.zeros(n, device="cuda", dtype=torch.bfloat16))
    sums = [Guarded(n, dt, skew[2]) for _ in range(R)]
    hp_, hm, hv, hw = f32_host(p0).copy(), np.zeros(n, np.float32), np.zeros(n, np.float32), np.zeros(n, np.uint16)
    for t in (1, 2):
        contribs = synth.contributions(R * D, N, N_pad, seed=seed, step=t, sigma=1e-3,
                                       dist=rnd.choice(["normal", "student_t"]), zero_frac=0.02, device="cuda")
        if layout == z3.Z3_CONTRIB_OWNED:
            contribs = [c[rank * S:(rank + 1) * S].clone() for c in contribs]
        gc = [Guarded(c.numel(), torch.bfloat16, skew[3], fill=c) for c in contribs]
        for k in range(R):
            z3.zero3_node_sum(plan, rank, [g.t for g in gc[k * D:(k + 1) * D]], sums[k].t, contrib_layout=layout,
                              reduce_dtype=mode)
        z3.zero3_fold_adamw(plan, rank, [g.t for g in sums], gp.t, gm.t, gv.t, gw.t, z3.adamw(**hp_for(t)),
                            reduce_dtype=mode)
        oracle.reduce_adamw_hybrid([synth.bf16_bits(c) for c in contribs], R, S, rank, hp_, hm, hv, hw,
                                   oracle_hp(t), layout=layout, reduce_dtype=mode)
        torch.cuda.synchronize()
        assert_f32_parity(f32_host(gp.t), hp_, "master " + desc)
        assert_f32_parity(f32_host(gm.t), hm, "exp_avg " + desc)
        assert_f32_parity(f32_host(gv.t), hv, "exp_avg_sq " + desc)
        assert_bf16_parity(synth.bf16_bits(gw.t), hw, "work " + desc)
        for g in [gp, gm, gv, gw, *sums, *gc]:
            assert g.guards_intact(), "canary " + desc


@pytest.mark.parametrize("block", range(2))
def test_fuzz_node_sums_then_fold_against_oracle(z3, block):
    for k in range(25):
        seed = 90_000 + 1000 * block + k
        node_fold_case(z3, random.Random(seed), seed)
