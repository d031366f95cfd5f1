"""GPU parity of the HYBRID_SHARD step (R nodes of D ranks: the nodes' rank
folds, then the node sums across nodes, then 1/(R*D), AdamW and the bf16
cast) against the oracle, through the C ABI, on the same seeded inputs.

Small cases span several 8-element chunks and ragged tails, the specialised
shape (4 nodes of 8) and the generic kernel (any R and D, up to 64
contributions), both reduce dtypes, both layouts, single ranks and all ranks
in one launch, and misaligned buffers (scalar path), with canary bands around
every buffer.  One node must give exactly the plain step.  The full-size case
is the pages' 4-node x 8-GPU LLaMA-7B block in the benchmark's launch
configuration, compared on sampled elements.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from parity_util import (assert_bf16_parity, assert_f32_parity, checked_plan, f32_host, Guarded, hp_for,
                         oracle_hp, state_init)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def z3():
    assert torch.cuda.is_available(), "the GPU tests need a CUDA device"
    from fsdp_sharded_mixed_flat_b200 import build
    build.build()
    from fsdp_sharded_mixed_flat_b200 import zero3
    return zero3


def run_small(z3, numels, R, D, A, rank, layout, mode, steps=6, seed=0, skew=0):
    plan, ref = checked_plan(z3, [(k,) for k in numels], D, A)
    N, N_pad, S = ref.N, ref.N_pad, ref.S
    n = N_pad if rank < 0 else S
    p_full, _, _ = state_init(N, N_pad, seed)
    p0 = p_full if rank < 0 else p_full[rank * S:(rank + 1) * S]
    gp = Guarded(n, torch.float32, skew, fill=p0)
    gm = Guarded(n, torch.float32, 0, fill=torch.zeros(n, device="cuda"))
    gv = Guarded(n, torch.float32, 0, fill=torch.zeros(n, device="cuda"))
    gw = Guarded(n, torch.bfloat16, 0, fill=torch.zeros(n, device="cuda", dtype=torch.bfloat16))
    hp_, hm, hv = f32_host(p0).copy(), np.zeros(n, np.float32), np.zeros(n, np.float32)
    hw = np.zeros(n, np.uint16)
    for t in range(1, steps + 1):
        contribs = synth.contributions(R * D, N, N_pad, seed=seed, step=t, sigma=1e-3, device="cuda")
        if layout == z3.Z3_CONTRIB_OWNED:
            contribs = [c[rank * S:(rank + 1) * S].clone() for c in contribs]
        gc = [Guarded(c.numel(), torch.bfloat16, 0, fill=c) for c in contribs]
        z3.zero3_reduce_adamw_hybrid(plan, rank, R, [g.t for g in gc], gp.t, gm.t, gv.t, gw.t,
                                     z3.adamw(**hp_for(t)), contrib_layout=layout, reduce_dtype=mode)
        oracle.reduce_adamw_hybrid([synth.bf16_bits(c) for c in contribs], R, S, rank, hp_, hm, hv, hw,
                                   oracle_hp(t), layout=layout, reduce_dtype=mode)
        torch.cuda.synchronize()
        what = f"numels={numels} R={R} D={D} A={A} rank={rank} layout={layout} mode={mode} step={t}"
        assert_f32_parity(f32_host(gp.t), hp_, "master " + what)
        assert_f32_parity(f32_host(gm.t), hm, "exp_avg " + what)
        assert_f32_parity(f32_host(gv.t), hv, "exp_avg_sq " + what)
        assert_bf16_parity(synth.bf16_bits(gw.t), hw, "work_bf16 " + what)
        for g in (gp, gm, gv, gw, *gc):
            assert g.guards_intact(), "canary overwritten: " + what
        for g, c in zip(gc, contribs):
            assert torch.equal(g.t.view(torch.int16), c.view(torch.int16)), "contribution modified"
    return plan


SMALL = [
    ([123457], 4, 8, 128),        # the specialised kernels: 2, 4 and 8 nodes of 8
    ([60001, 7], 2, 8, 128),
    ([30011], 8, 8, 8),
    ([5000, 77], 4, 8, 1),        # ... with a ragged tail
    ([3000, 17], 2, 3, 8),        # generic kernel
    ([20001], 3, 5, 1),
    ([4097, 33], 2, 16, 128),
    ([9000], 16, 4, 8),           # 64 contributions, the maximum
    ([9000], 8, 1, 8),            # one rank per node
    ([777], 5, 2, 1),
]


@pytest.mark.parametrize("mode", [0, 1], ids=["fp32", "bf16"])
@pytest.mark.parametrize("numels,R,D,A", SMALL)
def test_hybrid_all_ranks_one_launch(z3, numels, R, D, A, mode):
    run_small(z3, numels, R, D, A, -1, z3.Z3_CONTRIB_FULL, mode)


@pytest.mark.parametrize("mode", [0, 1], ids=["fp32", "bf16"])
@pytest.mark.parametrize("numels,R,D,A", SMALL)
def test_hybrid_single_rank_full_and_owned(z3, numels, R, D, A, mode):
    run_small(z3, numels, R, D, A, D // 2, z3.Z3_CONTRIB_FULL, mode, steps=3)
    run_small(z3, numels, R, D, A, D - 1, z3.Z3_CONTRIB_OWNED, mode, steps=3)


@pytest.mark.parametrize("skew", [1, 2])
def test_hybrid_misaligned_master_takes_the_scalar_path(z3, skew):
    for mode in (0, 1):
        run_small(z3, [3000, 17], 4, 8, 8, -1, z3.Z3_CONTRIB_FULL, mode, steps=3, skew=skew)
        run_small(z3, [3000, 17], 3, 2, 8, 1, z3.Z3_CONTRIB_OWNED, mode, steps=2, skew=skew)


@pytest.mark.parametrize("mode", [0, 1], ids=["fp32", "bf16"])
def test_one_node_is_exactly_the_plain_step(z3, mode):
    """n_nodes = 1 through the HYBRID_SHARD entry point gives the plain step's bits."""
    plan = z3.zero3_plan([(50000,), (333,)], 8, 128)
    out = []
    for hybrid in (False, True):
        p, m, v = state_init(plan.N, plan.N_pad, 4)
        w = torch.zeros(plan.N_pad, dtype=torch.bfloat16, device="cuda")
        for t in (1, 2, 3):
            c = synth.contributions(8, plan.N, plan.N_pad, seed=4, step=t, sigma=1e-3, device="cuda")
            if hybrid:
                z3.zero3_reduce_adamw_hybrid(plan, -1, 1, c, p, m, v, w, z3.adamw(**hp_for(t)), reduce_dtype=mode)
            else:
                z3.zero3_reduce_adamw(plan, -1, c, p, m, v, w, z3.adamw(**hp_for(t)), reduce_dtype=mode)
        out.append((p, m, v, w))
    torch.cuda.synchronize()
    for a, b in zip(*out):
        assert torch.equal(a.view(torch.int16), b.view(torch.int16))


@pytest.mark.parametrize("mode,steps", [(0, 10), (1, 3)], ids=["fp32", "bf16"])
def test_llama7b_block_4_nodes_of_8_bench_configuration(z3, mode, steps):
    """The benchmark's launch: 4 nodes of 8 ranks, all 8 local ranks in one
    launch, full layout; sampled elements against the oracle."""
    w = synth.WORKLOADS["llama7b_hybrid"]
    R, D = w["nodes"], w["D"]
    plan, ref = checked_plan(z3, [s for _, s in w["tensors"]], D, synth.ALIGN)
    N, N_pad, S = ref.N, ref.N_pad, ref.S
    p, m, v = state_init(N, N_pad, 0)
    wk = torch.zeros(N_pad, dtype=torch.bfloat16, device="cuda")
    rng = np.random.default_rng(1)
    picks = [rng.choice(N_pad, size=200_000, replace=False), np.arange(64), np.arange(N_pad - 64, N_pad)]
    picks += [np.arange(r * S - 16, r * S + 16) for r in range(1, D)]
    idx = torch.from_numpy(np.unique(np.concatenate(picks))).cuda()
    hp_, hm, hv = f32_host(p[idx]).copy(), np.zeros(idx.numel(), np.float32), np.zeros(idx.numel(), np.float32)
    hw = np.zeros(idx.numel(), np.uint16)
    for t in range(1, steps + 1):
        c = synth.contributions(R * D, N, N_pad, seed=0, step=t, sigma=w["sigma"], device="cuda")
        z3.zero3_reduce_adamw_hybrid(plan, -1, R, c, p, m, v, wk, z3.adamw(**hp_for(t)), reduce_dtype=mode)
        sub = [synth.bf16_bits(x[idx]) for x in c]
        oracle.reduce_adamw_hybrid(sub, R, idx.numel(), 0, hp_, hm, hv, hw, oracle_hp(t),
                                   layout=oracle.LAYOUT_OWNED, reduce_dtype=mode)
        del c
    torch.cuda.synchronize()
    what = f"llama7b_hybrid mode={mode}"
    assert_f32_parity(f32_host(p[idx]), hp_, "master " + what)
    assert_f32_parity(f32_host(m[idx]), hm, "exp_avg " + what)
    assert_f32_parity(f32_host(v[idx]), hv, "exp_avg_sq " + what)
    assert_bf16_parity(synth.bf16_bits(wk[idx]), hw, "work_bf16 " + what)
