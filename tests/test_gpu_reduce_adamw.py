"""GPU parity of the fused reduce-scatter + AdamW + bf16-cast kernel against the
oracle, called through the C ABI, on the same seeded inputs.

Small cases (seconds for the oracle) span several 8-element chunks, thread
blocks and ragged tails, every rank count class (1, powers of two, odd, the
maximum 64), both contribution layouts, both reduce dtypes, single ranks and
all ranks in one launch, and misaligned buffers (scalar path); every buffer
sits between canary bands that must come back untouched.  Full-size cases run
the workloads in the launch configuration the benchmark times and compare
sampled elements (every element is independent of the others, so the oracle
run on the gathered sample equals the full run at those indices).
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from parity_util import (Guarded, assert_bf16_parity, assert_f32_parity, checked_plan, f32_host, hp_for,
                         oracle_hp, state_init)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def z3():
    assert torch.cuda.is_available(), "the GPU tests need a CUDA device"
    from fsdp_sharded_mixed_flat_b200 import build
    build.build()
    from fsdp_sharded_mixed_flat_b200 import zero3
    return zero3


def run_small(z3, numels, D, A, rank, layout, mode, steps=10, seed=0, skew=(0, 0, 0, 0, 0),
              dist="normal", sigma=1e-3, zero_frac=0.0):
    plan, ref = checked_plan(z3, [(k,) for k in numels], D, A)
    N, N_pad, S = ref.N, ref.N_pad, ref.S
    n = N_pad if rank < 0 else S
    p_full, _, _ = state_init(N, N_pad, seed)
    p0 = p_full if rank < 0 else p_full[rank * S:(rank + 1) * S]
    gp = Guarded(n, torch.float32, skew[0], fill=p0)
    gm = Guarded(n, torch.float32, skew[1], fill=torch.zeros(n, device="cuda"))
    gv = Guarded(n, torch.float32, skew[2], fill=torch.zeros(n, device="cuda"))
    gw = Guarded(n, torch.bfloat16, skew[3], fill=torch.zeros(n, device="cuda", dtype=torch.bfloat16))
    hp_, hm, hv = f32_host(p0).copy(), np.zeros(n, np.float32), np.zeros(n, np.float32)
    hw = np.zeros(n, np.uint16)
    for t in range(1, steps + 1):
        contribs = synth.contributions(D, N, N_pad, seed=seed, step=t, sigma=sigma, dist=dist,
                                       zero_frac=zero_frac, device="cuda")
        if layout == z3.Z3_CONTRIB_OWNED:
            contribs = [c[rank * S:(rank + 1) * S].clone() for c in contribs]
        gc = [Guarded(c.numel(), torch.bfloat16, skew[4], fill=c) for c in contribs]
        z3.zero3_reduce_adamw(plan, rank, [g.t for g in gc], gp.t, gm.t, gv.t, gw.t, z3.adamw(**hp_for(t)),
                              contrib_layout=layout, reduce_dtype=mode)
        oracle.reduce_adamw([synth.bf16_bits(c) for c in contribs], S, rank, hp_, hm, hv, hw, oracle_hp(t),
                            layout=layout, reduce_dtype=mode)
        torch.cuda.synchronize()
        what = f"numels={numels} D={D} A={A} rank={rank} layout={layout} mode={mode} step={t}"
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
    ([13], 1, 1), ([1], 8, 1), ([5, 7, 1], 4, 1), ([13], 3, 1), ([999], 5, 1),
    ([300, 77, 1000], 4, 8), ([1000, 2000], 3, 8), ([4097, 33], 32, 128), ([123457], 8, 128),
    ([2 ** 16 + 3], 64, 8), ([50000], 16, 1), ([70001], 2, 128), ([6000, 1, 2], 7, 16),
]


@pytest.mark.parametrize("mode", [0, 1], ids=["fp32", "bf16"])
@pytest.mark.parametrize("numels,D,A", SMALL)
def test_all_ranks_one_launch(z3, numels, D, A, mode):
    run_small(z3, numels, D, A, -1, z3.Z3_CONTRIB_FULL, mode)


@pytest.mark.parametrize("mode", [0, 1], ids=["fp32", "bf16"])
@pytest.mark.parametrize("numels,D,A", SMALL)
def test_single_rank_full_and_owned(z3, numels, D, A, mode):
    run_small(z3, numels, D, A, D // 2, z3.Z3_CONTRIB_FULL, mode, steps=4)
    run_small(z3, numels, D, A, D - 1, z3.Z3_CONTRIB_OWNED, mode, steps=4)


@pytest.mark.parametrize("skew", [(1, 0, 0, 0, 0), (0, 0, 0, 1, 0), (0, 0, 0, 0, 1), (1, 1, 1, 1, 1),
                                  (2, 0, 2, 0, 0)])
def test_misaligned_buffers_take_the_scalar_path(z3, skew):
    run_small(z3, [3000, 17], 4, 8, -1, z3.Z3_CONTRIB_FULL, 0, steps=3, skew=skew)
    run_small(z3, [3000, 17], 4, 8, 1, z3.Z3_CONTRIB_OWNED, 1, steps=2, skew=skew)


def test_heavy_tails_and_exact_zeros(z3):
    for mode in (0, 1):
        run_small(z3, [40000, 123], 8, 128, -1, z3.Z3_CONTRIB_FULL, mode, steps=5, dist="student_t",
                  zero_frac=0.01)


def test_subnormal_contributions(z3):
    """Gradients in the bf16 / fp32 subnormal range: the packed bf16 add and the
    fp32 path keep subnormals exactly as the oracle does (no flush to zero)."""
    for mode in (0, 1):
        run_small(z3, [20000, 77], 8, 8, -1, z3.Z3_CONTRIB_FULL, mode, steps=3, dist="subnormal")
        run_small(z3, [20000, 77], 16, 8, 3, z3.Z3_CONTRIB_OWNED, mode, steps=2, dist="subnormal")


def test_integer_contributions_give_the_same_step_in_both_reduce_dtypes(z3):
    """Exact partial sums: the bf16 and fp32 reductions must coincide."""
    out = []
    for mode in (0, 1):
        plan = z3.zero3_plan([(4096,)], 8, 8)
        p, m, v = state_init(plan.N, plan.N_pad, 1)
        w = torch.zeros(plan.N_pad, dtype=torch.bfloat16, device="cuda")
        c = synth.contributions(8, plan.N, plan.N_pad, seed=2, step=1, sigma=0, dist="integers", device="cuda")
        z3.zero3_reduce_adamw(plan, -1, c, p, m, v, w, z3.adamw(step=1), reduce_dtype=mode)
        out.append((p, m, v, w))
    for a, b in zip(*out):
        assert torch.equal(a.view(torch.int16 if a.dtype == torch.bfloat16 else torch.int32),
                           b.view(torch.int16 if b.dtype == torch.bfloat16 else torch.int32))


def test_pad_stays_exactly_zero(z3):
    plan = run_small(z3, [1000 * 32 + 1], 32, 128, -1, z3.Z3_CONTRIB_FULL, 0, steps=3)
    assert plan.N_pad - plan.N == 767   # 32001 elements padded to 8 * 4096


def test_empty_plan_and_stream_argument(z3):
    plan = z3.zero3_plan([], 4, 128)
    z = torch.zeros(16, device="cuda")
    zb = torch.zeros(16, device="cuda", dtype=torch.bfloat16)
    z3.zero3_reduce_adamw(plan, -1, [zb] * 4, z, z.clone(), z.clone(), zb.clone(), z3.adamw(step=1))
    s = torch.cuda.Stream()
    run_on = z3.zero3_plan([(4096,)], 2, 8)
    p, m, v = state_init(run_on.N, run_on.N_pad, 3)
    w = torch.zeros(run_on.N_pad, dtype=torch.bfloat16, device="cuda")
    c = synth.contributions(2, run_on.N, run_on.N_pad, seed=3, step=1, sigma=1e-3, device="cuda")
    torch.cuda.synchronize()
    ref = [p.clone(), m.clone(), v.clone(), w.clone()]
    with torch.cuda.stream(s):
        z3.zero3_reduce_adamw(run_on, -1, c, p, m, v, w, z3.adamw(step=1))
    z3.zero3_reduce_adamw(run_on, -1, c, *ref, z3.adamw(step=1), stream=torch.cuda.current_stream())
    torch.cuda.synchronize()
    assert torch.equal(p, ref[0]) and torch.equal(w.view(torch.int16), ref[3].view(torch.int16))


# ------------------------------------------- fused all-gather (ZeRO-1/2 step)
SENTINEL = 0x7FAB  # a bf16 NaN pattern the kernel never produces


def run_fused(z3, numels, D, A, rank, layout, mode, n_gathered, with_work, steps=3, skew=0, seed=5):
    plan, ref = checked_plan(z3, [(k,) for k in numels], D, A)
    N, N_pad, S = ref.N, ref.N_pad, ref.S
    n = N_pad if rank < 0 else S
    p_full, _, _ = state_init(N, N_pad, seed)
    p0 = p_full if rank < 0 else p_full[rank * S:(rank + 1) * S]
    gp = Guarded(n, torch.float32, skew, fill=p0)
    gm = Guarded(n, torch.float32, 0, fill=torch.zeros(n, device="cuda"))
    gv = Guarded(n, torch.float32, 0, fill=torch.zeros(n, device="cuda"))
    gw = Guarded(n, torch.bfloat16, skew, fill=torch.zeros(n, device="cuda", dtype=torch.bfloat16)) \
        if with_work else None
    gg = []
    for k in range(n_gathered):
        g = Guarded(N_pad, torch.bfloat16, skew if k == 0 else 0)
        g.t.view(torch.int16).fill_(SENTINEL)
        gg.append(g)
    hp_, hm, hv = f32_host(p0).copy(), np.zeros(n, np.float32), np.zeros(n, np.float32)
    hw = np.zeros(n, np.uint16)
    lo = 0 if rank < 0 else rank * S
    for t in range(1, steps + 1):
        contribs = synth.contributions(D, N, N_pad, seed=seed, step=t, sigma=1e-3, device="cuda")
        if layout == z3.Z3_CONTRIB_OWNED:
            contribs = [c[rank * S:(rank + 1) * S].clone() for c in contribs]
        z3.zero3_reduce_adamw_gather(plan, rank, contribs, gp.t, gm.t, gv.t, None if gw is None else gw.t,
                                     [g.t for g in gg], z3.adamw(**hp_for(t)), contrib_layout=layout,
                                     reduce_dtype=mode)
        oracle.reduce_adamw([synth.bf16_bits(c) for c in contribs], S, rank, hp_, hm, hv, hw, oracle_hp(t),
                            layout=layout, reduce_dtype=mode)
        torch.cuda.synchronize()
        what = f"fused numels={numels} D={D} rank={rank} layout={layout} mode={mode} ng={n_gathered} step={t}"
        assert_f32_parity(f32_host(gp.t), hp_, "master " + what)
        assert_f32_parity(f32_host(gm.t), hm, "exp_avg " + what)
        assert_f32_parity(f32_host(gv.t), hv, "exp_avg_sq " + what)
        if gw is not None:
            assert_bf16_parity(synth.bf16_bits(gw.t), hw, "work_bf16 " + what)
            assert gw.guards_intact()
        for k, g in enumerate(gg):
            bits = synth.bf16_bits(g.t)
            assert_bf16_parity(bits[lo:lo + n], hw, f"gathered[{k}] " + what)
            rest = np.concatenate([bits[:lo], bits[lo + n:]])
            assert (rest == SENTINEL).all(), "a gathered position outside the updated partitions was written"
            assert g.guards_intact(), f"canary of gathered[{k}] " + what
        for g in (gp, gm, gv):
            assert g.guards_intact()


@pytest.mark.parametrize("mode", [0, 1], ids=["fp32", "bf16"])
@pytest.mark.parametrize("numels,D,A", [([300, 77, 1000], 4, 8), ([123457], 8, 128), ([13], 3, 1),
                                        ([4097, 33], 32, 128)])
def test_fused_gather_matches_oracle(z3, numels, D, A, mode):
    run_fused(z3, numels, D, A, -1, z3.Z3_CONTRIB_FULL, mode, 1, with_work=False)
    run_fused(z3, numels, D, A, -1, z3.Z3_CONTRIB_FULL, mode, 3, with_work=True)
    run_fused(z3, numels, D, A, D - 1, z3.Z3_CONTRIB_FULL, mode, 2, with_work=True)
    run_fused(z3, numels, D, A, D // 2, z3.Z3_CONTRIB_OWNED, mode, 8, with_work=False)


def test_fused_gather_misaligned_scalar_path(z3):
    run_fused(z3, [3000, 17], 4, 8, -1, z3.Z3_CONTRIB_FULL, 0, 2, with_work=True, skew=1)
    run_fused(z3, [3000, 17], 4, 8, 2, z3.Z3_CONTRIB_OWNED, 1, 1, with_work=False, skew=1)


# ------------------------------------------------ offloaded optimiser state
@pytest.mark.parametrize("mode", [0, 1], ids=["fp32", "bf16"])
@pytest.mark.parametrize("numels,D,A,rank", [([300, 77, 1000], 4, 8, -1), ([123457], 8, 128, -1),
                                             ([4097, 33], 32, 128, 7), ([999], 5, 1, 2)])
def test_offloaded_state_matches_oracle(z3, numels, D, A, rank, mode):
    """fp32 master / m / v in page-locked host memory, read and written by the kernel
    over PCIe (the CPU-offload placement): same results as in HBM."""
    plan, ref = checked_plan(z3, [(k,) for k in numels], D, A)
    N, N_pad, S = ref.N, ref.N_pad, ref.S
    n = N_pad if rank < 0 else S
    p_full, _, _ = state_init(N, N_pad, 8)
    p0 = (p_full if rank < 0 else p_full[rank * S:(rank + 1) * S]).cpu()
    p, m, v = p0.clone().pin_memory(), torch.zeros(n).pin_memory(), torch.zeros(n).pin_memory()
    w = torch.zeros(n, dtype=torch.bfloat16).pin_memory()
    g = torch.zeros(N_pad, dtype=torch.bfloat16, device="cuda")
    hp_, hm, hv, hw = p0.numpy().copy(), np.zeros(n, np.float32), np.zeros(n, np.float32), np.zeros(n, np.uint16)
    for t in range(1, 4):
        c = synth.contributions(D, N, N_pad, seed=8, step=t, sigma=1e-3, device="cuda")
        if t == 3:
            z3.zero3_reduce_adamw_gather(plan, rank, c, p, m, v, w, [g], z3.adamw(**hp_for(t)), reduce_dtype=mode)
        else:
            z3.zero3_reduce_adamw(plan, rank, c, p, m, v, w, z3.adamw(**hp_for(t)), reduce_dtype=mode)
        oracle.reduce_adamw([synth.bf16_bits(x) for x in c], S, rank, hp_, hm, hv, hw, oracle_hp(t),
                            reduce_dtype=mode)
    torch.cuda.synchronize()
    assert_f32_parity(p.numpy(), hp_, "master")
    assert_f32_parity(m.numpy(), hm, "exp_avg")
    assert_f32_parity(v.numpy(), hv, "exp_avg_sq")
    assert_bf16_parity(synth.bf16_bits(w), hw, "work_bf16")
    lo = 0 if rank < 0 else rank * S
    assert_bf16_parity(synth.bf16_bits(g)[lo:lo + n], hw, "gathered")


@pytest.mark.parametrize("mode", [0, 1], ids=["fp32", "bf16"])
@pytest.mark.parametrize("numels,D,A,n_stage", [([300, 77, 1000], 4, 8, 3), ([123457], 8, 128, 2),
                                                ([4097, 33], 32, 128, 3), ([999], 5, 1, 1)])
def test_staged_offload_matches_oracle(z3, numels, D, A, n_stage, mode):
    """The optimiser state in pinned host memory, streamed partition by partition
    through device staging buffers: same results as the whole-block kernel."""
    from fsdp_sharded_mixed_flat_b200.offload import OffloadedState
    plan, ref = checked_plan(z3, [(k,) for k in numels], D, A)
    N, N_pad, S = ref.N, ref.N_pad, ref.S
    p_full, _, _ = state_init(N, N_pad, 9)
    p = p_full.cpu().pin_memory()
    m, v = torch.zeros(N_pad).pin_memory(), torch.zeros(N_pad).pin_memory()
    w = torch.zeros(N_pad, dtype=torch.bfloat16, device="cuda")
    off = OffloadedState(plan, p, m, v, w, "cuda", n_stage=n_stage, reduce_dtype=mode)
    hp_, hm, hv, hw = p_full.cpu().numpy().copy(), np.zeros(N_pad, np.float32), np.zeros(N_pad, np.float32), \
        np.zeros(N_pad, np.uint16)
    for t in range(1, 5):
        c = synth.contributions(D, N, N_pad, seed=9, step=t, sigma=1e-3, device="cuda")
        off.step(c, z3.adamw(**hp_for(t)))
        oracle.reduce_adamw([synth.bf16_bits(x) for x in c], S, -1, hp_, hm, hv, hw, oracle_hp(t),
                            reduce_dtype=mode)
    torch.cuda.synchronize()
    assert_f32_parity(p.numpy(), hp_, "master")
    assert_f32_parity(m.numpy(), hm, "exp_avg")
    assert_f32_parity(v.numpy(), hv, "exp_avg_sq")
    assert_bf16_parity(synth.bf16_bits(w), hw, "work_bf16")


def test_unpinned_host_state_is_refused(z3):
    plan = z3.zero3_plan([(64,)], 2, 8)
    c = [torch.zeros(plan.N_pad, dtype=torch.bfloat16, device="cuda")] * 2
    host = torch.zeros(plan.N_pad)                   # pageable: the device cannot reach it
    with pytest.raises(ValueError):
        z3.zero3_reduce_adamw(plan, -1, c, host, host.clone(), host.clone(),
                              torch.zeros(plan.N_pad, dtype=torch.bfloat16, device="cuda"), z3.adamw(step=1))


# ------------------------------------------------------------- full sizes
def sample_indices(n: int, S: int, D: int, k: int, seed: int) -> torch.Tensor:
    rng = np.random.default_rng(seed)
    picks = [rng.choice(n, size=min(k, n), replace=False), np.arange(min(64, n)), np.arange(max(0, n - 64), n)]
    for r in range(1, D):
        picks.append(np.arange(max(0, r * S - 16), min(n, r * S + 16)))
    return torch.from_numpy(np.unique(np.concatenate(picks))).cuda()


def run_sampled(z3, workload: str, D: int, rank: int, layout: int, mode: int, steps: int,
                k: int = 200_000, seed: int = 0):
    w = synth.WORKLOADS[workload]
    plan, ref = checked_plan(z3, [s for _, s in w["tensors"]], D, synth.ALIGN)
    N, N_pad, S = ref.N, ref.N_pad, ref.S
    n = N_pad if rank < 0 else S
    p_full, _, _ = state_init(N, N_pad, seed)
    p = (p_full if rank < 0 else p_full[rank * S:(rank + 1) * S]).contiguous()
    del p_full
    m, v = torch.zeros_like(p), torch.zeros_like(p)
    wk = torch.zeros(n, dtype=torch.bfloat16, device="cuda")
    idx = sample_indices(n, S if rank < 0 else n, D if rank < 0 else 1, k, seed + 1)
    hp_, hm, hv = f32_host(p[idx]).copy(), np.zeros(idx.numel(), np.float32), np.zeros(idx.numel(), np.float32)
    hw = np.zeros(idx.numel(), np.uint16)
    for t in range(1, steps + 1):
        if layout == z3.Z3_CONTRIB_OWNED:
            c = [synth.contribution(min(S, max(0, N - rank * S)), S, seed=seed, step=t, rank=d,
                                    sigma=w["sigma"], dist=w["dist"], zero_frac=w.get("zero_frac", 0.0),
                                    device="cuda") for d in range(D)]
        else:
            c = synth.contributions(D, N, N_pad, seed=seed, step=t, sigma=w["sigma"], dist=w["dist"],
                                    zero_frac=w.get("zero_frac", 0.0), device="cuda")
        z3.zero3_reduce_adamw(plan, rank, c, p, m, v, wk, z3.adamw(**hp_for(t)), contrib_layout=layout,
                              reduce_dtype=mode)
        base = 0 if (rank < 0 or layout == z3.Z3_CONTRIB_OWNED) else rank * S
        sub = [synth.bf16_bits(x[idx + base]) for x in c]
        oracle.reduce_adamw(sub, idx.numel(), 0, hp_, hm, hv, hw, oracle_hp(t), layout=oracle.LAYOUT_OWNED,
                            reduce_dtype=mode)
        del c
    torch.cuda.synchronize()
    what = f"{workload} D={D} rank={rank} mode={mode}"
    assert_f32_parity(f32_host(p[idx]), hp_, "master " + what)
    assert_f32_parity(f32_host(m[idx]), hm, "exp_avg " + what)
    assert_f32_parity(f32_host(v[idx]), hv, "exp_avg_sq " + what)
    assert_bf16_parity(synth.bf16_bits(wk[idx]), hw, "work_bf16 " + what)
    return plan, p, m, v, wk


def test_llama7b_block_d8_bench_configuration(z3):
    """The benchmark's launch: all 8 ranks in one launch, full layout, fp32 reduce, 10 steps."""
    run_sampled(z3, "llama7b_d8", 8, -1, z3.Z3_CONTRIB_FULL, 0, steps=10)


def test_llama7b_block_d32_padded(z3):
    plan, p, m, v, wk = run_sampled(z3, "llama7b_d32", 32, -1, z3.Z3_CONTRIB_FULL, 0, steps=10)
    assert plan.N_pad - plan.N == 4095
    for t in (p, m, v):
        assert not t[plan.N:].any()
    assert not wk[plan.N:].view(torch.int16).any()


@pytest.mark.parametrize("mode", [0, 1], ids=["fp32", "bf16"])
def test_llama7b_d32_sharded_equals_unsharded_full_size(z3, mode):
    """The padded 7B block at D = 32 (N = 202,387,457, N_pad = 202,391,552, the
    4095 pad elements in rank 31's shard), 3 steps run two ways on the same
    contributions: 32 separate rank-r launches (full layout), each into its own
    S-element master / m / v / bf16 buffers, and one all-ranks launch on a copy of
    the same state.  Sharding leaves the arithmetic of DDP unchanged ("Building
    GPT from Scratch — Part 8", "Key Takeaways"; "7.10 — Fully-sharded data
    parallel", §3), so the 32 shards concatenated must equal the unsharded result
    bit for bit, and both must equal the oracle on sampled elements that include
    every shard boundary and the whole pad; the pad must stay exactly zero."""
    w = synth.WORKLOADS["llama7b_d32"]
    D = 32
    plan, ref = checked_plan(z3, [s for _, s in w["tensors"]], D, synth.ALIGN)
    N, N_pad, S = ref.N, ref.N_pad, ref.S
    assert (N, N_pad, S) == (202_387_457, 202_391_552, 6_324_736)
    p_full, _, _ = state_init(N, N_pad, 3)
    big = [p_full.clone(), torch.zeros_like(p_full), torch.zeros_like(p_full),
           torch.zeros(N_pad, dtype=torch.bfloat16, device="cuda")]
    shard = [[p_full[r * S:(r + 1) * S].clone() for r in range(D)],
             [torch.zeros(S, device="cuda") for _ in range(D)],
             [torch.zeros(S, device="cuda") for _ in range(D)],
             [torch.zeros(S, dtype=torch.bfloat16, device="cuda") for _ in range(D)]]
    idx = torch.from_numpy(np.unique(np.concatenate([sample_indices(N_pad, S, D, 100_000, 4).cpu().numpy(),
                                                     np.arange(N, N_pad)]))).cuda()
    hp_, hm, hv = f32_host(p_full[idx]).copy(), np.zeros(idx.numel(), np.float32), np.zeros(idx.numel(), np.float32)
    hw = np.zeros(idx.numel(), np.uint16)
    del p_full
    for t in range(1, 4):
        c = synth.contributions(D, N, N_pad, seed=3, step=t, sigma=w["sigma"], device="cuda")
        hp = z3.adamw(**hp_for(t))
        for r in range(D):
            z3.zero3_reduce_adamw(plan, r, c, shard[0][r], shard[1][r], shard[2][r], shard[3][r], hp,
                                  contrib_layout=z3.Z3_CONTRIB_FULL, reduce_dtype=mode)
        z3.zero3_reduce_adamw(plan, -1, c, *big, hp, reduce_dtype=mode)
        oracle.reduce_adamw([synth.bf16_bits(x[idx]) for x in c], idx.numel(), 0, hp_, hm, hv, hw, oracle_hp(t),
                            layout=oracle.LAYOUT_OWNED, reduce_dtype=mode)
        del c
    torch.cuda.synchronize()
    for name, whole, parts in zip(("master", "exp_avg", "exp_avg_sq", "work_bf16"), big, shard):
        bits = torch.int16 if whole.dtype == torch.bfloat16 else torch.int32
        cat = torch.cat(parts)
        differ = int((cat.view(bits) != whole.view(bits)).sum().item())
        assert differ == 0, f"{name}: {differ} elements of the 32 shards differ from the unsharded step"
        assert not whole[N:].view(bits).any(), f"{name}: the pad is no longer zero"
    what = f"7B block D=32 mode={mode}"
    assert_f32_parity(f32_host(big[0][idx]), hp_, "master " + what)
    assert_f32_parity(f32_host(big[1][idx]), hm, "exp_avg " + what)
    assert_f32_parity(f32_host(big[2][idx]), hv, "exp_avg_sq " + what)
    assert_bf16_parity(synth.bf16_bits(big[3][idx]), hw, "work_bf16 " + what)


@pytest.mark.parametrize("D", [2, 4, 8, 16])
def test_llama7b_policy_sweep_bf16_reduce(z3, D):
    run_sampled(z3, "llama7b_policy", D, -1, z3.Z3_CONTRIB_FULL, 1, steps=3, k=100_000)


@pytest.mark.parametrize("D", [2, 4, 8, 16])
def test_policy_sweep_hundred_steps_every_element(z3, D):
    """The policy sweep's 100 steps (Student-t nu=3 gradients, 1% exact zeros, fresh
    every step) on a 2^20-element slice of the 7B block, both reduce dtypes, every
    element compared after the last step."""
    w = synth.WORKLOADS["llama7b_policy"]
    n_real = 1 << 20
    plan, ref = checked_plan(z3, [(n_real,)], D, synth.ALIGN)
    N, N_pad, S = ref.N, ref.N_pad, ref.S
    for mode in (0, 1):
        p, m, v = state_init(N, N_pad, 31)
        wk = torch.zeros(N_pad, dtype=torch.bfloat16, device="cuda")
        hp_, hm, hv, hw = f32_host(p).copy(), np.zeros(N_pad, np.float32), np.zeros(N_pad, np.float32), \
            np.zeros(N_pad, np.uint16)
        for t in range(1, w["steps"] + 1):
            c = synth.contributions(D, N, N_pad, seed=31, step=t, sigma=w["sigma"], dist=w["dist"],
                                    zero_frac=w["zero_frac"], device="cuda")
            z3.zero3_reduce_adamw(plan, -1, c, p, m, v, wk, z3.adamw(**hp_for(t)), reduce_dtype=mode)
            oracle.reduce_adamw([synth.bf16_bits(x) for x in c], S, -1, hp_, hm, hv, hw, oracle_hp(t),
                                reduce_dtype=mode)
        torch.cuda.synchronize()
        what = f"100 steps D={D} mode={mode}"
        assert_f32_parity(f32_host(p), hp_, "master " + what)
        assert_f32_parity(f32_host(m), hm, "exp_avg " + what)
        assert_f32_parity(f32_host(v), hv, "exp_avg_sq " + what)
        assert_bf16_parity(synth.bf16_bits(wk), hw, "work_bf16 " + what)


def test_llama70b_layer_owned_rank(z3):
    """One 70B layer's owned shard of rank 3 at D = 8, contributions in the owned layout."""
    run_sampled(z3, "llama70b_layer", 8, 3, z3.Z3_CONTRIB_OWNED, 0, steps=2, k=100_000)


def test_tiny_gpt_full_ten_steps_then_gather(z3):
    """Config of the 3.3M-parameter GPT, every element compared, then the gather."""
    w = synth.WORKLOADS["tiny_gpt"]
    shapes = [s for _, s in w["tensors"]]
    plan, ref = checked_plan(z3, shapes, w["D"], synth.ALIGN)
    N, N_pad, S, D = ref.N, ref.N_pad, ref.S, ref.D
    p, m, v = state_init(N, N_pad, 0)
    wk = torch.zeros(N_pad, dtype=torch.bfloat16, device="cuda")
    hp_, hm, hv, hw = f32_host(p).copy(), np.zeros(N_pad, np.float32), np.zeros(N_pad, np.float32), \
        np.zeros(N_pad, np.uint16)
    for t in range(1, 11):
        c = synth.contributions(D, N, N_pad, seed=0, step=t, sigma=w["sigma"], device="cuda")
        z3.zero3_reduce_adamw(plan, -1, c, p, m, v, wk, z3.adamw(**hp_for(t)))
        oracle.reduce_adamw([synth.bf16_bits(x) for x in c], S, -1, hp_, hm, hv, hw, oracle_hp(t))
    torch.cuda.synchronize()
    assert_f32_parity(f32_host(p), hp_, "master")
    assert_f32_parity(f32_host(m), hm, "exp_avg")
    assert_f32_parity(f32_host(v), hv, "exp_avg_sq")
    assert_bf16_parity(synth.bf16_bits(wk), hw, "work_bf16")
    flat = torch.empty(N_pad, dtype=torch.bfloat16, device="cuda")
    outs = [torch.empty(s, dtype=torch.bfloat16, device="cuda") for s in shapes]
    z3.zero3_gather_block(plan, [wk[r * S:(r + 1) * S] for r in range(D)], flat, outs)
    torch.cuda.synchronize()
    ref_flat = oracle.all_gather([hw[r * S:(r + 1) * S] for r in range(D)], S)
    assert np.array_equal(synth.bf16_bits(flat), ref_flat)
    ref_t = oracle.unflatten(ref_flat, ref.offsets, ref.numels)
    for o, r, view in zip(outs, ref_t, plan.views(flat)):
        assert np.array_equal(synth.bf16_bits(o).ravel(), r)
        assert np.array_equal(synth.bf16_bits(view).ravel(), r)


def test_single_launch_beyond_2_31_elements(z3):
    """One launch over more than 2^31 elements (no 32-bit index anywhere): the fused
    kernel and the flat gather, sampled around 2^31 and at the end."""
    D = 2
    N = 2 ** 31 + 777
    torch.cuda.empty_cache()
    free, _ = torch.cuda.mem_get_info()
    if free < 48e9:
        pytest.skip("needs about 45 GB of free device memory")
    plan, ref = checked_plan(z3, [(N,)], D, synth.ALIGN)
    N_pad, S = ref.N_pad, ref.S
    p = synth.master_weights(N, N_pad, seed=21, device="cuda")
    m, v = torch.zeros_like(p), torch.zeros_like(p)
    w = torch.zeros(N_pad, dtype=torch.bfloat16, device="cuda")
    c = synth.contributions(D, N, N_pad, seed=21, step=1, sigma=1e-3, device="cuda")
    rng = np.random.default_rng(21)
    idx = np.unique(np.concatenate([rng.choice(N_pad, 50_000, replace=False),
                                    np.arange(2 ** 31 - 64, 2 ** 31 + 64), np.arange(S - 64, S + 64),
                                    np.arange(N - 64, N_pad)]))
    ti = torch.from_numpy(idx).cuda()
    hp_ = f32_host(p[ti]).copy()
    hm, hv, hw = np.zeros(idx.size, np.float32), np.zeros(idx.size, np.float32), np.zeros(idx.size, np.uint16)
    z3.zero3_reduce_adamw(plan, -1, c, p, m, v, w, z3.adamw(**hp_for(1)))
    oracle.reduce_adamw([synth.bf16_bits(x[ti]) for x in c], idx.size, 0, hp_, hm, hv, hw, oracle_hp(1),
                        layout=oracle.LAYOUT_OWNED)
    del c
    flat = torch.empty(N_pad, dtype=torch.bfloat16, device="cuda")
    z3.zero3_gather_block(plan, [w[r * S:(r + 1) * S] for r in range(D)], flat)
    torch.cuda.synchronize()
    assert_f32_parity(f32_host(p[ti]), hp_, "master")
    assert_f32_parity(f32_host(m[ti]), hm, "exp_avg")
    assert_f32_parity(f32_host(v[ti]), hv, "exp_avg_sq")
    assert_bf16_parity(synth.bf16_bits(w[ti]), hw, "work_bf16")
    assert np.array_equal(synth.bf16_bits(flat[ti]), hw)
    assert not p[N:].any() and not w[N:].view(torch.int16).any()
    del p, m, v, w, flat
    torch.cuda.empty_cache()


def test_random_hyperparameters_match_oracle(z3):
    """Bit-exact parity across AdamW hyper-parameters (momentum off, large eps,
    large learning rate, no decay, late steps) and both reduce dtypes."""
    import random
    rnd = random.Random(99)
    plan, ref = checked_plan(z3, [(30000,), (4097,)], 4, 8)
    N, N_pad, S = ref.N, ref.N_pad, ref.S
    for case in range(12):
        a = dict(lr=10 ** rnd.uniform(-5, -1.5), beta1=rnd.choice([0.0, 0.5, 0.9, 0.99]),
                 beta2=rnd.choice([0.5, 0.95, 0.999]), eps=10 ** rnd.uniform(-10, -2),
                 weight_decay=rnd.choice([0.0, 0.01, 0.1, 0.5]))
        t0 = rnd.choice([1, 1, 7, 1000, 123456])
        mode = case % 2
        p, m, v = state_init(N, N_pad, case)
        w = torch.zeros(N_pad, dtype=torch.bfloat16, device="cuda")
        hp_, hm, hv, hw = f32_host(p).copy(), np.zeros(N_pad, np.float32), np.zeros(N_pad, np.float32), \
            np.zeros(N_pad, np.uint16)
        for t in range(t0, t0 + 3):
            c = synth.contributions(4, N, N_pad, seed=case, step=t, sigma=1e-3, device="cuda")
            z3.zero3_reduce_adamw(plan, -1, c, p, m, v, w, z3.adamw(step=t, **a), reduce_dtype=mode)
            oracle.reduce_adamw([synth.bf16_bits(x) for x in c], S, -1, hp_, hm, hv, hw,
                                oracle.hp(a["lr"], a["beta1"], a["beta2"], a["eps"], a["weight_decay"], t),
                                reduce_dtype=mode)
        torch.cuda.synchronize()
        what = f"case {case} {a} t0={t0} mode={mode}"
        assert_f32_parity(f32_host(p), hp_, "master " + what)
        assert_f32_parity(f32_host(m), hm, "exp_avg " + what)
        assert_f32_parity(f32_host(v), hv, "exp_avg_sq " + what)
        assert_bf16_parity(synth.bf16_bits(w), hw, "work_bf16 " + what)


@pytest.mark.parametrize("extra", [1, 2, 3, 4, 5, 7])
def test_four_element_folds_every_tail_residue(z3, extra):
    """The instantiations that take 4 elements per thread (the bf16 fold of 16 ranks,
    and of 4 and 8 nodes of 8 ranks; the generic one-node fp32 fold; the generic
    HYBRID_SHARD fold in both dtypes): single-rank launches whose partition length
    leaves every remainder mod 4 and mod 8 for the scalar tail, owned and full
    layouts, against the oracle."""
    S = 1000 + extra                       # partition length; A = 1 keeps it unpadded
    run_small(z3, [16 * S], 16, 1, 0, z3.Z3_CONTRIB_FULL, 1, steps=2)       # rank 0: aligned at offset 0
    run_small(z3, [16 * S], 16, 1, 11, z3.Z3_CONTRIB_OWNED, 1, steps=2)
    for D in (3, 12):                      # runtime rank count: one chunk of 8 ranks, and a partial second
        run_small(z3, [D * S], D, 1, 0, z3.Z3_CONTRIB_FULL, 0, steps=2)
        run_small(z3, [D * S], D, 1, D - 1, z3.Z3_CONTRIB_OWNED, 0, steps=2)
    from test_gpu_hybrid import run_small as run_hybrid
    for R in (4, 8):
        run_hybrid(z3, [8 * S], R, 8, 1, 0, z3.Z3_CONTRIB_FULL, 1, steps=2)
        run_hybrid(z3, [8 * S], R, 8, 1, 5, z3.Z3_CONTRIB_OWNED, 1, steps=2)
    for R, D, mode in ((3, 5, 0), (2, 3, 1)):   # runtime node and rank counts
        run_hybrid(z3, [D * S], R, D, 1, 0, z3.Z3_CONTRIB_FULL, mode, steps=2)
        run_hybrid(z3, [D * S], R, D, 1, D - 1, z3.Z3_CONTRIB_OWNED, mode, steps=2)
