"""Pins for the oracle: each checks it against something other than itself --
the pages' worked examples and printed figures (tests/golden/), closed forms,
invariants, brute force with exact arithmetic, and independent library
routines (torch's bf16 cast and arithmetic, torch.optim.AdamW in float64).

Every function of the oracle has at least one pin here; a plausible mistake
(a dropped rank, a wrong slice index, a missing 1/D, a flipped sign, a missing
bias correction, coupled weight decay, a wrong pad) fails at least one test.
"""
import random
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
import synth

U = 2.0 ** -24  # binary32 unit roundoff


def bf16_torch_bits(x: np.ndarray) -> np.ndarray:
    return synth.bf16_bits(torch.from_numpy(np.asarray(x, dtype=np.float32)).to(torch.bfloat16))


def rand_bf16(rng: np.random.Generator, n: int, scale: float = 1e-3) -> np.ndarray:
    return bf16_torch_bits((rng.standard_normal(n) * scale).astype(np.float32))


# --------------------------------------------------------------- conversions
def test_bf16_rne_matches_torch_cast():
    """Pin: the oracle's own RNE cast equals torch's fp32->bf16 cast bit for bit."""
    rng = np.random.default_rng(1)
    vals = [0.0, -0.0, 1.0, -1.0, np.inf, -np.inf, 3.4028235e38, -3.4028235e38,
            1e-45, -1e-45, 1.1754944e-38, 2.0 ** -130, 65504.0, 1.00390625, 1.01171875]
    # exact halfway cases with even and odd kept parts, and just above / below
    for kept in (0x3F80, 0x3F81, 0x0001, 0x0002, 0x7F7F, 0x8001, 0xBF80):
        for low in (0x7FFF, 0x8000, 0x8001, 0x0000, 0xFFFF):
            vals.append(np.array([(kept << 16) | low], dtype=np.uint32).view(np.float32)[0])
    x = np.concatenate([np.array(vals, dtype=np.float32),
                        (rng.standard_normal(20000) * 10.0 ** rng.integers(-40, 38, 20000)).astype(np.float32),
                        rng.integers(0, 2 ** 32, 20000, dtype=np.uint64).astype(np.uint32).view(np.float32)])
    x = x[~np.isnan(x)]
    mine = oracle.bf16_from_f32(x)
    ref = bf16_torch_bits(x)
    assert np.array_equal(mine, ref)


def test_bf16_nan_stays_nan():
    x = np.array([np.nan, -np.nan], dtype=np.float32)
    x = np.concatenate([x, np.array([0x7F800001, 0xFFFFFFFF, 0x7FC00000], dtype=np.uint32).view(np.float32)])
    back = oracle.f32_from_bf16(oracle.bf16_from_f32(x))
    assert np.all(np.isnan(back))


# ----------------------------------------------------------------------- plan
def test_plan_invariants_brute_force():
    """Pin: offsets are the exclusive prefix sum, the padded size is the least
    multiple of D*A not below N, and the D partitions tile [0, N_pad)."""
    rnd = random.Random(7)
    for _ in range(400):
        n = rnd.randint(0, 7)
        numel = [rnd.randint(0, 40) for _ in range(n)]
        D = rnd.randint(1, 9)
        A = rnd.choice([1, 2, 3, 8, 128])
        offs, N, N_pad, S = oracle.plan(numel, D, A)
        assert N == sum(numel)
        assert list(offs) == list(np.concatenate([[0], np.cumsum(numel)[:-1]]).astype(np.int64)) if n else True
        assert N_pad % (D * A) == 0 and N <= N_pad < N + D * A
        smallest = next(k for k in range(0, N + D * A + 1, D * A) if k >= N)
        assert N_pad == smallest
        assert S * D == N_pad
        covered = []
        for r in range(D):
            b, e = oracle.rank_range(N, S, r)
            assert b == r * S and b <= e <= b + S
            covered += list(range(b, b + S))
            assert e - b == max(0, min(N, (r + 1) * S) - r * S)
        assert covered == list(range(N_pad))
        # every tensor lies inside [0, N)
        for o, k in zip(offs, numel):
            assert 0 <= o and o + k <= N


def test_plan_rejects_bad_arguments():
    with pytest.raises(ValueError):
        oracle.plan([3], 0, 1)
    with pytest.raises(ValueError):
        oracle.plan([3], 1, 0)
    with pytest.raises(ValueError):
        oracle.plan([3, -1], 2, 1)


def test_plan_workloads_golden(golden):
    """Pin: the plan figures derived by hand for the synthetic workloads."""
    g = golden("plan_workloads.json")
    for w in g["workloads"]:
        tensors = synth.WORKLOADS[w["name"]]["tensors"]
        assert len(tensors) == w["n_tensors"]
        offs, N, N_pad, S = oracle.plan([synth.numel(s) for _, s in tensors], w["D"], w["A"])
        assert (N, N_pad, S) == (w["N"], w["N_pad"], w["S"])
        if "last_rank_real" in w:
            b, e = oracle.rank_range(N, S, w["D"] - 1)
            assert e - b == w["last_rank_real"] and S - (e - b) == w["last_rank_pad"]


# --------------------------------------------------------------- memory ledger
def test_memory_buckets_golden(golden):
    """Pin: the per-parameter buckets of page 2 §2 at 7B."""
    g = golden("memory_figures.json")["bytes_per_param_buckets"]
    N = g["N"]
    assert oracle.memory_bytes(N, 1, 0) == pytest.approx(g["total_GB"] * 1e9)
    # ZeRO-3 at D = 1 shards nothing: every stage equals pure DP.
    for stage in (1, 2, 3):
        assert oracle.memory_bytes(N, 1, stage) == pytest.approx(g["total_GB"] * 1e9)


def test_memory_figures_golden(golden):
    """Pin: the printed per-device figures the formulas reproduce; the ones
    they do not are recorded as disagreements of the pages, not pins."""
    g = golden("memory_figures.json")
    for f in g["figures"]:
        got = oracle.memory_bytes(f["N"], f["D"], f["stage"]) / 1e9
        close = abs(got - f["GB"]) <= f["rel_tol"] * f["GB"] + 0.5
        assert close == f["consistent"], (f["source"], got)
    for b in g["sharded_buckets"]:
        got = b["bytes_per_param"] * b["N"] / b["D"] / 1e9
        assert got == pytest.approx(b["GB"], rel=b["rel_tol"] + 1e-12)
    # the per-stage formulas differ exactly by the buckets they shard
    N, D = 7e9, 32
    z1, z2, z3 = (oracle.memory_bytes(N, D, s) for s in (1, 2, 3))
    assert z1 - z2 == pytest.approx(6 * N - 6 * N / D)
    assert z2 - z3 == pytest.approx(2 * N - 2 * N / D)
    assert z3 == pytest.approx(20 * N / D)
    assert oracle.memory_bytes(N, D, 9) == -1.0


def test_transient_and_steady_state_golden(golden):
    g = golden("memory_figures.json")
    t = g["transient"]
    block = 12 * t["d"] * t["d"]
    assert oracle.transient_bytes(block, 1) / 1e6 == pytest.approx(t["one_buffer_MB"], rel=t["rel_tol"])
    assert oracle.transient_bytes(block, 2) / 1e6 == pytest.approx(t["two_buffers_MB"], rel=t["rel_tol"])
    s = g["steady_state"]
    got = (oracle.memory_bytes(s["N"], s["D"], 3) + s["transient_MB"] * 1e6) / 1e9
    assert got == pytest.approx(s["GB"], rel=s["rel_tol"])


def test_allgather_volume_golden(golden):
    """Pin: page 2 §5.3's forward and backward all-gather volume per device
    (each block gathered once per pass; a device receives the (D-1)/D it does
    not own), and the cases the formula fixes exactly."""
    a = golden("memory_figures.json")["allgather"]
    got = oracle.allgather_bytes(a["block_MB"] * 1e6, a["L"], a["D"]) / 1e9
    assert got == pytest.approx(a["forward_GB"], rel=a["rel_tol"])
    assert got == pytest.approx(a["backward_GB"], rel=a["rel_tol"])
    assert oracle.allgather_bytes(123456.0, 7, 1) == 0.0            # one rank holds everything
    for block, L, D in [(1000, 3, 2), (4096, 5, 8), (999, 1, 3)]:
        exact = Fraction(L) * block * (D - 1) / D
        assert oracle.allgather_bytes(block, L, D) == pytest.approx(float(exact), rel=1e-15)


# ----------------------------------------------------------------- reduction
def test_reduce_scatter_worked_example(golden):
    """Pin: page 3's 4-GPU reduce-scatter: GPU x gets the sum of slice x."""
    g = golden("reduce_scatter_worked_example.json")
    D, L = g["D"], g["slice_len"]
    contribs = [bf16_torch_bits(np.array(sum(row, []), dtype=np.float32)) for row in g["grads"]]
    offs, N, N_pad, S = oracle.plan([D * L], D, 1)
    assert S == L
    for mode in (oracle.REDUCE_FP32, oracle.REDUCE_BF16):
        for x in range(D):
            got = oracle.reduce_scatter(contribs, S, x, oracle.LAYOUT_FULL, mode)
            assert np.array_equal(got * D, np.array(g["expected_sum_per_gpu"][x], dtype=np.float32))
            owned = [c[x * S:(x + 1) * S].copy() for c in contribs]
            got_owned = oracle.reduce_scatter(owned, S, x, oracle.LAYOUT_OWNED, mode)
            assert np.array_equal(got_owned, got)
        every = oracle.reduce_scatter(contribs, S, -1, oracle.LAYOUT_FULL, mode)
        assert np.array_equal(every * D, np.array(sum(g["expected_sum_per_gpu"], []), dtype=np.float32))


@pytest.mark.parametrize("D", [1, 2, 3, 4, 5, 7, 8, 9, 16, 32, 64])
def test_reduce_fp32_matches_torch_left_fold(D):
    """Pin: fp32 reduce equals a torch fp32 left fold over ranks 0..D-1 times fp32(1/D)."""
    rng = np.random.default_rng(D)
    S = 37
    contribs = [rand_bf16(rng, D * S) for _ in range(D)]
    got = oracle.reduce_scatter(contribs, S, -1)
    t = [torch.from_numpy(c.view(np.int16)).view(torch.bfloat16).float() for c in contribs]
    acc = t[0].clone()
    for d in range(1, D):
        acc = acc + t[d]
    ref = (acc * torch.tensor(1.0 / D, dtype=torch.float32)).numpy()
    assert np.array_equal(got.view(np.uint32), ref.view(np.uint32))


@pytest.mark.parametrize("D", [2, 3, 8, 13, 32])
def test_reduce_fp32_error_bound_exact_sum(D):
    """Pin: against the exact rational sum, the fp32 fold errs by at most
    (D-1) u sum|c| (standard recursive-summation bound), plus one rounding
    of the 1/D scale."""
    rng = np.random.default_rng(100 + D)
    S = 23
    contribs = [rand_bf16(rng, D * S, scale=10.0 ** rng.integers(-5, 2)) for _ in range(D)]
    got = oracle.reduce_scatter(contribs, S, -1).astype(np.float64)
    vals = [oracle.f32_from_bf16(c).astype(np.float64) for c in contribs]
    for i in range(D * S):
        exact = sum(Fraction(float(v[i])) for v in vals) / D
        mag = sum(abs(float(v[i])) for v in vals) / D
        bound = ((D - 1) * U * (1 + U) ** D) * mag + U * (abs(float(exact)) + (D - 1) * U * mag) + 1e-45
        assert abs(Fraction(float(got[i])) - exact) <= Fraction(bound)


@pytest.mark.parametrize("D", [1, 2, 4, 6, 8, 16])
def test_reduce_bf16_matches_torch_bf16_adds(D):
    """Pin: the bf16 reduce equals torch's bf16 tensor adds (each partial sum
    rounded to bf16), then a bf16-rounded 1/D scale."""
    rng = np.random.default_rng(200 + D)
    S = 41
    contribs = [rand_bf16(rng, D * S) for _ in range(D)]
    got = oracle.reduce_scatter(contribs, S, -1, reduce_dtype=oracle.REDUCE_BF16)
    t = [torch.from_numpy(c.view(np.int16)).view(torch.bfloat16) for c in contribs]
    acc = t[0].clone()
    for d in range(1, D):
        acc = acc + t[d]
    ref = (acc.float() * torch.tensor(1.0 / D, dtype=torch.float32)).to(torch.bfloat16).float().numpy()
    assert np.array_equal(got.view(np.uint32), ref.view(np.uint32))


def test_reduce_integers_modes_agree_and_are_exact():
    """Pin: with small-integer contributions every partial sum is exact, so
    both reduce dtypes give exactly sum/D for power-of-two D."""
    for D in (1, 2, 4, 8, 16):
        S = 64
        contribs = [synth.bf16_bits(synth.contribution(D * S, D * S, seed=3, step=1, rank=r, sigma=0,
                                                       dist="integers")) for r in range(D)]
        a = oracle.reduce_scatter(contribs, S, -1, reduce_dtype=oracle.REDUCE_FP32)
        b = oracle.reduce_scatter(contribs, S, -1, reduce_dtype=oracle.REDUCE_BF16)
        exact = np.sum([oracle.f32_from_bf16(c).astype(np.float64) for c in contribs], axis=0) / D
        assert np.array_equal(a, b) and np.array_equal(a.astype(np.float64), exact)


def test_reduce_rejects_bad_arguments():
    c = [np.zeros(8, dtype=np.uint16)] * 2
    with pytest.raises(ValueError):
        oracle.reduce_scatter(c, 4, 2)                 # rank >= D
    with pytest.raises(ValueError):
        oracle.reduce_scatter(c, 4, -1, oracle.LAYOUT_OWNED)   # owned layout needs one rank
    with pytest.raises(ValueError):
        oracle.reduce_scatter(c, 4, 0, reduce_dtype=5)


# --------------------------------------------------------------------- AdamW
def test_adamw_step1_closed_form():
    """Pin: at step 1 from m = v = 0, m = (1-b1) g, v = (1-b2) g^2 and the
    bias-corrected update is lr * g / (|g| + eps) after decay (1 - lr wd)."""
    rng = np.random.default_rng(5)
    n = 5000
    g = (rng.standard_normal(n) * 1e-3).astype(np.float32)
    p0 = (rng.standard_normal(n) * 0.02).astype(np.float32)
    p, m, v = p0.copy(), np.zeros(n, np.float32), np.zeros(n, np.float32)
    lr, b1, b2, eps, wd = 3e-4, 0.9, 0.95, 1e-8, 0.1
    oracle.adamw(g, p, m, v, oracle.hp(lr, b1, b2, eps, wd, 1))
    g64 = g.astype(np.float64)
    np.testing.assert_allclose(m, (1 - b1) * g64, rtol=3e-7)
    np.testing.assert_allclose(v, (1 - b2) * g64 * g64, rtol=5e-7)
    expect = p0.astype(np.float64) * (1 - lr * wd) - lr * g64 / (np.abs(g64) + eps)
    # the update is lr*sign(g) to within eps/|g|, so p moves by about lr
    moved = np.abs(p0.astype(np.float64) * (1 - lr * wd) - p)
    assert np.all(np.abs(moved - lr) <= lr * eps / np.abs(g64) + 8 * U * (np.abs(p0) + lr))
    np.testing.assert_allclose(p, expect, rtol=0, atol=4 * U * 0.1)


def test_adamw_zero_gradient_keeps_zero_pad():
    """Pin: a zero parameter with zero gradient stays exactly zero (the pad)."""
    n = 64
    p, m, v = np.zeros(n, np.float32), np.zeros(n, np.float32), np.zeros(n, np.float32)
    g = np.zeros(n, np.float32)
    for t in range(1, 11):
        oracle.adamw(g, p, m, v, oracle.hp(step=t))
    assert not p.any() and not m.any() and not v.any()


def torch_adamw64(p0, grads, lr, b1, b2, eps, wd):
    p = torch.nn.Parameter(torch.from_numpy(p0.astype(np.float64)))
    opt = torch.optim.AdamW([p], lr=lr, betas=(b1, b2), eps=eps, weight_decay=wd,
                            foreach=False, fused=False)
    for g in grads:
        p.grad = torch.from_numpy(np.asarray(g, dtype=np.float64))
        opt.step()
    st = opt.state[p]
    return p.detach().numpy(), st["exp_avg"].numpy(), st["exp_avg_sq"].numpy()


def test_adamw_ten_steps_matches_torch_adamw_float64():
    """Pin: ten fp32 steps track torch.optim.AdamW run in float64 (an
    independent implementation) within the binary32 rounding of ten steps."""
    rng = np.random.default_rng(11)
    n = 4000
    p0 = (rng.standard_normal(n) * 0.02).astype(np.float32)
    grads = [(rng.standard_normal(n) * 1e-3).astype(np.float32) for _ in range(10)]
    lr, b1, b2, eps, wd = 3e-4, 0.9, 0.95, 1e-8, 0.1
    p, m, v = p0.copy(), np.zeros(n, np.float32), np.zeros(n, np.float32)
    for t, g in enumerate(grads, 1):
        oracle.adamw(g, p, m, v, oracle.hp(lr, b1, b2, eps, wd, t))
    rp, rm, rv = torch_adamw64(p0, grads, lr, b1, b2, eps, wd)
    np.testing.assert_allclose(m, rm, rtol=2e-6, atol=1e-6 * np.abs(rm).max())
    np.testing.assert_allclose(v, rv, rtol=2e-6, atol=1e-6 * np.abs(rv).max())
    np.testing.assert_allclose(p, rp, rtol=1e-6, atol=1e-6 * np.abs(rp).max())


@pytest.mark.parametrize("lr,b1,b2,eps,wd,t0", [
    (1e-3, 0.0, 0.999, 1e-8, 0.0, 1),       # no momentum, no decay
    (1e-2, 0.95, 0.99, 1e-3, 0.3, 1),      # a large eps: its place in the denominator shows
    (5e-5, 0.5, 0.5, 1e-6, 0.01, 1),
    (3e-4, 0.9, 0.95, 1e-8, 0.1, 990),     # late steps: the bias corrections are nearly 1
])
def test_adamw_hyperparameters_match_torch_adamw_float64(lr, b1, b2, eps, wd, t0):
    """Pin: with t0 = 1, ten fp32 steps track torch.optim.AdamW run in float64
    across the hyper-parameters.  torch always counts steps from 1, so a late
    step (t0 > 1) is checked instead as one step from zero moments against the
    closed form in float64, where the bias corrections are nearly 1."""
    rng = np.random.default_rng(int(lr * 1e6) + t0)
    n = 3000
    p0 = (rng.standard_normal(n) * 0.02).astype(np.float32)
    grads = [(rng.standard_normal(n) * 1e-3).astype(np.float32) for _ in range(10)]
    if t0 == 1:
        p, m, v = p0.copy(), np.zeros(n, np.float32), np.zeros(n, np.float32)
        for t, g in enumerate(grads, 1):
            oracle.adamw(g, p, m, v, oracle.hp(lr, b1, b2, eps, wd, t))
        rp, rm, rv = torch_adamw64(p0, grads, lr, b1, b2, eps, wd)
        np.testing.assert_allclose(m, rm, rtol=2e-6, atol=1e-6 * np.abs(rm).max())
        np.testing.assert_allclose(v, rv, rtol=2e-6, atol=1e-6 * np.abs(rv).max())
        np.testing.assert_allclose(p, rp, rtol=1e-6, atol=1e-6 * np.abs(rp).max())
    else:
        # one step at t0 from zero moments, against the closed form in float64
        g = grads[0].astype(np.float64)
        p, m, v = p0.copy(), np.zeros(n, np.float32), np.zeros(n, np.float32)
        oracle.adamw(grads[0], p, m, v, oracle.hp(lr, b1, b2, eps, wd, t0))
        m64, v64 = (1 - b1) * g, (1 - b2) * g * g
        step = lr / (1 - b1 ** t0)
        denom = np.sqrt(v64) / np.sqrt(1 - b2 ** t0) + eps
        p64 = p0.astype(np.float64) * (1 - lr * wd) - step * m64 / denom
        np.testing.assert_allclose(p, p64, rtol=1e-6, atol=1e-6 * np.abs(p64).max())


def test_adamw_detects_coupled_decay_and_missing_bias_correction():
    """The torch pin separates the plausible wrong variants of AdamW."""
    rng = np.random.default_rng(12)
    n = 2000
    p0 = (rng.standard_normal(n) * 0.02).astype(np.float32)
    g = (rng.standard_normal(n) * 1e-3).astype(np.float32)
    p, m, v = p0.copy(), np.zeros(n, np.float32), np.zeros(n, np.float32)
    oracle.adamw(g, p, m, v, oracle.hp(step=1))
    # Adam with L2 (coupled) decay: the decay enters the gradient instead
    pa = torch.nn.Parameter(torch.from_numpy(p0.astype(np.float64)))
    opt = torch.optim.Adam([pa], lr=3e-4, betas=(0.9, 0.95), eps=1e-8, weight_decay=0.1)
    pa.grad = torch.from_numpy(g.astype(np.float64))
    opt.step()
    assert np.abs(p - pa.detach().numpy()).max() > 1e-6
    # no bias correction would move p by (1-b1)/sqrt(1-b2) lr ~ 0.45 lr, not lr
    moved = np.abs(p0.astype(np.float64) * (1 - 3e-5) - p)
    assert np.all(np.abs(moved - 3e-4) <= 3e-4 * 1e-8 / np.abs(g.astype(np.float64)) + 8 * U * (np.abs(p0) + 3e-4))


def test_reduce_adamw_d1_is_plain_adamw_on_the_contribution():
    """Pin: with one rank the reduce is the identity and the step is AdamW."""
    rng = np.random.default_rng(13)
    n = 1024
    c = rand_bf16(rng, n)
    p0 = (rng.standard_normal(n) * 0.02).astype(np.float32)
    p, m, v, w = p0.copy(), np.zeros(n, np.float32), np.zeros(n, np.float32), np.zeros(n, np.uint16)
    oracle.reduce_adamw([c], n, 0, p, m, v, w, oracle.hp(step=1))
    rp, rm, rv = torch_adamw64(p0, [oracle.f32_from_bf16(c)], 3e-4, 0.9, 0.95, 1e-8, 0.1)
    np.testing.assert_allclose(p, rp, rtol=1e-6, atol=1e-9)
    assert np.array_equal(w, bf16_torch_bits(p))


# ------------------------------------------------------- sharded = unsharded
@pytest.mark.parametrize("D,A,numels", [(4, 1, [5, 7, 1]), (8, 2, [33, 1, 60]), (3, 8, [10, 20]),
                                        (16, 1, [255]), (2, 128, [300, 1])])
def test_sharded_steps_equal_one_unsharded_step(D, A, numels):
    """Pin: the pages state that sharding leaves the math identical to DDP.
    Ten steps run rank by rank on each owned shard, concatenated, equal ten
    unsharded steps (one pass over the whole padded block) bit for bit, and
    track float64 torch AdamW on the exactly averaged gradient."""
    _, N, N_pad, S = oracle.plan(numels, D, A)
    rng = np.random.default_rng(D * 1000 + A)
    p0 = np.zeros(N_pad, np.float32)
    p0[:N] = (rng.standard_normal(N) * 0.02).astype(np.float32)
    shard_state = [[p0[r * S:(r + 1) * S].copy(), np.zeros(S, np.float32), np.zeros(S, np.float32),
                    np.zeros(S, np.uint16)] for r in range(D)]
    full = [p0.copy(), np.zeros(N_pad, np.float32), np.zeros(N_pad, np.float32), np.zeros(N_pad, np.uint16)]
    avg64 = []
    for t in range(1, 11):
        contribs = []
        for r in range(D):
            c = np.zeros(N_pad, np.uint16)
            c[:N] = rand_bf16(rng, N)
            contribs.append(c)
        h = oracle.hp(step=t)
        for r in range(D):
            p, m, v, w = shard_state[r]
            oracle.reduce_adamw(contribs, S, r, p, m, v, w, h)
        oracle.reduce_adamw(contribs, S, -1, *full, h)
        avg64.append(np.sum([oracle.f32_from_bf16(c).astype(np.float64) for c in contribs], axis=0) / D)
    for k in range(4):
        cat = np.concatenate([shard_state[r][k] for r in range(D)])
        assert np.array_equal(cat.view(np.uint8), full[k].view(np.uint8))
    assert not full[0][N:].any() and not full[3][N:].any()   # pad stays zero
    rp, _, _ = torch_adamw64(p0, avg64, 3e-4, 0.9, 0.95, 1e-8, 0.1)
    np.testing.assert_allclose(full[0], rp, rtol=1e-6, atol=2e-6 * np.abs(rp).max())


def test_reduce_adamw_composes_reduce_then_adamw():
    """The fused oracle step is the reduce followed by AdamW and the bf16 cast."""
    rng = np.random.default_rng(21)
    D, S = 4, 50
    contribs = [rand_bf16(rng, D * S) for _ in range(D)]
    p0 = (rng.standard_normal(D * S) * 0.02).astype(np.float32)
    for mode in (oracle.REDUCE_FP32, oracle.REDUCE_BF16):
        a = [p0.copy(), np.zeros(D * S, np.float32), np.zeros(D * S, np.float32), np.zeros(D * S, np.uint16)]
        oracle.reduce_adamw(contribs, S, -1, *a, oracle.hp(step=3), reduce_dtype=mode)
        g = oracle.reduce_scatter(contribs, S, -1, reduce_dtype=mode)
        b = [p0.copy(), np.zeros(D * S, np.float32), np.zeros(D * S, np.float32)]
        oracle.adamw(g, *b, oracle.hp(step=3))
        for x, y in zip(a[:3], b):
            assert np.array_equal(x, y)
        assert np.array_equal(a[3], bf16_torch_bits(b[0]))


# -------------------------------------------------------------- HYBRID_SHARD
def test_hybrid_worked_examples(golden):
    """Pin: hand-derived HYBRID_SHARD reductions (R nodes of D ranks) in which
    the node-then-cross-node order, the rank-to-node map, the node order, the
    bf16 rounding of every partial sum and the 1/(R*D) scale each change the
    result."""
    g = golden("hybrid_worked_examples.json")
    for case in g["cases"]:
        R, D = case["R"], case["D"]
        contribs = [bf16_torch_bits(np.array([x], dtype=np.float32)) for x in case["contributions"]]
        assert [float(oracle.f32_from_bf16(c)[0]) for c in contribs] == case["contributions"]
        got = oracle.reduce_scatter_hybrid(contribs, R, 1, 0, oracle.LAYOUT_OWNED, case["reduce_dtype"])
        assert float(got[0]) == case["expected"], case["name"]


@pytest.mark.parametrize("mode", [0, 1])
@pytest.mark.parametrize("D", [1, 2, 3, 8])
def test_hybrid_one_node_is_the_plain_reduction(D, mode):
    """Pin: with one node, HYBRID_SHARD is FULL_SHARD: bit-identical to the
    plain reduce-scatter, for every rank and layout."""
    rng = np.random.default_rng(300 + D)
    S = 29
    contribs = [rand_bf16(rng, D * S) for _ in range(D)]
    every = oracle.reduce_scatter_hybrid(contribs, 1, S, -1, oracle.LAYOUT_FULL, mode)
    plain = oracle.reduce_scatter(contribs, S, -1, reduce_dtype=mode)
    assert np.array_equal(every.view(np.uint32), plain.view(np.uint32))
    for r in range(D):
        owned = [c[r * S:(r + 1) * S].copy() for c in contribs]
        got = oracle.reduce_scatter_hybrid(owned, 1, S, r, oracle.LAYOUT_OWNED, mode)
        assert np.array_equal(got.view(np.uint32), every[r * S:(r + 1) * S].view(np.uint32))


@pytest.mark.parametrize("mode", [0, 1])
@pytest.mark.parametrize("R", [2, 3, 4, 8])
def test_hybrid_one_rank_per_node_is_the_plain_fold_over_nodes(R, mode):
    """Pin: with one rank per node, the node sums are the contributions and the
    result is the plain left fold over R ranks times 1/R."""
    rng = np.random.default_rng(400 + R)
    S = 31
    contribs = [rand_bf16(rng, S) for _ in range(R)]
    got = oracle.reduce_scatter_hybrid(contribs, R, S, -1, oracle.LAYOUT_FULL, mode)
    ref = oracle.reduce_scatter(contribs, S, 0, oracle.LAYOUT_OWNED, mode)
    assert np.array_equal(got.view(np.uint32), ref.view(np.uint32))


@pytest.mark.parametrize("R,D", [(2, 2), (4, 8), (2, 16), (8, 4)])
def test_hybrid_integers_are_the_exact_mean(R, D):
    """Pin: with small-integer contributions every partial sum is exact, so
    both reduce dtypes give exactly sum / (R*D) for power-of-two R*D."""
    S = 16
    contribs = [synth.bf16_bits(synth.contribution(D * S, D * S, seed=5, step=1, rank=i, sigma=0,
                                                   dist="integers")) for i in range(R * D)]
    exact = np.sum([oracle.f32_from_bf16(c).astype(np.float64) for c in contribs], axis=0) / (R * D)
    for mode in (oracle.REDUCE_FP32, oracle.REDUCE_BF16):
        got = oracle.reduce_scatter_hybrid(contribs, R, S, -1, oracle.LAYOUT_FULL, mode)
        assert np.array_equal(got.astype(np.float64), exact)


@pytest.mark.parametrize("R,D", [(2, 3), (4, 8), (3, 5)])
def test_hybrid_matches_torch_two_level_fold(R, D):
    """Pin: torch's own fp32 and bf16 tensor additions, node by node and then
    across nodes, scaled by fp32(1/(R*D)) (rounded to bf16 in bf16 mode)."""
    rng = np.random.default_rng(500 + R * D)
    S = 19
    contribs = [rand_bf16(rng, D * S) for _ in range(R * D)]
    t = [torch.from_numpy(c.view(np.int16)).view(torch.bfloat16) for c in contribs]
    inv = torch.tensor(1.0 / (R * D), dtype=torch.float32)
    for mode, cast in ((oracle.REDUCE_FP32, lambda x: x.float()), (oracle.REDUCE_BF16, lambda x: x)):
        nodes = []
        for k in range(R):
            acc = cast(t[k * D]).clone()
            for d in range(1, D):
                acc = acc + cast(t[k * D + d])
            nodes.append(acc)
        total = nodes[0]
        for k in range(1, R):
            total = total + nodes[k]
        ref = total.float() * inv
        if mode == oracle.REDUCE_BF16:
            ref = ref.to(torch.bfloat16).float()
        got = oracle.reduce_scatter_hybrid(contribs, R, S, -1, oracle.LAYOUT_FULL, mode)
        assert np.array_equal(got.view(np.uint32), ref.numpy().view(np.uint32))


def test_hybrid_step_composes_reduce_then_adamw():
    """The fused HYBRID_SHARD step is its reduction followed by AdamW and the cast."""
    rng = np.random.default_rng(22)
    R, D, S = 3, 4, 40
    contribs = [rand_bf16(rng, D * S) for _ in range(R * D)]
    p0 = (rng.standard_normal(D * S) * 0.02).astype(np.float32)
    for mode in (oracle.REDUCE_FP32, oracle.REDUCE_BF16):
        a = [p0.copy(), np.zeros(D * S, np.float32), np.zeros(D * S, np.float32), np.zeros(D * S, np.uint16)]
        oracle.reduce_adamw_hybrid(contribs, R, S, -1, *a, oracle.hp(step=2), reduce_dtype=mode)
        g = oracle.reduce_scatter_hybrid(contribs, R, S, -1, reduce_dtype=mode)
        b = [p0.copy(), np.zeros(D * S, np.float32), np.zeros(D * S, np.float32)]
        oracle.adamw(g, *b, oracle.hp(step=2))
        for x, y in zip(a[:3], b):
            assert np.array_equal(x, y)
        assert np.array_equal(a[3], bf16_torch_bits(b[0]))


@pytest.mark.parametrize("R,D", [(2, 3), (4, 8), (3, 1), (1, 4)])
def test_node_sums_then_fold_is_the_hybrid_step(R, D):
    """Pin: HYBRID_SHARD split across nodes (each node's sum, then the fold of
    the node sums with AdamW) is the pinned two-level step, bit for bit, for
    every partition at once and for one rank in the owned layout."""
    rng = np.random.default_rng(600 + 10 * R + D)
    S = 23
    contribs = [rand_bf16(rng, D * S) for _ in range(R * D)]
    p0 = (rng.standard_normal(D * S) * 0.02).astype(np.float32)
    for mode in (oracle.REDUCE_FP32, oracle.REDUCE_BF16):
        ref = [p0.copy(), np.zeros(D * S, np.float32), np.zeros(D * S, np.float32), np.zeros(D * S, np.uint16)]
        got = [p0.copy(), np.zeros(D * S, np.float32), np.zeros(D * S, np.float32), np.zeros(D * S, np.uint16)]
        for t in (1, 2):
            oracle.reduce_adamw_hybrid(contribs, R, S, -1, *ref, oracle.hp(step=t), reduce_dtype=mode)
            sums = [oracle.node_sum(contribs[k * D:(k + 1) * D], S, -1, reduce_dtype=mode) for k in range(R)]
            oracle.fold_adamw(sums, D, *got, oracle.hp(step=t), reduce_dtype=mode)
        for a, b in zip(got, ref):
            assert np.array_equal(a.view(np.uint8), b.view(np.uint8)), (R, D, mode)
        r = D - 1                                               # one rank, owned slices
        owned = [c[r * S:(r + 1) * S].copy() for c in contribs]
        one = [p0[r * S:(r + 1) * S].copy(), np.zeros(S, np.float32), np.zeros(S, np.float32),
               np.zeros(S, np.uint16)]
        sums = [oracle.node_sum(owned[k * D:(k + 1) * D], S, r, oracle.LAYOUT_OWNED, mode) for k in range(R)]
        oracle.fold_adamw(sums, D, *one, oracle.hp(step=1), reduce_dtype=mode)
        first = [p0.copy(), np.zeros(D * S, np.float32), np.zeros(D * S, np.float32), np.zeros(D * S, np.uint16)]
        oracle.reduce_adamw_hybrid(contribs, R, S, -1, *first, oracle.hp(step=1), reduce_dtype=mode)
        for a, b in zip(one, first):
            assert np.array_equal(a.view(np.uint8), b[r * S:(r + 1) * S].view(np.uint8))


def test_hybrid_worked_examples_through_the_two_parts(golden):
    """Pin: the hand-derived HYBRID_SHARD examples, reached through the node
    sums and their fold (AdamW with lr = 0 and no decay leaves the master, and
    the first moment is (1 - beta1) g, so g is read back from it)."""
    g = golden("hybrid_worked_examples.json")
    for case in g["cases"]:
        R, D = case["R"], case["D"]
        contribs = [bf16_torch_bits(np.array([x], dtype=np.float32)) for x in case["contributions"]]
        sums = [oracle.node_sum(contribs[k * D:(k + 1) * D], 1, 0, oracle.LAYOUT_OWNED, case["reduce_dtype"])
                for k in range(R)]
        p, m, v, w = np.zeros(1, np.float32), np.zeros(1, np.float32), np.zeros(1, np.float32), np.zeros(1, np.uint16)
        oracle.fold_adamw(sums, D, p, m, v, w, oracle.hp(lr=0.0, beta1=0.0, weight_decay=0.0), case["reduce_dtype"])
        assert float(m[0]) == case["expected"], case["name"]


@pytest.mark.parametrize("D", [1, 2, 5, 8])
def test_node_sum_matches_torch_folds(D):
    """Pin: the node sum is torch's own left fold, fp32 adds of the bf16 values
    or bf16 tensor adds, with no scaling."""
    rng = np.random.default_rng(700 + D)
    S = 29
    contribs = [rand_bf16(rng, D * S) for _ in range(D)]
    t = [torch.from_numpy(c.view(np.int16)).view(torch.bfloat16) for c in contribs]
    acc32, acc16 = t[0].float().clone(), t[0].clone()
    for d in range(1, D):
        acc32 = acc32 + t[d].float()
        acc16 = acc16 + t[d]
    got32 = oracle.node_sum(contribs, S, -1, reduce_dtype=oracle.REDUCE_FP32)
    got16 = oracle.node_sum(contribs, S, -1, reduce_dtype=oracle.REDUCE_BF16)
    assert np.array_equal(got32.view(np.uint32), acc32.numpy().view(np.uint32))
    assert np.array_equal(got16.view(np.uint32), acc16.float().numpy().view(np.uint32))


def test_hybrid_rejects_bad_arguments():
    c = [np.zeros(8, dtype=np.uint16)] * 4
    with pytest.raises(ValueError):
        oracle.reduce_scatter_hybrid(c, 3, 4, -1)          # 4 contributions do not split into 3 nodes
    with pytest.raises(ValueError):
        oracle.reduce_scatter_hybrid(c, 2, 4, 2)           # local rank out of range (D = 2)
    with pytest.raises(ValueError):
        oracle.reduce_scatter_hybrid(c, 2, 4, -1, oracle.LAYOUT_OWNED)


# --------------------------------------------------------- gather, unflatten
def test_allgather_worked_example(golden):
    """Pin: page 3's 4-GPU all-gather: every GPU ends with [A, B, C, D]."""
    g = golden("allgather_worked_example.json")
    shards = [bf16_torch_bits(np.array(s, dtype=np.float32)) for s in g["shards"]]
    flat = oracle.all_gather(shards, len(g["shards"][0]))
    assert np.array_equal(oracle.f32_from_bf16(flat), np.array(g["expected_block"], dtype=np.float32))


def test_gather_round_trip_and_unflatten():
    """Pin: gather(shard(x)) is x with its zero pad; unflatten gives back each
    tensor as numpy's reshape of its own row-major run."""
    rnd = random.Random(3)
    rng = np.random.default_rng(3)
    for _ in range(50):
        shapes = [tuple(rnd.randint(1, 6) for _ in range(rnd.randint(1, 3))) for _ in range(rnd.randint(1, 5))]
        tensors = [rand_bf16(rng, int(np.prod(s))).reshape(s) for s in shapes]
        D, A = rnd.randint(1, 8), rnd.choice([1, 4, 8])
        offs, N, N_pad, S = oracle.plan([t.size for t in tensors], D, A)
        x = np.concatenate([t.ravel() for t in tensors])
        padded = np.concatenate([x, np.zeros(N_pad - N, np.uint16)])
        shards = [padded[r * S:(r + 1) * S].copy() for r in range(D)]
        flat = oracle.all_gather(shards, S)
        assert np.array_equal(flat, padded)
        outs = oracle.unflatten(flat, offs, [t.size for t in tensors])
        for o, t in zip(outs, tensors):
            assert np.array_equal(o.reshape(t.shape), t)


def test_workload_inputs_are_seeded_and_padded():
    """The generator gives identical bits for identical keys and zero pads."""
    a = synth.contribution(100, 128, seed=0, step=1, rank=2, sigma=1e-3)
    b = synth.contribution(100, 128, seed=0, step=1, rank=2, sigma=1e-3)
    c = synth.contribution(100, 128, seed=0, step=2, rank=2, sigma=1e-3)
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    assert not torch.equal(a.view(torch.int16), c.view(torch.int16))
    assert not a[100:].view(torch.int16).any()
    t = synth.contribution(20000, 20000, seed=0, step=1, rank=0, sigma=1e-3, dist="student_t", zero_frac=0.01)
    zeros = (t.float() == 0).float().mean().item()
    assert 0.005 < zeros < 0.02
