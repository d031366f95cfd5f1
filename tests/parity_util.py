"""Helpers shared by the GPU parity tests: guarded device buffers, the
comparison rules, and the runs of the CUDA path and of the oracle on the same
seeded inputs.

Comparison rules (the tolerances this path is held to):
  fp32 master / m / v: max relative error <= 1e-6 per element, with
      rel = |x - y| / max(|y|, FLT_MIN), so an expected 0 must come out 0;
  bf16 working weights and every gathered byte: within 1 bf16 ulp (weights)
      and bit-exact (layout, gather, unflatten).
The kernels follow the oracle's operation order with explicitly rounded fp32
operations, so the tests also assert the stronger bit-exact result.
"""
import numpy as np
import torch

import oracle
import synth

FLT_MIN = np.float32(1.1754944e-38)
REL_TOL = 1e-6
GUARD = 64  # canary elements before and after every device buffer


class Guarded:
    """A device buffer of n elements with canary bands of GUARD elements on each
    side; `t` is the interior (offset by `skew` extra elements to misalign it)."""

    def __init__(self, n: int, dtype: torch.dtype, skew: int = 0, fill=None):
        self.n, self.skew = n, skew
        self.base = torch.empty(n + 2 * GUARD + skew, dtype=dtype, device="cuda")
        pattern = torch.tensor(0x5A5A5A5A if dtype == torch.float32 else 0x5A5A,
                               dtype=torch.int32 if dtype == torch.float32 else torch.int16)
        self.base.view(pattern.dtype).fill_(pattern.item())
        self.t = self.base[GUARD + skew: GUARD + skew + n]
        if fill is not None:
            self.t.copy_(fill)

    def guards_intact(self) -> bool:
        raw = self.base.view(torch.int32 if self.base.dtype == torch.float32 else torch.int16)
        want = 0x5A5A5A5A if self.base.dtype == torch.float32 else 0x5A5A
        head = raw[:GUARD + self.skew]
        tail = raw[GUARD + self.skew + self.n:]
        return bool((head == want).all().item() and (tail == want).all().item())


def f32_host(t: torch.Tensor) -> np.ndarray:
    return t.detach().contiguous().cpu().numpy().astype(np.float32, copy=False)


def assert_f32_parity(got: np.ndarray, ref: np.ndarray, what: str, exact: bool = True):
    got = np.asarray(got, dtype=np.float32)
    ref = np.asarray(ref, dtype=np.float32)
    assert got.shape == ref.shape
    rel = np.abs(got.astype(np.float64) - ref) / np.maximum(np.abs(ref.astype(np.float64)), FLT_MIN)
    worst = float(rel.max()) if rel.size else 0.0
    assert worst <= REL_TOL, f"{what}: max relative error {worst:.3e} > {REL_TOL}"
    if exact:
        diff = int(np.count_nonzero(got.view(np.uint32) != ref.view(np.uint32)))
        assert diff == 0, f"{what}: {diff} of {got.size} elements differ in their bits"


def bf16_ulp_distance(a: np.ndarray, b: np.ndarray) -> np.ndarray:
    """Distance in bf16 ulps between bit patterns (sign-magnitude -> ordered ints)."""
    def ordered(x):
        x = x.astype(np.int32)
        return np.where(x & 0x8000, 0x8000 - (x & 0x7FFF), 0x8000 + (x & 0x7FFF))
    return np.abs(ordered(a) - ordered(b))


def assert_bf16_parity(got: np.ndarray, ref: np.ndarray, what: str, exact: bool = True):
    assert got.shape == ref.shape
    d = bf16_ulp_distance(got, ref)
    worst = int(d.max()) if d.size else 0
    assert worst <= 1, f"{what}: {worst} bf16 ulps apart"
    if exact:
        n = int(np.count_nonzero(got != ref))
        assert n == 0, f"{what}: {n} of {got.size} bf16 values differ"


class RefPlan:
    """The oracle's plan of a tensor list: offsets, numels, N, N_pad, S."""

    def __init__(self, shapes, D: int, A: int):
        self.numels = [synth.numel(s) for s in shapes]
        offs, self.N, self.N_pad, self.S = oracle.plan(self.numels, D, A)
        self.offsets = [int(o) for o in offs]
        self.D = D


def checked_plan(z3, shapes, D: int, A: int):
    """The product's plan and the oracle's plan of the same tensor list, after
    asserting that they agree on every offset, numel, N, N_pad and S.  Expected
    values are built from the oracle's plan only, so a planner mistake cannot
    make the kernel and its expected value agree."""
    plan = z3.zero3_plan(shapes, D, A)
    ref = RefPlan(shapes, D, A)
    assert (plan.N, plan.N_pad, plan.S) == (ref.N, ref.N_pad, ref.S), \
        f"plan sizes {(plan.N, plan.N_pad, plan.S)} != oracle {(ref.N, ref.N_pad, ref.S)}"
    assert list(plan.offsets) == ref.offsets, "tensor offsets differ from the oracle's plan"
    assert list(plan.numels) == ref.numels, "tensor sizes differ from the oracle's plan"
    return plan, ref


def state_init(n_real: int, n_pad: int, seed: int):
    """fp32 master (zero pad) and zero moments, on the device."""
    p = synth.master_weights(n_real, n_pad, seed=seed, device="cuda")
    return p, torch.zeros_like(p), torch.zeros_like(p)


def hp_for(step: int):
    return dict(synth.ADAMW, step=step)


def oracle_hp(step: int):
    a = synth.ADAMW
    return oracle.hp(a["lr"], a["beta1"], a["beta2"], a["eps"], a["weight_decay"], step)
