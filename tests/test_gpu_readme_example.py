"""The README's usage example, run as written on the GPU, then checked: its
final master weights and gathered views against the oracle on the same
inputs (ten steps, every element)."""
import os
import re

import numpy as np
import pytest
import torch

import oracle
import synth

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def readme_example() -> str:
    text = open(os.path.join(ROOT, "README.md")).read()
    section = text[text.index("## Use"):]
    return re.search(r"```python\n(.*?)```", section, re.S).group(1)


def test_readme_example_runs_and_matches_the_oracle():
    assert torch.cuda.is_available(), "the GPU tests need a CUDA device"
    from fsdp_sharded_mixed_flat_b200 import build
    build.build()
    code = readme_example()
    # record the example's inputs: the same seed before running it, then replay the draws
    torch.manual_seed(1234)
    ns = {}
    exec(compile(code, "README.md", "exec"), ns)
    plan, grads, flat, weights = ns["plan"], ns["grads"], ns["flat"], ns["weights"]
    torch.manual_seed(1234)
    g0 = [torch.zeros(plan.N_pad, dtype=torch.bfloat16, device="cuda") for _ in range(plan.D)]
    for g in g0:
        g[:plan.N] = torch.randn(plan.N, device="cuda") * 1e-3
    p0 = torch.zeros(plan.N_pad, device="cuda")
    p0[:plan.N] = torch.randn(plan.N, device="cuda") * 0.02
    for a, b in zip(g0, grads):                          # the replay reproduces the example's inputs
        assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    hp_, hm, hv = p0.cpu().numpy().copy(), np.zeros(plan.N_pad, np.float32), np.zeros(plan.N_pad, np.float32)
    hw = np.zeros(plan.N_pad, np.uint16)
    c = [synth.bf16_bits(g) for g in grads]
    for t in range(1, 11):
        oracle.reduce_adamw(c, plan.S, -1, hp_, hm, hv, hw, oracle.hp(3e-4, 0.9, 0.95, 1e-8, 0.1, t))
    assert np.array_equal(ns["master"].cpu().numpy().view(np.uint32), hp_.view(np.uint32))
    assert np.array_equal(synth.bf16_bits(flat), hw)
    for view, shape, off, n in zip(weights, ns["shapes"], plan.offsets, plan.numels):
        assert tuple(view.shape) == tuple(shape)
        assert np.array_equal(synth.bf16_bits(view).ravel(), hw[off:off + n])
