"""The usage example (fsdp_sharded_mixed_flat_b200/example.py, the code the
project's overview shows) run on the GPU, then checked: its final master
weights, gathered block and views against the oracle on the same inputs (ten
steps, every element), with the expected layout taken from the oracle's plan."""
import numpy as np
import pytest
import torch

import oracle
import synth

pytestmark = pytest.mark.gpu


def test_usage_example_runs_and_matches_the_oracle():
    assert torch.cuda.is_available(), "the GPU tests need a CUDA device"
    from fsdp_sharded_mixed_flat_b200 import build
    build.build()
    from fsdp_sharded_mixed_flat_b200 import example
    out = example.run(steps=10, seed=1234)
    plan, grads, flat, weights, shapes = out["plan"], out["grads"], out["flat"], out["weights"], out["shapes"]
    numels = [synth.numel(s) for s in shapes]
    offsets, N, N_pad, S = oracle.plan(numels, 8, 128)
    assert (plan.N, plan.N_pad, plan.S) == (N, N_pad, S)
    # replay the example's draws from the same seed: its inputs are reproduced exactly
    torch.manual_seed(1234)
    g0 = [torch.zeros(N_pad, dtype=torch.bfloat16, device="cuda") for _ in range(8)]
    for g in g0:
        g[:N] = torch.randn(N, device="cuda") * 1e-3
    p0 = torch.zeros(N_pad, device="cuda")
    p0[:N] = torch.randn(N, device="cuda") * 0.02
    for a, b in zip(g0, grads):
        assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    hp_, hm, hv = p0.cpu().numpy().copy(), np.zeros(N_pad, np.float32), np.zeros(N_pad, np.float32)
    hw = np.zeros(N_pad, np.uint16)
    c = [synth.bf16_bits(g) for g in grads]
    for t in range(1, 11):
        oracle.reduce_adamw(c, S, -1, hp_, hm, hv, hw, oracle.hp(3e-4, 0.9, 0.95, 1e-8, 0.1, t))
    torch.cuda.synchronize()
    assert np.array_equal(out["master"].cpu().numpy().view(np.uint32), hp_.view(np.uint32))
    ref_flat = oracle.all_gather([hw[r * S:(r + 1) * S] for r in range(8)], S)
    assert np.array_equal(synth.bf16_bits(flat), ref_flat)
    for view, shape, ref in zip(weights, shapes, oracle.unflatten(ref_flat, offsets, numels)):
        assert tuple(view.shape) == tuple(shape)
        assert np.array_equal(synth.bf16_bits(view).ravel(), ref)
