"""GPU parity of the device-scalar kernels and of the CUDA-graph step.

zero3_reduce_adamw_dev reads the step's AdamW scalars from device memory, so a
captured graph can be replayed step after step; GraphedStep captures the ZeRO-3
step (fused kernel, then the gather) or the ZeRO-1/2 step (fused kernel writing
the gathered block) once and replays it.  Both are compared with the oracle,
element by element, over several steps."""
import numpy as np
import pytest
import torch

import oracle
import synth
from parity_util import (assert_bf16_parity, assert_f32_parity, checked_plan, f32_host, hp_for, oracle_hp,
                         state_init)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def z3():
    assert torch.cuda.is_available(), "the GPU tests need a CUDA device"
    from fsdp_sharded_mixed_flat_b200 import build
    build.build()
    from fsdp_sharded_mixed_flat_b200 import zero3
    return zero3


@pytest.mark.parametrize("mode", [0, 1], ids=["fp32", "bf16"])
@pytest.mark.parametrize("numels,D,A,rank", [([300, 77, 1000], 4, 8, -1), ([123457], 8, 128, -1),
                                             ([13], 3, 1, -1), ([4097, 33], 32, 128, 5), ([999], 5, 1, 2)])
def test_device_scalars_match_oracle(z3, numels, D, A, rank, mode):
    plan, ref = checked_plan(z3, [(k,) for k in numels], D, A)
    N, N_pad, S = ref.N, ref.N_pad, ref.S
    n = N_pad if rank < 0 else S
    p_full, _, _ = state_init(N, N_pad, 3)
    p = (p_full if rank < 0 else p_full[rank * S:(rank + 1) * S]).clone()
    m, v = torch.zeros_like(p), torch.zeros_like(p)
    w = torch.zeros(n, dtype=torch.bfloat16, device="cuda")
    g = torch.full((N_pad,), 7.0, dtype=torch.bfloat16, device="cuda")
    sc = torch.zeros(z3.Z3_SCALARS, dtype=torch.float32, device="cuda")
    hp_, hm, hv, hw = f32_host(p).copy(), np.zeros(n, np.float32), np.zeros(n, np.float32), np.zeros(n, np.uint16)
    for t in range(1, 5):
        c = synth.contributions(D, N, N_pad, seed=3, step=t, sigma=1e-3, device="cuda")
        sc.copy_(torch.tensor(z3.zero3_step_scalars(z3.adamw(**hp_for(t))), dtype=torch.float32))
        z3.zero3_reduce_adamw_dev(plan, rank, c, p, m, v, w, [g], sc, reduce_dtype=mode)
        oracle.reduce_adamw([synth.bf16_bits(x) for x in c], S, rank, hp_, hm, hv, hw, oracle_hp(t),
                            reduce_dtype=mode)
    torch.cuda.synchronize()
    assert_f32_parity(f32_host(p), hp_, "master")
    assert_f32_parity(f32_host(m), hm, "exp_avg")
    assert_f32_parity(f32_host(v), hv, "exp_avg_sq")
    assert_bf16_parity(synth.bf16_bits(w), hw, "work_bf16")
    lo = 0 if rank < 0 else rank * S
    assert_bf16_parity(synth.bf16_bits(g)[lo:lo + n], hw, "gathered")


@pytest.mark.parametrize("stage", [3, 2])
@pytest.mark.parametrize("mode", [0, 1], ids=["fp32", "bf16"])
def test_graphed_step_matches_oracle(z3, stage, mode):
    from fsdp_sharded_mixed_flat_b200.graph import GraphedStep
    w_ = synth.WORKLOADS["tiny_gpt"]
    shapes = [s for _, s in w_["tensors"]]
    plan, ref = checked_plan(z3, shapes, w_["D"], synth.ALIGN)
    N, N_pad, S, D = ref.N, ref.N_pad, ref.S, plan.D
    p, m, v = state_init(N, N_pad, 0)
    work = torch.zeros(N_pad, dtype=torch.bfloat16, device="cuda") if stage == 3 else None
    flat = torch.zeros(N_pad, dtype=torch.bfloat16, device="cuda")
    contribs = [torch.zeros(N_pad, dtype=torch.bfloat16, device="cuda") for _ in range(D)]
    gs = GraphedStep(plan, contribs, p, m, v, work, flat, stage=stage, reduce_dtype=mode)
    hp_, hm, hv, hw = f32_host(p).copy(), np.zeros(N_pad, np.float32), np.zeros(N_pad, np.float32), \
        np.zeros(N_pad, np.uint16)
    for t in range(1, 8):
        fresh = synth.contributions(D, N, N_pad, seed=0, step=t, sigma=w_["sigma"], device="cuda")
        for c, f in zip(contribs, fresh):
            c.copy_(f)                        # the graph reads the same buffers every step
        gs.step(z3.adamw(**hp_for(t)))
        oracle.reduce_adamw([synth.bf16_bits(x) for x in fresh], S, -1, hp_, hm, hv, hw, oracle_hp(t),
                            reduce_dtype=mode)
    torch.cuda.synchronize()
    assert_f32_parity(f32_host(p), hp_, "master")
    assert_f32_parity(f32_host(m), hm, "exp_avg")
    assert_f32_parity(f32_host(v), hv, "exp_avg_sq")
    if work is not None:
        assert_bf16_parity(synth.bf16_bits(work), hw, "work_bf16")
    ref_flat = oracle.all_gather([hw[r * S:(r + 1) * S] for r in range(D)], S)
    assert np.array_equal(synth.bf16_bits(flat), ref_flat)


def test_graph_ring_wraps(z3):
    """More steps than the ring of pinned scalar slots: the slots are reused safely."""
    from fsdp_sharded_mixed_flat_b200 import graph
    plan = z3.zero3_plan([(4096,)], 2, 8)
    p, m, v = state_init(plan.N, plan.N_pad, 1)
    flat = torch.zeros(plan.N_pad, dtype=torch.bfloat16, device="cuda")
    c = synth.contributions(2, plan.N, plan.N_pad, seed=1, step=1, sigma=1e-3, device="cuda")
    ref = [p.clone(), m.clone(), v.clone()]
    refw = torch.zeros_like(flat)
    gs = graph.GraphedStep(plan, c, p, m, v, None, flat, stage=2)
    steps = graph.RING + 5
    for t in range(1, steps + 1):
        gs.step(z3.adamw(step=t))
        z3.zero3_reduce_adamw(plan, -1, c, *ref, refw, z3.adamw(step=t))
    torch.cuda.synchronize()
    assert torch.equal(p, ref[0]) and torch.equal(m, ref[1]) and torch.equal(v, ref[2])
    assert torch.equal(flat.view(torch.int16), refw.view(torch.int16))
