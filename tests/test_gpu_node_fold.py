"""GPU parity of HYBRID_SHARD's two halves for separate nodes (zero3_node_sum,
zero3_fold_adamw) against the oracle, through the C ABI, on the same seeded
inputs: every element, several rank and node counts (specialised and generic
kernels), single ranks and all ranks, both layouts and reduce dtypes,
misaligned buffers (scalar kernels), canary bands around every buffer.  At
full size, the composition (four node sums, then the fold) must equal the
fused HYBRID_SHARD kernel byte for byte on the 7B block over 4 nodes of 8."""
import numpy as np
import pytest
import torch

import oracle
import synth
from parity_util import checked_plan, f32_host, Guarded, hp_for, oracle_hp, state_init

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def z3():
    assert torch.cuda.is_available(), "the GPU tests need a CUDA device"
    from fsdp_sharded_mixed_flat_b200 import build
    build.build()
    from fsdp_sharded_mixed_flat_b200 import zero3
    return zero3


def sum_bits(t: torch.Tensor) -> np.ndarray:
    """Node sums (float32 or bf16 on the device) as float32 bit patterns."""
    return t.float().cpu().numpy().view(np.uint32)


@pytest.mark.parametrize("mode", [0, 1], ids=["fp32", "bf16"])
@pytest.mark.parametrize("numels,D,A,skew", [
    ([5000, 77], 8, 128, 0), ([123457], 4, 8, 0), ([3000, 17], 3, 8, 0), ([9999], 16, 8, 0),
    ([4097, 33], 32, 128, 0), ([2 ** 12 + 5], 64, 8, 0), ([777], 1, 1, 0), ([5000, 77], 8, 8, 1),
])
def test_node_sum_matches_oracle(z3, numels, D, A, skew, mode):
    plan, ref = checked_plan(z3, [(k,) for k in numels], D, A)
    N, N_pad, S = ref.N, ref.N_pad, ref.S
    c = synth.contributions(D, N, N_pad, seed=D, step=1, sigma=1e-3, dist="student_t", zero_frac=0.02,
                            device="cuda")
    dt = torch.float32 if mode == 0 else torch.bfloat16
    for rank, layout in ((-1, 0), (D // 2, 0), (D - 1, 1)):
        n = N_pad if rank < 0 else S
        src = c if layout == 0 else [x[rank * S:(rank + 1) * S].clone() for x in c]
        gc = [Guarded(x.numel(), torch.bfloat16, skew, fill=x) for x in src]
        out = Guarded(n, dt, skew)
        z3.zero3_node_sum(plan, rank, [g.t for g in gc], out.t, contrib_layout=layout, reduce_dtype=mode)
        want = oracle.node_sum([synth.bf16_bits(x) for x in src], S, rank, layout, mode)
        torch.cuda.synchronize()
        assert np.array_equal(sum_bits(out.t), want.view(np.uint32)), (numels, D, rank, layout, mode)
        assert out.guards_intact() and all(g.guards_intact() for g in gc)


@pytest.mark.parametrize("mode", [0, 1], ids=["fp32", "bf16"])
@pytest.mark.parametrize("R,skew", [(1, 0), (2, 0), (3, 0), (4, 0), (8, 0), (16, 0), (4, 1)])
def test_fold_adamw_matches_oracle(z3, R, skew, mode):
    D = 4
    plan, ref = checked_plan(z3, [(20000,), (4097,)], D, 8)
    N, N_pad, S = ref.N, ref.N_pad, ref.S
    dt = torch.float32 if mode == 0 else torch.bfloat16
    for rank in (-1, 2):
        n = N_pad if rank < 0 else S
        p_full, _, _ = state_init(N, N_pad, R)
        p0 = p_full if rank < 0 else p_full[rank * S:(rank + 1) * S]
        gp = Guarded(n, torch.float32, skew, fill=p0)
        gm = Guarded(n, torch.float32, 0, fill=torch.zeros(n, device="cuda"))
        gv = Guarded(n, torch.float32, skew, fill=torch.zeros(n, device="cuda"))
        gw = Guarded(n, torch.bfloat16, 0, fill=torch.zeros(n, device="cuda", dtype=torch.bfloat16))
        hp_, hm, hv, hw = f32_host(p0).copy(), np.zeros(n, np.float32), np.zeros(n, np.float32), \
            np.zeros(n, np.uint16)
        for t in (1, 2, 3):
            # node sums as a node would send them: any fp32 value, or a bf16 value in bf16 mode
            sums = []
            for k in range(R):
                gen = torch.Generator(device="cuda").manual_seed(100 * t + k)
                x = torch.randn(n, device="cuda", generator=gen) * 4e-3
                sums.append(Guarded(n, dt, skew, fill=x.to(dt)))
            z3.zero3_fold_adamw(plan, rank, [g.t for g in sums], gp.t, gm.t, gv.t, gw.t, z3.adamw(**hp_for(t)),
                                reduce_dtype=mode)
            oracle.fold_adamw([g.t.float().cpu().numpy() for g in sums], D, hp_, hm, hv, hw, oracle_hp(t),
                              reduce_dtype=mode)
            torch.cuda.synchronize()
            what = f"R={R} rank={rank} mode={mode} skew={skew} step={t}"
            assert np.array_equal(f32_host(gp.t).view(np.uint32), hp_.view(np.uint32)), "master " + what
            assert np.array_equal(f32_host(gm.t).view(np.uint32), hm.view(np.uint32)), "exp_avg " + what
            assert np.array_equal(f32_host(gv.t).view(np.uint32), hv.view(np.uint32)), "exp_avg_sq " + what
            assert np.array_equal(synth.bf16_bits(gw.t), hw), "work " + what
            assert all(g.guards_intact() for g in (gp, gm, gv, gw, *sums)), "canary " + what


@pytest.mark.parametrize("mode", [0, 1], ids=["fp32", "bf16"])
def test_node_sums_then_fold_equal_the_fused_hybrid_kernel_at_full_size(z3, mode):
    """The 7B block over 4 nodes of 8, all partitions in one launch, 3 steps:
    four node sums, then the fold, against the fused HYBRID_SHARD kernel."""
    w = synth.WORKLOADS["llama7b_hybrid"]
    R, D = w["nodes"], w["D"]
    plan, ref = checked_plan(z3, [s for _, s in w["tensors"]], D, synth.ALIGN)
    N, N_pad = ref.N, ref.N_pad
    dt = torch.float32 if mode == 0 else torch.bfloat16
    a = list(state_init(N, N_pad, 3)) + [torch.zeros(N_pad, dtype=torch.bfloat16, device="cuda")]
    b = [x.clone() for x in a]
    sums = [torch.empty(N_pad, dtype=dt, device="cuda") for _ in range(R)]
    for t in (1, 2, 3):
        c = synth.contributions(R * D, N, N_pad, seed=3, step=t, sigma=w["sigma"], device="cuda")
        z3.zero3_reduce_adamw_hybrid(plan, -1, R, c, *a, z3.adamw(**hp_for(t)), reduce_dtype=mode)
        for k in range(R):
            z3.zero3_node_sum(plan, -1, c[k * D:(k + 1) * D], sums[k], reduce_dtype=mode)
        z3.zero3_fold_adamw(plan, -1, sums, *b, z3.adamw(**hp_for(t)), reduce_dtype=mode)
        del c
    torch.cuda.synchronize()
    for x, y in zip(a, b):
        assert torch.equal(x.view(torch.int16), y.view(torch.int16))
