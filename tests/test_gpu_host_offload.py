"""GPU parity of the CPU-offload step as "7.10 — Fully-sharded data parallel
(FSDP / ZeRO-3)", §8 describes it: the reduce-scatter's reduction alone on the
GPU (zero3_reduce_scatter) against the oracle's reduce-scatter, and the whole
pipeline (gradient down, AdamW on the host, bf16 weights up) against the
oracle's fused step, bit for bit, in both reduce dtypes."""
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


CASES = [([13], 1, 1), ([5, 7, 1], 4, 1), ([999], 5, 1), ([300, 77, 1000], 4, 8), ([4097, 33], 32, 128),
         ([123457], 8, 128), ([2 ** 16 + 3], 64, 8), ([50000], 16, 1), ([70001], 2, 128)]


@pytest.mark.parametrize("mode", [0, 1], ids=["fp32", "bf16"])
@pytest.mark.parametrize("numels,D,A", CASES)
def test_reduce_scatter_matches_oracle(z3, numels, D, A, mode):
    plan, ref = checked_plan(z3, [(k,) for k in numels], D, A)
    N, N_pad, S = ref.N, ref.N_pad, ref.S
    gdt = torch.float32 if mode == 0 else torch.bfloat16
    c = synth.contributions(D, N, N_pad, seed=D, step=1, sigma=1e-3, dist="student_t", zero_frac=0.02,
                            device="cuda")
    host = [synth.bf16_bits(x) for x in c]

    def expect(rank, layout):
        src = host if layout == 0 else [h[rank * S:(rank + 1) * S] for h in host]
        return oracle.reduce_scatter(src, S, rank, layout=layout, reduce_dtype=mode)

    def got_of(g):
        return f32_host(g.t if gdt == torch.float32 else g.t.float())

    for rank, layout, skew in ((-1, 0, 0), (D - 1, 0, 0), (D // 2, 1, 0), (-1, 0, 1), (0, 1, 1)):
        n = N_pad if rank < 0 else S
        src = c if layout == 0 else [x[rank * S:(rank + 1) * S].clone() for x in c]
        gc = [Guarded(x.numel(), torch.bfloat16, skew, fill=x) for x in src]
        g = Guarded(n, gdt, skew)
        z3.zero3_reduce_scatter(plan, rank, [x.t for x in gc], g.t, contrib_layout=layout, reduce_dtype=mode)
        torch.cuda.synchronize()
        assert_f32_parity(got_of(g), expect(rank, layout), f"grad rank={rank} layout={layout} skew={skew}")
        assert g.guards_intact()
        if mode == 1:   # in the bf16 reduce g is a bf16 value: stored exactly
            assert np.array_equal(f32_host(g.t.float()).view(np.uint32) & 0xFFFF, np.zeros(n, np.uint32))


@pytest.mark.parametrize("mode", [0, 1], ids=["fp32", "bf16"])
@pytest.mark.parametrize("numels,D,A,n_stage,chunks", [([300, 77, 1000], 4, 8, 2, 1), ([123457], 8, 128, 1, 4),
                                                       ([4097, 33], 32, 128, 3, 2), ([999], 5, 1, 2, 3),
                                                       ([2 ** 20 + 5], 8, 128, 2, 4), ([2 ** 20 + 5], 8, 128, 3, 7)])
def test_host_adamw_offload_matches_oracle(z3, numels, D, A, n_stage, chunks, mode):
    from fsdp_sharded_mixed_flat_b200.offload import HostAdamWOffload
    plan, ref = checked_plan(z3, [(k,) for k in numels], D, A)
    N, N_pad, S = ref.N, ref.N_pad, ref.S
    p_dev, _, _ = state_init(N, N_pad, 12)
    p = p_dev.cpu().pin_memory()
    m, v = torch.zeros(N_pad).pin_memory(), torch.zeros(N_pad).pin_memory()
    w = torch.zeros(N_pad, dtype=torch.bfloat16, device="cuda")
    off = HostAdamWOffload(plan, p, m, v, w, "cuda", n_stage=n_stage, reduce_dtype=mode, n_threads=4, chunks=chunks)
    assert sum(n for _, _, n in off.units) == N_pad and len(off.units) >= D
    hp_, hm, hv, hw = p.numpy().copy(), np.zeros(N_pad, np.float32), np.zeros(N_pad, np.float32), \
        np.zeros(N_pad, np.uint16)
    for t in range(1, 5):
        c = synth.contributions(D, N, N_pad, seed=12, step=t, sigma=1e-3, device="cuda")
        off.step(c, z3.adamw(**hp_for(t)))
        oracle.reduce_adamw([synth.bf16_bits(x) for x in c], S, -1, hp_, hm, hv, hw, oracle_hp(t),
                            reduce_dtype=mode)
        torch.cuda.synchronize()
        what = f"numels={numels} D={D} mode={mode} step={t}"
        assert_f32_parity(p.numpy(), hp_, "master " + what)
        assert_f32_parity(m.numpy(), hm, "exp_avg " + what)
        assert_f32_parity(v.numpy(), hv, "exp_avg_sq " + what)
        assert_bf16_parity(synth.bf16_bits(w), hw, "work_bf16 " + what)
    assert off.bytes_down == N_pad * (4 if mode == 0 else 2) and off.bytes_up == N_pad * 2


def test_reduce_scatter_composed_with_host_adamw_equals_the_fused_kernel(z3):
    """The two halves composed by hand on the 7B block's first 2^22 elements at
    D = 8 (one rank's partition): the same bits as the fused kernel."""
    n = 1 << 22
    plan, ref = checked_plan(z3, [(n,)], 8, 128)
    S = ref.S
    c = synth.contributions(8, n, ref.N_pad, seed=4, step=1, sigma=1e-4, device="cuda")
    p0 = synth.master_weights(n, ref.N_pad, seed=4, device="cuda")[3 * S:4 * S].clone()
    for mode in (0, 1):
        fp, fm, fv = p0.clone(), torch.zeros_like(p0), torch.zeros_like(p0)
        fw = torch.zeros(S, dtype=torch.bfloat16, device="cuda")
        z3.zero3_reduce_adamw(plan, 3, c, fp, fm, fv, fw, z3.adamw(step=1), reduce_dtype=mode)
        g = torch.empty(S, dtype=torch.float32 if mode == 0 else torch.bfloat16, device="cuda")
        z3.zero3_reduce_scatter(plan, 3, c, g, reduce_dtype=mode)
        torch.cuda.synchronize()
        hp_, hm, hv = p0.cpu(), torch.zeros(S), torch.zeros(S)
        hw = torch.zeros(S, dtype=torch.bfloat16)
        z3.zero3_host_adamw(g.cpu(), hp_, hm, hv, hw, z3.adamw(step=1))
        for a, b in ((fp, hp_), (fm, hm), (fv, hv)):
            assert torch.equal(a.cpu().view(torch.int32), b.view(torch.int32))
        assert torch.equal(fw.cpu().view(torch.int16), hw.view(torch.int16))


@pytest.mark.parametrize("mode", [0, 1], ids=["fp32", "bf16"])
def test_host_adamw_offload_full_size_llama7b_block(z3, mode):
    """The benchmark's offload step at full size: the LLaMA-7B block at D = 8, the
    state in pinned host memory, AdamW on the host, 2 steps; every element of the
    state and of the bf16 weights compared with the oracle on a sample that
    includes every partition boundary."""
    from fsdp_sharded_mixed_flat_b200.offload import HostAdamWOffload
    w = synth.WORKLOADS["llama7b_d8"]
    plan, ref = checked_plan(z3, [s for _, s in w["tensors"]], 8, synth.ALIGN)
    N, N_pad, S = ref.N, ref.N_pad, ref.S
    p = synth.master_weights(N, N_pad, seed=17, device="cuda").cpu().pin_memory()
    m, v = torch.zeros(N_pad).pin_memory(), torch.zeros(N_pad).pin_memory()
    wk = torch.zeros(N_pad, dtype=torch.bfloat16, device="cuda")
    rng = np.random.default_rng(17)
    idx = np.unique(np.concatenate([rng.choice(N_pad, 100_000, replace=False)] +
                                   [np.arange(max(0, r * S - 16), min(N_pad, r * S + 16)) for r in range(9)]))
    ti = torch.from_numpy(idx).cuda()
    hp_, hm, hv = p.numpy()[idx].copy(), np.zeros(idx.size, np.float32), np.zeros(idx.size, np.float32)
    hw = np.zeros(idx.size, np.uint16)
    off = HostAdamWOffload(plan, p, m, v, wk, "cuda", reduce_dtype=mode)
    for t in (1, 2):
        c = synth.contributions(8, N, N_pad, seed=17, step=t, sigma=w["sigma"], device="cuda")
        off.step(c, z3.adamw(**hp_for(t)))
        oracle.reduce_adamw([synth.bf16_bits(x[ti]) for x in c], idx.size, 0, hp_, hm, hv, hw, oracle_hp(t),
                            layout=oracle.LAYOUT_OWNED, reduce_dtype=mode)
        del c
    torch.cuda.synchronize()
    assert_f32_parity(p.numpy()[idx], hp_, "master")
    assert_f32_parity(m.numpy()[idx], hm, "exp_avg")
    assert_f32_parity(v.numpy()[idx], hv, "exp_avg_sq")
    assert_bf16_parity(synth.bf16_bits(wk[ti]), hw, "work_bf16")
