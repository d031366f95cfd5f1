"""GPU parity of the backward sweep with the next block's all-gather prefetched
into one of two transient buffers ("7.10 — Fully-sharded data parallel
(FSDP / ZeRO-3)", §5.1, §5.2, §5.4): every block's gathered weights, as the
block sees them, equal the oracle's all-gather of that block's shards at that
point of the sweep, and this rank's state and shards equal the oracle's
update, bit for bit, over several sweeps, with and without the prefetch."""
import numpy as np
import pytest
import torch

import oracle
import synth
from parity_util import assert_bf16_parity, assert_f32_parity, checked_plan, f32_host, hp_for, oracle_hp

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def z3():
    assert torch.cuda.is_available(), "the GPU tests need a CUDA device"
    from fsdp_sharded_mixed_flat_b200 import build
    build.build()
    from fsdp_sharded_mixed_flat_b200 import zero3
    return zero3


def owned_contribs(S, D, layer, step, device):
    return [synth.contribution(S, S, seed=100 + layer, step=step, rank=d, sigma=1e-3, device=device) for d in range(D)]


@pytest.mark.parametrize("prefetch", [True, False], ids=["prefetch", "serial"])
@pytest.mark.parametrize("shapes,D,A,L,rank,mode", [([(300,), (77, 13), (1000,)], 4, 8, 5, 1, 0),
                                                    ([(4097,), (33,)], 8, 128, 4, 7, 1),
                                                    ([(65, 256), (256, 768)], 3, 16, 3, 0, 0),
                                                    ([(5000,)], 2, 1, 1, 1, 1)])
def test_prefetched_sweep_matches_oracle(z3, shapes, D, A, L, rank, mode, prefetch):
    from fsdp_sharded_mixed_flat_b200.stream import PrefetchSweep
    plan, ref = checked_plan(z3, shapes, D, A)
    S, N_pad = ref.S, ref.N_pad
    gen = torch.Generator().manual_seed(L * D)
    host_shards = [[torch.randint(-32768, 32768, (S,), generator=gen, dtype=torch.int32).to(torch.int16)
                    .numpy().view(np.uint16).copy() for _ in range(D)] for _ in range(L)]
    shards = [[synth.bits_to_bf16(h, "cuda") for h in blk] for blk in host_shards]
    master = synth.master_weights(L * S, L * S, seed=9, device="cuda")
    m, v = torch.zeros_like(master), torch.zeros_like(master)
    hp_ = [f32_host(master[l * S:(l + 1) * S]).copy() for l in range(L)]
    hm = [np.zeros(S, np.float32) for _ in range(L)]
    hv = [np.zeros(S, np.float32) for _ in range(L)]
    sweep = PrefetchSweep(plan, shards, rank, master, m, v, reduce_dtype=mode)
    assert sweep.transient_bytes == 2 * 2 * N_pad
    seen = [torch.empty(N_pad, dtype=torch.bfloat16, device="cuda") for _ in range(L)]
    for t in range(1, 4):
        contribs = {l: owned_contribs(S, D, l, t, "cuda") for l in range(L)}
        sweep.step(lambda l: contribs[l], z3.adamw(**hp_for(t)),
                   consume=lambda l, buf: seen[l].copy_(buf), prefetch=prefetch)
        torch.cuda.synchronize()
        for l in range(L - 1, -1, -1):
            # the block's gathered weights are its shards as they stood before its update
            want = oracle.all_gather(host_shards[l], S)
            assert np.array_equal(synth.bf16_bits(seen[l]), want), f"gathered block {l} step {t}"
            new_w = np.zeros(S, np.uint16)
            oracle.reduce_adamw([synth.bf16_bits(c) for c in contribs[l]], S, rank, hp_[l], hm[l], hv[l], new_w,
                                oracle_hp(t), layout=oracle.LAYOUT_OWNED, reduce_dtype=mode)
            host_shards[l][rank] = new_w
        for l in range(L):
            sl = slice(l * S, (l + 1) * S)
            what = f"block {l} step {t}"
            assert_f32_parity(f32_host(master[sl]), hp_[l], "master " + what)
            assert_f32_parity(f32_host(m[sl]), hm[l], "exp_avg " + what)
            assert_f32_parity(f32_host(v[sl]), hv[l], "exp_avg_sq " + what)
            for d in range(D):
                assert_bf16_parity(synth.bf16_bits(shards[l][d]), host_shards[l][d], f"shard {d} " + what)


def test_prefetched_sweep_full_size_llama7b_blocks(z3):
    """The benchmark's sweep at full block size: 3 LLaMA-7B blocks at D = 8, rank 0,
    two sweeps.  Every gathered block (202,383,360 elements) equals the oracle's
    all-gather of that block's shards at that point, in full; the rank's state and
    shard equal the oracle's on a sample that includes every partition boundary."""
    from fsdp_sharded_mixed_flat_b200.stream import PrefetchSweep
    w = synth.WORKLOADS["llama7b_d8"]
    D, L, rank = 8, 3, 0
    plan, ref = checked_plan(z3, [s for _, s in w["tensors"]], D, synth.ALIGN)
    S, N_pad = ref.S, ref.N_pad
    g = torch.Generator(device="cuda").manual_seed(41)
    flat_all = torch.randint(-32768, 32768, (L * N_pad,), generator=g, device="cuda",
                             dtype=torch.int32).to(torch.int16).view(torch.bfloat16)
    shards = [[flat_all[l * N_pad + d * S:l * N_pad + (d + 1) * S] for d in range(D)] for l in range(L)]
    master = synth.master_weights(L * S, L * S, seed=41, device="cuda")
    m, v = torch.zeros_like(master), torch.zeros_like(master)
    rng = np.random.default_rng(41)
    idx = torch.from_numpy(np.unique(np.concatenate([rng.choice(S, 20_000, replace=False),
                                                     np.arange(64), np.arange(S - 64, S)]))).cuda()
    hp_ = [f32_host(master[l * S:(l + 1) * S][idx]).copy() for l in range(L)]
    hm = [np.zeros(idx.numel(), np.float32) for _ in range(L)]
    hv = [np.zeros(idx.numel(), np.float32) for _ in range(L)]
    hw = [np.zeros(idx.numel(), np.uint16) for _ in range(L)]
    sweep = PrefetchSweep(plan, shards, rank, master, m, v)
    for t in (1, 2):
        contribs = {l: owned_contribs(S, D, l, t, "cuda") for l in range(L)}
        before = [[synth.bf16_bits(x) for x in blk] for blk in shards]       # the shards each block gathers
        seen = {}
        sweep.step(lambda l: contribs[l], z3.adamw(**hp_for(t)),
                   consume=lambda l, buf: seen.__setitem__(l, buf.clone()))
        torch.cuda.synchronize()
        for l in range(L):
            assert np.array_equal(synth.bf16_bits(seen[l]), oracle.all_gather(before[l], S)), f"block {l} step {t}"
            sub = [synth.bf16_bits(c[idx]) for c in contribs[l]]
            oracle.reduce_adamw(sub, idx.numel(), 0, hp_[l], hm[l], hv[l], hw[l], oracle_hp(t),
                                layout=oracle.LAYOUT_OWNED)
            sl = slice(l * S, (l + 1) * S)
            what = f"block {l} step {t}"
            assert_f32_parity(f32_host(master[sl][idx]), hp_[l], "master " + what)
            assert_f32_parity(f32_host(m[sl][idx]), hm[l], "exp_avg " + what)
            assert_f32_parity(f32_host(v[sl][idx]), hv[l], "exp_avg_sq " + what)
            assert_bf16_parity(synth.bf16_bits(shards[l][rank][idx]), hw[l], "shard " + what)
        del contribs, seen
