"""GPU parity of the all-gather / unflatten kernels against the oracle, through
the C ABI: bit-exact flat blocks and per-tensor copies for random plans
(ragged tensors at every offset residue, odd rank counts, alignments 1..128),
misaligned shards and destinations (scalar paths), more segments than one
launch carries, skipped tensors, canary bands, and the full-size 7B block."""
import random

import numpy as np
import pytest
import torch

import oracle
import synth
from parity_util import Guarded, checked_plan

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def z3():
    assert torch.cuda.is_available(), "the GPU tests need a CUDA device"
    from fsdp_sharded_mixed_flat_b200 import build
    build.build()
    from fsdp_sharded_mixed_flat_b200 import zero3
    return zero3


def random_bits(n: int, gen: torch.Generator) -> torch.Tensor:
    return torch.randint(-32768, 32768, (n,), generator=gen, dtype=torch.int32).to(torch.int16) \
        .view(torch.bfloat16).cuda()


def run_gather(z3, shapes, D, A, shard_skew=0, dst_skews=None, skip=(), with_flat=True, seed=0):
    plan, ref = checked_plan(z3, shapes, D, A)
    S, N_pad = ref.S, ref.N_pad
    gen = torch.Generator().manual_seed(seed)
    shards = [Guarded(S, torch.bfloat16, shard_skew, fill=random_bits(S, gen)) for _ in range(D)]
    flat = Guarded(N_pad, torch.bfloat16, 0) if with_flat else None
    dst_skews = dst_skews or [0] * len(shapes)
    outs = [None if i in skip else Guarded(ref.numels[i], torch.bfloat16, dst_skews[i]) for i in range(len(shapes))]
    z3.zero3_gather_block(plan, [s.t for s in shards], None if flat is None else flat.t,
                          [None if o is None else o.t for o in outs])
    torch.cuda.synchronize()
    host_shards = [synth.bf16_bits(s.t) for s in shards]
    ref_flat = oracle.all_gather(host_shards, S)
    if flat is not None:
        assert np.array_equal(synth.bf16_bits(flat.t), ref_flat)
        assert flat.guards_intact()
    ref_t = oracle.unflatten(ref_flat, ref.offsets, ref.numels)
    for i, (o, r) in enumerate(zip(outs, ref_t)):
        if o is None:
            continue
        assert np.array_equal(synth.bf16_bits(o.t), r), f"tensor {i} (offset {ref.offsets[i]})"
        assert o.guards_intact(), f"canary of tensor {i}"
    for s in shards:
        assert s.guards_intact()
    return plan


def random_shapes(rnd, n_tensors, max_numel):
    return [(rnd.randint(1, max_numel),) if rnd.random() < 0.5 else
            (rnd.randint(1, 40), rnd.randint(1, max_numel // 40 + 1)) for _ in range(n_tensors)]


@pytest.mark.parametrize("seed", range(12))
def test_random_plans(z3, seed):
    rnd = random.Random(seed)
    shapes = random_shapes(rnd, rnd.randint(1, 9), 5000)
    D = rnd.choice([1, 2, 3, 4, 5, 8, 16, 32, 64])
    A = rnd.choice([1, 2, 8, 16, 128])
    run_gather(z3, shapes, D, A, dst_skews=[rnd.randint(0, 7) for _ in shapes], seed=seed)


@pytest.mark.parametrize("shard_skew", [1, 3])
def test_misaligned_shards_scalar_path(z3, shard_skew):
    run_gather(z3, [(1000,), (77, 13), (4096,)], 4, 8, shard_skew=shard_skew, dst_skews=[0, 1, 2])


def test_partition_not_multiple_of_8(z3):
    plan = run_gather(z3, [(1001,), (33,)], 3, 1, dst_skews=[0, 5])
    assert plan.S % 8 != 0


def test_every_destination_offset_residue(z3):
    # tensors of 1..17 elements make every offset residue mod 8 appear on both sides
    shapes = [(k,) for k in range(1, 18)] + [(5000,)]
    for skew in range(8):
        run_gather(z3, shapes, 4, 8, dst_skews=[skew] * len(shapes))


def test_more_segments_than_one_launch_carries(z3):
    rnd = random.Random(99)
    shapes = [(rnd.randint(1, 300),) for _ in range(400)]
    run_gather(z3, shapes, 4, 8, with_flat=False, dst_skews=[rnd.randint(0, 7) for _ in shapes])


def test_skipped_tensors_and_flat_only(z3):
    run_gather(z3, [(100,), (200,), (300,)], 2, 8, skip={1})
    plan = z3.zero3_plan([(500,)], 4, 8)
    shards = [torch.ones(plan.S, dtype=torch.bfloat16, device="cuda") * r for r in range(4)]
    flat = torch.empty(plan.N_pad, dtype=torch.bfloat16, device="cuda")
    z3.zero3_gather_block(plan, shards, flat)
    torch.cuda.synchronize()
    assert torch.equal(flat, torch.cat(shards))


def test_worked_example_all_gather(z3, golden):
    """The 4-GPU all-gather of page 3: [A], [B], [C], [D] -> [A, B, C, D]."""
    g = golden("allgather_worked_example.json")
    shards = [torch.tensor(s, dtype=torch.float32).to(torch.bfloat16).cuda() for s in g["shards"]]
    plan = z3.zero3_plan([(len(g["expected_block"]),)], 4, 1)
    flat = torch.empty(plan.N_pad, dtype=torch.bfloat16, device="cuda")
    z3.zero3_gather_block(plan, shards, flat)
    torch.cuda.synchronize()
    assert flat.float().cpu().tolist() == g["expected_block"]


def test_llama7b_block_full_size(z3):
    """The benchmark's gather: 8 shards of the 7B block into the flat block and
    the 9 separate tensors, every element compared."""
    w = synth.WORKLOADS["llama7b_d8"]
    shapes = [s for _, s in w["tensors"]]
    plan, ref = checked_plan(z3, shapes, 8, synth.ALIGN)
    S = ref.S
    gen = torch.Generator(device="cuda").manual_seed(5)
    work = torch.randint(-32768, 32768, (ref.N_pad,), generator=gen, device="cuda",
                         dtype=torch.int32).to(torch.int16).view(torch.bfloat16)
    flat = torch.empty(ref.N_pad, dtype=torch.bfloat16, device="cuda")
    outs = [torch.empty(s, dtype=torch.bfloat16, device="cuda") for s in shapes]
    z3.zero3_gather_block(plan, [work[r * S:(r + 1) * S] for r in range(8)], flat, outs)
    torch.cuda.synchronize()
    host = synth.bf16_bits(work)
    ref_flat = oracle.all_gather([host[r * S:(r + 1) * S] for r in range(8)], S)
    assert np.array_equal(synth.bf16_bits(flat), ref_flat)
    ref_t = oracle.unflatten(ref_flat, ref.offsets, ref.numels)
    for o, r in zip(outs, ref_t):
        assert np.array_equal(synth.bf16_bits(o).ravel(), r)
    for view, r in zip(plan.views(flat), ref_t):                 # the zero-copy unflatten
        assert np.array_equal(synth.bf16_bits(view).ravel(), r)


@pytest.mark.parametrize("own", [[2], [0, 3], [0, 1, 2, 3]])
def test_shards_in_place_inside_the_block(z3, own):
    """A shard that already sits at its place in the block (shards[r] is the view
    flat[r*S:(r+1)*S], how FSDP keeps a rank's own shard) is accepted and left as
    it is; the other shards are copied around it, and the per-tensor copies read
    it in place."""
    shapes = [(1000,), (77, 13), (4096,), (5,)]
    D = 4
    plan, ref = checked_plan(z3, shapes, D, 8)
    S, N_pad = ref.S, ref.N_pad
    gen = torch.Generator().manual_seed(31)
    flat = Guarded(N_pad, torch.bfloat16, 0)
    apart = [Guarded(S, torch.bfloat16, 0, fill=random_bits(S, gen)) for _ in range(D)]
    for r in own:
        flat.t[r * S:(r + 1) * S].copy_(apart[r].t)            # rank r's shard lives in the block
    shards = [flat.t[r * S:(r + 1) * S] if r in own else apart[r].t for r in range(D)]
    outs = [Guarded(k, torch.bfloat16, 1) for k in ref.numels]
    z3.zero3_gather_block(plan, shards, flat.t, [o.t for o in outs])
    torch.cuda.synchronize()
    ref_flat = oracle.all_gather([synth.bf16_bits(a.t) for a in apart], S)
    assert np.array_equal(synth.bf16_bits(flat.t), ref_flat)
    for o, r in zip(outs, oracle.unflatten(ref_flat, ref.offsets, ref.numels)):
        assert np.array_equal(synth.bf16_bits(o.t), r)
        assert o.guards_intact()
    assert flat.guards_intact()
    # a shard inside the block at another rank's place is refused before any work
    bad = list(shards)
    bad[1] = flat.t[2 * S:3 * S] if 1 not in own else flat.t[0:S]
    with pytest.raises(z3.Zero3Error):
        z3.zero3_gather_block(plan, bad, flat.t)
