"""The Python binding's own checks, on CPU (no device work): the C ABI takes
plain pointers and cannot check extents, so the binding refuses wrong counts,
non-tensors, host tensors where device memory is needed, and buffers smaller
than the plan asks for, before anything reaches the library."""
import pytest
import torch

from fsdp_sharded_mixed_flat_b200 import build

build.build()
from fsdp_sharded_mixed_flat_b200 import zero3 as z3  # noqa: E402


@pytest.fixture()
def plan():
    return z3.zero3_plan([(100,), (28,)], 2, 8)


def state(n, dtype=torch.float32):
    return torch.zeros(n, dtype=dtype)


def test_contribution_count_must_match_D(plan):
    with pytest.raises(ValueError, match="need 2 contributions"):
        z3.zero3_reduce_adamw(plan, -1, [state(128, torch.bfloat16)], state(128), state(128), state(128),
                              state(128, torch.bfloat16), z3.adamw())
    with pytest.raises(ValueError, match="need 2 shards"):
        z3.zero3_gather_block(plan, [state(64, torch.bfloat16)] * 3, state(128, torch.bfloat16))


def test_host_tensors_are_refused_where_device_memory_is_needed(plan):
    c = [state(128, torch.bfloat16)] * 2
    with pytest.raises(ValueError, match="CUDA tensor"):
        z3.zero3_reduce_adamw(plan, -1, c, state(128), state(128), state(128), state(128, torch.bfloat16),
                              z3.adamw())
    with pytest.raises(TypeError):
        z3.zero3_reduce_adamw(plan, -1, [object(), object()], state(128), state(128), state(128),
                              state(128, torch.bfloat16), z3.adamw())


def test_hybrid_node_and_contribution_counts(plan):
    c = [state(128, torch.bfloat16)] * 4
    args = (state(128), state(128), state(128), state(128, torch.bfloat16), z3.adamw())
    with pytest.raises(ValueError, match="n_nodes"):
        z3.zero3_reduce_adamw_hybrid(plan, -1, 0, c, *args)
    with pytest.raises(ValueError, match="n_nodes"):
        z3.zero3_reduce_adamw_hybrid(plan, -1, 33, c * 17, *args)
    with pytest.raises(ValueError, match="need 4 contributions"):
        z3.zero3_reduce_adamw_hybrid(plan, -1, 2, c[:3], *args)
    with pytest.raises(ValueError, match="CUDA tensor"):
        z3.zero3_reduce_adamw_hybrid(plan, -1, 2, c, *args)


def test_gathered_block_count_is_bounded(plan):
    c = [state(128, torch.bfloat16)] * 2
    with pytest.raises(ValueError, match="gathered blocks"):
        z3.zero3_reduce_adamw_gather(plan, -1, c, state(128), state(128), state(128), None, [], z3.adamw())
    with pytest.raises(ValueError, match="at most"):
        z3.zero3_reduce_adamw_dev(plan, -1, c, state(128), state(128), state(128), None,
                                  [state(128, torch.bfloat16)] * 9, state(8))


def test_tensor_output_count_must_match(plan):
    with pytest.raises(ValueError, match="tensor outputs"):
        z3.zero3_gather_block(plan, [state(64, torch.bfloat16)] * 2, None, [None])


def test_plan_views_and_lazy_offsets(plan):
    assert (plan.N, plan.N_pad, plan.S) == (128, 128, 64)
    assert plan.offsets == [0, 100] and plan.numels == [100, 28]
    flat = torch.arange(128, dtype=torch.float32)
    v = plan.views(flat)
    assert v[0].shape == (100,) and v[1].shape == (28,) and v[1][0].item() == 100.0
    v[1][0] = -1.0                                   # zero-copy: the view aliases the block
    assert flat[100].item() == -1.0
    with pytest.raises(ValueError):
        plan.views(torch.zeros(10))
    specs = z3.tensor_specs([(100,), (28,)])
    again = z3.Plan([(100,), (28,)], 2, 8, specs=specs)
    assert (again.N, again.N_pad, again.S, again.offsets) == (plan.N, plan.N_pad, plan.S, plan.offsets)
    with pytest.raises(ValueError):
        z3.tensor_specs([(1, 2, 3, 4, 5)])


def test_plan_alive_at_interpreter_exit_is_freed_quietly():
    """A plan still referenced when the interpreter exits is freed without errors
    (module globals may already be cleared when its finaliser runs)."""
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    code = ("import sys; sys.path.insert(0, %r)\n"
            "from fsdp_sharded_mixed_flat_b200 import zero3 as z3\n"
            "keep = z3.zero3_plan([(10,), (3, 4)], 2, 8)\n") % root
    r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0 and "Error" not in r.stderr and "Exception" not in r.stderr, r.stderr
