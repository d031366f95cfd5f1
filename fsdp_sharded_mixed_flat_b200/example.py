"""A complete use of the library: ten ZeRO-3 optimiser steps of one block
whose D = 8 ranks are simulated on one GPU, then the all-gather of the eight
bf16 shards and the zero-copy unflatten into per-tensor views.

    python -m fsdp_sharded_mixed_flat_b200.build      # once: libzero3.so for sm_100a
    python -m fsdp_sharded_mixed_flat_b200.example

run() returns every buffer it used, so a caller (or a test) can inspect them.
"""
import torch

from fsdp_sharded_mixed_flat_b200 import zero3 as z3


def run(steps: int = 10, seed: int = 1234, dev: str = "cuda"):
    torch.manual_seed(seed)
    shapes = [(4096, 4096), (4096, 11008), (4096,)]           # one block's tensors, row-major
    plan = z3.zero3_plan(shapes, D=8, align_elems=128)       # N, N_pad, S = N_pad / D, P_r = [r*S, (r+1)*S)

    grads = [torch.zeros(plan.N_pad, dtype=torch.bfloat16, device=dev) for _ in range(plan.D)]
    for g in grads:
        g[:plan.N] = torch.randn(plan.N, device=dev) * 1e-3    # rank d's flat gradient; the tail pad stays zero
    master = torch.zeros(plan.N_pad, device=dev)              # fp32 state of every P_r, back to back
    master[:plan.N] = torch.randn(plan.N, device=dev) * 0.02
    m, v = torch.zeros_like(master), torch.zeros_like(master)
    work = torch.empty(plan.N_pad, dtype=torch.bfloat16, device=dev)                  # the D bf16 shards

    for step in range(1, steps + 1):
        hp = z3.adamw(lr=3e-4, beta1=0.9, beta2=0.95, eps=1e-8, weight_decay=0.1, step=step)
        # reduce-scatter's reduction in rank order + AdamW + bf16 cast, every rank's partition at once
        z3.zero3_reduce_adamw(plan, -1, grads, master, m, v, work, hp, reduce_dtype=z3.Z3_REDUCE_FP32)

    flat = torch.empty(plan.N_pad, dtype=torch.bfloat16, device=dev)
    z3.zero3_gather_block(plan, [work[r * plan.S:(r + 1) * plan.S] for r in range(plan.D)], flat)
    weights = plan.views(flat)                               # zero-copy per-tensor views of the gathered block
    return dict(shapes=shapes, plan=plan, grads=grads, master=master, exp_avg=m, exp_avg_sq=v, work=work,
                flat=flat, weights=weights)


if __name__ == "__main__":
    out = run()
    torch.cuda.synchronize()
    plan = out["plan"]
    print(f"N={plan.N} N_pad={plan.N_pad} S={plan.S}; views: {[tuple(w.shape) for w in out['weights']]}")
