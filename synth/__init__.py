"""Seeded synthetic inputs for the ZeRO-3 per-rank step.

This module only describes workloads (tensor lists shaped like the pages'
models) and draws seeded random inputs for them.  It holds none of the
method's arithmetic: no planning, reduction, optimiser or gather.  Both the
CUDA path's tests/benchmark and the oracle take their inputs from here.

Workloads (shapes from the pages' models; the sizes are synthetic stand-ins,
no dataset or trained weights are involved):
  tiny_gpt      the 3.3M-parameter GPT of "Building GPT from Scratch — Part 8:
                FSDP" (section "The Problem"), 26 tensors, D = 4.
  llama7b_d8    one LLaMA-7B decoder block ("7.10 — Fully-sharded data parallel
                (FSDP / ZeRO-3)", §5.2), 9 tensors, D = 8.
  llama7b_d32   the same block plus a 4097-element bias, D = 32: the block size
                is not a multiple of D*A, so the last shard has a padded tail.
  llama7b_policy the same block for the reduce-dtype sweep, D in {2,4,8,16},
                heavy-tailed gradients with exact zeros.
  llama70b_layer one 70B decoder layer (d = 8192, GQA k/v 8192x1024, MLP 28672)
                of "Distributed LLM Fine-Tuning at Scale" §1's 70B model at D=8;
                80 of them form one rank's resident shard.

Input recipe:
  gradient contributions  N(0, sigma) in fp32, rounded to bf16 by torch's
                          round-to-nearest-even cast; pad tail = 0.
  student-t contributions z / sqrt(chi2_3 / 3) * scale, chi2_3 the sum of three
                          squared standard normals; a fraction of elements set to
                          exactly 0, drawn independently per (rank, step, element).
  master weights          N(0, 0.02) fp32; pad tail = 0.  m = v = 0.
Every draw comes from its own torch.Generator seeded from (seed, step, rank, stream).
"""
from __future__ import annotations

import torch

# AdamW hyper-parameters used by every workload.
ADAMW = dict(lr=3e-4, beta1=0.9, beta2=0.95, eps=1e-8, weight_decay=0.1)

ALIGN = 128  # planner alignment in elements


def _tiny_gpt():
    ts = [("emb", (65, 256))]
    for layer in range(4):
        ts += [(f"h{layer}.qkv", (256, 768)), (f"h{layer}.proj", (256, 256)),
               (f"h{layer}.fc", (256, 1024)), (f"h{layer}.fc2", (1024, 256)),
               (f"h{layer}.ln1", (256,)), (f"h{layer}.ln2", (256,))]
    # The listed tensors sum to 3,164,416; the stated block size is 3,276,800.
    # The remaining 439 x 256 stand in for the unlisted parameters.
    ts.append(("rest", (439, 256)))
    return ts


def _llama7b_block():
    d, f = 4096, 11008
    return [("q", (d, d)), ("k", (d, d)), ("v", (d, d)), ("o", (d, d)),
            ("gate", (d, f)), ("up", (d, f)), ("down", (f, d)),
            ("rms1", (d,)), ("rms2", (d,))]


def _llama70b_layer():
    d, kv, f = 8192, 1024, 28672
    return [("q", (d, d)), ("k", (d, kv)), ("v", (d, kv)), ("o", (d, d)),
            ("gate", (d, f)), ("up", (d, f)), ("down", (f, d)),
            ("rms1", (d,)), ("rms2", (d,))]


WORKLOADS = {
    "tiny_gpt": dict(tensors=_tiny_gpt(), D=4, sigma=1e-3, dist="normal", steps=10),
    "llama7b_d8": dict(tensors=_llama7b_block(), D=8, sigma=1e-4, dist="normal", steps=10),
    "llama7b_d32": dict(tensors=_llama7b_block() + [("bias", (4097,))], D=32, sigma=1e-4,
                        dist="normal", steps=10),
    "llama7b_policy": dict(tensors=_llama7b_block(), D=8, Ds=(2, 4, 8, 16), sigma=1e-3,
                           dist="student_t", zero_frac=0.01, steps=100),
    "llama70b_layer": dict(tensors=_llama70b_layer(), D=8, sigma=1e-4, dist="normal",
                           steps=10, layers=80),
    # HYBRID_SHARD over 4 nodes of 8 GPUs on the 7B block: sharded 8 ways inside a
    # node, replicated over the 4 nodes; 32 contributions per element
    "llama7b_hybrid": dict(tensors=_llama7b_block(), D=8, nodes=4, sigma=1e-4, dist="normal", steps=10),
    # a 33.5M-element slice of the 7B block (two 4096 x 4096 projections) at D = 8:
    # about 1.4 GB of traffic per step, larger than L2, small enough for profiler replays
    "profile_d8": dict(tensors=[("q", (4096, 4096)), ("k", (4096, 4096))], D=8, sigma=1e-4,
                       dist="normal", steps=10),
    # the same slice as 4 nodes of 8 ranks (HYBRID_SHARD): about 3 GB of traffic per step
    "profile_hybrid": dict(tensors=[("q", (4096, 4096)), ("k", (4096, 4096))], D=8, nodes=4, sigma=1e-4,
                           dist="normal", steps=10),
}


def numel(shape) -> int:
    n = 1
    for s in shape:
        n *= int(s)
    return n


def block_numel(tensors) -> int:
    return sum(numel(s) for _, s in tensors)


def _gen(device, seed: int, step: int, rank: int, stream: int) -> torch.Generator:
    g = torch.Generator(device=device)
    key = (((seed * 1_000_003 + step) * 1_009 + rank) * 131 + stream) & ((1 << 63) - 1)
    g.manual_seed(key)
    return g


def contribution(n_real: int, n_total: int, *, seed: int, step: int, rank: int,
                 sigma: float, dist: str = "normal", zero_frac: float = 0.0,
                 device="cpu") -> torch.Tensor:
    """One rank's bf16 gradient contribution: n_real drawn values, then zeros up to n_total."""
    out = torch.zeros(n_total, dtype=torch.bfloat16, device=device)
    if n_real == 0:
        return out
    g = _gen(device, seed, step, rank, 1)
    if dist == "normal":
        x = torch.randn(n_real, generator=g, device=device, dtype=torch.float32) * sigma
    elif dist == "student_t":
        z = torch.randn(n_real, generator=g, device=device, dtype=torch.float32)
        chi2 = torch.zeros(n_real, device=device, dtype=torch.float32)
        for _ in range(3):
            e = torch.randn(n_real, generator=g, device=device, dtype=torch.float32)
            chi2 += e * e
        x = z / torch.sqrt(chi2 / 3.0) * sigma
        del z, chi2
    elif dist == "subnormal":
        # scaled so that most values and partial sums are bf16 / fp32 subnormals
        x = torch.randn(n_real, generator=g, device=device, dtype=torch.float32) * 2.0 ** -130
    elif dist == "integers":
        # small integers, exactly representable in bf16 and in every partial sum
        x = torch.randint(-8, 9, (n_real,), generator=g, device=device).to(torch.float32)
    else:
        raise ValueError(dist)
    if zero_frac > 0.0:
        u = torch.rand(n_real, generator=g, device=device)
        x = torch.where(u < zero_frac, torch.zeros_like(x), x)
    out[:n_real] = x.to(torch.bfloat16)
    return out


def contributions(D: int, n_real: int, n_total: int, *, seed: int, step: int,
                  sigma: float, dist: str = "normal", zero_frac: float = 0.0,
                  device="cpu"):
    """D ranks' contributions (list of bf16 tensors of n_total elements each)."""
    return [contribution(n_real, n_total, seed=seed, step=step, rank=r, sigma=sigma, dist=dist,
                         zero_frac=zero_frac, device=device) for r in range(D)]


def master_weights(n_real: int, n_total: int, *, seed: int, device="cpu",
                   std: float = 0.02) -> torch.Tensor:
    """fp32 master weights N(0, std), zero pad tail."""
    out = torch.zeros(n_total, dtype=torch.float32, device=device)
    if n_real:
        g = _gen(device, seed, 0, 0, 2)
        out[:n_real] = torch.randn(n_real, generator=g, device=device, dtype=torch.float32) * std
    return out


def bf16_bits(t: torch.Tensor):
    """A bf16 tensor's bit patterns as a numpy uint16 array (host copy)."""
    import numpy as np
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def bits_to_bf16(a, device="cpu") -> torch.Tensor:
    """numpy uint16 bit patterns as a bf16 tensor."""
    import numpy as np
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(device)
