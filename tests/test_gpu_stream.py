"""GPU parity of the layer-streamed owned-shard step (two transient buffers, a
copy stream and a compute stream) against the oracle run layer by layer, and a
sampled check of the full 70B rank shard (80 layers, D = 8)."""
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


def owned_contribs(D, S, n_real, seed, step, layer, sigma=1e-3):
    """The D owned contribution slices of one layer, back to back (D * S bf16)."""
    return torch.cat([synth.contribution(n_real, S, seed=seed * 1000 + layer, step=step, rank=d, sigma=sigma,
                                         device="cuda") for d in range(D)])


@pytest.mark.parametrize("copy_in", [True, False], ids=["double_buffer", "in_place"])
@pytest.mark.parametrize("mode", [0, 1], ids=["fp32", "bf16"])
def test_streamed_layers_match_oracle(z3, mode, copy_in):
    from fsdp_sharded_mixed_flat_b200.stream import LayerStreamer
    L, D, rank = 7, 4, 2
    plan, ref = checked_plan(z3, [(300,), (77, 5), (1000,)], D, 8)
    S = ref.S
    n_real = max(0, min(S, ref.N - rank * S))
    master = synth.master_weights(L * S, L * S, seed=4, device="cuda")
    m, v = torch.zeros_like(master), torch.zeros_like(master)
    w = torch.zeros(L * S, dtype=torch.bfloat16, device="cuda")
    st = LayerStreamer(plan, L, rank, master, m, v, w, reduce_dtype=mode)
    hp_, hm, hv, hw = f32_host(master).copy(), np.zeros(L * S, np.float32), np.zeros(L * S, np.float32), \
        np.zeros(L * S, np.uint16)
    for t in range(1, 4):
        src = {l: owned_contribs(D, S, n_real, 9, t, l) for l in range(L)}
        st.step(lambda l: src[l], z3.adamw(**hp_for(t)), copy_in=copy_in)
        for l in range(L):
            host = synth.bf16_bits(src[l])
            sl = slice(l * S, (l + 1) * S)
            p_l, m_l, v_l, w_l = hp_[sl].copy(), hm[sl].copy(), hv[sl].copy(), hw[sl].copy()
            oracle.reduce_adamw([host[d * S:(d + 1) * S] for d in range(D)], S, rank, p_l, m_l, v_l, w_l,
                                oracle_hp(t), layout=oracle.LAYOUT_OWNED, reduce_dtype=mode)
            hp_[sl], hm[sl], hv[sl], hw[sl] = p_l, m_l, v_l, w_l
    torch.cuda.synchronize()
    assert_f32_parity(f32_host(master), hp_, "master")
    assert_f32_parity(f32_host(m), hm, "exp_avg")
    assert_f32_parity(f32_host(v), hv, "exp_avg_sq")
    assert_bf16_parity(synth.bf16_bits(w), hw, "work_bf16")


def test_streamed_layers_with_a_fill_refill(z3):
    """The fill hook writes each block's contributions into the transient buffer."""
    from fsdp_sharded_mixed_flat_b200.stream import LayerStreamer
    L, D, rank = 5, 4, 1
    plan, ref = checked_plan(z3, [(4000,)], D, 8)
    S = ref.S
    n_real = max(0, min(S, ref.N - rank * S))
    master = synth.master_weights(L * S, L * S, seed=6, device="cuda")
    m, v = torch.zeros_like(master), torch.zeros_like(master)
    w = torch.zeros(L * S, dtype=torch.bfloat16, device="cuda")
    st = LayerStreamer(plan, L, rank, master, m, v, w)
    src = {l: owned_contribs(D, S, n_real, 4, 1, l) for l in range(L)}
    hp_, hm, hv, hw = f32_host(master).copy(), np.zeros(L * S, np.float32), np.zeros(L * S, np.float32), \
        np.zeros(L * S, np.uint16)
    st.step(None, z3.adamw(**hp_for(1)), fill=lambda l, buf: buf.copy_(src[l]))
    for l in range(L):
        host = synth.bf16_bits(src[l])
        sl = slice(l * S, (l + 1) * S)
        p_l, m_l, v_l, w_l = hp_[sl].copy(), hm[sl].copy(), hv[sl].copy(), hw[sl].copy()
        oracle.reduce_adamw([host[d * S:(d + 1) * S] for d in range(D)], S, rank, p_l, m_l, v_l, w_l,
                            oracle_hp(1), layout=oracle.LAYOUT_OWNED)
        hp_[sl], hm[sl], hv[sl], hw[sl] = p_l, m_l, v_l, w_l
    torch.cuda.synchronize()
    assert_f32_parity(f32_host(master), hp_, "master")
    assert_bf16_parity(synth.bf16_bits(w), hw, "work_bf16")


def test_llama70b_rank_shard_80_layers_sampled(z3):
    """The full resident shard of one rank (8.556B owned params, about 120 GB with
    the bf16 shard), one streamed step over all 80 layers; the oracle checks
    every element of layers 79, 40 and 0 and a seeded 2^20-element subset of
    every other layer (master, moments and bf16 weights)."""
    from fsdp_sharded_mixed_flat_b200.stream import LayerStreamer
    w_ = synth.WORKLOADS["llama70b_layer"]
    L, D, rank = w_["layers"], w_["D"], 5
    plan, ref = checked_plan(z3, [s for _, s in w_["tensors"]], D, synth.ALIGN)
    S = ref.S
    torch.cuda.empty_cache()              # blocks cached by earlier tests count as used
    free, _ = torch.cuda.mem_get_info()
    need = L * S * 14 + 4 * D * S * 2 + (1 << 30)
    if free < need:
        pytest.skip(f"needs {need / 1e9:.0f} GB free, {free / 1e9:.0f} GB available")
    master = torch.empty(L * S, dtype=torch.float32, device="cuda")
    for l in range(L):
        master[l * S:(l + 1) * S] = synth.master_weights(S, S, seed=100 + l, device="cuda")
    m, v = torch.zeros_like(master), torch.zeros_like(master)
    w = torch.zeros(L * S, dtype=torch.bfloat16, device="cuda")
    pool = [owned_contribs(D, S, S, 77, 1, k, sigma=1e-4) for k in range(2)]
    st = LayerStreamer(plan, L, rank, master, m, v, w)
    rng = np.random.default_rng(0)
    idx = torch.from_numpy(np.unique(rng.choice(S, 1 << 20, replace=False))).cuda()
    full_layers = (0, L // 2, L - 1)
    before = {l: f32_host(master[l * S:(l + 1) * S][idx]) for l in range(L) if l not in full_layers}
    full_before = {l: f32_host(master[l * S:(l + 1) * S]) for l in full_layers}
    st.step(lambda l: pool[l % 2], z3.adamw(**hp_for(1)))
    torch.cuda.synchronize()
    hosts = [synth.bf16_bits(p) for p in pool]
    for l in range(L):
        c = hosts[l % 2]
        if l in full_before:
            sel = np.arange(S)
            p_l = full_before[l].copy()
            got = master[l * S:(l + 1) * S]
            got_w = w[l * S:(l + 1) * S]
        else:
            sel = idx.cpu().numpy()
            p_l = before[l].copy()
            got = master[l * S:(l + 1) * S][idx]
            got_w = w[l * S:(l + 1) * S][idx]
            got_m = m[l * S:(l + 1) * S][idx]
            got_v = v[l * S:(l + 1) * S][idx]
        m_l, v_l, w_l = np.zeros(sel.size, np.float32), np.zeros(sel.size, np.float32), np.zeros(sel.size, np.uint16)
        oracle.reduce_adamw([np.ascontiguousarray(c[d * S:(d + 1) * S][sel]) for d in range(D)], sel.size, 0,
                            p_l, m_l, v_l, w_l, oracle_hp(1), layout=oracle.LAYOUT_OWNED)
        assert_f32_parity(f32_host(got), p_l, f"master layer {l}")
        assert_bf16_parity(synth.bf16_bits(got_w), w_l, f"work layer {l}")
        if l in full_before:
            got_m, got_v = m[l * S:(l + 1) * S], v[l * S:(l + 1) * S]
        assert_f32_parity(f32_host(got_m), m_l, f"exp_avg layer {l}")
        assert_f32_parity(f32_host(got_v), v_l, f"exp_avg_sq layer {l}")
