"""The host optimiser of the CPU-offload step (zero3_host_adamw, libzero3.so)
against the oracle, on the CPU: bit-exact master / m / v after several steps
and bf16 weights equal to the oracle's nearest-even cast, for fp32 and bf16
gradients, ragged sizes, every thread count, random hyper-parameters, the zero
pad and subnormal gradients; concurrent callers; a child forked while another
thread's call runs; argument errors."""
import ctypes as C
import os
import random
import signal
import threading
import time

import numpy as np
import pytest
import torch

import oracle
from fsdp_sharded_mixed_flat_b200 import zero3 as z3


def host_state(n: int, seed: int):
    g = torch.Generator().manual_seed(seed)
    p = torch.randn(n, generator=g) * 0.02
    return p, torch.zeros(n), torch.zeros(n), torch.zeros(n, dtype=torch.bfloat16)


def grad_of(n: int, seed: int, step: int, dtype, scale: float = 1e-3):
    g = torch.Generator().manual_seed(seed * 1000 + step)
    x = torch.randn(n, generator=g) * scale
    return x.to(dtype)


def f32_of(g: torch.Tensor) -> np.ndarray:
    """The gradient the oracle sees: float32 values (bf16 gradients widened exactly)."""
    return g.float().numpy().copy()


def check(p, m, v, w, hp_, hm, hv, what):
    for name, got, ref in (("master", p, hp_), ("exp_avg", m, hm), ("exp_avg_sq", v, hv)):
        a = got.numpy().view(np.uint32)
        b = ref.view(np.uint32)
        assert np.array_equal(a, b), f"{name} {what}: {int((a != b).sum())} elements differ"
    wb = w.view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(wb, oracle.bf16_from_f32(hp_)), f"work_bf16 {what}"


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16], ids=["fp32", "bf16"])
@pytest.mark.parametrize("n,threads", [(1, 1), (15, 3), (17, 0), (16384 * 3 + 5, 2), (16384 * 3 + 5, 7),
                                       (1_000_003, 16), (1_000_003, 0), (65536, 64)])
def test_host_adamw_matches_oracle(n, threads, dtype):
    p, m, v, w = host_state(n, n)
    hp_, hm, hv = p.numpy().copy(), np.zeros(n, np.float32), np.zeros(n, np.float32)
    for t in range(1, 5):
        g = grad_of(n, n, t, dtype)
        z3.zero3_host_adamw(g, p, m, v, w, z3.adamw(step=t), n_threads=threads)
        oracle.adamw(f32_of(g), hp_, hm, hv, oracle.hp(step=t))
        check(p, m, v, w, hp_, hm, hv, f"n={n} threads={threads} {dtype} step={t}")


def test_random_hyperparameters_and_late_steps():
    rnd = random.Random(5)
    n = 40_000
    for case in range(10):
        a = dict(lr=10 ** rnd.uniform(-5, -1.5), beta1=rnd.choice([0.0, 0.5, 0.9, 0.99]),
                 beta2=rnd.choice([0.5, 0.95, 0.999]), eps=10 ** rnd.uniform(-10, -2),
                 weight_decay=rnd.choice([0.0, 0.01, 0.1, 0.5]))
        t0 = rnd.choice([1, 7, 1000, 123456])
        p, m, v, w = host_state(n, case)
        hp_, hm, hv = p.numpy().copy(), np.zeros(n, np.float32), np.zeros(n, np.float32)
        for t in range(t0, t0 + 3):
            g = grad_of(n, case, t, torch.float32, scale=10 ** rnd.uniform(-6, 0))
            z3.zero3_host_adamw(g, p, m, v, w, z3.adamw(step=t, **a), n_threads=rnd.choice([1, 4, 0]))
            oracle.adamw(f32_of(g), hp_, hm, hv, oracle.hp(a["lr"], a["beta1"], a["beta2"], a["eps"],
                                                          a["weight_decay"], t))
        check(p, m, v, w, hp_, hm, hv, f"case {case} {a} t0={t0}")


def test_zero_pad_stays_zero_and_subnormal_gradients():
    n = 20_000
    p, m, v, w = host_state(n, 3)
    p[-4096:] = 0.0
    hp_, hm, hv = p.numpy().copy(), np.zeros(n, np.float32), np.zeros(n, np.float32)
    for t in range(1, 4):
        g = grad_of(n, 3, t, torch.float32, scale=2.0 ** -130)      # fp32 subnormals
        g[-4096:] = 0.0
        z3.zero3_host_adamw(g, p, m, v, w, z3.adamw(step=t), n_threads=4)
        oracle.adamw(f32_of(g), hp_, hm, hv, oracle.hp(step=t))
        check(p, m, v, w, hp_, hm, hv, f"subnormal step={t}")
    assert not p[-4096:].any() and not m[-4096:].any() and not v[-4096:].any()
    assert not w[-4096:].view(torch.int16).any()


def test_concurrent_callers_share_the_pool():
    n = 300_000
    results = {}

    def worker(k):
        p, m, v, w = host_state(n, 100 + k)
        g = grad_of(n, 100 + k, 1, torch.float32)
        for t in range(1, 4):
            z3.zero3_host_adamw(g, p, m, v, w, z3.adamw(step=t), n_threads=3 + k)
        results[k] = (p, m, v, w, g)

    ts = [threading.Thread(target=worker, args=(k,)) for k in range(4)]
    for t in ts:
        t.start()
    for t in ts:
        t.join()
    for k in range(4):
        p, m, v, w, g = results[k]
        p0, _, _, _ = host_state(n, 100 + k)
        hp_, hm, hv = p0.numpy().copy(), np.zeros(n, np.float32), np.zeros(n, np.float32)
        for t in range(1, 4):
            oracle.adamw(f32_of(g), hp_, hm, hv, oracle.hp(step=t))
        check(p, m, v, w, hp_, hm, hv, f"caller {k}")


@pytest.mark.filterwarnings("ignore::DeprecationWarning")
def test_forked_child_gets_a_pool_of_its_own():
    """fork() while another thread's call holds the pool (its lock taken, a worker
    busy): the child's own calls run on a fresh pool, since the parent's workers
    and their locks do not exist in it, and give the oracle's bits."""
    nb = 16_000_000                        # one call of the busy thread: tens of ms on two threads
    big = host_state(nb, 7)
    gbig = grad_of(nb, 7, 1, torch.float32)
    n = 100_003                            # several tasks: the child's call goes through the pool
    p, m, v, w = host_state(n, 8)
    g = grad_of(n, 8, 1, torch.float32)
    hp_, hm, hv = p.numpy().copy(), np.zeros(n, np.float32), np.zeros(n, np.float32)
    oracle.adamw(f32_of(g), hp_, hm, hv, oracle.hp(step=1))
    entering, stop = threading.Event(), threading.Event()

    def busy():
        t = 1
        while not stop.is_set():
            entering.set()
            z3.zero3_host_adamw(gbig, *big, z3.adamw(step=t), n_threads=2)
            t += 1

    th = threading.Thread(target=busy)
    th.start()
    try:
        entering.wait()
        time.sleep(0.005)                  # the busy thread is now inside a call, back to back
        pid = os.fork()
        if pid == 0:                       # the child: one call on its own pool, then leave at once
            code = 1
            try:
                z3.zero3_host_adamw(g, p, m, v, w, z3.adamw(step=1), n_threads=4)
                ok = all(np.array_equal(a.numpy().view(np.uint32), b.view(np.uint32))
                         for a, b in ((p, hp_), (m, hm), (v, hv)))
                code = 0 if ok else 2
            finally:
                os._exit(code)
        deadline = time.monotonic() + 60
        while True:
            done, status = os.waitpid(pid, os.WNOHANG)
            if done:
                break
            if time.monotonic() > deadline:
                os.kill(pid, signal.SIGKILL)
                os.waitpid(pid, 0)
                pytest.fail("the forked child did not finish its call")
            time.sleep(0.05)
        assert os.WIFEXITED(status) and os.WEXITSTATUS(status) == 0, f"child status {status}"
    finally:
        stop.set()
        th.join()


P16 = 0x10000  # fake host addresses: the argument checks run before any access


def call(n=1024, grad=P16 * 1, dtype=0, ptrs=None, hp=None, threads=0):
    ptrs = ptrs or [P16 * 10, P16 * 20, P16 * 30, P16 * 40]
    hp = hp or z3.adamw(step=1)
    return z3.lib().zero3_host_adamw(n, None if grad is None else C.c_void_p(grad), dtype,
                                     *[None if x is None else C.c_void_p(x) for x in ptrs], C.byref(hp), threads)


def test_host_adamw_argument_errors():
    E = z3.Z3_EINVAL
    assert call(n=-1) == E
    assert call(threads=-1) == E
    assert call(dtype=2) == E
    assert call(hp=z3.adamw(eps=0.0)) == E
    assert call(hp=z3.adamw(step=0)) == E
    assert call(grad=None) == E
    assert call(ptrs=[P16 * 10, None, P16 * 30, P16 * 40]) == E
    assert call(ptrs=[P16 * 10 + 2, P16 * 20, P16 * 30, P16 * 40]) == z3.Z3_EALIGN
    assert call(grad=P16 + 2) == z3.Z3_EALIGN                    # fp32 gradient off 4 bytes
    assert call(grad=P16 + 2, dtype=1, ptrs=[P16 * 10, P16 * 20, P16 * 30, P16 * 40 + 1]) == z3.Z3_EALIGN
    assert call(ptrs=[P16 * 10, P16 * 10 + 4, P16 * 30, P16 * 40]) == E   # master over exp_avg
    assert call(grad=P16 * 30 + 8) == E                           # gradient inside exp_avg_sq
    assert call(n=1 << 61) == z3.Z3_EOVERFLOW
    assert call(n=0, grad=None, ptrs=[None] * 4) == z3.Z3_OK      # nothing to do
