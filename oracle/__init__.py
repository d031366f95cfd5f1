"""The oracle: a plain, slow, single-threaded CPU restatement of the per-rank
ZeRO-3 / FSDP step (plan, memory ledger, reduce-scatter, AdamW, bf16 cast,
all-gather, unflatten, and the HYBRID_SHARD form of the reduction), written in
C (oracle/zero3_ref.c) and driven here through ctypes on numpy arrays.

TEST INFRASTRUCTURE ONLY.  Only tests/, the package's smoke check and the
benchmark's CPU-baseline leg may import this module.  It shares no code with
the CUDA product path and never imports it.

Arrays: bf16 values travel as numpy uint16 bit patterns, fp32 as float32.
"""
import ctypes as C

import numpy as np

from . import build as _build

_lib = None

REDUCE_FP32 = 0
REDUCE_BF16 = 1
LAYOUT_FULL = 0
LAYOUT_OWNED = 1


class AdamWHP(C.Structure):
    _fields_ = [("lr", C.c_double), ("beta1", C.c_double), ("beta2", C.c_double),
                ("eps", C.c_double), ("weight_decay", C.c_double), ("step", C.c_int64)]


def lib():
    """Load (building first if needed) the oracle's shared library."""
    global _lib
    if _lib is None:
        _lib = _bind(C.CDLL(_build.build()))
    return _lib


def use_library(path):
    """Swap in another build of the oracle's C source (the mutation tests plant a
    mistake in a copy of the source, build it, and check that the pins fail).
    Returns the library that was in use, for restoring."""
    global _lib
    previous = _lib
    _lib = None if path is None else _bind(C.CDLL(path))
    return previous


def restore_library(previous):
    global _lib
    _lib = previous


def _bind(L):
    """Declare the C signatures on a loaded oracle library."""
    p = C.c_void_p
    i64, i32 = C.c_int64, C.c_int32
    L.ref_bf16_from_f32.argtypes = [C.c_float]
    L.ref_bf16_from_f32.restype = C.c_uint16
    L.ref_f32_from_bf16.argtypes = [C.c_uint16]
    L.ref_f32_from_bf16.restype = C.c_float
    L.ref_bf16_from_f32_array.argtypes = [p, i64, p]
    L.ref_bf16_from_f32_array.restype = None
    L.ref_plan.argtypes = [i32, p, i32, i32, p, p, p, p]
    L.ref_plan.restype = C.c_int
    L.ref_rank_range.argtypes = [i64, i64, i32, p, p]
    L.ref_rank_range.restype = None
    L.ref_memory_bytes.argtypes = [C.c_double, C.c_double, i32]
    L.ref_memory_bytes.restype = C.c_double
    L.ref_transient_bytes.argtypes = [C.c_double, i32]
    L.ref_transient_bytes.restype = C.c_double
    L.ref_allgather_bytes.argtypes = [C.c_double, i32, i32]
    L.ref_allgather_bytes.restype = C.c_double
    L.ref_reduce_scatter.argtypes = [i32, i64, i32, p, i32, i32, p]
    L.ref_reduce_scatter.restype = C.c_int
    L.ref_adamw_consts_of.argtypes = [C.POINTER(AdamWHP), p]
    L.ref_adamw_consts_of.restype = None
    L.ref_adamw.argtypes = [i64, p, p, p, p, C.POINTER(AdamWHP)]
    L.ref_adamw.restype = C.c_int
    L.ref_reduce_adamw.argtypes = [i32, i64, i32, p, i32, p, p, p, p, i32, C.POINTER(AdamWHP)]
    L.ref_reduce_adamw.restype = C.c_int
    L.ref_reduce_scatter_hybrid.argtypes = [i32, i32, i64, i32, p, i32, i32, p]
    L.ref_reduce_scatter_hybrid.restype = C.c_int
    L.ref_reduce_adamw_hybrid.argtypes = [i32, i32, i64, i32, p, i32, p, p, p, p, i32, C.POINTER(AdamWHP)]
    L.ref_reduce_adamw_hybrid.restype = C.c_int
    L.ref_node_sum.argtypes = [i32, i64, i32, p, i32, i32, p]
    L.ref_node_sum.restype = C.c_int
    L.ref_fold_adamw.argtypes = [i32, i32, i64, p, p, p, p, p, i32, C.POINTER(AdamWHP)]
    L.ref_fold_adamw.restype = C.c_int
    L.ref_all_gather.argtypes = [i32, i64, p, p]
    L.ref_all_gather.restype = None
    L.ref_unflatten.argtypes = [p, i32, p, p, p]
    L.ref_unflatten.restype = None
    return L


def _ptr(a: np.ndarray):
    return C.c_void_p(a.ctypes.data)


def _ptr_array(arrays):
    arr = (C.c_void_p * max(1, len(arrays)))()
    for k, a in enumerate(arrays):
        arr[k] = a.ctypes.data
    return arr


def _u16(a) -> np.ndarray:
    a = np.ascontiguousarray(a)
    assert a.dtype == np.uint16, a.dtype
    return a


def _f32(a) -> np.ndarray:
    a = np.ascontiguousarray(a)
    assert a.dtype == np.float32, a.dtype
    return a


def hp(lr=3e-4, beta1=0.9, beta2=0.95, eps=1e-8, weight_decay=0.1, step=1) -> AdamWHP:
    return AdamWHP(lr, beta1, beta2, eps, weight_decay, step)


# ---------------------------------------------------------------- conversions
def bf16_from_f32(x) -> np.ndarray:
    x = _f32(np.asarray(x, dtype=np.float32))
    out = np.empty(x.shape, dtype=np.uint16)
    lib().ref_bf16_from_f32_array(_ptr(x), x.size, _ptr(out))
    return out


def f32_from_bf16(h) -> np.ndarray:
    h = _u16(np.asarray(h, dtype=np.uint16))
    return (h.astype(np.uint32) << 16).view(np.float32)


# ----------------------------------------------------------------------- plan
def plan(numels, D: int, A: int):
    """Returns (offsets, N, N_pad, S) for the tensors' element counts."""
    numel = np.ascontiguousarray(np.asarray(numels, dtype=np.int64))
    offsets = np.zeros(max(1, len(numel)), dtype=np.int64)
    out = np.zeros(3, dtype=np.int64)
    rc = lib().ref_plan(len(numel), _ptr(numel), D, A, _ptr(offsets), C.c_void_p(out.ctypes.data),
                        C.c_void_p(out.ctypes.data + 8), C.c_void_p(out.ctypes.data + 16))
    if rc != 0:
        raise ValueError("invalid plan arguments")
    return offsets[:len(numel)], int(out[0]), int(out[1]), int(out[2])


def rank_range(N: int, S: int, r: int):
    b, e = C.c_int64(), C.c_int64()
    lib().ref_rank_range(N, S, r, C.byref(b), C.byref(e))
    return b.value, e.value


def memory_bytes(N: float, D: float, stage: int) -> float:
    return lib().ref_memory_bytes(float(N), float(D), stage)


def transient_bytes(block_params: float, n_buffers: int = 1) -> float:
    return lib().ref_transient_bytes(float(block_params), n_buffers)


def allgather_bytes(block_bytes: float, n_blocks: int, D: int) -> float:
    return lib().ref_allgather_bytes(float(block_bytes), n_blocks, D)


# ----------------------------------------------------------- reduce and AdamW
def reduce_scatter(contribs, S: int, rank: int, layout: int = LAYOUT_FULL,
                   reduce_dtype: int = REDUCE_FP32) -> np.ndarray:
    contribs = [_u16(c) for c in contribs]
    D = len(contribs)
    out = np.empty(D * S if rank < 0 else S, dtype=np.float32)
    rc = lib().ref_reduce_scatter(D, S, rank, _ptr_array(contribs), layout, reduce_dtype, _ptr(out))
    if rc != 0:
        raise ValueError("invalid reduce_scatter arguments")
    return out


def adamw_consts(h: AdamWHP) -> np.ndarray:
    out = np.zeros(8, dtype=np.float32)
    lib().ref_adamw_consts_of(C.byref(h), _ptr(out))
    return out


def adamw(g, master, exp_avg, exp_avg_sq, h: AdamWHP) -> None:
    """In place on master / exp_avg / exp_avg_sq (float32 arrays)."""
    g, master, exp_avg, exp_avg_sq = _f32(g), _f32(master), _f32(exp_avg), _f32(exp_avg_sq)
    rc = lib().ref_adamw(g.size, _ptr(g), _ptr(master), _ptr(exp_avg), _ptr(exp_avg_sq), C.byref(h))
    if rc != 0:
        raise ValueError("invalid adamw arguments")


def reduce_adamw(contribs, S: int, rank: int, master, exp_avg, exp_avg_sq, work_bf16,
                 h: AdamWHP, layout: int = LAYOUT_FULL, reduce_dtype: int = REDUCE_FP32) -> None:
    """In place on master / exp_avg / exp_avg_sq; writes work_bf16."""
    contribs = [_u16(c) for c in contribs]
    for a in (master, exp_avg, exp_avg_sq):
        assert a.flags.c_contiguous and a.dtype == np.float32
    assert work_bf16.flags.c_contiguous and work_bf16.dtype == np.uint16
    rc = lib().ref_reduce_adamw(len(contribs), S, rank, _ptr_array(contribs), layout, _ptr(master),
                                _ptr(exp_avg), _ptr(exp_avg_sq), _ptr(work_bf16), reduce_dtype,
                                C.byref(h))
    if rc != 0:
        raise ValueError("invalid reduce_adamw arguments")


# ------------------------------------------------------------- HYBRID_SHARD
def _replica_split(contribs, R: int) -> int:
    if R < 1 or len(contribs) % R:
        raise ValueError(f"{len(contribs)} contributions do not split into {R} nodes")
    return len(contribs) // R


def reduce_scatter_hybrid(contribs, R: int, S: int, rank: int, layout: int = LAYOUT_FULL,
                          reduce_dtype: int = REDUCE_FP32) -> np.ndarray:
    """The averaged gradient for R nodes of D = len(contribs) / R ranks; the
    contribution of local rank d on node k is contribs[k * D + d]."""
    contribs = [_u16(c) for c in contribs]
    D = _replica_split(contribs, R)
    out = np.empty(D * S if rank < 0 else S, dtype=np.float32)
    rc = lib().ref_reduce_scatter_hybrid(R, D, S, rank, _ptr_array(contribs), layout, reduce_dtype, _ptr(out))
    if rc != 0:
        raise ValueError("invalid reduce_scatter_hybrid arguments")
    return out


def reduce_adamw_hybrid(contribs, R: int, S: int, rank: int, master, exp_avg, exp_avg_sq, work_bf16,
                        h: AdamWHP, layout: int = LAYOUT_FULL, reduce_dtype: int = REDUCE_FP32) -> None:
    """The HYBRID_SHARD step, in place on master / exp_avg / exp_avg_sq; writes work_bf16."""
    contribs = [_u16(c) for c in contribs]
    D = _replica_split(contribs, R)
    for a in (master, exp_avg, exp_avg_sq):
        assert a.flags.c_contiguous and a.dtype == np.float32
    assert work_bf16.flags.c_contiguous and work_bf16.dtype == np.uint16
    rc = lib().ref_reduce_adamw_hybrid(R, D, S, rank, _ptr_array(contribs), layout, _ptr(master),
                                       _ptr(exp_avg), _ptr(exp_avg_sq), _ptr(work_bf16), reduce_dtype,
                                       C.byref(h))
    if rc != 0:
        raise ValueError("invalid reduce_adamw_hybrid arguments")


def node_sum(contribs, S: int, rank: int, layout: int = LAYOUT_FULL, reduce_dtype: int = REDUCE_FP32) -> np.ndarray:
    """HYBRID_SHARD across nodes, part 1: the node's unscaled rank-ordered sum of
    its D contributions (D = len(contribs)) for one partition or all of them."""
    contribs = [_u16(c) for c in contribs]
    D = len(contribs)
    out = np.empty(D * S if rank < 0 else S, dtype=np.float32)
    rc = lib().ref_node_sum(D, S, rank, _ptr_array(contribs), layout, reduce_dtype, _ptr(out))
    if rc != 0:
        raise ValueError("invalid node_sum arguments")
    return out


def fold_adamw(node_sums, D: int, master, exp_avg, exp_avg_sq, work_bf16, h: AdamWHP,
               reduce_dtype: int = REDUCE_FP32) -> None:
    """HYBRID_SHARD across nodes, part 2: the R = len(node_sums) node sums folded
    in node order, 1/(R*D), AdamW and the cast; in place, writes work_bf16."""
    sums = [_f32(x) for x in node_sums]
    for a in (master, exp_avg, exp_avg_sq):
        assert a.flags.c_contiguous and a.dtype == np.float32
    assert work_bf16.flags.c_contiguous and work_bf16.dtype == np.uint16
    rc = lib().ref_fold_adamw(len(sums), D, master.size, _ptr_array(sums), _ptr(master), _ptr(exp_avg),
                              _ptr(exp_avg_sq), _ptr(work_bf16), reduce_dtype, C.byref(h))
    if rc != 0:
        raise ValueError("invalid fold_adamw arguments")


# ------------------------------------------------------- gather and unflatten
def all_gather(shards, S: int) -> np.ndarray:
    shards = [_u16(s) for s in shards]
    flat = np.empty(len(shards) * S, dtype=np.uint16)
    lib().ref_all_gather(len(shards), S, _ptr_array(shards), _ptr(flat))
    return flat


def unflatten(flat, offsets, numels):
    flat = _u16(flat)
    offsets = np.ascontiguousarray(np.asarray(offsets, dtype=np.int64))
    numels = np.ascontiguousarray(np.asarray(numels, dtype=np.int64))
    outs = [np.empty(int(n), dtype=np.uint16) for n in numels]
    lib().ref_unflatten(_ptr(flat), len(outs), _ptr(offsets), _ptr(numels), _ptr_array(outs))
    return outs
