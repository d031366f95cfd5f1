"""Python binding of libzero3.so (the C ABI declared in include/zero3.h).

Argument marshalling only: torch tensors are turned into device pointers,
sizes are checked against the plan (the C ABI sees plain pointers and cannot
check extents), the tensors' device is made current and the call is enqueued
on the given (default: torch's current) stream.  Every step of the path runs
in the library's CUDA kernels; there is no fallback.  If the library is not
built, importing this module raises.
"""
from __future__ import annotations

import ctypes as C
import os
from typing import Optional, Sequence

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libzero3.so")

Z3_OK, Z3_EINVAL, Z3_EALIGN, Z3_ENOMEM, Z3_ECUDA, Z3_EOVERFLOW = 0, -1, -2, -3, -4, -5
Z3_D_MAX = 64
Z3_GATHER_MAX = 8
Z3_SCALARS = 8
Z3_REDUCE_FP32, Z3_REDUCE_BF16 = 0, 1
Z3_CONTRIB_FULL, Z3_CONTRIB_OWNED = 0, 1
Z3_STAGE_DDP, Z3_STAGE_ZERO1, Z3_STAGE_ZERO2, Z3_STAGE_ZERO3 = 0, 1, 2, 3


class TensorSpec(C.Structure):
    _fields_ = [("numel", C.c_int64), ("ndim", C.c_int32), ("shape", C.c_int64 * 4)]


class AdamW(C.Structure):
    _fields_ = [("lr", C.c_double), ("beta1", C.c_double), ("beta2", C.c_double),
                ("eps", C.c_double), ("weight_decay", C.c_double), ("step", C.c_int64)]


class Zero3Error(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {status_string(status)} ({status})")
        self.status = status


def _load() -> C.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is not built: run `python -m fsdp_sharded_mixed_flat_b200.build`")
    L = C.CDLL(LIB_PATH)
    vp, i32, i64 = C.c_void_p, C.c_int32, C.c_int64
    L.zero3_status_string.argtypes = [C.c_int]
    L.zero3_status_string.restype = C.c_char_p
    L.zero3_plan.argtypes = [C.POINTER(TensorSpec), i32, i32, i32, C.POINTER(vp)]
    L.zero3_plan.restype = C.c_int
    L.zero3_plan_free.argtypes = [vp]
    L.zero3_plan_free.restype = None
    L.zero3_plan_info.argtypes = [vp, C.POINTER(i32), C.POINTER(i32), C.POINTER(i32),
                                  C.POINTER(i64), C.POINTER(i64), C.POINTER(i64)]
    L.zero3_plan_info.restype = C.c_int
    L.zero3_plan_tensor.argtypes = [vp, i32, C.POINTER(i64), C.POINTER(i64)]
    L.zero3_plan_tensor.restype = C.c_int
    L.zero3_plan_rank.argtypes = [vp, i32, C.POINTER(i64), C.POINTER(i64)]
    L.zero3_plan_rank.restype = C.c_int
    L.zero3_memory_bytes.argtypes = [i64, i32, i32, C.POINTER(i64)]
    L.zero3_memory_bytes.restype = C.c_int
    L.zero3_transient_bytes.argtypes = [i64, i32, C.POINTER(i64)]
    L.zero3_transient_bytes.restype = C.c_int
    L.zero3_allgather_bytes.argtypes = [i64, i32, i32, C.POINTER(i64)]
    L.zero3_allgather_bytes.restype = C.c_int
    L.zero3_reduce_adamw.argtypes = [vp, i32, vp, i32, vp, vp, vp, vp, i32, C.POINTER(AdamW), vp]
    L.zero3_reduce_adamw.restype = C.c_int
    L.zero3_reduce_adamw_hybrid.argtypes = [vp, i32, i32, vp, i32, vp, vp, vp, vp, i32, C.POINTER(AdamW), vp]
    L.zero3_reduce_adamw_hybrid.restype = C.c_int
    L.zero3_node_sum.argtypes = [vp, i32, vp, i32, i32, vp, vp]
    L.zero3_node_sum.restype = C.c_int
    L.zero3_fold_adamw.argtypes = [vp, i32, i32, vp, vp, vp, vp, vp, i32, C.POINTER(AdamW), vp]
    L.zero3_fold_adamw.restype = C.c_int
    L.zero3_reduce_adamw_gather.argtypes = [vp, i32, vp, i32, vp, vp, vp, vp, vp, i32, i32,
                                            C.POINTER(AdamW), vp]
    L.zero3_reduce_adamw_gather.restype = C.c_int
    L.zero3_step_scalars.argtypes = [C.POINTER(AdamW), vp]
    L.zero3_step_scalars.restype = C.c_int
    L.zero3_reduce_adamw_dev.argtypes = [vp, i32, vp, i32, vp, vp, vp, vp, vp, i32, i32, vp, vp]
    L.zero3_reduce_adamw_dev.restype = C.c_int
    L.zero3_gather_block.argtypes = [vp, vp, vp, vp, vp]
    L.zero3_gather_block.restype = C.c_int
    L.zero3_reduce_scatter.argtypes = [vp, i32, vp, i32, i32, vp, vp]
    L.zero3_reduce_scatter.restype = C.c_int
    L.zero3_host_adamw.argtypes = [i64, vp, i32, vp, vp, vp, vp, C.POINTER(AdamW), i32]
    L.zero3_host_adamw.restype = C.c_int
    L.zero3_ipc_export.argtypes = [vp, vp, C.POINTER(i64), C.POINTER(i64)]
    L.zero3_ipc_export.restype = C.c_int
    L.zero3_ipc_import.argtypes = [vp, i64, C.POINTER(vp), C.POINTER(vp)]
    L.zero3_ipc_import.restype = C.c_int
    L.zero3_ipc_close.argtypes = [vp]
    L.zero3_ipc_close.restype = C.c_int
    return L


_lib = _load()


def lib() -> C.CDLL:
    return _lib


def status_string(status: int) -> str:
    return _lib.zero3_status_string(status).decode()


def _check(rc: int, what: str) -> None:
    if rc != Z3_OK:
        raise Zero3Error(rc, what)


# ------------------------------------------------------------------- plan
def tensor_specs(shapes: Sequence[Sequence[int]]):
    """A host array of z3_tensor_spec for the given row-major shapes."""
    shapes = [tuple(int(x) for x in s) for s in shapes]
    specs = (TensorSpec * max(1, len(shapes)))()
    for i, s in enumerate(shapes):
        if len(s) > 4:
            raise ValueError("at most 4 dimensions per tensor")
        numel = 1
        for x in s:
            numel *= x
        specs[i].numel = numel
        specs[i].ndim = len(s)
        for k, x in enumerate(s):
            specs[i].shape[k] = x
    return specs


class Plan:
    """A flat-parameter plan (owns the C plan object).  `specs` may be passed in,
    prebuilt by tensor_specs(shapes), to re-plan the same block cheaply."""

    def __init__(self, shapes: Sequence[Sequence[int]], D: int, align_elems: int = 128, specs=None):
        self.shapes = [tuple(int(x) for x in s) for s in shapes]
        n = len(self.shapes)
        if specs is None:
            specs = tensor_specs(self.shapes)
        h = C.c_void_p()
        _check(_lib.zero3_plan(specs, n, D, align_elems, C.byref(h)), "zero3_plan")
        self._h = h
        self._free = _lib.zero3_plan_free   # held here: module globals may be gone when __del__ runs at exit
        d, nt, a = C.c_int32(), C.c_int32(), C.c_int32()
        N, N_pad, S = C.c_int64(), C.c_int64(), C.c_int64()
        _check(_lib.zero3_plan_info(h, C.byref(d), C.byref(nt), C.byref(a), C.byref(N),
                                    C.byref(N_pad), C.byref(S)), "zero3_plan_info")
        self.D, self.n_tensors, self.align_elems = d.value, nt.value, a.value
        self.N, self.N_pad, self.S = N.value, N_pad.value, S.value
        self._runs = None

    def _tensor_runs(self):
        if self._runs is None:
            runs = [zero3_plan_tensor(self, i) for i in range(self.n_tensors)]
            self._runs = ([o for o, _ in runs], [k for _, k in runs])
        return self._runs

    @property
    def offsets(self):
        return self._tensor_runs()[0]

    @property
    def numels(self):
        return self._tensor_runs()[1]

    @property
    def handle(self) -> C.c_void_p:
        return self._h

    def rank_range(self, r: int):
        return zero3_plan_rank(self, r)

    def views(self, flat: torch.Tensor):
        """Zero-copy per-tensor views of a gathered flat block (the unflatten)."""
        if flat.numel() < self.N_pad:
            raise ValueError("flat block smaller than N_pad")
        return [flat[o:o + k].view(s) for o, k, s in zip(self.offsets, self.numels, self.shapes)]

    def __del__(self):
        h, free = getattr(self, "_h", None), getattr(self, "_free", None)
        if h is not None and h.value and free is not None:
            free(h)
            self._h = None


def zero3_plan(shapes, D: int, align_elems: int = 128) -> Plan:
    return Plan(shapes, D, align_elems)


def zero3_plan_tensor(plan: Plan, i: int):
    off, n = C.c_int64(), C.c_int64()
    _check(_lib.zero3_plan_tensor(plan.handle, i, C.byref(off), C.byref(n)), "zero3_plan_tensor")
    return off.value, n.value


def zero3_plan_rank(plan: Plan, r: int):
    b, e = C.c_int64(), C.c_int64()
    _check(_lib.zero3_plan_rank(plan.handle, r, C.byref(b), C.byref(e)), "zero3_plan_rank")
    return b.value, e.value


def zero3_memory_bytes(N: int, D: int, stage: int) -> int:
    out = C.c_int64()
    _check(_lib.zero3_memory_bytes(N, D, stage, C.byref(out)), "zero3_memory_bytes")
    return out.value


def zero3_transient_bytes(block_params: int, n_buffers: int = 1) -> int:
    out = C.c_int64()
    _check(_lib.zero3_transient_bytes(block_params, n_buffers, C.byref(out)), "zero3_transient_bytes")
    return out.value


def zero3_allgather_bytes(block_params: int, n_blocks: int, D: int) -> int:
    out = C.c_int64()
    _check(_lib.zero3_allgather_bytes(block_params, n_blocks, D, C.byref(out)), "zero3_allgather_bytes")
    return out.value


# ------------------------------------------------------------- marshalling
def adamw(lr=3e-4, beta1=0.9, beta2=0.95, eps=1e-8, weight_decay=0.1, step=1) -> AdamW:
    return AdamW(lr, beta1, beta2, eps, weight_decay, step)


def _dev_tensor(t: torch.Tensor, dtype: torch.dtype, need: int, name: str, host_ok: bool = False) -> int:
    """The address of a contiguous tensor the kernels may access: a CUDA tensor, or
    with host_ok a page-locked host tensor (mapped into the device's address space,
    so the kernel reaches it over PCIe)."""
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda and not (host_ok and t.device.type == "cpu" and t.is_pinned()):
        raise ValueError(f"{name} must be a CUDA tensor" + (" or a pinned host tensor" if host_ok else ""))
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if t.numel() < need:
        raise ValueError(f"{name} holds {t.numel()} elements, needs {need}")
    return t.data_ptr()


def _launch_device(*candidates) -> int:
    """The device the kernels launch on: that of the first local CUDA tensor given
    (the state and outputs come first; contributions and shards may be mapped
    from peer GPUs)."""
    for t in candidates:
        if isinstance(t, torch.Tensor) and t.is_cuda:
            return t.get_device()
    raise ValueError("no CUDA tensor among the arguments")


def _call_on(dev: int, fn, *args) -> int:
    """fn(*args) with `dev` as the current CUDA device (the library launches on the
    current device); the device switch is skipped when it is current already."""
    if torch.cuda.current_device() == dev:
        return fn(*args)
    with torch.cuda.device(dev):
        return fn(*args)


def _stream_handle(stream, device) -> int:
    if stream is None:
        return torch.cuda.current_stream(device).cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def zero3_reduce_adamw(plan: Plan, rank: int, contrib: Sequence[torch.Tensor], master: torch.Tensor,
                       exp_avg: torch.Tensor, exp_avg_sq: torch.Tensor, work_bf16: torch.Tensor,
                       hp: AdamW, contrib_layout: int = Z3_CONTRIB_FULL,
                       reduce_dtype: int = Z3_REDUCE_FP32, stream=None) -> None:
    """Fused reduce-scatter reduction + AdamW + bf16 cast (see include/zero3.h)."""
    if len(contrib) != plan.D:
        raise ValueError(f"need {plan.D} contributions, got {len(contrib)}")
    n = plan.N_pad if rank < 0 else plan.S
    c_need = plan.N_pad if contrib_layout == Z3_CONTRIB_FULL else plan.S
    ptrs = (C.c_void_p * plan.D)()
    for d, c in enumerate(contrib):
        ptrs[d] = _dev_tensor(c, torch.bfloat16, c_need, f"contrib[{d}]")
    mp = _dev_tensor(master, torch.float32, n, "master", host_ok=True)
    ap = _dev_tensor(exp_avg, torch.float32, n, "exp_avg", host_ok=True)
    vp = _dev_tensor(exp_avg_sq, torch.float32, n, "exp_avg_sq", host_ok=True)
    wp = _dev_tensor(work_bf16, torch.bfloat16, n, "work_bf16", host_ok=True)
    dev = _launch_device(work_bf16, master, *contrib)
    rc = _call_on(dev, _lib.zero3_reduce_adamw, plan.handle, rank, ptrs, contrib_layout, mp, ap, vp, wp,
                  reduce_dtype, C.byref(hp), _stream_handle(stream, dev))
    _check(rc, "zero3_reduce_adamw")


def zero3_reduce_adamw_hybrid(plan: Plan, rank: int, n_nodes: int, contrib: Sequence[torch.Tensor],
                              master: torch.Tensor, exp_avg: torch.Tensor, exp_avg_sq: torch.Tensor,
                              work_bf16: torch.Tensor, hp: AdamW, contrib_layout: int = Z3_CONTRIB_FULL,
                              reduce_dtype: int = Z3_REDUCE_FP32, stream=None) -> None:
    """The HYBRID_SHARD step: n_nodes nodes of plan.D ranks, contrib[k * D + d] from
    local rank d of node k; node sums, then the node sums across nodes, then
    1/(n_nodes * D), AdamW and the bf16 cast (see include/zero3.h)."""
    if n_nodes < 1 or n_nodes * plan.D > Z3_D_MAX:
        raise ValueError(f"n_nodes * D must be in [1, {Z3_D_MAX}], got {n_nodes} * {plan.D}")
    if len(contrib) != n_nodes * plan.D:
        raise ValueError(f"need {n_nodes * plan.D} contributions, got {len(contrib)}")
    n = plan.N_pad if rank < 0 else plan.S
    c_need = plan.N_pad if contrib_layout == Z3_CONTRIB_FULL else plan.S
    ptrs = (C.c_void_p * len(contrib))()
    for d, c in enumerate(contrib):
        ptrs[d] = _dev_tensor(c, torch.bfloat16, c_need, f"contrib[{d}]")
    mp = _dev_tensor(master, torch.float32, n, "master", host_ok=True)
    ap = _dev_tensor(exp_avg, torch.float32, n, "exp_avg", host_ok=True)
    vp = _dev_tensor(exp_avg_sq, torch.float32, n, "exp_avg_sq", host_ok=True)
    wp = _dev_tensor(work_bf16, torch.bfloat16, n, "work_bf16", host_ok=True)
    dev = _launch_device(work_bf16, master, *contrib)
    rc = _call_on(dev, _lib.zero3_reduce_adamw_hybrid, plan.handle, rank, n_nodes, ptrs, contrib_layout, mp, ap,
                  vp, wp, reduce_dtype, C.byref(hp), _stream_handle(stream, dev))
    _check(rc, "zero3_reduce_adamw_hybrid")


def _node_sum_dtype(reduce_dtype: int) -> torch.dtype:
    return torch.float32 if reduce_dtype == Z3_REDUCE_FP32 else torch.bfloat16


def zero3_node_sum(plan: Plan, rank: int, contrib: Sequence[torch.Tensor], node_sum: torch.Tensor,
                   contrib_layout: int = Z3_CONTRIB_FULL, reduce_dtype: int = Z3_REDUCE_FP32, stream=None) -> None:
    """HYBRID_SHARD across nodes, part 1: this node's rank-ordered, unscaled sum of
    its plan.D contributions for the owned partition(s), written to node_sum
    (float32 for the fp32 reduce, bfloat16 for the bf16 reduce; see include/zero3.h)."""
    if len(contrib) != plan.D:
        raise ValueError(f"need {plan.D} contributions, got {len(contrib)}")
    n = plan.N_pad if rank < 0 else plan.S
    c_need = plan.N_pad if contrib_layout == Z3_CONTRIB_FULL else plan.S
    ptrs = (C.c_void_p * plan.D)()
    for d, c in enumerate(contrib):
        ptrs[d] = _dev_tensor(c, torch.bfloat16, c_need, f"contrib[{d}]")
    op = _dev_tensor(node_sum, _node_sum_dtype(reduce_dtype), n, "node_sum")
    dev = _launch_device(node_sum, *contrib)
    rc = _call_on(dev, _lib.zero3_node_sum, plan.handle, rank, ptrs, contrib_layout, reduce_dtype, op,
                  _stream_handle(stream, dev))
    _check(rc, "zero3_node_sum")


def zero3_fold_adamw(plan: Plan, rank: int, node_sums: Sequence[torch.Tensor], master: torch.Tensor,
                     exp_avg: torch.Tensor, exp_avg_sq: torch.Tensor, work_bf16: torch.Tensor, hp: AdamW,
                     reduce_dtype: int = Z3_REDUCE_FP32, stream=None) -> None:
    """HYBRID_SHARD across nodes, part 2: the node sums (node order) folded, scaled
    by 1/(len(node_sums) * plan.D), AdamW and the bf16 cast (see include/zero3.h)."""
    if not 1 <= len(node_sums) <= Z3_D_MAX:
        raise ValueError(f"need 1..{Z3_D_MAX} node sums, got {len(node_sums)}")
    n = plan.N_pad if rank < 0 else plan.S
    sp = (C.c_void_p * len(node_sums))()
    for k, x in enumerate(node_sums):
        sp[k] = _dev_tensor(x, _node_sum_dtype(reduce_dtype), n, f"node_sums[{k}]")
    mp = _dev_tensor(master, torch.float32, n, "master", host_ok=True)
    ap = _dev_tensor(exp_avg, torch.float32, n, "exp_avg", host_ok=True)
    vp = _dev_tensor(exp_avg_sq, torch.float32, n, "exp_avg_sq", host_ok=True)
    wp = _dev_tensor(work_bf16, torch.bfloat16, n, "work_bf16", host_ok=True)
    dev = _launch_device(work_bf16, master, *node_sums)
    rc = _call_on(dev, _lib.zero3_fold_adamw, plan.handle, rank, len(node_sums), sp, mp, ap, vp, wp, reduce_dtype,
                  C.byref(hp), _stream_handle(stream, dev))
    _check(rc, "zero3_fold_adamw")


def zero3_reduce_adamw_gather(plan: Plan, rank: int, contrib: Sequence[torch.Tensor], master: torch.Tensor,
                              exp_avg: torch.Tensor, exp_avg_sq: torch.Tensor,
                              work_bf16: Optional[torch.Tensor], gathered: Sequence[torch.Tensor], hp: AdamW,
                              contrib_layout: int = Z3_CONTRIB_FULL, reduce_dtype: int = Z3_REDUCE_FP32,
                              stream=None) -> None:
    """zero3_reduce_adamw whose kernel also writes every new bf16 weight into its place
    in each gathered block (N_pad bf16 each); work_bf16 may be None (see include/zero3.h)."""
    if len(contrib) != plan.D:
        raise ValueError(f"need {plan.D} contributions, got {len(contrib)}")
    if not 1 <= len(gathered) <= Z3_GATHER_MAX:
        raise ValueError(f"need 1..{Z3_GATHER_MAX} gathered blocks, got {len(gathered)}")
    n = plan.N_pad if rank < 0 else plan.S
    c_need = plan.N_pad if contrib_layout == Z3_CONTRIB_FULL else plan.S
    ptrs = (C.c_void_p * plan.D)()
    for d, c in enumerate(contrib):
        ptrs[d] = _dev_tensor(c, torch.bfloat16, c_need, f"contrib[{d}]")
    gp = (C.c_void_p * len(gathered))()
    for k, g in enumerate(gathered):
        gp[k] = _dev_tensor(g, torch.bfloat16, plan.N_pad, f"gathered[{k}]")
    mp = _dev_tensor(master, torch.float32, n, "master", host_ok=True)
    ap = _dev_tensor(exp_avg, torch.float32, n, "exp_avg", host_ok=True)
    vp = _dev_tensor(exp_avg_sq, torch.float32, n, "exp_avg_sq", host_ok=True)
    wp = None if work_bf16 is None else _dev_tensor(work_bf16, torch.bfloat16, n, "work_bf16", host_ok=True)
    dev = _launch_device(work_bf16, master, *contrib)
    rc = _call_on(dev, _lib.zero3_reduce_adamw_gather, plan.handle, rank, ptrs, contrib_layout, mp, ap, vp, wp,
                  gp, len(gathered), reduce_dtype, C.byref(hp), _stream_handle(stream, dev))
    _check(rc, "zero3_reduce_adamw_gather")


def zero3_step_scalars(hp: AdamW, out: Optional[int] = None):
    """The Z3_SCALARS fp32 scalars of one AdamW step.  With `out` (a host address of
    Z3_SCALARS floats, e.g. a pinned tensor's data_ptr()) they are written there;
    otherwise they are returned as a list."""
    if out is not None:
        _check(_lib.zero3_step_scalars(C.byref(hp), out), "zero3_step_scalars")
        return None
    buf = (C.c_float * Z3_SCALARS)()
    _check(_lib.zero3_step_scalars(C.byref(hp), buf), "zero3_step_scalars")
    return list(buf)


def zero3_reduce_adamw_dev(plan: Plan, rank: int, contrib: Sequence[torch.Tensor], master: torch.Tensor,
                           exp_avg: torch.Tensor, exp_avg_sq: torch.Tensor, work_bf16: Optional[torch.Tensor],
                           gathered: Sequence[torch.Tensor], scalars: torch.Tensor,
                           contrib_layout: int = Z3_CONTRIB_FULL, reduce_dtype: int = Z3_REDUCE_FP32,
                           stream=None) -> None:
    """The fused kernel reading the step's scalars from `scalars` (a CUDA float32
    tensor of Z3_SCALARS elements), so that the launch can be captured in a CUDA
    graph (see include/zero3.h)."""
    if len(contrib) != plan.D:
        raise ValueError(f"need {plan.D} contributions, got {len(contrib)}")
    if len(gathered) > Z3_GATHER_MAX:
        raise ValueError(f"at most {Z3_GATHER_MAX} gathered blocks")
    n = plan.N_pad if rank < 0 else plan.S
    c_need = plan.N_pad if contrib_layout == Z3_CONTRIB_FULL else plan.S
    ptrs = (C.c_void_p * plan.D)()
    for d, c in enumerate(contrib):
        ptrs[d] = _dev_tensor(c, torch.bfloat16, c_need, f"contrib[{d}]")
    gp = (C.c_void_p * max(1, len(gathered)))()
    for k, g in enumerate(gathered):
        gp[k] = _dev_tensor(g, torch.bfloat16, plan.N_pad, f"gathered[{k}]")
    sp = _dev_tensor(scalars, torch.float32, Z3_SCALARS, "scalars")
    mp = _dev_tensor(master, torch.float32, n, "master", host_ok=True)
    ap = _dev_tensor(exp_avg, torch.float32, n, "exp_avg", host_ok=True)
    vp = _dev_tensor(exp_avg_sq, torch.float32, n, "exp_avg_sq", host_ok=True)
    wp = None if work_bf16 is None else _dev_tensor(work_bf16, torch.bfloat16, n, "work_bf16", host_ok=True)
    dev = _launch_device(scalars, work_bf16, master, *contrib)
    rc = _call_on(dev, _lib.zero3_reduce_adamw_dev, plan.handle, rank, ptrs, contrib_layout, mp, ap, vp, wp,
                  gp if gathered else None, len(gathered), reduce_dtype, sp, _stream_handle(stream, dev))
    _check(rc, "zero3_reduce_adamw_dev")


def zero3_gather_block(plan: Plan, shards: Sequence[torch.Tensor], flat_out: Optional[torch.Tensor] = None,
                       tensor_out: Optional[Sequence[Optional[torch.Tensor]]] = None, stream=None) -> None:
    """All-gather of the D bf16 shards into the flat block and/or per-tensor buffers."""
    if len(shards) != plan.D:
        raise ValueError(f"need {plan.D} shards, got {len(shards)}")
    if tensor_out is not None and len(tensor_out) != plan.n_tensors:
        raise ValueError(f"need {plan.n_tensors} tensor outputs, got {len(tensor_out)}")
    sp = (C.c_void_p * plan.D)()
    for r, s in enumerate(shards):
        sp[r] = _dev_tensor(s, torch.bfloat16, plan.S, f"shards[{r}]")
    fp = None if flat_out is None else _dev_tensor(flat_out, torch.bfloat16, plan.N_pad, "flat_out")
    tp = None
    if tensor_out is not None:
        tp = (C.c_void_p * max(1, plan.n_tensors))()
        for i, t in enumerate(tensor_out):
            tp[i] = None if t is None else _dev_tensor(t, torch.bfloat16, plan.numels[i], f"tensor_out[{i}]")
    dev = _launch_device(flat_out, *(tensor_out or []), *shards)
    rc = _call_on(dev, _lib.zero3_gather_block, plan.handle, sp, fp, tp, _stream_handle(stream, dev))
    _check(rc, "zero3_gather_block")


def zero3_reduce_scatter(plan: Plan, rank: int, contrib: Sequence[torch.Tensor], grad: torch.Tensor,
                         contrib_layout: int = Z3_CONTRIB_FULL, reduce_dtype: int = Z3_REDUCE_FP32,
                         stream=None) -> None:
    """The reduce-scatter's reduction alone: the averaged gradient of the owned
    partition(s) into grad (float32 for the fp32 reduce, bfloat16 for the bf16
    reduce; see include/zero3.h)."""
    if len(contrib) != plan.D:
        raise ValueError(f"need {plan.D} contributions, got {len(contrib)}")
    n = plan.N_pad if rank < 0 else plan.S
    c_need = plan.N_pad if contrib_layout == Z3_CONTRIB_FULL else plan.S
    ptrs = (C.c_void_p * plan.D)()
    for d, c in enumerate(contrib):
        ptrs[d] = _dev_tensor(c, torch.bfloat16, c_need, f"contrib[{d}]")
    gp = _dev_tensor(grad, _node_sum_dtype(reduce_dtype), n, "grad", host_ok=True)
    dev = _launch_device(grad, *contrib)
    rc = _call_on(dev, _lib.zero3_reduce_scatter, plan.handle, rank, ptrs, contrib_layout, reduce_dtype, gp,
                  _stream_handle(stream, dev))
    _check(rc, "zero3_reduce_scatter")


def _host_tensor(t: torch.Tensor, dtype: torch.dtype, need: int, name: str) -> int:
    if not isinstance(t, torch.Tensor) or t.device.type != "cpu":
        raise ValueError(f"{name} must be a host (CPU) tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if t.numel() < need:
        raise ValueError(f"{name} holds {t.numel()} elements, needs {need}")
    return t.data_ptr()


def zero3_host_adamw(grad: torch.Tensor, master: torch.Tensor, exp_avg: torch.Tensor, exp_avg_sq: torch.Tensor,
                     work_bf16: torch.Tensor, hp: AdamW, n: Optional[int] = None, n_threads: int = 0) -> None:
    """AdamW and the bf16 cast of n elements in host memory, on host threads
    (n defaults to grad.numel()); grad is float32 or bfloat16 (see include/zero3.h).
    Synchronous; the GIL is released while it runs."""
    n = grad.numel() if n is None else n
    gdt = Z3_REDUCE_FP32 if grad.dtype == torch.float32 else Z3_REDUCE_BF16
    gp = _host_tensor(grad, torch.float32 if gdt == Z3_REDUCE_FP32 else torch.bfloat16, n, "grad")
    mp = _host_tensor(master, torch.float32, n, "master")
    ap = _host_tensor(exp_avg, torch.float32, n, "exp_avg")
    vp = _host_tensor(exp_avg_sq, torch.float32, n, "exp_avg_sq")
    wp = _host_tensor(work_bf16, torch.bfloat16, n, "work_bf16")
    _check(_lib.zero3_host_adamw(n, gp, gdt, mp, ap, vp, wp, C.byref(hp), n_threads), "zero3_host_adamw")


# ------------------------------------------------- peer memory through CUDA IPC
Z3_IPC_HANDLE_BYTES = 64


class _DeviceArray:
    """A device address range described by the CUDA array interface, so that torch
    can view it as a tensor without copying (used for imported peer memory)."""

    def __init__(self, ptr: int, numel: int, typestr: str):
        self.__cuda_array_interface__ = {"shape": (numel,), "typestr": typestr, "data": (ptr, False),
                                         "strides": None, "version": 2}


def zero3_ipc_export(t: torch.Tensor):
    """(handle bytes, byte offset of t in its allocation, allocation bytes) of a
    contiguous CUDA tensor, for another process's zero3_ipc_import."""
    if not isinstance(t, torch.Tensor) or not t.is_cuda or not t.is_contiguous():
        raise ValueError("zero3_ipc_export needs a contiguous CUDA tensor")
    h = (C.c_char * Z3_IPC_HANDLE_BYTES)()
    off, size = C.c_int64(), C.c_int64()
    rc = _call_on(t.get_device(), _lib.zero3_ipc_export, t.data_ptr(), h, C.byref(off), C.byref(size))
    _check(rc, "zero3_ipc_export")
    return bytes(h), off.value, size.value


def zero3_ipc_import(handle: bytes, offset: int, size: int, numel: int, dtype: torch.dtype, device: int):
    """Map another process's exported allocation into `device`'s address space
    (peer access to the owning GPU enabled as needed) and view the `numel`
    elements of `dtype` at `offset` as a tensor.  Returns (tensor, mapping base
    for zero3_ipc_close).  The tensor aliases the other process's memory; only
    the library's kernels should touch it, and only until the mapping is closed."""
    if len(handle) != Z3_IPC_HANDLE_BYTES:
        raise ValueError("an IPC handle is 64 bytes")
    itemsize = torch.empty((), dtype=dtype).element_size()
    if offset < 0 or offset + numel * itemsize > size:
        raise ValueError(f"{numel} elements at byte {offset} exceed the exported allocation of {size} bytes")
    buf = (C.c_char * Z3_IPC_HANDLE_BYTES).from_buffer_copy(handle)
    ptr, base = C.c_void_p(), C.c_void_p()
    _check(_call_on(device, _lib.zero3_ipc_import, buf, offset, C.byref(ptr), C.byref(base)), "zero3_ipc_import")
    raw = {2: "<i2", 4: "<f4"}.get(itemsize)
    if raw is None:
        raise TypeError(f"no peer view for {dtype}")
    t = torch.as_tensor(_DeviceArray(ptr.value, numel, raw))
    return (t.view(dtype) if t.dtype != dtype else t), base.value


def zero3_ipc_close(base: int, device: int) -> None:
    """Release one import of the mapping at `base` (the last release unmaps it)."""
    _check(_call_on(device, _lib.zero3_ipc_close, base), "zero3_ipc_close")
