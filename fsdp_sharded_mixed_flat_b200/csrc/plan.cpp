// plan.cpp -- the flat-parameter planner and the memory ledger (host only).
//
// "7.10 — Fully-sharded data parallel (FSDP / ZeRO-3)", §3: rank r owns a
// partition P_r of roughly 1/D of the parameters; §2: the per-stage byte
// formulas; §5.2: the transient buffer of the gathered block.
#include <cstdint>
#include <limits>
#include <new>

#include "plan_impl.h"
#include "zero3.h"

namespace {

constexpr int64_t kMaxElems = int64_t(1) << 62;

// a + b, or -1 if the sum leaves [0, limit].
int64_t add_checked(int64_t a, int64_t b, int64_t limit) {
    if (a < 0 || b < 0 || a > limit - b) return -1;
    return a + b;
}

// a * b for non-negative operands, or -1 on overflow of int64_t.
int64_t mul_checked(int64_t a, int64_t b) {
    if (a < 0 || b < 0) return -1;
    if (a != 0 && b > std::numeric_limits<int64_t>::max() / a) return -1;
    return a * b;
}

// ceil(a / b) for a >= 0, b >= 1.
int64_t ceil_div(int64_t a, int64_t b) { return a / b + (a % b != 0 ? 1 : 0); }

}  // namespace

extern "C" {

Z3_API const char* zero3_status_string(int status) {
    switch (status) {
    case Z3_OK: return "ok";
    case Z3_EINVAL: return "invalid argument";
    case Z3_EALIGN: return "misaligned pointer";
    case Z3_ENOMEM: return "host allocation failed";
    case Z3_ECUDA: return "CUDA error";
    case Z3_EOVERFLOW: return "size overflow";
    default: return "unknown status";
    }
}

Z3_API int zero3_plan(const z3_tensor_spec* t, int32_t n_tensors, int32_t D, int32_t align_elems,
                      z3_plan** out) {
    if (out == nullptr) return Z3_EINVAL;
    *out = nullptr;
    if (n_tensors < 0 || (n_tensors > 0 && t == nullptr)) return Z3_EINVAL;
    if (D < 1 || D > Z3_D_MAX || align_elems < 1) return Z3_EINVAL;

    z3_plan* p = new (std::nothrow) z3_plan;
    if (p == nullptr) return Z3_ENOMEM;
    try {
        p->offset.resize(static_cast<size_t>(n_tensors));
        p->numel.resize(static_cast<size_t>(n_tensors));
    } catch (...) {
        delete p;
        return Z3_ENOMEM;
    }
    int64_t N = 0;
    for (int32_t i = 0; i < n_tensors; ++i) {
        const z3_tensor_spec& s = t[i];
        if (s.numel < 0 || s.ndim < 0 || s.ndim > 4) { delete p; return Z3_EINVAL; }
        int64_t prod = 1;
        for (int32_t k = 0; k < s.ndim; ++k) {
            prod = mul_checked(prod, s.shape[k]);
            if (prod < 0) { delete p; return Z3_EINVAL; }
        }
        if (prod != s.numel) { delete p; return Z3_EINVAL; }
        p->offset[i] = N;   // list order, no gap between tensors
        p->numel[i] = s.numel;
        N = add_checked(N, s.numel, kMaxElems);
        if (N < 0) { delete p; return Z3_EOVERFLOW; }
    }
    const int64_t unit = int64_t(D) * int64_t(align_elems);  // <= 2^6 * 2^31
    const int64_t units = ceil_div(N, unit);
    const int64_t N_pad = mul_checked(units, unit);
    if (N_pad < 0 || N_pad > kMaxElems) { delete p; return Z3_EOVERFLOW; }
    p->D = D;
    p->A = align_elems;
    p->N = N;
    p->N_pad = N_pad;
    p->S = N_pad / D;
    *out = p;
    return Z3_OK;
}

Z3_API void zero3_plan_free(z3_plan* p) { delete p; }

Z3_API int zero3_plan_info(const z3_plan* p, int32_t* D, int32_t* n_tensors, int32_t* align_elems,
                           int64_t* N, int64_t* N_pad, int64_t* S) {
    if (p == nullptr) return Z3_EINVAL;
    if (D) *D = p->D;
    if (n_tensors) *n_tensors = static_cast<int32_t>(p->numel.size());
    if (align_elems) *align_elems = p->A;
    if (N) *N = p->N;
    if (N_pad) *N_pad = p->N_pad;
    if (S) *S = p->S;
    return Z3_OK;
}

Z3_API int zero3_plan_tensor(const z3_plan* p, int32_t i, int64_t* offset, int64_t* numel) {
    if (p == nullptr || i < 0 || static_cast<size_t>(i) >= p->numel.size()) return Z3_EINVAL;
    if (offset) *offset = p->offset[i];
    if (numel) *numel = p->numel[i];
    return Z3_OK;
}

Z3_API int zero3_plan_rank(const z3_plan* p, int32_t r, int64_t* begin, int64_t* end_real) {
    if (p == nullptr || r < 0 || r >= p->D) return Z3_EINVAL;
    const int64_t b = int64_t(r) * p->S;
    int64_t e = b + p->S;
    if (e > p->N) e = p->N;
    if (e < b) e = b;
    if (begin) *begin = b;
    if (end_real) *end_real = e;
    return Z3_OK;
}

Z3_API int zero3_memory_bytes(int64_t N, int32_t D, int32_t stage, int64_t* bytes) {
    if (bytes == nullptr || N < 0 || D < 1) return Z3_EINVAL;
    // Every product below is checked; sharded terms are rounded up to a byte.
    const int64_t w = mul_checked(2, N), g = mul_checked(6, N), o = mul_checked(12, N);
    const int64_t all = mul_checked(20, N);
    if (w < 0 || g < 0 || o < 0 || all < 0) return Z3_EOVERFLOW;
    int64_t total = -1;
    switch (stage) {
    case Z3_STAGE_DDP: total = all; break;
    case Z3_STAGE_ZERO1: total = add_checked(add_checked(ceil_div(o, D), w, INT64_MAX), g, INT64_MAX); break;
    case Z3_STAGE_ZERO2: total = add_checked(ceil_div(mul_checked(18, N), D), w, INT64_MAX); break;
    case Z3_STAGE_ZERO3: total = ceil_div(all, D); break;
    default: return Z3_EINVAL;
    }
    if (total < 0) return Z3_EOVERFLOW;
    *bytes = total;
    return Z3_OK;
}

Z3_API int zero3_transient_bytes(int64_t block_params, int32_t n_buffers, int64_t* bytes) {
    if (bytes == nullptr || block_params < 0 || n_buffers < 0) return Z3_EINVAL;
    const int64_t one = mul_checked(2, block_params);
    const int64_t all = one < 0 ? -1 : mul_checked(one, n_buffers);
    if (all < 0) return Z3_EOVERFLOW;
    *bytes = all;
    return Z3_OK;
}

Z3_API int zero3_allgather_bytes(int64_t block_params, int32_t n_blocks, int32_t D, int64_t* bytes) {
    if (bytes == nullptr || block_params < 0 || n_blocks < 0 || D < 1) return Z3_EINVAL;
    const int64_t one = mul_checked(2, block_params);            // one block in bf16
    const int64_t all = one < 0 ? -1 : mul_checked(one, n_blocks);
    if (all < 0) return Z3_EOVERFLOW;
    // all * (D - 1) / D rounded up, which is exactly all - floor(all / D)
    *bytes = all - all / D;
    return Z3_OK;
}

}  // extern "C"
