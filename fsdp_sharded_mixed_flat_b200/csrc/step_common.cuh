// step_common.cuh -- the pieces every optimiser-step kernel of this library
// shares: the AdamW element update (its scalars come from adamw_scalars.h),
// the bf16 conversions and the 16-byte memory accesses.
//
// Pages: "7.10 — Fully-sharded data parallel (FSDP / ZeRO-3)", §3 (rank r
// updates P_r from its fp32 master, m, v and gradient slice); "Building GPT
// from Scratch — Part 8", "Mixed Precision: Cutting Memory in Half" (fp32
// master, bf16 working weights).  AdamW with decoupled weight decay and
// bias-corrected moments (Loshchilov & Hutter, "Decoupled Weight Decay
// Regularization").
//
// Every arithmetic step is an explicitly rounded fp32 intrinsic, so nothing is
// contracted into an FMA and the results are fixed by the stated operation
// order.  Included by several translation units; everything has internal
// linkage.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>

#include "adamw_scalars.h"
#include "zero3.h"

namespace {

__device__ __forceinline__ float lo_bf16(uint32_t x) { return __uint_as_float(x << 16); }
__device__ __forceinline__ float hi_bf16(uint32_t x) { return __uint_as_float(x & 0xFFFF0000u); }
__device__ __forceinline__ float bf16_of(uint16_t h) { return __uint_as_float(uint32_t(h) << 16); }

// 16-byte load (default caching) and streaming store.  Among the cache hints
// measured on B200 for the fused step (streaming, read-only, last-use and
// default loads; streaming and default stores), default loads with streaming
// stores moved the most bytes per second at every D.
template <class T>
__device__ __forceinline__ T ld16(const T* p) { return *p; }
template <class T>
__device__ __forceinline__ void st16(T* p, const T& v) { __stcs(p, v); }

// fp32 -> nearest-even bf16 -> fp32.
__device__ __forceinline__ float round_to_bf16(float x) {
    return __bfloat162float(__float2bfloat16_rn(x));
}

// Two fp32 values -> two nearest-even bf16 in one 32-bit word (lo in bits 0..15).
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&h);
}

// Two bf16 values added pairwise by the packed hardware add, which rounds the
// exact sum to the nearest-even bf16.  That equals rounding the fp32 sum to
// bf16: double rounding through a format with more than 2p + 2 significand
// bits is innocuous (Figueroa, "When is double rounding innocuous?", 1995),
// and fp32's 24 bits exceed 18 for bf16's p = 8, also in the shared subnormal
// range, where both formats lose the same number of leading bits.
__device__ __forceinline__ uint32_t add_bf16x2(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("add.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

// Fold one rank's 8 bf16 values (one 16-byte vector) into fp32 accumulators.
__device__ __forceinline__ void fold8_fp32(float (&acc)[8], const uint4& q, bool first) {
    const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const float a = lo_bf16(w[k]), b = hi_bf16(w[k]);
        acc[2 * k] = first ? a : __fadd_rn(acc[2 * k], a);
        acc[2 * k + 1] = first ? b : __fadd_rn(acc[2 * k + 1], b);
    }
}

// Fold one rank's 8 bf16 values into packed bf16 accumulators (element 2k in
// the low half of word k).
__device__ __forceinline__ void fold8_bf16(uint32_t (&acc)[4], const uint4& q, bool first) {
    const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) acc[k] = first ? w[k] : add_bf16x2(acc[k], w[k]);
}

// One partial sum in the reduce dtype: the fp32 sum, rounded to bf16 in bf16 mode.
template <int MODE>
__device__ __forceinline__ float add_in(float x, float y) {
    const float s = __fadd_rn(x, y);
    return MODE == Z3_REDUCE_FP32 ? s : round_to_bf16(s);
}

// One AdamW element; each step a single fp32 operation rounded to nearest-even.
__device__ __forceinline__ void adamw_elem(const AdamScalars& s, float g, float& p, float& m, float& v) {
    const float p1 = __fmul_rn(p, s.decay);
    const float m1 = __fadd_rn(__fmul_rn(s.b1, m), __fmul_rn(s.omb1, g));
    const float v1 = __fadd_rn(__fmul_rn(s.b2, v), __fmul_rn(s.omb2, __fmul_rn(g, g)));
    const float denom = __fadd_rn(__fmul_rn(__fsqrt_rn(v1), s.inv_sqrt_bc2), s.eps);
    const float delta = __fmul_rn(s.step_size, __fdiv_rn(m1, denom));
    p = __fsub_rn(p1, delta);
    m = m1;
    v = v1;
}

// The scalars of a step read from device memory (a captured CUDA graph is
// replayed with only this 32-byte buffer rewritten in between).
__device__ __forceinline__ AdamScalars load_scalars(const AdamScalars* p) {
    const float4 x = __ldg(reinterpret_cast<const float4*>(p));
    const float4 y = __ldg(reinterpret_cast<const float4*>(p) + 1);
    return AdamScalars{x.x, x.y, x.z, x.w, y.x, y.y, y.z, y.w};
}

}  // namespace
