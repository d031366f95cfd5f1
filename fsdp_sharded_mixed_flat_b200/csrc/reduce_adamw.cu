// reduce_adamw.cu -- the fused per-rank optimiser pass for sm_100a:
// reduce-scatter's reduction of the D bf16 gradient contributions for the
// owned partition(s), AdamW on the owned fp32 master / m / v, and the cast of
// the new master to the bf16 working shard, in one streaming pass over HBM.
//
// Pages: "Building GPT from Scratch — Part 8: FSDP — When the Model Won't
// Fit", "AllGather vs AllReduce" (rank r receives the sum of the r-th slice of
// every rank's gradient) and "Mixed Precision: Cutting Memory in Half" (fp32
// master, bf16 params); "7.10 — Fully-sharded data parallel (FSDP / ZeRO-3)",
// §3 (rank r updates only P_r from its fp32 master, m, v and gradient slice)
// and §4 (reduce-scatter replaces the all-reduce).  The HYBRID_SHARD form
// ("Building GPT from Scratch — Part 8", "HYBRID_SHARD: The Multi-Node
// Strategy") reduces R nodes of D ranks in two levels: each node's ranks in
// rank order, then the node sums in node order.
//
// The pass is bound by HBM bandwidth: per owned element it reads 2*D bytes of
// contributions and 12 bytes of state, and writes 12 bytes of state and 2
// bytes of bf16 weights, against about 40 floating-point operations.  There is
// no contraction, so no tensor-core work.  Each thread owns 8 consecutive
// elements: one 16-byte load per rank, two per state array, all issued before
// the arithmetic so that (D + 6) x 16 bytes per thread are in flight; the
// ranks are folded in order 0..D-1 in chunks (8 ranks, 16 for the bf16 fold at
// D = 32) to bound registers at large D.  The folds that did not fit the
// register cap with 8 take 4 elements per thread instead (see k1_elems).
// Loading each tile with 1-D bulk copies (cp.async.bulk) into shared memory
// measured no faster on B200 (7044 against 7049 GB/s at D = 8, with more bytes
// in flight): the read/write mix of HBM is the bound, not the issue of the
// loads.  The grid covers the whole range rather than looping over a resident
// grid: HBM bandwidth does not divide evenly over the SMs, and a resident grid
// leaves the SMs that finish first idle, while the block scheduler keeps every
// SM fed until the end.  Stores carry the streaming cache hint: every
// byte is written exactly once.  Asking for three resident blocks per SM caps
// the registers at 80 (65,536 / (3 x 256), rounded down to the allocation
// granularity; left alone the compiler takes up to 128 at D >= 16); measured
// on B200 this never loses and gains up to 12 % (bf16 reduce at D = 16, before
// that instantiation moved to 4 elements per thread and 4 blocks per SM).
//
// Every arithmetic step is an explicitly rounded fp32 intrinsic, so nothing is
// contracted into an FMA and the results are fixed by the stated operation
// order.
//
// Measured ceilings of HBM on the B200s used here, for a full-grid kernel with
// two or more independent 16-byte vectors per thread: read-only 7.54 TB/s,
// write-only 7.56 TB/s, copy 6.94 TB/s, two reads per write 7.16 TB/s.  This
// pass reads 28 B and writes 14 B per element at D = 8, the two-to-one mix;
// the benchmark times torch's kernels of each mix beside it on the same GPU.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstring>

#include "plan_impl.h"
#include "step_common.cuh"
#include "zero3.h"

namespace {

struct K1Args {
    const uint16_t* c[Z3_D_MAX];  // contributions c[k*D + d] (node k, rank d), each at the launch's first element
    float* p;                     // master
    float* m;                     // exp_avg
    float* v;                     // exp_avg_sq
    uint16_t* w;                  // bf16 working weights (may be null when gathering)
    uint16_t* g[Z3_GATHER_MAX];   // gathered blocks, each at the launch's first element
    int32_t ng;                   // number of gathered blocks
    int64_t n;                    // elements in this launch
    int32_t D;                    // ranks per node
    float inv_n;                  // fp32 nearest to 1/(R*D)
    AdamScalars s;                // this step's scalars (unless s_dev is used)
    const AdamScalars* s_dev;     // device copy of the scalars (the DEVS kernels)
    int32_t R;                    // nodes (HYBRID_SHARD; 1 otherwise)
};

constexpr int kThreads = 256;
constexpr int kChunks = 1;                  // 8-element chunks per thread
constexpr int64_t kMaxBlocks = 1 << 30;     // grid.x cap; beyond it the kernel loops

// Elements per thread.  8 (16-byte loads of each contribution) by default; 4
// (8-byte loads of each contribution) where it measured faster on B200 (7B
// block), i.e. where 8 elements' contribution vectors and state did not fit the
// register cap and spilled, without a fused gather:
//   - the bf16 fold of one node of 16 ranks: 7066 -> 7276 GB/s;
//   - the bf16 folds of 4 and 8 nodes of 8 ranks: 7107 -> 7204, 7076 -> 7234;
//   - the generic one-node fp32 fold (rank counts without their own
//     instantiation): D = 3 / 6 / 12 / 24: 6088 / 6263 / 6658 / 6746 ->
//     6712 / 6978 / 6868 / 6997;
//   - the generic HYBRID_SHARD fold (any node count and D), both dtypes:
//     3 x 5 fp32 5764 -> 5976, 2 x 3 bf16 5346 -> 5889.
// It did not help elsewhere: the fp32 folds of D = 2, 4, 8, 16, 32, 2 nodes of 8
// and the generic one-node bf16 fold were within 0.5 % or slower with 4.
__host__ __device__ constexpr int k1_elems(int mode, int dt, int rt, bool gather) {
    return gather ? 8
         : dt == 0 ? ((rt == 0 || mode == Z3_REDUCE_FP32) ? 4 : 8)
         : (mode == Z3_REDUCE_BF16 && ((dt == 16 && rt == 1) || (dt == 8 && (rt == 4 || rt == 8)))) ? 4 : 8;
}

// Blocks per SM each vector kernel asks for (the register cap follows from it):
// 3 (80 registers), or 4 (64 registers) for the 4-element folds other than the
// specialised HYBRID_SHARD ones (where 3 measured better).
__host__ __device__ constexpr int k1_min_blocks(int mode, int dt, int rt, bool gather) {
    return (k1_elems(mode, dt, rt, gather) == 4 && (rt == 1 || rt == 0)) ? 4 : 3;
}

// Fold ranks base..base+D-1 for the 8 elements starting at e into the fp32 or
// packed-bf16 accumulators, left to right, in chunks of ranks (the chunk's
// loads are all issued before its folds).
template <int MODE, int DT>
__device__ __forceinline__ void fold_ranks(const K1Args& a, int base, int64_t e, float (&acc)[8],
                                           uint32_t (&accw)[4]) {
    const int D = DT > 0 ? DT : a.D;
    // ranks per chunk: 8, or 16 for the bf16 fold at D = 32 (measured 1.3 % faster there,
    // slower at D = 16; the fp32 fold did not change)
    constexpr int CH = (MODE != Z3_REDUCE_FP32 && DT >= 32) ? 16 : 8;
#pragma unroll
    for (int d0 = 0; d0 < (DT > 0 ? DT : Z3_D_MAX); d0 += CH) {
        if (DT == 0 && d0 >= D) break;
        uint4 q[CH];
#pragma unroll
        for (int k = 0; k < CH; ++k)
            if (d0 + k < D) q[k] = ld16(reinterpret_cast<const uint4*>(a.c[base + d0 + k] + e));
#pragma unroll
        for (int k = 0; k < CH; ++k) {
            if (d0 + k >= D) continue;
            if constexpr (MODE == Z3_REDUCE_FP32)
                fold8_fp32(acc, q[k], d0 + k == 0);
            else
                fold8_bf16(accw, q[k], d0 + k == 0);
        }
    }
}

// The averaged gradient g of the 8 elements starting at e, in the reduce dtype.
// RT = 1: ranks 0..D-1 folded in order, times 1/D.  RT != 1 (HYBRID_SHARD; 0
// means R from the arguments): each node's D ranks folded in order, the node
// sums folded in node order, times 1/(R*D).
template <int MODE, int DT, int RT>
__device__ __forceinline__ void reduce8(const K1Args& a, int64_t e, float (&g)[8]) {
    float acc[8];
    uint32_t accw[4];
    if constexpr (RT == 1) {
        fold_ranks<MODE, DT>(a, 0, e, acc, accw);
    } else {
        const int D = DT > 0 ? DT : a.D;
        const int R = RT > 0 ? RT : a.R;
        float node[8];
        uint32_t nodew[4];
#pragma unroll(RT > 0 ? RT : 1)
        for (int k = 0; k < R; ++k) {
            fold_ranks<MODE, DT>(a, k * D, e, node, nodew);
            if constexpr (MODE == Z3_REDUCE_FP32) {
#pragma unroll
                for (int i = 0; i < 8; ++i) acc[i] = k == 0 ? node[i] : __fadd_rn(acc[i], node[i]);
            } else {
#pragma unroll
                for (int i = 0; i < 4; ++i) accw[i] = k == 0 ? nodew[i] : add_bf16x2(accw[i], nodew[i]);
            }
        }
    }
    if constexpr (MODE == Z3_REDUCE_FP32) {
#pragma unroll
        for (int k = 0; k < 8; ++k) g[k] = __fmul_rn(acc[k], a.inv_n);
    } else {
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            g[2 * k] = round_to_bf16(__fmul_rn(lo_bf16(accw[k]), a.inv_n));
            g[2 * k + 1] = round_to_bf16(__fmul_rn(hi_bf16(accw[k]), a.inv_n));
        }
    }
}

// One element on the scalar path (tails and misaligned buffers).  RT = 1: the
// rank fold; otherwise the nodes' rank folds, then the fold of the node sums.
template <int MODE, int RT, bool GATHER>
__device__ __forceinline__ void scalar_elem(const K1Args& a, const AdamScalars& sc, int64_t i) {
    float total;
    if constexpr (RT == 1) {
        total = bf16_of(a.c[0][i]);
        for (int d = 1; d < a.D; ++d) total = add_in<MODE>(total, bf16_of(a.c[d][i]));
    } else {
        const int R = RT > 0 ? RT : a.R;
        for (int k = 0; k < R; ++k) {
            float node = bf16_of(a.c[k * a.D][i]);
            for (int d = 1; d < a.D; ++d) node = add_in<MODE>(node, bf16_of(a.c[k * a.D + d][i]));
            total = k == 0 ? node : add_in<MODE>(total, node);
        }
    }
    const float g0 = __fmul_rn(total, a.inv_n);
    const float g = MODE == Z3_REDUCE_FP32 ? g0 : round_to_bf16(g0);
    float p = a.p[i], m = a.m[i], v = a.v[i];
    adamw_elem(sc, g, p, m, v);
    a.p[i] = p;
    a.m[i] = m;
    a.v[i] = v;
    const uint16_t w = __bfloat16_as_ushort(__float2bfloat16_rn(p));
    if (!GATHER || a.w != nullptr) a.w[i] = w;
    if (GATHER)
        for (int k = 0; k < a.ng; ++k) a.g[k][i] = w;
}

// The 8 elements starting at e: state loads, the rank fold, AdamW, stores.
// GATHER: the bf16 result also goes to every gathered block (the all-gather's
// data movement done by the producer of the data).
template <int MODE, int DT, int RT, bool GATHER>
__device__ __forceinline__ void process8(const K1Args& a, const AdamScalars& sc, int64_t e) {
    const float4 p0 = ld16(reinterpret_cast<const float4*>(a.p + e));
    const float4 p1 = ld16(reinterpret_cast<const float4*>(a.p + e + 4));
    const float4 m0 = ld16(reinterpret_cast<const float4*>(a.m + e));
    const float4 m1 = ld16(reinterpret_cast<const float4*>(a.m + e + 4));
    const float4 v0 = ld16(reinterpret_cast<const float4*>(a.v + e));
    const float4 v1 = ld16(reinterpret_cast<const float4*>(a.v + e + 4));
    float g[8];
    reduce8<MODE, DT, RT>(a, e, g);
    float p[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
    float m[8] = {m0.x, m0.y, m0.z, m0.w, m1.x, m1.y, m1.z, m1.w};
    float v[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
#pragma unroll
    for (int k = 0; k < 8; ++k) adamw_elem(sc, g[k], p[k], m[k], v[k]);
    st16(reinterpret_cast<float4*>(a.p + e), make_float4(p[0], p[1], p[2], p[3]));
    st16(reinterpret_cast<float4*>(a.p + e + 4), make_float4(p[4], p[5], p[6], p[7]));
    st16(reinterpret_cast<float4*>(a.m + e), make_float4(m[0], m[1], m[2], m[3]));
    st16(reinterpret_cast<float4*>(a.m + e + 4), make_float4(m[4], m[5], m[6], m[7]));
    st16(reinterpret_cast<float4*>(a.v + e), make_float4(v[0], v[1], v[2], v[3]));
    st16(reinterpret_cast<float4*>(a.v + e + 4), make_float4(v[4], v[5], v[6], v[7]));
    const uint4 w = make_uint4(pack_bf16x2(p[0], p[1]), pack_bf16x2(p[2], p[3]), pack_bf16x2(p[4], p[5]),
                               pack_bf16x2(p[6], p[7]));
    if (!GATHER || a.w != nullptr) st16(reinterpret_cast<uint4*>(a.w + e), w);
    if (GATHER) {
#pragma unroll
        for (int k = 0; k < Z3_GATHER_MAX; ++k)
            if (k < a.ng) st16(reinterpret_cast<uint4*>(a.g[k] + e), w);
    }
}

// Fold ranks base..base+D-1 for the 4 elements starting at e into fp32 or
// packed-bf16 accumulators, left to right, in chunks of 8 ranks (the chunk's
// 8-byte loads all issued before its folds).  DT = 0: D from the arguments.
template <int MODE, int DT>
__device__ __forceinline__ void fold_ranks4(const K1Args& a, int base, int64_t e, float (&acc)[4],
                                            uint32_t (&accw)[2]) {
    const int D = DT > 0 ? DT : a.D;
#pragma unroll
    for (int d0 = 0; d0 < (DT > 0 ? DT : Z3_D_MAX); d0 += 8) {
        if (DT == 0 && d0 >= D) break;
        uint2 q[8];
#pragma unroll
        for (int k = 0; k < 8; ++k)
            if (d0 + k < D) q[k] = ld16(reinterpret_cast<const uint2*>(a.c[base + d0 + k] + e));
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            if (d0 + k >= D) continue;
            const bool first = d0 + k == 0;
            if constexpr (MODE == Z3_REDUCE_FP32) {
                const float x[4] = {lo_bf16(q[k].x), hi_bf16(q[k].x), lo_bf16(q[k].y), hi_bf16(q[k].y)};
#pragma unroll
                for (int i = 0; i < 4; ++i) acc[i] = first ? x[i] : __fadd_rn(acc[i], x[i]);
            } else {
                accw[0] = first ? q[k].x : add_bf16x2(accw[0], q[k].x);
                accw[1] = first ? q[k].y : add_bf16x2(accw[1], q[k].y);
            }
        }
    }
}

// The 4 elements starting at e (the k1_elems == 4 instantiations): one 8-byte
// load per rank, one 16-byte load per state array; the same operations in the
// same order as process8 (RT = 1: the rank fold; otherwise each node's rank
// fold, then the node sums in node order; DT = 0 / RT = 0: counts from the
// arguments).
template <int MODE, int DT, int RT>
__device__ __forceinline__ void process4(const K1Args& a, const AdamScalars& sc, int64_t e) {
    const float4 p0 = ld16(reinterpret_cast<const float4*>(a.p + e));
    const float4 m0 = ld16(reinterpret_cast<const float4*>(a.m + e));
    const float4 v0 = ld16(reinterpret_cast<const float4*>(a.v + e));
    float acc[4];
    uint32_t accw[2];
    if constexpr (RT == 1) {
        fold_ranks4<MODE, DT>(a, 0, e, acc, accw);
    } else {
        const int D = DT > 0 ? DT : a.D;
        const int R = RT > 0 ? RT : a.R;
        float node[4];
        uint32_t nodew[2];
#pragma unroll(RT > 0 ? RT : 1)
        for (int k = 0; k < R; ++k) {
            fold_ranks4<MODE, DT>(a, k * D, e, node, nodew);
            if constexpr (MODE == Z3_REDUCE_FP32) {
#pragma unroll
                for (int i = 0; i < 4; ++i) acc[i] = k == 0 ? node[i] : __fadd_rn(acc[i], node[i]);
            } else {
#pragma unroll
                for (int i = 0; i < 2; ++i) accw[i] = k == 0 ? nodew[i] : add_bf16x2(accw[i], nodew[i]);
            }
        }
    }
    float g[4];
    if constexpr (MODE == Z3_REDUCE_FP32) {
#pragma unroll
        for (int k = 0; k < 4; ++k) g[k] = __fmul_rn(acc[k], a.inv_n);
    } else {
#pragma unroll
        for (int k = 0; k < 2; ++k) {
            g[2 * k] = round_to_bf16(__fmul_rn(lo_bf16(accw[k]), a.inv_n));
            g[2 * k + 1] = round_to_bf16(__fmul_rn(hi_bf16(accw[k]), a.inv_n));
        }
    }
    float p[4] = {p0.x, p0.y, p0.z, p0.w};
    float m[4] = {m0.x, m0.y, m0.z, m0.w};
    float v[4] = {v0.x, v0.y, v0.z, v0.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) adamw_elem(sc, g[k], p[k], m[k], v[k]);
    st16(reinterpret_cast<float4*>(a.p + e), make_float4(p[0], p[1], p[2], p[3]));
    st16(reinterpret_cast<float4*>(a.m + e), make_float4(m[0], m[1], m[2], m[3]));
    st16(reinterpret_cast<float4*>(a.v + e), make_float4(v[0], v[1], v[2], v[3]));
    st16(reinterpret_cast<uint2*>(a.w + e), make_uint2(pack_bf16x2(p[0], p[1]), pack_bf16x2(p[2], p[3])));
}

// Vector kernel body: every pointer 16-byte aligned.  The grid covers the
// whole range (kChunks 8-element chunks per thread, consecutive threads on
// consecutive chunks), so the block scheduler hands blocks to whichever SM is
// free and every SM keeps streaming to the end; the outer loop only runs more
// than once when the range exceeds the largest grid.  The last n % 8 elements
// go through the scalar path.
template <int MODE, int DT, int RT, bool GATHER>
__device__ __forceinline__ void vec_body(const K1Args& a, const AdamScalars& sc) {
    if constexpr (k1_elems(MODE, DT, RT, GATHER) == 4) {
        const int64_t n4 = a.n >> 2;
        const int64_t step4 = int64_t(gridDim.x) * kThreads;
        for (int64_t q = int64_t(blockIdx.x) * kThreads + threadIdx.x; q < n4; q += step4)
            process4<MODE, DT, RT>(a, sc, q << 2);
        const int64_t tail4 = (n4 << 2) + int64_t(blockIdx.x) * kThreads + threadIdx.x;
        if (tail4 < a.n) scalar_elem<MODE, RT, GATHER>(a, sc, tail4);
        return;
    }
    const int64_t n8 = a.n >> 3;
    const int64_t span = int64_t(kThreads) * kChunks;
    const int64_t step = int64_t(gridDim.x) * span;
    for (int64_t first = int64_t(blockIdx.x) * span + threadIdx.x; first < n8; first += step) {
#pragma unroll
        for (int k = 0; k < kChunks; ++k) {
            const int64_t q = first + int64_t(k) * kThreads;
            if (q < n8) process8<MODE, DT, RT, GATHER>(a, sc, q << 3);
        }
    }
    const int64_t tail = (n8 << 3) + int64_t(blockIdx.x) * kThreads + threadIdx.x;
    if (tail < a.n) scalar_elem<MODE, RT, GATHER>(a, sc, tail);
}

template <int MODE, int DT, int RT, bool GATHER, bool DEVS>
__global__ void __launch_bounds__(kThreads, (k1_min_blocks(MODE, DT, RT, GATHER)))
    k_reduce_adamw_vec(const __grid_constant__ K1Args a) {
    if constexpr (DEVS) {
        const AdamScalars sc = load_scalars(a.s_dev);
        vec_body<MODE, DT, RT, GATHER>(a, sc);
    } else {
        vec_body<MODE, DT, RT, GATHER>(a, a.s);   // the scalars stay in the parameter block
    }
}

// Scalar kernel: any element-aligned pointers.
template <int MODE, int RT, bool GATHER>
__device__ __forceinline__ void scalar_body(const K1Args& a, const AdamScalars& sc) {
    const int64_t stride = int64_t(gridDim.x) * kThreads;
    for (int64_t i = int64_t(blockIdx.x) * kThreads + threadIdx.x; i < a.n; i += stride)
        scalar_elem<MODE, RT, GATHER>(a, sc, i);
}

template <int MODE, int RT, bool GATHER, bool DEVS>
__global__ void __launch_bounds__(kThreads) k_reduce_adamw_scalar(const __grid_constant__ K1Args a) {
    if constexpr (DEVS) {
        const AdamScalars sc = load_scalars(a.s_dev);
        scalar_body<MODE, RT, GATHER>(a, sc);
    } else {
        scalar_body<MODE, RT, GATHER>(a, a.s);
    }
}

using KernelFn = void (*)(K1Args);

template <int MODE, bool GATHER, bool DEVS>
KernelFn pick_vec(int D) {
    switch (D) {
    case 1: return k_reduce_adamw_vec<MODE, 1, 1, GATHER, DEVS>;
    case 2: return k_reduce_adamw_vec<MODE, 2, 1, GATHER, DEVS>;
    case 4: return k_reduce_adamw_vec<MODE, 4, 1, GATHER, DEVS>;
    case 8: return k_reduce_adamw_vec<MODE, 8, 1, GATHER, DEVS>;
    case 16: return k_reduce_adamw_vec<MODE, 16, 1, GATHER, DEVS>;
    case 32: return k_reduce_adamw_vec<MODE, 32, 1, GATHER, DEVS>;
    default: return k_reduce_adamw_vec<MODE, 0, 1, GATHER, DEVS>;
    }
}

template <bool GATHER, bool DEVS>
KernelFn pick(bool vec, int32_t reduce_dtype, int D) {
    if (vec)
        return reduce_dtype == Z3_REDUCE_FP32 ? pick_vec<Z3_REDUCE_FP32, GATHER, DEVS>(D)
                                              : pick_vec<Z3_REDUCE_BF16, GATHER, DEVS>(D);
    return reduce_dtype == Z3_REDUCE_FP32 ? k_reduce_adamw_scalar<Z3_REDUCE_FP32, 1, GATHER, DEVS>
                                          : k_reduce_adamw_scalar<Z3_REDUCE_BF16, 1, GATHER, DEVS>;
}

// HYBRID_SHARD kernels (no fused gather, scalars by value): specialised vector
// kernels for 2, 4 and 8 nodes of 8 ranks (measured on B200: the generic
// kernel ran 12-15 % slower at 2 and 8 nodes), and one for any other shape.
template <int MODE>
KernelFn pick_hybrid_vec(int R, int D) {
    if (D == 8) {
        switch (R) {
        case 2: return k_reduce_adamw_vec<MODE, 8, 2, false, false>;
        case 4: return k_reduce_adamw_vec<MODE, 8, 4, false, false>;
        case 8: return k_reduce_adamw_vec<MODE, 8, 8, false, false>;
        default: break;
        }
    }
    return k_reduce_adamw_vec<MODE, 0, 0, false, false>;
}

KernelFn pick_any(bool gather, bool devs, bool vec, int32_t reduce_dtype, int D, int R) {
    if (R > 1) {
        if (vec)
            return reduce_dtype == Z3_REDUCE_FP32 ? pick_hybrid_vec<Z3_REDUCE_FP32>(R, D)
                                                  : pick_hybrid_vec<Z3_REDUCE_BF16>(R, D);
        return reduce_dtype == Z3_REDUCE_FP32 ? k_reduce_adamw_scalar<Z3_REDUCE_FP32, 0, false, false>
                                              : k_reduce_adamw_scalar<Z3_REDUCE_BF16, 0, false, false>;
    }
    if (gather)
        return devs ? pick<true, true>(vec, reduce_dtype, D) : pick<true, false>(vec, reduce_dtype, D);
    return devs ? pick<false, true>(vec, reduce_dtype, D) : pick<false, false>(vec, reduce_dtype, D);
}

// Validation and launch shared by every entry point.  `gathered` holds
// n_gathered whole padded blocks (0 for the plain entry point); `work_bf16`
// may be null only when n_gathered > 0.
// Exactly one of hp (scalars computed here, passed by value) and dev_scalars
// (read by the kernel from device memory) is non-null.
// R: nodes of D ranks each (HYBRID_SHARD, contrib holds R*D pointers; only
// with n_gathered = 0 and hp), 1 otherwise.
int launch_k1(const z3_plan* p, int32_t rank, int32_t R, const uint16_t* const* contrib, int32_t contrib_layout,
              float* master, float* exp_avg, float* exp_avg_sq, uint16_t* work_bf16,
              uint16_t* const* gathered, int32_t n_gathered, int32_t reduce_dtype, const z3_adamw* hp,
              const float* dev_scalars, void* cuda_stream) {
    // ---- arguments
    if (p == nullptr || contrib == nullptr || (hp == nullptr) == (dev_scalars == nullptr)) return Z3_EINVAL;
    const int32_t D = p->D;
    if (R < 1 || R > Z3_D_MAX / D || (R > 1 && (n_gathered != 0 || hp == nullptr))) return Z3_EINVAL;
    const int32_t n_contrib = R * D;
    if (rank < -1 || rank >= D) return Z3_EINVAL;
    if (contrib_layout != Z3_CONTRIB_FULL && contrib_layout != Z3_CONTRIB_OWNED) return Z3_EINVAL;
    if (contrib_layout == Z3_CONTRIB_OWNED && rank < 0) return Z3_EINVAL;
    if (reduce_dtype != Z3_REDUCE_FP32 && reduce_dtype != Z3_REDUCE_BF16) return Z3_EINVAL;
    if (n_gathered < 0 || n_gathered > Z3_GATHER_MAX || (n_gathered > 0 && gathered == nullptr))
        return Z3_EINVAL;
    if (master == nullptr || exp_avg == nullptr || exp_avg_sq == nullptr ||
        (work_bf16 == nullptr && n_gathered == 0))
        return Z3_EINVAL;
    for (int32_t d = 0; d < n_contrib; ++d)
        if (contrib[d] == nullptr) return Z3_EINVAL;
    for (int32_t k = 0; k < n_gathered; ++k)
        if (gathered[k] == nullptr) return Z3_EINVAL;
    if (hp != nullptr && !hp_valid(hp)) return Z3_EINVAL;
    if (dev_scalars != nullptr && !z3::aligned(dev_scalars, 16)) return Z3_EALIGN;
    if (!z3::aligned(master, 4) || !z3::aligned(exp_avg, 4) || !z3::aligned(exp_avg_sq, 4) ||
        !z3::aligned(work_bf16, 2))
        return Z3_EALIGN;
    for (int32_t d = 0; d < n_contrib; ++d)
        if (!z3::aligned(contrib[d], 2)) return Z3_EALIGN;
    for (int32_t k = 0; k < n_gathered; ++k)
        if (!z3::aligned(gathered[k], 2)) return Z3_EALIGN;

    const int64_t n = rank < 0 ? p->N_pad : p->S;
    // first element of the launch inside each contribution buffer and gathered block
    const int64_t c_off = (contrib_layout == Z3_CONTRIB_FULL && rank >= 0) ? int64_t(rank) * p->S : 0;
    const int64_t g_off = rank >= 0 ? int64_t(rank) * p->S : 0;

    // ---- outputs must not overlap each other or any contribution they read
    const int64_t fb = n * 4, hb = n * 2;
    const void* outs[4 + Z3_GATHER_MAX] = {master, exp_avg, exp_avg_sq, work_bf16};
    int64_t out_bytes[4 + Z3_GATHER_MAX] = {fb, fb, fb, work_bf16 ? hb : 0};
    for (int32_t k = 0; k < n_gathered; ++k) {
        outs[4 + k] = gathered[k];
        out_bytes[4 + k] = p->N_pad * 2;  // the whole block is the caller's buffer
    }
    const int n_out = 4 + n_gathered;
    for (int x = 0; x < n_out; ++x) {
        for (int y = x + 1; y < n_out; ++y)
            if (z3::overlaps(outs[x], out_bytes[x], outs[y], out_bytes[y])) return Z3_EINVAL;
        for (int32_t d = 0; d < n_contrib; ++d)
            if (z3::overlaps(outs[x], out_bytes[x], contrib[d] + c_off, hb)) return Z3_EINVAL;
        if (dev_scalars != nullptr &&
            z3::overlaps(outs[x], out_bytes[x], dev_scalars, Z3_SCALARS * int64_t(sizeof(float))))
            return Z3_EINVAL;
    }
    if (n == 0) return Z3_OK;

    // ---- host scalars: double, then rounded to fp32 once
    K1Args a;
    a.s = hp != nullptr ? step_scalars(hp) : AdamScalars{};
    a.s_dev = reinterpret_cast<const AdamScalars*>(dev_scalars);
    a.inv_n = float(1.0 / double(n_contrib));
    a.D = D;
    a.R = R;
    a.n = n;
    a.p = master;
    a.m = exp_avg;
    a.v = exp_avg_sq;
    a.w = work_bf16;
    a.ng = n_gathered;
    bool vec = z3::aligned(master, 16) && z3::aligned(exp_avg, 16) && z3::aligned(exp_avg_sq, 16) &&
               z3::aligned(work_bf16, 16);
    for (int32_t d = 0; d < Z3_D_MAX; ++d) {
        a.c[d] = d < n_contrib ? contrib[d] + c_off : nullptr;
        if (d < n_contrib && !z3::aligned(a.c[d], 16)) vec = false;
    }
    for (int32_t k = 0; k < Z3_GATHER_MAX; ++k) {
        a.g[k] = k < n_gathered ? gathered[k] + g_off : nullptr;
        if (k < n_gathered && !z3::aligned(a.g[k], 16)) vec = false;
    }

    // ---- launch: the vector kernel's grid covers the range; the scalar kernel
    // runs a whole number of resident waves with a grid-stride loop
    const KernelFn fn = pick_any(n_gathered > 0, dev_scalars != nullptr, vec, reduce_dtype, D, R);
    int64_t blocks;
    if (vec) {
        // the template rank and node counts of the picked kernel (pick_vec, pick_hybrid_vec)
        int dt = 0, rt = 1;
        if (R == 1) {
            if (D == 1 || D == 2 || D == 4 || D == 8 || D == 16 || D == 32) dt = D;
        } else if (D == 8 && (R == 2 || R == 4 || R == 8)) {
            dt = 8;
            rt = R;
        } else {
            rt = 0;
        }
        const int elems = k1_elems(reduce_dtype, dt, rt, n_gathered > 0);
        const int64_t span = int64_t(kThreads) * (elems == 4 ? 1 : kChunks);
        blocks = ((n / elems) + span - 1) / span;
        if (blocks > kMaxBlocks) blocks = kMaxBlocks;
    } else {
        int per_sm = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, kThreads, 0) != cudaSuccess ||
            per_sm < 1)
            per_sm = 1;
        const int sms = z3::sm_count();
        if (sms < 1) return Z3_ECUDA;
        blocks = (n + kThreads - 1) / kThreads;
        const int64_t resident = int64_t(sms) * per_sm;
        if (blocks > resident) blocks = resident;
    }
    if (blocks < 1) blocks = 1;  // the vector kernel's scalar tail still needs one block
    fn<<<dim3(unsigned(blocks)), dim3(kThreads), 0, static_cast<cudaStream_t>(cuda_stream)>>>(a);
    return cudaGetLastError() == cudaSuccess ? Z3_OK : Z3_ECUDA;
}

}  // namespace

extern "C" Z3_API int zero3_reduce_adamw(const z3_plan* p, int32_t rank, const uint16_t* const* contrib,
                                         int32_t contrib_layout, float* master, float* exp_avg,
                                         float* exp_avg_sq, uint16_t* work_bf16, int32_t reduce_dtype,
                                         const z3_adamw* hp, void* cuda_stream) {
    if (hp == nullptr) return Z3_EINVAL;
    return launch_k1(p, rank, 1, contrib, contrib_layout, master, exp_avg, exp_avg_sq, work_bf16, nullptr, 0,
                     reduce_dtype, hp, nullptr, cuda_stream);
}

extern "C" Z3_API int zero3_reduce_adamw_hybrid(const z3_plan* p, int32_t rank, int32_t n_nodes,
                                                const uint16_t* const* contrib, int32_t contrib_layout,
                                                float* master, float* exp_avg, float* exp_avg_sq,
                                                uint16_t* work_bf16, int32_t reduce_dtype, const z3_adamw* hp,
                                                void* cuda_stream) {
    if (hp == nullptr || n_nodes < 1) return Z3_EINVAL;
    return launch_k1(p, rank, n_nodes, contrib, contrib_layout, master, exp_avg, exp_avg_sq, work_bf16, nullptr,
                     0, reduce_dtype, hp, nullptr, cuda_stream);
}

extern "C" Z3_API int zero3_reduce_adamw_gather(const z3_plan* p, int32_t rank, const uint16_t* const* contrib,
                                                int32_t contrib_layout, float* master, float* exp_avg,
                                                float* exp_avg_sq, uint16_t* work_bf16,
                                                uint16_t* const* gathered, int32_t n_gathered,
                                                int32_t reduce_dtype, const z3_adamw* hp, void* cuda_stream) {
    if (n_gathered < 1 || hp == nullptr) return Z3_EINVAL;
    return launch_k1(p, rank, 1, contrib, contrib_layout, master, exp_avg, exp_avg_sq, work_bf16, gathered,
                     n_gathered, reduce_dtype, hp, nullptr, cuda_stream);
}

extern "C" Z3_API int zero3_step_scalars(const z3_adamw* hp, float* out) {
    if (out == nullptr || !hp_valid(hp)) return Z3_EINVAL;
    const AdamScalars s = step_scalars(hp);
    std::memcpy(out, &s, sizeof s);
    return Z3_OK;
}

extern "C" Z3_API int zero3_reduce_adamw_dev(const z3_plan* p, int32_t rank, const uint16_t* const* contrib,
                                             int32_t contrib_layout, float* master, float* exp_avg,
                                             float* exp_avg_sq, uint16_t* work_bf16, uint16_t* const* gathered,
                                             int32_t n_gathered, int32_t reduce_dtype, const float* scalars,
                                             void* cuda_stream) {
    if (scalars == nullptr) return Z3_EINVAL;
    return launch_k1(p, rank, 1, contrib, contrib_layout, master, exp_avg, exp_avg_sq, work_bf16, gathered,
                     n_gathered, reduce_dtype, nullptr, scalars, cuda_stream);
}
