// node_fold.cu -- HYBRID_SHARD across nodes, for sm_100a: the two halves of
// the two-level reduction, for when the node sums have to cross a network.
//
// Pages: "Building GPT from Scratch — Part 8: FSDP — When the Model Won't
// Fit", "HYBRID_SHARD: The Multi-Node Strategy" (R nodes of D GPUs: sharded
// D ways inside a node, replicated across the nodes, the gradient crosses the
// nodes in one exchange per step) and "Key Takeaways" (the same gradient as on
// one GPU: the average over all R*D ranks).
//
//   k_node_sum:   a node's D contributions for the owned partition(s), folded
//                 left to right in rank order, not scaled; written as fp32
//                 (fp32 reduce) or bf16 (bf16 reduce, every partial sum
//                 rounded).  Reads 2*D bytes, writes 4 (or 2) per element.
//                 The same kernel with the 1/D scale is the reduce-scatter's
//                 reduction alone (zero3_reduce_scatter): the averaged gradient
//                 of the owned partition, for the CPU-offload step, whose
//                 optimiser runs on the host ("7.10 — Fully-sharded data
//                 parallel (FSDP / ZeRO-3)", §8).
//   k_fold_adamw: the R node sums folded in node order, times fp32(1/(R*D)),
//                 AdamW on the owned fp32 master / m / v and the bf16 cast.
//                 Reads 4*R (or 2*R) + 12 bytes, writes 14 per element.
//
// Composed, they compute exactly what the fused HYBRID_SHARD kernel in
// reduce_adamw.cu computes in one pass: the same partial sums in the same
// order, each explicitly rounded.  Both are streaming passes bound by HBM,
// built like the fused kernel: a grid covering the range, one 8-element chunk
// per thread, 16-byte loads issued before the arithmetic, streaming stores,
// and a scalar kernel for misaligned buffers and the n mod 8 tail.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "plan_impl.h"
#include "step_common.cuh"
#include "zero3.h"

namespace {

constexpr int kNfThreads = 256;
constexpr int64_t kNfMaxBlocks = 1 << 30;   // grid.x cap; beyond it the kernels loop

struct NodeSumArgs {
    const uint16_t* c[Z3_D_MAX];  // the node's D contributions, each at the launch's first element
    void* out;                    // n node sums: float (fp32 reduce) or bf16 bits (bf16 reduce)
    int64_t n;
    int32_t D;
    float inv_n;                  // SCALE kernels: fp32 nearest to 1/D
};

struct FoldArgs {
    const void* sums[Z3_D_MAX];   // the R node sums, each at the launch's first element
    float* p;                     // master
    float* m;                     // exp_avg
    float* v;                     // exp_avg_sq
    uint16_t* w;                  // bf16 working weights
    int64_t n;
    int32_t R;
    float inv_n;                  // fp32 nearest to 1/(R*D)
    AdamScalars s;
};

// ---------------------------------------------------------------- node sums
// SCALE = false: the node's unscaled sum.  SCALE = true: the reduce-scatter's
// averaged gradient, the sum times fp32(1/D) (rounded to bf16 in the bf16
// reduce), exactly the g the fused kernel hands to AdamW.
template <int MODE, bool SCALE>
__device__ __forceinline__ void node_sum1(const NodeSumArgs& a, int64_t i) {
    float acc = bf16_of(a.c[0][i]);
    for (int d = 1; d < a.D; ++d) acc = add_in<MODE>(acc, bf16_of(a.c[d][i]));
    if constexpr (SCALE) acc = __fmul_rn(acc, a.inv_n);
    if constexpr (MODE == Z3_REDUCE_FP32)
        static_cast<float*>(a.out)[i] = acc;
    else  // nearest-even: exact for the unscaled sum (already bf16), the rounding of g when scaled
        static_cast<uint16_t*>(a.out)[i] = __bfloat16_as_ushort(__float2bfloat16_rn(acc));
}

template <int MODE, int DT, bool SCALE>
__device__ __forceinline__ void node_sum8(const NodeSumArgs& a, int64_t e) {
    const int D = DT > 0 ? DT : a.D;
    float acc[8];
    uint32_t accw[4];
#pragma unroll
    for (int d0 = 0; d0 < (DT > 0 ? DT : Z3_D_MAX); d0 += 8) {
        if (DT == 0 && d0 >= D) break;
        uint4 q[8];
#pragma unroll
        for (int k = 0; k < 8; ++k)
            if (d0 + k < D) q[k] = ld16(reinterpret_cast<const uint4*>(a.c[d0 + k] + e));
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            if (d0 + k >= D) continue;
            if constexpr (MODE == Z3_REDUCE_FP32)
                fold8_fp32(acc, q[k], d0 + k == 0);
            else
                fold8_bf16(accw, q[k], d0 + k == 0);
        }
    }
    if constexpr (MODE == Z3_REDUCE_FP32) {
        if constexpr (SCALE) {
#pragma unroll
            for (int k = 0; k < 8; ++k) acc[k] = __fmul_rn(acc[k], a.inv_n);
        }
        float* o = static_cast<float*>(a.out) + e;
        st16(reinterpret_cast<float4*>(o), make_float4(acc[0], acc[1], acc[2], acc[3]));
        st16(reinterpret_cast<float4*>(o + 4), make_float4(acc[4], acc[5], acc[6], acc[7]));
    } else {
        if constexpr (SCALE) {
#pragma unroll
            for (int k = 0; k < 4; ++k)
                accw[k] = pack_bf16x2(__fmul_rn(lo_bf16(accw[k]), a.inv_n), __fmul_rn(hi_bf16(accw[k]), a.inv_n));
        }
        st16(reinterpret_cast<uint4*>(static_cast<uint16_t*>(a.out) + e),
             make_uint4(accw[0], accw[1], accw[2], accw[3]));
    }
}

// Blocks per SM the node-sum kernel asks for (the register cap follows from it).
// 3 blocks (80 registers) as in the fused kernel; the fp32 fold at 16 or more
// ranks hoists the loads of every rank chunk and spilled under that cap, so it
// gets 2 blocks (128 registers) at 16 ranks and 1 at 32: measured on B200 for
// the 7B block, 6771 -> 7242 GB/s at 16 ranks, 6022 -> 6432 GB/s at 32.
template <int MODE, int DT>
constexpr int node_sum_min_blocks() {
    return (MODE == Z3_REDUCE_FP32 && DT >= 32) ? 1 : (MODE == Z3_REDUCE_FP32 && DT >= 16) ? 2 : 3;
}

template <int MODE, int DT, bool SCALE>
__global__ void __launch_bounds__(kNfThreads, (node_sum_min_blocks<MODE, DT>()))
    k_node_sum_vec(const __grid_constant__ NodeSumArgs a) {
    const int64_t n8 = a.n >> 3;
    const int64_t step = int64_t(gridDim.x) * kNfThreads;
    for (int64_t q = int64_t(blockIdx.x) * kNfThreads + threadIdx.x; q < n8; q += step)
        node_sum8<MODE, DT, SCALE>(a, q << 3);
    const int64_t tail = (n8 << 3) + int64_t(blockIdx.x) * kNfThreads + threadIdx.x;
    if (tail < a.n) node_sum1<MODE, SCALE>(a, tail);
}

template <int MODE, bool SCALE>
__global__ void __launch_bounds__(kNfThreads) k_node_sum_scalar(const __grid_constant__ NodeSumArgs a) {
    const int64_t stride = int64_t(gridDim.x) * kNfThreads;
    for (int64_t i = int64_t(blockIdx.x) * kNfThreads + threadIdx.x; i < a.n; i += stride)
        node_sum1<MODE, SCALE>(a, i);
}

// ---------------------------------------------------- fold of the node sums
template <int MODE>
__device__ __forceinline__ float sum_at(const void* s, int64_t i) {
    if constexpr (MODE == Z3_REDUCE_FP32)
        return static_cast<const float*>(s)[i];
    else
        return bf16_of(static_cast<const uint16_t*>(s)[i]);
}

template <int MODE>
__device__ __forceinline__ void fold1(const FoldArgs& a, int64_t i) {
    float total = sum_at<MODE>(a.sums[0], i);
    for (int k = 1; k < a.R; ++k) total = add_in<MODE>(total, sum_at<MODE>(a.sums[k], i));
    const float g0 = __fmul_rn(total, a.inv_n);
    const float g = MODE == Z3_REDUCE_FP32 ? g0 : round_to_bf16(g0);
    float p = a.p[i], m = a.m[i], v = a.v[i];
    adamw_elem(a.s, g, p, m, v);
    a.p[i] = p;
    a.m[i] = m;
    a.v[i] = v;
    a.w[i] = __bfloat16_as_ushort(__float2bfloat16_rn(p));
}

template <int MODE, int RT>
__device__ __forceinline__ void fold8(const FoldArgs& a, int64_t e) {
    const int R = RT > 0 ? RT : a.R;
    const float4 p0 = ld16(reinterpret_cast<const float4*>(a.p + e));
    const float4 p1 = ld16(reinterpret_cast<const float4*>(a.p + e + 4));
    const float4 m0 = ld16(reinterpret_cast<const float4*>(a.m + e));
    const float4 m1 = ld16(reinterpret_cast<const float4*>(a.m + e + 4));
    const float4 v0 = ld16(reinterpret_cast<const float4*>(a.v + e));
    const float4 v1 = ld16(reinterpret_cast<const float4*>(a.v + e + 4));
    float g[8];
    if constexpr (MODE == Z3_REDUCE_FP32) {
        float tot[8];
#pragma unroll(RT > 0 ? RT : 1)
        for (int k = 0; k < R; ++k) {
            const float* s = static_cast<const float*>(a.sums[k]) + e;
            const float4 x = ld16(reinterpret_cast<const float4*>(s));
            const float4 y = ld16(reinterpret_cast<const float4*>(s + 4));
            const float xs[8] = {x.x, x.y, x.z, x.w, y.x, y.y, y.z, y.w};
#pragma unroll
            for (int i = 0; i < 8; ++i) tot[i] = k == 0 ? xs[i] : __fadd_rn(tot[i], xs[i]);
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) g[i] = __fmul_rn(tot[i], a.inv_n);
    } else {
        uint32_t tot[4];
#pragma unroll(RT > 0 ? RT : 1)
        for (int k = 0; k < R; ++k) {
            const uint4 q = ld16(reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(a.sums[k]) + e));
            fold8_bf16(tot, q, k == 0);
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            g[2 * i] = round_to_bf16(__fmul_rn(lo_bf16(tot[i]), a.inv_n));
            g[2 * i + 1] = round_to_bf16(__fmul_rn(hi_bf16(tot[i]), a.inv_n));
        }
    }
    float p[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
    float m[8] = {m0.x, m0.y, m0.z, m0.w, m1.x, m1.y, m1.z, m1.w};
    float v[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
#pragma unroll
    for (int k = 0; k < 8; ++k) adamw_elem(a.s, g[k], p[k], m[k], v[k]);
    st16(reinterpret_cast<float4*>(a.p + e), make_float4(p[0], p[1], p[2], p[3]));
    st16(reinterpret_cast<float4*>(a.p + e + 4), make_float4(p[4], p[5], p[6], p[7]));
    st16(reinterpret_cast<float4*>(a.m + e), make_float4(m[0], m[1], m[2], m[3]));
    st16(reinterpret_cast<float4*>(a.m + e + 4), make_float4(m[4], m[5], m[6], m[7]));
    st16(reinterpret_cast<float4*>(a.v + e), make_float4(v[0], v[1], v[2], v[3]));
    st16(reinterpret_cast<float4*>(a.v + e + 4), make_float4(v[4], v[5], v[6], v[7]));
    st16(reinterpret_cast<uint4*>(a.w + e), make_uint4(pack_bf16x2(p[0], p[1]), pack_bf16x2(p[2], p[3]),
                                                       pack_bf16x2(p[4], p[5]), pack_bf16x2(p[6], p[7])));
}

template <int MODE, int RT>
__global__ void __launch_bounds__(kNfThreads, 3) k_fold_adamw_vec(const __grid_constant__ FoldArgs a) {
    const int64_t n8 = a.n >> 3;
    const int64_t step = int64_t(gridDim.x) * kNfThreads;
    for (int64_t q = int64_t(blockIdx.x) * kNfThreads + threadIdx.x; q < n8; q += step) fold8<MODE, RT>(a, q << 3);
    const int64_t tail = (n8 << 3) + int64_t(blockIdx.x) * kNfThreads + threadIdx.x;
    if (tail < a.n) fold1<MODE>(a, tail);
}

template <int MODE>
__global__ void __launch_bounds__(kNfThreads) k_fold_adamw_scalar(const __grid_constant__ FoldArgs a) {
    const int64_t stride = int64_t(gridDim.x) * kNfThreads;
    for (int64_t i = int64_t(blockIdx.x) * kNfThreads + threadIdx.x; i < a.n; i += stride) fold1<MODE>(a, i);
}

// ------------------------------------------------------------------- launch
using NodeSumFn = void (*)(NodeSumArgs);
using FoldFn = void (*)(FoldArgs);

template <int MODE, bool SCALE>
NodeSumFn pick_node_sum(bool vec, int D) {
    if (!vec) return k_node_sum_scalar<MODE, SCALE>;
    switch (D) {
    case 1: return k_node_sum_vec<MODE, 1, SCALE>;
    case 2: return k_node_sum_vec<MODE, 2, SCALE>;
    case 4: return k_node_sum_vec<MODE, 4, SCALE>;
    case 8: return k_node_sum_vec<MODE, 8, SCALE>;
    case 16: return k_node_sum_vec<MODE, 16, SCALE>;
    case 32: return k_node_sum_vec<MODE, 32, SCALE>;
    default: return k_node_sum_vec<MODE, 0, SCALE>;
    }
}

template <int MODE>
FoldFn pick_fold(bool vec, int R) {
    if (!vec) return k_fold_adamw_scalar<MODE>;
    switch (R) {
    case 2: return k_fold_adamw_vec<MODE, 2>;
    case 4: return k_fold_adamw_vec<MODE, 4>;
    case 8: return k_fold_adamw_vec<MODE, 8>;
    default: return k_fold_adamw_vec<MODE, 0>;
    }
}

// Blocks for a launch over n elements: the vector kernels cover the range (one
// 8-element chunk per thread), the scalar kernels run whole resident waves.
template <class Fn>
int64_t grid_for(Fn fn, bool vec, int64_t n) {
    int64_t blocks;
    if (vec) {
        blocks = ((n >> 3) + kNfThreads - 1) / kNfThreads;
        if (blocks > kNfMaxBlocks) blocks = kNfMaxBlocks;
    } else {
        int per_sm = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, kNfThreads, 0) != cudaSuccess || per_sm < 1)
            per_sm = 1;
        const int sms = z3::sm_count();
        if (sms < 1) return -1;
        blocks = (n + kNfThreads - 1) / kNfThreads;
        const int64_t resident = int64_t(sms) * per_sm;
        if (blocks > resident) blocks = resident;
    }
    return blocks < 1 ? 1 : blocks;
}

}  // namespace

namespace {

// zero3_node_sum (scale = false) and zero3_reduce_scatter (scale = true).
int launch_node_sum(const z3_plan* p, int32_t rank, const uint16_t* const* contrib, int32_t contrib_layout,
                    int32_t reduce_dtype, void* node_sum, bool scale, void* cuda_stream) {
    if (p == nullptr || contrib == nullptr || node_sum == nullptr) return Z3_EINVAL;
    const int32_t D = p->D;
    if (rank < -1 || rank >= D) return Z3_EINVAL;
    if (contrib_layout != Z3_CONTRIB_FULL && contrib_layout != Z3_CONTRIB_OWNED) return Z3_EINVAL;
    if (contrib_layout == Z3_CONTRIB_OWNED && rank < 0) return Z3_EINVAL;
    if (reduce_dtype != Z3_REDUCE_FP32 && reduce_dtype != Z3_REDUCE_BF16) return Z3_EINVAL;
    const int64_t esz = reduce_dtype == Z3_REDUCE_FP32 ? 4 : 2;
    for (int32_t d = 0; d < D; ++d) {
        if (contrib[d] == nullptr) return Z3_EINVAL;
        if (!z3::aligned(contrib[d], 2)) return Z3_EALIGN;
    }
    if (!z3::aligned(node_sum, esz)) return Z3_EALIGN;
    const int64_t n = rank < 0 ? p->N_pad : p->S;
    const int64_t c_off = (contrib_layout == Z3_CONTRIB_FULL && rank >= 0) ? int64_t(rank) * p->S : 0;
    for (int32_t d = 0; d < D; ++d)
        if (z3::overlaps(node_sum, n * esz, contrib[d] + c_off, n * 2)) return Z3_EINVAL;
    if (n == 0) return Z3_OK;

    NodeSumArgs a;
    a.out = node_sum;
    a.n = n;
    a.D = D;
    a.inv_n = float(1.0 / double(D));
    bool vec = z3::aligned(node_sum, 16);
    for (int32_t d = 0; d < Z3_D_MAX; ++d) {
        a.c[d] = d < D ? contrib[d] + c_off : nullptr;
        if (d < D && !z3::aligned(a.c[d], 16)) vec = false;
    }
    NodeSumFn fn;
    if (scale)
        fn = reduce_dtype == Z3_REDUCE_FP32 ? pick_node_sum<Z3_REDUCE_FP32, true>(vec, D)
                                            : pick_node_sum<Z3_REDUCE_BF16, true>(vec, D);
    else
        fn = reduce_dtype == Z3_REDUCE_FP32 ? pick_node_sum<Z3_REDUCE_FP32, false>(vec, D)
                                            : pick_node_sum<Z3_REDUCE_BF16, false>(vec, D);
    const int64_t blocks = grid_for(fn, vec, n);
    if (blocks < 1) return Z3_ECUDA;
    fn<<<dim3(unsigned(blocks)), dim3(kNfThreads), 0, static_cast<cudaStream_t>(cuda_stream)>>>(a);
    return cudaGetLastError() == cudaSuccess ? Z3_OK : Z3_ECUDA;
}

}  // namespace

extern "C" Z3_API int zero3_node_sum(const z3_plan* p, int32_t rank, const uint16_t* const* contrib,
                                     int32_t contrib_layout, int32_t reduce_dtype, void* node_sum,
                                     void* cuda_stream) {
    return launch_node_sum(p, rank, contrib, contrib_layout, reduce_dtype, node_sum, false, cuda_stream);
}

extern "C" Z3_API int zero3_reduce_scatter(const z3_plan* p, int32_t rank, const uint16_t* const* contrib,
                                           int32_t contrib_layout, int32_t reduce_dtype, void* grad,
                                           void* cuda_stream) {
    return launch_node_sum(p, rank, contrib, contrib_layout, reduce_dtype, grad, true, cuda_stream);
}

extern "C" Z3_API int zero3_fold_adamw(const z3_plan* p, int32_t rank, int32_t n_nodes, const void* const* node_sums,
                                       float* master, float* exp_avg, float* exp_avg_sq, uint16_t* work_bf16,
                                       int32_t reduce_dtype, const z3_adamw* hp, void* cuda_stream) {
    if (p == nullptr || node_sums == nullptr || master == nullptr || exp_avg == nullptr || exp_avg_sq == nullptr ||
        work_bf16 == nullptr || !hp_valid(hp))
        return Z3_EINVAL;
    const int32_t D = p->D;
    if (rank < -1 || rank >= D || n_nodes < 1 || n_nodes > Z3_D_MAX) return Z3_EINVAL;
    if (reduce_dtype != Z3_REDUCE_FP32 && reduce_dtype != Z3_REDUCE_BF16) return Z3_EINVAL;
    const int64_t esz = reduce_dtype == Z3_REDUCE_FP32 ? 4 : 2;
    for (int32_t k = 0; k < n_nodes; ++k) {
        if (node_sums[k] == nullptr) return Z3_EINVAL;
        if (!z3::aligned(node_sums[k], esz)) return Z3_EALIGN;
    }
    if (!z3::aligned(master, 4) || !z3::aligned(exp_avg, 4) || !z3::aligned(exp_avg_sq, 4) ||
        !z3::aligned(work_bf16, 2))
        return Z3_EALIGN;
    const int64_t n = rank < 0 ? p->N_pad : p->S;
    // outputs overlap neither each other nor a node sum
    const void* outs[4] = {master, exp_avg, exp_avg_sq, work_bf16};
    const int64_t out_bytes[4] = {n * 4, n * 4, n * 4, n * 2};
    for (int x = 0; x < 4; ++x) {
        for (int y = x + 1; y < 4; ++y)
            if (z3::overlaps(outs[x], out_bytes[x], outs[y], out_bytes[y])) return Z3_EINVAL;
        for (int32_t k = 0; k < n_nodes; ++k)
            if (z3::overlaps(outs[x], out_bytes[x], node_sums[k], n * esz)) return Z3_EINVAL;
    }
    if (n == 0) return Z3_OK;

    FoldArgs a;
    a.p = master;
    a.m = exp_avg;
    a.v = exp_avg_sq;
    a.w = work_bf16;
    a.n = n;
    a.R = n_nodes;
    a.inv_n = float(1.0 / (double(n_nodes) * double(D)));
    a.s = step_scalars(hp);
    bool vec = z3::aligned(master, 16) && z3::aligned(exp_avg, 16) && z3::aligned(exp_avg_sq, 16) &&
               z3::aligned(work_bf16, 16);
    for (int32_t k = 0; k < Z3_D_MAX; ++k) {
        a.sums[k] = k < n_nodes ? node_sums[k] : nullptr;
        if (k < n_nodes && !z3::aligned(node_sums[k], 16)) vec = false;
    }
    const FoldFn fn = reduce_dtype == Z3_REDUCE_FP32 ? pick_fold<Z3_REDUCE_FP32>(vec, n_nodes)
                                                     : pick_fold<Z3_REDUCE_BF16>(vec, n_nodes);
    const int64_t blocks = grid_for(fn, vec, n);
    if (blocks < 1) return Z3_ECUDA;
    fn<<<dim3(unsigned(blocks)), dim3(kNfThreads), 0, static_cast<cudaStream_t>(cuda_stream)>>>(a);
    return cudaGetLastError() == cudaSuccess ? Z3_OK : Z3_ECUDA;
}
