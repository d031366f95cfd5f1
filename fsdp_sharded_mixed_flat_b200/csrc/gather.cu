// gather.cu -- the all-gather's data movement and the unflatten, for sm_100a.
//
// "Building GPT from Scratch — Part 8: FSDP — When the Model Won't Fit",
// "AllGather vs AllReduce": GPU r holds shard r; after the all-gather every GPU
// holds the whole block [A, B, C, D].  "7.10 — Fully-sharded data parallel
// (FSDP / ZeRO-3)", §5.1: the gathered parameters are then used as the block's
// tensors (the unflatten).
//
// Both kernels are pure copies bound by HBM bandwidth (2 bytes read + 2 bytes
// written per element).
//   - flat copy: grid.y = one row per shard to copy (a shard already in place
//     inside the block is skipped), grid.x covering the shard (2 independent
//     16-byte vectors per thread, consecutive threads on consecutive vectors),
//     so the block scheduler balances the SMs; streaming stores.
//   - per-tensor copy: the host cuts every tensor into segments, one per rank
//     partition it intersects, and numbers the 16-byte units of each
//     segment's destination.  A block takes a run of consecutive units; one
//     thread finds the run's first segment by binary search and shares it
//     through shared memory, and each thread steps forward from there to the
//     segment of each of its two units (segments are long, so this is
//     rarely more than one step).  A whole unit is written with one 16-byte
//     store.  When the segment's source run is 16-byte aligned, the unit is
//     one aligned 16-byte load; otherwise the source run may start at any
//     2-byte position, and the unit is assembled from the two aligned 16-byte
//     source vectors around it with funnel shifts.  Partial units at a
//     segment's ends are written element by element.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <vector>

#include "plan_impl.h"
#include "zero3.h"

namespace {

constexpr int kThreads = 256;
constexpr int kUnroll = 2;                 // 16-byte vectors per thread in the flat copy
constexpr int64_t kMaxBlocks = 1 << 30;   // grid.x cap; beyond it the kernels loop
constexpr int kSegMax = 100;  // segments per launch; keeps the parameter block under 4 KB

struct FlatArgs {
    const uint16_t* shard[Z3_D_MAX];  // the shards to copy, in grid.y order
    int32_t rank[Z3_D_MAX];           // the partition each of them fills
    uint16_t* flat;
    int64_t S;
};

struct Seg {
    const uint16_t* src;  // first source element
    uint16_t* dst;        // first destination element
    int64_t len;          // elements
    int64_t unit_begin;   // index of the segment's first destination unit in this launch
    int32_t src_aligned;  // 1: src and dst both 16-byte aligned (whole units load one aligned vector)
};

struct SegArgs {
    Seg seg[kSegMax];
    int32_t nseg;
    int32_t vec;          // 1: sources may be read as aligned 16-byte vectors
    int64_t units;        // destination units in this launch
};
static_assert(sizeof(SegArgs) <= 4096, "segment table must fit the 4 KB parameter block");

__global__ void __launch_bounds__(kThreads) k_gather_flat_vec(const __grid_constant__ FlatArgs a) {
    const int y = blockIdx.y;
    const uint4* src = reinterpret_cast<const uint4*>(a.shard[y]);
    uint4* dst = reinterpret_cast<uint4*>(a.flat + int64_t(a.rank[y]) * a.S);
    const int64_t n = a.S >> 3;
    const int64_t span = int64_t(kThreads) * kUnroll;
    for (int64_t i = int64_t(blockIdx.x) * span + threadIdx.x; i < n; i += int64_t(gridDim.x) * span) {
        uint4 q[kUnroll];
#pragma unroll
        for (int k = 0; k < kUnroll; ++k)
            if (i + k * kThreads < n) q[k] = src[i + k * kThreads];
#pragma unroll
        for (int k = 0; k < kUnroll; ++k)
            if (i + k * kThreads < n) __stcs(dst + i + k * kThreads, q[k]);
    }
}

__global__ void __launch_bounds__(kThreads) k_gather_flat_scalar(const __grid_constant__ FlatArgs a) {
    const int y = blockIdx.y;
    const uint16_t* src = a.shard[y];
    uint16_t* dst = a.flat + int64_t(a.rank[y]) * a.S;
    const int64_t stride = int64_t(gridDim.x) * kThreads;
    for (int64_t j = int64_t(blockIdx.x) * kThreads + threadIdx.x; j < a.S; j += stride) dst[j] = src[j];
}

// Eight consecutive bf16 values starting at element pointer s, read as aligned
// 16-byte vectors (the caller guarantees both vectors lie inside the source).
__device__ __forceinline__ uint4 load8_unaligned(const uint16_t* s) {
    const uintptr_t addr = reinterpret_cast<uintptr_t>(s);
    const uint32_t delta = uint32_t(addr >> 1) & 7u;  // elements past the 16-byte boundary
    const uint4* base = reinterpret_cast<const uint4*>(addr & ~uintptr_t(15));
    const uint4 A = __ldcs(base);
    if (delta == 0) return A;
    const uint4 B = __ldcs(base + 1);
    const uint32_t w[8] = {A.x, A.y, A.z, A.w, B.x, B.y, B.z, B.w};
    const uint32_t q = delta >> 1;              // whole words to skip
    const uint32_t sh = (delta & 1u) * 16u;     // plus half a word
    uint32_t o[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        // words k+q and k+q+1, picked without dynamic register indexing
        uint32_t lo = w[k], hi = w[k + 1];
#pragma unroll
        for (int j = 1; j < 4; ++j)
            if (q == uint32_t(j)) { lo = w[k + j]; hi = w[k + j + 1]; }
        o[k] = __funnelshift_r(lo, hi, sh);
    }
    return make_uint4(o[0], o[1], o[2], o[3]);
}

// The segment holding destination unit u: the last one whose unit_begin <= u.
__device__ __forceinline__ int find_segment(const SegArgs& a, int64_t u) {
    int lo = 0, hi = a.nseg - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (a.seg[mid].unit_begin <= u) lo = mid; else hi = mid - 1;
    }
    return lo;
}

// kSegUnits destination units per thread (consecutive threads on consecutive
// units); the whole units' source vectors are all loaded before any store, so
// a thread keeps several 16-byte loads in flight.
constexpr int kSegUnits = 2;

__global__ void __launch_bounds__(kThreads) k_gather_segments(const __grid_constant__ SegArgs a) {
    __shared__ int first_seg;
    const int64_t span = int64_t(kThreads) * kSegUnits;
    // the loop bounds are the same for every thread of the block, so the barriers are uniform
    for (int64_t ub = int64_t(blockIdx.x) * span; ub < a.units; ub += int64_t(gridDim.x) * span) {
        if (threadIdx.x == 0) first_seg = find_segment(a, ub);
        __syncthreads();
        int si = first_seg;
        __syncthreads();  // first_seg is rewritten in the next iteration
        uint4 q[kSegUnits];
        uintptr_t dst[kSegUnits];
        bool whole[kSegUnits];
#pragma unroll
        for (int k = 0; k < kSegUnits; ++k) {
            const int64_t u = ub + threadIdx.x + int64_t(k) * kThreads;
            whole[k] = false;
            if (u >= a.units) continue;
            while (si + 1 < a.nseg && a.seg[si + 1].unit_begin <= u) ++si;
            const Seg& s = a.seg[si];
            const uintptr_t d0 = reinterpret_cast<uintptr_t>(s.dst);
            const uintptr_t unit_addr = (d0 & ~uintptr_t(15)) + uintptr_t(u - s.unit_begin) * 16u;
            // elements of this unit inside the segment: [k0, k1) relative to s.dst
            const int64_t k_first = (int64_t(unit_addr) - int64_t(d0)) / 2;  // may be negative
            if (a.vec && k_first >= 0 && k_first + 8 <= s.len) {
                q[k] = s.src_aligned ? *reinterpret_cast<const uint4*>(s.src + k_first)
                                     : load8_unaligned(s.src + k_first);
                dst[k] = unit_addr;
                whole[k] = true;
            } else {
                const int64_t k0 = k_first < 0 ? 0 : k_first;
                const int64_t k1 = k_first + 8 < s.len ? k_first + 8 : s.len;
                for (int64_t e = k0; e < k1; ++e) s.dst[e] = s.src[e];
            }
        }
#pragma unroll
        for (int k = 0; k < kSegUnits; ++k)
            if (whole[k]) __stcs(reinterpret_cast<uint4*>(dst[k]), q[k]);
    }
}

}  // namespace

extern "C" Z3_API int zero3_gather_block(const z3_plan* p, const uint16_t* const* shards, uint16_t* flat_out,
                                         uint16_t* const* tensor_out, void* cuda_stream) {
    if (p == nullptr || shards == nullptr || (flat_out == nullptr && tensor_out == nullptr)) return Z3_EINVAL;
    const int32_t D = p->D;
    const int64_t S = p->S;
    const int32_t nt = static_cast<int32_t>(p->numel.size());
    for (int32_t r = 0; r < D; ++r) {
        if (shards[r] == nullptr) return Z3_EINVAL;
        if (!z3::aligned(shards[r], 2)) return Z3_EALIGN;
    }
    if (flat_out != nullptr && !z3::aligned(flat_out, 2)) return Z3_EALIGN;
    if (tensor_out != nullptr)
        for (int32_t i = 0; i < nt; ++i)
            if (tensor_out[i] != nullptr && !z3::aligned(tensor_out[i], 2)) return Z3_EALIGN;
    // Shard r may sit in place inside the block, at exactly flat_out + r*S (a
    // rank's own shard as a view of its gathered block, the usual FSDP layout):
    // that partition is already where it belongs and is not copied.  Otherwise
    // outputs overlap neither the shards nor each other.
    auto in_place = [&](int32_t r) { return flat_out != nullptr && shards[r] == flat_out + int64_t(r) * S; };
    for (int32_t r = 0; r < D; ++r) {
        if (flat_out && !in_place(r) && z3::overlaps(flat_out, p->N_pad * 2, shards[r], S * 2)) return Z3_EINVAL;
        if (tensor_out)
            for (int32_t i = 0; i < nt; ++i)
                if (tensor_out[i] && z3::overlaps(tensor_out[i], p->numel[i] * 2, shards[r], S * 2))
                    return Z3_EINVAL;
    }
    if (tensor_out) {
        for (int32_t i = 0; i < nt; ++i) {
            if (!tensor_out[i]) continue;
            if (flat_out && z3::overlaps(tensor_out[i], p->numel[i] * 2, flat_out, p->N_pad * 2))
                return Z3_EINVAL;
            for (int32_t k = i + 1; k < nt; ++k)
                if (tensor_out[k] &&
                    z3::overlaps(tensor_out[i], p->numel[i] * 2, tensor_out[k], p->numel[k] * 2))
                    return Z3_EINVAL;
        }
    }
    if (p->N_pad == 0) return Z3_OK;

    const cudaStream_t stream = static_cast<cudaStream_t>(cuda_stream);
    const int sms = z3::sm_count();
    if (sms < 1) return Z3_ECUDA;
    bool vec_src = (S % 8) == 0;
    for (int32_t r = 0; r < D; ++r) vec_src = vec_src && z3::aligned(shards[r], 16);

    // ---- the all-gather into the flat block: one grid row per shard not already in place
    FlatArgs a;
    int32_t n_copy = 0;
    bool vec = (S % 8) == 0 && flat_out != nullptr && z3::aligned(flat_out, 16);
    for (int32_t r = 0; r < D; ++r) {
        if (flat_out == nullptr || in_place(r)) continue;
        a.shard[n_copy] = shards[r];
        a.rank[n_copy] = r;
        vec = vec && z3::aligned(shards[r], 16);
        ++n_copy;
    }
    if (n_copy > 0) {
        for (int32_t k = n_copy; k < Z3_D_MAX; ++k) {
            a.shard[k] = nullptr;
            a.rank[k] = 0;
        }
        a.flat = flat_out;
        a.S = S;
        auto fn = vec ? k_gather_flat_vec : k_gather_flat_scalar;
        int64_t bx;
        if (vec) {
            bx = ((S >> 3) + int64_t(kThreads) * kUnroll - 1) / (int64_t(kThreads) * kUnroll);
            bx = std::max<int64_t>(1, std::min(bx, kMaxBlocks));
        } else {
            int per_sm = 0;
            if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, kThreads, 0) != cudaSuccess || per_sm < 1)
                per_sm = 1;
            bx = (S + kThreads - 1) / kThreads;
            const int64_t cap = std::max<int64_t>(1, (int64_t(sms) * per_sm + n_copy - 1) / n_copy);
            bx = std::max<int64_t>(1, std::min(bx, cap));
        }
        fn<<<dim3(unsigned(bx), unsigned(n_copy)), dim3(kThreads), 0, stream>>>(a);
        if (cudaGetLastError() != cudaSuccess) return Z3_ECUDA;
    }

    // ---- the per-tensor copies, straight from the shards
    if (tensor_out != nullptr) {
        std::vector<Seg> segs;
        try {  // the segment list is host memory: an allocation failure is a status, not an exception
            for (int32_t i = 0; i < nt; ++i) {
                if (!tensor_out[i] || p->numel[i] == 0) continue;
                const int64_t b = p->offset[i], e = b + p->numel[i];
                for (int64_t r = b / S; r < D && r * S < e; ++r) {
                    const int64_t lo = std::max(b, r * S), hi = std::min(e, (r + 1) * S);
                    if (hi <= lo) continue;
                    Seg g{shards[r] + (lo - r * S), tensor_out[i] + (lo - b), hi - lo, 0, 0};
                    g.src_aligned = z3::aligned(g.src, 16) && z3::aligned(g.dst, 16) ? 1 : 0;
                    segs.push_back(g);
                }
            }
        } catch (...) {
            return Z3_ENOMEM;
        }
        for (size_t first = 0; first < segs.size(); first += kSegMax) {
            SegArgs a;
            a.nseg = int32_t(std::min<size_t>(kSegMax, segs.size() - first));
            a.vec = vec_src ? 1 : 0;
            int64_t units = 0;
            for (int32_t k = 0; k < a.nseg; ++k) {
                Seg s = segs[first + k];
                const uintptr_t d0 = reinterpret_cast<uintptr_t>(s.dst);
                const uintptr_t d1 = d0 + uintptr_t(s.len) * 2 - 1;
                s.unit_begin = units;
                units += int64_t((d1 >> 4) - (d0 >> 4)) + 1;
                a.seg[k] = s;
            }
            a.units = units;
            int64_t blocks = (units + int64_t(kThreads) * kSegUnits - 1) / (int64_t(kThreads) * kSegUnits);
            blocks = std::max<int64_t>(1, std::min<int64_t>(blocks, kMaxBlocks));
            k_gather_segments<<<dim3(unsigned(blocks)), dim3(kThreads), 0, stream>>>(a);
            if (cudaGetLastError() != cudaSuccess) return Z3_ECUDA;
        }
    }
    return Z3_OK;
}
