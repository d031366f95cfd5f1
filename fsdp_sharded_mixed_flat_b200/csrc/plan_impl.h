// plan_impl.h -- the host-side plan object shared by the planner and the
// launch code of the kernels (never by the oracle).
#pragma once

#include <cstdint>
#include <vector>

#include "zero3.h"

struct z3_plan {
    int32_t D = 0;
    int32_t A = 0;
    int64_t N = 0;      // real elements
    int64_t N_pad = 0;  // padded elements, a multiple of D*A
    int64_t S = 0;      // elements per rank
    std::vector<int64_t> offset;  // per tensor: first flat element
    std::vector<int64_t> numel;   // per tensor: element count
};

namespace z3 {

// Overlap test of two byte ranges [a, a+na), [b, b+nb) (empty ranges never overlap).
inline bool overlaps(const void* a, int64_t na, const void* b, int64_t nb) {
    if (na <= 0 || nb <= 0) return false;
    auto x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
    return x < y + static_cast<uintptr_t>(nb) && y < x + static_cast<uintptr_t>(na);
}

inline bool aligned(const void* p, uintptr_t bytes) {
    return (reinterpret_cast<uintptr_t>(p) & (bytes - 1)) == 0;
}

// Number of streaming multiprocessors of the current device (cached per device).
int sm_count();

}  // namespace z3
