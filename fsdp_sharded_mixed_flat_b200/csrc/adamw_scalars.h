// adamw_scalars.h -- the host side of one AdamW step, shared by the GPU
// kernels' launch code and the host optimiser: the eight fp32 scalars of a
// step and the validation of the hyper-parameters.
//
// AdamW with decoupled weight decay and bias-corrected moments (Loshchilov &
// Hutter, "Decoupled Weight Decay Regularization"); the pages name the
// optimiser ("7.10 — Fully-sharded data parallel (FSDP / ZeRO-3)", §3: rank r
// updates P_r from its fp32 master, m and v).  Every scalar is formed in
// binary64 and rounded to fp32 once.  Host code only; everything has internal
// linkage.
#pragma once

#include <cmath>
#include <cstdint>

#include "zero3.h"

namespace {

// The eight fp32 scalars of one AdamW step, in the order the C ABI documents
// for zero3_step_scalars.
struct AdamScalars {
    float step_size;     // lr / (1 - b1^t)
    float inv_sqrt_bc2;  // 1 / sqrt(1 - b2^t)
    float decay;         // 1 - lr * wd
    float b1, omb1, b2, omb2, eps;
};

static_assert(sizeof(AdamScalars) == Z3_SCALARS * sizeof(float), "scalar layout");

// Host computation of one step's scalars: binary64, each rounded to fp32 once.
inline AdamScalars step_scalars(const z3_adamw* hp) {
    AdamScalars s;
    const double t = double(hp->step);
    const double bc1 = 1.0 - std::pow(hp->beta1, t);
    const double bc2 = 1.0 - std::pow(hp->beta2, t);
    s.step_size = float(hp->lr / bc1);
    s.inv_sqrt_bc2 = float(1.0 / std::sqrt(bc2));
    s.decay = float(1.0 - hp->lr * hp->weight_decay);
    s.b1 = float(hp->beta1);
    s.omb1 = float(1.0 - hp->beta1);
    s.b2 = float(hp->beta2);
    s.omb2 = float(1.0 - hp->beta2);
    s.eps = float(hp->eps);
    return s;
}

inline bool is_finite(double x) { return std::isfinite(x); }

// A usable set of hyper-parameters: step >= 1, everything finite, betas in
// [0, 1), eps > 0, lr >= 0 and weight_decay >= 0.  eps > 0 keeps the update's
// denominator away from zero: with eps = 0 a zero-padded element (g = m = v = 0)
// would compute 0/0 and turn the pad into NaN.
inline bool hp_valid(const z3_adamw* hp) {
    return hp != nullptr && hp->step >= 1 && is_finite(hp->lr) && is_finite(hp->beta1) &&
           is_finite(hp->beta2) && is_finite(hp->eps) && is_finite(hp->weight_decay) && hp->beta1 >= 0.0 &&
           hp->beta1 < 1.0 && hp->beta2 >= 0.0 && hp->beta2 < 1.0 && hp->eps > 0.0 && hp->lr >= 0.0 &&
           hp->weight_decay >= 0.0;
}

}  // namespace
