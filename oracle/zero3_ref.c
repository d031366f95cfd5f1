/*
 * zero3_ref.c -- the oracle.
 *
 * A plain, slow, single-threaded C99 restatement of the per-rank arithmetic of
 * one ZeRO-3 / FSDP training step, with the D data-parallel ranks simulated in
 * one address space.  Every loop walks the elements one by one, in the order
 * the method states; nothing is blocked, fused or reordered.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the package's smoke check and
 * the benchmark's CPU-baseline leg may load the library built from this file.
 * The CUDA product path shares no code, header, table or helper with it, and
 * neither side includes or loads the other.
 *
 * Build (oracle/build.py): gcc -std=c99 -O2 -ffp-contract=off -fno-fast-math
 * Every float expression below is a chain of single IEEE-754 binary32
 * operations, each rounded to nearest-even; -ffp-contract=off forbids fusing
 * a*b+c into one FMA.  Host scalars are computed in binary64 and rounded to
 * binary32 once.
 *
 * Precision.  The pages fix the precisions of this path: bf16 working weights,
 * fp32 master weights and fp32 Adam moments, and a reduce dtype of fp32 or
 * bf16.  The oracle computes in exactly those types, so binary32 (not
 * binary64) is the oracle's arithmetic.
 *
 * Sources, cited by page title and section:
 *   [P1] "Distributed LLM Fine-Tuning at Scale: FSDP, ZeRO-3, and Multi-GPU
 *         Orchestration", §1 The Memory Sharding Mathematics, §2 PyTorch FSDP
 *         Production Python Snippet (the MixedPrecision policy).
 *   [P2] "7.10 — Fully-sharded data parallel (FSDP / ZeRO-3)", §2 Recap: DP
 *         memory in three buckets, §3 ZeRO-1, §4 ZeRO-2, §5.1 Forward and
 *         backward pass under FSDP, §5.2 Memory accounting, §5.3 Extra
 *         communication.
 *   [P3] "Building GPT from Scratch — Part 8: FSDP — When the Model Won't
 *         Fit", sections "AllGather vs AllReduce", "Mixed Precision:
 *         Cutting Memory in Half", "HYBRID_SHARD: The Multi-Node Strategy"
 *         and "Key Takeaways".
 *
 * Readings where the pages are silent:
 *   - flat layout: tensors packed row-major in list order, no padding between
 *     tensors, zero padding at the tail to a multiple of D*A elements;
 *   - the reduction sums ranks 0..D-1 left to right, starting from rank 0's
 *     value, then multiplies by the binary32 constant 1/D;
 *   - bf16 reduce: every partial sum is rounded to bf16 (round-nearest-even);
 *   - HYBRID_SHARD: node sums first, then the node sums in node order, then
 *     1/(R*D) (reduce_hybrid_one() below);
 *   - AdamW: decoupled weight decay applied to every element, bias-corrected
 *     moments, 1-based step count, the operation order of adamw_one() below;
 *   - every fp32 -> bf16 conversion rounds to nearest-even.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

/* ------------------------------------------------------------------------ */
/* bf16 <-> binary32.  bf16 is the upper half of a binary32 bit pattern.     */
/* Rounding to nearest-even, written from the IEEE-754 definition: keep the  */
/* upper 16 bits; the lower 16 bits are the discarded fraction; round up if  */
/* it is above one half, or exactly one half and the kept part is odd.  A    */
/* carry out of the kept fraction correctly bumps the exponent (up to inf).  */
/* ------------------------------------------------------------------------ */
uint16_t ref_bf16_from_f32(float x)
{
    uint32_t u;
    memcpy(&u, &x, sizeof u);
    uint32_t kept = u >> 16;
    uint32_t dropped = u & 0xFFFFu;
    int is_nan = ((u & 0x7F800000u) == 0x7F800000u) && ((u & 0x007FFFFFu) != 0u);
    if (is_nan)
        return (uint16_t)(kept | 0x0040u); /* stay NaN: force a quiet-NaN fraction bit */
    if (dropped > 0x8000u || (dropped == 0x8000u && (kept & 1u)))
        kept += 1u;
    return (uint16_t)kept;
}

float ref_f32_from_bf16(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float x;
    memcpy(&x, &u, sizeof x);
    return x;
}

void ref_bf16_from_f32_array(const float* x, int64_t n, uint16_t* out)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = ref_bf16_from_f32(x[i]);
}

/* ------------------------------------------------------------------------ */
/* Flat-parameter plan.  [P2] §3: rank r owns a partition P_r of roughly 1/D */
/* of the parameters.  Tensors are laid out one after the other in list      */
/* order; the tail is padded with zeros so that N_pad is a multiple of D*A   */
/* and every partition has S = N_pad / D elements, P_r = [r*S, (r+1)*S).     */
/* Returns 0, or -1 on an invalid argument.                                   */
/* ------------------------------------------------------------------------ */
int ref_plan(int32_t n_tensors, const int64_t* numel, int32_t D, int32_t A,
             int64_t* offset_out, int64_t* N_out, int64_t* N_pad_out, int64_t* S_out)
{
    if (n_tensors < 0 || D < 1 || A < 1)
        return -1;
    int64_t N = 0;
    for (int32_t t = 0; t < n_tensors; ++t) {
        if (numel[t] < 0)
            return -1;
        offset_out[t] = N;
        N += numel[t];
    }
    int64_t unit = (int64_t)D * (int64_t)A;
    int64_t units = N / unit;
    if (units * unit < N)
        units += 1;
    *N_out = N;
    *N_pad_out = units * unit;
    *S_out = *N_pad_out / D;
    return 0;
}

/* Rank r's partition [r*S, (r+1)*S) and the end of its real (unpadded)
 * elements, min((r+1)*S, N), never below the partition's start. */
void ref_rank_range(int64_t N, int64_t S, int32_t r, int64_t* begin, int64_t* end_real)
{
    int64_t b = (int64_t)r * S;
    int64_t e = b + S;
    if (e > N)
        e = N;
    if (e < b)
        e = b;
    *begin = b;
    *end_real = e;
}

/* ------------------------------------------------------------------------ */
/* Memory ledger, bytes per device.  [P2] §2: under pure DP with bf16 mixed  */
/* precision and Adam, each parameter costs 2 B of working weights, about    */
/* 6 B of gradient (bf16 with an fp32 accumulator) and 12 B of optimiser     */
/* state (fp32 master, m, v): about 20 B in all.  ZeRO-1 shards the 12 B     */
/* bucket, ZeRO-2 also the 6 B bucket, ZeRO-3 all three.                     */
/* stage: 0 = pure DP, 1, 2, 3.  Returns -1.0 for an unknown stage.          */
/* ------------------------------------------------------------------------ */
double ref_memory_bytes(double N, double D, int32_t stage)
{
    const double weights = 2.0, grads = 6.0, optim = 12.0;
    switch (stage) {
    case 0: return (weights + grads + optim) * N;
    case 1: return optim * N / D + weights * N + grads * N;
    case 2: return (optim + grads) * N / D + weights * N;
    case 3: return (weights + grads + optim) * N / D;
    default: return -1.0;
    }
}

/* [P2] §5.2: the gathered full parameters of one block take |theta_block|*2
 * bytes in bf16; n_buffers of them are held at once (two when the forward
 * and backward gathers overlap). */
double ref_transient_bytes(double block_params, int32_t n_buffers)
{
    return (double)n_buffers * block_params * 2.0;
}

/* [P2] §5.3: every pass gathers each block once; a device already holds its
 * own 1/D of the block and receives the other (D-1)/D.  Bytes received per
 * device for n_blocks blocks of block_bytes each. */
double ref_allgather_bytes(double block_bytes, int32_t n_blocks, int32_t D)
{
    return (double)n_blocks * block_bytes * (double)(D - 1) / (double)D;
}

/* ------------------------------------------------------------------------ */
/* Reduce-scatter, one owned element.  [P3] "AllGather vs AllReduce": after  */
/* the reduce-scatter, GPU r holds the sum over all GPUs of the r-th slice   */
/* of their gradients; [P2] §4: rank r ends up with the summed gradient for  */
/* its partition P_r only.  The sum is scaled by 1/D to the average.         */
/* idx is the element's index inside every contribution buffer.              */
/* reduce_dtype 0: binary32 accumulator.  1: bf16 accumulator ([P1] §2's     */
/* reduce_dtype=bfloat16), each partial sum rounded to bf16.                 */
/* ------------------------------------------------------------------------ */
static float reduce_one(int32_t D, const uint16_t* const* contrib, int64_t idx,
                        int32_t reduce_dtype, float inv_D)
{
    if (reduce_dtype == 0) {
        float acc = ref_f32_from_bf16(contrib[0][idx]);
        for (int32_t d = 1; d < D; ++d)
            acc = acc + ref_f32_from_bf16(contrib[d][idx]);
        return acc * inv_D;
    } else {
        uint16_t acc = contrib[0][idx];
        for (int32_t d = 1; d < D; ++d)
            acc = ref_bf16_from_f32(ref_f32_from_bf16(acc) + ref_f32_from_bf16(contrib[d][idx]));
        return ref_f32_from_bf16(ref_bf16_from_f32(ref_f32_from_bf16(acc) * inv_D));
    }
}

/* The binary32 constant 1/D. */
static float inverse_of(int32_t D)
{
    return (float)(1.0 / (double)D);
}

/* Index of owned element j of rank r inside a contribution buffer.
 * layout 0 (full): every contribution spans the whole padded block [0, N_pad).
 * layout 1 (owned): every contribution already starts at P_r. */
static int64_t contrib_index(int32_t layout, int64_t S, int32_t r, int64_t j)
{
    return layout == 0 ? (int64_t)r * S + j : j;
}

/* The reduced (averaged) gradient for rank `rank`'s partition (S elements),
 * or for every rank in order (rank = -1: N_pad elements, g_out[r*S + j]).
 * Returns 0, or -1 on an invalid argument. */
int ref_reduce_scatter(int32_t D, int64_t S, int32_t rank, const uint16_t* const* contrib,
                       int32_t layout, int32_t reduce_dtype, float* g_out)
{
    if (D < 1 || S < 0 || rank < -1 || rank >= D || (layout != 0 && layout != 1) ||
        (reduce_dtype != 0 && reduce_dtype != 1) || (rank == -1 && layout == 1))
        return -1;
    float inv_D = inverse_of(D);
    int32_t r0 = rank < 0 ? 0 : rank;
    int32_t r1 = rank < 0 ? D : rank + 1;
    for (int32_t r = r0; r < r1; ++r)
        for (int64_t j = 0; j < S; ++j) {
            int64_t out = rank < 0 ? (int64_t)r * S + j : j;
            g_out[out] = reduce_one(D, contrib, contrib_index(layout, S, r, j), reduce_dtype, inv_D);
        }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* AdamW on the owned shard.  [P2] §3: rank r updates only the parameters in */
/* P_r, from its local fp32 master, m and v and the rank-r slice of the      */
/* gradient; [P3] "Mixed Precision": the fp32 master stays, the working      */
/* weights are bf16.  The pages name AdamW but print no equations; this is   */
/* the plain reading of decoupled weight decay with bias-corrected moments   */
/* (Loshchilov & Hutter, "Decoupled Weight Decay Regularization").           */
/* ------------------------------------------------------------------------ */
typedef struct {
    double lr, beta1, beta2, eps, weight_decay;
    int64_t step; /* 1-based */
} ref_adamw_hp;

typedef struct {
    float step_size, inv_sqrt_bc2, decay, b1, omb1, b2, omb2, eps;
} ref_adamw_consts;

/* Host scalars: computed in binary64, each rounded to binary32 once. */
static ref_adamw_consts adamw_consts(const ref_adamw_hp* hp)
{
    ref_adamw_consts c;
    double t = (double)hp->step;
    double bias_correction1 = 1.0 - pow(hp->beta1, t);
    double bias_correction2 = 1.0 - pow(hp->beta2, t);
    c.step_size = (float)(hp->lr / bias_correction1);
    c.inv_sqrt_bc2 = (float)(1.0 / sqrt(bias_correction2));
    c.decay = (float)(1.0 - hp->lr * hp->weight_decay);
    c.b1 = (float)hp->beta1;
    c.omb1 = (float)(1.0 - hp->beta1);
    c.b2 = (float)hp->beta2;
    c.omb2 = (float)(1.0 - hp->beta2);
    c.eps = (float)hp->eps;
    return c;
}

void ref_adamw_consts_of(const ref_adamw_hp* hp, float* out8)
{
    ref_adamw_consts c = adamw_consts(hp);
    out8[0] = c.step_size;
    out8[1] = c.inv_sqrt_bc2;
    out8[2] = c.decay;
    out8[3] = c.b1;
    out8[4] = c.omb1;
    out8[5] = c.b2;
    out8[6] = c.omb2;
    out8[7] = c.eps;
}

/* One element, one binary32 operation per statement. */
static void adamw_one(const ref_adamw_consts* c, float g, float* p, float* m, float* v)
{
    float p1 = *p * c->decay;                      /* decoupled weight decay */
    float m_old = c->b1 * *m;
    float m_new_part = c->omb1 * g;
    float m1 = m_old + m_new_part;                 /* first moment */
    float g2 = g * g;
    float v_old = c->b2 * *v;
    float v_new_part = c->omb2 * g2;
    float v1 = v_old + v_new_part;                 /* second moment */
    float root = sqrtf(v1);
    float root_hat = root * c->inv_sqrt_bc2;       /* sqrt of the bias-corrected v */
    float denom = root_hat + c->eps;
    float ratio = m1 / denom;
    float delta = c->step_size * ratio;            /* step_size carries 1/bias_correction1 */
    float p2 = p1 - delta;
    *p = p2;
    *m = m1;
    *v = v1;
}

/* AdamW alone on n elements, gradient given in binary32. */
int ref_adamw(int64_t n, const float* g, float* master, float* exp_avg, float* exp_avg_sq,
              const ref_adamw_hp* hp)
{
    if (n < 0 || hp->step < 1)
        return -1;
    ref_adamw_consts c = adamw_consts(hp);
    for (int64_t i = 0; i < n; ++i)
        adamw_one(&c, g[i], &master[i], &exp_avg[i], &exp_avg_sq[i]);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* The whole per-rank step: reduce-scatter of the D contributions for P_r,   */
/* AdamW on the owned master / m / v, and the cast of the new master to the  */
/* bf16 working shard ([P2] §3; [P3] "Mixed Precision").                      */
/* rank = r: state arrays hold P_r (S elements, index j).                     */
/* rank = -1: every rank in turn; state arrays hold the whole padded block    */
/*            (N_pad = D*S elements, index r*S + j).                          */
/* Returns 0, or -1 on an invalid argument.                                   */
/* ------------------------------------------------------------------------ */
int ref_reduce_adamw(int32_t D, int64_t S, int32_t rank, const uint16_t* const* contrib,
                     int32_t layout, float* master, float* exp_avg, float* exp_avg_sq,
                     uint16_t* work_bf16, int32_t reduce_dtype, const ref_adamw_hp* hp)
{
    if (D < 1 || S < 0 || rank < -1 || rank >= D || (layout != 0 && layout != 1) ||
        (reduce_dtype != 0 && reduce_dtype != 1) || (rank == -1 && layout == 1) || hp->step < 1)
        return -1;
    ref_adamw_consts c = adamw_consts(hp);
    float inv_D = inverse_of(D);
    int32_t r0 = rank < 0 ? 0 : rank;
    int32_t r1 = rank < 0 ? D : rank + 1;
    for (int32_t r = r0; r < r1; ++r)
        for (int64_t j = 0; j < S; ++j) {
            int64_t s = rank < 0 ? (int64_t)r * S + j : j;
            float g = reduce_one(D, contrib, contrib_index(layout, S, r, j), reduce_dtype, inv_D);
            adamw_one(&c, g, &master[s], &exp_avg[s], &exp_avg_sq[s]);
            work_bf16[s] = ref_bf16_from_f32(master[s]);
        }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* HYBRID_SHARD.  [P3] "HYBRID_SHARD: The Multi-Node Strategy": R nodes of D */
/* GPUs; the model is sharded D ways inside each node and replicated across  */
/* the nodes, and the gradient crosses nodes in one all-reduce.  [P3] "Key   */
/* Takeaways": the result is the same gradient as on one GPU, so the sum is  */
/* scaled by 1/(R*D), the average over every data-parallel rank.             */
/* Reading: global rank k*D + d is local rank d of node k, and its           */
/* contribution is contrib[k*D + d].  Inside node k the ranks are folded     */
/* 0..D-1 left to right (the node's reduce-scatter); the R node sums are     */
/* then folded in node order 0..R-1 (the cross-node all-reduce, which leaves */
/* the same sum on every node, so the replicas stay identical); the total is */
/* multiplied by the binary32 constant 1/(R*D).  In bf16 mode every partial  */
/* sum, inside a node and across nodes, is rounded to bf16.  R = 1 is the    */
/* plain reduction above.                                                    */
/* ------------------------------------------------------------------------ */
static float reduce_hybrid_one(int32_t R, int32_t D, const uint16_t* const* contrib, int64_t idx,
                               int32_t reduce_dtype, float inv_RD)
{
    if (reduce_dtype == 0) {
        float total = 0.0f;
        for (int32_t k = 0; k < R; ++k) {
            const uint16_t* const* node = contrib + (int64_t)k * D;
            float node_sum = ref_f32_from_bf16(node[0][idx]);
            for (int32_t d = 1; d < D; ++d)
                node_sum = node_sum + ref_f32_from_bf16(node[d][idx]);
            total = (k == 0) ? node_sum : total + node_sum;
        }
        return total * inv_RD;
    } else {
        uint16_t total = 0;
        for (int32_t k = 0; k < R; ++k) {
            const uint16_t* const* node = contrib + (int64_t)k * D;
            uint16_t node_sum = node[0][idx];
            for (int32_t d = 1; d < D; ++d)
                node_sum = ref_bf16_from_f32(ref_f32_from_bf16(node_sum) + ref_f32_from_bf16(node[d][idx]));
            total = (k == 0) ? node_sum
                             : ref_bf16_from_f32(ref_f32_from_bf16(total) + ref_f32_from_bf16(node_sum));
        }
        return ref_f32_from_bf16(ref_bf16_from_f32(ref_f32_from_bf16(total) * inv_RD));
    }
}

static int hybrid_args_invalid(int32_t R, int32_t D, int64_t S, int32_t rank, int32_t layout,
                               int32_t reduce_dtype)
{
    return R < 1 || D < 1 || S < 0 || rank < -1 || rank >= D || (layout != 0 && layout != 1) ||
           (reduce_dtype != 0 && reduce_dtype != 1) || (rank == -1 && layout == 1);
}

/* The averaged gradient of the HYBRID_SHARD step for local rank `rank`'s
 * partition (S elements), or for every local rank in order (rank = -1: the
 * node's N_pad elements).  contrib holds R*D buffers; layouts as for
 * ref_reduce_scatter.  Returns 0, or -1 on an invalid argument. */
int ref_reduce_scatter_hybrid(int32_t R, int32_t D, int64_t S, int32_t rank, const uint16_t* const* contrib,
                              int32_t layout, int32_t reduce_dtype, float* g_out)
{
    if (hybrid_args_invalid(R, D, S, rank, layout, reduce_dtype))
        return -1;
    float inv_RD = inverse_of(R * D);
    int32_t r0 = rank < 0 ? 0 : rank;
    int32_t r1 = rank < 0 ? D : rank + 1;
    for (int32_t r = r0; r < r1; ++r)
        for (int64_t j = 0; j < S; ++j) {
            int64_t out = rank < 0 ? (int64_t)r * S + j : j;
            g_out[out] = reduce_hybrid_one(R, D, contrib, contrib_index(layout, S, r, j), reduce_dtype, inv_RD);
        }
    return 0;
}

/* The whole HYBRID_SHARD step of local rank `rank` (or of every local rank):
 * the two-level reduction above, AdamW on the owned state, the bf16 cast.
 * Every node's replica of the rank computes exactly this. */
int ref_reduce_adamw_hybrid(int32_t R, int32_t D, int64_t S, int32_t rank, const uint16_t* const* contrib,
                            int32_t layout, float* master, float* exp_avg, float* exp_avg_sq,
                            uint16_t* work_bf16, int32_t reduce_dtype, const ref_adamw_hp* hp)
{
    if (hybrid_args_invalid(R, D, S, rank, layout, reduce_dtype) || hp->step < 1)
        return -1;
    ref_adamw_consts c = adamw_consts(hp);
    float inv_RD = inverse_of(R * D);
    int32_t r0 = rank < 0 ? 0 : rank;
    int32_t r1 = rank < 0 ? D : rank + 1;
    for (int32_t r = r0; r < r1; ++r)
        for (int64_t j = 0; j < S; ++j) {
            int64_t s = rank < 0 ? (int64_t)r * S + j : j;
            float g = reduce_hybrid_one(R, D, contrib, contrib_index(layout, S, r, j), reduce_dtype, inv_RD);
            adamw_one(&c, g, &master[s], &exp_avg[s], &exp_avg_sq[s]);
            work_bf16[s] = ref_bf16_from_f32(master[s]);
        }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* HYBRID_SHARD across nodes, in two parts.  Between nodes the node sums have */
/* to exist in memory: each rank computes its node's sum for its partition,  */
/* the sums cross the nodes (one exchange per step), and every node folds    */
/* them in node order.  Composed, the two parts are reduce_hybrid_one above. */
/* ------------------------------------------------------------------------ */

/* Part 1: the node's sum for local rank `rank`'s partition (S elements), or for
 * every partition (rank = -1, D*S elements): its D contributions folded left
 * to right in rank order, not scaled.  reduce_dtype 1 rounds every partial sum
 * to bf16, so every result is a bf16 value (held here in binary32).
 * Returns 0, or -1 on an invalid argument. */
int ref_node_sum(int32_t D, int64_t S, int32_t rank, const uint16_t* const* contrib, int32_t layout,
                 int32_t reduce_dtype, float* out)
{
    if (hybrid_args_invalid(1, D, S, rank, layout, reduce_dtype))
        return -1;
    int32_t r0 = rank < 0 ? 0 : rank;
    int32_t r1 = rank < 0 ? D : rank + 1;
    for (int32_t r = r0; r < r1; ++r)
        for (int64_t j = 0; j < S; ++j) {
            int64_t idx = contrib_index(layout, S, r, j);
            int64_t o = rank < 0 ? (int64_t)r * S + j : j;
            if (reduce_dtype == 0) {
                float acc = ref_f32_from_bf16(contrib[0][idx]);
                for (int32_t d = 1; d < D; ++d)
                    acc = acc + ref_f32_from_bf16(contrib[d][idx]);
                out[o] = acc;
            } else {
                uint16_t acc = contrib[0][idx];
                for (int32_t d = 1; d < D; ++d)
                    acc = ref_bf16_from_f32(ref_f32_from_bf16(acc) + ref_f32_from_bf16(contrib[d][idx]));
                out[o] = ref_f32_from_bf16(acc);
            }
        }
    return 0;
}

/* Part 2: for n owned elements, the R node sums (node_sums[k][i], node k's sum,
 * as part 1 wrote it) folded in node order 0..R-1, multiplied by the binary32
 * constant 1/(R*D), then AdamW on master / exp_avg / exp_avg_sq and the cast
 * of the new master to work_bf16.  In bf16 mode every partial sum across nodes
 * and the scaled result are rounded to bf16.  Returns 0, or -1 on an invalid
 * argument. */
int ref_fold_adamw(int32_t R, int32_t D, int64_t n, const float* const* node_sums, float* master,
                   float* exp_avg, float* exp_avg_sq, uint16_t* work_bf16, int32_t reduce_dtype,
                   const ref_adamw_hp* hp)
{
    if (R < 1 || D < 1 || n < 0 || (reduce_dtype != 0 && reduce_dtype != 1) || hp->step < 1)
        return -1;
    ref_adamw_consts c = adamw_consts(hp);
    float inv_RD = inverse_of(R * D);
    for (int64_t i = 0; i < n; ++i) {
        float total = node_sums[0][i];
        for (int32_t k = 1; k < R; ++k) {
            total = total + node_sums[k][i];
            if (reduce_dtype == 1)
                total = ref_f32_from_bf16(ref_bf16_from_f32(total));
        }
        float g = total * inv_RD;
        if (reduce_dtype == 1)
            g = ref_f32_from_bf16(ref_bf16_from_f32(g));
        adamw_one(&c, g, &master[i], &exp_avg[i], &exp_avg_sq[i]);
        work_bf16[i] = ref_bf16_from_f32(master[i]);
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* All-gather.  [P3] "AllGather vs AllReduce": GPU r holds shard r; after    */
/* the all-gather every GPU holds [shard 0, shard 1, ..., shard D-1].        */
/* [P2] §5.1: full_params = all_gather(local_shard) before the block runs.   */
/* ------------------------------------------------------------------------ */
void ref_all_gather(int32_t D, int64_t S, const uint16_t* const* shards, uint16_t* flat)
{
    for (int32_t r = 0; r < D; ++r)
        for (int64_t j = 0; j < S; ++j)
            flat[(int64_t)r * S + j] = shards[r][j];
}

/* Unflatten: tensor t is the row-major run flat[offset[t], offset[t] + numel[t]).
 * Copies each run into its own buffer. */
void ref_unflatten(const uint16_t* flat, int32_t n_tensors, const int64_t* offset,
                   const int64_t* numel, uint16_t* const* out)
{
    for (int32_t t = 0; t < n_tensors; ++t)
        for (int64_t k = 0; k < numel[t]; ++k)
            out[t][k] = flat[offset[t] + k];
}
