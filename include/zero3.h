/*
 * zero3.h -- C ABI of the B200 library for the per-rank arithmetic of one
 * ZeRO-3 / FSDP training step, with D data-parallel ranks simulated on one GPU.
 *
 * Pages cited (by title and section):
 *   [P1] "Distributed LLM Fine-Tuning at Scale: FSDP, ZeRO-3, and Multi-GPU
 *         Orchestration"
 *   [P2] "7.10 — Fully-sharded data parallel (FSDP / ZeRO-3)"
 *   [P3] "Building GPT from Scratch — Part 8: FSDP — When the Model Won't Fit"
 *
 * Conventions for every entry point
 *   - Return value: Z3_OK (0) or a negative Z3_E* status.  No C++ exception
 *     ever crosses this boundary.
 *   - bf16 values are passed as uint16_t bit patterns.
 *   - Device pointers are plain CUDA global-memory addresses on the current
 *     device.  The caller owns and allocates every device buffer; the library
 *     never allocates, frees or keeps device memory.  Host arrays of device
 *     pointers (contrib, gathered, shards, tensor_out) are read during the
 *     call only.  zero3_host_adamw alone works on host memory, synchronously;
 *     it keeps a pool of host threads for later calls.
 *   - Device work is enqueued on `cuda_stream` (a cudaStream_t; NULL means the
 *     legacy default stream) and the call returns without synchronising.
 *     Argument and alignment errors are reported synchronously, before any
 *     device work is enqueued; a failed launch returns Z3_ECUDA; errors that
 *     happen while the kernels run surface at the caller's next synchronise.
 *   - Outputs must not overlap inputs or each other unless stated (the
 *     optimiser state is updated in place, which is the one sanctioned
 *     input/output pairing).  Overlaps the library can see are rejected with
 *     Z3_EINVAL.
 *   - Element counts are int64_t; a plan may describe up to 2^62 elements.
 *   - A plan is an immutable host object: it can be shared between threads
 *     and streams, and must outlive the calls that use it.
 */
#ifndef ZERO3_H
#define ZERO3_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define Z3_API __attribute__((visibility("default")))
#else
#define Z3_API
#endif

/* ----------------------------------------------------------------- status */
enum {
    Z3_OK = 0,
    Z3_EINVAL = -1,    /* a NULL pointer, a value out of range, overlapping buffers */
    Z3_EALIGN = -2,    /* a pointer not aligned to its element size */
    Z3_ENOMEM = -3,    /* host allocation failed (a plan, a segment list, a host thread) */
    Z3_ECUDA = -4,     /* a CUDA runtime call or kernel launch failed */
    Z3_EOVERFLOW = -5  /* a size does not fit in int64_t */
};

/* Largest number of simulated ranks D one call accepts (with HYBRID_SHARD,
 * the largest n_nodes * D). */
#define Z3_D_MAX 64

/* Largest number of gathered blocks zero3_reduce_adamw_gather writes in one call. */
#define Z3_GATHER_MAX 8

/* Number of fp32 scalars zero3_step_scalars writes. */
#define Z3_SCALARS 8

/* Reduce dtype, the MixedPrecision policy's reduce_dtype ([P1] §2 uses
 * bfloat16; [P3] "Mixed Precision: Cutting Memory in Half" uses float32). */
enum {
    Z3_REDUCE_FP32 = 0, /* fp32 accumulator: each partial sum rounded to fp32 */
    Z3_REDUCE_BF16 = 1  /* bf16 accumulator: each partial sum rounded to bf16 */
};

/* Layout of the D gradient contributions handed to zero3_reduce_adamw. */
enum {
    Z3_CONTRIB_FULL = 0, /* contrib[d] spans the whole padded block [0, N_pad);
                            rank r's owned element j is contrib[d][r*S + j] */
    Z3_CONTRIB_OWNED = 1 /* contrib[d] starts at rank r's partition: element j is
                            contrib[d][j] (only with one rank per call) */
};

/* Stages of the memory ledger ([P2] §2). */
enum { Z3_STAGE_DDP = 0, Z3_STAGE_ZERO1 = 1, Z3_STAGE_ZERO2 = 2, Z3_STAGE_ZERO3 = 3 };

/* One tensor of a flat-parameter block: `ndim` sizes in `shape` (row-major,
 * 0 <= ndim <= 4; ndim = 0 is a scalar), whose product must equal `numel`. */
typedef struct {
    int64_t numel;
    int32_t ndim;
    int64_t shape[4];
} z3_tensor_spec;

/* AdamW hyper-parameters for one optimiser step.  `step` is the 1-based step
 * count t used for the bias corrections. */
typedef struct {
    double lr, beta1, beta2, eps, weight_decay;
    int64_t step;
} z3_adamw;

/* Opaque host-side plan of one flat-parameter block. */
typedef struct z3_plan z3_plan;

/* Text for a status code (a static string; never NULL). */
Z3_API const char* zero3_status_string(int status);

/* ------------------------------------------------------------------ plan
 * zero3_plan: lay a block's tensors out as one flat buffer and partition it
 * over D ranks.  [P2] §3: rank r owns a partition P_r of roughly 1/D of the
 * parameters; [P2] §5.1 and [P1] §2: the unit of sharding is one block (one
 * wrapped transformer layer), gathered whole before it runs.
 *   Layout: tensors packed row-major in list order with no gaps; the tail is
 *   zero-padded so that N_pad = ceil(N / (D*A)) * D*A; every rank owns
 *   S = N_pad / D elements, P_r = [r*S, (r+1)*S).  align_elems = A >= 1;
 *   A = 128 keeps every partition 256-byte aligned in bf16 and 512-byte
 *   aligned in fp32, which the vectorised kernels need (A*D % 8 == 0).
 *   t: host array of n_tensors specs (may be NULL when n_tensors == 0).
 *   *out: receives a new plan; release it with zero3_plan_free.
 * Errors: Z3_EINVAL (n_tensors < 0, D outside [1, Z3_D_MAX], A < 1, a spec
 * with numel < 0, ndim outside [0,4] or a shape product != numel, out NULL),
 * Z3_EOVERFLOW (N_pad beyond 2^62), Z3_ENOMEM. */
Z3_API int zero3_plan(const z3_tensor_spec* t, int32_t n_tensors, int32_t D, int32_t align_elems,
                      z3_plan** out);
Z3_API void zero3_plan_free(z3_plan* p);

/* Sizes of a plan; any output pointer may be NULL.  N = real elements,
 * N_pad = padded elements, S = elements per rank. */
Z3_API int zero3_plan_info(const z3_plan* p, int32_t* D, int32_t* n_tensors, int32_t* align_elems,
                           int64_t* N, int64_t* N_pad, int64_t* S);

/* Tensor i's run in the flat block: elements [*offset, *offset + *numel).
 * This is the unflatten of [P2] §5.1 ("full_params" used as the block's
 * tensors): a view of tensor i is the flat block at that offset, reshaped to
 * its row-major shape.  Errors: Z3_EINVAL (p NULL or i out of range). */
Z3_API int zero3_plan_tensor(const z3_plan* p, int32_t i, int64_t* offset, int64_t* numel);

/* Rank r's partition: *begin = r*S; *end_real = min((r+1)*S, N), never below
 * *begin.  Elements [*end_real, *begin + S) are tail padding.
 * Errors: Z3_EINVAL (p NULL or r outside [0, D)). */
Z3_API int zero3_plan_rank(const z3_plan* p, int32_t r, int64_t* begin, int64_t* end_real);

/* ---------------------------------------------------------- memory ledger
 * Bytes per device for N parameters over D ranks ([P2] §2, per-stage
 * formulas): 2 B of bf16 weights, about 6 B of gradient (bf16 with an fp32
 * accumulator) and 12 B of fp32 master + m + v per parameter;
 *   stage 0 (pure DP)  20 N
 *   stage 1 (ZeRO-1)   12 N / D + 2 N + 6 N
 *   stage 2 (ZeRO-2)   (12 + 6) N / D + 2 N
 *   stage 3 (ZeRO-3)   20 N / D
 * Each term that divides by D is rounded up to a whole byte.
 * Errors: Z3_EINVAL (N < 0, D < 1, unknown stage, bytes NULL), Z3_EOVERFLOW. */
Z3_API int zero3_memory_bytes(int64_t N, int32_t D, int32_t stage, int64_t* bytes);

/* Transient bytes for gathered blocks ([P2] §5.2): one gathered block of
 * block_params bf16 values takes 2 * block_params bytes, and n_buffers of
 * them are live at once (two when the next block's gather overlaps).
 * Errors: Z3_EINVAL (negative argument, bytes NULL), Z3_EOVERFLOW. */
Z3_API int zero3_transient_bytes(int64_t block_params, int32_t n_buffers, int64_t* bytes);

/* All-gather volume ([P2] §5.3): each pass (forward, and again backward)
 * gathers every block once; a device already holds its own 1/D of a block
 * and receives the other (D-1)/D.  *bytes = the bf16 bytes one device
 * receives for n_blocks blocks of block_params parameters each,
 * ceil(n_blocks * 2 * block_params * (D-1) / D).  D = 1 gives 0.
 * Errors: Z3_EINVAL (negative argument, D < 1, bytes NULL), Z3_EOVERFLOW. */
Z3_API int zero3_allgather_bytes(int64_t block_params, int32_t n_blocks, int32_t D, int64_t* bytes);

/* ------------------------------------------- reduce-scatter + AdamW + cast
 * zero3_reduce_adamw: one fused pass over the owned partition(s):
 *   1. reduce-scatter's reduction ([P3] "AllGather vs AllReduce": rank r
 *      receives the sum of the r-th slice of every rank's gradient; [P2] §4):
 *      g = (c_0 + c_1 + ... + c_{D-1}) * (1/D), summed left to right in rank
 *      order in the reduce dtype (Z3_REDUCE_FP32 or Z3_REDUCE_BF16), the 1/D
 *      factor being the fp32 constant nearest 1/D;
 *   2. AdamW on the owned fp32 master / m / v ([P2] §3: rank r updates only
 *      P_r from its local fp32 master, m, v and its gradient slice), in place:
 *        p = p*(1 - lr*wd);  m = b1*m + (1-b1)*g;  v = b2*v + (1-b2)*g*g;
 *        p = p - (lr/(1-b1^t)) * m / (sqrt(v)/sqrt(1-b2^t) + eps)
 *      with each scalar factor formed in double and rounded to fp32 once and
 *      each array operation one fp32 operation rounded to nearest-even;
 *   3. the cast of the new master to the bf16 working shard ([P3] "Mixed
 *      Precision"; [P1] §2 param_dtype=bfloat16), round-to-nearest-even.
 *
 *   p      plan of the block.
 *   rank   r in [0, D) runs rank r's partition; -1 runs every rank in one
 *          launch (state arrays then hold all D partitions back to back).
 *   contrib host array of D device pointers, the ranks' bf16 gradient
 *          contributions in `contrib_layout` (Z3_CONTRIB_OWNED needs rank >= 0).
 *          A pointer may address any memory this device can read with plain
 *          loads: its own, or another GPU's mapped through peer access or
 *          CUDA IPC (the kernel's loads then are the reduce-scatter's data
 *          movement, [P2] §4), read only, never with TMA.
 *   master, exp_avg, exp_avg_sq  fp32, S elements (N_pad if rank = -1), read
 *          and updated in place.  In device memory, or in page-locked host
 *          memory mapped into the device's address space (the CPU-offload
 *          placement of [P2] §8: the optimiser state leaves the GPU, which
 *          then reads and writes it over PCIe; the arithmetic is unchanged).
 *   work_bf16 bf16 output, same extent as master; device or mapped host memory.
 *   reduce_dtype  Z3_REDUCE_FP32 or Z3_REDUCE_BF16.
 *   hp     host struct; hp->step >= 1, all values finite, betas in [0, 1),
 *          eps > 0 (a zero eps turns the zero pad into 0/0), lr >= 0 and
 *          weight_decay >= 0.
 *   cuda_stream  stream to enqueue on.
 * Pad elements are processed like real ones: a zero master with zero
 * contributions stays exactly zero.
 * Alignment: every pointer must be aligned to its element size (Z3_EALIGN
 * otherwise).  When every contribution (at its partition offset), master,
 * m, v and work_bf16 is 16-byte aligned the kernel moves 16-byte vectors;
 * otherwise it falls back to a scalar kernel with the same results.
 * Errors: Z3_EINVAL, Z3_EALIGN, Z3_ECUDA (launch failed). */
Z3_API int zero3_reduce_adamw(const z3_plan* p, int32_t rank, const uint16_t* const* contrib,
                              int32_t contrib_layout, float* master, float* exp_avg,
                              float* exp_avg_sq, uint16_t* work_bf16, int32_t reduce_dtype,
                              const z3_adamw* hp, void* cuda_stream);

/* ------------------------ reduce-scatter + AdamW + cast + all-gather, fused
 * zero3_reduce_adamw_gather: zero3_reduce_adamw whose kernel also stores each
 * new bf16 working weight straight into its place in n_gathered whole padded
 * blocks: the value of rank r's owned element j goes to gathered[k][r*S + j]
 * for every k.  This is the all-gather's data movement ([P3] "AllGather vs
 * AllReduce": afterwards every GPU holds [A, B, C, D]; [P2] §3: rank r sends
 * its updated P_r slice to all other ranks) done by the kernel that produces
 * the data, so no separate pass reads the shards back.  It is the per-rank
 * step of ZeRO-1 and ZeRO-2, which keep the bf16 working weights replicated
 * and all-gather them at the end of every step ([P2] §3, §4); ZeRO-3 instead
 * gathers each block just before it runs (zero3_gather_block, [P2] §5.1).
 *   gathered    host array of n_gathered (1..Z3_GATHER_MAX) device pointers,
 *               each a bf16 block of N_pad elements.  Only the positions of
 *               the partitions this call updates are written (all of them for
 *               rank = -1, [r*S, (r+1)*S) for rank r).  A pointer may address
 *               any memory this device can store to with plain stores (its
 *               own, or another GPU's mapped through peer access).
 *   work_bf16   as in zero3_reduce_adamw, or NULL to write the gathered blocks
 *               only.
 * Every other argument, the arithmetic and the results are those of
 * zero3_reduce_adamw; the vector path also needs every gathered pointer at
 * its partition offset 16-byte aligned.
 * Errors: those of zero3_reduce_adamw, plus Z3_EINVAL for n_gathered outside
 * [1, Z3_GATHER_MAX], a NULL gathered pointer, or a gathered block that
 * overlaps another output or a contribution. */
Z3_API int zero3_reduce_adamw_gather(const z3_plan* p, int32_t rank, const uint16_t* const* contrib,
                                     int32_t contrib_layout, float* master, float* exp_avg,
                                     float* exp_avg_sq, uint16_t* work_bf16, uint16_t* const* gathered,
                                     int32_t n_gathered, int32_t reduce_dtype, const z3_adamw* hp,
                                     void* cuda_stream);

/* ------------------------------------- HYBRID_SHARD: reduce + AdamW + cast
 * zero3_reduce_adamw_hybrid: the per-rank step of HYBRID_SHARD ([P3]
 * "HYBRID_SHARD: The Multi-Node Strategy": n_nodes nodes of D GPUs; the block
 * is sharded D ways inside each node, as the plan describes, and replicated
 * across the nodes; the gradient crosses nodes in one all-reduce).  The
 * reduction has two levels:
 *   node k's sum   n_k = c_{k,0} + c_{k,1} + ... + c_{k,D-1}  (its reduce-scatter)
 *   total          (n_0 + n_1) + ... + n_{n_nodes-1}          (the cross-node all-reduce)
 *   g              total * (1/(n_nodes*D))
 * each sum left to right in the reduce dtype (every partial sum rounded to
 * fp32 or to bf16), the factor being the fp32 constant nearest 1/(n_nodes*D):
 * the average over every data-parallel rank, the same gradient as on one GPU
 * ([P3] "Key Takeaways").  Steps 2 and 3 are those of zero3_reduce_adamw.  The
 * all-reduce leaves the same sum on every node, so every node's replica of a
 * local rank computes exactly this update; one call stands for all of them.
 *   n_nodes  number of nodes, >= 1, with n_nodes * D <= Z3_D_MAX.  n_nodes = 1
 *            is zero3_reduce_adamw.
 *   contrib  host array of n_nodes * D device pointers: contrib[k*D + d] is the
 *            bf16 contribution of local rank d on node k (global rank k*D + d),
 *            each in `contrib_layout` as for zero3_reduce_adamw.
 * Every other argument, the alignment rules and the state placement are those
 * of zero3_reduce_adamw.
 * Errors: those of zero3_reduce_adamw, plus Z3_EINVAL for n_nodes < 1 or
 * n_nodes * D > Z3_D_MAX. */
Z3_API int zero3_reduce_adamw_hybrid(const z3_plan* p, int32_t rank, int32_t n_nodes,
                                     const uint16_t* const* contrib, int32_t contrib_layout, float* master,
                                     float* exp_avg, float* exp_avg_sq, uint16_t* work_bf16,
                                     int32_t reduce_dtype, const z3_adamw* hp, void* cuda_stream);

/* ------------------------------------ HYBRID_SHARD across nodes, in two parts
 * When the R nodes are separate machines, each node's sum has to exist in
 * memory so that it can cross the network once per step ([P3] "HYBRID_SHARD:
 * The Multi-Node Strategy").  The two calls below split the two-level
 * reduction of zero3_reduce_adamw_hybrid at that point; composed (node sums of
 * nodes 0..R-1, in node order), they give its results exactly.
 *
 * zero3_node_sum: a node's sum for rank `rank`'s partition (S elements), or for
 * every partition in one launch (rank = -1: N_pad elements): the node's D
 * contributions (the plan's D) folded left to right in rank order, not scaled.
 *   contrib, contrib_layout  as for zero3_reduce_adamw (D device pointers).
 *   reduce_dtype  Z3_REDUCE_FP32: every partial sum rounded to fp32, node_sum is
 *                 float; Z3_REDUCE_BF16: every partial sum rounded to bf16,
 *                 node_sum holds bf16 (uint16_t), half the bytes to send.
 *   node_sum      device output, S (or N_pad) elements of that type.
 * The vector path needs node_sum and every contribution (at its partition
 * offset) 16-byte aligned; otherwise a scalar kernel gives the same results.
 * Errors: Z3_EINVAL (NULL pointer, rank, layout or dtype out of range, output
 * over a contribution), Z3_EALIGN (a pointer off its element size), Z3_ECUDA.
 *
 * zero3_fold_adamw: for rank `rank`'s partition (or every partition, rank = -1),
 * the n_nodes node sums folded in node order 0..n_nodes-1 (partial sums in the
 * reduce dtype), times the fp32 constant nearest 1/(n_nodes * D), then AdamW on
 * master / exp_avg / exp_avg_sq and the bf16 cast to work_bf16, exactly as in
 * zero3_reduce_adamw.
 *   node_sums  host array of n_nodes (1..Z3_D_MAX) device pointers, node k's sum
 *              as zero3_node_sum wrote it (float or bf16 by reduce_dtype), each
 *              S (or N_pad) elements.
 *   master, exp_avg, exp_avg_sq, work_bf16, hp  as for zero3_reduce_adamw.
 * Errors: Z3_EINVAL (NULL pointer, bad rank, n_nodes or dtype, invalid hp,
 * overlapping outputs, an output over a node sum), Z3_EALIGN, Z3_ECUDA. */
Z3_API int zero3_node_sum(const z3_plan* p, int32_t rank, const uint16_t* const* contrib, int32_t contrib_layout,
                          int32_t reduce_dtype, void* node_sum, void* cuda_stream);
Z3_API int zero3_fold_adamw(const z3_plan* p, int32_t rank, int32_t n_nodes, const void* const* node_sums,
                            float* master, float* exp_avg, float* exp_avg_sq, uint16_t* work_bf16,
                            int32_t reduce_dtype, const z3_adamw* hp, void* cuda_stream);

/* ------------------------------------ CPU offload: optimiser on the host
 * The CPU-offload variant of [P2] §8: the Adam state (fp32 master, m, v)
 * lives in host memory; every step the GPU reduces the owned gradient shard,
 * the shard goes down over PCIe, AdamW runs on the host, and the bf16 weights
 * go back up (4 or 2 bytes per parameter down, 2 up, instead of moving the
 * 12 bytes of state each way).  These two calls are the GPU and host halves;
 * composed (zero3_reduce_scatter, then zero3_host_adamw on its output) they
 * give exactly the results of zero3_reduce_adamw.
 *
 * zero3_reduce_scatter: the reduce-scatter's reduction alone ([P3] "AllGather
 * vs AllReduce": rank r receives the sum of the r-th slice of every rank's
 * gradient; [P2] §4) for rank `rank`'s partition (S elements) or every
 * partition (rank = -1, N_pad elements): the averaged gradient
 *   g = (c_0 + c_1 + ... + c_{D-1}) * (1/D)
 * folded left to right in rank order in the reduce dtype, the factor the
 * fp32 constant nearest 1/D -- the g zero3_reduce_adamw hands to AdamW.
 *   contrib, contrib_layout  as for zero3_reduce_adamw (D device pointers).
 *   reduce_dtype  Z3_REDUCE_FP32: grad is float; Z3_REDUCE_BF16: every partial
 *                 sum rounded to bf16 and g rounded to bf16, grad holds bf16
 *                 (uint16_t) bits.
 *   grad          device output (or mapped page-locked host memory), S (or
 *                 N_pad) elements of that type.
 * The vector path needs grad and every contribution (at its partition offset)
 * 16-byte aligned; otherwise a scalar kernel gives the same results.
 * Errors: Z3_EINVAL (NULL pointer, rank, layout or dtype out of range, grad
 * over a contribution), Z3_EALIGN (a pointer off its element size), Z3_ECUDA.
 *
 * zero3_host_adamw: AdamW and the bf16 cast of n elements in HOST memory, on
 * host threads, with the same operations in the same order as the GPU kernels
 * (each one IEEE binary32 operation rounded to nearest-even, no fused
 * multiply-add), so the results are bit-identical to zero3_reduce_adamw's:
 *   p = p*(1 - lr*wd); m = b1*m + (1-b1)*g; v = b2*v + (1-b2)*g*g;
 *   p = p - (lr/(1-b1^t)) * m / (sqrt(v)/sqrt(1-b2^t) + eps);  w = bf16(p)
 *   grad        host array of n gradients: float (grad_dtype Z3_REDUCE_FP32)
 *               or bf16 bits (Z3_REDUCE_BF16), e.g. zero3_reduce_scatter's
 *               output copied down.
 *   master, exp_avg, exp_avg_sq  host fp32 arrays of n elements, in place.
 *   work_bf16   host bf16 output, n elements (to be copied up).
 *   hp          as for zero3_reduce_adamw.
 *   n_threads   host threads to use (0: all the hardware threads).  The
 *               threads are kept in a pool for later calls; concurrent calls
 *               run one after the other.
 * Synchronous: returns when every element is updated.  Nothing touches the GPU.
 * Errors: Z3_EINVAL (n < 0, n_threads < 0, NULL pointer with n > 0, bad
 * grad_dtype, invalid hp, overlapping arrays), Z3_EALIGN (a pointer off its
 * element size), Z3_EOVERFLOW (n beyond 2^60), Z3_ENOMEM (no thread could be
 * started). */
Z3_API int zero3_reduce_scatter(const z3_plan* p, int32_t rank, const uint16_t* const* contrib,
                                int32_t contrib_layout, int32_t reduce_dtype, void* grad, void* cuda_stream);
Z3_API int zero3_host_adamw(int64_t n, const void* grad, int32_t grad_dtype, float* master, float* exp_avg,
                            float* exp_avg_sq, uint16_t* work_bf16, const z3_adamw* hp, int32_t n_threads);

/* ------------------------------------- scalars in device memory (graphs)
 * zero3_step_scalars: the Z3_SCALARS fp32 scalars of one AdamW step, formed in
 * binary64 from *hp and rounded to fp32 once, exactly as zero3_reduce_adamw
 * forms them, in this order:
 *   [0] lr / (1 - beta1^t)    [1] 1 / sqrt(1 - beta2^t)   [2] 1 - lr * weight_decay
 *   [3] beta1   [4] 1 - beta1   [5] beta2   [6] 1 - beta2   [7] eps
 *   out: host array of Z3_SCALARS floats.
 * Errors: Z3_EINVAL (out or hp NULL, hp->step < 1, a value not finite, a beta
 * outside [0, 1), eps <= 0, lr < 0 or weight_decay < 0).
 *
 * zero3_reduce_adamw_dev: zero3_reduce_adamw (n_gathered = 0) or
 * zero3_reduce_adamw_gather (n_gathered >= 1, up to Z3_GATHER_MAX) whose kernel
 * reads the step's scalars from `scalars`, a device array of Z3_SCALARS floats
 * (16-byte aligned) laid out as above, instead of taking them as launch
 * arguments.  Nothing else in the launch depends on the step, so the launch can
 * be captured into a CUDA graph once and the graph replayed every step, with
 * only the scalars rewritten (stream-ordered) before each replay.  The
 * arithmetic and results are those of zero3_reduce_adamw.  work_bf16 may be
 * NULL only when n_gathered >= 1.
 * Errors: those of zero3_reduce_adamw_gather, Z3_EINVAL (scalars NULL, or
 * overlapping an output), Z3_EALIGN (scalars not 16-byte aligned). */
Z3_API int zero3_step_scalars(const z3_adamw* hp, float* out);
Z3_API int zero3_reduce_adamw_dev(const z3_plan* p, int32_t rank, const uint16_t* const* contrib,
                                  int32_t contrib_layout, float* master, float* exp_avg, float* exp_avg_sq,
                                  uint16_t* work_bf16, uint16_t* const* gathered, int32_t n_gathered,
                                  int32_t reduce_dtype, const float* scalars, void* cuda_stream);

/* ------------------------------------------------ all-gather + unflatten
 * zero3_gather_block: the all-gather's data movement ([P3] "AllGather vs
 * AllReduce": GPU r holds shard r; afterwards every GPU holds [A, B, C, D];
 * [P2] §5.1: full_params = all_gather(local_shard) before the block runs) and
 * the optional unflatten into separate per-tensor buffers.
 *   shards     host array of D device pointers, shard r = rank r's S bf16
 *              working weights.  A pointer may address another GPU's memory
 *              mapped through peer access or CUDA IPC (plain loads; the
 *              all-gather done by the receiving GPU's kernel).
 *   flat_out   device bf16, N_pad elements: flat_out[r*S + j] = shards[r][j].
 *              May be NULL when tensor_out is given.  A shard may already
 *              sit in place inside it, shards[r] == flat_out + r*S (a rank's
 *              own shard kept as a view of its gathered block, as FSDP lays
 *              it out); that partition is left as it is and not copied.
 *   tensor_out host array of n_tensors device pointers, or NULL: tensor i's
 *              buffer receives its numel elements (flat elements
 *              [offset_i, offset_i + numel_i)), read straight from the shards.
 *              An entry may be NULL to skip that tensor.
 * Zero-copy views need no call: zero3_plan_tensor gives each tensor's offset
 * in flat_out.  The vector path needs S % 8 == 0 and 16-byte aligned
 * pointers; otherwise a scalar kernel gives the same bytes.
 * Errors: Z3_EINVAL (both outputs NULL, a NULL shard, an output overlapping a
 * shard other than in the in-place position above, outputs overlapping each
 * other), Z3_EALIGN, Z3_ENOMEM (the host list of per-tensor segments could not
 * be allocated), Z3_ECUDA. */
Z3_API int zero3_gather_block(const z3_plan* p, const uint16_t* const* shards, uint16_t* flat_out,
                              uint16_t* const* tensor_out, void* cuda_stream);

/* ------------------------------------ another process's memory, through CUDA IPC
 * The D-GPU form of the step ([P2] §4, §5.1): the fused kernel on rank r reads
 * slice P_r of every rank's gradient, and the gather kernel every rank's shard,
 * from the other GPUs' memory with plain loads.  Each rank exports the device
 * allocation that holds a buffer; every other rank imports it, which maps it
 * into the address space of the importing thread's CURRENT device (the device
 * its kernels launch on) with peer access to the owning GPU enabled as needed
 * (cudaIpcMemLazyEnablePeerAccess).
 *
 * zero3_ipc_export: for a pointer into device memory from cudaMalloc (e.g.
 * PyTorch's caching allocator), the IPC handle of the allocation holding it
 * (Z3_IPC_HANDLE_BYTES bytes written to handle_out), the pointer's byte offset
 * in the allocation and the allocation's size in bytes.
 * Errors: Z3_EINVAL (a NULL argument, ptr not inside a device allocation),
 * Z3_ECUDA (the runtime cannot export the allocation, e.g. virtual-memory
 * mapped memory).
 *
 * zero3_ipc_import: maps the allocation of another process's handle and sets
 * *ptr_out = mapping + offset and *base_out = the mapping (for zero3_ipc_close).
 * The caller checks offset against the exporter's size.  Importing a handle
 * this process holds already returns the same mapping and counts the import.
 * A handle exported by this same process cannot be imported.
 * Errors: Z3_EINVAL (a NULL argument, offset < 0), Z3_ECUDA (the runtime
 * refused the mapping), Z3_ENOMEM (host bookkeeping).
 *
 * zero3_ipc_close: releases one import of the mapping at base; the last
 * release unmaps it.  Nothing the device still has in flight may use it.
 * Errors: Z3_EINVAL (NULL, or not a mapping from zero3_ipc_import), Z3_ECUDA. */
#define Z3_IPC_HANDLE_BYTES 64
Z3_API int zero3_ipc_export(const void* ptr, void* handle_out, int64_t* offset_out, int64_t* size_out);
Z3_API int zero3_ipc_import(const void* handle, int64_t offset, void** ptr_out, void** base_out);
Z3_API int zero3_ipc_close(void* base);

#ifdef __cplusplus
}
#endif

#endif /* ZERO3_H */
