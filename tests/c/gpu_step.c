/*
 * gpu_step.c -- a plain C99 program that runs ZeRO-3 steps through the C ABI
 * on the GPU and checks them, bit for bit, against the oracle's C library.
 *
 * Built and run by tests/test_c_consumers.py (the GPU test).  The product side
 * is include/zero3.h + libzero3.so only; device memory comes from the CUDA
 * runtime API.  The oracle (oracle/zero3_ref.c, test infrastructure) is linked
 * as a second library; its prototypes are declared below.
 *
 * What runs, for each reduce dtype:
 *   - 3 steps of zero3_reduce_adamw over every rank's partition of a 3-tensor
 *     block at D = 4 (ragged tensor sizes, tail padding), then
 *     zero3_gather_block into the flat block and into one buffer per tensor
 *     ("7.10 — Fully-sharded data parallel (FSDP / ZeRO-3)", §3 and §5.1);
 *   - 3 steps of zero3_reduce_adamw_hybrid with 3 nodes of 4 ranks
 *     ("Building GPT from Scratch — Part 8", "HYBRID_SHARD: The Multi-Node
 *     Strategy");
 *   - 3 steps of the CPU-offload step ("7.10", §8): zero3_reduce_scatter of
 *     every rank's partition on the GPU, the gradient copied down, and
 *     zero3_host_adamw on host memory.
 * Inputs are drawn from splitmix64 (Steele, Lea and Flood, "Fast splittable
 * pseudorandom number generators", 2014), keyed by (step, contributor,
 * element), and fed identically to both sides.  Exit status 0 means every
 * result matched.
 */
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <cuda_runtime_api.h>

#include "zero3.h"

/* ---- the oracle's entry points (oracle/zero3_ref.c) */
typedef struct {
    double lr, beta1, beta2, eps, weight_decay;
    int64_t step;
} oracle_hp;
int ref_reduce_adamw(int32_t D, int64_t S, int32_t rank, const uint16_t* const* contrib, int32_t layout,
                     float* master, float* exp_avg, float* exp_avg_sq, uint16_t* work_bf16,
                     int32_t reduce_dtype, const oracle_hp* hp);
int ref_reduce_adamw_hybrid(int32_t R, int32_t D, int64_t S, int32_t rank, const uint16_t* const* contrib,
                            int32_t layout, float* master, float* exp_avg, float* exp_avg_sq,
                            uint16_t* work_bf16, int32_t reduce_dtype, const oracle_hp* hp);
int ref_reduce_scatter(int32_t D, int64_t S, int32_t rank, const uint16_t* const* contrib, int32_t layout,
                       int32_t reduce_dtype, float* out);
void ref_all_gather(int32_t D, int64_t S, const uint16_t* const* shards, uint16_t* flat);
void ref_unflatten(const uint16_t* flat, int32_t n_tensors, const int64_t* offset, const int64_t* numel,
                   uint16_t* const* out);

#define D 4
#define NODES 3
#define NT 3
#define MAXC (NODES * D)

static int failures = 0;

#define CHECK(cond)                                                                   \
    do {                                                                              \
        if (!(cond)) {                                                                \
            fprintf(stderr, "%s:%d: check failed: %s\n", __FILE__, __LINE__, #cond); \
            ++failures;                                                               \
        }                                                                             \
    } while (0)

#define CUDA(call)                                                                               \
    do {                                                                                         \
        cudaError_t e_ = (call);                                                                 \
        if (e_ != cudaSuccess) {                                                                 \
            fprintf(stderr, "%s:%d: %s: %s\n", __FILE__, __LINE__, #call, cudaGetErrorString(e_)); \
            exit(2);                                                                             \
        }                                                                                        \
    } while (0)

static uint64_t splitmix64(uint64_t x)
{
    uint64_t z = x + 0x9E3779B97F4A7C15ULL;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}

/* uniform in [0, 1) from the draw keyed (a, b, i) */
static double uniform(uint64_t a, uint64_t b, uint64_t i)
{
    uint64_t h = splitmix64(splitmix64(splitmix64(a) ^ b) ^ i);
    return (double)(h >> 11) * (1.0 / 9007199254740992.0);
}

/* an input gradient value as a bf16 bit pattern: the upper half of a float draw */
static uint16_t grad_bits(uint64_t step, uint64_t who, uint64_t i)
{
    float x = (float)((uniform(step, who, i) - 0.5) * 2e-3);
    uint32_t u;
    memcpy(&u, &x, sizeof u);
    return (uint16_t)(u >> 16);
}

static z3_tensor_spec spec(int64_t a, int64_t b)
{
    z3_tensor_spec t;
    memset(&t, 0, sizeof t);
    t.numel = a * b;
    t.ndim = b > 1 ? 2 : 1;
    t.shape[0] = a;
    t.shape[1] = b;
    return t;
}

static void* dalloc(size_t bytes)
{
    void* p = NULL;
    CUDA(cudaMalloc(&p, bytes));
    return p;
}

static void run(int32_t mode, int32_t nodes)
{
    const z3_tensor_spec t[NT] = {spec(1000, 1), spec(257, 33), spec(4097, 1)};
    z3_plan* plan = NULL;
    CHECK(zero3_plan(t, NT, D, 8, &plan) == Z3_OK);
    int64_t N = 0, N_pad = 0, S = 0;
    zero3_plan_info(plan, NULL, NULL, NULL, &N, &N_pad, &S);
    const int nc = nodes * D;

    /* host state: the oracle's copy and the staging for the device */
    float* hp_ = calloc((size_t)N_pad, 4);
    float* hm = calloc((size_t)N_pad, 4);
    float* hv = calloc((size_t)N_pad, 4);
    uint16_t* hw = calloc((size_t)N_pad, 2);
    float* back = calloc((size_t)N_pad, 4);
    uint16_t* back16 = calloc((size_t)N_pad, 2);
    uint16_t* hc[MAXC];
    for (int64_t i = 0; i < N; ++i) hp_[i] = (float)((uniform(0, 999, (uint64_t)i) - 0.5) * 0.08);

    float* dp = dalloc((size_t)N_pad * 4);
    float* dm = dalloc((size_t)N_pad * 4);
    float* dv = dalloc((size_t)N_pad * 4);
    uint16_t* dw = dalloc((size_t)N_pad * 2);
    const uint16_t* dc[MAXC];
    CUDA(cudaMemcpy(dp, hp_, (size_t)N_pad * 4, cudaMemcpyHostToDevice));
    CUDA(cudaMemset(dm, 0, (size_t)N_pad * 4));
    CUDA(cudaMemset(dv, 0, (size_t)N_pad * 4));
    for (int c = 0; c < nc; ++c) {
        hc[c] = calloc((size_t)N_pad, 2);
        dc[c] = dalloc((size_t)N_pad * 2);
    }

    for (int64_t step = 1; step <= 3; ++step) {
        for (int c = 0; c < nc; ++c) {
            for (int64_t i = 0; i < N; ++i) hc[c][i] = grad_bits((uint64_t)step, (uint64_t)c, (uint64_t)i);
            CUDA(cudaMemcpy((void*)dc[c], hc[c], (size_t)N_pad * 2, cudaMemcpyHostToDevice));
        }
        const z3_adamw hp = {3e-4, 0.9, 0.95, 1e-8, 0.1, step};
        const oracle_hp ohp = {3e-4, 0.9, 0.95, 1e-8, 0.1, step};
        int rc;
        if (nodes > 1) {
            rc = zero3_reduce_adamw_hybrid(plan, -1, nodes, dc, Z3_CONTRIB_FULL, dp, dm, dv, dw, mode, &hp, NULL);
            CHECK(ref_reduce_adamw_hybrid(nodes, D, S, -1, (const uint16_t* const*)hc, 0, hp_, hm, hv, hw, mode,
                                          &ohp) == 0);
        } else {
            rc = zero3_reduce_adamw(plan, -1, dc, Z3_CONTRIB_FULL, dp, dm, dv, dw, mode, &hp, NULL);
            CHECK(ref_reduce_adamw(D, S, -1, (const uint16_t* const*)hc, 0, hp_, hm, hv, hw, mode, &ohp) == 0);
        }
        CHECK(rc == Z3_OK);
        CUDA(cudaDeviceSynchronize());
        CUDA(cudaMemcpy(back, dp, (size_t)N_pad * 4, cudaMemcpyDeviceToHost));
        CHECK(memcmp(back, hp_, (size_t)N_pad * 4) == 0);
        CUDA(cudaMemcpy(back, dm, (size_t)N_pad * 4, cudaMemcpyDeviceToHost));
        CHECK(memcmp(back, hm, (size_t)N_pad * 4) == 0);
        CUDA(cudaMemcpy(back, dv, (size_t)N_pad * 4, cudaMemcpyDeviceToHost));
        CHECK(memcmp(back, hv, (size_t)N_pad * 4) == 0);
        CUDA(cudaMemcpy(back16, dw, (size_t)N_pad * 2, cudaMemcpyDeviceToHost));
        CHECK(memcmp(back16, hw, (size_t)N_pad * 2) == 0);
    }

    if (nodes == 1) {
        /* all-gather of the D shards into the flat block and into one buffer per tensor */
        const uint16_t* shards[D];
        const uint16_t* hshards[D];
        for (int r = 0; r < D; ++r) {
            shards[r] = dw + r * S;
            hshards[r] = hw + r * S;
        }
        uint16_t* dflat = dalloc((size_t)N_pad * 2);
        uint16_t* dt[NT];
        uint16_t* ht[NT];
        int64_t off[NT], num[NT];
        for (int i = 0; i < NT; ++i) {
            zero3_plan_tensor(plan, i, &off[i], &num[i]);
            dt[i] = dalloc((size_t)num[i] * 2);
            ht[i] = calloc((size_t)num[i], 2);
        }
        CHECK(zero3_gather_block(plan, shards, dflat, dt, NULL) == Z3_OK);
        uint16_t* hflat = calloc((size_t)N_pad, 2);
        ref_all_gather(D, S, hshards, hflat);
        ref_unflatten(hflat, NT, off, num, ht);
        CUDA(cudaDeviceSynchronize());
        CUDA(cudaMemcpy(back16, dflat, (size_t)N_pad * 2, cudaMemcpyDeviceToHost));
        CHECK(memcmp(back16, hflat, (size_t)N_pad * 2) == 0);
        for (int i = 0; i < NT; ++i) {
            CUDA(cudaMemcpy(back16, dt[i], (size_t)num[i] * 2, cudaMemcpyDeviceToHost));
            CHECK(memcmp(back16, ht[i], (size_t)num[i] * 2) == 0);
            CUDA(cudaFree(dt[i]));
            free(ht[i]);
        }
        CUDA(cudaFree(dflat));
        free(hflat);
    }

    for (int c = 0; c < nc; ++c) {
        CUDA(cudaFree((void*)dc[c]));
        free(hc[c]);
    }
    CUDA(cudaFree(dp));
    CUDA(cudaFree(dm));
    CUDA(cudaFree(dv));
    CUDA(cudaFree(dw));
    free(hp_);
    free(hm);
    free(hv);
    free(hw);
    free(back);
    free(back16);
    zero3_plan_free(plan);
    printf("mode %d, %d node(s) of %d ranks, N=%lld N_pad=%lld: %s\n", (int)mode, (int)nodes, D, (long long)N,
           (long long)N_pad, failures ? "MISMATCH" : "bit-identical to the oracle");
}

/* The CPU-offload step: per rank partition, the averaged gradient on the GPU
 * (compared with the oracle's reduce-scatter), copied down, then AdamW and
 * the cast on the host; the host state is compared with the oracle's step. */
static void run_offload(int32_t mode)
{
    const z3_tensor_spec t[NT] = {spec(1000, 1), spec(257, 33), spec(4097, 1)};
    z3_plan* plan = NULL;
    CHECK(zero3_plan(t, NT, D, 8, &plan) == Z3_OK);
    int64_t N = 0, N_pad = 0, S = 0;
    zero3_plan_info(plan, NULL, NULL, NULL, &N, &N_pad, &S);
    const size_t gsz = mode == Z3_REDUCE_FP32 ? 4 : 2;

    float* hp_ = calloc((size_t)N_pad, 4); /* the oracle's state */
    float* hm = calloc((size_t)N_pad, 4);
    float* hv = calloc((size_t)N_pad, 4);
    uint16_t* hw = calloc((size_t)N_pad, 2);
    float* op = calloc((size_t)N_pad, 4); /* the offloaded state, on the host */
    float* om = calloc((size_t)N_pad, 4);
    float* ov = calloc((size_t)N_pad, 4);
    uint16_t* ow = calloc((size_t)N_pad, 2);
    void* hg = calloc((size_t)S, gsz);
    float* ref_g = calloc((size_t)S, 4);
    uint16_t* hc[D];
    const uint16_t* dc[D];
    for (int64_t i = 0; i < N; ++i) hp_[i] = op[i] = (float)((uniform(0, 998, (uint64_t)i) - 0.5) * 0.08);
    for (int c = 0; c < D; ++c) {
        hc[c] = calloc((size_t)N_pad, 2);
        dc[c] = dalloc((size_t)N_pad * 2);
    }
    void* dg = dalloc((size_t)S * gsz);

    for (int64_t step = 1; step <= 3; ++step) {
        for (int c = 0; c < D; ++c) {
            for (int64_t i = 0; i < N; ++i) hc[c][i] = grad_bits((uint64_t)step + 10, (uint64_t)c, (uint64_t)i);
            CUDA(cudaMemcpy((void*)dc[c], hc[c], (size_t)N_pad * 2, cudaMemcpyHostToDevice));
        }
        const z3_adamw hp = {3e-4, 0.9, 0.95, 1e-8, 0.1, step};
        const oracle_hp ohp = {3e-4, 0.9, 0.95, 1e-8, 0.1, step};
        for (int32_t r = 0; r < D; ++r) {
            CHECK(zero3_reduce_scatter(plan, r, dc, Z3_CONTRIB_FULL, mode, dg, NULL) == Z3_OK);
            CUDA(cudaMemcpy(hg, dg, (size_t)S * gsz, cudaMemcpyDeviceToHost));
            CHECK(ref_reduce_scatter(D, S, r, (const uint16_t* const*)hc, 0, mode, ref_g) == 0);
            for (int64_t j = 0; j < S; ++j) {
                float g;
                if (mode == Z3_REDUCE_FP32) {
                    g = ((const float*)hg)[j];
                } else {
                    const uint32_t u = (uint32_t)((const uint16_t*)hg)[j] << 16;
                    memcpy(&g, &u, sizeof g);
                }
                if (memcmp(&g, &ref_g[j], 4) != 0) {
                    CHECK(!"reduce-scatter output differs from the oracle");
                    break;
                }
            }
            CHECK(zero3_host_adamw(S, hg, mode, op + r * S, om + r * S, ov + r * S, ow + r * S, &hp, 3) == Z3_OK);
        }
        CHECK(ref_reduce_adamw(D, S, -1, (const uint16_t* const*)hc, 0, hp_, hm, hv, hw, mode, &ohp) == 0);
        CHECK(memcmp(op, hp_, (size_t)N_pad * 4) == 0);
        CHECK(memcmp(om, hm, (size_t)N_pad * 4) == 0);
        CHECK(memcmp(ov, hv, (size_t)N_pad * 4) == 0);
        CHECK(memcmp(ow, hw, (size_t)N_pad * 2) == 0);
    }
    for (int c = 0; c < D; ++c) {
        CUDA(cudaFree((void*)dc[c]));
        free(hc[c]);
    }
    CUDA(cudaFree(dg));
    free(hp_);
    free(hm);
    free(hv);
    free(hw);
    free(op);
    free(om);
    free(ov);
    free(ow);
    free(hg);
    free(ref_g);
    zero3_plan_free(plan);
    printf("mode %d, CPU offload (GPU reduce-scatter, host AdamW), N=%lld N_pad=%lld: %s\n", (int)mode,
           (long long)N, (long long)N_pad, failures ? "MISMATCH" : "bit-identical to the oracle");
}

int main(void)
{
    int count = 0;
    if (cudaGetDeviceCount(&count) != cudaSuccess || count < 1) {
        fprintf(stderr, "no CUDA device\n");
        return 2;
    }
    for (int32_t mode = Z3_REDUCE_FP32; mode <= Z3_REDUCE_BF16; ++mode) {
        run(mode, 1);
        run(mode, NODES);
        run_offload(mode);
    }
    return failures ? 1 : 0;
}
