/*
 * host_abi.c -- a plain C99 consumer of the library's host-side entry points.
 *
 * Built and run by tests/test_c_consumers.py.  It includes only
 * include/zero3.h and links only libzero3.so, which checks that the header is
 * valid C99 (no C++ in the signatures) and that the host-side calls behave as
 * the header documents: the plan of the LLaMA-7B decoder block ("7.10 —
 * Fully-sharded data parallel (FSDP / ZeRO-3)", §3: rank r owns P_r), the tail
 * padding of the same block with a 4097-element bias at D = 32, the memory
 * ledger of §2 and the transient buffers of §5.2, the step scalars, and the
 * error codes.  Expected values are closed forms written out below.  No GPU
 * is touched.  Exit status 0 means every check passed.
 */
#include <math.h>
#include <stdio.h>
#include <string.h>

#include "zero3.h"

static int failures = 0;

#define CHECK(cond)                                                             \
    do {                                                                        \
        if (!(cond)) {                                                          \
            fprintf(stderr, "%s:%d: check failed: %s\n", __FILE__, __LINE__, #cond); \
            ++failures;                                                         \
        }                                                                       \
    } while (0)

static z3_tensor_spec spec2(int64_t a, int64_t b)
{
    z3_tensor_spec t;
    memset(&t, 0, sizeof t);
    t.numel = a * b;
    t.ndim = 2;
    t.shape[0] = a;
    t.shape[1] = b;
    return t;
}

static z3_tensor_spec spec1(int64_t a)
{
    z3_tensor_spec t;
    memset(&t, 0, sizeof t);
    t.numel = a;
    t.ndim = 1;
    t.shape[0] = a;
    return t;
}

/* q, k, v, o 4096 x 4096; gate, up 4096 x 11008; down 11008 x 4096; two RMSNorm 4096 */
static int llama7b_block(z3_tensor_spec* t)
{
    int n = 0;
    for (int i = 0; i < 4; ++i) t[n++] = spec2(4096, 4096);
    t[n++] = spec2(4096, 11008);
    t[n++] = spec2(4096, 11008);
    t[n++] = spec2(11008, 4096);
    t[n++] = spec1(4096);
    t[n++] = spec1(4096);
    return n;
}

static void check_plan_d8(void)
{
    z3_tensor_spec t[10];
    int n = llama7b_block(t);
    z3_plan* p = NULL;
    CHECK(zero3_plan(t, n, 8, 128, &p) == Z3_OK && p != NULL);
    if (p == NULL) return;
    int32_t D = 0, nt = 0, A = 0;
    int64_t N = 0, N_pad = 0, S = 0;
    CHECK(zero3_plan_info(p, &D, &nt, &A, &N, &N_pad, &S) == Z3_OK);
    const int64_t N_expect = 4LL * 4096 * 4096 + 3LL * 4096 * 11008 + 2LL * 4096;  /* 202,383,360 */
    CHECK(D == 8 && nt == 9 && A == 128);
    CHECK(N == N_expect && N_pad == N_expect && S == N_expect / 8);
    /* offsets: prefix sums in list order */
    int64_t off = 0, numel = 0, expect = 0;
    for (int i = 0; i < n; ++i) {
        CHECK(zero3_plan_tensor(p, i, &off, &numel) == Z3_OK);
        CHECK(off == expect && numel == t[i].numel);
        expect += t[i].numel;
    }
    int64_t b = 0, e = 0;
    for (int r = 0; r < 8; ++r) {
        CHECK(zero3_plan_rank(p, r, &b, &e) == Z3_OK);
        CHECK(b == r * S && e == (r + 1) * S);
    }
    CHECK(zero3_plan_tensor(p, 9, &off, &numel) == Z3_EINVAL);
    CHECK(zero3_plan_rank(p, 8, &b, &e) == Z3_EINVAL);
    zero3_plan_free(p);
}

static void check_plan_d32_padded(void)
{
    z3_tensor_spec t[10];
    int n = llama7b_block(t);
    t[n++] = spec1(4097);
    z3_plan* p = NULL;
    CHECK(zero3_plan(t, n, 32, 128, &p) == Z3_OK && p != NULL);
    if (p == NULL) return;
    int64_t N = 0, N_pad = 0, S = 0;
    CHECK(zero3_plan_info(p, NULL, NULL, NULL, &N, &N_pad, &S) == Z3_OK);
    /* N = 49,410 * 4096 + 4097 = 49,411 * 4096 + 1 = 202,387,457, padded to the next
     * multiple of 32 * 128 = 4096: 49,412 * 4096 = 202,391,552 */
    CHECK(N == 202387457LL && N_pad == 49412LL * 4096 && S == N_pad / 32);
    int64_t b = 0, e = 0;
    CHECK(zero3_plan_rank(p, 31, &b, &e) == Z3_OK);
    CHECK(b == 31 * S && e == N);                   /* the 4,095 pad elements sit in rank 31's shard */
    CHECK(N_pad - N == 4095);
    zero3_plan_free(p);
}

static void check_ledger(void)
{
    const int64_t N = 7000000000LL;                 /* 7B parameters */
    int64_t bytes = 0;
    CHECK(zero3_memory_bytes(N, 32, Z3_STAGE_ZERO3, &bytes) == Z3_OK && bytes == 20 * N / 32);
    CHECK(zero3_memory_bytes(N, 32, Z3_STAGE_DDP, &bytes) == Z3_OK && bytes == 20 * N);
    CHECK(zero3_memory_bytes(N, 32, Z3_STAGE_ZERO1, &bytes) == Z3_OK && bytes == 12 * N / 32 + 8 * N);
    CHECK(zero3_memory_bytes(N, 32, Z3_STAGE_ZERO2, &bytes) == Z3_OK && bytes == 18 * N / 32 + 2 * N);
    CHECK(zero3_memory_bytes(7, 2, Z3_STAGE_ZERO3, &bytes) == Z3_OK && bytes == 70);   /* 140 / 2 */
    CHECK(zero3_memory_bytes(7, 3, Z3_STAGE_ZERO3, &bytes) == Z3_OK && bytes == 47);   /* ceil(140 / 3) */
    CHECK(zero3_memory_bytes(N, 32, 4, &bytes) == Z3_EINVAL);
    CHECK(zero3_memory_bytes(-1, 32, 3, &bytes) == Z3_EINVAL);
    CHECK(zero3_memory_bytes(N, 32, 3, NULL) == Z3_EINVAL);
    /* all-gather volume: 32 blocks of 100M bf16 parameters (200 MB) at D = 32 receive 31/32 of each */
    CHECK(zero3_allgather_bytes(100000000LL, 32, 32, &bytes) == Z3_OK && bytes == 6200000000LL);
    CHECK(zero3_allgather_bytes(7, 1, 3, &bytes) == Z3_OK && bytes == 10);   /* ceil(14 * 2 / 3) */
    CHECK(zero3_allgather_bytes(7, 1, 1, &bytes) == Z3_OK && bytes == 0);
    CHECK(zero3_allgather_bytes(7, 1, 0, &bytes) == Z3_EINVAL);
    /* one 12 x 4096^2 block in bf16, two buffers live (next block's gather overlapping) */
    CHECK(zero3_transient_bytes(12LL * 4096 * 4096, 2, &bytes) == Z3_OK && bytes == 4LL * 12 * 4096 * 4096);
}

static void check_scalars(void)
{
    z3_adamw hp = {3e-4, 0.9, 0.95, 1e-8, 0.1, 1};
    float s[Z3_SCALARS];
    CHECK(zero3_step_scalars(&hp, s) == Z3_OK);
    /* step 1: lr / (1 - beta1), 1 / sqrt(1 - beta2), 1 - lr * wd, then the betas and eps */
    CHECK(s[0] == (float)(3e-4 / (1.0 - 0.9)));
    CHECK(s[1] == (float)(1.0 / sqrt(1.0 - 0.95)));
    CHECK(s[2] == (float)(1.0 - 3e-4 * 0.1));
    CHECK(s[3] == 0.9f && s[4] == (float)(1.0 - 0.9) && s[5] == 0.95f && s[6] == (float)(1.0 - 0.95));
    CHECK(s[7] == 1e-8f);
    hp.step = 0;
    CHECK(zero3_step_scalars(&hp, s) == Z3_EINVAL);
    hp.step = 1;
    hp.beta2 = 1.0;
    CHECK(zero3_step_scalars(&hp, s) == Z3_EINVAL);
}

/* The host optimiser of the CPU-offload step, from C: one step from m = v = 0
 * moves every weight by about lr against the sign of its gradient (the
 * update is lr * g / (|g| + eps * sqrt(1 - beta2)) once the bias corrections
 * cancel), a zero pad with a zero gradient stays exactly zero, the bf16
 * weights are the masters rounded to bf16, and the work is the same on 1 and
 * on 7 threads. */
static void check_host_adamw(void)
{
    enum { n = 5000, pad = 96 };
    static float g[n], p1[n], m1[n], v1[n], p7[n], m7[n], v7[n];
    static uint16_t w1[n], w7[n];
    for (int i = 0; i < n; ++i) {
        g[i] = i >= n - pad ? 0.0f : (i % 2 ? 1e-3f : -2e-3f) * (float)(1 + i % 7);
        p1[i] = p7[i] = i >= n - pad ? 0.0f : 0.01f * (float)((i % 11) - 5);
        m1[i] = m7[i] = v1[i] = v7[i] = 0.0f;
    }
    const z3_adamw hp = {3e-4, 0.9, 0.95, 1e-8, 0.0, 1};
    CHECK(zero3_host_adamw(n, g, Z3_REDUCE_FP32, p1, m1, v1, w1, &hp, 1) == Z3_OK);
    CHECK(zero3_host_adamw(n, g, Z3_REDUCE_FP32, p7, m7, v7, w7, &hp, 7) == Z3_OK);
    CHECK(memcmp(p1, p7, sizeof p1) == 0 && memcmp(m1, m7, sizeof m1) == 0 && memcmp(v1, v7, sizeof v1) == 0);
    CHECK(memcmp(w1, w7, sizeof w1) == 0);
    for (int i = 0; i < n; ++i) {
        const float p0 = i >= n - pad ? 0.0f : 0.01f * (float)((i % 11) - 5);
        if (i >= n - pad) {
            CHECK(p1[i] == 0.0f && m1[i] == 0.0f && v1[i] == 0.0f && w1[i] == 0);
            continue;
        }
        const double step = (double)p1[i] - (double)p0;
        CHECK(fabs(fabs(step) - 3e-4) < 3e-6);          /* |update| = lr, within eps's share */
        CHECK((step < 0) == (g[i] > 0));                 /* against the gradient */
        uint32_t u;
        memcpy(&u, &p1[i], sizeof u);
        const uint32_t lsb = (u >> 16) & 1u;
        CHECK(w1[i] == (uint16_t)((u + 0x7FFFu + lsb) >> 16));   /* nearest-even bf16 */
    }
    CHECK(zero3_host_adamw(-1, g, Z3_REDUCE_FP32, p1, m1, v1, w1, &hp, 1) == Z3_EINVAL);
    CHECK(zero3_host_adamw(n, g, 7, p1, m1, v1, w1, &hp, 1) == Z3_EINVAL);
    CHECK(zero3_host_adamw(n, g, Z3_REDUCE_FP32, p1, p1, v1, w1, &hp, 1) == Z3_EINVAL);   /* master = exp_avg */
    CHECK(zero3_host_adamw(0, NULL, Z3_REDUCE_FP32, NULL, NULL, NULL, NULL, &hp, 0) == Z3_OK);
}

static void check_errors(void)
{
    z3_tensor_spec t = spec2(3, 5);
    z3_plan* p = NULL;
    CHECK(zero3_plan(&t, 1, 0, 8, &p) == Z3_EINVAL);
    CHECK(zero3_plan(&t, 1, Z3_D_MAX + 1, 8, &p) == Z3_EINVAL);
    CHECK(zero3_plan(&t, 1, 4, 0, &p) == Z3_EINVAL);
    CHECK(zero3_plan(&t, 1, 4, 8, NULL) == Z3_EINVAL);
    t.shape[1] = 6;                                  /* shape product != numel */
    CHECK(zero3_plan(&t, 1, 4, 8, &p) == Z3_EINVAL);
    CHECK(zero3_plan(NULL, 0, 4, 8, &p) == Z3_OK && p != NULL);   /* an empty block */
    int64_t N = -1, N_pad = -1;
    CHECK(zero3_plan_info(p, NULL, NULL, NULL, &N, &N_pad, NULL) == Z3_OK && N == 0 && N_pad == 0);
    zero3_plan_free(p);
    zero3_plan_free(NULL);
    const int codes[] = {Z3_OK, Z3_EINVAL, Z3_EALIGN, Z3_ENOMEM, Z3_ECUDA, Z3_EOVERFLOW, 12345};
    for (unsigned i = 0; i < sizeof codes / sizeof codes[0]; ++i) {
        const char* text = zero3_status_string(codes[i]);
        CHECK(text != NULL && text[0] != '\0');
    }
    /* device entry points reject bad arguments before touching any device */
    CHECK(zero3_reduce_adamw(NULL, 0, NULL, 0, NULL, NULL, NULL, NULL, 0, NULL, NULL) == Z3_EINVAL);
    CHECK(zero3_reduce_adamw_hybrid(NULL, 0, 2, NULL, 0, NULL, NULL, NULL, NULL, 0, NULL, NULL) == Z3_EINVAL);
    CHECK(zero3_gather_block(NULL, NULL, NULL, NULL, NULL) == Z3_EINVAL);
}

int main(void)
{
    check_plan_d8();
    check_plan_d32_padded();
    check_ledger();
    check_scalars();
    check_errors();
    check_host_adamw();
    if (failures) {
        fprintf(stderr, "%d check(s) failed\n", failures);
        return 1;
    }
    printf("host ABI ok\n");
    return 0;
}
