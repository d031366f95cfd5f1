// host_adamw.cpp -- AdamW and the bf16 cast on the host, for the CPU-offload
// form of the step ("7.10 — Fully-sharded data parallel (FSDP / ZeRO-3)", §8,
// the CPU-offload variant: the Adam state lives in CPU memory; every step the
// averaged gradient shard goes down to the CPU, the optimiser runs there, and
// the updated bf16 weights go back up).
//
// The arithmetic is element for element the GPU kernels': each step one IEEE
// binary32 operation rounded to nearest-even, in the same order, with no
// contraction into fused multiply-adds (this file is compiled with
// -ffp-contract=off and without any fast-math flag), so the host step gives
// the same bits as the fused kernel.  The loop is plain C++ that the compiler
// vectorises; square root and division are the correctly rounded IEEE ones.
//
// The work is split over a pool of host threads that lives for the rest of the
// process (created on first use, never torn down: its threads may still wait
// for work when the process exits).  One call runs at a time; a second caller
// waits for the first to finish.  A child made by fork() starts a pool of its
// own on its first call.
#include <algorithm>
#include <atomic>
#include <condition_variable>
#include <cstdint>
#include <cstring>
#include <functional>
#include <mutex>
#include <thread>
#include <vector>

#include <pthread.h>

#include "adamw_scalars.h"
#include "plan_impl.h"
#include "zero3.h"

namespace {

// fp32 -> bf16, round to nearest, ties to even, on the bit pattern: add half a
// bf16 ulp (0x7FFF, plus one when the kept last bit is odd) and truncate.
// Finite values round correctly across the subnormal range and overflow to
// infinity; NaN stays a quiet NaN.
inline uint16_t bf16_rne(float x) {
    uint32_t u;
    std::memcpy(&u, &x, sizeof u);
    if ((u & 0x7FFFFFFFu) > 0x7F800000u) return uint16_t((u >> 16) | 0x0040u);
    u += 0x7FFFu + ((u >> 16) & 1u);
    return uint16_t(u >> 16);
}

inline float f32_of_bf16(uint16_t h) {
    const uint32_t u = uint32_t(h) << 16;
    float x;
    std::memcpy(&x, &u, sizeof x);
    return x;
}

// Elements [b, e) of one AdamW step.  G is float (fp32 reduce) or uint16_t
// (bf16 gradient bits).
template <class G>
void adamw_range(const AdamScalars s, const G* __restrict g, float* __restrict p, float* __restrict m,
                 float* __restrict v, uint16_t* __restrict w, int64_t b, int64_t e) {
    for (int64_t i = b; i < e; ++i) {
        float gi;
        if constexpr (sizeof(G) == 2)
            gi = f32_of_bf16(g[i]);
        else
            gi = g[i];
        const float p1 = p[i] * s.decay;
        const float m1 = s.b1 * m[i] + s.omb1 * gi;
        const float g2 = gi * gi;
        const float v1 = s.b2 * v[i] + s.omb2 * g2;
        const float denom = std::sqrt(v1) * s.inv_sqrt_bc2 + s.eps;
        const float delta = s.step_size * (m1 / denom);
        const float p2 = p1 - delta;
        p[i] = p2;
        m[i] = m1;
        v[i] = v1;
        w[i] = bf16_rne(p2);
    }
}

// A pool of worker threads; run(n, f) calls f(0) .. f(n-1) spread over the
// workers and the calling thread and returns when every call has returned.
class Pool;
Pool* g_pool = nullptr;  // never destroyed: workers may still wait at exit

class Pool {
  public:
    static Pool& get() {
        static std::once_flag once;
        std::call_once(once, [] {
            g_pool = new Pool();
            pthread_atfork(nullptr, nullptr, &Pool::after_fork_in_child);
        });
        return *g_pool;
    }

    void run(int workers, int n_tasks, const std::function<void(int)>& f) {
        std::lock_guard<std::mutex> one_job(job_mutex_);
        grow(workers);
        {
            std::lock_guard<std::mutex> lk(m_);
            job_ = &f;
            n_tasks_ = n_tasks;
            next_.store(0);
            pending_ = n_tasks;
            wanted_ = workers;
            ++generation_;
        }
        cv_.notify_all();
        drain(f, n_tasks);
        std::unique_lock<std::mutex> lk(m_);
        done_.wait(lk, [&] { return pending_ == 0 && busy_ == 0; });
        job_ = nullptr;
    }

  private:
    // Only the forking thread lives on in the child: the workers are gone and
    // a lock of the pool may have been held by one of them.  The child gets a
    // fresh, empty pool; the old one is left as it is (its thread handles
    // cannot be destroyed).
    static void after_fork_in_child() { g_pool = new Pool(); }

    void grow(int n) {
        while (int(threads_.size()) < n) {
            const int id = int(threads_.size());
            threads_.emplace_back([this, id] { loop(id); });
        }
    }

    // Claim and run tasks until none is left; returns how many this thread ran.
    int drain(const std::function<void(int)>& f, int n_tasks) {
        int ran = 0;
        for (int t = next_.fetch_add(1); t < n_tasks; t = next_.fetch_add(1)) {
            f(t);
            ++ran;
        }
        if (ran > 0) {
            std::lock_guard<std::mutex> lk(m_);
            pending_ -= ran;
            if (pending_ == 0) done_.notify_all();
        }
        return ran;
    }

    void loop(int id) {
        uint64_t seen = 0;
        for (;;) {
            const std::function<void(int)>* f;
            int n;
            {
                std::unique_lock<std::mutex> lk(m_);
                cv_.wait(lk, [&] { return generation_ != seen; });
                seen = generation_;
                if (id >= wanted_ || job_ == nullptr) continue;  // this job asked for fewer threads
                f = job_;
                n = n_tasks_;
                ++busy_;
            }
            drain(*f, n);
            std::lock_guard<std::mutex> lk(m_);
            if (--busy_ == 0 && pending_ == 0) done_.notify_all();
        }
    }

    std::mutex job_mutex_;  // one job at a time
    std::mutex m_;
    std::condition_variable cv_, done_;
    std::vector<std::thread> threads_;
    const std::function<void(int)>* job_ = nullptr;
    int n_tasks_ = 0, pending_ = 0, busy_ = 0, wanted_ = 0;
    uint64_t generation_ = 0;
    std::atomic<int> next_{0};
};

constexpr int64_t kGrain = 1 << 14;  // elements per task at least (64 KB of fp32 per array)
constexpr int kMaxThreads = 256;

}  // namespace

extern "C" Z3_API int zero3_host_adamw(int64_t n, const void* grad, int32_t grad_dtype, float* master,
                                       float* exp_avg, float* exp_avg_sq, uint16_t* work_bf16, const z3_adamw* hp,
                                       int32_t n_threads) {
    if (n < 0 || n_threads < 0 || !hp_valid(hp)) return Z3_EINVAL;
    if (grad_dtype != Z3_REDUCE_FP32 && grad_dtype != Z3_REDUCE_BF16) return Z3_EINVAL;
    if (n == 0) return Z3_OK;
    if (grad == nullptr || master == nullptr || exp_avg == nullptr || exp_avg_sq == nullptr || work_bf16 == nullptr)
        return Z3_EINVAL;
    const int64_t gsz = grad_dtype == Z3_REDUCE_FP32 ? 4 : 2;
    if (!z3::aligned(grad, uintptr_t(gsz)) || !z3::aligned(master, 4) || !z3::aligned(exp_avg, 4) ||
        !z3::aligned(exp_avg_sq, 4) || !z3::aligned(work_bf16, 2))
        return Z3_EALIGN;
    if (n > (int64_t(1) << 60)) return Z3_EOVERFLOW;
    // the outputs overlap neither each other nor the gradient
    const void* outs[4] = {master, exp_avg, exp_avg_sq, work_bf16};
    const int64_t bytes[4] = {n * 4, n * 4, n * 4, n * 2};
    for (int x = 0; x < 4; ++x) {
        if (z3::overlaps(outs[x], bytes[x], grad, n * gsz)) return Z3_EINVAL;
        for (int y = x + 1; y < 4; ++y)
            if (z3::overlaps(outs[x], bytes[x], outs[y], bytes[y])) return Z3_EINVAL;
    }

    const AdamScalars s = step_scalars(hp);
    int threads = n_threads > 0 ? n_threads : int(std::thread::hardware_concurrency());
    threads = std::max(1, std::min({threads, kMaxThreads, int((n + kGrain - 1) / kGrain)}));
    // about four tasks per thread for balance, each a whole number of 16-element groups
    const int64_t tasks = std::min<int64_t>(int64_t(threads) * 4, (n + kGrain - 1) / kGrain);
    const int64_t per = ((n + tasks - 1) / tasks + 15) / 16 * 16;
    auto body = [&](int t) {
        const int64_t b = int64_t(t) * per, e = std::min(n, b + per);
        if (b >= e) return;
        if (grad_dtype == Z3_REDUCE_FP32)
            adamw_range(s, static_cast<const float*>(grad), master, exp_avg, exp_avg_sq, work_bf16, b, e);
        else
            adamw_range(s, static_cast<const uint16_t*>(grad), master, exp_avg, exp_avg_sq, work_bf16, b, e);
    };
    if (threads == 1) {
        for (int64_t t = 0; t < tasks; ++t) body(int(t));
        return Z3_OK;
    }
    try {
        Pool::get().run(threads - 1, int(tasks), body);
    } catch (...) {  // thread creation failed: nothing crosses the C boundary
        return Z3_ENOMEM;
    }
    return Z3_OK;
}
