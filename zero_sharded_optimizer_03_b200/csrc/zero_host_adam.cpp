// zero_host_adam.cpp -- host (CPU) side of ZeRO-Offload: a multithreaded AdamW over fp32 state
// held in host memory, and the thread pool that runs it.
//
// [P2] "ZeRO-Offload": optimizer state and gradients live in CPU memory; the GPU produces the
// gradients, the CPU updates the optimizer state, and the updated parameters go back to the GPU.
// The update rule and its operation order are those of the device kernels (zero_adam_shard in
// include/zero.h): every operation is one IEEE fp32 round-to-nearest step, no contraction (this
// file is compiled with -ffp-contract=off, -fno-math-errno so that sqrt is the IEEE instruction),
// so the host and the device produce the same bits.  The loop is written so the compiler can
// vectorize it; target_clones picks an AVX-512 / AVX2 / baseline body at run time, and every
// variant computes the same correctly rounded results.
#include <cmath>
#include <condition_variable>
#include <cstdint>
#include <cstring>
#include <functional>
#include <memory>
#include <mutex>
#include <thread>
#include <vector>

#include "zero.h"

// sets the thread-local message returned by zero_last_error (zero_abi.cu)
int zero_internal_fail(int code, const char* msg);

namespace zh {

struct Scalars {
  float b1, b2, omb1, omb2, eps, decay, step_size, sbc2, coef;
};

// b^e by binary exponentiation in double, the same sequence of products as the device kernels.
static double pow_binary(double b, long long e) {
  double r = 1.0;
  while (e > 0) {
    if (e & 1) r = r * b;
    b = b * b;
    e >>= 1;
  }
  return r;
}

static Scalars make_scalars(const zero_hparams_t* hp, int64_t t, float coef) {
  Scalars c;
  c.b1 = (float)hp->beta1;
  c.b2 = (float)hp->beta2;
  c.omb1 = (float)(1.0 - hp->beta1);
  c.omb2 = (float)(1.0 - hp->beta2);
  c.eps = (float)hp->eps;
  c.decay = (float)(1.0 - hp->lr * hp->weight_decay);
  c.step_size = (float)(hp->lr / (1.0 + -pow_binary(hp->beta1, t)));
  c.sbc2 = (float)std::sqrt(1.0 + -pow_binary(hp->beta2, t));
  c.coef = coef;
  return c;
}

static inline uint16_t bf16_nearest_even(float x) {
  uint32_t u;
  std::memcpy(&u, &x, 4);
  // round to nearest, ties to even (NaN never reaches here: an overflowed step is skipped)
  u += 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

__attribute__((target_clones("avx512f", "avx2", "default"))) static void adam_range(
    float* __restrict p, float* __restrict m, float* __restrict v, const float* __restrict g,
    uint16_t* __restrict out16, int64_t n, const Scalars c) {
  for (int64_t i = 0; i < n; ++i) {
    const float gi = g[i] * c.coef;
    float pi = p[i] * c.decay;
    const float mi = c.b1 * m[i] + c.omb1 * gi;
    const float vi = c.b2 * v[i] + (c.omb2 * gi) * gi;
    const float den = std::sqrt(vi) / c.sbc2 + c.eps;
    pi = pi - c.step_size * (mi / den);
    p[i] = pi;
    m[i] = mi;
    v[i] = vi;
    if (out16) out16[i] = bf16_nearest_even(pi);
  }
}

// A small persistent pool: run(n_tasks, fn) executes fn(k) for k in [0, n_tasks) on the pool's
// threads plus the calling thread and returns when all are done.
class Pool {
 public:
  explicit Pool(int nthreads) {
    for (int k = 0; k + 1 < nthreads; ++k) workers_.emplace_back([this] { loop(); });
  }
  ~Pool() {
    {
      std::lock_guard<std::mutex> lk(mu_);
      stop_ = true;
    }
    cv_.notify_all();
    for (auto& t : workers_) t.join();
  }
  int size() const { return (int)workers_.size() + 1; }
  void run(int n_tasks, const std::function<void(int)>& fn) {
    {
      std::lock_guard<std::mutex> lk(mu_);
      fn_ = &fn;
      n_tasks_ = n_tasks;
      next_ = 0;
      done_ = 0;
      ++gen_;
    }
    cv_.notify_all();
    work();
    std::unique_lock<std::mutex> lk(mu_);
    done_cv_.wait(lk, [&] { return done_ == n_tasks_; });
    fn_ = nullptr;
  }

 private:
  void work() {
    while (true) {
      int k;
      const std::function<void(int)>* fn;
      {
        std::lock_guard<std::mutex> lk(mu_);
        if (!fn_ || next_ >= n_tasks_) return;
        k = next_++;
        fn = fn_;
      }
      (*fn)(k);
      {
        std::lock_guard<std::mutex> lk(mu_);
        if (++done_ == n_tasks_) done_cv_.notify_all();
      }
    }
  }
  void loop() {
    long long seen = 0;
    while (true) {
      {
        std::unique_lock<std::mutex> lk(mu_);
        cv_.wait(lk, [&] { return stop_ || gen_ != seen; });
        if (stop_) return;
        seen = gen_;
      }
      work();
    }
  }
  std::vector<std::thread> workers_;
  std::mutex mu_;
  std::condition_variable cv_, done_cv_;
  const std::function<void(int)>* fn_ = nullptr;
  int n_tasks_ = 0, next_ = 0, done_ = 0;
  long long gen_ = 0;
  bool stop_ = false;
};

// One pool per requested size, kept for the life of the process.
static Pool& pool_for(int nthreads) {
  static std::mutex mu;
  static std::vector<std::unique_ptr<Pool>> pools;
  std::lock_guard<std::mutex> lk(mu);
  for (auto& p : pools)
    if (p->size() == nthreads) return *p;
  pools.emplace_back(new Pool(nthreads));
  return *pools.back();
}

int resolve_threads(int nthreads) {
  if (nthreads > 0) return nthreads;
  const unsigned hc = std::thread::hardware_concurrency();
  return hc > 0 ? (int)hc : 1;
}

// Updates n elements, split into blocks of 64K elements over `nthreads` threads.
void adam_host(float* p, float* m, float* v, const float* g, uint16_t* out16, int64_t n, const zero_hparams_t* hp,
               int64_t t, float coef, int nthreads) {
  const Scalars c = make_scalars(hp, t, coef);
  const int64_t block = 1 << 16;
  const int64_t nblocks = (n + block - 1) / block;
  nthreads = resolve_threads(nthreads);
  if (nthreads == 1 || nblocks <= 1) {
    adam_range(p, m, v, g, out16, n, c);
    return;
  }
  Pool& pool = pool_for(nthreads);
  std::function<void(int)> fn = [&](int k) {
    const int64_t lo = (int64_t)k * block;
    const int64_t len = n - lo < block ? n - lo : block;
    adam_range(p + lo, m + lo, v + lo, g + lo, out16 ? out16 + lo : nullptr, len, c);
  };
  pool.run((int)nblocks, fn);
}

float clip_factor(double max_norm, double sumsq) {
  if (!(max_norm > 0.0)) return 1.0f;
  double coef = max_norm / (std::sqrt(sumsq) + 1e-6);
  if (coef > 1.0) coef = 1.0;
  return (float)coef;
}

}  // namespace zh

extern "C" int zero_host_adam(float* master, float* exp_avg, float* exp_avg_sq, const float* grad, int64_t n,
                              const zero_hparams_t* hp, int64_t t, float clip_coef, uint16_t* param_out,
                              int nthreads) {
  if (!hp) return zero_internal_fail(ZERO_EINVAL, "hparams is NULL");
  if (n < 0 || t < 1) return zero_internal_fail(ZERO_EINVAL, "need n >= 0 and step t >= 1");
  if (!(clip_coef > 0.0f) || clip_coef > 1.0f) return zero_internal_fail(ZERO_EINVAL, "clip_coef must be in (0, 1]");
  if (n == 0) return ZERO_OK;
  if (!master || !exp_avg || !exp_avg_sq || !grad)
    return zero_internal_fail(ZERO_EINVAL, "master, exp_avg, exp_avg_sq and grad must be non-NULL");
  zh::adam_host(master, exp_avg, exp_avg_sq, grad, param_out, n, hp, t, clip_coef, nthreads);
  return ZERO_OK;
}
