// zero_kernels.cuh -- sm_100a kernels of the sharded mixed-precision Adam step (ZeRO-1/2/3).
//
// Every kernel here streams HBM: per element it does a few dozen fp32 operations against
// tens of bytes of traffic (about 0.35 flop/byte), far below the ridge point, so there are
// no tensor-core paths.  The design choices are the ones that matter for a bandwidth-bound
// kernel on B200: 16-byte vector loads/stores with streaming cache hints, an Nd-way fan-in
// issued as independent loads in flight per thread, persistent grids sized to a multiple of
// the 148 SMs, and a single pass over the data wherever the algorithm allows.
//
// Simulated collectives ([P1] §二 and §三, [P3] core operations; page titles in include/zero.h):
// the Nd "ranks" are Nd buffers in this GPU's memory.  A reduce-scatter is the Nd-way read of
// the gradient replicas at an index (each index belongs to exactly one rank's shard), an
// all-gather is the Nd-way write of the bf16 weight at that index.  Because both act on the
// same index as the Adam update, the fused kernel does RS + Adam + AG in one pass.
//
// Numerics: every fp32 operation is an explicit round-to-nearest intrinsic (no contraction),
// replicas are summed in rank order, and the per-element rule is the one documented for
// zero_adam_shard in include/zero.h.  The overflow flag is an OR (exact), the sum of squares
// is accumulated in double in a fixed order for a given grid.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace zb {

constexpr int kMaxNd = 64;
constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kMaxCtas = 8192;

// Step bookkeeping at the start of the workspace.
struct Header {
  unsigned int done;      // CTAs of the current launch that have finished (reset by the last one)
  int pending_flag;       // overflow seen by the step in progress
  double pending_sumsq;   // sum of squares accumulated by the step in progress
  long long t;            // completed updates
  long long skipped;      // skipped steps
  int live;               // state copy holding the current state (fused path)
  int last_flag;          // overflow of the last finished step
  double last_sumsq;      // sum of squares of the last finished step
  int error;              // nonzero once a kernel gave up a bounded wait (sticky until init)
  int dyn;                // dynamic loss scaling on: the gradients carry `scale`
  double scale;           // current loss scale (dynamic)
  double growth, backoff; // scale factors after `interval` clean steps / after an overflow
  long long interval;
  long long good;         // clean steps since the last change of the scale
  unsigned long long chunk;  // next work chunk of a dynamically scheduled launch (0 between launches)
};
static_assert(sizeof(Header) <= 256, "header must fit its slot");

struct Partial {
  double sumsq;
  int flag;
  int pad;
};

constexpr size_t kHeaderBytes = 256;
constexpr size_t kWorkspaceBytes = kHeaderBytes + sizeof(Partial) * kMaxCtas;

// What the last CTA of a launch does with the launch's totals.
enum : int {
  kAccSet = 1,    // pending := launch totals (first launch of a step)
  kAccAdd = 2,    // pending += launch totals
  kFinalize = 4,  // end the step: t += 1 unless overflow (else skipped += 1)
  kFlip = 8,      // with kFinalize and no overflow: swap the live state copy
};

// Element-independent scalars, rounded once to fp32 on the host (see include/zero.h).
struct Consts {
  float inv;    // 1/(Nd*loss_scale) or 1/loss_scale
  float b1, b2;
  float omb1, omb2;
  float eps;
  float decay;  // 1 - lr*wd
  float unused;
  double lr, b1d, b2d;  // for the step-dependent bias corrections
  double inv_base;      // Nd (mean) or 1 (sum): the unscale factor is 1/(inv_base * loss scale)
  double max_norm;      // global-norm clipping bound (<= 0: off)
};

// Unscale factor of the step: from the host (static loss scale) or, with dynamic loss scaling,
// 1/(inv_base * scale) from the workspace, evaluated in double and rounded once to fp32.
__device__ __forceinline__ float step_inv(const Consts& c, const Header* h) {
  if (!__ldcg(&h->dyn)) return c.inv;
  return __double2float_rn(__ddiv_rn(1.0, __dmul_rn(c.inv_base, __ldcg(&h->scale))));
}

// Clipping factor min(1, max_norm/(sqrt(sumsq) + 1e-6)) in double, rounded once to fp32.
__device__ __forceinline__ float clip_coef(double max_norm, double sumsq) {
  if (!(max_norm > 0.0)) return 1.0f;
  double coef = __ddiv_rn(max_norm, __dadd_rn(__dsqrt_rn(sumsq), 1e-6));
  if (coef > 1.0) coef = 1.0;
  return __double2float_rn(coef);
}

// End of a step: bookkeeping of the counters and of the dynamic loss scale.
__device__ __forceinline__ void end_step(Header& h, int flip) {
  const int of = h.pending_flag;
  h.last_flag = of;
  h.last_sumsq = h.pending_sumsq;
  if (!of) {
    h.t += 1;
    if (flip) h.live ^= 1;
  } else {
    h.skipped += 1;
  }
  if (h.dyn) {
    if (of) {
      h.scale = __dmul_rn(h.scale, h.backoff);
      h.good = 0;
    } else if (++h.good >= h.interval) {
      const double grown = __dmul_rn(h.scale, h.growth);
      if (grown <= 3.4028234663852886e38) h.scale = grown;  // stays finite in fp32
      h.good = 0;
    }
  }
  h.pending_flag = 0;
  h.pending_sumsq = 0.0;
}

struct Bias {
  float step_size;  // lr / (1 - b1^t)
  float sbc2;       // sqrt(1 - b2^t)
};

// b^e for e >= 0 by binary exponentiation (square-and-multiply, Knuth TAOCP vol. 2, 4.6.3),
// every product one double round-to-nearest step.
__device__ __forceinline__ double pow_binary(double b, long long e) {
  double r = 1.0;
  while (e > 0) {
    if (e & 1) r = __dmul_rn(r, b);
    b = __dmul_rn(b, b);
    e >>= 1;
  }
  return r;
}

__device__ __forceinline__ Bias bias_for(const Consts& c, long long t) {
  Bias o;
  o.step_size = __double2float_rn(__ddiv_rn(c.lr, __dadd_rn(1.0, -pow_binary(c.b1d, t))));
  o.sbc2 = __double2float_rn(__dsqrt_rn(__dadd_rn(1.0, -pow_binary(c.b2d, t))));
  return o;
}

// One Adam/AdamW update of one element (the rule of zero_adam_shard).  With wd = 0 the decay
// factor is exactly 1 and the first multiply changes nothing.
__device__ __forceinline__ void adam_elem(float g, float& p, float& m, float& v, const Consts& c,
                                          const Bias& b) {
  p = __fmul_rn(p, c.decay);
  m = __fadd_rn(__fmul_rn(c.b1, m), __fmul_rn(c.omb1, g));
  v = __fadd_rn(__fmul_rn(c.b2, v), __fmul_rn(__fmul_rn(c.omb2, g), g));
  const float den = __fadd_rn(__fdiv_rn(__fsqrt_rn(v), b.sbc2), c.eps);
  p = __fsub_rn(p, __fmul_rn(b.step_size, __fdiv_rn(m, den)));
}

__device__ __forceinline__ int nonfinite(float x) {
  return (__float_as_uint(x) & 0x7f800000u) == 0x7f800000u;
}

// ------------------------------------------------------------------ memory helpers

__device__ __forceinline__ uint4 ld_stream(const uint16_t* p) {
  return __ldcs(reinterpret_cast<const uint4*>(p));
}
__device__ __forceinline__ float4 ld_stream(const float* p) {
  return __ldcs(reinterpret_cast<const float4*>(p));
}
__device__ __forceinline__ void st_stream(uint16_t* p, uint4 v) {
  __stcs(reinterpret_cast<uint4*>(p), v);
}
__device__ __forceinline__ void st_stream(float* p, float4 v) {
  __stcs(reinterpret_cast<float4*>(p), v);
}

// 16-bit gradient decoding (exact).
template <int DT>
struct Dec;

template <>
struct Dec<0> {  // bf16: the upper half of an fp32 word
  __device__ static __forceinline__ float one(uint16_t h) { return __uint_as_float((uint32_t)h << 16); }
  __device__ static __forceinline__ void add2(float& a, float& b, uint32_t w) {
    a = __fadd_rn(a, __uint_as_float(w << 16));
    b = __fadd_rn(b, __uint_as_float(w & 0xffff0000u));
  }
};

template <>
struct Dec<1> {  // IEEE fp16
  __device__ static __forceinline__ float one(uint16_t h) { return __half2float(__ushort_as_half(h)); }
  __device__ static __forceinline__ void add2(float& a, float& b, uint32_t w) {
    __half2 h2;
    *reinterpret_cast<uint32_t*>(&h2) = w;
    const float2 f = __half22float2(h2);
    a = __fadd_rn(a, f.x);
    b = __fadd_rn(b, f.y);
  }
};

template <int DT>
__device__ __forceinline__ void add8(float (&s)[8], const uint4& q) {
  Dec<DT>::add2(s[0], s[1], q.x);
  Dec<DT>::add2(s[2], s[3], q.y);
  Dec<DT>::add2(s[4], s[5], q.z);
  Dec<DT>::add2(s[6], s[7], q.w);
}

// Rank-order sum of the Nd replicas at 8 consecutive elements starting at i (16-byte aligned).
// Loads are issued CH ranks at a time so that up to CH x 16 bytes per thread are in flight; a
// small CH (small fan-in) leaves registers for more resident warps.
template <int DT, int CH = 8>
__device__ __forceinline__ void fan_in8(const uint16_t* const* grads, int Nd, int64_t i, float (&s)[8]) {
#pragma unroll
  for (int k = 0; k < 8; ++k) s[k] = 0.0f;
#pragma unroll 1
  for (int r0 = 0; r0 < Nd; r0 += CH) {
    uint4 q[CH];
#pragma unroll
    for (int u = 0; u < CH; ++u)
      if (r0 + u < Nd) q[u] = ld_stream(grads[r0 + u] + i);
#pragma unroll
    for (int u = 0; u < CH; ++u)
      if (r0 + u < Nd) add8<DT>(s, q[u]);
  }
}

template <int DT>
__device__ __forceinline__ float fan_in1(const uint16_t* const* grads, int Nd, int64_t i) {
  float s = 0.0f;
  for (int r = 0; r < Nd; ++r) s = __fadd_rn(s, Dec<DT>::one(grads[r][i]));
  return s;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);  // .x (low half) = lo, round to nearest even
  return *reinterpret_cast<const uint32_t*>(&h);
}

__device__ __forceinline__ uint4 pack_bf16x8(const float (&p)[8]) {
  return make_uint4(pack_bf16x2(p[0], p[1]), pack_bf16x2(p[2], p[3]), pack_bf16x2(p[4], p[5]),
                    pack_bf16x2(p[6], p[7]));
}

__device__ __forceinline__ uint16_t to_bf16(float x) {
  const __nv_bfloat16 h = __float2bfloat16_rn(x);
  return *reinterpret_cast<const uint16_t*>(&h);
}

__device__ __forceinline__ void unpack(const float4& a, const float4& b, float (&x)[8]) {
  x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
  x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
}

// Vector bounds of a window: the 8-aligned interior [vlo, vhi) and the scalar remainder.
struct Span {
  int64_t vlo, vhi, nvec, nhead, nrest;
  __device__ __forceinline__ Span(int64_t lo, int64_t hi, int vec) {
    vlo = lo;
    vhi = lo;
    if (vec) {
      vlo = (lo + 7) & ~int64_t(7);
      if (vlo > hi) vlo = hi;
      vhi = hi & ~int64_t(7);
      if (vhi < vlo) vhi = vlo;
    }
    nvec = (vhi - vlo) >> 3;
    nhead = vlo - lo;
    nrest = nhead + (hi - vhi);
  }
  // e-th scalar element: the head [lo, vlo) then the tail [vhi, hi)
  __device__ __forceinline__ int64_t scalar_index(int64_t lo, int64_t e) const {
    return e < nhead ? lo + e : vhi + (e - nhead);
  }
};

__device__ __forceinline__ double warp_sum(double x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x = __dadd_rn(x, __shfl_xor_sync(0xffffffffu, x, o));
  return x;
}

// Launch epilogue: per-CTA totals into the partials, and the last CTA to arrive reduces them
// in CTA order and applies `mode` to the header.  No CTA waits for another (the last one to
// arrive does the work), so there is no spin and no co-residency assumption.
//
// Arrival: thread 0 publishes the CTA's partial and counts the CTA in with one acquire-release
// atomic add at device scope.  As a release it publishes the partial and every thread's earlier
// stores (state copies, replicas: the barrier before it orders them first); as an acquire, on the
// CTA that arrives last, it makes what every other CTA published before its own arrival visible
// to the loads after the next barrier.  (Separate fences around a relaxed add measured 0.34 us
// slower on a one-round step of 1M elements.)  The last CTA's loads are issued together: each
// thread its partials (thread k adds partials k, k + 32 NW, ... in that order, as one load chain
// would) and thread 0 the header words the step's end reads, so the two wait for memory once.
// The kernel boundary publishes the header, so no fence follows the update.
template <int NW = kWarps>
__device__ __forceinline__ int block_finish(double sq, int bad, Header* hdr, Partial* part, int mode) {
  if (mode == 0) return 0;
  constexpr int BT = NW * 32;
  constexpr int U = 4;  // partials in flight per thread
  __shared__ double r_sq[NW];
  __shared__ int r_bad[NW];
  __shared__ int am_last;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  sq = warp_sum(sq);
  bad = __any_sync(0xffffffffu, bad);
  if (lane == 0) {
    r_sq[warp] = sq;
    r_bad[warp] = bad;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    double s = 0.0;
    int f = 0;
    for (int w = 0; w < NW; ++w) {
      s = __dadd_rn(s, r_sq[w]);
      f |= r_bad[w];
    }
    part[blockIdx.x].sumsq = s;
    part[blockIdx.x].flag = f;
    unsigned prev;
    asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], 1;" : "=r"(prev) : "l"(&hdr->done) : "memory");
    am_last = prev == gridDim.x - 1;
  }
  __syncthreads();
  if (!am_last) return 0;
  Header hv;
  if (threadIdx.x == 0) hv = *hdr;
  const int nparts = (int)gridDim.x;
  double s = 0.0;
  int f = 0;
  for (int k0 = threadIdx.x; k0 < nparts; k0 += U * BT) {
    double ps[U];
    int pf[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int k = k0 + u * BT;
      if (k < nparts) {
        ps[u] = __ldcg(&part[k].sumsq);
        pf[u] = __ldcg(&part[k].flag);
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      if (k0 + u * BT < nparts) {
        s = __dadd_rn(s, ps[u]);
        f |= pf[u];
      }
    }
  }
  s = warp_sum(s);
  f = __any_sync(0xffffffffu, f);
  __syncthreads();
  if (lane == 0) {
    r_sq[warp] = s;
    r_bad[warp] = f;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    double tot = 0.0;
    int fl = 0;
    for (int w = 0; w < NW; ++w) {
      tot = __dadd_rn(tot, r_sq[w]);
      fl |= r_bad[w];
    }
    if (mode & kAccSet) {
      hv.pending_flag = fl;
      hv.pending_sumsq = tot;
    } else if (mode & kAccAdd) {
      hv.pending_flag |= fl;
      hv.pending_sumsq = __dadd_rn(hv.pending_sumsq, tot);
    }
    int skipped = 0;
    if (mode & kFinalize) {
      end_step(hv, mode & kFlip);
      skipped = hv.last_flag;
      hdr->last_flag = hv.last_flag;
      hdr->last_sumsq = hv.last_sumsq;
      hdr->t = hv.t;
      hdr->skipped = hv.skipped;
      hdr->live = hv.live;
      hdr->scale = hv.scale;
      hdr->good = hv.good;
    }
    if (mode & (kAccSet | kAccAdd | kFinalize)) {
      hdr->pending_flag = hv.pending_flag;
      hdr->pending_sumsq = hv.pending_sumsq;
    }
    hdr->done = 0u;
    hdr->chunk = 0ull;  // every CTA has left its chunk loop: ready for the next launch
    return skipped;
  }
  return 0;
}

// ------------------------------------------------------------------ K1: fused RS + Adam + AG

struct FusedArgs {
  const uint16_t* grads[kMaxNd];  // Nd gradient replicas
  uint16_t* reps[kMaxNd];         // Nd bf16 weight replicas
  float* p[2];                    // master weights, two copies (read live, write 1-live)
  float* m[2];
  float* v[2];
  int64_t lo, hi;                 // window of global indices
  Consts c;
  Header* hdr;
  Partial* part;
  int Nd;
  int mode;
  int vec;
  int nrep;     // bf16 outputs per element: the Nd replicas (ZeRO-1/2), or 1 (a ZeRO-3 layer's shard)
  int chunked;  // 1: CTAs take chunks of kChunkVecs vectors from hdr->chunk (needs mode != 0)
  int trigger_late;  // 1: a dependent launch may start only once this CTA's main loop is done
  int wait_first;    // 1: launched as a programmatic dependent of whatever precedes it on the
                     // stream (the first launch of a step); waits for it before anything else
  int self_repair;   // 1: (a step's only launch) after an overflowed step the last CTA rewrites
                     // the window of every replica from the unchanged state itself
  int prefetch;      // 1: a thread's second vector is prefetched to L2 (set only where every
                     // buffer is this GPU's memory; never for a window that reads peers' memory)
  // ZeRO-3 layer with its gather (kernel variant G): gsrc is the layer's bf16 weights before the
  // update (the concatenated shards, the same memory as reps[0]); each element's old word is
  // copied to the Nd gathered-layer buffers gout[r] before the new weight overwrites it
  const uint16_t* gsrc;
  uint16_t* gout[kMaxNd];
};

// Compiler-only ordering point: memory accesses written before it are emitted before those
// written after it (used where a thread reads a word and later overwrites the same word).
__device__ __forceinline__ void compiler_fence() { asm volatile("" ::: "memory"); }

// Programmatic dependent launch: a grid launched with programmatic stream serialization may
// start while the previous grid in the stream finishes.  launch_dependents lets the next grid
// start; wait blocks until the previous grid has completed and its memory is visible (it
// returns at once for a grid launched without the attribute).
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Starts the transfer of the line holding `p` into L2 (no register result, no ordering).
__device__ __forceinline__ void prefetch_l2(const void* p) {
  asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

// Vectors per dynamically scheduled chunk: 4 per thread of a CTA.
constexpr int kChunkIters = 4;
constexpr int64_t kChunkVecs = (int64_t)kChunkIters * kThreads;

// CH: gradient replicas loaded per batch (1, 2, 4 or 8).  Small batches leave registers for more
// resident warps (the budgets are below), so more loads are in flight at small fan-in, where each
// element carries few bytes.
//
// Work distribution: a grid-stride loop over one wave of resident CTAs (every SM owns a fixed
// share of the window), or, with a.chunked, chunks of kChunkVecs vectors handed out by an atomic
// counter in the workspace header, so that SMs that stream faster take more of the window; the
// last CTA to finish resets the counter.  Which vector a thread updates does not change any
// result (every element is independent); only the order in which the per-CTA sums of squares
// are formed does.
//
// Consecutive buckets of one step may be launched as programmatic dependents (fixed split
// only): the next bucket's CTAs start streaming while this one's last CTAs finish.  The header
// fields read at the start (t, live, loss scale) change only when a step ends, and a dependent
// grid waits for its predecessor before it touches the partials and the counters.  The first
// launch of a step (wait_first) is a programmatic dependent of whatever precedes it and waits for
// it before its first instruction, so only its launch overlaps the predecessor.
//
// G (ZeRO-3 layer with its gather): every element j of the layer is also the layer's gathered
// weight j (the gather concatenates the Nd shards, which lie back to back), so one pass reads
// the old bf16 word, fans it out to the Nd gathered buffers, and then writes the updated
// weight over it: 2 + 2Nd bytes of gather traffic ride along with the update's 26 + 2Nd.
//
// Start of a launch.  With EARLY (every instantiation but batches of 2 without the gather),
// every thread reads the live copy index itself (one broadcast load per warp), because the
// state loads depend on it; the bias corrections and the unscale factor, which thread 0
// evaluates in double, are needed only once the data has arrived, so the barrier that publishes
// them comes after each thread has issued its first vector's loads (1-2% faster at 1 and 4-8
// replicas than waiting for them).  Without EARLY, thread 0 reads the header and evaluates the
// scalars before a barrier, the loads start after it, and the loop body keeps its vector in
// registers of its own: at Nd = 2 that form measured faster than the restructured one.
// Registers are budgeted for 4 resident CTAs per SM at single-replica batches (3 with the
// gather, which would spill at 64 registers), 3 up to batches of 4 and 2 at 8.
template <int DT, int CH, bool G = false>
__global__ void __launch_bounds__(kThreads, (CH <= 1 && !G) ? 4 : CH <= 4 ? 3 : 2) fused_step_kernel(const __grid_constant__ FusedArgs a) {
  constexpr int BT = kThreads;
  constexpr bool EARLY = CH != 2 || G;
  if (a.wait_first) pdl_wait();  // the predecessor has completed and its memory is visible
  __shared__ Bias s_bias;
  __shared__ float s_inv;
  __shared__ int s_live;
  __shared__ long long s_chunk;
  __shared__ int s_repair;
  int live;
  if constexpr (EARLY) {
    live = __ldcg(&a.hdr->live) & 1;
    if (threadIdx.x == 0) {
      s_bias = bias_for(a.c, __ldcg(&a.hdr->t) + 1);
      s_inv = step_inv(a.c, a.hdr);
    }
  } else {
    if (threadIdx.x == 0) {
      s_bias = bias_for(a.c, __ldcg(&a.hdr->t) + 1);
      s_live = __ldcg(&a.hdr->live) & 1;
      s_inv = step_inv(a.c, a.hdr);
    }
    __syncthreads();
    live = s_live;
  }
  if (!a.trigger_late) pdl_launch_dependents();  // the next bucket may fill this launch's tail
  const float* __restrict__ sp = a.p[live];
  const float* __restrict__ sm = a.m[live];
  const float* __restrict__ sv = a.v[live];
  float* __restrict__ dp = a.p[live ^ 1];
  float* __restrict__ dm = a.m[live ^ 1];
  float* __restrict__ dv = a.v[live ^ 1];

  double sq = 0.0;
  int bad = 0;
  const Span sp8(a.lo, a.hi, a.vec);
  // One 8-element vector between its loads and its update.
  struct Vec {
    float P[8], M[8], V[8], s[8];
    uint4 w_old;
  };
  // The loads of vector j: (G) the old weights, the state copy `live`, the first batch of
  // gradient replicas; then the rank-order sum of the Nd replicas, the later batches loaded as
  // the earlier ones are added.
  auto load = [&](int64_t j, Vec& R) {
    const int64_t i = sp8.vlo + (j << 3);
    uint4 q[CH];
    if (G) R.w_old = ld_stream(a.gsrc + i);
    unpack(ld_stream(sp + i), ld_stream(sp + i + 4), R.P);
    unpack(ld_stream(sm + i), ld_stream(sm + i + 4), R.M);
    unpack(ld_stream(sv + i), ld_stream(sv + i + 4), R.V);
#pragma unroll
    for (int u = 0; u < CH; ++u)
      if (u < a.Nd) q[u] = ld_stream(a.grads[u] + i);
#pragma unroll
    for (int k = 0; k < 8; ++k) R.s[k] = 0.0f;
#pragma unroll
    for (int u = 0; u < CH; ++u)
      if (u < a.Nd) add8<DT>(R.s, q[u]);
#pragma unroll 1
    for (int r0 = CH; r0 < a.Nd; r0 += CH) {
#pragma unroll
      for (int u = 0; u < CH; ++u)
        if (r0 + u < a.Nd) q[u] = ld_stream(a.grads[r0 + u] + i);
#pragma unroll
      for (int u = 0; u < CH; ++u)
        if (r0 + u < a.Nd) add8<DT>(R.s, q[u]);
    }
  };
  // The rest of vector j: (G) the gather of the old weights, unscale, flag / sum of squares,
  // AdamW from copy `live` into copy 1-live, bf16 cast fanned out to the nrep outputs.
  auto finish = [&](int64_t j, Vec& R, const Bias& b, float inv) {
    const int64_t i = sp8.vlo + (j << 3);
    if (G) {  // the old weights to every rank's layer buffer, before they are replaced
      for (int r = 0; r < a.Nd; ++r) st_stream(a.gout[r] + i, R.w_old);
      compiler_fence();
    }
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const float g = __fmul_rn(R.s[k], inv);
      bad |= nonfinite(g);
      sq = __dadd_rn(sq, __dmul_rn((double)g, (double)g));
      adam_elem(g, R.P[k], R.M[k], R.V[k], a.c, b);
    }
    st_stream(dp + i, make_float4(R.P[0], R.P[1], R.P[2], R.P[3]));
    st_stream(dp + i + 4, make_float4(R.P[4], R.P[5], R.P[6], R.P[7]));
    st_stream(dm + i, make_float4(R.M[0], R.M[1], R.M[2], R.M[3]));
    st_stream(dm + i + 4, make_float4(R.M[4], R.M[5], R.M[6], R.M[7]));
    st_stream(dv + i, make_float4(R.V[0], R.V[1], R.V[2], R.V[3]));
    st_stream(dv + i + 4, make_float4(R.V[4], R.V[5], R.V[6], R.V[7]));
    const uint4 w = pack_bf16x8(R.P);
    for (int r = 0; r < a.nrep; ++r) st_stream(a.reps[r] + i, w);
  };
  Bias b;
  float inv;
  if (a.chunked) {
    if (EARLY) __syncthreads();  // thread 0's bias corrections and unscale factor are published
    b = s_bias;
    inv = s_inv;
    const int64_t nchunks = (sp8.nvec + kChunkVecs - 1) / kChunkVecs;
    for (;;) {
      if (threadIdx.x == 0) s_chunk = (long long)atomicAdd(&a.hdr->chunk, 1ull);
      __syncthreads();
      const int64_t c = s_chunk;
      __syncthreads();  // every thread has read s_chunk before thread 0 takes the next one
      if (c >= nchunks) break;
      const int64_t j0 = c * kChunkVecs + threadIdx.x;
#pragma unroll 1
      for (int u = 0; u < (int)(kChunkVecs / BT); ++u) {
        const int64_t j = j0 + (int64_t)u * BT;
        if (j < sp8.nvec) {
          Vec R;
          load(j, R);
          finish(j, R, b, inv);
        }
      }
    }
  } else {
    const int64_t stride = (int64_t)gridDim.x * BT;
    int64_t j = (int64_t)blockIdx.x * BT + threadIdx.x;
    if constexpr (EARLY) {
      Vec R;
      const bool first = j < sp8.nvec;
      if (first) load(j, R);  // in flight while thread 0 evaluates the step scalars
      // A window a little larger than one round of the grid leaves a second vector to some
      // threads; its lines start for L2 now, with the first round's loads, so that its loads
      // after the first update hit L2 (1M elements at Nd = 4: 0.2 us of a 14.7 us step).
      if (a.prefetch && j + stride < sp8.nvec) {
        const int64_t i2 = sp8.vlo + ((j + stride) << 3);
        prefetch_l2(sp + i2);
        prefetch_l2(sm + i2);
        prefetch_l2(sv + i2);
        if (G) prefetch_l2(a.gsrc + i2);
        for (int r = 0; r < a.Nd; ++r) prefetch_l2(a.grads[r] + i2);
      }
      __syncthreads();
      b = s_bias;
      inv = s_inv;
      if (first) finish(j, R, b, inv);
#pragma unroll 1
      for (j += stride; j < sp8.nvec; j += stride) {
        load(j, R);
        finish(j, R, b, inv);
      }
    } else {
      // one vector per iteration with everything in the loop body's own registers (the same
      // arithmetic as load + finish, in the loop shape this instantiation measured fastest in)
      const Bias bb = s_bias;
      const float ii = s_inv;
      b = bb;
      inv = ii;
#pragma unroll 1
      for (; j < sp8.nvec; j += stride) {
        const int64_t i = sp8.vlo + (j << 3);
        float P[8], M[8], V[8], sg[8];
        unpack(ld_stream(sp + i), ld_stream(sp + i + 4), P);
        unpack(ld_stream(sm + i), ld_stream(sm + i + 4), M);
        unpack(ld_stream(sv + i), ld_stream(sv + i + 4), V);
        fan_in8<DT, CH>(a.grads, a.Nd, i, sg);
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const float g = __fmul_rn(sg[k], ii);
          bad |= nonfinite(g);
          sq = __dadd_rn(sq, __dmul_rn((double)g, (double)g));
          adam_elem(g, P[k], M[k], V[k], a.c, bb);
        }
        st_stream(dp + i, make_float4(P[0], P[1], P[2], P[3]));
        st_stream(dp + i + 4, make_float4(P[4], P[5], P[6], P[7]));
        st_stream(dm + i, make_float4(M[0], M[1], M[2], M[3]));
        st_stream(dm + i + 4, make_float4(M[4], M[5], M[6], M[7]));
        st_stream(dv + i, make_float4(V[0], V[1], V[2], V[3]));
        st_stream(dv + i + 4, make_float4(V[4], V[5], V[6], V[7]));
        const uint4 w = pack_bf16x8(P);
        for (int r = 0; r < a.nrep; ++r) st_stream(a.reps[r] + i, w);
      }
    }
  }
  // before a dependent that only waits for this grid (the overflow-repair check), trigger late:
  // its CTAs would otherwise sit on the SMs for the whole of this launch
  if (a.trigger_late) pdl_launch_dependents();
  const int64_t stride = (int64_t)gridDim.x * BT;
  for (int64_t e = (int64_t)blockIdx.x * BT + threadIdx.x; e < sp8.nrest; e += stride) {
    const int64_t i = sp8.scalar_index(a.lo, e);
    if (G) {
      const uint16_t w_old = a.gsrc[i];
      for (int r = 0; r < a.Nd; ++r) a.gout[r][i] = w_old;
      compiler_fence();
    }
    const float g = __fmul_rn(fan_in1<DT>(a.grads, a.Nd, i), inv);
    bad |= nonfinite(g);
    sq = __dadd_rn(sq, __dmul_rn((double)g, (double)g));
    float P = sp[i], M = sm[i], V = sv[i];
    adam_elem(g, P, M, V, a.c, b);
    dp[i] = P;
    dm[i] = M;
    dv[i] = V;
    const uint16_t w = to_bf16(P);
    for (int r = 0; r < a.nrep; ++r) a.reps[r][i] = w;
  }
  pdl_wait();  // a programmatic dependent: the previous bucket has completed
  const int skipped = block_finish<BT / 32>(sq, bad, a.hdr, a.part, a.mode);
  // short window: the last CTA to finish repairs the replicas after a skip.  Every other CTA has
  // published its speculative stores (fence, then its arrival) before the last one arrived, so
  // these stores come after them.
  if (a.self_repair) {
    __syncthreads();
    if (threadIdx.x == 0) s_repair = skipped;
    __syncthreads();
    if (s_repair) {
      for (int64_t j = threadIdx.x; j < sp8.nvec; j += BT) {
        const int64_t i = sp8.vlo + (j << 3);
        float P[8];
        unpack(ld_stream(sp + i), ld_stream(sp + i + 4), P);
        const uint4 w = pack_bf16x8(P);
        for (int r = 0; r < a.nrep; ++r) st_stream(a.reps[r] + i, w);
      }
      for (int64_t e = threadIdx.x; e < sp8.nrest; e += BT) {
        const int64_t i = sp8.scalar_index(a.lo, e);
        const uint16_t w = to_bf16(sp[i]);
        for (int r = 0; r < a.nrep; ++r) a.reps[r][i] = w;
      }
    }
  }
}

// ------------------------------------------------------------------ K3: RS into an fp32 shard

struct RsArgs {
  const uint16_t* grads[kMaxNd];
  float* out;        // reduced gradient, indexed like the replicas (fp32 variant)
  uint16_t* out16;   // reduced gradient rounded to bf16 (bf16 variant)
  int64_t lo, hi;
  float inv;         // static unscale factor
  double inv_base;   // Nd or 1, for the dynamic loss scale
  int Nd;
  Header* hdr;
  Partial* part;
  int mode;
  int vec;
};

// bf16 round trip of a reduced gradient value (nearest even), as the bf16 variant keeps it.
__device__ __forceinline__ float round_bf16(float x) { return __uint_as_float((uint32_t)to_bf16(x) << 16); }

// OUT16: keep the reduced gradient as bf16; the flag and the norm then use the rounded value.
template <int DT, bool OUT16>
__global__ void __launch_bounds__(kThreads) reduce_scatter_kernel(const __grid_constant__ RsArgs a) {
  __shared__ float s_inv;
  if (threadIdx.x == 0) {
    s_inv = a.inv;
    if (__ldcg(&a.hdr->dyn))
      s_inv = __double2float_rn(__ddiv_rn(1.0, __dmul_rn(a.inv_base, __ldcg(&a.hdr->scale))));
  }
  __syncthreads();
  const float inv = s_inv;
  double sq = 0.0;
  int bad = 0;
  float* __restrict__ out = a.out;
  const Span sp8(a.lo, a.hi, a.vec);
  const int64_t stride = (int64_t)gridDim.x * kThreads;
  for (int64_t j = (int64_t)blockIdx.x * kThreads + threadIdx.x; j < sp8.nvec; j += stride) {
    const int64_t i = sp8.vlo + (j << 3);
    float s[8];
    fan_in8<DT>(a.grads, a.Nd, i, s);
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      s[k] = __fmul_rn(s[k], inv);
      if (OUT16) s[k] = round_bf16(s[k]);
      bad |= nonfinite(s[k]);
      sq = __dadd_rn(sq, __dmul_rn((double)s[k], (double)s[k]));
    }
    if (OUT16) {
      st_stream(a.out16 + i, pack_bf16x8(s));  // exact: the values are already bf16
    } else {
      st_stream(out + i, make_float4(s[0], s[1], s[2], s[3]));
      st_stream(out + i + 4, make_float4(s[4], s[5], s[6], s[7]));
    }
  }
  for (int64_t e = (int64_t)blockIdx.x * kThreads + threadIdx.x; e < sp8.nrest; e += stride) {
    const int64_t i = sp8.scalar_index(a.lo, e);
    float g = __fmul_rn(fan_in1<DT>(a.grads, a.Nd, i), inv);
    if (OUT16) g = round_bf16(g);
    bad |= nonfinite(g);
    sq = __dadd_rn(sq, __dmul_rn((double)g, (double)g));
    if (OUT16)
      a.out16[i] = to_bf16(g);
    else
      out[i] = g;
  }
  block_finish(sq, bad, a.hdr, a.part, a.mode);
}

// ------------------------------------------------------------------ K4: gated Adam (+ cast / AG)

struct AdamArgs {
  float* p[2];        // state copies; the kernel updates copy `live` in place
  float* m[2];
  float* v[2];
  const float* g;     // reduced gradient (fp32 variant)
  const uint16_t* g16;  // reduced gradient kept as bf16 (bf16 variant)
  uint16_t* out16;    // optional bf16 copy of the new weights (ZeRO-3 shard)
  uint16_t* reps[kMaxNd];  // optional bf16 replicas (fused all-gather of the two-pass path)
  int nrep;
  int use_live;       // 0: always copy 0
  int64_t lo, hi;
  Consts c;
  Header* hdr;
  Partial* part;
  int mode;
  int vec;
};

template <bool G16>
__global__ void __launch_bounds__(kThreads) adam_kernel(const __grid_constant__ AdamArgs a) {
  __shared__ Bias s_bias;
  __shared__ int s_live, s_skip;
  __shared__ float s_coef;
  if (threadIdx.x == 0) {
    s_bias = bias_for(a.c, __ldcg(&a.hdr->t) + 1);
    s_live = a.use_live ? (__ldcg(&a.hdr->live) & 1) : 0;
    s_skip = __ldcg(&a.hdr->pending_flag);
    s_coef = clip_coef(a.c.max_norm, __ldcg(&a.hdr->pending_sumsq));
  }
  __syncthreads();
  if (!s_skip) {
    const Bias b = s_bias;
    const float coef = s_coef;  // 1 unless the step's gradient norm is clipped
    float* __restrict__ P_ = a.p[s_live];
    float* __restrict__ M_ = a.m[s_live];
    float* __restrict__ V_ = a.v[s_live];
    const float* __restrict__ G_ = a.g;
    const Span sp8(a.lo, a.hi, a.vec);
    const int64_t stride = (int64_t)gridDim.x * kThreads;
    for (int64_t j = (int64_t)blockIdx.x * kThreads + threadIdx.x; j < sp8.nvec; j += stride) {
      const int64_t i = sp8.vlo + (j << 3);
      float P[8], M[8], V[8], G[8];
      unpack(ld_stream(P_ + i), ld_stream(P_ + i + 4), P);
      unpack(ld_stream(M_ + i), ld_stream(M_ + i + 4), M);
      unpack(ld_stream(V_ + i), ld_stream(V_ + i + 4), V);
      if (G16) {
        const uint4 q = ld_stream(a.g16 + i);
        const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          G[2 * k] = __uint_as_float(w[k] << 16);
          G[2 * k + 1] = __uint_as_float(w[k] & 0xffff0000u);
        }
      } else {
        unpack(ld_stream(G_ + i), ld_stream(G_ + i + 4), G);
      }
#pragma unroll
      for (int k = 0; k < 8; ++k) adam_elem(__fmul_rn(G[k], coef), P[k], M[k], V[k], a.c, b);
      st_stream(P_ + i, make_float4(P[0], P[1], P[2], P[3]));
      st_stream(P_ + i + 4, make_float4(P[4], P[5], P[6], P[7]));
      st_stream(M_ + i, make_float4(M[0], M[1], M[2], M[3]));
      st_stream(M_ + i + 4, make_float4(M[4], M[5], M[6], M[7]));
      st_stream(V_ + i, make_float4(V[0], V[1], V[2], V[3]));
      st_stream(V_ + i + 4, make_float4(V[4], V[5], V[6], V[7]));
      if (a.out16 || a.nrep) {
        const uint4 w = pack_bf16x8(P);
        if (a.out16) st_stream(a.out16 + i, w);
        for (int r = 0; r < a.nrep; ++r) st_stream(a.reps[r] + i, w);
      }
    }
    for (int64_t e = (int64_t)blockIdx.x * kThreads + threadIdx.x; e < sp8.nrest; e += stride) {
      const int64_t i = sp8.scalar_index(a.lo, e);
      float P = P_[i], M = M_[i], V = V_[i];
      const float gi = G16 ? __uint_as_float((uint32_t)a.g16[i] << 16) : G_[i];
      adam_elem(__fmul_rn(gi, coef), P, M, V, a.c, b);
      P_[i] = P;
      M_[i] = M;
      V_[i] = V;
      const uint16_t w = to_bf16(P);
      if (a.out16) a.out16[i] = w;
      for (int r = 0; r < a.nrep; ++r) a.reps[r][i] = w;
    }
  }
  block_finish(0.0, 0, a.hdr, a.part, a.mode);
}

// ------------------------------------------------------------------ K5: cast + all-gather

enum : int {
  kGateAlways = 0,
  kGateNoOverflow = 1,  // skip if the step in progress has overflowed
  kGateRepair = 2,      // run only if the last finished step overflowed; source = copy `live`
};

struct CastArgs {
  const float* src[2];
  uint16_t* reps[kMaxNd];
  int nrep;
  int gate;
  int64_t lo, hi;
  const Header* hdr;
  int vec;
  int unused;
};

// The overflow repair after a fused step may be launched as a programmatic dependent of the last
// fused launch: it waits for that grid (its header and replica writes) before anything else.  It
// then lets its own dependents launch at once: the only launches that follow it as programmatic
// dependents are the first fused launch of a next step, which waits at its start, so their
// launch overlaps this kernel without reading or writing anything before it has completed.
__global__ void __launch_bounds__(kThreads) cast_allgather_kernel(const __grid_constant__ CastArgs a) {
  __shared__ int s_run, s_live;
  pdl_wait();
  pdl_launch_dependents();
  if (threadIdx.x == 0) {
    int run = 1, live = 0;
    if (a.gate == kGateNoOverflow) run = !__ldcg(&a.hdr->pending_flag);
    if (a.gate == kGateRepair) {
      run = __ldcg(&a.hdr->last_flag);
      live = __ldcg(&a.hdr->live) & 1;
    }
    s_run = run;
    s_live = live;
  }
  __syncthreads();
  if (!s_run) return;
  const float* __restrict__ src = a.src[s_live];
  const Span sp8(a.lo, a.hi, a.vec);
  const int64_t stride = (int64_t)gridDim.x * kThreads;
  for (int64_t j = (int64_t)blockIdx.x * kThreads + threadIdx.x; j < sp8.nvec; j += stride) {
    const int64_t i = sp8.vlo + (j << 3);
    float P[8];
    unpack(ld_stream(src + i), ld_stream(src + i + 4), P);
    const uint4 w = pack_bf16x8(P);
    for (int r = 0; r < a.nrep; ++r) st_stream(a.reps[r] + i, w);
  }
  for (int64_t e = (int64_t)blockIdx.x * kThreads + threadIdx.x; e < sp8.nrest; e += stride) {
    const int64_t i = sp8.scalar_index(a.lo, e);
    const uint16_t w = to_bf16(src[i]);
    for (int r = 0; r < a.nrep; ++r) a.reps[r][i] = w;
  }
}

// ------------------------------------------------------------------ K2: ZeRO-3 layer gather

struct GatherArgs {
  const uint16_t* shards[kMaxNd];
  uint16_t* out[kMaxNd];
  int Nd, nout;
  int64_t L, S;
  int vec;  // S % 8 == 0 and every pointer 16-byte aligned
  int unused;
};

// grid.y = source rank r; grid.x strides over the shard.  out[o][r*S + k] = shards[r][k].
__global__ void __launch_bounds__(kThreads) gather_layer_kernel(const __grid_constant__ GatherArgs a) {
  const int r = blockIdx.y;
  const int64_t base = (int64_t)r * a.S;
  int64_t len = a.L - base;  // real elements in shard r
  if (len > a.S) len = a.S;
  if (len <= 0) return;
  const uint16_t* __restrict__ src = a.shards[r];
  const int64_t stride = (int64_t)gridDim.x * kThreads;
  if (a.vec) {
    const int64_t nvec = len >> 3;
    for (int64_t j = (int64_t)blockIdx.x * kThreads + threadIdx.x; j < nvec; j += stride) {
      const uint4 w = ld_stream(src + (j << 3));
      for (int o = 0; o < a.nout; ++o) st_stream(a.out[o] + base + (j << 3), w);
    }
    const int64_t rest = len - (nvec << 3);
    for (int64_t e = (int64_t)blockIdx.x * kThreads + threadIdx.x; e < rest; e += stride) {
      const int64_t k = (nvec << 3) + e;
      const uint16_t w = src[k];
      for (int o = 0; o < a.nout; ++o) a.out[o][base + k] = w;
    }
  } else {
    for (int64_t k = (int64_t)blockIdx.x * kThreads + threadIdx.x; k < len; k += stride) {
      const uint16_t w = src[k];
      for (int o = 0; o < a.nout; ++o) a.out[o][base + k] = w;
    }
  }
}

// ------------------------------------------------------------------ workspace control

enum : int { kWsInit = 0, kWsBegin = 1, kWsEnd = 2, kWsEndFlip = 3 };

__global__ void ws_ctl_kernel(Header* h, int op, long long t0) {
  if (threadIdx.x != 0 || blockIdx.x != 0) return;
  if (op == kWsInit) {
    h->done = 0u;
    h->t = t0;
    h->skipped = 0;
    h->live = 0;
    h->last_flag = 0;
    h->last_sumsq = 0.0;
    h->error = 0;
    h->dyn = 0;
    h->scale = 1.0;
    h->growth = 1.0;
    h->backoff = 1.0;
    h->interval = 1;
    h->good = 0;
    h->chunk = 0ull;
  }
  if (op == kWsInit || op == kWsBegin) {
    h->pending_flag = 0;
    h->pending_sumsq = 0.0;
  }
  if (op == kWsEnd || op == kWsEndFlip) end_step(*h, op == kWsEndFlip);
  __threadfence();
}

// Turns on dynamic loss scaling in the workspace.
__global__ void scaler_init_kernel(Header* h, double scale, double growth, double backoff, long long interval) {
  if (threadIdx.x != 0 || blockIdx.x != 0) return;
  h->dyn = 1;
  h->scale = scale;
  h->growth = growth;
  h->backoff = backoff;
  h->interval = interval;
  h->good = 0;
  __threadfence();
}

}  // namespace zb
