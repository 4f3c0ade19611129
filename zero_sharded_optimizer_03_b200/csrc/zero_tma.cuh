// zero_tma.cuh -- TMA-pipelined fused ZeRO step (reduce-scatter + Adam + all-gather) for sm_100a.
//
// Same arithmetic as fused_step_kernel (zero_kernels.cuh), bit for bit; different data movement.
// The register kernel keeps every load in registers, which caps the bytes in flight per SM at
// what the register file holds (about 64-115 KB at 16 warps per SM) and hurts most when the
// gradient fan-in is wide (Nd = 16, 64).  Here the Tensor Memory Accelerator moves the data:
//
//   producer (1 warp)    : 1-D bulk copies (cp.async.bulk) global -> shared of every load unit
//                          into a ring of input stages; completion counted on the stage's "full"
//                          mbarrier (expect_tx bytes)
//   consumers (8 warps)  : one 8-element vector per thread per tile; sum the replicas in rank
//                          order from shared memory into registers and release each input stage
//                          as soon as it has been read; for the state unit, the Adam update, then
//                          the new fp32 state and the bf16 weights go into an output buffer
//   storer (1 warp)      : bulk copies shared -> global of the output buffer: the three state
//                          streams, and the one bf16 tile to every one of the Nd weight replicas
//                          (the all-gather is a TMA fan-out of one shared tile)
//
// A tile is kTile elements; its load units are ceil(Nd/8) gradient chunks of up to 8 replicas
// (8 x 4 KB) followed by the state unit (master, m, v: 3 x 8 KB).  Units stream through
// kStages input stages of 32 KB; results go through kOutBufs output buffers of 28 KB, so the
// time stores take to drain never holds an input stage.  One CTA per SM, 216 KB of shared
// memory; up to ~160 KB of loads per SM are in flight whatever Nd is, while the per-element
// rank-order sums stay in registers across the chunks of a tile.  Elements outside whole tiles
// (a ragged head or tail) are done by the consumers with plain loads and stores.
//
// Every mbarrier wait is bounded (kWaitTimeoutNs on %globaltimer).  A wait that runs out sets a
// CTA-wide abort flag; all roles leave their loops (consumers together, through a barrier
// reduction), loads already issued are waited for (again bounded), bulk stores are drained, the
// workspace error word is set, and the step is reported as overflowed so that it is skipped.
#pragma once

#include "zero_kernels.cuh"

namespace zb {

constexpr int kTile = 2048;       // elements per tile
constexpr int kChunkRanks = 8;    // gradient replicas per load unit
constexpr int kStages = 5;        // input stages
constexpr int kStageBytes = 32768;
constexpr int kOutBufs = 2;       // output buffers
constexpr int kOutBytes = 28672;  // master, m, v (fp32) + bf16 weights of one tile
constexpr int kConsumerWarps = 8;
constexpr int kConsumers = kConsumerWarps * 32;  // 256 threads x 8 elements = one tile
constexpr int kTmaThreads = kConsumers + 64;     // + producer warp + storer warp
constexpr int kTmaWarps = kTmaThreads / 32;
constexpr int kProducerWarp = kConsumerWarps;
constexpr int kStorerWarp = kConsumerWarps + 1;
constexpr size_t kOutOffset = (size_t)kStages * kStageBytes;
constexpr size_t kBarOffset = kOutOffset + (size_t)kOutBufs * kOutBytes;
constexpr int kNumBars = 2 * kStages + 2 * kOutBufs;
constexpr size_t kTmaSmemBytes = kBarOffset + kNumBars * sizeof(uint64_t);
constexpr unsigned long long kWaitTimeoutNs = 1000000000ull;  // 1 s

// state unit layout inside an input stage, and output buffer layout: master, m, v, bf16 weights
constexpr int kOffP = 0;
constexpr int kOffM = kTile * 4;
constexpr int kOffV = 2 * kTile * 4;
constexpr int kOffW = 3 * kTile * 4;
static_assert(3 * kTile * 4 <= kStageBytes, "state unit fits a stage");
static_assert(kOffW + kTile * 2 <= kOutBytes, "results fit an output buffer");
static_assert(kChunkRanks * kTile * 2 <= kStageBytes, "gradient chunk fits a stage");
static_assert(kConsumers * 8 == kTile, "one 8-element vector per consumer thread");
static_assert(kOutOffset % 128 == 0 && kOutBytes % 128 == 0, "output buffers 128-byte aligned");
static_assert(kTmaSmemBytes + 512 <= 227 * 1024, "shared memory per CTA");

enum : int { kErrTimeout = 1 };

// ------------------------------------------------------------------ PTX wrappers

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n"
      " .reg .pred p;\n"
      " mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n"
      "}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ unsigned long long global_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
// 1-D bulk copy global -> shared, completion reported to `bar` (bytes and addresses 16-aligned)
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "l"(src), "r"(bytes), "r"(bar)
               : "memory");
}
// 1-D bulk copy shared -> global (bulk async-group completion)
__device__ __forceinline__ void bulk_store(void* dst, uint32_t src, uint32_t bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst), "r"(src), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read_all() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
__device__ __forceinline__ void fence_smem_to_async() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }
// barrier 1 over the consumer warps only
__device__ __forceinline__ void consumer_sync() { asm volatile("bar.sync 1, %0;" ::"n"(kConsumers) : "memory"); }
// barrier 1 over the consumer warps, returning the AND of `pred` over them
__device__ __forceinline__ int consumer_all(int pred) {
  int r;
  asm volatile(
      "{\n"
      " .reg .pred p, q;\n"
      " setp.ne.s32 p, %1, 0;\n"
      " bar.red.and.pred q, 1, %2, p;\n"
      " selp.s32 %0, 1, 0, q;\n"
      "}\n"
      : "=r"(r)
      : "r"(pred), "n"(kConsumers)
      : "memory");
  return r;
}

// Waits for the phase of parity `parity` to complete.  Returns false when *abort is set or when
// the wait exceeds kWaitTimeoutNs (then it sets *abort itself).
__device__ __forceinline__ bool wait_bounded(uint32_t bar, uint32_t parity, volatile int* abort) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = global_ns();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort) return false;
    if (global_ns() - t0 > kWaitTimeoutNs) {
      *abort = 1;
      return false;
    }
  }
}

// Bounded wait that ignores the abort flag (draining copies already issued).
__device__ __forceinline__ void wait_drain(uint32_t bar, uint32_t parity) {
  const unsigned long long t0 = global_ns();
  while (!mbar_try_wait(bar, parity) && global_ns() - t0 < kWaitTimeoutNs) {
  }
}

// ------------------------------------------------------------------ kernel

struct TmaArgs {
  const uint16_t* grads[kMaxNd];
  uint16_t* reps[kMaxNd];
  float* p[2];
  float* m[2];
  float* v[2];
  int64_t lo, hi;    // window of global indices
  int64_t tiles_lo;  // first element of tile 0 (a multiple of 8, >= lo)
  int64_t ntiles;    // whole tiles in [tiles_lo, hi)
  Consts c;
  Header* hdr;
  Partial* part;
  int Nd;
  int mode;
  int trigger_late;    // 1: a dependent launch may start only once this CTA's tiles are done
  int unused;
  int64_t stall_unit;  // test hook: CTA 0 issues no copies for this load unit (-1: none)
};

template <int DT>
__global__ void __launch_bounds__(kTmaThreads, 1) fused_step_tma_kernel(const __grid_constant__ TmaArgs a) {
  extern __shared__ __align__(128) unsigned char smem[];
  unsigned char* outbuf = smem + kOutOffset;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kBarOffset);
  __shared__ Bias s_bias;
  __shared__ int s_live;
  __shared__ float s_inv;
  __shared__ volatile int s_abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    s_bias = bias_for(a.c, __ldcg(&a.hdr->t) + 1);
    s_live = __ldcg(&a.hdr->live) & 1;
    s_inv = step_inv(a.c, a.hdr);
    s_abort = (smem_u32(smem) & 127u) ? 1 : 0;  // bulk copies need aligned buffers: never start misaligned
    for (int k = 0; k < kNumBars; ++k) mbar_init(smem_u32(&bars[k]), 1);
    fence_barrier_init();
  }
  __syncthreads();
  if (!a.trigger_late) pdl_launch_dependents();  // a later bucket may take each SM as soon as this CTA leaves it
  const Bias b = s_bias;
  const int live = s_live;
  const float inv = s_inv;
  // full[s]: loads landed; empty[s]: consumers done with input stage s;
  // out_full[o]: results written to output buffer o; out_free[o]: its stores have read it
  auto full_bar = [&](int s) { return smem_u32(&bars[s]); };
  auto empty_bar = [&](int s) { return smem_u32(&bars[kStages + s]); };
  auto out_full_bar = [&](int o) { return smem_u32(&bars[2 * kStages + o]); };
  auto out_free_bar = [&](int o) { return smem_u32(&bars[2 * kStages + kOutBufs + o]); };

  const int nchunks = (a.Nd + kChunkRanks - 1) / kChunkRanks;
  const int per_tile = nchunks + 1;  // gradient chunks, then the state unit
  const int64_t my_tiles =
      a.ntiles > (int64_t)blockIdx.x ? (a.ntiles - 1 - (int64_t)blockIdx.x) / gridDim.x + 1 : 0;
  const int64_t my_units = my_tiles * per_tile;

  double sq = 0.0;
  int bad = 0;
  int64_t issued = 0;  // load units the producer has issued (drained on abort)

  if (warp == kProducerWarp) {
    // the whole warp walks the units (and agrees on leaving); lane 0 issues the copies
    for (int64_t u = 0; u < my_units; ++u) {
      const int s = (int)(u % kStages);
      const uint32_t ph = (uint32_t)((u / kStages) & 1);
      if (__any_sync(0xffffffffu, s_abort)) break;
      if (!__all_sync(0xffffffffu, wait_bounded(empty_bar(s), ph ^ 1u, &s_abort))) break;
      const bool stall = blockIdx.x == 0 && u == a.stall_unit;  // nothing will complete this unit
      if (lane == 0 && !stall) {
        const int64_t tile = (int64_t)blockIdx.x + (u / per_tile) * gridDim.x;
        const int j = (int)(u % per_tile);
        const int64_t i0 = a.tiles_lo + tile * kTile;
        unsigned char* st = smem + (size_t)s * kStageBytes;
        if (j < nchunks) {
          const int r0 = j * kChunkRanks;
          const int nr = a.Nd - r0 < kChunkRanks ? a.Nd - r0 : kChunkRanks;
          mbar_expect_tx(full_bar(s), (uint32_t)(nr * kTile * 2));
          for (int q = 0; q < nr; ++q)
            bulk_load(smem_u32(st + q * kTile * 2), a.grads[r0 + q] + i0, kTile * 2, full_bar(s));
        } else {
          mbar_expect_tx(full_bar(s), 3u * kTile * 4);
          bulk_load(smem_u32(st + kOffP), a.p[live] + i0, kTile * 4, full_bar(s));
          bulk_load(smem_u32(st + kOffM), a.m[live] + i0, kTile * 4, full_bar(s));
          bulk_load(smem_u32(st + kOffV), a.v[live] + i0, kTile * 4, full_bar(s));
        }
      }
      __syncwarp();
      issued = u + 1;
    }
  } else if (warp == kStorerWarp) {
    for (int64_t n = 0; n < my_tiles; ++n) {
      const int o = (int)(n % kOutBufs);
      const uint32_t ph = (uint32_t)((n / kOutBufs) & 1);
      if (!__all_sync(0xffffffffu, wait_bounded(out_full_bar(o), ph, &s_abort))) break;
      if (lane == 0) {
        const int64_t tile = (int64_t)blockIdx.x + n * gridDim.x;
        const int64_t i0 = a.tiles_lo + tile * kTile;
        const unsigned char* ob = outbuf + (size_t)o * kOutBytes;
        bulk_store(a.p[live ^ 1] + i0, smem_u32(ob + kOffP), kTile * 4);
        bulk_store(a.m[live ^ 1] + i0, smem_u32(ob + kOffM), kTile * 4);
        bulk_store(a.v[live ^ 1] + i0, smem_u32(ob + kOffV), kTile * 4);
        for (int r = 0; r < a.Nd; ++r) bulk_store(a.reps[r] + i0, smem_u32(ob + kOffW), kTile * 2);
        bulk_commit();
        bulk_wait_read_all();  // the buffer may be rewritten once the stores have read it
        mbar_arrive(out_free_bar(o));
      }
      __syncwarp();
    }
    if (lane == 0) bulk_wait_all();
    __syncwarp();
  } else {
    const int t = threadIdx.x;  // 0 .. kConsumers-1
    float acc[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) acc[k] = 0.0f;
    int64_t n = 0;  // tiles finished by this CTA
    for (int64_t u = 0; u < my_units; ++u) {
      const int s = (int)(u % kStages);
      const uint32_t ph = (uint32_t)((u / kStages) & 1);
      const int ok = wait_bounded(full_bar(s), ph, &s_abort);
      if (!consumer_all(ok)) {
        bad = 1;
        break;
      }
      const int j = (int)(u % per_tile);
      const unsigned char* st = smem + (size_t)s * kStageBytes;
      if (j == 0) {
#pragma unroll
        for (int k = 0; k < 8; ++k) acc[k] = 0.0f;
      }
      if (j < nchunks) {
        const int r0 = j * kChunkRanks;
        const int nr = a.Nd - r0 < kChunkRanks ? a.Nd - r0 : kChunkRanks;
        for (int q = 0; q < nr; ++q)
          add8<DT>(acc, *reinterpret_cast<const uint4*>(st + q * kTile * 2 + t * 16));
        consumer_sync();  // every consumer is done reading the stage
        if (t == 0) mbar_arrive(empty_bar(s));
        continue;
      }
      float P[8], M[8], V[8];
      {
        const float4* sp4 = reinterpret_cast<const float4*>(st + kOffP + t * 32);
        const float4* sm4 = reinterpret_cast<const float4*>(st + kOffM + t * 32);
        const float4* sv4 = reinterpret_cast<const float4*>(st + kOffV + t * 32);
        unpack(sp4[0], sp4[1], P);
        unpack(sm4[0], sm4[1], M);
        unpack(sv4[0], sv4[1], V);
      }
      consumer_sync();  // the input stage has been read: hand it back to the producer
      if (t == 0) mbar_arrive(empty_bar(s));
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const float g = __fmul_rn(acc[k], inv);
        bad |= nonfinite(g);
        sq = __dadd_rn(sq, __dmul_rn((double)g, (double)g));
        adam_elem(g, P[k], M[k], V[k], a.c, b);
      }
      const int o = (int)(n % kOutBufs);
      const uint32_t oph = (uint32_t)((n / kOutBufs) & 1);
      const int ok2 = wait_bounded(out_free_bar(o), oph ^ 1u, &s_abort);
      if (!consumer_all(ok2)) {
        bad = 1;
        break;
      }
      unsigned char* ob = outbuf + (size_t)o * kOutBytes;
      float4* op4 = reinterpret_cast<float4*>(ob + kOffP + t * 32);
      float4* om4 = reinterpret_cast<float4*>(ob + kOffM + t * 32);
      float4* ov4 = reinterpret_cast<float4*>(ob + kOffV + t * 32);
      op4[0] = make_float4(P[0], P[1], P[2], P[3]);
      op4[1] = make_float4(P[4], P[5], P[6], P[7]);
      om4[0] = make_float4(M[0], M[1], M[2], M[3]);
      om4[1] = make_float4(M[4], M[5], M[6], M[7]);
      ov4[0] = make_float4(V[0], V[1], V[2], V[3]);
      ov4[1] = make_float4(V[4], V[5], V[6], V[7]);
      *reinterpret_cast<uint4*>(ob + kOffW + t * 16) = pack_bf16x8(P);
      fence_smem_to_async();  // make the generic-proxy writes visible to the bulk stores
      consumer_sync();
      if (t == 0) mbar_arrive(out_full_bar(o));
      ++n;
    }
    if (!s_abort) {
      // elements outside whole tiles: [lo, tiles_lo) and [tiles_lo + ntiles * kTile, hi)
      const float* __restrict__ sp = a.p[live];
      const float* __restrict__ sm = a.m[live];
      const float* __restrict__ sv = a.v[live];
      float* __restrict__ dp = a.p[live ^ 1];
      float* __restrict__ dm = a.m[live ^ 1];
      float* __restrict__ dv = a.v[live ^ 1];
      const int64_t tail_lo = a.tiles_lo + a.ntiles * kTile;
      const int64_t nhead = a.tiles_lo - a.lo;
      const int64_t nrest = nhead + (a.hi - tail_lo);
      for (int64_t e = (int64_t)blockIdx.x * kConsumers + t; e < nrest; e += (int64_t)gridDim.x * kConsumers) {
        const int64_t i = e < nhead ? a.lo + e : tail_lo + (e - nhead);
        const float g = __fmul_rn(fan_in1<DT>(a.grads, a.Nd, i), inv);
        bad |= nonfinite(g);
        sq = __dadd_rn(sq, __dmul_rn((double)g, (double)g));
        float P = sp[i], M = sm[i], V = sv[i];
        adam_elem(g, P, M, V, a.c, b);
        dp[i] = P;
        dm[i] = M;
        dv[i] = V;
        const uint16_t w = to_bf16(P);
        for (int r = 0; r < a.Nd; ++r) a.reps[r][i] = w;
      }
    }
  }
  __syncthreads();
  if (s_abort) {
    bad = 1;  // an aborted launch never commits: the step is reported as overflowed
    if (threadIdx.x == 0) atomicOr(&a.hdr->error, kErrTimeout);
    if (warp == kProducerWarp && lane == 0) {
      // let the copies already issued land before the CTA's shared memory goes away; the
      // last kStages issued units are the only ones that can still be in flight
      const int64_t first = issued > kStages ? issued - kStages : 0;
      for (int64_t u = first; u < issued; ++u)
        wait_drain(full_bar((int)(u % kStages)), (uint32_t)((u / kStages) & 1));
    }
  }
  if (a.trigger_late) pdl_launch_dependents();
  pdl_wait();  // a programmatic dependent: the previous bucket has completed
  block_finish<kTmaWarps>(sq, bad, a.hdr, a.part, a.mode);
}

}  // namespace zb

namespace zb {

// ------------------------------------------------------------------ TMA ZeRO-3 layer gather
//
// The gather is a pure fan-out copy: 2 bytes read and 2*nout written per element.  Issued as
// 16-byte stores from registers it saturates the load/store units (lg_throttle stalls) before
// DRAM; here one thread per CTA drives the Tensor Memory Accelerator instead: a 1-D bulk load of
// a chunk of the source shard into shared memory (the next chunk prefetched while the current
// one is stored), then nout bulk stores of that one shared tile.  A stage is refilled only once
// the stores that read it have finished reading (bulk async-group accounting).  Waits are
// bounded as in the fused kernel; a timeout sets the workspace error word.

constexpr int kGTile = 4096;   // elements per chunk (8 KB)
constexpr int kGStages = 4;
constexpr size_t kGSmemBytes = (size_t)kGStages * kGTile * 2 + kGStages * sizeof(uint64_t);

struct GatherTmaArgs {
  const uint16_t* shards[kMaxNd];
  uint16_t* out[kMaxNd];
  int Nd, nout;
  int64_t L, S;
  Header* hdr;  // error word
};

__device__ __forceinline__ void bulk_wait_read_2() { asm volatile("cp.async.bulk.wait_group.read 2;" ::: "memory"); }

// grid.y = source rank r, grid.x strides over the chunks of shard r; 32 threads per CTA.
__global__ void __launch_bounds__(32) gather_layer_tma_kernel(const __grid_constant__ GatherTmaArgs a) {
  extern __shared__ __align__(128) unsigned char smem[];
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + (size_t)kGStages * kGTile * 2);
  const int r = blockIdx.y;
  const int64_t base = (int64_t)r * a.S;
  int64_t len = a.L - base;
  if (len > a.S) len = a.S;
  if (len <= 0) return;
  const int64_t len8 = len & ~int64_t(7);  // bulk part (multiples of 16 bytes)
  const int64_t nchunks = (len8 + kGTile - 1) / kGTile;
  const int64_t mine = nchunks > (int64_t)blockIdx.x ? (nchunks - 1 - (int64_t)blockIdx.x) / gridDim.x + 1 : 0;
  const uint16_t* src = a.shards[r];
  if (threadIdx.x == 0 && mine > 0 && (smem_u32(smem) & 127u) == 0) {
    for (int k = 0; k < kGStages; ++k) mbar_init(smem_u32(&bars[k]), 1);
    fence_barrier_init();
    auto chunk = [&](int64_t it, int64_t* k0, uint32_t* bytes) {
      *k0 = ((int64_t)blockIdx.x + it * gridDim.x) * kGTile;
      const int64_t n = len8 - *k0 < kGTile ? len8 - *k0 : kGTile;
      *bytes = (uint32_t)(n * 2);
    };
    auto load = [&](int64_t it) {
      int64_t k0;
      uint32_t bytes;
      chunk(it, &k0, &bytes);
      const int s = (int)(it % kGStages);
      mbar_expect_tx(smem_u32(&bars[s]), bytes);
      bulk_load(smem_u32(smem + (size_t)s * kGTile * 2), src + k0, bytes, smem_u32(&bars[s]));
    };
    volatile int abort = 0;
    int64_t issued = 1;
    load(0);
    for (int64_t it = 0; it < mine; ++it) {
      if (it + 1 < mine) {
        bulk_wait_read_2();  // the stage chunk it+1 will use was last read by the stores of it-3
        load(it + 1);
        issued = it + 2;
      }
      const int s = (int)(it % kGStages);
      if (!wait_bounded(smem_u32(&bars[s]), (uint32_t)((it / kGStages) & 1), &abort)) break;
      int64_t k0;
      uint32_t bytes;
      chunk(it, &k0, &bytes);
      for (int o = 0; o < a.nout; ++o) bulk_store(a.out[o] + base + k0, smem_u32(smem + (size_t)s * kGTile * 2), bytes);
      bulk_commit();
    }
    bulk_wait_all();
    if (abort) {
      atomicOr(&a.hdr->error, kErrTimeout);
      for (int64_t it = issued > 2 ? issued - 2 : 0; it < issued; ++it)  // loads still in flight
        wait_drain(smem_u32(&bars[it % kGStages]), (uint32_t)((it / kGStages) & 1));
    }
  } else if (threadIdx.x == 0 && mine > 0) {
    atomicOr(&a.hdr->error, kErrTimeout);  // misaligned shared memory: nothing copied
  }
  __syncwarp();
  if (blockIdx.x == 0)  // the last < 8 elements of the shard
    for (int64_t k = len8 + threadIdx.x; k < len; k += 32) {
      const uint16_t w = src[k];
      for (int o = 0; o < a.nout; ++o) a.out[o][base + k] = w;
    }
}

}  // namespace zb
