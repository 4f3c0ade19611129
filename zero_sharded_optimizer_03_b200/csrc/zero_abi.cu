// zero_abi.cu -- host side of the C ABI declared in include/zero.h.
//
// Validates arguments, derives the element-independent scalars, sizes persistent grids to
// the GPU, and enqueues the kernels of zero_kernels.cuh on the caller's stream.  It never
// allocates memory and never synchronizes except in zero_read_result.
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>

#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <vector>

#include "zero.h"
#include "zero_kernels.cuh"
#include "zero_tma.cuh"

namespace {

thread_local char g_err[512] = "";

int fail(int code, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof g_err, fmt, ap);
  va_end(ap);
  return code;
}

int cuda_fail(cudaError_t e, const char* what) {
  return fail(ZERO_ECUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// The kernels read and update the workspace's doubles and 64-bit counters in place: a NULL
// workspace, or one off a 16-byte boundary, is rejected before anything is launched.
int check_ws(const void* ws) {
  if (!ws) return fail(ZERO_EINVAL, "workspace is NULL");
  if (!aligned16(ws)) return fail(ZERO_EINVAL, "workspace %p is not 16-byte aligned", ws);
  return ZERO_OK;
}

// Resident CTAs per SM for each kernel, cached per device (occupancy does not change).
constexpr int kMaxDevices = 64;
enum KernelId {
  kRsBf16, kRsFp16, kRsBf16Out16, kRsFp16Out16, kAdam, kAdamG16, kCast, kGather,
  kFusedBase,  // 16 fused-kernel variants: (gather, rank batch 1/2/4/8, gradient dtype)
  kNumKernels = kFusedBase + 16
};

// Occupancy id of fused_step_kernel<DT, CH, G>.
constexpr int ch_index(int CH) { return CH == 1 ? 0 : CH == 2 ? 1 : CH == 4 ? 2 : 3; }
constexpr int fused_kid(int DT, int CH, bool G) { return kFusedBase + (G ? 8 : 0) + 2 * ch_index(CH) + DT; }

template <int DT, int CH, bool G>
const void* fused_ptr() {
  return reinterpret_cast<const void*>(&zb::fused_step_kernel<DT, CH, G>);
}

const void* kernel_ptr(int id) {
  if (id >= kFusedBase) {
    static const void* const table[16] = {
        fused_ptr<0, 1, false>(), fused_ptr<1, 1, false>(), fused_ptr<0, 2, false>(), fused_ptr<1, 2, false>(),
        fused_ptr<0, 4, false>(), fused_ptr<1, 4, false>(), fused_ptr<0, 8, false>(), fused_ptr<1, 8, false>(),
        fused_ptr<0, 1, true>(),  fused_ptr<1, 1, true>(),  fused_ptr<0, 2, true>(),  fused_ptr<1, 2, true>(),
        fused_ptr<0, 4, true>(),  fused_ptr<1, 4, true>(),  fused_ptr<0, 8, true>(),  fused_ptr<1, 8, true>()};
    return table[id - kFusedBase];
  }
  switch (id) {
    case kRsBf16: return reinterpret_cast<const void*>(&zb::reduce_scatter_kernel<0, false>);
    case kRsFp16: return reinterpret_cast<const void*>(&zb::reduce_scatter_kernel<1, false>);
    case kRsBf16Out16: return reinterpret_cast<const void*>(&zb::reduce_scatter_kernel<0, true>);
    case kRsFp16Out16: return reinterpret_cast<const void*>(&zb::reduce_scatter_kernel<1, true>);
    case kAdam: return reinterpret_cast<const void*>(&zb::adam_kernel<false>);
    case kAdamG16: return reinterpret_cast<const void*>(&zb::adam_kernel<true>);
    case kCast: return reinterpret_cast<const void*>(&zb::cast_allgather_kernel);
    default: return reinterpret_cast<const void*>(&zb::gather_layer_kernel);
  }
}

struct DeviceInfo {
  int sms = 0;
  int per_sm[kNumKernels] = {};
  bool tma_ready = false;  // dynamic shared memory attribute set for the TMA kernels
  int gather_tma_per_sm = 0;
};
DeviceInfo g_dev[kMaxDevices];
std::mutex g_dev_mu;

// Grid for `work` units of one thread each: a grid-stride loop over at most `waves` full waves
// of resident CTAs (`waves` x SMs x CTAs per SM).  Several waves let the block scheduler hand
// the later CTAs to whichever SMs finish first, instead of every SM owning a fixed 1/148 of the
// data; measured on B200 (same-box sweeps of 1, 2, 4, 8 and 16 waves), that balancing is worth
// up to 20% for the in-place Adam kernel and 12% for the layer gather.  (The register fused
// kernel keeps one wave and balances with chunks instead, see use_chunks.)  Kernels that leave
// a per-CTA partial in the workspace are capped at kMaxCtas CTAs.
int grid_for(int kid, int64_t work, int* grid, int waves = 1, bool partials = true) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(ZERO_EINVAL, "device ordinal %d unsupported", dev);
  DeviceInfo& d = g_dev[dev];
  {
    std::lock_guard<std::mutex> lk(g_dev_mu);
    if (d.sms == 0) {
      e = cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev);
      if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute");
    }
    if (d.per_sm[kid] == 0) {
      int n = 0;
      e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel_ptr(kid), zb::kThreads, 0);
      if (e != cudaSuccess) return cuda_fail(e, "cudaOccupancyMaxActiveBlocksPerMultiprocessor");
      d.per_sm[kid] = n > 0 ? n : 1;
    }
  }
  int64_t need = (work + zb::kThreads - 1) / zb::kThreads;
  if (need < 1) need = 1;
  const int64_t wave = (int64_t)d.sms * d.per_sm[kid];
  int64_t cap = wave;
  // only long loops (>= 16 iterations per thread in one wave) are split into several waves: on
  // short ones a partial extra wave costs more than the balancing gains (1M elements: +13%)
  if (waves > 1 && need >= 16 * wave) cap = wave * waves;
  if (partials && cap > zb::kMaxCtas) cap = zb::kMaxCtas;
  if (cap > (int64_t)1 << 30) cap = (int64_t)1 << 30;
  *grid = (int)(need < cap ? need : cap);
  return ZERO_OK;
}

// Waves per kernel (see grid_for), from the same-box sweeps: reduce-scatter 4, in-place Adam 8,
// layer gather 16 (it has no partials).  The fused kernel balances its SMs with dynamically
// scheduled chunks instead (use_chunks), and the TMA kernel with waves of its own (tma_grid).
constexpr int kWavesRs = 4;
constexpr int kWavesAdam = 8;
constexpr int kWavesGather = 16;
constexpr int kWavesGatherTma = 32;

// Longest unbucketed register-path step whose overflow repair the fused kernel's last CTA does
// itself (zero_step); longer steps keep the repair launch, whose full grid repairs fast.
constexpr int64_t kSelfRepairMax = int64_t(1) << 21;

// Fused kernel over a long window: chunks handed out by the workspace counter, or the fixed
// grid-stride split.  Same-box sweeps at 2^25-2^28 elements, chunks against the best fixed grid:
// +15% at Nd = 1, +7% at Nd = 4 and, with batches of 4 replicas, +1.4% (124M) to +3.7% (2^28)
// at Nd = 8, +4% at Nd = 16, +2% at Nd = 64; -2% at Nd = 2 and with a single bf16 output
// (ZeRO-3 layers, nrep = 1 < Nd).
inline bool use_chunks(int Nd, int nrep) { return nrep == Nd && Nd != 2; }

// SM count of the current device, and the TMA kernels' shared-memory attribute set once.
int tma_setup(int* sms) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(ZERO_EINVAL, "device ordinal %d unsupported", dev);
  DeviceInfo& d = g_dev[dev];
  std::lock_guard<std::mutex> lk(g_dev_mu);
  if (d.sms == 0) {
    e = cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute");
  }
  if (!d.tma_ready) {
    e = cudaFuncSetAttribute(zb::fused_step_tma_kernel<0>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)zb::kTmaSmemBytes);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(zb::fused_step_tma_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)zb::kTmaSmemBytes);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(TMA shared memory)");
    e = cudaFuncSetAttribute(zb::gather_layer_tma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)zb::kGSmemBytes);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(TMA gather shared memory)");
    int n = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, zb::gather_layer_tma_kernel, 32, zb::kGSmemBytes);
    if (e != cudaSuccess) return cuda_fail(e, "cudaOccupancyMaxActiveBlocksPerMultiprocessor");
    d.gather_tma_per_sm = n > 0 ? n : 1;
    d.tma_ready = true;
  }
  *sms = d.sms;
  return ZERO_OK;
}

int gather_tma_per_sm() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 1;
  return g_dev[dev].gather_tma_per_sm > 0 ? g_dev[dev].gather_tma_per_sm : 1;
}

// An NVTX range over a scope (host timeline of a profiler: one range per step, per ZeRO-3
// layer, per offload chunk).  Without a profiler attached the calls return at once.
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

int check_launch(const char* what) {
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? ZERO_OK : cuda_fail(e, what);
}

zb::Header* header(void* ws) { return static_cast<zb::Header*>(ws); }
zb::Partial* partials(void* ws) {
  return reinterpret_cast<zb::Partial*>(static_cast<char*>(ws) + zb::kHeaderBytes);
}

int check_hp(const zero_hparams_t* hp) {
  if (!hp) return fail(ZERO_EINVAL, "hparams is NULL");
  if (!std::isfinite(hp->lr) || hp->lr < 0) return fail(ZERO_EINVAL, "lr must be finite and >= 0");
  if (!(hp->beta1 >= 0 && hp->beta1 < 1)) return fail(ZERO_EINVAL, "beta1 must be in [0, 1)");
  if (!(hp->beta2 >= 0 && hp->beta2 < 1)) return fail(ZERO_EINVAL, "beta2 must be in [0, 1)");
  if (!(hp->eps > 0) || !std::isfinite(hp->eps)) return fail(ZERO_EINVAL, "eps must be finite and > 0");
  if (!std::isfinite(hp->weight_decay)) return fail(ZERO_EINVAL, "weight_decay must be finite");
  if (!(hp->loss_scale > 0) || !std::isfinite(hp->loss_scale))
    return fail(ZERO_EINVAL, "loss_scale must be finite and > 0");
  if (!(hp->max_grad_norm >= 0) || !std::isfinite(hp->max_grad_norm))
    return fail(ZERO_EINVAL, "max_grad_norm must be finite and >= 0");
  return ZERO_OK;
}

zb::Consts make_consts(const zero_hparams_t* hp, int Nd) {
  zb::Consts c;
  const double denom = hp->grad_average ? (double)Nd * hp->loss_scale : hp->loss_scale;
  c.inv = (float)(1.0 / denom);
  c.b1 = (float)hp->beta1;
  c.b2 = (float)hp->beta2;
  c.omb1 = (float)(1.0 - hp->beta1);
  c.omb2 = (float)(1.0 - hp->beta2);
  c.eps = (float)hp->eps;
  c.decay = (float)(1.0 - hp->lr * hp->weight_decay);
  c.unused = 0.0f;
  c.lr = hp->lr;
  c.b1d = hp->beta1;
  c.b2d = hp->beta2;
  c.inv_base = hp->grad_average ? (double)Nd : 1.0;
  c.max_norm = hp->max_grad_norm;
  return c;
}

int check_nd(int Nd) {
  if (Nd < 1 || Nd > ZERO_MAX_ND) return fail(ZERO_EINVAL, "Nd=%d outside [1, %d]", Nd, ZERO_MAX_ND);
  return ZERO_OK;
}

int check_window(int64_t lo, int64_t hi) {
  if (lo < 0 || hi < lo) return fail(ZERO_EINVAL, "bad window [%lld, %lld)", (long long)lo, (long long)hi);
  return ZERO_OK;
}

template <typename T>
int check_ptrs(T* const* ptrs, int n, const char* what, bool* all_aligned) {
  if (!ptrs) return fail(ZERO_EINVAL, "%s array is NULL", what);
  for (int r = 0; r < n; ++r) {
    if (!ptrs[r]) return fail(ZERO_EINVAL, "%s[%d] is NULL", what, r);
    if (!aligned16(ptrs[r])) *all_aligned = false;
  }
  return ZERO_OK;
}

// Optional CUDA events recorded around the data-moving kernels of the next zero_step call
// on this thread (one-shot; see zero_profile_events).
thread_local int64_t g_test_stall = -1;  // zero_test_inject_stall (one-shot)
thread_local cudaEvent_t g_prof_start = nullptr;
thread_local cudaEvent_t g_prof_stop = nullptr;

void prof_mark(bool start, cudaStream_t s) {
  cudaEvent_t& e = start ? g_prof_start : g_prof_stop;
  if (e) {
    cudaEventRecord(e, s);
    e = nullptr;
  }
}

// ------------------------------------------------------------------ launchers

template <int DT, int CH, bool G>
int launch_fused_ch(zb::FusedArgs a, bool dependent, cudaStream_t s) {
  int grid = 0;
  const int64_t work = (a.hi - a.lo + 7) / 8;
  int rc = grid_for(fused_kid(DT, CH, G), work, &grid);
  if (rc) return rc;
  // chunks only for long windows (>= 64 vectors per thread of the wave: on the 25M-element
  // buckets of a 1.3e9-parameter fp16 job at Nd = 16, 16 per thread, they measured 1% slower)
  // and launches whose last CTA resets the counter (mode != 0)
  a.chunked = a.mode != 0 && work >= 64 * (int64_t)grid * zb::kThreads && use_chunks(a.Nd, G ? a.Nd : a.nrep);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(zb::kThreads);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  // a later bucket of the same step may overlap the previous one's tail (fixed split only: the
  // chunk counter is shared between launches)
  if ((dependent && !a.chunked) || a.wait_first) {
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
  }
  cudaError_t e = cudaLaunchKernelEx(&cfg, zb::fused_step_kernel<DT, CH, G>, a);
  if (e != cudaSuccess) return cuda_fail(e, "fused_step_kernel launch");
  return check_launch("fused_step_kernel launch");
}

// The rank batch width follows the fan-in: 1 or 2 replicas per batch for Nd <= 2, 4 up to
// Nd = 8 (at Nd = 8 two batches of 4 with 24 resident warps per SM beat one batch of 8 with 16:
// +1.4% to +3.7% with chunks, +3.5% for a single output), else 8.
// dependent: a later bucket of the same step, launched right after the previous bucket's fused
// kernel on the same stream (programmatic dependent launch).
template <bool G>
int launch_fused_g(int dtype, const zb::FusedArgs& a, cudaStream_t s, bool d) {
  const bool f16 = dtype == ZERO_FP16;
  if (a.Nd <= 1) return f16 ? launch_fused_ch<1, 1, G>(a, d, s) : launch_fused_ch<0, 1, G>(a, d, s);
  if (a.Nd <= 2) return f16 ? launch_fused_ch<1, 2, G>(a, d, s) : launch_fused_ch<0, 2, G>(a, d, s);
  if (a.Nd <= 8) return f16 ? launch_fused_ch<1, 4, G>(a, d, s) : launch_fused_ch<0, 4, G>(a, d, s);
  return f16 ? launch_fused_ch<1, 8, G>(a, d, s) : launch_fused_ch<0, 8, G>(a, d, s);
}

// a.gsrc != NULL selects the variant that also gathers a ZeRO-3 layer (see fused_step_kernel).
int launch_fused(int dtype, const zb::FusedArgs& a, cudaStream_t s, bool dependent = false) {
  return a.gsrc ? launch_fused_g<true>(dtype, a, s, dependent) : launch_fused_g<false>(dtype, a, s, dependent);
}

// TMA-pipelined fused step over [a.lo, a.hi): whole tiles through the bulk-copy pipeline, the
// rest by the same kernel's consumers.  Every pointer must be 16-byte aligned.
int launch_fused_tma(int dtype, zb::TmaArgs& a, cudaStream_t s, bool dependent = false) {
  int sms = 0;
  int rc = tma_setup(&sms);
  if (rc) return rc;
  a.tiles_lo = (a.lo + 7) & ~int64_t(7);
  if (a.tiles_lo > a.hi) a.tiles_lo = a.hi;
  a.ntiles = (a.hi - a.tiles_lo) / zb::kTile;
  // Several waves of one-CTA-per-SM blocks (at least 16 tiles per CTA, at most 32 waves) let the
  // block scheduler give more tiles to the SMs that stream faster: same-box sweep at Nd = 64,
  // 2^28 elements: 1 wave 6080 GB/s, 8 waves 6499, 16 6656, 32 6671; at Nd = 16, 1.3e9
  // elements: 1 wave 5978, 16 waves 6635.
  int64_t waves = a.ntiles / (16 * (int64_t)sms);
  if (waves > 32) waves = 32;
  if (waves < 1) waves = 1;
  int64_t grid = (int64_t)sms * waves;
  if (grid > zb::kMaxCtas) grid = zb::kMaxCtas;
  if (grid > a.ntiles) grid = a.ntiles;
  if (grid < 1) grid = 1;
  a.stall_unit = g_test_stall;
  g_test_stall = -1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(zb::kTmaThreads);
  cfg.dynamicSmemBytes = zb::kTmaSmemBytes;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  if (dependent) {  // a later bucket of the same step: may overlap the previous bucket's tail
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
  }
  const cudaError_t e = dtype == ZERO_FP16 ? cudaLaunchKernelEx(&cfg, zb::fused_step_tma_kernel<1>, a)
                                           : cudaLaunchKernelEx(&cfg, zb::fused_step_tma_kernel<0>, a);
  if (e != cudaSuccess) return cuda_fail(e, "fused_step_tma_kernel launch");
  return check_launch("fused_step_tma_kernel launch");
}

int launch_rs(int dtype, const zb::RsArgs& a, cudaStream_t s) {
  const bool o16 = a.out16 != nullptr;
  const int kid = dtype == ZERO_FP16 ? (o16 ? kRsFp16Out16 : kRsFp16) : (o16 ? kRsBf16Out16 : kRsBf16);
  int grid = 0;
  int rc = grid_for(kid, (a.hi - a.lo + 7) / 8, &grid, kWavesRs);
  if (rc) return rc;
  if (dtype == ZERO_FP16 && o16)
    zb::reduce_scatter_kernel<1, true><<<grid, zb::kThreads, 0, s>>>(a);
  else if (dtype == ZERO_FP16)
    zb::reduce_scatter_kernel<1, false><<<grid, zb::kThreads, 0, s>>>(a);
  else if (o16)
    zb::reduce_scatter_kernel<0, true><<<grid, zb::kThreads, 0, s>>>(a);
  else
    zb::reduce_scatter_kernel<0, false><<<grid, zb::kThreads, 0, s>>>(a);
  return check_launch("reduce_scatter_kernel launch");
}

int launch_adam(const zb::AdamArgs& a, cudaStream_t s) {
  const bool g16 = a.g16 != nullptr;
  int grid = 0;
  int rc = grid_for(g16 ? kAdamG16 : kAdam, (a.hi - a.lo + 7) / 8, &grid, kWavesAdam);
  if (rc) return rc;
  if (g16)
    zb::adam_kernel<true><<<grid, zb::kThreads, 0, s>>>(a);
  else
    zb::adam_kernel<false><<<grid, zb::kThreads, 0, s>>>(a);
  return check_launch("adam_kernel launch");
}

// dependent: the overflow repair right after the step's last fused launch on the same stream
// (programmatic dependent launch: its launch overlaps the fused kernel's tail).
int launch_cast(const zb::CastArgs& a, cudaStream_t s, bool dependent = false) {
  int grid = 0;
  int rc = grid_for(kCast, (a.hi - a.lo + 7) / 8, &grid);
  if (rc) return rc;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(zb::kThreads);
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  if (dependent) {
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
  }
  cudaError_t e = cudaLaunchKernelEx(&cfg, zb::cast_allgather_kernel, a);
  if (e != cudaSuccess) return cuda_fail(e, "cast_allgather_kernel launch");
  return check_launch("cast_allgather_kernel launch");
}

int launch_ws(void* ws, int op, long long t0, cudaStream_t s) {
  zb::ws_ctl_kernel<<<1, 32, 0, s>>>(header(ws), op, t0);
  return check_launch("ws_ctl_kernel launch");
}

// ZeRO-3 layer gather through the TMA (zero_step stage 3): needs S % 8 == 0 and 16-byte aligned
// buffers; falls back to the register kernel otherwise.
int do_gather_tma(const uint16_t* const* shards, int Nd, int64_t L, uint16_t* const* out, int nout, void* ws,
                  cudaStream_t s);

int do_gather(const uint16_t* const* shards, int Nd, int64_t L, uint16_t* const* out, int nout,
              cudaStream_t s) {
  if (L == 0) return ZERO_OK;
  zb::GatherArgs a;
  std::memset(&a, 0, sizeof a);
  bool al = true;
  int rc = check_ptrs(shards, Nd, "shards", &al);
  if (rc) return rc;
  rc = check_ptrs(out, nout, "out", &al);
  if (rc) return rc;
  const int64_t S = (L + Nd - 1) / Nd;
  for (int r = 0; r < Nd; ++r) a.shards[r] = shards[r];
  for (int o = 0; o < nout; ++o) a.out[o] = out[o];
  a.Nd = Nd;
  a.nout = nout;
  a.L = L;
  a.S = S;
  a.vec = al && (S % 8 == 0);
  // one thread per 8 elements of a shard; about kWavesGather waves in total over the Nd rows
  const int64_t row = (S + 7) / 8;
  int grid = 0;
  rc = grid_for(kGather, row * Nd, &grid, kWavesGather, false);
  if (rc) return rc;
  int64_t gx = (grid + Nd - 1) / Nd;
  const int64_t row_ctas = (row + zb::kThreads - 1) / zb::kThreads;
  if (gx > row_ctas) gx = row_ctas;
  if (gx < 1) gx = 1;
  zb::gather_layer_kernel<<<dim3((unsigned)gx, Nd), zb::kThreads, 0, s>>>(a);
  return check_launch("gather_layer_kernel launch");
}

int do_gather_tma(const uint16_t* const* shards, int Nd, int64_t L, uint16_t* const* out, int nout, void* ws,
                  cudaStream_t s) {
  if (L == 0) return ZERO_OK;
  bool al = true;
  int rc = check_ptrs(shards, Nd, "shards", &al);
  if (rc) return rc;
  rc = check_ptrs(out, nout, "out", &al);
  if (rc) return rc;
  const int64_t S = (L + Nd - 1) / Nd;
  if (!al || S % 8 != 0 || !ws) return do_gather(shards, Nd, L, out, nout, s);
  int sms = 0;
  if ((rc = tma_setup(&sms))) return rc;
  zb::GatherTmaArgs a;
  std::memset(&a, 0, sizeof a);
  for (int r = 0; r < Nd; ++r) a.shards[r] = shards[r];
  for (int o = 0; o < nout; ++o) a.out[o] = out[o];
  a.Nd = Nd;
  a.nout = nout;
  a.L = L;
  a.S = S;
  a.hdr = header(ws);
  const int64_t chunks = (S + zb::kGTile - 1) / zb::kGTile;
  // about kWavesGatherTma waves over the Nd rows (same-box sweep on a 202M-element layer, Nd = 8:
  // 1 wave 5708 GB/s, 8 waves 6335, 32 waves 6570; the register gather with 16 waves 5979)
  int64_t gx = ((int64_t)sms * gather_tma_per_sm() * kWavesGatherTma + Nd - 1) / Nd;
  if (gx > chunks) gx = chunks;
  if (gx < 1) gx = 1;
  zb::gather_layer_tma_kernel<<<dim3((unsigned)gx, Nd), 32, zb::kGSmemBytes, s>>>(a);
  return check_launch("gather_layer_tma_kernel launch");
}

}  // namespace

int zero_internal_fail(int code, const char* msg) { return fail(code, "%s", msg); }

namespace zh {  // zero_host_adam.cpp
void adam_host(float* p, float* m, float* v, const float* g, uint16_t* out16, int64_t n, const zero_hparams_t* hp,
               int64_t t, float coef, int nthreads);
float clip_factor(double max_norm, double sumsq);
}  // namespace zh

// ZeRO-3 step with one fused pass per layer (flag ZERO_FUSED_LAYERS): the gather of layer l and
// the layer's reduce-scatter, unscale, flag / sum of squares, AdamW and bf16 cast in one kernel
// (the K1 kernel with a single bf16 output, the layer's concatenated shards, whose G variant
// copies each old shard word to the Nd gathered-layer buffers before replacing it; with
// ZERO_FORCE_TMA the gather is a TMA fan-out kernel of its own before the pass).  The
// global overflow decision is known only after the last layer, so every layer's update goes into
// the other state copy (read `live`, write 1 - live) and the bf16 shards are written
// speculatively; the last layer's launch ends the step and makes the new copy live unless the
// step overflowed, and an overflowed step has its bf16 shards rewritten from the unchanged live
// copy.  Same arithmetic, same results as the two-phase stage 3 (no reduced-gradient shard), at
// 28 + 4 Nd bytes per parameter instead of 36 + 4 Nd, for twice the fp32 state.
static int zero3_fused_layers(int Nd, int64_t N, int64_t bucket, const zero_state_t* st, const zero_hparams_t* hp,
                              const zb::Consts& c, cudaStream_t s) {
  if (hp->max_grad_norm > 0)
    return fail(ZERO_EINVAL,
                "ZERO_FUSED_LAYERS cannot clip (the update would need the whole gradient's norm first): "
                "use the two-phase stage 3");
  if (st->flags & ZERO_BF16_GRAD_SHARD)
    return fail(ZERO_EINVAL, "ZERO_FUSED_LAYERS keeps no reduced-gradient shard (ZERO_BF16_GRAD_SHARD)");
  for (int i = 0; i < 2; ++i)
    if (!st->master[i] || !st->exp_avg[i] || !st->exp_avg_sq[i])
      return fail(ZERO_EINVAL, "ZERO_FUSED_LAYERS needs both state copies (master/exp_avg/exp_avg_sq [0] and [1])");
  if (!st->param_shard) return fail(ZERO_EINVAL, "stage 3 needs param_shard");
  bool al = true;
  int rc = check_ptrs(st->grads, Nd, "grads", &al);
  if (rc) return rc;
  if ((rc = check_ptrs(st->params, Nd, "params", &al))) return rc;
  void* ws = st->workspace;
  const int64_t L = bucket > 0 ? bucket : N;
  const int64_t nl = (N + L - 1) / L;
  prof_mark(true, s);
  int64_t off = 0;
  for (int64_t l = 0; l < nl; ++l) {
    NvtxRange layer_range("zero3 layer: gather + fused update");
    const int64_t Ll = (l + 1) * L <= N ? L : N - l * L;
    const int64_t Sl = (Ll + Nd - 1) / Nd;
    const uint16_t* shards[ZERO_MAX_ND];
    uint16_t* outs[ZERO_MAX_ND];
    for (int r = 0; r < Nd; ++r) {
      shards[r] = st->param_shard + off + r * Sl;
      outs[r] = st->params[r] + l * st->param_layer_stride;
    }
    // The gather rides in the fused pass (one kernel per layer, see fused_step_kernel's G
    // variant) unless ZERO_FORCE_TMA asks for the TMA fan-out as a kernel of its own.
    const bool tma_gather = (st->flags & ZERO_FORCE_TMA) != 0;
    if (tma_gather && (rc = do_gather_tma(shards, Nd, Ll, outs, Nd, ws, s))) return rc;
    zb::FusedArgs a;
    std::memset(&a, 0, sizeof a);
    a.prefetch = 1;  // the step's own buffers: this GPU's memory
    bool fal = true;
    for (int r = 0; r < Nd; ++r) {
      a.grads[r] = st->grads[r] + l * st->grad_layer_stride;
      fal = fal && aligned16(a.grads[r]);
    }
    if (!tma_gather) {
      a.gsrc = st->param_shard + off;
      for (int r = 0; r < Nd; ++r) {
        a.gout[r] = outs[r];
        fal = fal && aligned16(outs[r]);
      }
    }
    a.reps[0] = st->param_shard + off;
    a.nrep = 1;
    for (int i = 0; i < 2; ++i) {  // the layer's slice of each state copy, indexed from the layer start
      a.p[i] = st->master[i] + off;
      a.m[i] = st->exp_avg[i] + off;
      a.v[i] = st->exp_avg_sq[i] + off;
      fal = fal && aligned16(a.p[i]) && aligned16(a.m[i]) && aligned16(a.v[i]);
    }
    fal = fal && aligned16(a.reps[0]);
    a.lo = 0;
    a.hi = Ll;
    a.c = c;
    a.hdr = header(ws);
    a.part = partials(ws);
    a.Nd = Nd;
    a.vec = fal;
    a.mode = (l == 0 ? zb::kAccSet : zb::kAccAdd) | (l == nl - 1 ? (zb::kFinalize | zb::kFlip) : 0);
    a.trigger_late = l == nl - 1;  // followed by the repair check
    if ((rc = launch_fused(st->grad_dtype, a, s))) return rc;
    off += Sl * Nd;
  }
  // overflow repair: the bf16 shards from the unchanged live copy (runs only after a skip); the
  // shards and the state share one padded layout, so one launch covers every layer.  Launched
  // as a programmatic dependent of the last fused launch, inside the traced span.
  zb::CastArgs r;
  std::memset(&r, 0, sizeof r);
  r.src[0] = st->master[0];
  r.src[1] = st->master[1];
  r.reps[0] = st->param_shard;
  r.nrep = 1;
  r.gate = zb::kGateRepair;
  r.lo = 0;
  r.hi = off;
  r.hdr = header(ws);
  r.vec = aligned16(r.src[0]) && aligned16(r.src[1]) && aligned16(r.reps[0]);
  rc = launch_cast(r, s, true);
  prof_mark(false, s);
  return rc;
}

// ==================================================================== C ABI

extern "C" {

const char* zero_last_error(void) { return g_err; }

const char* zero_version(void) { return "zero-b200 1.0 sm_100a"; }

int zero_partition(int64_t N, int Nd, zero_partition_t* out) {
  if (!out) return fail(ZERO_EINVAL, "out is NULL");
  if (N < 0) return fail(ZERO_EINVAL, "N=%lld < 0", (long long)N);
  int rc = check_nd(Nd);
  if (rc) return rc;
  const int64_t S = (N + Nd - 1) / Nd;
  out->N = N;
  out->Nd = Nd;
  out->reserved = 0;
  out->S = S;
  out->Np = S * Nd;
  out->pad = S * Nd - N;
  return ZERO_OK;
}

size_t zero_workspace_bytes(void) { return zb::kWorkspaceBytes; }

int zero_workspace_init(void* ws, int64_t t, void* stream) {
  if (const int rc = check_ws(ws)) return rc;
  if (t < 0) return fail(ZERO_EINVAL, "t=%lld < 0", (long long)t);
  return launch_ws(ws, zb::kWsInit, t, (cudaStream_t)stream);
}

int zero_read_result(const void* ws, zero_step_result_t* out, void* stream) {
  if (!out) return fail(ZERO_EINVAL, "out is NULL");
  if (const int rc = check_ws(ws)) return rc;
  zb::Header h;
  cudaError_t e = cudaMemcpyAsync(&h, ws, sizeof h, cudaMemcpyDeviceToHost, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpyAsync(result)");
  e = cudaStreamSynchronize((cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  out->step = h.t;
  out->skipped = h.skipped;
  out->overflow = h.last_flag;
  out->live = h.live;
  out->grad_sumsq = h.last_sumsq;
  out->pending_overflow = h.pending_flag;
  out->reserved = 0;
  out->pending_sumsq = h.pending_sumsq;
  out->error = h.error;
  out->reserved2 = 0;
  out->loss_scale = h.dyn ? h.scale : 0.0;
  out->good_steps = h.dyn ? h.good : 0;
  out->dynamic_scale = h.dyn;
  out->reserved3 = 0;
  if (h.error)
    return fail(ZERO_ETIMEOUT,
                "a kernel gave up a bounded internal wait (error word %d); the step it belonged to was "
                "skipped; the word stays set until zero_workspace_init",
                h.error);
  return ZERO_OK;
}

int zero_profile_events(void* start_event, void* stop_event) {
  g_prof_start = (cudaEvent_t)start_event;
  g_prof_stop = (cudaEvent_t)stop_event;
  return ZERO_OK;
}

int zero_loss_scaler_init(void* ws, double init_scale, double growth_factor, double backoff_factor,
                          int64_t growth_interval, void* stream) {
  if (const int rc = check_ws(ws)) return rc;
  if (!(init_scale > 0) || !std::isfinite(init_scale)) return fail(ZERO_EINVAL, "init_scale must be finite and > 0");
  if (!(growth_factor >= 1) || !std::isfinite(growth_factor)) return fail(ZERO_EINVAL, "growth_factor must be >= 1");
  if (!(backoff_factor > 0 && backoff_factor <= 1)) return fail(ZERO_EINVAL, "backoff_factor must be in (0, 1]");
  if (growth_interval < 1) return fail(ZERO_EINVAL, "growth_interval must be >= 1");
  zb::scaler_init_kernel<<<1, 32, 0, (cudaStream_t)stream>>>(header(ws), init_scale, growth_factor, backoff_factor,
                                                             (long long)growth_interval);
  return check_launch("scaler_init_kernel launch");
}

int zero_test_inject_stall(int64_t unit) {
  if (unit < -1) return fail(ZERO_EINVAL, "unit=%lld < -1", (long long)unit);
  g_test_stall = unit;
  return ZERO_OK;
}

int zero_begin_step(void* ws, void* stream) {
  if (const int rc = check_ws(ws)) return rc;
  return launch_ws(ws, zb::kWsBegin, 0, (cudaStream_t)stream);
}

int zero_end_step(void* ws, void* stream) {
  if (const int rc = check_ws(ws)) return rc;
  return launch_ws(ws, zb::kWsEnd, 0, (cudaStream_t)stream);
}

int zero_reduce_scatter(const uint16_t* const* grads, int dtype, int Nd, int64_t lo, int64_t hi,
                        const zero_hparams_t* hp, float* grad_out, void* ws, void* stream) {
  int rc = check_nd(Nd);
  if (rc) return rc;
  if ((rc = check_window(lo, hi))) return rc;
  if ((rc = check_hp(hp))) return rc;
  if (dtype != ZERO_BF16 && dtype != ZERO_FP16) return fail(ZERO_EINVAL, "dtype=%d", dtype);
  if (lo == hi) return ZERO_OK;  // empty window: nothing to reduce or to report
  if (!grad_out) return fail(ZERO_EINVAL, "grad_out is NULL");
  if ((rc = check_ws(ws))) return rc;
  zb::RsArgs a;
  std::memset(&a, 0, sizeof a);
  bool al = aligned16(grad_out);
  if ((rc = check_ptrs(grads, Nd, "grads", &al))) return rc;
  for (int r = 0; r < Nd; ++r) a.grads[r] = grads[r];
  a.out = grad_out;
  a.lo = lo;
  a.hi = hi;
  const zb::Consts c = make_consts(hp, Nd);
  a.inv = c.inv;
  a.inv_base = c.inv_base;
  a.Nd = Nd;
  a.hdr = header(ws);
  a.part = partials(ws);
  a.mode = zb::kAccAdd;
  a.vec = al;
  return launch_rs(dtype, a, (cudaStream_t)stream);
}

int zero_adam_shard(float* master, float* exp_avg, float* exp_avg_sq, const float* grad, int64_t lo,
                    int64_t hi, const zero_hparams_t* hp, uint16_t* param_out, void* ws, void* stream) {
  int rc = check_window(lo, hi);
  if (rc) return rc;
  if ((rc = check_hp(hp))) return rc;
  if (lo == hi) return ZERO_OK;
  if (!master || !exp_avg || !exp_avg_sq || !grad)
    return fail(ZERO_EINVAL, "master, exp_avg, exp_avg_sq and grad must be non-NULL");
  if ((rc = check_ws(ws))) return rc;
  zb::AdamArgs a;
  std::memset(&a, 0, sizeof a);
  a.p[0] = a.p[1] = master;
  a.m[0] = a.m[1] = exp_avg;
  a.v[0] = a.v[1] = exp_avg_sq;
  a.g = grad;
  a.out16 = param_out;
  a.nrep = 0;
  a.use_live = 0;
  a.lo = lo;
  a.hi = hi;
  a.c = make_consts(hp, 1);
  a.hdr = header(ws);
  a.part = partials(ws);
  a.mode = 0;
  a.vec = aligned16(master) && aligned16(exp_avg) && aligned16(exp_avg_sq) && aligned16(grad) &&
          (param_out == nullptr || aligned16(param_out));
  return launch_adam(a, (cudaStream_t)stream);
}

int zero_allgather(const float* master, uint16_t* const* replicas, int Nd, int64_t lo, int64_t hi, int gate,
                   const void* ws, void* stream) {
  int rc = check_nd(Nd);
  if (rc) return rc;
  if ((rc = check_window(lo, hi))) return rc;
  if (gate != ZERO_GATE_ALWAYS && gate != ZERO_GATE_NO_OVERFLOW) return fail(ZERO_EINVAL, "gate=%d", gate);
  if (gate == ZERO_GATE_NO_OVERFLOW && (rc = check_ws(ws))) return rc;
  if (lo == hi) return ZERO_OK;
  if (!master) return fail(ZERO_EINVAL, "master is NULL");
  zb::CastArgs a;
  std::memset(&a, 0, sizeof a);
  bool al = aligned16(master);
  if ((rc = check_ptrs(replicas, Nd, "replicas", &al))) return rc;
  a.src[0] = a.src[1] = master;
  for (int r = 0; r < Nd; ++r) a.reps[r] = replicas[r];
  a.nrep = Nd;
  a.gate = gate == ZERO_GATE_NO_OVERFLOW ? zb::kGateNoOverflow : zb::kGateAlways;
  a.lo = lo;
  a.hi = hi;
  a.hdr = static_cast<const zb::Header*>(ws);
  a.vec = al;
  return launch_cast(a, (cudaStream_t)stream);
}

int zero3_gather_layer(const uint16_t* const* shards, int Nd, int64_t L, uint16_t* const* out, int nout,
                       void* stream) {
  int rc = check_nd(Nd);
  if (rc) return rc;
  if (nout < 1 || nout > ZERO_MAX_ND) return fail(ZERO_EINVAL, "nout=%d outside [1, %d]", nout, ZERO_MAX_ND);
  if (L < 0) return fail(ZERO_EINVAL, "L=%lld < 0", (long long)L);
  return do_gather(shards, Nd, L, out, nout, (cudaStream_t)stream);
}

int zero_step(int stage, int Nd, int64_t N, int64_t bucket, const zero_state_t* st, const zero_hparams_t* hp,
              void* stream) {
  int rc = check_nd(Nd);
  if (rc) return rc;
  if ((rc = check_hp(hp))) return rc;
  if (!st) return fail(ZERO_EINVAL, "state is NULL");
  if (stage < 1 || stage > 3) return fail(ZERO_EINVAL, "stage=%d outside [1, 3]", stage);
  if (N < 0 || bucket < 0) return fail(ZERO_EINVAL, "N and bucket must be >= 0");
  if (st->grad_dtype != ZERO_BF16 && st->grad_dtype != ZERO_FP16)
    return fail(ZERO_EINVAL, "grad_dtype=%d", st->grad_dtype);
  if ((rc = check_ws(st->workspace))) return rc;
  static const char* const kStepNames[4] = {"", "zero_step stage 1", "zero_step stage 2", "zero_step stage 3"};
  NvtxRange range(kStepNames[stage]);
  cudaStream_t s = (cudaStream_t)stream;
  const zb::Consts c = make_consts(hp, Nd);
  void* ws = st->workspace;
  if (N == 0) {  // nothing to reduce or update: the (empty) step completes without overflow
    prof_mark(true, s);
    prof_mark(false, s);
    return launch_ws(ws, zb::kWsEnd, 0, s);
  }

  if (stage == 3 && (st->flags & ZERO_FUSED_LAYERS)) return zero3_fused_layers(Nd, N, bucket, st, hp, c, s);
  if (stage == 3) {
    if (!st->master[0] || !st->exp_avg[0] || !st->exp_avg_sq[0] || !st->grad_shard || !st->param_shard)
      return fail(ZERO_EINVAL, "stage 3 needs master[0], exp_avg[0], exp_avg_sq[0], grad_shard, param_shard");
    bool al = true;
    if ((rc = check_ptrs(st->grads, Nd, "grads", &al))) return rc;
    if ((rc = check_ptrs(st->params, Nd, "params", &al))) return rc;
    const int64_t L = bucket > 0 ? bucket : N;
    const int64_t nl = (N + L - 1) / L;
    const bool g16 = (st->flags & ZERO_BF16_GRAD_SHARD) != 0;
    uint16_t* gsh16 = reinterpret_cast<uint16_t*>(st->grad_shard);
    prof_mark(true, s);
    int64_t off = 0;
    for (int64_t l = 0; l < nl; ++l) {  // forward gathers + backward reduce-scatters, layer by layer
      NvtxRange layer_range("zero3 layer: gather + reduce-scatter");
      const int64_t Ll = (l + 1) * L <= N ? L : N - l * L;
      const int64_t Sl = (Ll + Nd - 1) / Nd;
      const uint16_t* shards[ZERO_MAX_ND];
      uint16_t* outs[ZERO_MAX_ND];
      const uint16_t* gl[ZERO_MAX_ND];
      for (int r = 0; r < Nd; ++r) {
        shards[r] = st->param_shard + off + r * Sl;
        outs[r] = st->params[r] + l * st->param_layer_stride;
        gl[r] = st->grads[r] + l * st->grad_layer_stride;
      }
      // register gather by default; ZERO_FORCE_TMA selects the TMA fan-out.  Alone on a
      // 202M-element layer the TMA one is faster (32 waves: 6.57 TB/s against 5.98), but inside
      // the ZeRO-3 step the two measured the same (69.16 against 68.93 ms per step)
      rc = (st->flags & ZERO_FORCE_TMA) ? do_gather_tma(shards, Nd, Ll, outs, Nd, ws, s)
                                        : do_gather(shards, Nd, Ll, outs, Nd, s);
      if (rc) return rc;
      zb::RsArgs a;
      std::memset(&a, 0, sizeof a);
      bool ral = g16 ? aligned16(gsh16 + off) : aligned16(st->grad_shard + off);
      for (int r = 0; r < Nd; ++r) {
        a.grads[r] = gl[r];
        ral = ral && aligned16(gl[r]);
      }
      if (g16)
        a.out16 = gsh16 + off;
      else
        a.out = st->grad_shard + off;
      a.lo = 0;
      a.hi = Ll;
      a.inv = c.inv;
      a.inv_base = c.inv_base;
      a.Nd = Nd;
      a.hdr = header(ws);
      a.part = partials(ws);
      a.mode = l == 0 ? zb::kAccSet : zb::kAccAdd;
      a.vec = ral;
      if ((rc = launch_rs(st->grad_dtype, a, s))) return rc;
      off += Sl * Nd;
    }
    off = 0;
    for (int64_t l = 0; l < nl; ++l) {  // optimizer step on every shard, gated on the overflow flag
      const int64_t Ll = (l + 1) * L <= N ? L : N - l * L;
      const int64_t Sl = (Ll + Nd - 1) / Nd;
      zb::AdamArgs a;
      std::memset(&a, 0, sizeof a);
      a.p[0] = a.p[1] = st->master[0] + off;
      a.m[0] = a.m[1] = st->exp_avg[0] + off;
      a.v[0] = a.v[1] = st->exp_avg_sq[0] + off;
      if (g16)
        a.g16 = gsh16 + off;
      else
        a.g = st->grad_shard + off;
      a.out16 = st->param_shard + off;
      a.lo = 0;
      a.hi = Ll;
      a.c = c;
      a.hdr = header(ws);
      a.part = partials(ws);
      a.mode = l == nl - 1 ? zb::kFinalize : 0;
      a.vec = aligned16(a.p[0]) && aligned16(a.m[0]) && aligned16(a.v[0]) &&
              (g16 ? aligned16(a.g16) : aligned16(a.g)) && aligned16(a.out16);
      if ((rc = launch_adam(a, s))) return rc;
      off += Sl * Nd;
    }
    prof_mark(false, s);
    return ZERO_OK;
  }

  // stages 1 and 2
  bool al = true;
  if ((rc = check_ptrs(st->grads, Nd, "grads", &al))) return rc;
  if ((rc = check_ptrs(st->params, Nd, "params", &al))) return rc;
  const int64_t B = bucket > 0 ? bucket : N;
  const int64_t nb = (N + B - 1) / B;

  if ((st->flags & ZERO_BF16_GRAD_SHARD) && !(st->flags & ZERO_TWO_PASS))
    return fail(ZERO_EINVAL, "ZERO_BF16_GRAD_SHARD needs a gradient shard: ZERO_TWO_PASS or stage 3");
  if (st->flags & ZERO_TWO_PASS) {
    if (!st->master[0] || !st->exp_avg[0] || !st->exp_avg_sq[0] || !st->grad_shard)
      return fail(ZERO_EINVAL, "ZERO_TWO_PASS needs master[0], exp_avg[0], exp_avg_sq[0], grad_shard");
    const bool g16 = (st->flags & ZERO_BF16_GRAD_SHARD) != 0;
    uint16_t* gsh16 = reinterpret_cast<uint16_t*>(st->grad_shard);
    prof_mark(true, s);
    for (int64_t k = 0; k < nb; ++k) {
      zb::RsArgs a;
      std::memset(&a, 0, sizeof a);
      for (int r = 0; r < Nd; ++r) a.grads[r] = st->grads[r];
      if (g16)
        a.out16 = gsh16;
      else
        a.out = st->grad_shard;
      a.lo = k * B;
      a.hi = (k + 1) * B < N ? (k + 1) * B : N;
      a.inv = c.inv;
      a.inv_base = c.inv_base;
      a.Nd = Nd;
      a.hdr = header(ws);
      a.part = partials(ws);
      a.mode = k == 0 ? zb::kAccSet : zb::kAccAdd;
      a.vec = al && aligned16(st->grad_shard);
      if ((rc = launch_rs(st->grad_dtype, a, s))) return rc;
    }
    // copy 1 may be absent on this path; `live` then must be 0
    const bool two = st->master[1] && st->exp_avg[1] && st->exp_avg_sq[1];
    for (int64_t k = 0; k < nb; ++k) {
      zb::AdamArgs a;
      std::memset(&a, 0, sizeof a);
      for (int i = 0; i < 2; ++i) {
        a.p[i] = two ? st->master[i] : st->master[0];
        a.m[i] = two ? st->exp_avg[i] : st->exp_avg[0];
        a.v[i] = two ? st->exp_avg_sq[i] : st->exp_avg_sq[0];
      }
      if (g16)
        a.g16 = gsh16;
      else
        a.g = st->grad_shard;
      for (int r = 0; r < Nd; ++r) a.reps[r] = st->params[r];
      a.nrep = Nd;
      a.use_live = 1;
      a.lo = k * B;
      a.hi = (k + 1) * B < N ? (k + 1) * B : N;
      a.c = c;
      a.hdr = header(ws);
      a.part = partials(ws);
      a.mode = k == nb - 1 ? zb::kFinalize : 0;
      a.vec = al && aligned16(a.p[0]) && aligned16(a.p[1]) && aligned16(a.m[0]) && aligned16(a.m[1]) &&
              aligned16(a.v[0]) && aligned16(a.v[1]) && aligned16(st->grad_shard);
      if ((rc = launch_adam(a, s))) return rc;
    }
    prof_mark(false, s);
    return ZERO_OK;
  }

  if (hp->max_grad_norm > 0)
    return fail(ZERO_EINVAL,
                "gradient clipping needs the whole gradient's norm before the update: use "
                "ZERO_TWO_PASS (or stage 3); the fused one-pass step cannot clip");
  for (int i = 0; i < 2; ++i)
    if (!st->master[i] || !st->exp_avg[i] || !st->exp_avg_sq[i])
      return fail(ZERO_EINVAL, "ZERO_FUSED needs both state copies (master/exp_avg/exp_avg_sq [0] and [1])");
  zb::FusedArgs a;
  std::memset(&a, 0, sizeof a);
  a.prefetch = 1;  // the step's own buffers: this GPU's memory
  for (int r = 0; r < Nd; ++r) {
    a.grads[r] = st->grads[r];
    a.reps[r] = st->params[r];
  }
  for (int i = 0; i < 2; ++i) {
    a.p[i] = st->master[i];
    a.m[i] = st->exp_avg[i];
    a.v[i] = st->exp_avg_sq[i];
    al = al && aligned16(a.p[i]) && aligned16(a.m[i]) && aligned16(a.v[i]);
  }
  a.c = c;
  a.hdr = header(ws);
  a.part = partials(ws);
  a.Nd = Nd;
  a.nrep = Nd;
  a.vec = al;
  // The TMA pipeline wins where many loads must be in flight per element (one B200, with its
  // multi-wave grid: Nd = 64, 2^28: 6671 GB/s against 6091 for the register kernel; Nd = 16,
  // 1.3e9 in one bucket: 6635 against 6229; in 52 buckets of 25M, with the buckets launched as
  // programmatic dependents, which hides the TMA kernel's per-launch set-up: 6555 against 6115);
  // at Nd = 8 the two are equal.  Windows under 2^24 elements keep the register kernel.
  const bool tma_auto = Nd >= 16 && B >= (int64_t(1) << 24);
  const bool tma = al && !(st->flags & ZERO_NO_TMA) && ((st->flags & ZERO_FORCE_TMA) || tma_auto);
  // A short unbucketed step skips the separate overflow-repair launch: after an overflow the
  // fused kernel's last CTA rewrites the replicas alone.  On such a step that launch is a large
  // part of the time (1M elements at Nd = 4: 16.75 -> 15.64 us per step), while a skipped step
  // becomes slower (one CTA moves the window's 4 + 2Nd bytes per element); skips are rare.
  const bool self_repair = !tma && nb == 1 && N <= kSelfRepairMax;
  zb::TmaArgs ta;
  if (tma) {
    std::memset(&ta, 0, sizeof ta);
    for (int r = 0; r < Nd; ++r) {
      ta.grads[r] = a.grads[r];
      ta.reps[r] = a.reps[r];
    }
    for (int i = 0; i < 2; ++i) {
      ta.p[i] = a.p[i];
      ta.m[i] = a.m[i];
      ta.v[i] = a.v[i];
    }
    ta.c = c;
    ta.hdr = a.hdr;
    ta.part = a.part;
    ta.Nd = Nd;
  }
  prof_mark(true, s);
  for (int64_t k = 0; k < nb; ++k) {
    a.lo = k * B < N ? k * B : N;
    a.hi = (k + 1) * B < N ? (k + 1) * B : N;
    a.mode = (k == 0 ? zb::kAccSet : zb::kAccAdd) | (k == nb - 1 ? (zb::kFinalize | zb::kFlip) : 0);
    a.trigger_late = k == nb - 1;  // followed by the repair check, not by another bucket
    // the first bucket waits for its predecessor at its start, so it may be a programmatic
    // dependent of it: after the repair check of a previous step (which triggers at once) its
    // launch latency is hidden; after any other kernel it starts when that kernel completes
    a.wait_first = k == 0;
    a.self_repair = self_repair;
    if (self_repair) a.trigger_late = 1;  // the next step may launch once the main loops are done
    if (tma) {
      ta.lo = a.lo;
      ta.hi = a.hi;
      ta.mode = a.mode;
      ta.trigger_late = a.trigger_late;
      if ((rc = launch_fused_tma(st->grad_dtype, ta, s, k > 0))) return rc;
    } else if ((rc = launch_fused(st->grad_dtype, a, s, k > 0))) {
      return rc;
    }
  }
  if (self_repair) {  // the fused kernel's last CTA repairs after a skip: no repair launch
    prof_mark(false, s);
    return ZERO_OK;
  }
  // overflow repair: rewrite the replicas from the unchanged state (runs only after a skip);
  // launched as a programmatic dependent of the last fused launch, inside the traced span
  zb::CastArgs r;
  std::memset(&r, 0, sizeof r);
  r.src[0] = st->master[0];
  r.src[1] = st->master[1];
  for (int q = 0; q < Nd; ++q) r.reps[q] = st->params[q];
  r.nrep = Nd;
  r.gate = zb::kGateRepair;
  r.lo = 0;
  r.hi = N;
  r.hdr = header(ws);
  r.vec = al;
  rc = launch_cast(r, s, true);
  prof_mark(false, s);
  return rc;
}

}  // extern "C"

// ==================================================================== no-allocation variant
//
// zero_reduce_scatter_noalloc: the reduce-scatter of zero_reduce_scatter for callers that cannot
// allocate device memory.  Its only scratch (the arrival counter and one partial per CTA) lives
// in the file-scope array below instead of a caller-provided workspace.

namespace {

constexpr int kNoAllocTile = zb::kThreads * 8;  // elements per CTA: one 16-byte vector per thread
constexpr size_t kNoAllocHeader = 256;          // arrival counter, padded to the array alignment
constexpr size_t kNoAllocBytes = kNoAllocHeader + sizeof(zb::Partial) * ZERO_NOALLOC_MAX_CTAS;
// The window limit the header publishes is exactly the CTA count that has scratch slots: a
// window it accepts never launches more CTAs than there are partial slots.
static_assert(ZERO_NOALLOC_MAX_WINDOW == (int64_t)ZERO_NOALLOC_MAX_CTAS * kNoAllocTile,
              "ZERO_NOALLOC_MAX_WINDOW must equal ZERO_NOALLOC_MAX_CTAS x elements per CTA");

// Shared by every call on a device; held by every GPU that loads the library until exit.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocBytes];

void* g_noalloc_addr[kMaxDevices] = {};
std::mutex g_noalloc_mu;

struct NoAllocRsArgs {
  const uint16_t* grads[zb::kMaxNd];
  float* out;
  int64_t lo, hi;
  float inv;
  int Nd;
  unsigned int* done;          // scratch: arrival counter (cleared before every launch)
  zb::Partial* part;           // scratch: one slot per CTA
  zero_rs_summary_t* summary;  // caller's output
  int accumulate;
  int vec;
};

template <int DT>
__global__ void __launch_bounds__(zb::kThreads) reduce_scatter_noalloc_kernel(const __grid_constant__ NoAllocRsArgs a) {
  double sq = 0.0;
  int bad = 0;
  float* __restrict__ out = a.out;
  const zb::Span sp8(a.lo, a.hi, a.vec);
  const int64_t stride = (int64_t)gridDim.x * zb::kThreads;
  for (int64_t j = (int64_t)blockIdx.x * zb::kThreads + threadIdx.x; j < sp8.nvec; j += stride) {
    const int64_t i = sp8.vlo + (j << 3);
    float s[8];
    zb::fan_in8<DT>(a.grads, a.Nd, i, s);
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      s[k] = __fmul_rn(s[k], a.inv);
      bad |= zb::nonfinite(s[k]);
      sq = __dadd_rn(sq, __dmul_rn((double)s[k], (double)s[k]));
    }
    zb::st_stream(out + i, make_float4(s[0], s[1], s[2], s[3]));
    zb::st_stream(out + i + 4, make_float4(s[4], s[5], s[6], s[7]));
  }
  for (int64_t e = (int64_t)blockIdx.x * zb::kThreads + threadIdx.x; e < sp8.nrest; e += stride) {
    const int64_t i = sp8.scalar_index(a.lo, e);
    const float g = __fmul_rn(zb::fan_in1<DT>(a.grads, a.Nd, i), a.inv);
    bad |= zb::nonfinite(g);
    sq = __dadd_rn(sq, __dmul_rn((double)g, (double)g));
    out[i] = g;
  }
  // per-CTA partial into the scratch slot; the last CTA to arrive combines them in CTA order
  __shared__ double r_sq[zb::kWarps];
  __shared__ int r_bad[zb::kWarps];
  __shared__ int am_last;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  sq = zb::warp_sum(sq);
  bad = __any_sync(0xffffffffu, bad);
  if (lane == 0) {
    r_sq[warp] = sq;
    r_bad[warp] = bad;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    double s = 0.0;
    int f = 0;
    for (int w = 0; w < zb::kWarps; ++w) {
      s = __dadd_rn(s, r_sq[w]);
      f |= r_bad[w];
    }
    a.part[blockIdx.x].sumsq = s;
    a.part[blockIdx.x].flag = f;
    __threadfence();
    am_last = (atomicAdd(a.done, 1u) == gridDim.x - 1);
  }
  __syncthreads();
  if (!am_last) return;
  __threadfence();
  double s = 0.0;
  int f = 0;
  for (int k = threadIdx.x; k < (int)gridDim.x; k += zb::kThreads) {
    s = __dadd_rn(s, __ldcg(&a.part[k].sumsq));
    f |= __ldcg(&a.part[k].flag);
  }
  s = zb::warp_sum(s);
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
    for (int w = 0; w < zb::kWarps; ++w) {
      tot = __dadd_rn(tot, r_sq[w]);
      fl |= r_bad[w];
    }
    if (a.accumulate) {
      a.summary->overflow |= fl;
      a.summary->sumsq = __dadd_rn(a.summary->sumsq, tot);
    } else {
      a.summary->overflow = fl;
      a.summary->reserved = 0;
      a.summary->sumsq = tot;
    }
  }
}

// Device address of the scratch array for the current device (looked up once per device).
int noalloc_scratch(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(ZERO_EINVAL, "device ordinal %d unsupported", dev);
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (!g_noalloc_addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(no-alloc scratch)");
    g_noalloc_addr[dev] = p;
  }
  *out = g_noalloc_addr[dev];
  return ZERO_OK;
}

}  // namespace

extern "C" int zero_reduce_scatter_noalloc(const uint16_t* const* grads, int dtype, int Nd, int64_t lo, int64_t hi,
                                           const zero_hparams_t* hp, float* grad_out, zero_rs_summary_t* summary,
                                           int accumulate, void* stream) {
  int rc = check_nd(Nd);
  if (rc) return rc;
  if ((rc = check_window(lo, hi))) return rc;
  if ((rc = check_hp(hp))) return rc;
  if (dtype != ZERO_BF16 && dtype != ZERO_FP16) return fail(ZERO_EINVAL, "dtype=%d", dtype);
  if (hi - lo > ZERO_NOALLOC_MAX_WINDOW)
    return fail(ZERO_ENOMEM,
                "window of %lld elements exceeds the no-allocation limit of %lld elements "
                "(%d scratch slots of %d elements); split it into smaller windows",
                (long long)(hi - lo), (long long)ZERO_NOALLOC_MAX_WINDOW, ZERO_NOALLOC_MAX_CTAS, kNoAllocTile);
  if (!summary) return fail(ZERO_EINVAL, "summary is NULL");
  bool al = true;
  if (hi > lo) {
    if (!grad_out) return fail(ZERO_EINVAL, "grad_out is NULL");
    al = aligned16(grad_out);
    if ((rc = check_ptrs(grads, Nd, "grads", &al))) return rc;
  }
  void* scratch = nullptr;
  if ((rc = noalloc_scratch(&scratch))) return rc;
  cudaStream_t s = (cudaStream_t)stream;
  // the arrival counter must start at zero; the partial slots are written before they are read
  cudaError_t e = cudaMemsetAsync(scratch, 0, sizeof(unsigned int), s);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(no-alloc counter)");
  NoAllocRsArgs a;
  std::memset(&a, 0, sizeof a);
  if (hi > lo)
    for (int r = 0; r < Nd; ++r) a.grads[r] = grads[r];
  a.out = grad_out;
  a.lo = lo;
  a.hi = hi;
  a.inv = make_consts(hp, Nd).inv;
  a.Nd = Nd;
  a.done = static_cast<unsigned int*>(scratch);
  a.part = reinterpret_cast<zb::Partial*>(static_cast<unsigned char*>(scratch) + kNoAllocHeader);
  a.summary = summary;
  a.accumulate = accumulate != 0;
  a.vec = al;
  int64_t grid = (hi - lo + kNoAllocTile - 1) / kNoAllocTile;
  if (grid < 1) grid = 1;  // an empty window still writes (or keeps) the summary
  if (dtype == ZERO_FP16)
    reduce_scatter_noalloc_kernel<1><<<(unsigned)grid, zb::kThreads, 0, s>>>(a);
  else
    reduce_scatter_noalloc_kernel<0><<<(unsigned)grid, zb::kThreads, 0, s>>>(a);
  return check_launch("reduce_scatter_noalloc_kernel launch");
}

// ==================================================================== ZeRO-Offload step

namespace {

struct EventRing {  // per-chunk completion events, destroyed on every exit path
  std::vector<cudaEvent_t> ev;
  ~EventRing() {
    for (cudaEvent_t e : ev)
      if (e) cudaEventDestroy(e);
  }
};

}  // namespace

extern "C" int zero_offload_step(int Nd, int64_t N, int64_t chunk, const zero_offload_state_t* st,
                                 const zero_hparams_t* hp, void* stream) {
  int rc = check_nd(Nd);
  if (rc) return rc;
  if ((rc = check_hp(hp))) return rc;
  if (!st) return fail(ZERO_EINVAL, "state is NULL");
  if (N < 0 || chunk < 0) return fail(ZERO_EINVAL, "N and chunk must be >= 0");
  if (st->grad_dtype != ZERO_BF16 && st->grad_dtype != ZERO_FP16) return fail(ZERO_EINVAL, "grad_dtype=%d", st->grad_dtype);
  if ((rc = check_ws(st->workspace))) return rc;
  cudaStream_t s = (cudaStream_t)stream;
  void* ws = st->workspace;
  NvtxRange range("zero_offload_step");
  if (N == 0) return launch_ws(ws, zb::kWsEnd, 0, s);
  if (!st->grad_dev || !st->param_dev || !st->grad_host || !st->param_host || !st->master_host ||
      !st->exp_avg_host || !st->exp_avg_sq_host)
    return fail(ZERO_EINVAL, "offload state needs grad_dev, param_dev, grad_host, param_host and the host fp32 state");
  bool al = aligned16(st->grad_dev) && aligned16(st->param_dev);
  if ((rc = check_ptrs(st->grads, Nd, "grads", &al))) return rc;
  if ((rc = check_ptrs(st->params, Nd, "params", &al))) return rc;
  cudaStream_t up = st->upload_stream ? (cudaStream_t)st->upload_stream : s;
  const zb::Consts c = make_consts(hp, Nd);
  const int64_t C = chunk > 0 ? chunk : N;
  const int64_t nc = (N + C - 1) / C;
  EventRing ring;
  ring.ev.assign((size_t)nc + 2, nullptr);
  for (auto& e : ring.ev) {
    cudaError_t e2 = cudaEventCreateWithFlags(&e, cudaEventDisableTiming);
    if (e2 != cudaSuccess) return cuda_fail(e2, "cudaEventCreateWithFlags");
  }
  cudaEvent_t ev_rs = ring.ev[nc], ev_up = ring.ev[nc + 1];
  prof_mark(true, s);
  // 1. reduce-scatter every chunk into the fp32 staging buffer (overflow flag and norm
  //    accumulate in the workspace), then stream the chunks to host memory
  for (int64_t k = 0; k < nc; ++k) {
    zb::RsArgs a;
    std::memset(&a, 0, sizeof a);
    for (int r = 0; r < Nd; ++r) a.grads[r] = st->grads[r];
    a.out = st->grad_dev;
    a.lo = k * C;
    a.hi = (k + 1) * C < N ? (k + 1) * C : N;
    a.inv = c.inv;
    a.inv_base = c.inv_base;
    a.Nd = Nd;
    a.hdr = header(ws);
    a.part = partials(ws);
    a.mode = k == 0 ? zb::kAccSet : zb::kAccAdd;
    a.vec = al;
    if ((rc = launch_rs(st->grad_dtype, a, s))) return rc;
  }
  cudaError_t e = cudaEventRecord(ev_rs, s);
  if (e != cudaSuccess) return cuda_fail(e, "cudaEventRecord");
  for (int64_t k = 0; k < nc; ++k) {
    const int64_t lo = k * C, len = (k + 1) * C < N ? C : N - lo;
    e = cudaMemcpyAsync(st->grad_host + lo, st->grad_dev + lo, (size_t)len * 4, cudaMemcpyDeviceToHost, s);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpyAsync(gradient to host)");
    if ((e = cudaEventRecord(ring.ev[k], s)) != cudaSuccess) return cuda_fail(e, "cudaEventRecord");
  }
  // 2. the overflow decision and the norm, once every chunk is reduced
  if ((e = cudaEventSynchronize(ev_rs)) != cudaSuccess) return cuda_fail(e, "cudaEventSynchronize");
  zb::Header h;
  if ((e = cudaMemcpyAsync(&h, ws, sizeof h, cudaMemcpyDeviceToHost, up)) != cudaSuccess)
    return cuda_fail(e, "cudaMemcpyAsync(workspace)");
  if ((e = cudaStreamSynchronize(up)) != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  if (!h.pending_flag) {
    // 3. host AdamW chunk by chunk as the gradients land; each chunk's bf16 weights go back
    //    and are fanned out to the Nd replicas on the upload stream, overlapping the next chunk
    const float coef = zh::clip_factor(hp->max_grad_norm, h.pending_sumsq);
    for (int64_t k = 0; k < nc; ++k) {
      const int64_t lo = k * C, len = (k + 1) * C < N ? C : N - lo;
      if ((e = cudaEventSynchronize(ring.ev[k])) != cudaSuccess) return cuda_fail(e, "cudaEventSynchronize");
      NvtxRange chunk_range("host AdamW chunk");
      zh::adam_host(st->master_host + lo, st->exp_avg_host + lo, st->exp_avg_sq_host + lo, st->grad_host + lo,
                    st->param_host + lo, len, hp, h.t + 1, coef, st->host_threads);
      e = cudaMemcpyAsync(st->param_dev + lo, st->param_host + lo, (size_t)len * 2, cudaMemcpyHostToDevice, up);
      if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpyAsync(weights to device)");
      const uint16_t* src[1] = {st->param_dev + lo};
      uint16_t* dst[ZERO_MAX_ND];
      for (int r = 0; r < Nd; ++r) dst[r] = st->params[r] + lo;
      if ((rc = do_gather(src, 1, len, dst, Nd, up))) return rc;
    }
  }
  if ((e = cudaEventRecord(ev_up, up)) != cudaSuccess) return cuda_fail(e, "cudaEventRecord");
  if ((e = cudaStreamWaitEvent(s, ev_up, 0)) != cudaSuccess) return cuda_fail(e, "cudaStreamWaitEvent");
  prof_mark(false, s);
  // 4. end of step on the device: t, skip count and the dynamic loss scale
  rc = launch_ws(ws, zb::kWsEnd, 0, s);
  if (rc) return rc;
  // the events may be destroyed now: pending work that refers to them still completes
  return ZERO_OK;
}

// ==================================================================== windows (multi-GPU)

extern "C" int zero_fused_window(int Nd, int64_t lo, int64_t hi, const zero_state_t* st, const zero_hparams_t* hp,
                                 int finalize, void* stream) {
  int rc = check_nd(Nd);
  if (rc) return rc;
  if ((rc = check_window(lo, hi))) return rc;
  if ((rc = check_hp(hp))) return rc;
  if (!st) return fail(ZERO_EINVAL, "state is NULL");
  if ((rc = check_ws(st->workspace))) return rc;
  if (st->grad_dtype != ZERO_BF16 && st->grad_dtype != ZERO_FP16) return fail(ZERO_EINVAL, "grad_dtype=%d", st->grad_dtype);
  if (hp->max_grad_norm > 0) return fail(ZERO_EINVAL, "the fused pass cannot clip (needs the global norm first)");
  bool al = true;
  if ((rc = check_ptrs(st->grads, Nd, "grads", &al))) return rc;
  if ((rc = check_ptrs(st->params, Nd, "params", &al))) return rc;
  zb::FusedArgs a;
  std::memset(&a, 0, sizeof a);
  for (int r = 0; r < Nd; ++r) {
    a.grads[r] = st->grads[r];
    a.reps[r] = st->params[r];
  }
  for (int i = 0; i < 2; ++i) {
    if (!st->master[i] || !st->exp_avg[i] || !st->exp_avg_sq[i])
      return fail(ZERO_EINVAL, "the fused pass needs both state copies");
    a.p[i] = st->master[i];
    a.m[i] = st->exp_avg[i];
    a.v[i] = st->exp_avg_sq[i];
    al = al && aligned16(a.p[i]) && aligned16(a.m[i]) && aligned16(a.v[i]);
  }
  a.c = make_consts(hp, Nd);
  a.hdr = header(st->workspace);
  a.part = partials(st->workspace);
  a.Nd = Nd;
  a.nrep = Nd;
  a.vec = al;
  a.lo = lo;
  a.hi = hi;
  a.mode = zb::kAccSet | (finalize ? (zb::kFinalize | zb::kFlip) : 0);
  a.trigger_late = finalize != 0;  // followed by the repair check
  cudaStream_t s = (cudaStream_t)stream;
  prof_mark(true, s);
  rc = launch_fused(st->grad_dtype, a, s);
  if (!rc && finalize) {  // the step ended here: after an overflow, rewrite the window's replicas
    zb::CastArgs r;
    std::memset(&r, 0, sizeof r);
    r.src[0] = st->master[0];
    r.src[1] = st->master[1];
    for (int q = 0; q < Nd; ++q) r.reps[q] = st->params[q];
    r.nrep = Nd;
    r.gate = zb::kGateRepair;
    r.lo = lo;
    r.hi = hi;
    r.hdr = header(st->workspace);
    r.vec = al;
    rc = launch_cast(r, s, true);
  }
  prof_mark(false, s);
  return rc;
}

extern "C" int zero_end_step_flip(void* ws, void* stream) {
  if (const int rc = check_ws(ws)) return rc;
  return launch_ws(ws, zb::kWsEndFlip, 0, (cudaStream_t)stream);
}

extern "C" int zero_repair_window(int Nd, int64_t lo, int64_t hi, const zero_state_t* st, void* stream) {
  int rc = check_nd(Nd);
  if (rc) return rc;
  if ((rc = check_window(lo, hi))) return rc;
  if (!st || !st->workspace || !st->master[0] || !st->master[1]) return fail(ZERO_EINVAL, "state is incomplete");
  if ((rc = check_ws(st->workspace))) return rc;
  if (lo == hi) return ZERO_OK;
  bool al = aligned16(st->master[0]) && aligned16(st->master[1]);
  if ((rc = check_ptrs(st->params, Nd, "params", &al))) return rc;
  zb::CastArgs r;
  std::memset(&r, 0, sizeof r);
  r.src[0] = st->master[0];
  r.src[1] = st->master[1];
  for (int q = 0; q < Nd; ++q) r.reps[q] = st->params[q];
  r.nrep = Nd;
  r.gate = zb::kGateRepair;
  r.lo = lo;
  r.hi = hi;
  r.hdr = header(st->workspace);
  r.vec = al;
  return launch_cast(r, (cudaStream_t)stream);
}
