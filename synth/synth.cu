// synth.cu -- device implementation of the seeded input generator of synth/__init__.py.
//
// Test and benchmark infrastructure: it writes synthetic gradient replicas, master weights
// and moments straight into device memory so that multi-gigabyte inputs need no host
// round trip.  It holds none of the optimizer's arithmetic.  The definition (SplitMix64
// outputs, Irwin-Hall(12) sum of 16-bit fields, value kinds, output types)
// is documented in synth/__init__.py; this file implements it bit for bit.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace {

constexpr uint64_t kGamma = 0x9E3779B97F4A7C15ull;
constexpr uint64_t kTail = 1ull << 62;

__host__ __device__ inline uint64_t mix(uint64_t z) {
  z ^= z >> 30;
  z *= 0xBF58476D1CE4E5B9ull;
  z ^= z >> 27;
  z *= 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

__host__ __device__ inline uint64_t out(uint64_t s, uint64_t k) { return mix(s + (k + 1) * kGamma); }

__device__ inline uint32_t fields16(uint64_t h) {
  return (uint32_t)(h & 0xFFFF) + (uint32_t)((h >> 16) & 0xFFFF) + (uint32_t)((h >> 32) & 0xFFFF) +
         (uint32_t)(h >> 48);
}

struct FillArgs {
  void* dst;
  int dtype;  // 0 bf16, 1 fp16, 2 fp32
  int kind;   // 0 normal, 1 abs, 2 square, 3 heavy, 4 zero
  uint64_t s, s_tail;
  int64_t first, n;
  float sigma, tail_sigma;
  uint32_t tail_mod;
};

__global__ void fill_kernel(const FillArgs a) {
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < a.n;
       e += (int64_t)gridDim.x * blockDim.x) {
    uint64_t k = (uint64_t)(a.first + e);
    float x = 0.0f;
    if (a.kind != 4) {
      uint32_t total = fields16(out(a.s, 3 * k)) + fields16(out(a.s, 3 * k + 1)) + fields16(out(a.s, 3 * k + 2));
      float z = __fmul_rn((float)((int32_t)total - 393210), 1.52587890625e-05f);  // 2^-16, exact
      float sg = a.sigma;
      if (a.kind == 3 && (out(a.s_tail, k) % a.tail_mod) == 0) sg = a.tail_sigma;
      x = __fmul_rn(z, sg);
      if (a.kind == 1) x = fabsf(x);
      if (a.kind == 2) x = __fmul_rn(x, x);
    }
    if (a.dtype == 2) {
      static_cast<float*>(a.dst)[e] = x;
    } else if (a.dtype == 1) {
      static_cast<__half*>(a.dst)[e] = __float2half_rn(x);
    } else {
      static_cast<uint16_t*>(a.dst)[e] = (uint16_t)(__float_as_uint(x) >> 16);  // upper half
    }
  }
}

}  // namespace

extern "C" int synth_fill(void* dst, int dtype, int kind, uint64_t seed, uint64_t stream, int64_t first, int64_t n,
                          float sigma, float tail_sigma, uint32_t tail_mod, void* cuda_stream) {
  if (n < 0 || first < 0 || dtype < 0 || dtype > 2 || kind < 0 || kind > 4) return -1;
  if (n == 0) return 0;
  if (!dst || (kind == 3 && tail_mod == 0)) return -1;
  FillArgs a;
  a.dst = dst;
  a.dtype = dtype;
  a.kind = kind;
  a.s = out(seed, stream);
  a.s_tail = out(seed, stream ^ kTail);
  a.first = first;
  a.n = n;
  a.sigma = sigma;
  a.tail_sigma = tail_sigma;
  a.tail_mod = tail_mod;
  int64_t blocks = (n + 255) / 256;
  if (blocks > 148 * 32) blocks = 148 * 32;
  fill_kernel<<<(unsigned)blocks, 256, 0, (cudaStream_t)cuda_stream>>>(a);
  return cudaGetLastError() == cudaSuccess ? 0 : -2;
}
