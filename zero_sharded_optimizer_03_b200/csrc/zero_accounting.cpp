// zero_accounting.cpp -- host-only closed forms of include/zero.h: per-GPU model-state memory
// and per-rank communication volume of plain data parallelism and ZeRO stages 1-3.
#include "zero.h"

int zero_internal_fail(int code, const char* msg);  // zero_abi.cu: sets zero_last_error

extern "C" {

// [P1] §二 code: weights and gradients take bytes_per_param each, Adam's fp32 copy + m + v take
// bytes_per_opt_state; ZeRO-1 shards the optimizer state, ZeRO-2 also the gradients, ZeRO-3
// the weights too.  Results in GiB (2^30 bytes), as the page's helper reports them.
int zero_memory_estimate(double N, int Nd, int bytes_per_param, int bytes_per_opt_state, zero_mem_t out[4]) {
  if (!out) return zero_internal_fail(ZERO_EINVAL, "out is NULL");
  if (!(N >= 0)) return zero_internal_fail(ZERO_EINVAL, "N must be >= 0");
  if (Nd < 1) return zero_internal_fail(ZERO_EINVAL, "Nd must be >= 1");
  if (bytes_per_param < 0 || bytes_per_opt_state < 0)
    return zero_internal_fail(ZERO_EINVAL, "bytes_per_param and bytes_per_opt_state must be >= 0");
  const double gib = 1073741824.0;
  const double weights = N * bytes_per_param / gib;
  const double grads = N * bytes_per_param / gib;
  const double opt = N * bytes_per_opt_state / gib;
  const double d = Nd;
  const double shard_opt[4] = {1.0, d, d, d};  // divisor per stage
  const double shard_grad[4] = {1.0, 1.0, d, d};
  const double shard_w[4] = {1.0, 1.0, 1.0, d};
  for (int s = 0; s < 4; ++s) {
    out[s].optimizer_states = opt / shard_opt[s];
    out[s].gradients = grads / shard_grad[s];
    out[s].parameters = weights / shard_w[s];
    out[s].total = out[s].optimizer_states + out[s].gradients + out[s].parameters;
  }
  return ZERO_OK;
}

// [P1] §二 / §三, [P3] core operations.  A ring reduce-scatter or all-gather sends (Nd-1)/Nd of
// the vector per rank.  Plain DP: one all-reduce (= RS + AG).  ZeRO-1/2: RS of gradients + AG
// of weights.  ZeRO-3: AG of weights before forward, again before backward, RS of gradients.
double zero_comm_volume(int stage, double N, int Nd) {
  if (Nd < 1 || stage < 0 || stage > 3) return -1.0;
  const double per_collective = N * (double)(Nd - 1) / (double)Nd;
  const int collectives = stage == 3 ? 3 : 2;
  return collectives * per_collective;
}

}  // extern "C"
