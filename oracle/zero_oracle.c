/*
 * zero_oracle.c -- CPU oracle for the sharded mixed-precision Adam step (ZeRO-1/2/3).
 *
 * TEST INFRASTRUCTURE, NOT PART OF THE PRODUCT.  Only the tests, the smoke check of
 * __graft_entry__ and the cpu_baseline leg of bench.py may load this library.  It shares
 * no code, header, table or helper with the CUDA library, and neither one includes or
 * links the other.
 *
 * Sources, cited by title and section:
 *   [P1] "ZeRO 优化器的三个阶段深度对比：显存节省与通信开销的量化分析" (wmrh.cn/news/520095)
 *   [P2] "ZeRO 优化器：把显存“分”着用" (5688vip.com course note, 多卡分布式训练显存优化与通信协同 03)
 *   [P3] "ZeRO Optimization（零冗余优化）" (ai-master.cc glossary entry)
 *
 * What is computed.  ZeRO only changes where each piece of model state is stored and which
 * rank updates it; the arithmetic is that of plain data parallelism ([P3] "vs 数据并行" and
 * "vs 模型并行": the computation graph is unchanged, only storage is sharded).  So every
 * stage computes, per element: the data-parallel mean of the Nd gradient replicas, one
 * Adam/AdamW step on fp32 master weights and moments, and a bf16 copy of the new weights.
 * This file writes each stage out with its own loops over ranks and shards:
 *   ZeRO-1/2 ([P1] §二, [P2] "ZeRO Stage 1/2"): reduce-scatter of the gradients into each
 *     rank's contiguous 1/Nd shard, Adam on that shard, all-gather of the bf16 weights.
 *   ZeRO-3 ([P1] §三, [P2] "ZeRO Stage 3", [P3] core operations): per layer, all-gather of
 *     the layer's bf16 weights from the Nd shards just before use, reduce-scatter of the
 *     layer's gradients after backward, then Adam on each shard and a bf16 copy kept in
 *     the shard only.
 *   Plain data parallelism ([P1] §一, [P2] "ZeRO Stage 2" all-reduce): all-reduce, Adam on
 *     the full vector, every replica receives the new weights.  It is the reference the
 *     sharded stages must equal.
 *   Per-GPU memory and per-rank communication volume ([P1] §二 code and §三, [P3]).
 *
 * Readings where the pages are silent (every one is also listed in the design notes):
 *   - The update rule is not printed anywhere (the pages name only the fp32 copy and the two
 *     moments, [P1] §一, [P2] "ZeRO Stage 1").  Read as textbook Adam with bias correction
 *     (Kingma & Ba, 2015) and decoupled weight decay (AdamW, Loshchilov & Hutter, 2019), with
 *     eps added after the bias-corrected square root:
 *         p <- p * (1 - lr*wd)
 *         m <- b1*m + (1-b1)*g
 *         v <- b2*v + ((1-b2)*g)*g
 *         p <- p - (lr/(1-b1^t)) * (m / (sqrt(v)/sqrt(1-b2^t) + eps))
 *     every operation one fp32 round-to-nearest step, no fused multiply-add.  With wd = 0 the
 *     first line is skipped (it would multiply by exactly 1).
 *   - Scalars that do not depend on the element (1-b1, 1-b2, 1-lr*wd, lr/(1-b1^t),
 *     sqrt(1-b2^t), 1/(Nd*loss_scale)) are computed once in double and rounded once to fp32.
 *   - The reduced gradient is the mean over ranks (data-parallel all-reduce averages) divided
 *     by the loss scale: g = (sum over ranks, fp32, rank 0 first) * (1/(Nd*loss_scale)).
 *     A plain sum is available with grad_average = 0.
 *   - Overflow: if any reduced gradient element is inf or NaN anywhere in the vector, the
 *     whole step is skipped: master, m, v and the bf16 replicas keep their values and the
 *     step counter t is not advanced.
 *   - Shard r of a vector of N elements is [r*S, min((r+1)*S, N)) with S = ceil(N/Nd); the
 *     padded length is Nd*S and pad elements are zero.
 *   - fp32 -> bf16 is round to nearest, ties to even.
 *   - Communication volume counts elements sent per rank by ring collectives.
 *
 * Everything here is plain, single-threaded, one element per loop iteration.  It is built
 * with -O2 -ffp-contract=off and without -ffast-math so that every float operation is one
 * IEEE round-to-nearest step.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_BF16 0
#define ORACLE_FP16 1

/* ---------------------------------------------------------------- partition */

/* [P1] §二: each rank keeps 1/Nd of the optimizer state; [P3] core operations: each process
 * keeps only its own shard.  out = {S, padded length Nd*S, pad count}. */
int oracle_partition(int64_t N, int Nd, int64_t out[3])
{
    if (N < 0 || Nd < 1) return -1;
    int64_t S = N / Nd;
    if (S * Nd < N) S = S + 1; /* ceil(N / Nd) */
    out[0] = S;
    out[1] = S * Nd;
    out[2] = S * Nd - N;
    return 0;
}

/* Rank that owns global element i. */
int64_t oracle_owner(int64_t i, int64_t S)
{
    return i / S;
}

/* ---------------------------------------------------------------- number formats */

/* bf16 is the upper half of an IEEE binary32 word. */
float oracle_bf16_to_f32(uint16_t h)
{
    uint32_t u = ((uint32_t)h) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* IEEE binary16: 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits. */
float oracle_f16_to_f32(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 0x1f;
    int frac = h & 0x3ff;
    double mag;
    if (e == 0)
        mag = ldexp((double)frac, -24);              /* subnormal: frac * 2^-24 */
    else if (e == 31)
        mag = frac ? (double)NAN : (double)INFINITY; /* inf / NaN */
    else
        mag = ldexp((double)(1024 + frac), e - 25);  /* (1 + frac/1024) * 2^(e-15) */
    float f = (float)mag;
    return sign ? -f : f;
}

/* fp32 -> bf16, round to nearest, ties to even.  NaN stays NaN (quiet bit set). */
uint16_t oracle_f32_to_bf16(float f)
{
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    if (isnan(f)) return (uint16_t)((u >> 16) | 0x0040);
    uint32_t kept = u >> 16;
    uint32_t dropped = u & 0xffffu;
    if (dropped > 0x8000u || (dropped == 0x8000u && (kept & 1u))) kept = kept + 1u;
    return (uint16_t)kept;
}

static float grad_value(const uint16_t *g, int64_t i, int dtype)
{
    return dtype == ORACLE_FP16 ? oracle_f16_to_f32(g[i]) : oracle_bf16_to_f32(g[i]);
}

/* ---------------------------------------------------------------- step scalars */

typedef struct {
    float inv;        /* 1/(Nd*loss_scale) (mean) or 1/loss_scale (sum) */
    float beta1, beta2, omb1, omb2, eps;
    float decay;      /* 1 - lr*wd */
    float step_size;  /* lr / (1 - beta1^t) */
    float sbc2;       /* sqrt(1 - beta2^t) */
    int apply_decay;  /* wd != 0 */
} oracle_scalars_t;

/* hp = {lr, beta1, beta2, eps, weight_decay, loss_scale, grad_average} */
void oracle_scalars(const double hp[7], int Nd, int64_t t, oracle_scalars_t *c)
{
    double lr = hp[0], b1 = hp[1], b2 = hp[2], eps = hp[3], wd = hp[4], ls = hp[5];
    int average = hp[6] != 0.0;
    double denom = average ? (double)Nd * ls : ls;
    c->inv = (float)(1.0 / denom);
    c->beta1 = (float)b1;
    c->beta2 = (float)b2;
    c->omb1 = (float)(1.0 - b1);
    c->omb2 = (float)(1.0 - b2);
    c->eps = (float)eps;
    c->decay = (float)(1.0 - lr * wd);
    c->apply_decay = wd != 0.0;
    double bc1 = 1.0 - pow(b1, (double)t);
    double bc2 = 1.0 - pow(b2, (double)t);
    c->step_size = (float)(lr / bc1);
    c->sbc2 = (float)sqrt(bc2);
}

/* ---------------------------------------------------------------- collectives + Adam */

/* Reduce-scatter ([P1] §二 ZeRO-2, [P3] backward: ReduceScatter).  Rank r receives the reduced
 * gradient of its own shard.  `out` holds the Nd shards back to back (Nd*S floats); pad
 * elements are written as 0.  Elements are reduced in rank order 0..Nd-1.  Only global
 * elements in [lo, hi) are produced (a window of the flat vector; [0, N) for no bucketing). */
void oracle_reduce_scatter_window(int Nd, int64_t N, int dtype, const uint16_t *const *grads,
                                  float inv, int64_t lo, int64_t hi, float *out,
                                  int *overflow, double *sumsq)
{
    int64_t part[3] = {0, 0, 0};
    oracle_partition(N, Nd, part);
    int64_t S = part[0];
    for (int r = 0; r < Nd; r++) {
        for (int64_t k = 0; k < S; k++) {
            int64_t i = (int64_t)r * S + k;
            if (i < lo || i >= hi) continue;
            if (i >= N) {
                out[i] = 0.0f;
                continue;
            }
            float s = 0.0f;
            for (int q = 0; q < Nd; q++) s = s + grad_value(grads[q], i, dtype);
            float g = s * inv;
            out[i] = g;
            if (!isfinite(g)) *overflow = 1;
            *sumsq += (double)g * (double)g;
        }
    }
}

/* One Adam/AdamW update of n consecutive elements (one rank's shard). */
void oracle_adam(float *p, float *m, float *v, const float *g, int64_t n, const oracle_scalars_t *c)
{
    for (int64_t i = 0; i < n; i++) {
        float pi = p[i];
        if (c->apply_decay) pi = pi * c->decay;
        float mi = c->beta1 * m[i] + c->omb1 * g[i];
        float vi = c->beta2 * v[i] + (c->omb2 * g[i]) * g[i];
        float den = sqrtf(vi) / c->sbc2 + c->eps;
        pi = pi - c->step_size * (mi / den);
        p[i] = pi;
        m[i] = mi;
        v[i] = vi;
    }
}

/* All-gather ([P1] §二 ZeRO-1, [P3] forward: AllGather): every destination replica receives
 * every rank's shard of the new weights, as bf16. */
void oracle_allgather(int Nd, int64_t N, const float *master, uint16_t *const *replicas)
{
    int64_t part[3] = {0, 0, 0};
    oracle_partition(N, Nd, part);
    int64_t S = part[0];
    for (int dst = 0; dst < Nd; dst++)
        for (int r = 0; r < Nd; r++)
            for (int64_t k = 0; k < S; k++) {
                int64_t i = (int64_t)r * S + k;
                if (i < N) replicas[dst][i] = oracle_f32_to_bf16(master[i]);
            }
}

static int64_t shard_len(int64_t N, int64_t S, int r)
{
    int64_t lo = (int64_t)r * S;
    if (lo >= N) return 0;
    return (N - lo < S) ? (N - lo) : S;
}

/* ZeRO-1/2 step ([P1] §二, [P2] "ZeRO Stage 1" / "ZeRO Stage 2").  master/m/v hold Nd*S
 * floats (the shards back to back).  `bucket` > 0 runs the reduce-scatter over windows
 * [k*bucket, (k+1)*bucket) of the flat vector; 0 means one window.  On overflow nothing is
 * written and t is unchanged.  Returns 0, or -1 on bad arguments / no memory. */
int oracle_zero12_step(int Nd, int64_t N, int64_t bucket, int dtype,
                       const uint16_t *const *grads, float *master, float *m, float *v,
                       uint16_t *const *replicas, const double hp[7], int64_t *t,
                       int *overflow, double *sumsq)
{
    int64_t part[3] = {0, 0, 0};
    if (oracle_partition(N, Nd, part) != 0 || bucket < 0) return -1;
    int64_t S = part[0], Np = part[1];
    float *g = (float *)malloc((size_t)(Np > 0 ? Np : 1) * sizeof(float));
    if (!g) return -1;
    oracle_scalars_t c;
    oracle_scalars(hp, Nd, 1, &c); /* only c.inv is used before the skip decision */
    *overflow = 0;
    *sumsq = 0.0;
    int64_t w = bucket > 0 ? bucket : (Np > 0 ? Np : 1);
    for (int64_t lo = 0; lo < Np; lo += w) {
        int64_t hi = lo + w < Np ? lo + w : Np;
        oracle_reduce_scatter_window(Nd, N, dtype, grads, c.inv, lo, hi, g, overflow, sumsq);
    }
    if (*overflow) {
        free(g);
        return 0;
    }
    *t = *t + 1;
    oracle_scalars(hp, Nd, *t, &c);
    for (int r = 0; r < Nd; r++) {
        int64_t off = (int64_t)r * S;
        oracle_adam(master + off, m + off, v + off, g + off, shard_len(N, S, r), &c);
    }
    oracle_allgather(Nd, N, master, replicas);
    free(g);
    return 0;
}

/* Plain data parallelism ([P1] §一, [P2] "ZeRO Stage 2": all-reduce of the gradients): every
 * rank holds the full state; the all-reduced gradient updates the full vector and every
 * replica gets the new weights.  Same arguments as oracle_zero12_step (master/m/v hold N). */
int oracle_dp_step(int Nd, int64_t N, int dtype, const uint16_t *const *grads, float *master,
                   float *m, float *v, uint16_t *const *replicas, const double hp[7],
                   int64_t *t, int *overflow, double *sumsq)
{
    if (N < 0 || Nd < 1) return -1;
    float *g = (float *)malloc((size_t)(N > 0 ? N : 1) * sizeof(float));
    if (!g) return -1;
    oracle_scalars_t c;
    oracle_scalars(hp, Nd, 1, &c);
    *overflow = 0;
    *sumsq = 0.0;
    for (int64_t i = 0; i < N; i++) {
        float s = 0.0f;
        for (int q = 0; q < Nd; q++) s = s + grad_value(grads[q], i, dtype);
        g[i] = s * c.inv;
        if (!isfinite(g[i])) *overflow = 1;
        *sumsq += (double)g[i] * (double)g[i];
    }
    if (*overflow) {
        free(g);
        return 0;
    }
    *t = *t + 1;
    oracle_scalars(hp, Nd, *t, &c);
    oracle_adam(master, m, v, g, N, &c);
    for (int q = 0; q < Nd; q++)
        for (int64_t i = 0; i < N; i++) replicas[q][i] = oracle_f32_to_bf16(master[i]);
    free(g);
    return 0;
}

/* ZeRO-3 just-in-time gather of one layer ([P1] §三, [P2] "ZeRO Stage 3", [P3] forward):
 * rebuild the layer's L weights from its Nd shards of length S = ceil(L/Nd). */
void oracle_zero3_gather(int Nd, int64_t L, const uint16_t *const *shards, uint16_t *full)
{
    int64_t part[3] = {0, 0, 0};
    oracle_partition(L, Nd, part);
    int64_t S = part[0];
    for (int r = 0; r < Nd; r++)
        for (int64_t k = 0; k < S; k++) {
            int64_t j = (int64_t)r * S + k;
            if (j < L) full[j] = shards[r][k];
        }
}

/* One ZeRO-3 step over `nlayers` layers of lengths layer_len[].  Each layer is one flat unit
 * sharded contiguously; layer l occupies Nd*S_l padded elements of master/m/v/shard16 (the
 * layers back to back).  For every layer: gather the full bf16 weights from the Nd shards
 * into gathered[l*Nd + dst] (skipped when gathered is NULL), then reduce-scatter the layer's
 * gradient replicas grads[l*Nd + q] into the fp32 gradient shard.  After the last layer: skip
 * on overflow, else Adam on every shard and shard16 = bf16(master) (no all-gather; the next
 * forward gathers). */
int oracle_zero3_step(int Nd, int nlayers, const int64_t *layer_len, int dtype,
                      const uint16_t *const *grads, float *master, float *m, float *v,
                      uint16_t *shard16, uint16_t *const *gathered, const double hp[7],
                      int64_t *t, int *overflow, double *sumsq)
{
    if (Nd < 1 || nlayers < 0) return -1;
    int64_t total = 0;
    for (int l = 0; l < nlayers; l++) {
        int64_t part[3] = {0, 0, 0};
        if (oracle_partition(layer_len[l], Nd, part) != 0) return -1;
        total += part[1];
    }
    float *g = (float *)malloc((size_t)(total > 0 ? total : 1) * sizeof(float));
    const uint16_t **sh = (const uint16_t **)malloc(sizeof(uint16_t *) * (size_t)Nd);
    if (!g || !sh) {
        free(g);
        free(sh);
        return -1;
    }
    oracle_scalars_t c;
    oracle_scalars(hp, Nd, 1, &c);
    *overflow = 0;
    *sumsq = 0.0;
    int64_t off = 0;
    for (int l = 0; l < nlayers; l++) {
        int64_t part[3] = {0, 0, 0};
        oracle_partition(layer_len[l], Nd, part);
        int64_t S = part[0];
        for (int r = 0; r < Nd; r++) sh[r] = shard16 + off + (int64_t)r * S;
        if (gathered)
            for (int dst = 0; dst < Nd; dst++)
                oracle_zero3_gather(Nd, layer_len[l], sh, gathered[(int64_t)l * Nd + dst]);
        oracle_reduce_scatter_window(Nd, layer_len[l], dtype, grads + (int64_t)l * Nd, c.inv, 0,
                                     part[1], g + off, overflow, sumsq);
        off += part[1];
    }
    if (*overflow) {
        free(g);
        free(sh);
        return 0;
    }
    *t = *t + 1;
    oracle_scalars(hp, Nd, *t, &c);
    off = 0;
    for (int l = 0; l < nlayers; l++) {
        int64_t part[3] = {0, 0, 0};
        oracle_partition(layer_len[l], Nd, part);
        int64_t S = part[0];
        for (int r = 0; r < Nd; r++) {
            int64_t o = off + (int64_t)r * S;
            int64_t n = shard_len(layer_len[l], S, r);
            oracle_adam(master + o, m + o, v + o, g + o, n, &c);
            for (int64_t k = 0; k < n; k++) shard16[o + k] = oracle_f32_to_bf16(master[o + k]);
        }
        off += part[1];
    }
    free(g);
    free(sh);
    return 0;
}

/* Same element-wise update evaluated for a list of independent elements (sampled checks at
 * sizes where the full vector is too large for the host).  For element e: the Nd gradient
 * values grads[e*Nd + q], the state p/m/v[e] (updated in place), the bf16 result out16[e].
 * The caller supplies the overflow decision of the full vector (`skip`). */
void oracle_update_elements(int Nd, int64_t n, int dtype, const uint16_t *grads, float *p,
                            float *m, float *v, uint16_t *out16, float *gout,
                            const double hp[7], int64_t t_new, int skip)
{
    oracle_scalars_t c;
    oracle_scalars(hp, Nd, t_new, &c);
    for (int64_t e = 0; e < n; e++) {
        float s = 0.0f;
        for (int q = 0; q < Nd; q++) s = s + grad_value(grads, e * Nd + q, dtype);
        float g = s * c.inv;
        if (gout) gout[e] = g;
        if (!skip) oracle_adam(p + e, m + e, v + e, &g, 1, &c);
        out16[e] = oracle_f32_to_bf16(p[e]);
    }
}

/* ---------------------------------------------------------------- accounting */

typedef struct {
    double optimizer_states, gradients, parameters, total; /* GiB (2^30 bytes) */
} oracle_mem_t;

/* Per-GPU model-state memory of plain data parallelism and of the three ZeRO stages
 * ([P1] §二 code: 2-byte parameters and gradients, 12 bytes of Adam state = fp32 copy + m + v;
 * stage 1 divides the optimizer state by Nd, stage 2 also the gradients, stage 3 everything).
 * out[0] = DP, out[1] = ZeRO-1, out[2] = ZeRO-2, out[3] = ZeRO-3. */
void oracle_memory_estimate(double N, int Nd, int bytes_per_param, int bytes_per_opt_state,
                            oracle_mem_t out[4])
{
    const double GiB = 1024.0 * 1024.0 * 1024.0;
    double P = N * bytes_per_param;   /* 16-bit weights */
    double G = N * bytes_per_param;   /* 16-bit gradients */
    double O = N * bytes_per_opt_state;
    double d = (double)Nd;
    double o[4] = {O, O / d, O / d, O / d};
    double g[4] = {G, G, G / d, G / d};
    double p[4] = {P, P, P, P / d};
    for (int s = 0; s < 4; s++) {
        out[s].optimizer_states = o[s] / GiB;
        out[s].gradients = g[s] / GiB;
        out[s].parameters = p[s] / GiB;
        out[s].total = (s == 3 ? (O + G + P) / d : o[s] + g[s] + p[s]) / GiB;
    }
}

/* Elements each rank sends in one training step with ring collectives ([P1] §二 and §三,
 * [P3] core operations).  A ring reduce-scatter or all-gather of N elements sends
 * (Nd-1)/Nd*N per rank; an all-reduce is one of each.
 *   stage 0 (plain DP): all-reduce of the gradients.
 *   stage 1, 2: reduce-scatter of the gradients + all-gather of the weights.
 *   stage 3: all-gather of the weights in forward and again in backward + reduce-scatter. */
double oracle_comm_volume(int stage, double N, int Nd)
{
    double one = (double)(Nd - 1) / (double)Nd * N;
    if (stage == 0 || stage == 1 || stage == 2) return 2.0 * one;
    if (stage == 3) return 3.0 * one;
    return -1.0;
}

/* ---------------------------------------------------------------- array helpers */

void oracle_bf16_array_to_f32(const uint16_t *src, float *dst, int64_t n)
{
    for (int64_t i = 0; i < n; i++) dst[i] = oracle_bf16_to_f32(src[i]);
}

void oracle_f16_array_to_f32(const uint16_t *src, float *dst, int64_t n)
{
    for (int64_t i = 0; i < n; i++) dst[i] = oracle_f16_to_f32(src[i]);
}

void oracle_f32_array_to_bf16(const float *src, uint16_t *dst, int64_t n)
{
    for (int64_t i = 0; i < n; i++) dst[i] = oracle_f32_to_bf16(src[i]);
}

/* ---------------------------------------------------------------- loss scaler and clipping */

/* Dynamic loss scaling (the pages only name mixed precision, [P3] "vs 混合精度"; reading: the
 * standard backoff / growth rule).  After a step that overflowed, the scale is multiplied by
 * `backoff` and the count of clean steps restarts; after `interval` clean steps in a row it is
 * multiplied by `growth`, unless that would take it past the largest finite fp32 value (the
 * scale multiplies fp32 losses, so it must stay finite there). */
void oracle_scaler_update(double *scale, int64_t *good, int overflow, double growth, double backoff,
                          int64_t interval)
{
    const double fp32_max = 3.4028234663852886e38;
    if (overflow) {
        *scale = *scale * backoff;
        *good = 0;
        return;
    }
    *good = *good + 1;
    if (*good >= interval) {
        double grown = *scale * growth;
        if (grown <= fp32_max) *scale = grown;
        *good = 0;
    }
}

/* Global-norm clipping factor (reading: the usual rule, g <- g * min(1, max_norm/(||g|| + 1e-6)),
 * with ||g|| the 2-norm of the whole reduced, unscaled gradient).  Evaluated in double, rounded
 * once to fp32; 1 when max_norm <= 0 (no clipping). */
float oracle_clip_coef(double sumsq, double max_norm)
{
    if (!(max_norm > 0.0)) return 1.0f;
    double coef = max_norm / (sqrt(sumsq) + 1e-6);
    if (coef > 1.0) coef = 1.0;
    return (float)coef;
}

/* Reduce-scatter whose result is kept as bf16 (16-bit gradient partitions, a memory-saving
 * variant the pages do not describe; reading: the reduced fp32 mean is rounded to bf16, nearest
 * even, and the overflow check, the sum of squares and the update all use the rounded value).
 * `out` receives the rounded values widened back to fp32. */
void oracle_reduce_scatter_window_bf16(int Nd, int64_t N, int dtype, const uint16_t *const *grads,
                                       float inv, int64_t lo, int64_t hi, float *out, int *overflow,
                                       double *sumsq)
{
    int64_t part[3] = {0, 0, 0};
    oracle_partition(N, Nd, part);
    int64_t S = part[0];
    for (int r = 0; r < Nd; r++) {
        for (int64_t k = 0; k < S; k++) {
            int64_t i = (int64_t)r * S + k;
            if (i < lo || i >= hi) continue;
            if (i >= N) {
                out[i] = 0.0f;
                continue;
            }
            float s = 0.0f;
            for (int q = 0; q < Nd; q++) s = s + grad_value(grads[q], i, dtype);
            float g = oracle_bf16_to_f32(oracle_f32_to_bf16(s * inv));
            out[i] = g;
            if (!isfinite(g)) *overflow = 1;
            *sumsq += (double)g * (double)g;
        }
    }
}

/* ZeRO-1/2 step with the extensions.  hpx = {lr, beta1, beta2, eps, weight_decay,
 * loss_scale, grad_average, max_grad_norm, growth, backoff, interval, dynamic, bf16_grad}
 * (bf16_grad != 0: the reduced gradient is kept as bf16, see above).  With dynamic
 * != 0 the gradients carry the scale *scale (updated on return, with *good) instead of
 * hpx[5].  Order: reduce-scatter (mean, unscaled), overflow check, clipping of the reduced
 * gradient, Adam per shard, all-gather, scaler update. */
int oracle_zero12_step_ex(int Nd, int64_t N, int64_t bucket, int dtype, const uint16_t *const *grads,
                          float *master, float *m, float *v, uint16_t *const *replicas,
                          const double hpx[13], int64_t *t, double *scale, int64_t *good,
                          int *overflow, double *sumsq)
{
    int64_t part[3] = {0, 0, 0};
    if (oracle_partition(N, Nd, part) != 0 || bucket < 0) return -1;
    int64_t S = part[0], Np = part[1];
    double hp[7];
    for (int k = 0; k < 7; k++) hp[k] = hpx[k];
    int dynamic = hpx[11] != 0.0;
    if (dynamic) hp[5] = *scale;
    float *g = (float *)malloc((size_t)(Np > 0 ? Np : 1) * sizeof(float));
    if (!g) return -1;
    oracle_scalars_t c;
    oracle_scalars(hp, Nd, 1, &c);
    *overflow = 0;
    *sumsq = 0.0;
    int64_t w = bucket > 0 ? bucket : (Np > 0 ? Np : 1);
    for (int64_t lo = 0; lo < Np; lo += w) {
        int64_t hi = lo + w < Np ? lo + w : Np;
        if (hpx[12] != 0.0)
            oracle_reduce_scatter_window_bf16(Nd, N, dtype, grads, c.inv, lo, hi, g, overflow, sumsq);
        else
            oracle_reduce_scatter_window(Nd, N, dtype, grads, c.inv, lo, hi, g, overflow, sumsq);
    }
    if (!*overflow) {
        float coef = oracle_clip_coef(*sumsq, hpx[7]);
        for (int64_t i = 0; i < N; i++) g[i] = g[i] * coef;
        *t = *t + 1;
        oracle_scalars(hp, Nd, *t, &c);
        for (int r = 0; r < Nd; r++) {
            int64_t off = (int64_t)r * S;
            oracle_adam(master + off, m + off, v + off, g + off, shard_len(N, S, r), &c);
        }
        oracle_allgather(Nd, N, master, replicas);
    }
    if (dynamic) oracle_scaler_update(scale, good, *overflow, hpx[8], hpx[9], (int64_t)hpx[10]);
    free(g);
    return 0;
}

/* Sampled-element form of the extended step: element e's gradients, state and result as in
 * oracle_update_elements; the caller supplies the overflow decision, the clipping factor and
 * the loss scale of the full vector. */
void oracle_update_elements_ex(int Nd, int64_t n, int dtype, const uint16_t *grads, float *p, float *m,
                               float *v, uint16_t *out16, const double hp[7], int64_t t_new,
                               int skip, float coef)
{
    oracle_scalars_t c;
    oracle_scalars(hp, Nd, t_new, &c);
    for (int64_t e = 0; e < n; e++) {
        float s = 0.0f;
        for (int q = 0; q < Nd; q++) s = s + grad_value(grads, e * Nd + q, dtype);
        float g = (s * c.inv) * coef;
        if (!skip) oracle_adam(p + e, m + e, v + e, &g, 1, &c);
        out16[e] = oracle_f32_to_bf16(p[e]);
    }
}
