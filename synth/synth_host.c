/* synth_host.c -- host (C) implementation of the seeded input generator of synth/__init__.py.
 *
 * Test and benchmark infrastructure, the fast twin of the numpy reference implementation
 * (same definition, bit for bit; a CPU test checks they agree).  It holds none of the
 * optimizer's arithmetic. */
#include <stdint.h>
#include <string.h>

static const uint64_t GAMMA = 0x9E3779B97F4A7C15ull;
static const uint64_t TAIL = 1ull << 62;

static uint64_t mix(uint64_t z)
{
    z ^= z >> 30;
    z *= 0xBF58476D1CE4E5B9ull;
    z ^= z >> 27;
    z *= 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

static uint64_t out(uint64_t s, uint64_t k) { return mix(s + (k + 1) * GAMMA); }

static uint32_t fields16(uint64_t h)
{
    return (uint32_t)(h & 0xFFFF) + (uint32_t)((h >> 16) & 0xFFFF) + (uint32_t)((h >> 32) & 0xFFFF) +
           (uint32_t)(h >> 48);
}

/* dtype 0 bf16 (upper 16 bits), 1 fp16 (round to nearest even), 2 fp32;
 * kind 0 normal, 1 abs, 2 square, 3 heavy, 4 zero. */
int synth_fill_host(void *dst, int dtype, int kind, uint64_t seed, uint64_t stream, int64_t first,
                    int64_t n, float sigma, float tail_sigma, uint32_t tail_mod)
{
    if (n < 0 || first < 0 || dtype < 0 || dtype > 2 || kind < 0 || kind > 4) return -1;
    if (kind == 3 && tail_mod == 0) return -1;
    uint64_t s = out(seed, stream), st = out(seed, stream ^ TAIL);
    for (int64_t e = 0; e < n; e++) {
        uint64_t k = (uint64_t)(first + e);
        float x = 0.0f;
        if (kind != 4) {
            uint32_t total = fields16(out(s, 3 * k)) + fields16(out(s, 3 * k + 1)) + fields16(out(s, 3 * k + 2));
            float z = (float)((int32_t)total - 393210) * 1.52587890625e-05f; /* 2^-16, exact */
            float sg = sigma;
            if (kind == 3 && (out(st, k) % tail_mod) == 0) sg = tail_sigma;
            x = z * sg;
            if (kind == 1 && x < 0.0f) x = -x;
            if (kind == 2) x = x * x;
        }
        if (dtype == 2) {
            ((float *)dst)[e] = x;
        } else if (dtype == 1) {
            _Float16 h = (_Float16)x;
            memcpy((uint16_t *)dst + e, &h, 2);
        } else {
            uint32_t u;
            memcpy(&u, &x, 4);
            ((uint16_t *)dst)[e] = (uint16_t)(u >> 16);
        }
    }
    return 0;
}
