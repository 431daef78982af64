/*
 * synth.c - seeded synthetic inputs for the TIDE hot path (host side).
 *
 * This file draws the bf16 values that stand in for gradients and all-gather
 * shards.  It knows nothing about sharding, layouts or reductions: it fills a
 * flat array of n elements, element idx taking a value that depends only on
 * (seed, stream, rank, param, idx).  Both the CPU oracle and the CUDA path get
 * their inputs from here (or from the bit-identical device twin in
 * synth_dev.cu); neither side's arithmetic lives here.
 *
 * Value recipe, per element:
 *   key = sm64(sm64(seed) ^ (stream << 48 ^ rank << 32 ^ param))
 *   h   = sm64(key ^ idx)
 *   s   = lane0(h) + lane1(h) + lane2(h) + lane3(h) - 131070   (16-bit lanes)
 *   x   = fl32((float)s * fl32(sigma / 37837.2272372))
 *   out = bf16 round-to-nearest-even of x
 * sm64 is the SplitMix64 output function (Steele, Lea and Flood, "Fast
 * splittable pseudorandom number generators", OOPSLA 2014; constants as in
 * Vigna's public-domain splitmix64.c): add the golden gamma, then two
 * xor-shift-multiply rounds and a final xor-shift.  s is an Irwin-Hall(4)
 * variate centred at zero; 37837.2272... is its standard deviation
 * (sqrt(4 * (65536^2 - 1) / 12)), so x is approximately N(0, sigma).  The
 * pipeline is integer-only apart from one fp32 multiply, so host and device
 * produce identical bits.
 */
#include <stdint.h>
#include <string.h>

#define SYNTH_GAMMA 0x9e3779b97f4a7c15ULL

uint64_t synth_splitmix64(uint64_t x) {
    uint64_t z = x + SYNTH_GAMMA;
    z = (z ^ (z >> 30)) * 0xbf58476d1ce4e5b9ULL;
    z = (z ^ (z >> 27)) * 0x94d049bb133111ebULL;
    return z ^ (z >> 31);
}

uint64_t synth_key(uint64_t seed, uint64_t stream, uint64_t rank, uint64_t param) {
    return synth_splitmix64(synth_splitmix64(seed) ^ ((stream << 48) ^ (rank << 32) ^ param));
}

/* fl32(sigma / 37837.2272372): the per-unit multiplier applied to s. */
float synth_sigma_scale(double sigma) {
    return (float)(sigma / 37837.2272372);
}

static uint16_t f32_to_bf16_rne(float x) {
    uint32_t u;
    memcpy(&u, &x, 4);
    u += 0x7fffu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}

static uint16_t value_at(uint64_t key, uint64_t idx, float mul) {
    uint64_t h = synth_splitmix64(key ^ idx);
    int32_t s = (int32_t)(h & 0xffff) + (int32_t)((h >> 16) & 0xffff) +
                (int32_t)((h >> 32) & 0xffff) + (int32_t)(h >> 48) - 131070;
    volatile float x = (float)s * mul; /* one fp32 multiply, no contraction */
    return f32_to_bf16_rne(x);
}

/* Fill out[0..n) with the values of (seed, stream, rank, param) at idx0+0..n-1. */
void synth_fill_bf16(uint16_t* out, int64_t n, uint64_t idx0, uint64_t seed,
                     uint64_t stream, uint64_t rank, uint64_t param, float mul) {
    uint64_t key = synth_key(seed, stream, rank, param);
    /* every element is independent, so threads cannot change the result */
#pragma omp parallel for schedule(static) if (n > (1 << 20))
    for (int64_t j = 0; j < n; ++j) out[j] = value_at(key, idx0 + (uint64_t)j, mul);
}

/* Values at an arbitrary list of indices (for sampled checks at full size). */
void synth_gather_bf16(uint16_t* out, const int64_t* idx, int64_t n, uint64_t seed,
                       uint64_t stream, uint64_t rank, uint64_t param, float mul) {
    uint64_t key = synth_key(seed, stream, rank, param);
    for (int64_t j = 0; j < n; ++j) out[j] = value_at(key, (uint64_t)idx[j], mul);
}

/*
 * Unrouted experts: for one rank, mark n_zero of n_experts as "received no
 * tokens".  Each expert e gets the score h(seed, stream 2, rank, e, idx 0);
 * the n_zero lowest scores are chosen, ties broken by the lower e.
 */
void synth_zero_experts(uint8_t* mask, int32_t n_experts, int32_t n_zero,
                        uint64_t seed, uint64_t rank) {
    for (int32_t e = 0; e < n_experts; ++e) mask[e] = 0;
    for (int32_t pick = 0; pick < n_zero && pick < n_experts; ++pick) {
        int32_t best = -1;
        uint64_t best_score = 0;
        for (int32_t e = 0; e < n_experts; ++e) {
            if (mask[e]) continue;
            uint64_t sc = synth_splitmix64(synth_key(seed, 2, rank, (uint64_t)e));
            if (best < 0 || sc < best_score) { best = e; best_score = sc; }
        }
        mask[best] = 1;
    }
}
