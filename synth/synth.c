/*
 * Seeded synthetic-input generators shared by the CPU oracle, the tests and the
 * benchmark.  This file holds no arithmetic of the decoding method: it only
 * produces weights, prompts and window states from (seed, stream, index)
 * counters, so both sides of every parity check start from identical bytes.
 *
 * Generator: element i of stream s under seed q is
 *     u = mix64(key(q, s) + (i + 1) * 0x9E3779B97F4A7C15)
 * where mix64 is the SplitMix64 output finaliser (Steele, Lea and Flood,
 * "Fast splittable pseudorandom number generators", OOPSLA 2014).  Because
 * every element is a pure function of its index, the result does not depend on
 * the number of threads or on the order in which elements are produced.
 *
 * Normal-shaped weights use the Irwin-Hall sum of the four 16-bit lanes of u,
 * centred and scaled to the requested standard deviation.  Only integer
 * operations, one integer-to-float conversion (exact below 2^24) and one
 * correctly rounded fp32 multiply are involved, so the values are reproducible
 * on any IEEE-754 machine.  bf16 outputs are the round-to-nearest-even
 * truncation of those fp32 values.
 */
#include <stdint.h>
#include <stddef.h>
#include <math.h>

static inline uint64_t mix64(uint64_t z) {
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}

static inline uint64_t stream_key(uint64_t seed, uint64_t stream) {
    return mix64(mix64(seed ^ 0x5EEDULL) ^ (stream * 0xD1B54A32D192ED03ULL + 0x632BE59BD9B4E019ULL));
}

static inline uint64_t draw(uint64_t key, uint64_t i) {
    return mix64(key + (i + 1) * 0x9E3779B97F4A7C15ULL);
}

/* Irwin-Hall(4) sample centred on zero: an integer in [-131070, 131070]. */
static inline int32_t ih4(uint64_t u) {
    int32_t s = (int32_t)(u & 0xFFFF) + (int32_t)((u >> 16) & 0xFFFF)
              + (int32_t)((u >> 32) & 0xFFFF) + (int32_t)((u >> 48) & 0xFFFF);
    return s - 131070;
}

/* fp32 scale that maps the Irwin-Hall(4) integer to standard deviation `std`:
 * Var(sum of four uniform 16-bit lanes) = 65536^2 / 3 (to within 1e-9 rel). */
float synth_normal_scale(double std) {
    return (float)(std * sqrt(3.0) / 65536.0);
}

static inline uint16_t f32_to_bf16_rne(float f) {
    union { float f; uint32_t u; } v;
    v.f = f;
    uint32_t u = v.u;
    if ((u & 0x7F800000u) == 0x7F800000u) {           /* inf / nan */
        return (uint16_t)((u >> 16) | ((u & 0xFFFF) ? 0x40 : 0));
    }
    uint32_t lsb = (u >> 16) & 1u;
    u += 0x7FFFu + lsb;
    return (uint16_t)(u >> 16);
}

void synth_normal_f32(uint64_t seed, uint64_t stream, double std, float* out, int64_t n) {
    const uint64_t key = stream_key(seed, stream);
    const float c = synth_normal_scale(std);
    #pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) {
        out[i] = (float)ih4(draw(key, (uint64_t)i)) * c;
    }
}

void synth_normal_bf16(uint64_t seed, uint64_t stream, double std, uint16_t* out, int64_t n) {
    const uint64_t key = stream_key(seed, stream);
    const float c = synth_normal_scale(std);
    #pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) {
        out[i] = f32_to_bf16_rne((float)ih4(draw(key, (uint64_t)i)) * c);
    }
}

/* Uniform token ids in [0, vocab) with `exclude` (if >= 0) never produced. */
void synth_token_ids(uint64_t seed, uint64_t stream, int32_t vocab, int32_t exclude,
                     int32_t* out, int64_t n) {
    const uint64_t key = stream_key(seed, stream);
    const uint64_t span = (uint64_t)vocab - (exclude >= 0 && exclude < vocab ? 1u : 0u);
    #pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) {
        int32_t r = (int32_t)(draw(key, (uint64_t)i) % span);
        if (exclude >= 0 && exclude < vocab && r >= exclude) r += 1;
        out[i] = r;
    }
}

/* Uniform doubles in [0, 1) with 53 random bits. */
void synth_uniform01(uint64_t seed, uint64_t stream, double* out, int64_t n) {
    const uint64_t key = stream_key(seed, stream);
    #pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) {
        out[i] = (double)(draw(key, (uint64_t)i) >> 11) * (1.0 / 9007199254740992.0);
    }
}

/* Raw 64-bit draws (for tests of the generator itself). */
void synth_raw_u64(uint64_t seed, uint64_t stream, uint64_t* out, int64_t n) {
    const uint64_t key = stream_key(seed, stream);
    for (int64_t i = 0; i < n; ++i) out[i] = draw(key, (uint64_t)i);
}
