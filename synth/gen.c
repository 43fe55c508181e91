/*
 * Seeded synthetic input generator for the QK4V8 attention workloads.
 *
 * This module only draws random numbers and writes bf16 bit patterns. It holds
 * none of the quantization or attention arithmetic, and both the CPU oracle and
 * the CUDA path consume its output unchanged.
 *
 * Random numbers are counter based, so every element can be drawn
 * independently and in parallel:
 *   key(seed, stream)        = mix64(seed * 0x9E3779B97F4A7C15 + stream * 0xD1B54A32D192ED03 + 1)
 *   u64(seed, stream, index) = mix64(key + (index + 1) * 0x9E3779B97F4A7C15)
 * where mix64 is the splitmix64 output function (Steele, Lea, Flood,
 * "Fast splittable pseudorandom number generators", OOPSLA 2014).
 * A uniform in (0,1) is ((u >> 11) + 0.5) * 2^-53, and standard normals come in
 * pairs from the Box-Muller transform of two uniforms with consecutive indices.
 *
 * Tensors are written as bf16 bit patterns (round to nearest even from the
 * float32 value) in [B, T, H, D] order, T the token axis.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

static inline uint64_t mix64(uint64_t z) {
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}

static inline uint64_t stream_key(uint64_t seed, uint64_t stream) {
    return mix64(seed * 0x9E3779B97F4A7C15ULL + stream * 0xD1B54A32D192ED03ULL + 1ULL);
}

static inline uint64_t draw_u64(uint64_t key, uint64_t index) {
    return mix64(key + (index + 1ULL) * 0x9E3779B97F4A7C15ULL);
}

static inline double uniform01(uint64_t key, uint64_t index) {
    return ((double)(draw_u64(key, index) >> 11) + 0.5) * (1.0 / 9007199254740992.0);
}

/* Standard normal number `index` of a stream: Box-Muller on the uniform pair
 * (2*(index/2), 2*(index/2)+1); even indices take the cosine branch. */
static inline double normal_at(uint64_t key, uint64_t index) {
    uint64_t pair = index >> 1;
    double u1 = uniform01(key, 2 * pair);
    double u2 = uniform01(key, 2 * pair + 1);
    double r = sqrt(-2.0 * log(u1));
    double th = 6.283185307179586476925286766559 * u2;
    return (index & 1) ? r * sin(th) : r * cos(th);
}

static inline uint16_t f32_to_bf16_rne(float f) {
    uint32_t u;
    memcpy(&u, &f, 4);
    if ((u & 0x7F800000u) == 0x7F800000u) return (uint16_t)(u >> 16); /* never produced */
    uint32_t lsb = (u >> 16) & 1u;
    u += 0x7FFFu + lsb;
    return (uint16_t)(u >> 16);
}

enum { DIST_NORMAL = 0, DIST_STUDENT_T3 = 1 };

/*
 * Fill out[B][T][H][D] (bf16 bits) for the tokens t < T_valid[b] (T_valid may be
 * NULL: all tokens). Tokens at or past T_valid[b] are set to `pad_bits`.
 * dist: DIST_NORMAL draws N(0,1); DIST_STUDENT_T3 draws Z / sqrt(chi2_3 / 3) with
 * chi2_3 the sum of three squared standard normals (four normal streams).
 * chan_mult[H][D] (may be NULL) multiplies each value before rounding to bf16,
 * which is how outlier channels are planted.
 */
int synth_fill(uint16_t *out, int64_t B, int64_t T, int64_t H, int64_t D,
               const int32_t *T_valid, uint64_t seed, uint64_t stream, int dist,
               const float *chan_mult, uint16_t pad_bits) {
    if (!out || B < 0 || T < 0 || H <= 0 || D <= 0) return -1;
    const uint64_t k0 = stream_key(seed, stream * 4 + 0);
    const uint64_t k1 = stream_key(seed, stream * 4 + 1);
    const uint64_t k2 = stream_key(seed, stream * 4 + 2);
    const uint64_t k3 = stream_key(seed, stream * 4 + 3);
    const int64_t row = H * D;
    const int64_t rows = B * T;
#pragma omp parallel for schedule(static)
    for (int64_t bt = 0; bt < rows; ++bt) {
        const int64_t b = bt / T, t = bt % T;
        uint16_t *dst = out + bt * row;
        const int64_t tv = T_valid ? (int64_t)T_valid[b] : T;
        if (t >= tv) {
            for (int64_t i = 0; i < row; ++i) dst[i] = pad_bits;
            continue;
        }
        for (int64_t i = 0; i < row; ++i) {
            const uint64_t idx = (uint64_t)(bt * row + i);
            double v = normal_at(k0, idx);
            if (dist == DIST_STUDENT_T3) {
                double a = normal_at(k1, idx), c = normal_at(k2, idx), e = normal_at(k3, idx);
                v = v / sqrt((a * a + c * c + e * e) / 3.0);
            }
            if (chan_mult) v *= (double)chan_mult[i];
            dst[i] = f32_to_bf16_rne((float)v);
        }
    }
    return 0;
}

/* Pick `n_pick` distinct channels out of `n` for each of `groups` groups with a
 * seeded partial Fisher-Yates shuffle; out[groups][n_pick]. */
int synth_pick_channels(int32_t *out, int groups, int n, int n_pick, uint64_t seed, uint64_t stream) {
    if (!out || n_pick > n || n <= 0 || n > 4096) return -1;
    int32_t perm[4096];
    for (int g = 0; g < groups; ++g) {
        const uint64_t key = stream_key(seed, stream * 4096 + (uint64_t)g);
        for (int i = 0; i < n; ++i) perm[i] = i;
        for (int i = 0; i < n_pick; ++i) {
            uint64_t r = draw_u64(key, (uint64_t)i);
            int j = i + (int)(r % (uint64_t)(n - i));
            int32_t tmp = perm[i]; perm[i] = perm[j]; perm[j] = tmp;
            out[g * n_pick + i] = perm[i];
        }
    }
    return 0;
}

/* Integers uniform in [lo, hi] (inclusive), one per index. */
int synth_uniform_ints(int32_t *out, int64_t n, int32_t lo, int32_t hi, uint64_t seed, uint64_t stream) {
    if (!out || hi < lo) return -1;
    const uint64_t key = stream_key(seed, stream);
    const uint64_t span = (uint64_t)((int64_t)hi - (int64_t)lo + 1);
    for (int64_t i = 0; i < n; ++i) out[i] = lo + (int32_t)(draw_u64(key, (uint64_t)i) % span);
    return 0;
}

int synth_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
