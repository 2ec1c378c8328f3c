/*
 * Seeded synthetic input generator shared by the CPU oracle and the CUDA path.
 *
 * It holds none of the attention method's arithmetic: it only turns
 * (seed, tensor id, element index) into a normal deviate and rounds it to
 * the storage type.  Every element is a pure function of its coordinates
 * (counter-based), so any token range of any tensor can be regenerated
 * independently and in any order, on any number of threads.
 *
 *   uniforms : Philox4x32-10 (Salmon, Moraes, Dror, Shaw, "Parallel random
 *              numbers: as easy as 1, 2, 3", SC'11), counter
 *              (g_lo, g_hi, tensor_id, 0x494E464C), key (seed_lo, seed_hi),
 *              where g = element_index / 4.
 *   normals  : Box-Muller in float32 on the two uniform pairs of each
 *              Philox output; element e takes output lane e % 4.
 *   rounding : float32 -> bfloat16 round-to-nearest-even (bf16 outputs).
 *
 * Built with -ffp-contract=off and no fast-math so that results are
 * bit-reproducible for a given libm.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#define PHILOX_M0 0xD2511F53u
#define PHILOX_M1 0xCD9E8D57u
#define PHILOX_W0 0x9E3779B9u
#define PHILOX_W1 0xBB67AE85u

static inline void philox4x32_10(const uint32_t ctr_in[4], const uint32_t key_in[2], uint32_t out[4]) {
    uint32_t c0 = ctr_in[0], c1 = ctr_in[1], c2 = ctr_in[2], c3 = ctr_in[3];
    uint32_t k0 = key_in[0], k1 = key_in[1];
    for (int r = 0; r < 10; ++r) {
        uint64_t p0 = (uint64_t)PHILOX_M0 * (uint64_t)c0;
        uint64_t p1 = (uint64_t)PHILOX_M1 * (uint64_t)c2;
        uint32_t hi0 = (uint32_t)(p0 >> 32), lo0 = (uint32_t)p0;
        uint32_t hi1 = (uint32_t)(p1 >> 32), lo1 = (uint32_t)p1;
        uint32_t n0 = hi1 ^ c1 ^ k0;
        uint32_t n1 = lo1;
        uint32_t n2 = hi0 ^ c3 ^ k1;
        uint32_t n3 = lo0;
        c0 = n0; c1 = n1; c2 = n2; c3 = n3;
        k0 += PHILOX_W0;
        k1 += PHILOX_W1;
    }
    out[0] = c0; out[1] = c1; out[2] = c2; out[3] = c3;
}

/* uniform in (0, 1]: 24 random bits, never zero (log stays finite) */
static inline float u01_open_low(uint32_t x) { return ((float)(x >> 8) + 1.0f) * (1.0f / 16777216.0f); }
/* uniform in [0, 1) */
static inline float u01(uint32_t x) { return (float)(x >> 8) * (1.0f / 16777216.0f); }

static inline void normal4(uint64_t g, uint32_t tensor_id, uint64_t seed, float z[4]) {
    uint32_t ctr[4] = {(uint32_t)g, (uint32_t)(g >> 32), tensor_id, 0x494E464Cu};
    uint32_t key[2] = {(uint32_t)seed, (uint32_t)(seed >> 32)};
    uint32_t r[4];
    philox4x32_10(ctr, key, r);
    const float two_pi = 6.28318530717958647692f;
    float ra = sqrtf(-2.0f * logf(u01_open_low(r[0])));
    float ta = two_pi * u01(r[1]);
    float rb = sqrtf(-2.0f * logf(u01_open_low(r[2])));
    float tb = two_pi * u01(r[3]);
    z[0] = ra * cosf(ta);
    z[1] = ra * sinf(ta);
    z[2] = rb * cosf(tb);
    z[3] = rb * sinf(tb);
}

static inline uint16_t f32_to_bf16_rne(float f) {
    uint32_t u;
    memcpy(&u, &f, 4);
    if ((u & 0x7fffffffu) > 0x7f800000u) return (uint16_t)((u >> 16) | 0x40u); /* quiet NaN */
    u += 0x7fffu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}

/*
 * Fill out[t][h][i] for t in [0, n_tok), h < n_head, i < dim with
 *     value = scale * z(seed, tensor_id, ((t0 + t) * n_head + h) * dim + i) + bias[h][i]
 * computed in float32, then stored as float32 (dtype 0) or bfloat16 bits (dtype 1).
 * bias may be NULL.  Parallel over tokens with OpenMP.
 */
void synth_normal(uint64_t seed, uint32_t tensor_id, int64_t t0, int64_t n_tok, int32_t n_head, int32_t dim,
                  float scale, const float* bias, int32_t dtype, void* out) {
    const int64_t row = (int64_t)n_head * dim;
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < n_tok; ++t) {
        const int64_t e0 = (t0 + t) * row;
        uint64_t g_cached = UINT64_MAX;
        float z4[4];
        for (int64_t j = 0; j < row; ++j) {
            const uint64_t e = (uint64_t)(e0 + j);
            const uint64_t g = e >> 2;
            if (g != g_cached) {
                normal4(g, tensor_id, seed, z4);
                g_cached = g;
            }
            float v = scale * z4[e & 3u];
            if (bias) v = v + bias[j];
            if (dtype == 0) {
                ((float*)out)[t * row + j] = v;
            } else {
                ((uint16_t*)out)[t * row + j] = f32_to_bf16_rne(v);
            }
        }
    }
}

/* Raw float32 normals z(seed, tensor_id, e) for e in [e0, e0 + n): used for small draws (biases, directions). */
void synth_normal_flat(uint64_t seed, uint32_t tensor_id, int64_t e0, int64_t n, float* out) {
#pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < n; ++j) {
        const uint64_t e = (uint64_t)(e0 + j);
        float z4[4];
        normal4(e >> 2, tensor_id, seed, z4);
        out[j] = z4[e & 3u];
    }
}

/* Raw Philox4x32-10 block, exposed so tests can check the published known-answer vectors. */
void synth_philox4x32_10(const uint32_t ctr[4], const uint32_t key[2], uint32_t out[4]) { philox4x32_10(ctr, key, out); }

/* float32 -> bfloat16 round-to-nearest-even for n values. */
void synth_round_bf16(const float* in, int64_t n, uint16_t* out) {
#pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < n; ++j) out[j] = f32_to_bf16_rne(in[j]);
}
