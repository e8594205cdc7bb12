/*
 * Seeded synthetic input generator, host side (plain C, OpenMP).
 *
 * This module holds no arithmetic of the serving iteration itself. It only
 * produces the inputs (weights, cached K/V, hidden states, token ids, batch
 * shapes) that both the CPU oracle and the CUDA path consume. The device-side
 * twin in synth_gpu.cu implements the same specification independently and is
 * tested for bitwise equality against this file.
 *
 * Specification
 * -------------
 * Counter-based generator: Philox4x32-10 (Salmon, Moraes, Dror, Shaw,
 * "Parallel random numbers: as easy as 1, 2, 3", SC'11), with the
 * multipliers 0xD2511F53 / 0xCD9E8D57 and Weyl key increments
 * 0x9E3779B9 / 0xBB67AE85.
 *
 *   key     = (seed, tensor_id)
 *   counter = (lo32(i), hi32(i), 0, 0) for element i of the tensor
 *
 * Normal values (Irwin-Hall of eight 16-bit uniforms):
 *   S     = sum of the eight 16-bit halves of the four output words (exact int)
 *   t     = (float)(S - 262140) * scale        one IEEE fp32 multiply
 *   v     = t + mean                           one IEEE fp32 add
 *   out   = bf16 round-to-nearest-even of v
 *   scale = (float)(sigma / sqrt(8 * (65536^2 - 1) / 12)), computed in double
 *           by the caller and passed in, so that sd(v) = sigma.
 *
 * Uniform integers in [lo, hi]: lo + ((uint64)word0 * (hi - lo + 1)) >> 32.
 */
#include <stdint.h>
#include <string.h>
#include <math.h>

#define PHILOX_M0 0xD2511F53u
#define PHILOX_M1 0xCD9E8D57u
#define PHILOX_W0 0x9E3779B9u
#define PHILOX_W1 0xBB67AE85u

static inline void philox_round(uint32_t c[4], const uint32_t k[2]) {
    uint64_t p0 = (uint64_t)PHILOX_M0 * c[0];
    uint64_t p1 = (uint64_t)PHILOX_M1 * c[2];
    uint32_t hi0 = (uint32_t)(p0 >> 32), lo0 = (uint32_t)p0;
    uint32_t hi1 = (uint32_t)(p1 >> 32), lo1 = (uint32_t)p1;
    uint32_t n0 = hi1 ^ c[1] ^ k[0];
    uint32_t n2 = hi0 ^ c[3] ^ k[1];
    c[0] = n0; c[1] = lo1; c[2] = n2; c[3] = lo0;
}

void nfs_philox4x32_10(const uint32_t ctr[4], const uint32_t key[2], uint32_t out[4]) {
    uint32_t c[4] = {ctr[0], ctr[1], ctr[2], ctr[3]};
    uint32_t k[2] = {key[0], key[1]};
    for (int r = 0; r < 10; ++r) {
        philox_round(c, k);
        if (r != 9) { k[0] += PHILOX_W0; k[1] += PHILOX_W1; }
    }
    memcpy(out, c, sizeof(c));
}

static inline void philox_at(uint32_t seed, uint32_t tid, uint64_t i, uint32_t out[4]) {
    uint32_t ctr[4] = {(uint32_t)i, (uint32_t)(i >> 32), 0u, 0u};
    uint32_t key[2] = {seed, tid};
    nfs_philox4x32_10(ctr, key, out);
}

static inline int32_t irwin_hall_centered(const uint32_t w[4]) {
    int32_t s = 0;
    for (int j = 0; j < 4; ++j) s += (int32_t)(w[j] & 0xFFFFu) + (int32_t)(w[j] >> 16);
    return s - 262140;
}

static inline uint16_t f32_to_bf16_rne(float f) {
    uint32_t u;
    memcpy(&u, &f, 4);
    u += 0x7FFFu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}

static inline float normal_f32(uint32_t seed, uint32_t tid, uint64_t i, float scale, float mean) {
    uint32_t w[4];
    philox_at(seed, tid, i, w);
    /* built with -ffp-contract=off: the multiply and the add round separately */
    float t = (float)irwin_hall_centered(w) * scale;
    return t + mean;
}

/* out[j] = bf16 normal value of element offset + j, j in [0, n). */
void nfs_fill_normal_bf16(uint32_t seed, uint32_t tid, uint64_t offset, uint64_t n,
                          float scale, float mean, uint16_t* out) {
#pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < (int64_t)n; ++j)
        out[j] = f32_to_bf16_rne(normal_f32(seed, tid, offset + (uint64_t)j, scale, mean));
}

/* Same values for an arbitrary list of element indices. */
void nfs_gather_normal_bf16(uint32_t seed, uint32_t tid, const uint64_t* idx, uint64_t n,
                            float scale, float mean, uint16_t* out) {
#pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < (int64_t)n; ++j)
        out[j] = f32_to_bf16_rne(normal_f32(seed, tid, idx[j], scale, mean));
}

/* Element ranges: for r in [0, nranges), fill out with elements [starts[r], starts[r]+len). */
void nfs_fill_normal_bf16_ranges(uint32_t seed, uint32_t tid, const uint64_t* starts, uint64_t nranges,
                                 uint64_t len, float scale, float mean, uint16_t* out) {
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < (int64_t)nranges; ++r)
        for (uint64_t j = 0; j < len; ++j)
            out[(uint64_t)r * len + j] =
                f32_to_bf16_rne(normal_f32(seed, tid, starts[r] + j, scale, mean));
}

/* fp32 normal values (no bf16 rounding), used for batch-shape draws. */
void nfs_fill_normal_f32(uint32_t seed, uint32_t tid, uint64_t offset, uint64_t n,
                         float scale, float mean, float* out) {
    for (uint64_t j = 0; j < n; ++j) out[j] = normal_f32(seed, tid, offset + j, scale, mean);
}

/* Uniform integers in [lo, hi] (inclusive), one Philox block per element (word 0). */
void nfs_fill_uniform_int(uint32_t seed, uint32_t tid, uint64_t offset, uint64_t n,
                          int64_t lo, int64_t hi, int64_t* out) {
    uint64_t span = (uint64_t)(hi - lo + 1);
    for (uint64_t j = 0; j < n; ++j) {
        uint32_t w[4];
        philox_at(seed, tid, offset + j, w);
        out[j] = lo + (int64_t)(((uint64_t)w[0] * span) >> 32);
    }
}

/* Raw Philox words for element indices [offset, offset+n): out[4*j .. 4*j+3]. */
void nfs_fill_raw(uint32_t seed, uint32_t tid, uint64_t offset, uint64_t n, uint32_t* out) {
    for (uint64_t j = 0; j < n; ++j) philox_at(seed, tid, offset + j, out + 4 * j);
}
