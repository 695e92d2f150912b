/*
 * Seeded synthetic tensors for the MoE layer workloads.
 *
 * Every value is a pure function of (seed, tensor id, element index): a
 * splitmix64 counter hash (Steele, Lea, Flood, "Fast splittable pseudorandom
 * number generators", OOPSLA 2014) gives 53-bit uniforms, and the Box-Muller
 * transform (Box & Muller 1958) turns pairs of them into normals.  Results do
 * not depend on the number of threads.  This file holds no arithmetic of the
 * MoE layer itself; it only draws numbers.
 *
 * bf16 outputs are the float value rounded to nearest-even on the upper 16 bits.
 */
#include <math.h>
#include <stdint.h>

#define GOLDEN 0x9E3779B97F4A7C15ull

static inline uint64_t mix64(uint64_t z) {
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

static inline uint64_t stream_key(uint64_t seed, uint64_t tid) {
    return mix64(seed * GOLDEN + mix64(tid + 0x632BE59BD9B4E019ull));
}

static inline uint64_t draw(uint64_t key, uint64_t i) { return mix64(key + (i + 1) * GOLDEN); }

/* uniform on the open interval (0, 1) */
static inline double u01(uint64_t r) { return ((double)(r >> 11) + 0.5) * 0x1.0p-53; }

static inline uint16_t f32_to_bf16_rne(float f) {
    union { float f; uint32_t u; } v = {f};
    if ((v.u & 0x7F800000u) == 0x7F800000u && (v.u & 0x007FFFFFu)) return (uint16_t)((v.u >> 16) | 0x40);
    v.u += 0x7FFFu + ((v.u >> 16) & 1u);
    return (uint16_t)(v.u >> 16);
}

static inline void normal_pair(uint64_t key, uint64_t p, double* z0, double* z1) {
    double u1 = u01(draw(key, 2 * p)), u2 = u01(draw(key, 2 * p + 1));
    double r = sqrt(-2.0 * log(u1));
    double a = 6.283185307179586476925 * u2;
    *z0 = r * cos(a);
    *z1 = r * sin(a);
}

/* out[i] = (float)(mean + std * N_i), i in [0, n) */
void synth_normal_f32(float* out, uint64_t n, uint64_t seed, uint64_t tid, double mean, double std) {
    uint64_t key = stream_key(seed, tid);
    int64_t npairs = (int64_t)((n + 1) / 2);
#pragma omp parallel for schedule(static)
    for (int64_t p = 0; p < npairs; ++p) {
        double z0, z1;
        normal_pair(key, (uint64_t)p, &z0, &z1);
        uint64_t i = 2 * (uint64_t)p;
        out[i] = (float)(mean + std * z0);
        if (i + 1 < n) out[i + 1] = (float)(mean + std * z1);
    }
}

/* bf16 bits of (float)(mean + std * N_i) */
void synth_normal_bf16(uint16_t* out, uint64_t n, uint64_t seed, uint64_t tid, double mean, double std) {
    uint64_t key = stream_key(seed, tid);
    int64_t npairs = (int64_t)((n + 1) / 2);
#pragma omp parallel for schedule(static)
    for (int64_t p = 0; p < npairs; ++p) {
        double z0, z1;
        normal_pair(key, (uint64_t)p, &z0, &z1);
        uint64_t i = 2 * (uint64_t)p;
        out[i] = f32_to_bf16_rne((float)(mean + std * z0));
        if (i + 1 < n) out[i + 1] = f32_to_bf16_rne((float)(mean + std * z1));
    }
}

/* out[i] = (float)(lo + (hi - lo) * U_i) */
void synth_uniform_f32(float* out, uint64_t n, uint64_t seed, uint64_t tid, double lo, double hi) {
    uint64_t key = stream_key(seed, tid);
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < (int64_t)n; ++i) out[i] = (float)(lo + (hi - lo) * u01(draw(key, (uint64_t)i)));
}

/* uniform integers in [lo, hi] (inclusive), for index-valued test inputs */
void synth_uniform_i32(int32_t* out, uint64_t n, uint64_t seed, uint64_t tid, int32_t lo, int32_t hi) {
    uint64_t key = stream_key(seed, tid);
    uint64_t span = (uint64_t)((int64_t)hi - (int64_t)lo + 1);
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < (int64_t)n; ++i) out[i] = (int32_t)((int64_t)lo + (int64_t)(draw(key, (uint64_t)i) % span));
}

/* one raw 64-bit draw per element (for permutations / sampling done by the caller) */
void synth_raw_u64(uint64_t* out, uint64_t n, uint64_t seed, uint64_t tid) {
    uint64_t key = stream_key(seed, tid);
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < (int64_t)n; ++i) out[i] = draw(key, (uint64_t)i);
}
