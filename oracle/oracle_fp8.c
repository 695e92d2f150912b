/*
 * CPU oracle of the block-FP8 expert MLP (FP8 E4M3 codes with fp32 block
 * scales).
 *
 * TEST INFRASTRUCTURE ONLY, under the same rules as oracle.c: nothing on the
 * product path calls, links or loads it, and it shares no code with the CUDA
 * library.
 *
 * Source: [P5] "「赤兔」Chitu 框架深度解读（七）：混合专家模型 (MoE) 的高效处理",
 * §专家计算实现: the DeepGEMM expert backends run FP8 GEMMs (fp8_gemm_nt) on
 * expert-contiguous tokens, and the quantised MoE experts follow a
 * "blockfp8" scheme.  The page names the scheme without defining it; the
 * reading implemented here (the usual block-FP8 layout) is:
 *   - E4M3 codes: sign, 4 exponent bits (bias 7), 3 mantissa bits; no
 *     infinities; S.1111.111 is NaN; the largest finite magnitude is 448;
 *     exponent field 0 holds subnormals m * 2^-9.
 *   - encoding rounds to the nearest code, ties to the even mantissa, and
 *     saturates finite values beyond 448 to +-448.
 *   - a weight matrix [n][k] has one fp32 scale per 128 x 128 block; a GEMM
 *     input [rows][k] has one fp32 scale per (row, 128 consecutive columns).
 *     For a block with largest magnitude a: s = a / 448 (fp32 division), or
 *     s = 1 when a = 0; each element x gets the code of the fp32 quotient x / s.
 *     Codes are decided in fp32 on both sides, so they compare exactly.
 *   - a dequantised element is code_value * s; each GEMM is the exact dot
 *     product of dequantised operands (fp64 here, in index order).
 *   - gate/up: h = SiLU(g) * u from the dequantised products; h is quantised
 *     per (row, 128 features) from its fp32 rounding, which is the down
 *     projection's input.
 *
 * Parity status: every function is pinned by tests/test_oracle_fp8.py
 * (all 256 codes against an independent library decoder, round trips, tie and
 * saturation cases, quantisation bounds, brute force on tiny GEMMs).
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

double oracle_silu(double x);  /* oracle.c */
double oracle_load(const void* p, int dt, int64_t i);

/* value of an E4M3 code (NaN for S.1111.111) */
double oracle_e4m3_decode(uint8_t c) {
    const int sign = c >> 7, e = (c >> 3) & 15, m = c & 7;
    if (e == 15 && m == 7) return NAN;
    const double mag = e == 0 ? ldexp((double)m, -9) : ldexp(1.0 + m / 8.0, e - 7);
    return sign ? -mag : mag;
}

/* nearest E4M3 code of x (ties to even mantissa), finite overflow saturated to +-448 */
uint8_t oracle_e4m3_encode(float x) {
    if (isnan(x)) return 0x7F;
    const uint8_t sign = signbit(x) ? 0x80 : 0x00;
    const double a = fabs((double)x);
    uint32_t code;
    if (a < ldexp(1.0, -6)) {
        /* subnormal range: multiples of 2^-9; m == 8 is the smallest normal, code 8 */
        code = (uint32_t)nearbyint(ldexp(a, 9));
    } else {
        int e2;
        frexp(a, &e2);           /* a = f * 2^e2, f in [0.5, 1) */
        const int e = e2 - 1;    /* a in [2^e, 2^(e+1)) */
        const double m = nearbyint(ldexp(a, 3 - e));  /* 8 .. 16 */
        if (e + 7 > 15) return sign | 0x7E;
        code = (uint32_t)(((e + 7) << 3) + (int)m - 8);  /* m == 16 carries into the exponent */
    }
    if (code > 0x7E) code = 0x7E;  /* beyond 448, and the NaN pattern, saturate */
    return sign | (uint8_t)code;
}

/*
 * Quantise x [rows][cols] (dtype dt: 0 f32, 1 bf16) in blocks of blk_rows x 128:
 * q [rows][cols] codes, s [ceil(rows / blk_rows)][cols / 128] fp32 scales.
 */
void oracle_quantize_blocks(const void* x, int dt, int64_t rows, int64_t cols, int64_t blk_rows, uint8_t* q,
                            float* s) {
    const int64_t nbc = cols / 128, nbr = (rows + blk_rows - 1) / blk_rows;
    for (int64_t br = 0; br < nbr; ++br)
        for (int64_t bc = 0; bc < nbc; ++bc) {
            float amax = 0.f;
            for (int64_t r = br * blk_rows; r < rows && r < (br + 1) * blk_rows; ++r)
                for (int64_t c = bc * 128; c < (bc + 1) * 128; ++c) {
                    const float v = fabsf((float)oracle_load(x, dt, r * cols + c));
                    if (v > amax) amax = v;
                }
            const float sc = amax > 0.f ? amax / 448.0f : 1.0f;
            s[br * nbc + bc] = sc;
            for (int64_t r = br * blk_rows; r < rows && r < (br + 1) * blk_rows; ++r)
                for (int64_t c = bc * 128; c < (bc + 1) * 128; ++c)
                    q[r * cols + c] = oracle_e4m3_encode((float)oracle_load(x, dt, r * cols + c) / sc);
        }
}

/* the 256 code values, filled from oracle_e4m3_decode on first use (a speed-up only) */
static double code_value(uint8_t c) {
    static double tab[256];
    static int ready = 0;
    if (!ready) {
        for (int i = 0; i < 256; ++i) tab[i] = oracle_e4m3_decode((uint8_t)i);
        ready = 1;
    }
    return tab[c];
}

/* dequantised element (r, c) of a block-quantised matrix with cols columns */
static double deq(const uint8_t* q, const float* s, int64_t cols, int64_t blk_rows, int64_t r, int64_t c) {
    return code_value(q[r * cols + c]) * (double)s[(r / blk_rows) * (cols / 128) + c / 128];
}

/*
 * Block-FP8 grouped SwiGLU MLP over expert segments [offsets[e], offsets[e] + counts[e]):
 *   xq [S][d] codes + xs [S][d/128]            (GEMM input, per-row blocks)
 *   W*_q codes + W*_s scales [E][n/128][k/128]  (weights, 128 x 128 blocks)
 * Outputs for the segment rows: h [S][d_ff] (fp64), hq [S][d_ff] + hs [S][d_ff/128] (the quantised
 * down input), y [S][d] (fp64).  If hq_in/hs_in are given, y uses them instead of hq/hs.
 */
void oracle_fp8_grouped_mlp(const uint8_t* xq, const float* xs, const int32_t* counts, const int32_t* offsets,
                            int64_t E, int64_t d, int64_t d_ff, const uint8_t* wg_q, const float* wg_s,
                            const uint8_t* wu_q, const float* wu_s, const uint8_t* wd_q, const float* wd_s, double* h,
                            uint8_t* hq, float* hs, const uint8_t* hq_in, const float* hs_in, double* y) {
    const int64_t nfb = d_ff / 128;
    for (int64_t e = 0; e < E; ++e) {
        const uint8_t* gq = wg_q + e * d_ff * d;
        const uint8_t* uq = wu_q + e * d_ff * d;
        const uint8_t* dq = wd_q + e * d * d_ff;
        const float* gs = wg_s + e * nfb * (d / 128);
        const float* us = wu_s + e * nfb * (d / 128);
        const float* ds = wd_s + e * (d / 128) * nfb;
        for (int64_t r = offsets[e]; r < offsets[e] + counts[e]; ++r) {
            for (int64_t f = 0; f < d_ff; ++f) {
                double g = 0.0, u = 0.0;
                for (int64_t j = 0; j < d; ++j) {
                    const double a = deq(xq, xs, d, 1, r, j);
                    g += a * deq(gq, gs, d, 128, f, j);
                    u += a * deq(uq, us, d, 128, f, j);
                }
                h[r * d_ff + f] = oracle_silu(g) * u;
            }
            for (int64_t b = 0; b < nfb; ++b) {
                float amax = 0.f;
                for (int64_t f = b * 128; f < (b + 1) * 128; ++f) {
                    const float v = fabsf((float)h[r * d_ff + f]);
                    if (v > amax) amax = v;
                }
                const float sc = amax > 0.f ? amax / 448.0f : 1.0f;
                hs[r * nfb + b] = sc;
                for (int64_t f = b * 128; f < (b + 1) * 128; ++f)
                    hq[r * d_ff + f] = oracle_e4m3_encode((float)h[r * d_ff + f] / sc);
            }
            const uint8_t* hqr = hq_in ? hq_in : hq;
            const float* hsr = hs_in ? hs_in : hs;
            for (int64_t o = 0; o < d; ++o) {
                double acc = 0.0;
                for (int64_t f = 0; f < d_ff; ++f) acc += deq(hqr, hsr, d_ff, 1, r, f) * deq(dq, ds, d_ff, 128, o, f);
                y[r * d + o] = acc;
            }
        }
    }
}
