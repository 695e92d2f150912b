/*
 * CPU oracle for one MoE feed-forward layer: R = X + MoE(RMSNorm(X)).
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call, link or load
 * this file; only the tests, the smoke check and the benchmark's CPU-baseline
 * leg do.  It shares no code, header or table with the CUDA library.
 *
 * Plain, single-threaded, fp64 arithmetic on exactly converted inputs (f32 or
 * bf16 bits).  Every sum runs in index order.  The only place the result is
 * decided in fp32 is the top-8 choice of experts, because there a float
 * comparison decides an integer: the selection score is taken in the same
 * precision as the GPU kernel (fp32 logit -> fp32 sigmoid -> fp32 add of b).
 *
 * Sources (web pages on MoE inference):
 *   [P1] "推理计算流梳理" (huanyp.cn): §Norm&Residual (pre-norm block and the
 *        RMSNorm equation), §实际 MLP 计算策略 (gated MLP equation),
 *        §专家并行 / MoE Router 过程 (router equation), §EP 路径 (grouped GEMM,
 *        weighted sum at the source).
 *   [P5] "「赤兔」Chitu 框架深度解读（七）：混合专家模型 (MoE) 的高效处理":
 *        §Token 分发策略 (token_permutation / token_unpermutation),
 *        §专家计算实现 (tokens laid out contiguously by expert id).
 *
 * Readings where the pages are silent or garbled (each is also a pinned test):
 *   - the RMSNorm divisor printed as 4096 is the hidden size d; eps sits inside
 *     the square root; gamma multiplies directly;
 *   - SiLU(x) = x * sigmoid(x);
 *   - Top8 ties go to the lower expert index; I is listed by descending score,
 *     then ascending index;
 *   - slots inside one expert's segment are ordered by ascending token index;
 *     segments follow expert order with no padding between them.
 *
 * Parity status: every function below is pinned by tests under tests/
 * (closed forms, invariants, brute force); none is "parity unpinned".
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

enum { OR_F32 = 0, OR_BF16 = 1 };

static double load(const void* p, int dt, int64_t i) {
    if (dt == OR_F32) return (double)((const float*)p)[i];
    uint32_t bits = (uint32_t)((const uint16_t*)p)[i] << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

double oracle_load(const void* p, int dt, int64_t i) { return load(p, dt, i); }

/* logistic sigmoid 1 / (1 + e^-z) [P1 §MoE Router 过程] */
double oracle_sigmoid(double z) { return 1.0 / (1.0 + exp(-z)); }

/* SiLU(x) = x * sigmoid(x), the gate activation of [P1 §实际 MLP 计算策略] */
double oracle_silu(double x) { return x * oracle_sigmoid(x); }

/*
 * RMSNorm [P1 §Norm&Residual]:
 *   v_j = gamma_j * x_j / sqrt((1/d) * sum_k x_k^2 + eps)
 * x: [T][d] (dtype x_dt); v: [T][d] fp64.
 */
void oracle_rmsnorm(const void* x, int x_dt, const float* gamma, int64_t T, int64_t d, double eps, double* v) {
    for (int64_t t = 0; t < T; ++t) {
        double ss = 0.0;
        for (int64_t k = 0; k < d; ++k) {
            double a = load(x, x_dt, t * d + k);
            ss += a * a;
        }
        double denom = sqrt(ss / (double)d + eps);
        for (int64_t j = 0; j < d; ++j) v[t * d + j] = (double)gamma[j] * load(x, x_dt, t * d + j) / denom;
    }
}

/*
 * One row through a linear map stored out x in (row o of W holds the weights
 * of output o):  y_o = sum_i W[o][i] * x_i.  This is Y = X W of [P1 §张量并行和通信]
 * with W kept transposed in memory.
 */
void oracle_linear(const double* x, const void* W, int w_dt, int64_t n_out, int64_t n_in, double* y) {
    for (int64_t o = 0; o < n_out; ++o) {
        double acc = 0.0;
        for (int64_t i = 0; i < n_in; ++i) acc += load(W, w_dt, o * n_in + i) * x[i];
        y[o] = acc;
    }
}

/* router logits z = v W_r^T [P1 §MoE Router 过程]; v [T][d] fp64, W_r [E][d] f32, z [T][E] */
void oracle_router_logits(const double* v, const float* W_r, int64_t T, int64_t d, int64_t E, double* z) {
    for (int64_t t = 0; t < T; ++t) oracle_linear(v + t * d, W_r, OR_F32, E, d, z + t * E);
}

/* the fp32 selection score sigmoid(z) + b, with sigmoid evaluated in double and rounded once */
float oracle_selection_score(float z, float b) {
    float s = (float)oracle_sigmoid((double)z);
    volatile float r = s + b; /* fp32 addition */
    return r;
}

/* a NaN score sorts below every number */
static float sel_key(float s) { return isnan(s) ? -INFINITY : s; }

/*
 * Top-k selection and weights [P1 §MoE Router 过程]:
 *   I = TopK(sigmoid(z) + b),   w_i = s_i / sum_{j in I} s_j  (b takes no part in w).
 * z_sel [T][E] fp32 logits that decide I (score taken in fp32, see above);
 * z_w [T][E] fp64 logits for the weights, or NULL to use z_sel.
 * Outputs: idx [T][k] (descending score, ties to the lower index), w [T][k] fp64,
 * margin [T] = score of the k-th pick minus the best unpicked score (fp32), +inf if E == k.
 * Returns 0, or -1 on bad arguments.
 */
int oracle_select_topk(const float* z_sel, const double* z_w, const float* b, int64_t T, int64_t E, int k,
                       int32_t* idx, double* w, float* margin) {
    if (k < 1 || k > E || E > 4096 || k > 64) return -1;
    float score[4096];
    unsigned char taken[4096];
    for (int64_t t = 0; t < T; ++t) {
        for (int64_t e = 0; e < E; ++e) {
            score[e] = sel_key(oracle_selection_score(z_sel[t * E + e], b[e]));
            taken[e] = 0;
        }
        float kth = 0.0f;
        for (int i = 0; i < k; ++i) {
            int64_t best = -1;
            for (int64_t e = 0; e < E; ++e) {
                if (taken[e]) continue;
                if (best < 0 || score[e] > score[best]) best = e; /* strict '>' keeps the lower index on ties */
            }
            taken[best] = 1;
            idx[t * k + i] = (int32_t)best;
            kth = score[best];
        }
        if (margin) {
            float next = -INFINITY;
            int any = 0;
            for (int64_t e = 0; e < E; ++e)
                if (!taken[e] && (!any || score[e] > next)) { next = score[e]; any = 1; }
            volatile float m = any ? kth - next : INFINITY;
            margin[t] = m;
        }
        double sum = 0.0, s[64];
        for (int i = 0; i < k; ++i) {
            int64_t e = idx[t * k + i];
            double zz = z_w ? z_w[t * E + e] : (double)z_sel[t * E + e];
            s[i] = oracle_sigmoid(zz);
            sum += s[i];
        }
        for (int i = 0; i < k; ++i) w[t * k + i] = s[i] / sum;
    }
    return 0;
}

/*
 * Gated expert MLP of expert e [P1 §实际 MLP 计算策略]:
 *   y = (SiLU(v W_gate) ⊙ (v W_up)) W_down
 * W_gate, W_up: [E][d_ff][d]; W_down: [E][d][d_ff] (out x in).  v [d] fp64.
 * h [d_ff] (optional) receives the gated hidden row; y [d].
 */
void oracle_expert_mlp(const double* v, const void* W_gate, const void* W_up, const void* W_down, int w_dt,
                       int64_t e, int64_t d, int64_t d_ff, double* h, double* y) {
    double* g = (double*)malloc(sizeof(double) * d_ff);
    double* u = (double*)malloc(sizeof(double) * d_ff);
    double* hh = h ? h : (double*)malloc(sizeof(double) * d_ff);
    const int64_t wsz = (w_dt == OR_F32) ? 4 : 2;
    const char* wg = (const char*)W_gate + e * d_ff * d * wsz;
    const char* wu = (const char*)W_up + e * d_ff * d * wsz;
    const char* wd = (const char*)W_down + e * d * d_ff * wsz;
    oracle_linear(v, wg, w_dt, d_ff, d, g);
    oracle_linear(v, wu, w_dt, d_ff, d, u);
    for (int64_t f = 0; f < d_ff; ++f) hh[f] = oracle_silu(g[f]) * u[f];
    oracle_linear(hh, wd, w_dt, d, d_ff, y);
    if (!h) free(hh);
    free(g);
    free(u);
}

/*
 * Token permutation into expert-contiguous order [P5 §Token 分发策略, token_permutation;
 * §专家计算实现, tokens contiguous by expert id].
 * idx [T][k] expert ids in [0, E).  Outputs:
 *   counts [E]          rows routed to each expert,
 *   offsets [E+1]       start row of each expert's segment (no padding), offsets[E] = T*k,
 *   slot_token [T*k]    source token of each row,
 *   token_slot [T][k]   row that holds pick i of token t.
 * Inside a segment rows follow ascending token index.  Returns 0, or -1 if an id is out of range.
 */
int oracle_permute(const int32_t* idx, int64_t T, int64_t E, int k, int32_t* counts, int32_t* offsets,
                   int32_t* slot_token, int32_t* token_slot) {
    for (int64_t n = 0; n < T * k; ++n)
        if (idx[n] < 0 || idx[n] >= E) return -1;
    int64_t next = 0;
    for (int64_t e = 0; e < E; ++e) {
        offsets[e] = (int32_t)next;
        for (int64_t t = 0; t < T; ++t)
            for (int i = 0; i < k; ++i)
                if (idx[t * k + i] == e) {
                    slot_token[next] = (int32_t)t;
                    token_slot[t * k + i] = (int32_t)next;
                    ++next;
                }
        counts[e] = (int32_t)(next - offsets[e]);
    }
    offsets[E] = (int32_t)next;
    return 0;
}

/* gathered rows xp[s] = v[slot_token[s]] (the permuted activations), fp64 out */
void oracle_gather(const void* v, int v_dt, const int32_t* slot_token, int64_t S, int64_t d, double* xp) {
    for (int64_t s = 0; s < S; ++s)
        for (int64_t j = 0; j < d; ++j) xp[s * d + j] = load(v, v_dt, (int64_t)slot_token[s] * d + j);
}

/*
 * Grouped expert MLP over expert-contiguous rows [P1 §EP 路径, grouped GEMM]:
 * rows offsets[e] .. offsets[e]+counts[e]-1 of xp [S][d] go through expert e.
 * h [S][d_ff] (optional) and y [S][d] fp64; rows outside every segment are left untouched.
 */
void oracle_grouped_mlp(const void* xp, int x_dt, const int32_t* counts, const int32_t* offsets, int64_t E,
                        int64_t d, int64_t d_ff, const void* W_gate, const void* W_up, const void* W_down, int w_dt,
                        double* h, double* y) {
    double* row = (double*)malloc(sizeof(double) * d);
    for (int64_t e = 0; e < E; ++e) {
        for (int64_t r = offsets[e]; r < (int64_t)offsets[e] + counts[e]; ++r) {
            for (int64_t j = 0; j < d; ++j) row[j] = load(xp, x_dt, r * d + j);
            oracle_expert_mlp(row, W_gate, W_up, W_down, w_dt, e, d, d_ff, h ? h + r * d_ff : NULL, y + r * d);
        }
    }
    free(row);
}

/*
 * Weighted un-permute and residual [P1 §EP 路径, weighted sum at the source;
 * §Norm&Residual, X' = R + FFN(V); P5 token_unpermutation]:
 *   out[t] = res[t] + sum_i w[t][i] * y[token_slot[t][i]]
 */
void oracle_combine(const void* y, int y_dt, const int32_t* token_slot, const float* w, const void* res, int r_dt,
                    int64_t T, int64_t d, int k, double* out) {
    for (int64_t t = 0; t < T; ++t)
        for (int64_t j = 0; j < d; ++j) {
            double acc = 0.0;
            for (int i = 0; i < k; ++i)
                acc += (double)w[t * k + i] * load(y, y_dt, (int64_t)token_slot[t * k + i] * d + j);
            out[t * d + j] = load(res, r_dt, t * d + j) + acc;
        }
}

/*
 * The whole layer, token by token, straight from the definition (no permutation):
 *   v = RMSNorm(x_t); z = v W_r^T; I = Top_k(sigmoid(z) + b); w_i = s_i / sum_I s;
 *   out_t = x_t + sum_{i} w_i * MLP_{I_i}(v).
 * x: n rows [n][d].  If force_idx / force_w are given ([n][k]) they replace the
 * oracle's own routing (used to compare the expert path on the GPU's choice).
 * Optional outputs: idx [n][k], w [n][k] fp64, z32 [n][E] (the fp32 logits that
 * decided I), margin [n].  out [n][d] fp64.  Returns 0 or -1.
 */
int oracle_moe_layer(const void* x, int x_dt, int64_t n, const float* gamma, const float* W_r, const float* b,
                     const void* W_gate, const void* W_up, const void* W_down, int w_dt, int64_t d, int64_t E,
                     int k, int64_t d_ff, double eps, const int32_t* force_idx, const float* force_w, double* out,
                     int32_t* idx_out, double* w_out, float* z32_out, float* margin_out) {
    if (k < 1 || k > E || k > 64) return -1;
    double* v = (double*)malloc(sizeof(double) * d);
    double* z = (double*)malloc(sizeof(double) * E);
    float* z32 = (float*)malloc(sizeof(float) * E);
    double* y = (double*)malloc(sizeof(double) * d);
    int32_t sel[64];
    double wt[64];
    int rc = 0;
    for (int64_t t = 0; t < n && rc == 0; ++t) {
        /* x row t, as its own 1-row tensor */
        const char* xr = (const char*)x + t * d * (x_dt == OR_F32 ? 4 : 2);
        oracle_rmsnorm(xr, x_dt, gamma, 1, d, eps, v);
        oracle_router_logits(v, W_r, 1, d, E, z);
        for (int64_t e = 0; e < E; ++e) z32[e] = (float)z[e];
        float m = 0.0f;
        rc = oracle_select_topk(z32, z, b, 1, E, k, sel, wt, &m);
        if (z32_out) memcpy(z32_out + t * E, z32, sizeof(float) * E);
        if (margin_out) margin_out[t] = m;
        if (idx_out) memcpy(idx_out + t * k, sel, sizeof(int32_t) * k);
        if (w_out) memcpy(w_out + t * k, wt, sizeof(double) * k);
        if (force_idx) {
            for (int i = 0; i < k; ++i) {
                sel[i] = force_idx[t * k + i];
                wt[i] = (double)force_w[t * k + i];
                if (sel[i] < 0 || sel[i] >= E) rc = -1;
            }
            if (rc) break;
        }
        for (int64_t j = 0; j < d; ++j) out[t * d + j] = 0.0;
        for (int i = 0; i < k; ++i) {
            oracle_expert_mlp(v, W_gate, W_up, W_down, w_dt, sel[i], d, d_ff, NULL, y);
            for (int64_t j = 0; j < d; ++j) out[t * d + j] += wt[i] * y[j];
        }
        for (int64_t j = 0; j < d; ++j) out[t * d + j] += load(xr, x_dt, j);
    }
    free(v);
    free(z);
    free(z32);
    free(y);
    return rc;
}
