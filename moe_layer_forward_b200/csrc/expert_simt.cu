// Step 4 for fp32 expert weights: grouped gated MLP on CUDA cores.
//
// "推理计算流梳理" (huanyp.cn), §实际 MLP 计算策略: Y = (SiLU(X W_gate) ⊙ X W_up) W_down,
// run per expert over its contiguous rows (§EP 路径: one grouped GEMM for all
// active experts).  fp32 operands have no full-precision tensor-core form on
// sm_100 (tf32 would drop mantissa bits), so this path is plain fp32 FMA.
//
// C[r][n] = sum_k A[r][k] * W[e][n][k] for r in expert e's rows, over 32x32
// output tiles; the grid's x index enumerates row blocks of all experts (an
// upper bound, blocks past the real total exit), y the column blocks.  With
// SWIGLU two weight tiles give C = SiLU(A W1^T) * (A W2^T).
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace moe {

constexpr int SR = 32, SC = 32, SK = 32;

template <bool SWIGLU>
__global__ void __launch_bounds__(256) simt_grouped_kernel(const float* __restrict__ A, const float* __restrict__ W1,
                                                           const float* __restrict__ W2,
                                                           const int32_t* __restrict__ counts,
                                                           const int32_t* __restrict__ offsets, int E, int K, int N,
                                                           float* __restrict__ C, int S, int32_t* status) {
    __shared__ int rb_start[kMaxExperts + 1];
    __shared__ int cnt_s[kMaxExperts], off_s[kMaxExperts];
    __shared__ float As[SK][SR + 1];
    __shared__ float B1[SK][SC + 1];
    __shared__ float B2[SWIGLU ? SK : 1][SC + 1];
    pdl_wait();
    pdl_trigger();
    if (threadIdx.x == 0) {
        // segments that do not fit the S-row buffers are clamped into them and flagged (by block 0)
        int run = 0;
        for (int e = 0; e < E; ++e) {
            int o, n;
            if (!clamp_segment(offsets[e], counts[e], S, o, n) && blockIdx.x == 0 && blockIdx.y == 0)
                set_status(status, DEV_BAD_COUNT);
            cnt_s[e] = n;
            off_s[e] = o;
            rb_start[e] = run;
            run += (n + SR - 1) / SR;
        }
        rb_start[E] = run;
    }
    __syncthreads();
    const int rbg = blockIdx.x;
    if (rbg >= rb_start[E]) return;
    int lo = 0, hi = E - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (rb_start[mid] <= rbg) lo = mid; else hi = mid - 1;
    }
    const int e = lo;
    const int rb = rbg - rb_start[e];
    const int64_t row0 = (int64_t)off_s[e] + (int64_t)rb * SR;
    const int rows = min(SR, cnt_s[e] - rb * SR);
    const int col0 = blockIdx.y * SC;
    const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
    float g[2][2] = {{0.f, 0.f}, {0.f, 0.f}}, u[2][2] = {{0.f, 0.f}, {0.f, 0.f}};
    const float* W1e = W1 + (int64_t)e * N * K;
    const float* W2e = SWIGLU ? W2 + (int64_t)e * N * K : nullptr;
    for (int k0 = 0; k0 < K; k0 += SK) {
        __syncthreads();
        for (int n = threadIdx.x; n < SK * SR; n += 256) {
            const int r = n / SK, kk = n % SK;
            const int kg = k0 + kk;
            As[kk][r] = (r < rows && kg < K) ? A[(row0 + r) * K + kg] : 0.f;
            const int cg = col0 + r;
            B1[kk][r] = (cg < N && kg < K) ? W1e[(int64_t)cg * K + kg] : 0.f;
            if (SWIGLU) B2[kk][r] = (cg < N && kg < K) ? W2e[(int64_t)cg * K + kg] : 0.f;
        }
        __syncthreads();
#pragma unroll 8
        for (int kk = 0; kk < SK; ++kk) {
            const float a0 = As[kk][ty * 2], a1 = As[kk][ty * 2 + 1];
            const float b0 = B1[kk][tx * 2], b1 = B1[kk][tx * 2 + 1];
            g[0][0] = fmaf(a0, b0, g[0][0]);
            g[0][1] = fmaf(a0, b1, g[0][1]);
            g[1][0] = fmaf(a1, b0, g[1][0]);
            g[1][1] = fmaf(a1, b1, g[1][1]);
            if (SWIGLU) {
                const float c0 = B2[kk][tx * 2], c1 = B2[kk][tx * 2 + 1];
                u[0][0] = fmaf(a0, c0, u[0][0]);
                u[0][1] = fmaf(a0, c1, u[0][1]);
                u[1][0] = fmaf(a1, c0, u[1][0]);
                u[1][1] = fmaf(a1, c1, u[1][1]);
            }
        }
    }
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const int r = ty * 2 + i;
        if (r >= rows) continue;
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            const int cg = col0 + tx * 2 + j;
            if (cg >= N) continue;
            float val = g[i][j];
            if (SWIGLU) val = val / (1.0f + expf(-val)) * u[i][j];
            C[(row0 + r) * N + cg] = val;
        }
    }
}

static dim3 simt_grid(int S, int E, int N) {
    // sum_e ceil(count_e / 32) <= S / 32 + E
    return dim3((unsigned)((S + SR - 1) / SR + E), (unsigned)((N + SC - 1) / SC));
}

cudaError_t launch_gate_up_f32(const Ctx& c, const float* xp, const float* Wg, const float* Wu, const int32_t* counts,
                               const int32_t* offsets, int S, int E, int d, int d_ff, float* h, int32_t* status) {
    if (S == 0) return cudaSuccess;
    return launch(simt_grouped_kernel<true>, simt_grid(S, E, d_ff), dim3(256), 0, c, xp, Wg, Wu, counts, offsets, E,
                  d, d_ff, h, S, status);
}

cudaError_t launch_down_f32(const Ctx& c, const float* h, const float* Wd, const int32_t* counts,
                            const int32_t* offsets, int S, int E, int d, int d_ff, float* y, int32_t* status) {
    if (S == 0) return cudaSuccess;
    return launch(simt_grouped_kernel<false>, simt_grid(S, E, d), dim3(256), 0, c, h, Wd, (const float*)nullptr,
                  counts, offsets, E, d_ff, d, y, S, status);
}

}  // namespace moe
