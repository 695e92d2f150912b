// Step 5 of the MoE layer: weighted un-permute back to token order, plus the residual.
//
// "推理计算流梳理" (huanyp.cn), §EP 路径 (the expert outputs are summed with their
// router weights at the token's source) and §Norm&Residual (X_{l+1} = R_l + FFN(V_l));
// the Chitu MoE page calls this token_unpermutation.
//
//   out[t][j] = residual[t][j] + sum_{i<k} w[t][i] * y[token_slot[t][i]][j]
//
// One thread owns 8 consecutive columns of one token: it gathers the k expert
// rows (16-byte loads), accumulates in fp32 in pick order, adds the residual
// and writes once.  Grid-stride over (token, column chunk); HBM-bound.
#include "common.cuh"
#include "kernels.h"

namespace moe {

template <int YDT, int RDT, int ODT>
__global__ void __launch_bounds__(256) combine_kernel(const void* __restrict__ y, const int32_t* __restrict__ token_slot,
                                                      const float* __restrict__ w, const void* __restrict__ res, int T,
                                                      int d, int k, void* __restrict__ out) {
    pdl_wait();
    pdl_trigger();
    const int cpr = d / 8;
    const int64_t n = (int64_t)T * cpr;
    for (int64_t u = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; u < n; u += (int64_t)gridDim.x * blockDim.x) {
        const int64_t t = u / cpr;
        const int64_t j = (u - t * cpr) * 8;
        int slot[kMaxTopK];
        float wt[kMaxTopK];
#pragma unroll
        for (int i = 0; i < kMaxTopK; ++i) {
            slot[i] = -1;
            wt[i] = 0.f;
            if (i < k) {
                slot[i] = __ldg(token_slot + t * k + i);
                wt[i] = __ldg(w + t * k + i);
            }
        }
        float acc[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) acc[q] = 0.f;
#pragma unroll
        for (int i = 0; i < kMaxTopK; ++i) {
            if (slot[i] < 0) continue;
            float yv[8];
            load8<YDT>(y, (int64_t)slot[i] * d + j, yv);
#pragma unroll
            for (int q = 0; q < 8; ++q) acc[q] = fmaf(wt[i], yv[q], acc[q]);
        }
        float r[8], o[8];
        load8<RDT>(res, t * d + j, r);
#pragma unroll
        for (int q = 0; q < 8; ++q) o[q] = r[q] + acc[q];
        store8<ODT>(out, t * d + j, o);
    }
}

template <int YDT, int RDT>
static cudaError_t launch_combine_o(const Ctx& c, dim3 g, const void* y, const int32_t* ts, const float* w,
                                   const void* res, int T, int d, int k, void* out, int out_dt) {
    if (out_dt == DT_BF16) return launch(combine_kernel<YDT, RDT, DT_BF16>, g, dim3(256), 0, c, y, ts, w, res, T, d, k, out);
    return launch(combine_kernel<YDT, RDT, DT_F32>, g, dim3(256), 0, c, y, ts, w, res, T, d, k, out);
}

cudaError_t launch_combine(const Ctx& c, const void* y, int y_dt, const int32_t* token_slot, const float* w,
                           const void* res, int r_dt, int T, int d, int k, void* out, int out_dt) {
    if (T == 0) return cudaSuccess;
    const int64_t n = (int64_t)T * (d / 8);
    int64_t blocks = (n + 255) / 256;
    const int64_t cap = (int64_t)c.num_sms * 16;
    if (blocks > cap) blocks = cap;
    dim3 g((unsigned)blocks);
    if (y_dt == DT_BF16 && r_dt == DT_BF16) return launch_combine_o<DT_BF16, DT_BF16>(c, g, y, token_slot, w, res, T, d, k, out, out_dt);
    if (y_dt == DT_BF16) return launch_combine_o<DT_BF16, DT_F32>(c, g, y, token_slot, w, res, T, d, k, out, out_dt);
    if (r_dt == DT_BF16) return launch_combine_o<DT_F32, DT_BF16>(c, g, y, token_slot, w, res, T, d, k, out, out_dt);
    return launch_combine_o<DT_F32, DT_F32>(c, g, y, token_slot, w, res, T, d, k, out, out_dt);
}

}  // namespace moe
