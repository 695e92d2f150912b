// Step 5 of the MoE layer: weighted un-permute back to token order, plus the residual.
//
// "推理计算流梳理" (huanyp.cn), §EP 路径 (the expert outputs are summed with their
// router weights at the token's source) and §Norm&Residual (X_{l+1} = R_l + FFN(V_l));
// the Chitu MoE page calls this token_unpermutation.
//
//   out[t][j] = residual[t][j] + sum_{i<k} w[t][i] * y[token_slot[t][i]][j]
//
// A pick whose slot is negative (the permutation marks a pick with a bad
// expert id that way) is skipped: neither its row is read nor its weight used.
//
// One warp owns a (token, 256-column segment) unit: lanes below k load the
// token's k slots and weights once and broadcast them by shuffle; each lane
// then gathers its 8 columns from the k expert rows (16-byte loads, all
// independent), accumulates in fp32 in pick order, adds the residual and
// writes once.  Warp-grid-stride over units; HBM-bound.
#include "common.cuh"
#include "kernels.h"

namespace moe {

template <int YDT, int RDT, int ODT>
__global__ void __launch_bounds__(256) combine_kernel(const void* __restrict__ y, const int32_t* __restrict__ token_slot,
                                                      const float* __restrict__ w, const void* __restrict__ res, int T,
                                                      int d, int k, void* __restrict__ out) {
    pdl_wait();
    pdl_trigger();
    const int lane = threadIdx.x & 31;
    const int nseg = (d + 255) / 256;
    const int64_t n = (int64_t)T * nseg;
    const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
    for (int64_t u = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); u < n; u += warps) {
        const int64_t t = u / nseg;
        const int64_t j = (u - t * nseg) * 256 + lane * 8;
        int my_slot = 0;
        float my_w = 0.f;
        if (lane < k) {
            my_slot = __ldg(token_slot + t * k + lane);
            my_w = __ldg(w + t * k + lane);
        }
        int slot[kMaxTopK];
        float wt[kMaxTopK];
#pragma unroll
        for (int i = 0; i < kMaxTopK; ++i) {
            slot[i] = __shfl_sync(0xffffffffu, my_slot, i);
            wt[i] = __shfl_sync(0xffffffffu, my_w, i);
        }
        if (j >= d) continue;
        // all k row loads first (raw 16-byte vectors), then convert and accumulate in pick order
        constexpr int V = YDT == DT_BF16 ? 1 : 2;  // 16-byte vectors per 8 columns
        uint4 raw[kMaxTopK][V];
#pragma unroll
        for (int i = 0; i < kMaxTopK; ++i) {
            if (i < k && slot[i] >= 0) {
                const int64_t e0 = (int64_t)slot[i] * d + j;
#pragma unroll
                for (int v = 0; v < V; ++v)
                    raw[i][v] = YDT == DT_BF16 ? ld16(static_cast<const uint16_t*>(y) + e0)
                                               : ld16(static_cast<const float*>(y) + e0 + 4 * v);
            }
        }
        float acc[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) acc[q] = 0.f;
#pragma unroll
        for (int i = 0; i < kMaxTopK; ++i) {
            if (i < k && slot[i] >= 0) {
                float yv[8];
                if constexpr (YDT == DT_BF16) {
                    const uint32_t wv[4] = {raw[i][0].x, raw[i][0].y, raw[i][0].z, raw[i][0].w};
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        yv[2 * q] = bf16_bits_to_f32(wv[q] & 0xFFFFu);
                        yv[2 * q + 1] = bf16_bits_to_f32(wv[q] >> 16);
                    }
                } else {
                    yv[0] = __uint_as_float(raw[i][0].x); yv[1] = __uint_as_float(raw[i][0].y);
                    yv[2] = __uint_as_float(raw[i][0].z); yv[3] = __uint_as_float(raw[i][0].w);
                    yv[4] = __uint_as_float(raw[i][V - 1].x); yv[5] = __uint_as_float(raw[i][V - 1].y);
                    yv[6] = __uint_as_float(raw[i][V - 1].z); yv[7] = __uint_as_float(raw[i][V - 1].w);
                }
#pragma unroll
                for (int q = 0; q < 8; ++q) acc[q] = fmaf(wt[i], yv[q], acc[q]);
            }
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
    const int64_t n = (int64_t)T * ((d + 255) / 256);  // warp units
    int64_t blocks = (n + 7) / 8;
    const int64_t cap = (int64_t)c.num_sms * 16;
    if (blocks > cap) blocks = cap;
    dim3 g((unsigned)blocks);
    if (y_dt == DT_BF16 && r_dt == DT_BF16) return launch_combine_o<DT_BF16, DT_BF16>(c, g, y, token_slot, w, res, T, d, k, out, out_dt);
    if (y_dt == DT_BF16) return launch_combine_o<DT_BF16, DT_F32>(c, g, y, token_slot, w, res, T, d, k, out, out_dt);
    if (r_dt == DT_BF16) return launch_combine_o<DT_F32, DT_BF16>(c, g, y, token_slot, w, res, T, d, k, out, out_dt);
    return launch_combine_o<DT_F32, DT_F32>(c, g, y, token_slot, w, res, T, d, k, out, out_dt);
}

}  // namespace moe
