// Steps 1-2 of the MoE layer: RMSNorm and the sigmoid/bias top-k router.
//
// RMSNorm — "推理计算流梳理" (huanyp.cn), §Norm&Residual, RMSNorm equation:
//   v_j = gamma_j * x_j / sqrt((1/d) sum_k x_k^2 + eps)
// Router — same page, §专家并行 / MoE Router 过程:
//   z = v W_r^T, s = sigmoid(z), I = Top8(s + b), w_i = s_i / sum_{j in I} s_j
//
// Kernels
//   rmsnorm_kernel       one warp per row, 16-byte loads, fp32 sum of squares by
//                        warp shuffle; writes v (f32/bf16) and 1/rms per row.
//   rmsnorm_row_kernel   the same with a 256-thread CTA per row, for batches of
//                        fewer rows than two waves of warps would cover.
//   router_logits_kernel fp32 CUDA-core GEMM z = a W_r^T over 64x64 tiles with a
//                        K split: W_r is staged in shared memory once per tile of
//                        64 tokens instead of re-read per token; the next K block
//                        is fetched into registers while the current one is used.  The A operand is
//                        either v, or x*rstd*gamma formed on the fly (the router
//                        then sees the unrounded fp32 normalised row).
//   router_topk_kernel   one warp per token: sums the K-split partials in split
//                        order, scores sigmoid(z)+b in fp32 (sigmoid in double,
//                        rounded once), then k rounds of a warp-wide argmax (two
//                        warp reductions: the largest score key, then the lowest
//                        expert index holding it) plus one more for the margin.
//   router_topk_token_kernel  the same for few tokens: a CTA per token, a thread
//                        per expert for the split sum, then one warp selects.
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace moe {

// ----------------------------------------------------------------------------- RMSNorm
template <int XDT, int VDT>
__global__ void __launch_bounds__(256) rmsnorm_kernel(const void* __restrict__ x, const float* __restrict__ gamma,
                                                      int T, int d, float eps, void* __restrict__ v,
                                                      float* __restrict__ rstd_out) {
    pdl_wait();
    pdl_trigger();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t t = (int64_t)blockIdx.x * 8 + warp;
    if (t >= T) return;
    const int64_t row = t * d;
    float ss = 0.f;
    for (int j = lane * 8; j < d; j += 256) {
        float a[8];
        load8<XDT>(x, row + j, a);
#pragma unroll
        for (int i = 0; i < 8; ++i) ss = fmaf(a[i], a[i], ss);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    const float r = 1.0f / sqrtf(ss / (float)d + eps);
    if (lane == 0 && rstd_out) rstd_out[t] = r;
    if (v == nullptr) return;
    for (int j = lane * 8; j < d; j += 256) {
        float a[8], g[8], o[8];
        load8<XDT>(x, row + j, a);
        load8<DT_F32>(gamma, j, g);
#pragma unroll
        for (int i = 0; i < 8; ++i) o[i] = (a[i] * r) * g[i];
        store8<VDT>(v, row + j, o);
    }
}

// The same with the whole row held in registers (d <= 256 NC): every load of the row is issued before
// the first is used, so a warp has NC 16-byte loads per lane in flight and x is read once.  Same
// arithmetic and summation order as rmsnorm_kernel, so the same results bit for bit.
template <int XDT, int VDT, int NC>
__global__ void __launch_bounds__(256) rmsnorm_reg_kernel(const void* __restrict__ x, const float* __restrict__ gamma,
                                                          int T, int d, float eps, void* __restrict__ v,
                                                          float* __restrict__ rstd_out) {
    pdl_wait();
    pdl_trigger();
    constexpr int V = XDT == DT_BF16 ? 1 : 2;  // 16-byte vectors per 8 elements
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t t = (int64_t)blockIdx.x * 8 + warp;
    if (t >= T) return;
    const int64_t row = t * d;
    uint4 raw[NC][V];
#pragma unroll
    for (int c = 0; c < NC; ++c) {
        const int j = lane * 8 + c * 256;
        if (j < d) {
#pragma unroll
            for (int q = 0; q < V; ++q)
                raw[c][q] = XDT == DT_BF16 ? ld16(static_cast<const uint16_t*>(x) + row + j)
                                           : ld16(static_cast<const float*>(x) + row + j + 4 * q);
        }
    }
    auto unpack = [&](int c, float (&a)[8]) {
        if constexpr (XDT == DT_BF16) {
            const uint32_t wv[4] = {raw[c][0].x, raw[c][0].y, raw[c][0].z, raw[c][0].w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                a[2 * i] = bf16_bits_to_f32(wv[i] & 0xFFFFu);
                a[2 * i + 1] = bf16_bits_to_f32(wv[i] >> 16);
            }
        } else {
            a[0] = __uint_as_float(raw[c][0].x); a[1] = __uint_as_float(raw[c][0].y);
            a[2] = __uint_as_float(raw[c][0].z); a[3] = __uint_as_float(raw[c][0].w);
            a[4] = __uint_as_float(raw[c][V - 1].x); a[5] = __uint_as_float(raw[c][V - 1].y);
            a[6] = __uint_as_float(raw[c][V - 1].z); a[7] = __uint_as_float(raw[c][V - 1].w);
        }
    };
    float ss = 0.f;
#pragma unroll
    for (int c = 0; c < NC; ++c) {
        if (lane * 8 + c * 256 < d) {
            float a[8];
            unpack(c, a);
#pragma unroll
            for (int i = 0; i < 8; ++i) ss = fmaf(a[i], a[i], ss);
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    const float r = 1.0f / sqrtf(ss / (float)d + eps);
    if (lane == 0 && rstd_out) rstd_out[t] = r;
    if (v == nullptr) return;
#pragma unroll
    for (int c = 0; c < NC; ++c) {
        const int j = lane * 8 + c * 256;
        if (j < d) {
            float a[8], g[8], o[8];
            unpack(c, a);
            load8<DT_F32>(gamma, j, g);
#pragma unroll
            for (int i = 0; i < 8; ++i) o[i] = (a[i] * r) * g[i];
            store8<VDT>(v, row + j, o);
        }
    }
}

// One CTA of 256 threads per row: for batches too small to fill the GPU with a warp per row.
template <int XDT, int VDT>
__global__ void __launch_bounds__(256) rmsnorm_row_kernel(const void* __restrict__ x, const float* __restrict__ gamma,
                                                          int T, int d, float eps, void* __restrict__ v,
                                                          float* __restrict__ rstd_out) {
    __shared__ float part[8];
    pdl_wait();
    pdl_trigger();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t row = (int64_t)blockIdx.x * d;
    float ss = 0.f;
    for (int j = threadIdx.x * 8; j < d; j += 2048) {
        float a[8];
        load8<XDT>(x, row + j, a);
#pragma unroll
        for (int i = 0; i < 8; ++i) ss = fmaf(a[i], a[i], ss);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    if (lane == 0) part[warp] = ss;
    __syncthreads();
    ss = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) ss += part[w];
    const float r = 1.0f / sqrtf(ss / (float)d + eps);
    if (threadIdx.x == 0 && rstd_out) rstd_out[blockIdx.x] = r;
    if (v == nullptr) return;
    for (int j = threadIdx.x * 8; j < d; j += 2048) {
        float a[8], g[8], o[8];
        load8<XDT>(x, row + j, a);
        load8<DT_F32>(gamma, j, g);
#pragma unroll
        for (int i = 0; i < 8; ++i) o[i] = (a[i] * r) * g[i];
        store8<VDT>(v, row + j, o);
    }
}

template <int XDT, int VDT>
static cudaError_t launch_rms(const Ctx& c, const void* x, const float* gamma, int T, int d, float eps, void* v,
                              float* rstd) {
    if (T <= 2 * 8 * c.num_sms)  // fewer rows than two waves of warp-per-row CTAs
        return launch(rmsnorm_row_kernel<XDT, VDT>, dim3(T), dim3(256), 0, c, x, gamma, T, d, eps, v, rstd);
    const dim3 g((T + 7) / 8);
    if (d <= 1024) return launch(rmsnorm_reg_kernel<XDT, VDT, 4>, g, dim3(256), 0, c, x, gamma, T, d, eps, v, rstd);
    if (d <= 2048) return launch(rmsnorm_reg_kernel<XDT, VDT, 8>, g, dim3(256), 0, c, x, gamma, T, d, eps, v, rstd);
    if (d <= 4096) return launch(rmsnorm_reg_kernel<XDT, VDT, 16>, g, dim3(256), 0, c, x, gamma, T, d, eps, v, rstd);
    return launch(rmsnorm_kernel<XDT, VDT>, g, dim3(256), 0, c, x, gamma, T, d, eps, v, rstd);
}

cudaError_t launch_rmsnorm(const Ctx& c, const void* x, int x_dt, const float* gamma, int T, int d, float eps, void* v,
                           int v_dt, float* rstd) {
    if (T == 0) return cudaSuccess;
    if (x_dt == DT_BF16 && v_dt == DT_BF16) return launch_rms<DT_BF16, DT_BF16>(c, x, gamma, T, d, eps, v, rstd);
    if (x_dt == DT_BF16 && v_dt == DT_F32) return launch_rms<DT_BF16, DT_F32>(c, x, gamma, T, d, eps, v, rstd);
    if (x_dt == DT_F32 && v_dt == DT_BF16) return launch_rms<DT_F32, DT_BF16>(c, x, gamma, T, d, eps, v, rstd);
    return launch_rms<DT_F32, DT_F32>(c, x, gamma, T, d, eps, v, rstd);
}

// ----------------------------------------------------------------------------- top-k
// Scores, top-k selection and weights of token t from its logits z[j] = z(lane + 32 j), by one
// warp: sigmoid in double rounded once to fp32, + b in fp32, k rounds of a warp-wide argmax (a max
// reduction of the order-preserving score keys, then a min reduction of the expert indices holding
// the maximum: ties go to the lower index) and one more for the margin to the first expert left out.
// Order-preserving 32-bit image of a non-NaN float (a larger float gives a larger unsigned; -0 is +0).
__device__ __forceinline__ uint32_t ordered_bits(float f) {
    const uint32_t u = __float_as_uint(f + 0.0f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float from_ordered(uint32_t o) {
    return __uint_as_float((o & 0x80000000u) ? (o & 0x7FFFFFFFu) : ~o);
}
__device__ __forceinline__ void select_topk_warp(const float (&z)[8], int lane, int t, const float* __restrict__ b,
                                                 int E, int k, int32_t* __restrict__ idx, float* __restrict__ w,
                                                 float* __restrict__ logits, float* __restrict__ margin) {
    // key of entry e = lane + 32 j: the order-preserving image of its score (NaN as -inf), 0 = no candidate
    uint32_t key[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const int e = lane + 32 * j;
        key[j] = 0;
        if (e < E) {
            const float acc = z[j];
            if (logits) logits[(int64_t)t * E + e] = acc;
            const float sg = (float)(1.0 / (1.0 + exp(-(double)acc)));
            const float sc = sg + b[e];
            key[j] = ordered_bits(isnan(sc) ? -INFINITY : sc);
        }
    }
    // this lane's best remaining entry (largest key, the lowest expert index among equal keys) and its logit
    uint32_t best = 0;
    int best_e = 0;
    float best_z = 0.f;
    auto refresh = [&]() {
        best = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j)
            if (key[j] > best) {
                best = key[j];
                best_e = lane + 32 * j;
                best_z = z[j];
            }
    };
    refresh();
    int sel_e[kMaxTopK];
    float sel_z[kMaxTopK];
    float kth = 0.f, next = INFINITY;
    const int rounds = k + (E > k ? 1 : 0);
    // each round: the warp's largest key (one reduction), then the lowest expert index holding it (a second)
#pragma unroll
    for (int r = 0; r < kMaxTopK + 1; ++r) {
        if (r >= rounds) break;
        const uint32_t m = __reduce_max_sync(0xffffffffu, best);
        const int be = (int)__reduce_min_sync(0xffffffffu, best == m ? (uint32_t)best_e : 0xFFFFFFFFu);
        const float bk = from_ordered(m);
        if (r < k) {
            sel_z[r] = __shfl_sync(0xffffffffu, best_z, be & 31);
            sel_e[r] = be;
            kth = bk;
            if ((be & 31) == lane) {  // the winner's lane drops it and finds its next best
#pragma unroll
                for (int j = 0; j < 8; ++j)
                    if (j == (be >> 5)) key[j] = 0;
                refresh();
            }
        } else {
            next = bk;
        }
    }
    // w_i = s_i / sum_j s_j with s in double: lane i < k takes pick i; the sum runs in pick order
    float my_z = 0.f;
    int my_e = 0;
#pragma unroll
    for (int i = 0; i < kMaxTopK; ++i)
        if (i == lane) {
            my_z = sel_z[i];
            my_e = sel_e[i];
        }
    const double sd = lane < k ? 1.0 / (1.0 + exp(-(double)my_z)) : 0.0;
    double sum = 0.0;
#pragma unroll
    for (int i = 0; i < kMaxTopK; ++i)
        if (i < k) sum += __shfl_sync(0xffffffffu, sd, i);
    if (lane < k) {
        idx[(int64_t)t * k + lane] = my_e;
        w[(int64_t)t * k + lane] = (float)(sd / sum);
    }
    if (margin && lane == 0) margin[t] = (E > k) ? (kth - next) : INFINITY;
}

__global__ void __launch_bounds__(256) router_topk_kernel(const float* __restrict__ partial, int splitk,
                                                          const float* __restrict__ b, int T, int E, int k,
                                                          int32_t* __restrict__ idx, float* __restrict__ w,
                                                          float* __restrict__ logits, float* __restrict__ margin) {
    pdl_wait();
    pdl_trigger();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t = blockIdx.x * 8 + warp;
    if (t >= T) return;
    float z[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) z[j] = 0.f;
    // sum the K-split partials in split order; the loads of one split are independent of each other
#pragma unroll 4
    for (int s = 0; s < splitk; ++s) {
        const float* ps = partial + ((int64_t)s * T + t) * E;
        float pv[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) pv[j] = (lane + 32 * j < E) ? __ldg(ps + lane + 32 * j) : 0.f;
#pragma unroll
        for (int j = 0; j < 8; ++j) z[j] += pv[j];
    }
    select_topk_warp(z, lane, t, b, E, k, idx, w, logits, margin);
}

// Few tokens (decode): one CTA per token, one thread per expert, so the split partials of all
// experts load in parallel (each thread's own sum still runs in split order: the same logits as
// the warp-per-token kernel bit for bit); then warp 0 selects.
__global__ void __launch_bounds__(256) router_topk_token_kernel(const float* __restrict__ partial, int splitk,
                                                                const float* __restrict__ b, int T, int E, int k,
                                                                int32_t* __restrict__ idx, float* __restrict__ w,
                                                                float* __restrict__ logits,
                                                                float* __restrict__ margin) {
    __shared__ float zs[kMaxExperts];
    pdl_wait();
    pdl_trigger();
    const int t = blockIdx.x, e = threadIdx.x;
    if (e < E) {
        const float* pe = partial + (int64_t)t * E + e;
        const int64_t stride = (int64_t)T * E;
        float acc = 0.f;
#pragma unroll 8
        for (int s = 0; s < splitk; ++s) acc += __ldg(pe + s * stride);
        zs[e] = acc;
    }
    __syncthreads();
    if (threadIdx.x >= 32) return;
    const int lane = threadIdx.x;
    float z[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) z[j] = (lane + 32 * j < E) ? zs[lane + 32 * j] : 0.f;
    select_topk_warp(z, lane, t, b, E, k, idx, w, logits, margin);
}

cudaError_t launch_router_topk(const Ctx& c, const RouterPlan& p, const float* partial, const float* b, int T, int E,
                               int k, int32_t* idx, float* w, float* logits, float* margin) {
    if (T == 0) return cudaSuccess;
    if (T <= c.num_sms && p.splitk > 2) {  // a warp per token would occupy only T / 8 SMs
        const int threads = (E + 31) / 32 * 32;
        return launch(router_topk_token_kernel, dim3(T), dim3(threads < 32 ? 32 : threads), 0, c, partial, p.splitk,
                      b, T, E, k, idx, w, logits, margin);
    }
    return launch(router_topk_kernel, dim3((T + 7) / 8), dim3(256), 0, c, partial, p.splitk, b, T, E, k, idx, w,
                  logits, margin);
}

}  // namespace moe
