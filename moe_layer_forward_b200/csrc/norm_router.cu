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
//   router_logits_kernel fp32 CUDA-core GEMM z = a W_r^T over 64x64 tiles with a
//                        K split: W_r is staged in shared memory once per tile of
//                        64 tokens instead of re-read per token.  The A operand is
//                        either v, or x*rstd*gamma formed on the fly (the router
//                        then sees the unrounded fp32 normalised row).
//   router_topk_kernel   one warp per token: sums the K-split partials in split
//                        order, scores sigmoid(z)+b in fp32 (sigmoid in double,
//                        rounded once), then k rounds of a warp-shuffle argmax
//                        (ties to the lower index) plus one more for the margin.
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

cudaError_t launch_rmsnorm(const Ctx& c, const void* x, int x_dt, const float* gamma, int T, int d, float eps, void* v,
                           int v_dt, float* rstd) {
    if (T == 0) return cudaSuccess;
    dim3 grid((T + 7) / 8), block(256);
    if (x_dt == DT_BF16 && v_dt == DT_BF16) return launch(rmsnorm_kernel<DT_BF16, DT_BF16>, grid, block, 0, c, x, gamma, T, d, eps, v, rstd);
    if (x_dt == DT_BF16 && v_dt == DT_F32) return launch(rmsnorm_kernel<DT_BF16, DT_F32>, grid, block, 0, c, x, gamma, T, d, eps, v, rstd);
    if (x_dt == DT_F32 && v_dt == DT_BF16) return launch(rmsnorm_kernel<DT_F32, DT_BF16>, grid, block, 0, c, x, gamma, T, d, eps, v, rstd);
    return launch(rmsnorm_kernel<DT_F32, DT_F32>, grid, block, 0, c, x, gamma, T, d, eps, v, rstd);
}

// ----------------------------------------------------------------------------- router logits
constexpr int RT = 64, RE = 64, RK = 32;

// NORM: the A row is x * rstd[t] * gamma (x of type ADT); otherwise A = v of type ADT.
template <bool NORM, int ADT>
__global__ void __launch_bounds__(256) router_logits_kernel(const void* __restrict__ a, const float* __restrict__ rstd,
                                                            const float* __restrict__ gamma,
                                                            const float* __restrict__ W_r, int T, int d, int E,
                                                            int kchunk, float* __restrict__ partial) {
    __shared__ __align__(16) float As[RK][RT + 4];  // [k][token]
    __shared__ __align__(16) float Bs[RK][RE + 4];  // [k][expert]
    const int t0 = blockIdx.y * RT, e0 = blockIdx.x * RE, split = blockIdx.z;
    const int kbeg = split * kchunk, kend = min(d, kbeg + kchunk);
    pdl_wait();
    pdl_trigger();
    const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
    const int lrow = tid >> 2, lk = (tid & 3) * 8;
    const int ta = t0 + lrow, eb = e0 + lrow;
    float rs = 1.f;
    if (NORM && ta < T) rs = rstd[ta];
    float acc[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;

    for (int k0 = kbeg; k0 < kend; k0 += RK) {
        float av[8], bv[8];
        const int kk = k0 + lk;
        if (ta < T && kk < kend) {
            load8<ADT>(a, (int64_t)ta * d + kk, av);
            if (NORM) {
                float g[8];
                load8<DT_F32>(gamma, kk, g);
#pragma unroll
                for (int i = 0; i < 8; ++i) av[i] = (av[i] * rs) * g[i];
            }
        } else {
#pragma unroll
            for (int i = 0; i < 8; ++i) av[i] = 0.f;
        }
        if (eb < E && kk < kend) {
            load8<DT_F32>(W_r, (int64_t)eb * d + kk, bv);
        } else {
#pragma unroll
            for (int i = 0; i < 8; ++i) bv[i] = 0.f;
        }
        __syncthreads();
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            As[lk + i][lrow] = av[i];
            Bs[lk + i][lrow] = bv[i];
        }
        __syncthreads();
#pragma unroll
        for (int k = 0; k < RK; ++k) {
            const float4 a4 = *reinterpret_cast<const float4*>(&As[k][ty * 4]);
            const float4 b4 = *reinterpret_cast<const float4*>(&Bs[k][tx * 4]);
            const float ar[4] = {a4.x, a4.y, a4.z, a4.w}, br[4] = {b4.x, b4.y, b4.z, b4.w};
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(ar[i], br[j], acc[i][j]);
        }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int t = t0 + ty * 4 + i;
        if (t >= T) continue;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int e = e0 + tx * 4 + j;
            if (e < E) partial[((int64_t)split * T + t) * E + e] = acc[i][j];
        }
    }
}

RouterPlan plan_router(int T, int d, int E, int num_sms) {
    RouterPlan p;
    const int tiles = ((T + RT - 1) / RT) * ((E + RE - 1) / RE);
    const int kblocks = (d + RK - 1) / RK;
    int split = (2 * num_sms + tiles - 1) / (tiles > 0 ? tiles : 1);
    split = split < 1 ? 1 : split;
    // keep at least 8 K-blocks (256 columns) per split
    const int max_split = kblocks / 8 > 1 ? kblocks / 8 : 1;
    if (split > max_split) split = max_split;
    const int kb_per = (kblocks + split - 1) / split;
    p.kchunk = kb_per * RK;
    p.splitk = (d + p.kchunk - 1) / p.kchunk;
    p.partial_bytes = (size_t)p.splitk * (size_t)T * (size_t)E * sizeof(float);
    return p;
}

cudaError_t launch_router_logits(const Ctx& c, const RouterPlan& p, const void* a, int a_dt, const float* rstd,
                                 const float* gamma, const float* W_r, int T, int d, int E, float* partial) {
    if (T == 0) return cudaSuccess;
    dim3 grid((E + RE - 1) / RE, (T + RT - 1) / RT, p.splitk), block(256);
    const bool norm = rstd != nullptr;
    if (norm && a_dt == DT_BF16) return launch(router_logits_kernel<true, DT_BF16>, grid, block, 0, c, a, rstd, gamma, W_r, T, d, E, p.kchunk, partial);
    if (norm) return launch(router_logits_kernel<true, DT_F32>, grid, block, 0, c, a, rstd, gamma, W_r, T, d, E, p.kchunk, partial);
    if (a_dt == DT_BF16) return launch(router_logits_kernel<false, DT_BF16>, grid, block, 0, c, a, rstd, gamma, W_r, T, d, E, p.kchunk, partial);
    return launch(router_logits_kernel<false, DT_F32>, grid, block, 0, c, a, rstd, gamma, W_r, T, d, E, p.kchunk, partial);
}

// ----------------------------------------------------------------------------- top-k
__device__ __forceinline__ bool better(float ka, int ea, float kb, int eb) { return ka > kb || (ka == kb && ea < eb); }

__global__ void __launch_bounds__(256) router_topk_kernel(const float* __restrict__ partial, int splitk,
                                                          const float* __restrict__ b, int T, int E, int k,
                                                          int32_t* __restrict__ idx, float* __restrict__ w,
                                                          float* __restrict__ logits, float* __restrict__ margin) {
    pdl_wait();
    pdl_trigger();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t = blockIdx.x * 8 + warp;
    if (t >= T) return;
    float z[8], key[8];
    uint32_t taken = 0;  // bit j: entry lane + 32 j unavailable
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const int e = lane + 32 * j;
        z[j] = 0.f;
        key[j] = -INFINITY;
        if (e < E) {
            float acc = 0.f;
            for (int s = 0; s < splitk; ++s) acc += partial[((int64_t)s * T + t) * E + e];
            z[j] = acc;
            if (logits) logits[(int64_t)t * E + e] = acc;
            const float sg = (float)(1.0 / (1.0 + exp(-(double)acc)));
            const float sc = sg + b[e];
            key[j] = isnan(sc) ? -INFINITY : sc;
        } else {
            taken |= 1u << j;
        }
    }
    int sel_e[kMaxTopK];
    float sel_z[kMaxTopK];
    float kth = 0.f, next = INFINITY;
    const int rounds = k + (E > k ? 1 : 0);
#pragma unroll
    for (int r = 0; r < kMaxTopK + 1; ++r) {
        if (r >= rounds) break;
        float bk = -INFINITY;
        int be = 0x7fffffff;
        float bz = 0.f;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int e = lane + 32 * j;
            if (!(taken & (1u << j)) && better(key[j], e, bk, be)) {
                bk = key[j];
                be = e;
                bz = z[j];
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const float ok = __shfl_xor_sync(0xffffffffu, bk, o);
            const int oe = __shfl_xor_sync(0xffffffffu, be, o);
            const float oz = __shfl_xor_sync(0xffffffffu, bz, o);
            if (better(ok, oe, bk, be)) {
                bk = ok;
                be = oe;
                bz = oz;
            }
        }
        if (r < k) {
            if ((be & 31) == lane) taken |= 1u << (be >> 5);
            sel_e[r] = be;
            sel_z[r] = bz;
            kth = bk;
        } else {
            next = bk;
        }
    }
    double sd[kMaxTopK], sum = 0.0;
#pragma unroll
    for (int i = 0; i < kMaxTopK; ++i) {
        if (i < k) {
            sd[i] = 1.0 / (1.0 + exp(-(double)sel_z[i]));
            sum += sd[i];
        }
    }
#pragma unroll
    for (int i = 0; i < kMaxTopK; ++i) {
        if (i < k && lane == i) {
            idx[(int64_t)t * k + i] = sel_e[i];
            w[(int64_t)t * k + i] = (float)(sd[i] / sum);
        }
    }
    if (margin && lane == 0) margin[t] = (E > k) ? (kth - next) : INFINITY;
}

cudaError_t launch_router_topk(const Ctx& c, const RouterPlan& p, const float* partial, const float* b, int T, int E,
                               int k, int32_t* idx, float* w, float* logits, float* margin) {
    if (T == 0) return cudaSuccess;
    return launch(router_topk_kernel, dim3((T + 7) / 8), dim3(256), 0, c, partial, p.splitk, b, T, E, k, idx, w,
                  logits, margin);
}

}  // namespace moe
