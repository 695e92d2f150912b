// Step 3 of the MoE layer: token permutation into expert-contiguous rows.
//
// "「赤兔」Chitu 框架深度解读（七）：混合专家模型 (MoE) 的高效处理", §Token 分发策略
// (token_permutation) and §专家计算实现 (the contiguous layout of the grouped GEMM:
// the rows of one expert are adjacent).  Without expert parallelism the
// dispatch is a local permutation (the page's MoEEmptyTokenDispatcher case).
//
// A deterministic counting sort, no atomics on global memory, no host sync:
//   perm_hist_kernel    per chunk of 256 tokens: shared-memory histogram over experts
//   perm_scan_kernel    one CTA: per expert, exclusive scan over chunks (in place);
//                       counts; exclusive scan over experts -> offsets
//   perm_scatter_kernel per chunk: a 256-bit token mask per expert in shared
//                       memory; the rank of token t inside expert e's segment is
//                       popcount(mask bits below t) + the chunk's base -> rows in
//                       ascending token order.  Writes token_slot, slot_token.
//   perm_single_kernel  the three above in one CTA when all tokens fit one chunk
//                       (T <= 256, decode batches): same counts, offsets and
//                       slots, one launch instead of three.
//   perm_gather_kernel  16-byte chunks: each token row of v is read once and
//                       written to its k rows of xp.
#include "common.cuh"
#include "kernels.h"

namespace moe {

constexpr int PC = kPermuteChunk;  // tokens per chunk == threads per CTA

__global__ void __launch_bounds__(PC) perm_hist_kernel(const int32_t* __restrict__ idx, int T, int E, int k,
                                                       int32_t* __restrict__ hist, int32_t* status) {
    __shared__ int h[kMaxExperts];
    pdl_wait();
    pdl_trigger();
    for (int e = threadIdx.x; e < E; e += PC) h[e] = 0;
    __syncthreads();
    const int t = blockIdx.x * PC + threadIdx.x;
    if (t < T) {
        for (int i = 0; i < k; ++i) {
            const int e = idx[(int64_t)t * k + i];
            if (e >= 0 && e < E)
                atomicAdd(&h[e], 1);
            else
                set_status(status, DEV_BAD_EXPERT_ID);
        }
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += PC) hist[(int64_t)blockIdx.x * E + e] = h[e];
}

// exclusive scan of one value per thread over a 256-thread block
__device__ __forceinline__ int block_exclusive_scan_256(int v, int* warp_tot) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += n;
    }
    if (lane == 31) warp_tot[warp] = incl;
    __syncthreads();
    int before = 0;
    for (int w = 0; w < warp; ++w) before += warp_tot[w];
    return before + incl - v;
}

__global__ void __launch_bounds__(256) perm_scan_kernel(int32_t* __restrict__ hist, int nchunks, int E,
                                                        int32_t* __restrict__ counts, int32_t* __restrict__ offsets) {
    __shared__ int warp_tot[8];
    pdl_wait();
    pdl_trigger();
    const int e = threadIdx.x;
    int run = 0;
    if (e < E) {
        // batches of 16 chunks: the loads of a batch are independent and in flight together
        for (int c0 = 0; c0 < nchunks; c0 += 16) {
            int v[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) v[i] = c0 + i < nchunks ? hist[(int64_t)(c0 + i) * E + e] : 0;
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                if (c0 + i < nchunks) hist[(int64_t)(c0 + i) * E + e] = run;
                run += v[i];
            }
        }
        counts[e] = run;
    }
    const int off = block_exclusive_scan_256(e < E ? run : 0, warp_tot);
    if (e < E) offsets[e] = off;
    if (e == 255) offsets[E] = off + (e < E ? run : 0);
}

__global__ void __launch_bounds__(PC) perm_scatter_kernel(const int32_t* __restrict__ idx, int T, int E, int k,
                                                          const int32_t* __restrict__ base,
                                                          const int32_t* __restrict__ offsets,
                                                          int32_t* __restrict__ slot_token,
                                                          int32_t* __restrict__ token_slot) {
    __shared__ uint32_t mask[kMaxExperts][PC / 32];
    __shared__ int off_s[kMaxExperts];
    pdl_wait();
    pdl_trigger();
    for (int n = threadIdx.x; n < E * (PC / 32); n += PC) (&mask[0][0])[n] = 0u;
    for (int e = threadIdx.x; e < E; e += PC) off_s[e] = offsets[e] + base[(int64_t)blockIdx.x * E + e];
    __syncthreads();
    const int tl = threadIdx.x;
    const int t = blockIdx.x * PC + tl;
    int ev[kMaxTopK];
#pragma unroll
    for (int i = 0; i < kMaxTopK; ++i) {
        ev[i] = -1;
        if (i < k && t < T) {
            const int e = idx[(int64_t)t * k + i];
            if (e >= 0 && e < E) {
                ev[i] = e;
                atomicOr(&mask[e][tl >> 5], 1u << (tl & 31));
            }
        }
    }
    __syncthreads();
    if (t >= T) return;
    const int wi = tl >> 5;
    const uint32_t below = (1u << (tl & 31)) - 1u;
#pragma unroll
    for (int i = 0; i < kMaxTopK; ++i) {
        if (i >= k) break;
        const int e = ev[i];
        int slot = -1;
        if (e >= 0) {
            int r = __popc(mask[e][wi] & below);
            for (int w = 0; w < wi; ++w) r += __popc(mask[e][w]);
            slot = off_s[e] + r;
            slot_token[slot] = t;
        }
        token_slot[(int64_t)t * k + i] = slot;
    }
}

// T <= PC: histogram, scan over experts and scatter in one CTA (thread = token, then thread = expert)
__global__ void __launch_bounds__(PC) perm_single_kernel(const int32_t* __restrict__ idx, int T, int E, int k,
                                                         int32_t* __restrict__ counts, int32_t* __restrict__ offsets,
                                                         int32_t* __restrict__ slot_token,
                                                         int32_t* __restrict__ token_slot, int32_t* status) {
    __shared__ uint32_t mask[kMaxExperts][PC / 32];
    __shared__ int h[kMaxExperts];
    __shared__ int off_s[kMaxExperts];
    __shared__ int warp_tot[PC / 32];
    pdl_wait();
    pdl_trigger();
    for (int n = threadIdx.x; n < E * (PC / 32); n += PC) (&mask[0][0])[n] = 0u;
    for (int e = threadIdx.x; e < E; e += PC) h[e] = 0;
    __syncthreads();
    const int t = threadIdx.x;
    int ev[kMaxTopK];
#pragma unroll
    for (int i = 0; i < kMaxTopK; ++i) {
        ev[i] = -1;
        if (i < k && t < T) {
            const int e = idx[(int64_t)t * k + i];
            if (e >= 0 && e < E) {
                ev[i] = e;
                atomicAdd(&h[e], 1);
                atomicOr(&mask[e][t >> 5], 1u << (t & 31));
            } else {
                set_status(status, DEV_BAD_EXPERT_ID);
            }
        }
    }
    __syncthreads();
    const int e = threadIdx.x;  // PC == 256 >= E threads
    const int cnt = e < E ? h[e] : 0;
    const int off = block_exclusive_scan_256(cnt, warp_tot);
    if (e < E) {
        counts[e] = cnt;
        offsets[e] = off;
        off_s[e] = off;
    }
    if (e == PC - 1) offsets[E] = off + cnt;
    __syncthreads();
    if (t >= T) return;
    const int wi = t >> 5;
    const uint32_t below = (1u << (t & 31)) - 1u;
#pragma unroll
    for (int i = 0; i < kMaxTopK; ++i) {
        if (i >= k) break;
        const int ee = ev[i];
        int slot = -1;
        if (ee >= 0) {
            int r = __popc(mask[ee][wi] & below);
            for (int w = 0; w < wi; ++w) r += __popc(mask[ee][w]);
            slot = off_s[ee] + r;
            slot_token[slot] = t;
        }
        token_slot[(int64_t)t * k + i] = slot;
    }
}

// each thread moves 16 bytes of one token row to the rows of its k picks
__global__ void __launch_bounds__(256) perm_gather_kernel(const uint8_t* __restrict__ v, int64_t row_bytes,
                                                          const int32_t* __restrict__ token_slot, int T, int k,
                                                          uint8_t* __restrict__ xp) {
    pdl_wait();
    pdl_trigger();
    const int64_t cpr = row_bytes / 16;
    const int64_t n = (int64_t)T * cpr;
    for (int64_t u = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; u < n; u += (int64_t)gridDim.x * blockDim.x) {
        const int64_t t = u / cpr, c = u - t * cpr;
        const uint4 val = ld16(v + t * row_bytes + c * 16);
#pragma unroll
        for (int i = 0; i < kMaxTopK; ++i) {
            if (i >= k) break;
            const int s = token_slot[t * k + i];
            if (s >= 0) st16(xp + (int64_t)s * row_bytes + c * 16, val);
        }
    }
}

cudaError_t launch_permute(const Ctx& c, const void* v, int v_dt, const int32_t* idx, int T, int d, int E, int k,
                           int32_t* counts, int32_t* offsets, int32_t* slot_token, int32_t* token_slot, void* xp,
                           int32_t* hist, int32_t* status) {
    const int nchunks = (T + PC - 1) / PC;
    cudaError_t err;
    if (nchunks <= 1) {  // one chunk: the whole sort in one CTA
        err = launch(perm_single_kernel, dim3(1), dim3(PC), 0, c, idx, T, E, k, counts, offsets, slot_token,
                     token_slot, status);
        if (err != cudaSuccess || T == 0 || xp == nullptr) return err;
        const int64_t row_bytes1 = (int64_t)d * (v_dt == DT_BF16 ? 2 : 4);
        const int64_t n1 = (int64_t)T * (row_bytes1 / 16);
        int64_t blocks1 = (n1 + 255) / 256;
        if (blocks1 > (int64_t)c.num_sms * 16) blocks1 = (int64_t)c.num_sms * 16;
        return launch(perm_gather_kernel, dim3((unsigned)blocks1), dim3(256), 0, c, static_cast<const uint8_t*>(v),
                      row_bytes1, token_slot, T, k, static_cast<uint8_t*>(xp));
    }
    if (T > 0) {
        err = launch(perm_hist_kernel, dim3(nchunks), dim3(PC), 0, c, idx, T, E, k, hist, status);
        if (err != cudaSuccess) return err;
    }
    // the scan also runs for T == 0 so that counts/offsets are always written
    err = launch(perm_scan_kernel, dim3(1), dim3(256), 0, c, hist, nchunks, E, counts, offsets);
    if (err != cudaSuccess || T == 0) return err;
    err = launch(perm_scatter_kernel, dim3(nchunks), dim3(PC), 0, c, idx, T, E, k, hist, offsets, slot_token,
                 token_slot);
    if (err != cudaSuccess || xp == nullptr) return err;
    const int64_t row_bytes = (int64_t)d * (v_dt == DT_BF16 ? 2 : 4);
    const int64_t n = (int64_t)T * (row_bytes / 16);
    int64_t blocks = (n + 255) / 256;
    const int64_t cap = (int64_t)c.num_sms * 16;
    if (blocks > cap) blocks = cap;
    return launch(perm_gather_kernel, dim3((unsigned)blocks), dim3(256), 0, c, static_cast<const uint8_t*>(v),
                  row_bytes, token_slot, T, k, static_cast<uint8_t*>(xp));
}

}  // namespace moe
