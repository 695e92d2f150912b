// Expert parallelism over peer memory: the token dispatch and the combine
// fused with their exchanges.
//
// "「赤兔」Chitu 框架深度解读（七）", §Token 分发策略: with expert parallelism
// every (token, expert) row is sent to the rank that owns the expert, the
// experts run there, and the results come back to be summed at the token's
// source; "推理计算流梳理", §EP 路径: the same exchange around the grouped GEMM,
// weighted sum at the source.
//
// Rank j of N owns experts [j E_loc, (j+1) E_loc), E_loc = E / N.  Every rank
// knows the count table C[s][e] (rows rank s routes to expert e, all ranks'
// counts exchanged beforehand).  Rank j's receive buffer holds its experts'
// rows expert-major, and within an expert source-rank-major, each source's rows
// in its own slot order (token order):
//
//   row of (source r, expert e, i-th row of r's segment for e)
//     = sum_{e' in [j E_loc, e)} sum_s C[s][e']  +  sum_{s<r} C[s][e]  +  i
//
// which is exactly the expert-contiguous layout the grouped GEMM consumes
// (counts_loc[e] = sum_s C[s][e]), so the receiver needs no second permutation.
// With tokens split over ranks in order, this is also the single-GPU
// permutation's row order.
//
//   ep_dispatch_kernel  the permutation's row copy, each row stored straight
//                       into its owner's receive buffer (peer memory); replaces
//                       the local row copy plus an All-to-All.
//   ep_layout_kernel    this rank's counts_loc / offsets_loc from the table.
//   ep_combine_kernel   step 5 reading every pick's expert output row from its
//                       owner's buffer (peer loads); the same arithmetic as
//                       combine_kernel (fp32 pick-order sum, then the residual).
//
// The kernels use plain loads and stores on the peer pointers (NVLink P2P);
// ordering between the ranks' kernels is the caller's (a barrier after the
// dispatch and one after the expert MLP).
#include "common.cuh"
#include "kernels.h"

namespace moe {

// dbase[e] = row of (this rank, expert e, i = 0) in e's owner's receive buffer
__device__ void ep_dest_base(const int32_t* __restrict__ table, int rank, int N, int E, int* dbase, int* scratch) {
    const int E_loc = E / N;
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        int col = 0, pre = 0;
        for (int s = 0; s < N; ++s) {
            const int c = table[(int64_t)s * E + e];
            col += c;
            if (s < rank) pre += c;
        }
        scratch[e] = col;
        dbase[e] = pre;
    }
    __syncthreads();
    if (threadIdx.x < 32) {  // exclusive prefix of the column sums: lane owns experts 8 lane .. 8 lane + 7
        const int lane = threadIdx.x;
        int loc[8], sum = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int e = lane * 8 + i;
            loc[i] = e < E ? scratch[e] : 0;
            sum += loc[i];
        }
        int incl = sum;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int n = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += n;
        }
        int run = incl - sum;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int e = lane * 8 + i;
            if (e < E) scratch[e] = run;
            run += loc[i];
        }
    }
    __syncthreads();
    // rebase each prefix to the start of its owner's expert range
    for (int e = threadIdx.x; e < E; e += blockDim.x) dbase[e] += scratch[e] - scratch[(e / E_loc) * E_loc];
    __syncthreads();
}

__global__ void __launch_bounds__(256) ep_dispatch_kernel(const uint8_t* __restrict__ v, int64_t row_bytes,
                                                          const int32_t* __restrict__ idx,
                                                          const int32_t* __restrict__ token_slot,
                                                          const int32_t* __restrict__ offsets,
                                                          const int32_t* __restrict__ table, int rank, int N, int E,
                                                          int T, int k, uint8_t* const* __restrict__ recv,
                                                          int64_t recv_rows, int32_t* status) {
    __shared__ int dbase[kMaxExperts], scratch[kMaxExperts], own[kMaxExperts];
    pdl_wait();
    pdl_trigger();
    ep_dest_base(table, rank, N, E, dbase, scratch);
    for (int e = threadIdx.x; e < E; e += blockDim.x) own[e] = table[(int64_t)rank * E + e];
    __syncthreads();
    const int E_loc = E / N;
    const int64_t cpr = row_bytes / 16;
    const int64_t n = (int64_t)T * cpr;
    for (int64_t u = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; u < n; u += (int64_t)gridDim.x * blockDim.x) {
        const int64_t t = u / cpr, c = u - t * cpr;
        const uint4 val = ld16(v + t * row_bytes + c * 16);
#pragma unroll
        for (int i = 0; i < kMaxTopK; ++i) {
            if (i >= k) break;
            const int e = idx[t * k + i];
            const int s = token_slot[t * k + i];
            if (e < 0 || e >= E || s < 0) {
                if (c == 0) set_status(status, DEV_BAD_EXPERT_ID);
                continue;
            }
            // the row must lie in this rank's part of e's segment and inside the receive buffer: a table
            // that disagrees with the routing (or a short buffer) skips the store and is reported
            const int i_e = s - offsets[e];
            const int64_t row = (int64_t)dbase[e] + i_e;
            if (i_e < 0 || i_e >= own[e] || row < 0 || row >= recv_rows) {
                if (c == 0) set_status(status, DEV_BAD_COUNT);
                continue;
            }
            st16(recv[e / E_loc] + row * row_bytes + c * 16, val);
        }
    }
    __threadfence_system();  // the stores reach the owners' memory before this kernel counts as complete
}

// counts_loc[e] = sum_s C[s][rank E_loc + e], offsets_loc = its exclusive prefix (E_loc + 1 entries)
__global__ void __launch_bounds__(256) ep_layout_kernel(const int32_t* __restrict__ table, int rank, int N, int E,
                                                        int32_t* __restrict__ counts_loc,
                                                        int32_t* __restrict__ offsets_loc) {
    __shared__ int col[kMaxExperts];
    pdl_wait();
    pdl_trigger();
    const int E_loc = E / N;
    for (int e = threadIdx.x; e < E_loc; e += blockDim.x) {
        int sum = 0;
        for (int s = 0; s < N; ++s) sum += table[(int64_t)s * E + rank * E_loc + e];
        col[e] = sum;
        counts_loc[e] = sum;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        int run = 0;
        for (int e = 0; e < E_loc; ++e) {
            offsets_loc[e] = run;
            run += col[e];
        }
        offsets_loc[E_loc] = run;
    }
}

__device__ __forceinline__ uint4 ld16_plain(const void* p) { return *reinterpret_cast<const uint4*>(p); }

template <int YDT, int RDT, int ODT>
__global__ void __launch_bounds__(256) ep_combine_kernel(const void* const* __restrict__ ybuf,
                                                         const int32_t* __restrict__ idx,
                                                         const int32_t* __restrict__ token_slot,
                                                         const int32_t* __restrict__ offsets,
                                                         const int32_t* __restrict__ table, int rank, int N, int E,
                                                         const float* __restrict__ w, const void* __restrict__ res,
                                                         int T, int d, int k, void* __restrict__ out,
                                                         int64_t recv_rows, int32_t* status) {
    __shared__ int dbase[kMaxExperts], scratch[kMaxExperts], own[kMaxExperts];
    pdl_wait();
    pdl_trigger();
    ep_dest_base(table, rank, N, E, dbase, scratch);
    for (int e = threadIdx.x; e < E; e += blockDim.x) own[e] = table[(int64_t)rank * E + e];
    __syncthreads();
    const int E_loc = E / N;
    const int lane = threadIdx.x & 31;
    const int nseg = (d + 255) / 256;
    const int64_t n = (int64_t)T * nseg;
    const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
    constexpr int ES = YDT == DT_BF16 ? 2 : 4;
    for (int64_t u = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); u < n; u += warps) {
        const int64_t t = u / nseg;
        const int64_t j = (u - t * nseg) * 256 + lane * 8;
        // lanes below k: the pick's owner and its row there
        int my_owner = 0;
        int64_t my_row = 0;
        float my_w = 0.f;
        int my_ok = 0;
        if (lane < k) {
            const int e = __ldg(idx + t * k + lane);
            const int s = __ldg(token_slot + t * k + lane);
            my_w = __ldg(w + t * k + lane);
            if (e >= 0 && e < E && s >= 0) {
                const int i_e = s - offsets[e];
                my_owner = e / E_loc;
                my_row = (int64_t)dbase[e] + i_e;
                my_ok = i_e >= 0 && i_e < own[e] && my_row >= 0 && my_row < recv_rows;
                if (!my_ok && u - t * nseg == 0) set_status(status, DEV_BAD_COUNT);
            } else if (u - t * nseg == 0) {
                set_status(status, DEV_BAD_EXPERT_ID);
            }
        }
        // a pick that is not valid is skipped: its row is neither read nor weighted
        int owner[kMaxTopK];
        int64_t row[kMaxTopK];
        float wt[kMaxTopK];
        bool ok[kMaxTopK];
#pragma unroll
        for (int i = 0; i < kMaxTopK; ++i) {
            owner[i] = __shfl_sync(0xffffffffu, my_owner, i);
            row[i] = __shfl_sync(0xffffffffu, my_row, i);
            wt[i] = __shfl_sync(0xffffffffu, my_w, i);
            ok[i] = __shfl_sync(0xffffffffu, my_ok, i) != 0;
        }
        if (j >= d) continue;
        constexpr int V = YDT == DT_BF16 ? 1 : 2;
        uint4 raw[kMaxTopK][V];
#pragma unroll
        for (int i = 0; i < kMaxTopK; ++i) {
            if (i < k && ok[i]) {
                const uint8_t* p = static_cast<const uint8_t*>(ybuf[owner[i]]) + (row[i] * d + j) * ES;
#pragma unroll
                for (int vv = 0; vv < V; ++vv) raw[i][vv] = ld16_plain(p + 16 * vv);
            }
        }
        float acc[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) acc[q] = 0.f;
#pragma unroll
        for (int i = 0; i < kMaxTopK; ++i) {
            if (i < k && ok[i]) {
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

cudaError_t launch_ep_dispatch(const Ctx& c, const void* v, int v_dt, const int32_t* idx, const int32_t* token_slot,
                               const int32_t* offsets, const int32_t* table, int rank, int N, int E, int T, int d,
                               int k, void* const* recv, int64_t recv_rows, int32_t* status) {
    if (T == 0) return cudaSuccess;
    const int64_t row_bytes = (int64_t)d * (v_dt == DT_BF16 ? 2 : 4);
    const int64_t n = (int64_t)T * (row_bytes / 16);
    int64_t blocks = (n + 255) / 256;
    const int64_t cap = (int64_t)c.num_sms * 8;
    if (blocks > cap) blocks = cap;
    return launch(ep_dispatch_kernel, dim3((unsigned)blocks), dim3(256), 0, c, static_cast<const uint8_t*>(v),
                  row_bytes, idx, token_slot, offsets, table, rank, N, E, T, k,
                  reinterpret_cast<uint8_t* const*>(recv), recv_rows, status);
}

cudaError_t launch_ep_layout(const Ctx& c, const int32_t* table, int rank, int N, int E, int32_t* counts_loc,
                             int32_t* offsets_loc) {
    return launch(ep_layout_kernel, dim3(1), dim3(256), 0, c, table, rank, N, E, counts_loc, offsets_loc);
}

template <int YDT, int RDT>
static cudaError_t launch_ep_combine_o(const Ctx& c, dim3 g, const void* const* y, const int32_t* idx,
                                      const int32_t* ts, const int32_t* off, const int32_t* table, int rank, int N,
                                      int E, const float* w, const void* res, int T, int d, int k, void* out,
                                      int out_dt, int64_t recv_rows, int32_t* status) {
    if (out_dt == DT_BF16)
        return launch(ep_combine_kernel<YDT, RDT, DT_BF16>, g, dim3(256), 0, c, y, idx, ts, off, table, rank, N, E, w,
                      res, T, d, k, out, recv_rows, status);
    return launch(ep_combine_kernel<YDT, RDT, DT_F32>, g, dim3(256), 0, c, y, idx, ts, off, table, rank, N, E, w, res,
                  T, d, k, out, recv_rows, status);
}

cudaError_t launch_ep_combine(const Ctx& c, const void* const* y, int y_dt, const int32_t* idx,
                              const int32_t* token_slot, const int32_t* offsets, const int32_t* table, int rank, int N,
                              int E, const float* w, const void* res, int r_dt, int T, int d, int k, void* out,
                              int out_dt, int64_t recv_rows, int32_t* status) {
    if (T == 0) return cudaSuccess;
    const int64_t n = (int64_t)T * ((d + 255) / 256);
    int64_t blocks = (n + 7) / 8;
    const int64_t cap = (int64_t)c.num_sms * 16;
    if (blocks > cap) blocks = cap;
    const dim3 g((unsigned)blocks);
    if (y_dt == DT_BF16 && r_dt == DT_BF16)
        return launch_ep_combine_o<DT_BF16, DT_BF16>(c, g, y, idx, token_slot, offsets, table, rank, N, E, w, res, T,
                                                     d, k, out, out_dt, recv_rows, status);
    if (y_dt == DT_BF16)
        return launch_ep_combine_o<DT_BF16, DT_F32>(c, g, y, idx, token_slot, offsets, table, rank, N, E, w, res, T, d,
                                                    k, out, out_dt, recv_rows, status);
    if (r_dt == DT_BF16)
        return launch_ep_combine_o<DT_F32, DT_BF16>(c, g, y, idx, token_slot, offsets, table, rank, N, E, w, res, T, d,
                                                    k, out, out_dt, recv_rows, status);
    return launch_ep_combine_o<DT_F32, DT_F32>(c, g, y, idx, token_slot, offsets, table, rank, N, E, w, res, T, d, k,
                                               out, out_dt, recv_rows, status);
}

}  // namespace moe
