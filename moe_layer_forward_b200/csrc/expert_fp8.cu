// Block-FP8 expert MLP: E4M3 codes with fp32 block scales, on tcgen05 tensor cores
// ("「赤兔」Chitu 框架深度解读（七）", §专家计算实现: FP8 expert GEMMs (DeepGEMM
// fp8_gemm_nt) and the blockfp8 quantised experts).  The page names the scheme
// without defining it; the reading implemented:
//   - weights [n][k]: one fp32 scale per 128 x 128 block; GEMM inputs [rows][k]:
//     one scale per (row, 128 consecutive columns);
//   - s = amax / 448 (IEEE division; 1 for an all-zero block), code = E4M3(x / s)
//     rounded to nearest even, saturating at +-448;
//   - every product is the dot product of dequantised operands (code * scale).
//
// Kernels:
//   quant_rows_kernel      a warp per (row, 128-column block) of a GEMM input
//   quant_tiles_kernel     a CTA per 128 x 128 block of a weight matrix
//   rmsnorm_quant_kernel   RMSNorm of a row (the same fp32 arithmetic as the bf16
//                          path) quantised per 128 columns, plus 1/rms for the router;
//                          rmsnorm_quant_row_kernel the same with a CTA per row (few rows)
//   grouped_gemm_fp8_kernel<SWIGLU, R, NA>
//       weights are the MMA's M operand: 128 weight rows = one row of scale blocks;
//       the expert's rows (tokens) are N <= R.  A tile stages NA = 2 such operands
//       (gate and up, or two consecutive 128-feature blocks of down), because the
//       promotion pass below, not the MMAs or the loads, sets the pace: two
//       operands bring 32 KB of weights per pass.  K runs in 128-wide blocks: a stage
//       holds one 128-byte swizzled row slice per operand (exactly one scale block),
//       and the MMA thread issues 4 kind::f8f6f4 MMAs (K = 32) per operand into one
//       of eight tensor-memory chunk buffers.  Four epilogue warps promote each chunk
//       into fp32 register sums with s_w * s_a(row) and release the buffer, so the
//       next blocks' MMAs overlap the promotion (whose scale loads run one block
//       ahead).  Gate/up ends with SiLU(g) * u and quantises h per (row, 128 features) for the down projection (an amax over
//       the 128 weight rows of the tile: warp shuffles, then the 4 warps in shared
//       memory); down ends with bf16 y.  Activation rows are copied by four loader
//       warps (16-byte cp.async into the swizzled layout, optionally through the
//       permutation's slot -> token map), weights by TMA.
// Every wait is bounded; a wait that gives up raises DEV_TIMEOUT and all roles unwind.
#include <cuda.h>
#include <cuda_fp8.h>
#include <math.h>

#include "common.cuh"
#include "kernels.h"
#include "tc_ptx.cuh"

namespace moe {
namespace fp8 {
using namespace tc;

__device__ __forceinline__ uint32_t e4m3(float x) {
    return (uint32_t)__nv_cvt_float_to_fp8(x, __NV_SATFINITE, __NV_E4M3);
}
__device__ __forceinline__ float block_scale(float amax) { return amax > 0.f ? __fdiv_rn(amax, 448.0f) : 1.0f; }
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

// 4 consecutive elements as fp32 (bf16 or f32; 8- or 16-byte aligned)
template <int DT>
__device__ __forceinline__ void load4(const void* base, int64_t elem, float (&o)[4]) {
    if constexpr (DT == DT_BF16) {
        const uint2 u = __ldg(reinterpret_cast<const uint2*>(static_cast<const uint16_t*>(base) + elem));
        o[0] = bf16_bits_to_f32(u.x & 0xFFFFu);
        o[1] = bf16_bits_to_f32(u.x >> 16);
        o[2] = bf16_bits_to_f32(u.y & 0xFFFFu);
        o[3] = bf16_bits_to_f32(u.y >> 16);
    } else {
        const float4 f = __ldg(reinterpret_cast<const float4*>(static_cast<const float*>(base) + elem));
        o[0] = f.x; o[1] = f.y; o[2] = f.z; o[3] = f.w;
    }
}

// quantise 4 values of a 128-wide block whose 32 lanes hold 4 values each; lane 0 gets the scale
__device__ __forceinline__ uint32_t quant_block4(const float (&v)[4], float& sc) {
    float m = fmaxf(fmaxf(fabsf(v[0]), fabsf(v[1])), fmaxf(fabsf(v[2]), fabsf(v[3])));
    sc = block_scale(warp_max(m));
    return e4m3(__fdiv_rn(v[0], sc)) | (e4m3(__fdiv_rn(v[1], sc)) << 8) | (e4m3(__fdiv_rn(v[2], sc)) << 16) |
           (e4m3(__fdiv_rn(v[3], sc)) << 24);
}

template <int DT>
__global__ void __launch_bounds__(256) quant_rows_kernel(const void* __restrict__ x, int64_t rows, int64_t cols,
                                                         uint8_t* __restrict__ q, float* __restrict__ s) {
    pdl_wait();
    pdl_trigger();
    const int lane = threadIdx.x & 31;
    const int64_t nb = cols / 128, units = rows * nb;
    for (int64_t u = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; u < units;
         u += ((int64_t)gridDim.x * blockDim.x) >> 5) {
        const int64_t r = u / nb, b = u - r * nb;
        const int64_t e0 = r * cols + b * 128 + 4 * lane;
        float v[4], sc;
        load4<DT>(x, e0, v);
        const uint32_t codes = quant_block4(v, sc);
        *reinterpret_cast<uint32_t*>(q + e0) = codes;
        if (lane == 0) s[u] = sc;
    }
}

// 256 threads per 128 x 128 block: thread t covers row t / 2, columns (t % 2) * 64 .. + 63
template <int DT>
__global__ void __launch_bounds__(256) quant_tiles_kernel(const void* __restrict__ x, int64_t rows, int64_t cols,
                                                          uint8_t* __restrict__ q, float* __restrict__ s) {
    __shared__ float red[8];
    pdl_wait();
    pdl_trigger();
    const int64_t nbc = cols / 128;
    const int64_t br = blockIdx.x / nbc, bc = blockIdx.x - br * nbc;
    const int64_t r = br * 128 + (threadIdx.x >> 1);
    const int64_t c0 = bc * 128 + (threadIdx.x & 1) * 64;
    const bool in = r < rows;
    float v[64];
    float m = 0.f;
#pragma unroll
    for (int i = 0; i < 64; i += 4) {
        float t[4] = {0.f, 0.f, 0.f, 0.f};
        if (in) load4<DT>(x, r * cols + c0 + i, t);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            v[i + j] = t[j];
            m = fmaxf(m, fabsf(t[j]));
        }
    }
    m = warp_max(m);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
    __syncthreads();
    float amax = red[0];
#pragma unroll
    for (int w = 1; w < 8; ++w) amax = fmaxf(amax, red[w]);
    const float sc = block_scale(amax);
    if (threadIdx.x == 0) s[blockIdx.x] = sc;
    if (!in) return;
#pragma unroll
    for (int i = 0; i < 64; i += 16) {
        uint32_t w4[4];
#pragma unroll
        for (int j = 0; j < 4; ++j)
            w4[j] = e4m3(__fdiv_rn(v[i + 4 * j], sc)) | (e4m3(__fdiv_rn(v[i + 4 * j + 1], sc)) << 8) |
                    (e4m3(__fdiv_rn(v[i + 4 * j + 2], sc)) << 16) | (e4m3(__fdiv_rn(v[i + 4 * j + 3], sc)) << 24);
        st16(q + r * cols + c0 + i, make_uint4(w4[0], w4[1], w4[2], w4[3]));
    }
}

// a warp per row: the bf16 path's RMSNorm arithmetic (sum of squares in the same order, v = (x r) gamma
// in fp32), then codes and scales per 128 columns
template <int XDT>
__global__ void __launch_bounds__(256) rmsnorm_quant_kernel(const void* __restrict__ x, const float* __restrict__ gamma,
                                                            int T, int d, float eps, uint8_t* __restrict__ q,
                                                            float* __restrict__ s, float* __restrict__ rstd_out) {
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
    if (lane == 0) rstd_out[t] = r;
    const int nb = d / 128;
    for (int b = 0; b < nb; ++b) {
        const int j = b * 128 + 4 * lane;
        float a[4], g[4], v[4], sc;
        load4<XDT>(x, row + j, a);
        load4<DT_F32>(gamma, j, g);
#pragma unroll
        for (int i = 0; i < 4; ++i) v[i] = (a[i] * r) * g[i];
        const uint32_t codes = quant_block4(v, sc);
        *reinterpret_cast<uint32_t*>(q + row + j) = codes;
        if (lane == 0) s[t * nb + b] = sc;
    }
}

// The same for batches of fewer rows than two waves of warp-per-row CTAs: a
// 256-thread CTA per row sums the squares in the order of the bf16 path's
// row kernel (so 1/rms is the same to the bit), then each warp quantises
// 128-column blocks w, w + 8, ... of the row.
template <int XDT>
__global__ void __launch_bounds__(256) rmsnorm_quant_row_kernel(const void* __restrict__ x,
                                                                const float* __restrict__ gamma, int T, int d,
                                                                float eps, uint8_t* __restrict__ q,
                                                                float* __restrict__ s, float* __restrict__ rstd_out) {
    __shared__ float part[8];
    pdl_wait();
    pdl_trigger();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t t = blockIdx.x, row = t * d;
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
    if (threadIdx.x == 0) rstd_out[t] = r;
    const int nb = d / 128;
    for (int b = warp; b < nb; b += 8) {
        const int j = b * 128 + 4 * lane;
        float a[4], g[4], v[4], sc;
        load4<XDT>(x, row + j, a);
        load4<DT_F32>(gamma, j, g);
#pragma unroll
        for (int i = 0; i < 4; ++i) v[i] = (a[i] * r) * g[i];
        const uint32_t codes = quant_block4(v, sc);
        *reinterpret_cast<uint32_t*>(q + row + j) = codes;
        if (lane == 0) s[t * nb + b] = sc;
    }
}

// ----------------------------------------------------------------------------- grouped GEMM
constexpr int kThreads = 320;
constexpr int kSmemLimit = 232448;

// NA = 128-row weight operands per tile: gate/up stages a gate and an up block
// (NA = 2); down stages one (128 output features) or two consecutive ones (256).
template <bool SWIGLU, int R, int NA>
struct Cfg {
    static_assert(R == 16 || R == 32, "token columns per tile");
    static_assert(NA == 2 || (!SWIGLU && NA == 1), "weight operands per tile");
    static constexpr int NUM_A = NA;
    static constexpr int WROWS = SWIGLU ? 128 : 128 * NA;  // output features of a tile
    static constexpr int A_BYTES = 128 * 128;  // 128 weight rows x one 128-byte K block
    static constexpr int B_BYTES = R * 128;
    static constexpr int STAGE_BYTES = NUM_A * A_BYTES + B_BYTES;
    static constexpr int AUX_BYTES = 5120;
    static constexpr int STAGES_MAX = (kSmemLimit - 1024 - AUX_BYTES) / STAGE_BYTES;
    static constexpr int STAGES = STAGES_MAX > 8 ? 8 : STAGES_MAX;
    static_assert(STAGES >= 3, "pipeline depth");
    static constexpr int CB = NUM_A * R;  // columns of one chunk buffer: gate | up, or the two down blocks
    static constexpr int NBUF = 8;        // chunk buffers: the MMAs run up to 7 K blocks ahead of the promotion
    static constexpr int TMEM_COLS = NBUF * CB <= 128 ? 128 : (NBUF * CB <= 256 ? 256 : 512);
    static_assert(NBUF * CB <= 512, "tensor memory");
    static constexpr int SMEM = 1024 + STAGES * STAGE_BYTES + AUX_BYTES;
};

struct Args {
    const int32_t* counts;
    const int32_t* offsets;
    int E;
    int K;      // reduction length (d for gate/up, d_ff for down), multiple of 128
    int n_out;  // weight rows per expert, multiple of 128
    const uint8_t* act;     // GEMM input codes [rows][K]
    const float* act_s;     // and scales [rows][K / 128]
    const int32_t* gather;  // optional: slot i reads input row gather[i]
    const float* w1_s;      // weight scales [E][n_out / 128][K / 128] (gate, or down)
    const float* w2_s;      // (up)
    uint8_t* out_q;         // gate/up: h codes [S][n_out]
    float* out_s;           //          h scales [S][n_out / 128]
    uint16_t* out;          // down:    y bf16 [S][n_out]
    int32_t* status;
    int S;                  // rows of the expert-contiguous outputs; a segment that does not fit is clamped and flagged
    int act_rows;           // rows of act when gather is set
    // bounded waits: the limit of one wait, and (failure-path tests only) an extra wait on a barrier
    // that nothing completes, made by the epilogue warps before their first tile
    uint64_t wait_ns = kTimeoutNs;
    int stall = 0;
};

// input row of expert-contiguous slot `slot`: the slot itself, or its entry of the gather map (a map
// entry outside the input reads row 0 instead and is flagged)
__device__ __forceinline__ int input_row(const Args& p, int slot) {
    if (!p.gather) return slot;
    const int t = p.gather[slot];
    if (t < 0 || t >= p.act_rows) {
        set_status(p.status, DEV_BAD_COUNT);
        return 0;
    }
    return t;
}

struct Aux {
    uint64_t full[8];
    uint64_t empty[8];
    uint64_t cfull[8];
    uint64_t cempty[8];
    uint64_t drain;
    uint64_t redbar;  // the 4 epilogue warps' per-tile rendezvous on red
    uint64_t never;   // completed by nothing: the injected stall waits on it
    uint32_t tmem_slot;
    int abort_flag;
    float red[2][4][32];  // by tile parity: a warp reaches tile j+2's rendezvous only after all read tile j's
    int tstart[kMaxExperts + 1];
    int cnt[kMaxExperts];
    int off[kMaxExperts];
};
static_assert(sizeof(Aux) <= 5120, "aux block");

__device__ __forceinline__ void decode_tile(const Aux& a, int E, int R, int tile, int& e, int& rb, int& cb) {
    int lo = 0, hi = E - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (a.tstart[mid] <= tile) lo = mid; else hi = mid - 1;
    }
    e = lo;
    const int local = tile - a.tstart[e];
    const int nrb = (a.cnt[e] + R - 1) / R;
    cb = local / nrb;
    rb = local - cb * nrb;
}

template <bool SWIGLU, int R, int NA>
__global__ void __launch_bounds__(kThreads, 1)
    grouped_gemm_fp8_kernel(const __grid_constant__ CUtensorMap tm_w1, const __grid_constant__ CUtensorMap tm_w2,
                            const Args p) {
    using C = Cfg<SWIGLU, R, NA>;
    constexpr int STAGES = C::STAGES;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    Aux& aux = *reinterpret_cast<Aux*>(smem + STAGES * C::STAGE_BYTES);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    volatile int* abort_flag = &aux.abort_flag;
    const uint64_t wait_ns = p.wait_ns;

    if (warp == 0 && lane == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(smem_u32(&aux.full[s]), 2);  // weight TMA (with its bytes) + the activation loader
            mbar_init(smem_u32(&aux.empty[s]), 1);
        }
        for (int c = 0; c < C::NBUF; ++c) {
            mbar_init(smem_u32(&aux.cfull[c]), 1);
            mbar_init(smem_u32(&aux.cempty[c]), 4);
        }
        mbar_init(smem_u32(&aux.drain), 1);
        mbar_init(smem_u32(&aux.redbar), 4);
        mbar_init(smem_u32(&aux.never), 1);
        aux.abort_flag = 0;
        fence_mbar_init();
        tma_prefetch(&tm_w1);
        if (SWIGLU) tma_prefetch(&tm_w2);
    }
    if (warp == 1) tmem_alloc(smem_u32(&aux.tmem_slot), C::TMEM_COLS);

    pdl_wait();
    const int E = p.E;
    for (int e = threadIdx.x; e < E; e += kThreads) {
        int o, n;
        if (!clamp_segment(p.offsets[e], p.counts[e], p.S, o, n)) set_status(p.status, DEV_BAD_COUNT);
        aux.cnt[e] = n;
        aux.off[e] = o;
    }
    __syncthreads();
    if (warp == 0) {
        const int ncb = p.n_out / C::WROWS;
        int loc[8], sum = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int e = lane * 8 + i;
            loc[i] = (e < E) ? ((aux.cnt[e] + R - 1) / R) * ncb : 0;
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
            if (e < E) aux.tstart[e] = run;
            run += loc[i];
        }
        if (lane == 31) aux.tstart[E] = incl;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    pdl_trigger();
    const uint32_t tmem_base = aux.tmem_slot;
    const int total = aux.tstart[E];
    const int nk = p.K / 128;

    auto give_up = [&]() {
        if (lane == 0) {
            *abort_flag = 1;
            set_status(p.status, DEV_TIMEOUT);
        }
    };

    if (warp == 0) {
        // ================= weight TMA producer
        int stage = 0;
        uint32_t phase = 0, used = 0, last_parity = 0;
        for (int tile = blockIdx.x; tile < total && !*abort_flag; tile += gridDim.x) {
            int e, rb, cb;
            decode_tile(aux, E, R, tile, e, rb, cb);
            const int w_row = e * p.n_out + cb * C::WROWS;
            bool ok = true;
            for (int kb = 0; kb < nk; ++kb) {
                const uint32_t full = smem_u32(&aux.full[stage]);
                if (!warp_wait(smem_u32(&aux.empty[stage]), phase ^ 1u, abort_flag, wait_ns)) {
                    give_up();
                    ok = false;
                    break;
                }
                if (lane == 0) {
                    const uint32_t a0 = smem_u32(smem + stage * C::STAGE_BYTES);
                    mbar_expect_tx(full, C::NUM_A * C::A_BYTES);
                    tma_load_2d(a0, &tm_w1, kb * 128, w_row, full);
                    if (SWIGLU) tma_load_2d(a0 + C::A_BYTES, &tm_w2, kb * 128, w_row, full);
                    else if (NA == 2) tma_load_2d(a0 + C::A_BYTES, &tm_w1, kb * 128, w_row + 128, full);
                }
                used |= 1u << stage;
                last_parity = (last_parity & ~(1u << stage)) | (phase << stage);
                if (++stage == STAGES) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
            if (!ok) break;
        }
        {
            const uint64_t dl = drain_deadline();
            for (int s = 0; s < STAGES; ++s)
                if (used & (1u << s)) mbar_drain(smem_u32(&aux.full[s]), (last_parity >> s) & 1u, dl);
        }
    } else if (warp == 1) {
        // ================= MMA issuer
        int stage = 0;
        uint32_t phase = 0, q = 0;
        bool ok = true;
        for (int tile = blockIdx.x; tile < total && ok && !*abort_flag; tile += gridDim.x) {
            int e, rb, cb;
            decode_tile(aux, E, R, tile, e, rb, cb);
            const int rows = min(R, aux.cnt[e] - rb * R);
            const uint32_t idesc = idesc_e4m3(128, (rows + 15) & ~15);
            for (int kb = 0; kb < nk; ++kb, ++q) {
                const uint32_t c = q % C::NBUF, use = q / C::NBUF;
                if (!warp_wait(smem_u32(&aux.full[stage]), phase, abort_flag, wait_ns) ||
                    !warp_wait(smem_u32(&aux.cempty[c]), (use & 1u) ^ 1u, abort_flag, wait_ns)) {
                    give_up();
                    ok = false;
                    break;
                }
                tc_fence_after();
                if (lane == 0) {
                    const uint32_t a0 = smem_u32(smem + stage * C::STAGE_BYTES);
                    const uint32_t b0 = a0 + C::NUM_A * C::A_BYTES;
                    const uint32_t d = tmem_base + c * C::CB;
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        const uint64_t bd = sdesc_sw128(b0 + kk * 32);
                        tc_mma_f8(d, sdesc_sw128(a0 + kk * 32), bd, idesc, kk > 0 ? 1u : 0u);
                        if (NA == 2) tc_mma_f8(d + R, sdesc_sw128(a0 + C::A_BYTES + kk * 32), bd, idesc, kk > 0 ? 1u : 0u);
                    }
                    tc_commit(smem_u32(&aux.empty[stage]));
                    tc_commit(smem_u32(&aux.cfull[c]));
                }
                __syncwarp();
                if (++stage == STAGES) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
        }
        if (lane == 0) {
            tc_commit(smem_u32(&aux.drain));
            mbar_drain(smem_u32(&aux.drain), 0, drain_deadline());
        }
        __syncwarp();
    } else if (warp >= 6) {
        // ================= activation loaders: warp gw fills stages gw, gw + 4, ...
        constexpr int RPL = R / 4;  // rows per lane: lane covers rows lane / 8 + 4 i, 16-byte chunk lane % 8
        const int gw = warp - 6, c = lane & 7, r0 = lane >> 3;
        int src_row[RPL];
        int cur = -1, rows = 0;
        for (int g = gw;; g += 4) {
            const int ti = g / nk, kb = g - ti * nk;
            const int tile = blockIdx.x + ti * gridDim.x;
            // (no abort check here: a stage the producer armed is always filled, so its drain completes)
            if (tile >= total) break;
            if (tile != cur) {
                int e, rb, cb;
                decode_tile(aux, E, R, tile, e, rb, cb);
                rows = min(R, aux.cnt[e] - rb * R);
                const int base = aux.off[e] + rb * R;
#pragma unroll
                for (int i = 0; i < RPL; ++i) {
                    const int r = r0 + 4 * i;
                    src_row[i] = r < rows ? input_row(p, base + r) : 0;
                }
                cur = tile;
            }
            const int stage = g % STAGES;
            const uint32_t use = (uint32_t)(g / STAGES);
            if (!warp_wait(smem_u32(&aux.empty[stage]), (use & 1u) ^ 1u, abort_flag, wait_ns)) {
                give_up();
                break;
            }
            const uint32_t dst = smem_u32(smem + stage * C::STAGE_BYTES) + C::NUM_A * C::A_BYTES;
#pragma unroll
            for (int i = 0; i < RPL; ++i) {
                const int r = r0 + 4 * i;
                if (r < rows)  // rows past the tile's count feed only columns that are never stored
                    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst + r * 128 + ((c ^ (r & 7)) << 4)),
                                 "l"(p.act + (int64_t)src_row[i] * p.K + kb * 128 + c * 16)
                                 : "memory");
            }
            asm volatile("cp.async.wait_all;" ::: "memory");
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&aux.full[stage]));
        }
    } else {
        // ================= promotion and epilogue (warps 2..5: TMEM lane quarter qw = weight rows 32 qw ..)
        const int qw = warp & 3;
        const int f = 32 * qw + lane;  // weight row inside the tile's 128
        uint32_t q = 0, j = 0;
        bool ok = true;
        if (p.stall && !warp_wait(smem_u32(&aux.never), 0, abort_flag, wait_ns)) {
            give_up();
            ok = false;
        }
        for (int tile = blockIdx.x; tile < total && ok && !*abort_flag; tile += gridDim.x, ++j) {
            int e, rb, cb;
            decode_tile(aux, E, R, tile, e, rb, cb);
            const int rows = min(R, aux.cnt[e] - rb * R);
            const int base = aux.off[e] + rb * R;
            // lane n < rows: input row of token column n (its activation scales)
            const int my_row = lane < rows ? input_row(p, base + lane) : 0;
            // weight scale rows: gate and up of block cb, or down blocks NA*cb (and NA*cb + 1)
            const int64_t wb = (int64_t)e * (p.n_out / 128) + (SWIGLU ? cb : NA * cb);
            const float* s1 = p.w1_s + wb * nk;
            const float* s2 = SWIGLU ? p.w2_s + wb * nk : (NA == 2 ? p.w1_s + (wb + 1) * nk : nullptr);
            float g[R], u[R];
#pragma unroll
            for (int n = 0; n < R; ++n) g[n] = u[n] = 0.f;
            // scales of the next block load while this block's chunk is awaited
            float sw1_n = __ldg(s1), sw2_n = NA == 2 ? __ldg(s2) : 0.f;
            float sa_n = lane < rows ? __ldg(p.act_s + (int64_t)my_row * nk) : 0.f;
            for (int kb = 0; kb < nk; ++kb, ++q) {
                const float sw1 = sw1_n, sw2 = sw2_n, my_sa = sa_n;
                if (kb + 1 < nk) {
                    sw1_n = __ldg(s1 + kb + 1);
                    if (NA == 2) sw2_n = __ldg(s2 + kb + 1);
                    sa_n = lane < rows ? __ldg(p.act_s + (int64_t)my_row * nk + kb + 1) : 0.f;
                }
                const uint32_t c = q % C::NBUF, use = q / C::NBUF;
                if (!warp_wait(smem_u32(&aux.cfull[c]), use & 1u, abort_flag, wait_ns)) {
                    give_up();
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t ta = tmem_base + c * C::CB + ((uint32_t)(32 * qw) << 16);
                uint32_t cg[R], cu[R];
                tmem_ld<R>(ta, cg);
                if (NA == 2) tmem_ld<R>(ta + R, cu);
                tmem_wait_ld(cg);
                if (NA == 2) tmem_wait_ld(cu);
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_u32(&aux.cempty[c]));
#pragma unroll
                for (int n = 0; n < R; ++n) {
                    const float sa = __shfl_sync(0xffffffffu, my_sa, n);
                    g[n] = fmaf(__uint_as_float(cg[n]), sw1 * sa, g[n]);
                    if (NA == 2) u[n] = fmaf(__uint_as_float(cu[n]), sw2 * sa, u[n]);
                }
            }
            if (!ok) break;
            if constexpr (SWIGLU) {
                // h = SiLU(g) * u, then codes per (row, these 128 features): amax over the tile's 128 weight rows
                float h[R];
                float(&red)[4][32] = aux.red[j & 1u];
#pragma unroll
                for (int n = 0; n < R; ++n) {
                    h[n] = n < rows ? g[n] / (1.0f + expf(-g[n])) * u[n] : 0.f;
                    const float m = warp_max(fabsf(h[n]));
                    if (lane == 0) red[qw][n] = m;
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_u32(&aux.redbar));
                if (!warp_wait(smem_u32(&aux.redbar), j & 1u, abort_flag, wait_ns)) {
                    give_up();
                    break;
                }
                const int nfb = p.n_out / 128;
#pragma unroll
                for (int n = 0; n < R; ++n) {
                    if (n < rows) {
                        const float amax = fmaxf(fmaxf(red[0][n], red[1][n]), fmaxf(red[2][n], red[3][n]));
                        const float sc = block_scale(amax);
                        const int64_t slot = base + n;
                        p.out_q[slot * p.n_out + cb * 128 + f] = (uint8_t)e4m3(__fdiv_rn(h[n], sc));
                        if (f == 0) p.out_s[slot * nfb + cb] = sc;
                    }
                }
            } else {
#pragma unroll
                for (int n = 0; n < R; ++n)
                    if (n < rows) {
                        uint16_t* o = p.out + (int64_t)(base + n) * p.n_out + cb * C::WROWS + f;
                        o[0] = (uint16_t)f32_to_bf16_bits(g[n]);
                        if (NA == 2) o[128] = (uint16_t)f32_to_bf16_bits(u[n]);
                    }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem_base, C::TMEM_COLS);
}

// 8-bit matrix [rows][inner], box = 128 bytes x 128 rows, 128-byte swizzle
static bool encode_u8(CUtensorMap* tm, const void* base, uint64_t inner, uint64_t rows) {
    EncodeTiledFn fn = encode_tiled_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {inner, rows};
    cuuint64_t strides[1] = {inner};
    cuuint32_t box[2] = {128, 128};
    cuuint32_t estr[2] = {1, 1};
    return fn(tm, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <bool SWIGLU, int R, int NA = 2>
static cudaError_t run(const Ctx& c, int S, const void* w1, const void* w2, Args a) {
    using CF = Cfg<SWIGLU, R, NA>;
    set_wait_args(a);
    auto kern = grouped_gemm_fp8_kernel<SWIGLU, R, NA>;
    static bool attr_done[64] = {};
    if (c.device < 0 || c.device >= 64) return cudaErrorInvalidDevice;
    if (!attr_done[c.device]) {
        cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, CF::SMEM);
        if (err != cudaSuccess) return err;
        attr_done[c.device] = true;
    }
    CUtensorMap tm_w1, tm_w2;
    const uint64_t wrows = (uint64_t)a.E * a.n_out;
    if (!encode_u8(&tm_w1, w1, (uint64_t)a.K, wrows)) return cudaErrorInvalidValue;
    if (!encode_u8(&tm_w2, SWIGLU ? w2 : w1, (uint64_t)a.K, wrows)) return cudaErrorInvalidValue;
    const int64_t max_tiles = ((int64_t)S / R + a.E) * (a.n_out / CF::WROWS);
    const int grid = (int)(max_tiles < c.num_sms ? max_tiles : c.num_sms);
    if (grid <= 0) return cudaSuccess;
    return launch(kern, dim3(grid), dim3(kThreads), (size_t)CF::SMEM, c, tm_w1, tm_w2, a);
}

}  // namespace fp8

cudaError_t launch_quant_fp8(const Ctx& c, const void* x, int dt, int64_t rows, int64_t cols, int blk_rows,
                             uint8_t* q, float* s) {
    if (rows == 0) return cudaSuccess;
    if (blk_rows == 128) {
        const int64_t blocks = ((rows + 127) / 128) * (cols / 128);
        if (dt == DT_BF16) return launch(fp8::quant_tiles_kernel<DT_BF16>, dim3((unsigned)blocks), dim3(256), 0, c, x, rows, cols, q, s);
        return launch(fp8::quant_tiles_kernel<DT_F32>, dim3((unsigned)blocks), dim3(256), 0, c, x, rows, cols, q, s);
    }
    int64_t blocks = (rows * (cols / 128) + 7) / 8;
    const int64_t cap = (int64_t)c.num_sms * 16;
    if (blocks > cap) blocks = cap;
    if (dt == DT_BF16) return launch(fp8::quant_rows_kernel<DT_BF16>, dim3((unsigned)blocks), dim3(256), 0, c, x, rows, cols, q, s);
    return launch(fp8::quant_rows_kernel<DT_F32>, dim3((unsigned)blocks), dim3(256), 0, c, x, rows, cols, q, s);
}

cudaError_t launch_rmsnorm_quant(const Ctx& c, const void* x, int x_dt, const float* gamma, int T, int d, float eps,
                                 uint8_t* q, float* s, float* rstd) {
    if (T == 0) return cudaSuccess;
    if (T <= 2 * 8 * c.num_sms) {  // fewer rows than two waves of warp-per-row CTAs
        if (x_dt == DT_BF16)
            return launch(fp8::rmsnorm_quant_row_kernel<DT_BF16>, dim3(T), dim3(256), 0, c, x, gamma, T, d, eps, q, s,
                          rstd);
        return launch(fp8::rmsnorm_quant_row_kernel<DT_F32>, dim3(T), dim3(256), 0, c, x, gamma, T, d, eps, q, s, rstd);
    }
    const dim3 g((T + 7) / 8);
    if (x_dt == DT_BF16) return launch(fp8::rmsnorm_quant_kernel<DT_BF16>, g, dim3(256), 0, c, x, gamma, T, d, eps, q, s, rstd);
    return launch(fp8::rmsnorm_quant_kernel<DT_F32>, g, dim3(256), 0, c, x, gamma, T, d, eps, q, s, rstd);
}

// token columns per tile: 16 up to 8 rows per expert on average, else 32 (more row blocks)
static int fp8_rows(int S, int E) { return E > 0 && S / E <= 8 ? 16 : 32; }

cudaError_t launch_gate_up_fp8(const Ctx& c, const uint8_t* xq, const float* xs, const int32_t* gather,
                               const uint8_t* Wg, const float* Wg_s, const uint8_t* Wu, const float* Wu_s,
                               const int32_t* counts, const int32_t* offsets, int S, int E, int d, int d_ff,
                               uint8_t* hq, float* hs, int32_t* status, int act_rows) {
    if (S == 0) return cudaSuccess;
    fp8::Args a{counts, offsets, E, d, d_ff, xq, xs, gather, Wg_s, Wu_s, hq, hs, nullptr, status, S,
                gather ? act_rows : S};
    if (fp8_rows(S, E) == 16) return fp8::run<true, 16>(c, S, Wg, Wu, a);
    return fp8::run<true, 32>(c, S, Wg, Wu, a);
}

cudaError_t launch_down_fp8(const Ctx& c, const uint8_t* hq, const float* hs, const uint8_t* Wd, const float* Wd_s,
                            const int32_t* counts, const int32_t* offsets, int S, int E, int d, int d_ff, void* y,
                            int32_t* status) {
    if (S == 0) return cudaSuccess;
    fp8::Args a{counts, offsets, E, d_ff, d, hq, hs, nullptr, Wd_s, nullptr, nullptr, nullptr,
                static_cast<uint16_t*>(y), status, S, S};
    // two 128-row weight blocks per tile where d allows: each promotion pass then covers 32 KB of
    // weights instead of 16 (the pass, not the MMAs or the loads, paces the 128-row tile)
    const bool wide = d % 256 == 0;
    if (fp8_rows(S, E) == 16)
        return wide ? fp8::run<false, 16, 2>(c, S, Wd, nullptr, a) : fp8::run<false, 16, 1>(c, S, Wd, nullptr, a);
    return wide ? fp8::run<false, 32, 2>(c, S, Wd, nullptr, a) : fp8::run<false, 32, 1>(c, S, Wd, nullptr, a);
}

}  // namespace moe
