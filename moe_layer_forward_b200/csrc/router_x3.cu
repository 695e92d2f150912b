// Router logits for bf16 token rows: z = rstd * (x (gamma ⊙ W_r)^T) on the tensor cores at fp32 accuracy.
//
// "推理计算流梳理" (huanyp.cn), §专家并行 / MoE Router 过程: z = v W_r^T with v the
// RMSNorm output, v_j = rstd * gamma_j * x_j (§Norm&Residual).  rstd is one
// scalar per token and gamma one per column, so
//     z_e = rstd * sum_j x_j * (gamma_j W_r[e][j]).
// When x is bf16 it is an exact MMA operand.  W' = gamma ⊙ W_r is rounded
// once to fp32 and split exactly into three bf16 terms,
//     W' = w_hi + w_mid + w_lo   (w_hi = bf16(W'), w_mid = bf16(W' - w_hi),
//                                 w_lo = bf16(W' - w_hi - w_mid), no remainder),
// so x·W' = x·w_hi + x·w_mid + x·w_lo with every product exact in fp32: three
// bf16 MMAs per K = 16 accumulate it in fp32 in tensor memory.  Against the
// 3xTF32 form (router_tc.cu) this moves half the bytes through shared memory
// per K (x needs no split, and bf16 K = 16 fills the 32-byte MMA row that
// tf32 fills with K = 8) and needs no warps to build the A operand: x comes
// straight from HBM by TMA.  As there, each 128 columns of K accumulate in
// their own TMEM chunk, added in fp32 round-to-nearest to a running sum
// (the tensor core's long accumulations drift), and rstd multiplies the final
// sum of each K split.
//
// router_w3split_kernel  W' = gamma ⊙ W_r -> (w_hi, w_mid, w_lo), [3][E][d] bf16.
// router_x3_kernel       persistent over (128-token tile, block of <= 128 experts,
//                        K split) units:
//   warp 0       TMA: the x tile (128 rows x 64 columns) and the three weight
//                slices of each 64-column stage (128-byte swizzle)
//   warp 1       TMEM owner; lane 0 issues 3 bf16 MMAs per K = 16 into one of
//                two chunk accumulators
//   warps 2..5   add each finished chunk to the running sum in TMEM; after the
//                last chunk of a unit, write rstd * sum as the fp32 partial
//                logits [split][T][E] that router_topk_kernel sums
#include <cuda.h>
#include <math.h>

#include "common.cuh"
#include "kernels.h"
#include "tc_ptx.cuh"

namespace moe {
namespace rx3 {
using namespace tc;

constexpr int BM = 128;          // tokens per tile (MMA M)
constexpr int BK = 64;           // bf16 K elements per stage: one 128-byte swizzled row
constexpr int kChunkStages = 2;  // stages (128 columns of K) per TMEM chunk before promotion
constexpr int kThreads = 192;
constexpr int kSmemLimit = 232448;

template <int NP>
struct XCfg {
    static_assert(NP % 16 == 0 && NP >= 32 && NP <= 128, "padded expert block");
    static constexpr int A_BYTES = BM * 128;
    static constexpr int B_BYTES = NP * 128;
    static constexpr int STAGE_BYTES = A_BYTES + 3 * B_BYTES;
    static constexpr int AUX_BYTES = 1024;
    static constexpr int ST = (kSmemLimit - 1024 - AUX_BYTES) / STAGE_BYTES;
    static constexpr int STAGES = ST > 4 ? 4 : ST;
    static_assert(STAGES >= 2, "pipeline depth");
    // columns [0, NP): running sum; [NP, 2NP) and [2NP, 3NP): chunk accumulators
    static constexpr int TMEM_COLS = (3 * NP <= 128) ? 128 : (3 * NP <= 256) ? 256 : 512;
    static constexpr int SMEM = 1024 + STAGES * STAGE_BYTES + AUX_BYTES;
};

struct XAux {
    uint64_t full[4];
    uint64_t empty[4];
    uint64_t cfull[2];
    uint64_t cempty[2];
    uint64_t drain;
    uint64_t never;  // completed by nothing: the injected stall waits on it
    uint32_t tmem_slot;
    int abort_flag;
};

struct XArgs {
    const float* rstd;  // [T]
    float* partial;     // [ksplit][T][E]
    int T, d, E;
    int neb;               // expert blocks of NP
    int ksplit;            // K splits (= slices of partial)
    int chunks_per_split;  // 128-column chunks of K per split; trailing splits may be empty
    int32_t* status;
    // bounded waits: the limit of one wait, and (failure-path tests only) an extra wait on a barrier
    // that nothing completes, made by the epilogue warps before their first unit
    uint64_t wait_ns = kTimeoutNs;
    int stall = 0;
};

__global__ void __launch_bounds__(256) router_w3split_kernel(const float* __restrict__ W,
                                                             const float* __restrict__ gamma, int d, int64_t n,
                                                             uint16_t* __restrict__ parts) {
    pdl_wait();
    pdl_trigger();
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
        const float w = W[i] * gamma[i % d];
        const uint32_t hi = f32_to_bf16_bits(w);
        const float r1 = w - bf16_bits_to_f32(hi);  // exact
        const uint32_t mid = f32_to_bf16_bits(r1);
        const float r2 = r1 - bf16_bits_to_f32(mid);  // exact, and exactly a bf16 value
        parts[i] = (uint16_t)hi;
        parts[n + i] = (uint16_t)mid;
        parts[2 * n + i] = (uint16_t)f32_to_bf16_bits(r2);
    }
}

template <int NP>
__global__ void __launch_bounds__(kThreads, 1)
    router_x3_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
                     const XArgs p) {
    using C = XCfg<NP>;
    constexpr int STAGES = C::STAGES;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    XAux& aux = *reinterpret_cast<XAux*>(smem + STAGES * C::STAGE_BYTES);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    volatile int* abort_flag = &aux.abort_flag;
    const uint64_t wait_ns = p.wait_ns;

    if (warp == 0 && lane == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(smem_u32(&aux.full[s]), 1);
            mbar_init(smem_u32(&aux.empty[s]), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(smem_u32(&aux.cfull[b]), 1);
            mbar_init(smem_u32(&aux.cempty[b]), 4);
        }
        mbar_init(smem_u32(&aux.drain), 1);
        mbar_init(smem_u32(&aux.never), 1);
        aux.abort_flag = 0;
        fence_mbar_init();
        tma_prefetch(&tm_x);
        tma_prefetch(&tm_w);
    }
    if (warp == 1) tmem_alloc(smem_u32(&aux.tmem_slot), C::TMEM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = aux.tmem_slot;
    pdl_wait();
    pdl_trigger();

    const int tiles = (p.T + BM - 1) / BM;
    const int per_tile = p.neb * p.ksplit;
    const int units = tiles * per_tile;
    const int nchunks = p.d / 128;
    // 128-column chunks [c0, c1) of unit u's K split (empty for a trailing split)
    auto chunk_range = [&](int u, int& c0, int& c1) {
        const int split = (u % per_tile) % p.ksplit;
        c0 = split * p.chunks_per_split;
        c1 = min(nchunks, c0 + p.chunks_per_split);
    };
    auto raise_abort = [&]() {
        if (lane == 0) {
            *abort_flag = 1;
            set_status(p.status, DEV_TIMEOUT);
        }
    };

    if (warp == 0) {
        // ================= TMA: x tile and the three weight slices of each stage
        int stage = 0;
        uint32_t phase = 0, used = 0, last_parity = 0;
        for (int u = blockIdx.x; u < units && !*abort_flag; u += gridDim.x) {
            const int tile = u / per_tile, eblk = (u % per_tile) / p.ksplit;
            int c0, c1;
            chunk_range(u, c0, c1);
            bool ok = true;
            for (int kb = kChunkStages * c0; kb < kChunkStages * c1; ++kb) {
                if (!warp_wait(smem_u32(&aux.empty[stage]), phase ^ 1u, abort_flag, wait_ns)) {
                    ok = false;
                    break;
                }
                if (lane == 0) {
                    const uint32_t st = smem_u32(smem + stage * C::STAGE_BYTES);
                    const uint32_t full = smem_u32(&aux.full[stage]);
                    mbar_expect_tx(full, C::STAGE_BYTES);
                    tma_load_2d(st, &tm_x, kb * BK, tile * BM, full);
#pragma unroll
                    for (int q = 0; q < 3; ++q)
                        tma_load_2d(st + C::A_BYTES + q * C::B_BYTES, &tm_w, kb * BK, q * p.E + eblk * NP, full);
                }
                used |= 1u << stage;
                last_parity = (last_parity & ~(1u << stage)) | (phase << stage);
                if (++stage == STAGES) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
            if (!ok) {
                raise_abort();
                break;
            }
        }
        {
            const uint64_t dl = drain_deadline();
            for (int s = 0; s < STAGES; ++s)
                if (used & (1u << s)) mbar_drain(smem_u32(&aux.full[s]), (last_parity >> s) & 1u, dl);
        }
    } else if (warp == 1) {
        // ================= MMA issuer: one chunk accumulator per kChunkStages stages, alternating
        int stage = 0;
        uint32_t phase = 0;
        int g = 0;  // chunks issued so far
        const uint32_t idesc = idesc_bf16(BM, NP);
        bool ok = true;
        for (int u = blockIdx.x; u < units && ok && !*abort_flag; u += gridDim.x) {
            int c0, c1;
            chunk_range(u, c0, c1);
            for (int ch = c0; ch < c1 && ok; ++ch, ++g) {
                const int buf = g & 1;
                if (!warp_wait(smem_u32(&aux.cempty[buf]), ((uint32_t)(g >> 1) & 1u) ^ 1u, abort_flag, wait_ns)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)((1 + buf) * NP);
                for (int s = 0; s < kChunkStages; ++s) {
                    if (!warp_wait(smem_u32(&aux.full[stage]), phase, abort_flag, wait_ns)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    if (lane == 0) {
                        const uint32_t a0 = smem_u32(smem + stage * C::STAGE_BYTES);
#pragma unroll
                        for (int kk = 0; kk < BK / 16; ++kk) {
                            const uint32_t o = kk * 32;
#pragma unroll
                            for (int q = 0; q < 3; ++q)
                                tc_mma(d_tmem, sdesc_sw128(a0 + o), sdesc_sw128(a0 + C::A_BYTES + q * C::B_BYTES + o),
                                       idesc, (s | kk | q) ? 1u : 0u);
                        }
                        tc_commit(smem_u32(&aux.empty[stage]));
                    }
                    __syncwarp();
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok) break;
                if (lane == 0) tc_commit(smem_u32(&aux.cfull[buf]));
                __syncwarp();
            }
        }
        if (!ok) raise_abort();
        if (lane == 0) {
            tc_commit(smem_u32(&aux.drain));
            mbar_drain(smem_u32(&aux.drain), 0, drain_deadline());
        }
        __syncwarp();
    } else {
        // ================= promotion + epilogue (warps 2..5 -> TMEM lane quarters 2,3,0,1)
        const int q = warp & 3;
        int g = 0;
        bool ok = true;
        if (p.stall && !warp_wait(smem_u32(&aux.never), 0, abort_flag, wait_ns)) ok = false;
        for (int u = blockIdx.x; u < units && ok && !*abort_flag; u += gridDim.x) {
            const int tile = u / per_tile, rem = u % per_tile, eblk = rem / p.ksplit, split = rem % p.ksplit;
            int c0, c1;
            chunk_range(u, c0, c1);
            const int nch = c1 - c0;
            const int t = tile * BM + 32 * q + lane;
            const int e0 = eblk * NP;
            const int ne = p.E - e0 < NP ? p.E - e0 : NP;  // columns of this block that exist
            float* out = p.partial + ((int64_t)split * p.T + t) * p.E + e0;
            const float rs = t < p.T ? p.rstd[t] : 0.f;
            if (nch <= 0) {  // a trailing split with no columns: its slice of the partial sums is zero
                if (t < p.T)
                    for (int i = 0; i < ne; ++i) out[i] = 0.f;
                continue;
            }
            const uint32_t lane_off = (uint32_t)(32 * q) << 16;
            for (int ci = 0; ci < nch; ++ci, ++g) {
                const int buf = g & 1;
                if (!warp_wait(smem_u32(&aux.cfull[buf]), (uint32_t)(g >> 1) & 1u, abort_flag, wait_ns)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t tchunk = tmem_base + (uint32_t)((1 + buf) * NP) + lane_off;
                const uint32_t trun = tmem_base + lane_off;
                const bool last = ci == nch - 1;
#pragma unroll 1
                for (int c = 0; c < NP; c += 32) {
                    uint32_t r[32], run[32];
                    tmem_ld32(tchunk + c, r);
                    if (ci > 0) {
                        tmem_ld32(trun + c, run);
                        tmem_wait_ld(run);
                    }
                    tmem_wait_ld(r);
                    if (ci > 0) {
#pragma unroll
                        for (int i = 0; i < 32; ++i)
                            r[i] = __float_as_uint(__uint_as_float(run[i]) + __uint_as_float(r[i]));
                    }
                    if (!last) {
                        tmem_st32(trun + c, r);
                    } else if (t < p.T) {
                        if ((p.E & 3) == 0 && c + 32 <= ne) {
#pragma unroll
                            for (int i = 0; i < 32; i += 4)
                                *reinterpret_cast<float4*>(out + c + i) =
                                    make_float4(rs * __uint_as_float(r[i]), rs * __uint_as_float(r[i + 1]),
                                                rs * __uint_as_float(r[i + 2]), rs * __uint_as_float(r[i + 3]));
                        } else {
#pragma unroll
                            for (int i = 0; i < 32; ++i)
                                if (c + i < ne) out[c + i] = rs * __uint_as_float(r[i]);
                        }
                    }
                }
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_u32(&aux.cempty[buf]));
            }
        }
        if (!ok) raise_abort();
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem_base, C::TMEM_COLS);
}

// bf16 matrix [rows][inner], box = 64 x box_rows, 128-byte swizzle
static bool encode_bf16(CUtensorMap* tm, const void* base, uint64_t inner, uint64_t rows, uint32_t box_rows) {
    EncodeTiledFn fn = encode_tiled_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {inner, rows};
    cuuint64_t strides[1] = {inner * 2};
    cuuint32_t box[2] = {(cuuint32_t)BK, box_rows};
    cuuint32_t estr[2] = {1, 1};
    return fn(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int NP>
static cudaError_t run(const Ctx& c, const CUtensorMap& tx, const CUtensorMap& tw, XArgs a, int units) {
    using C = XCfg<NP>;
    set_wait_args(a);
    auto kern = router_x3_kernel<NP>;
    static bool attr_done[64] = {};
    if (c.device < 0 || c.device >= 64) return cudaErrorInvalidDevice;
    if (!attr_done[c.device]) {
        cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
        if (err != cudaSuccess) return err;
        attr_done[c.device] = true;
    }
    const int grid = units < c.num_sms ? units : c.num_sms;
    return launch(kern, dim3(grid), dim3(kThreads), (size_t)C::SMEM, c, tx, tw, a);
}

}  // namespace rx3

cudaError_t launch_router_logits_x3(const Ctx& c, const RouterPlan& p, const void* x, const float* rstd,
                                    const float* gamma, const float* W_r, int T, int d, int E, int np,
                                    float* partial, void* ws, int32_t* status) {
    if (T == 0) return cudaSuccess;
    if (d % 128 != 0) return cudaErrorInvalidValue;
    uint16_t* parts = static_cast<uint16_t*>(ws);
    const int64_t n = (int64_t)E * d;
    int64_t blocks = (n + 255) / 256;
    if (blocks > (int64_t)c.num_sms * 8) blocks = (int64_t)c.num_sms * 8;
    cudaError_t err = launch(rx3::router_w3split_kernel, dim3((unsigned)blocks), dim3(256), 0, c, W_r, gamma, d, n, parts);
    if (err != cudaSuccess) return err;
    const int neb = (E + np - 1) / np;
    CUtensorMap tm_x, tm_w;
    if (!rx3::encode_bf16(&tm_x, x, (uint64_t)d, (uint64_t)T, (uint32_t)rx3::BM) ||
        !rx3::encode_bf16(&tm_w, parts, (uint64_t)d, (uint64_t)3 * E, (uint32_t)np))
        return cudaErrorInvalidValue;
    const int nchunks = d / 128;
    const int cps = (nchunks + p.splitk - 1) / p.splitk;
    rx3::XArgs args{rstd, partial, T, d, E, neb, p.splitk, cps, status};
    const int units = ((T + rx3::BM - 1) / rx3::BM) * neb * p.splitk;
    switch (np) {
        case 32: return rx3::run<32>(c, tm_x, tm_w, args, units);
        case 64: return rx3::run<64>(c, tm_x, tm_w, args, units);
        default: return rx3::run<128>(c, tm_x, tm_w, args, units);
    }
}

}  // namespace moe
