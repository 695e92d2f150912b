// Router logits z = v W_r^T on the tensor cores at fp32 accuracy.
//
// "推理计算流梳理" (huanyp.cn), §专家并行 / MoE Router 过程: z = x W_r^T feeds
// s = sigmoid(z), I = Top8(s + b).  The logits are a dense contraction
// (T x d by d x E), so they run on tcgen05 — but the selection needs fp32
// logits, and tf32 keeps only 11 significant bits.  Each fp32 operand is
// therefore split into two tf32 terms, a = a_hi + a_lo (a_hi = tf32(a),
// a_lo = tf32(a - a_hi)), and
//     a·b ≈ a_hi·b_hi + a_hi·b_lo + a_lo·b_hi
// accumulated in fp32 in tensor memory (the dropped a_lo·b_lo is ~2^-22 of
// a·b), the accuracy of an fp32 dot product.
//
// The tensor core adds each MMA's result into its fp32 accumulator with a
// rounding biased toward zero, so a long accumulation drifts (measured on
// B200: -4.8e-5 relative after K = 4096 of positive terms).  The kernel
// therefore accumulates at most kChunkSlabs x 32 = 128 columns of K per TMEM
// accumulator and adds the chunks in fp32 round-to-nearest on the CUDA cores
// (a running sum kept in tensor memory), like an fp32 dot product.
//
// router_wsplit_kernel  W_r -> (W_hi, W_lo), elementwise, into the workspace.
// router_tc_kernel      persistent over (128-token tile, block of <= 128
//                       experts, K slice) units:
//   warp 0       TMA loads of the W_hi / W_lo slices (fp32, 128-byte swizzle)
//   warp 1       TMEM owner; lane 0 issues 3 tf32 MMAs per K=8 step into one
//                of two chunk accumulators
//   warps 2..9   build A: v = x * rstd * gamma (or v itself), split into
//                hi / lo and stored into shared memory in the swizzled
//                K-major layout the MMA reads (fence.proxy.async before
//                arriving on the stage barrier)
//   warps 10..13 add each finished chunk to the running sum in TMEM; after
//                the last chunk of a unit, write fp32 partial logits
//                [split][T][E]
// The K-split partials are summed in split order by router_topk_kernel.
#include <math.h>

#include "common.cuh"
#include "kernels.h"
#include "tc_ptx.cuh"

namespace moe {
namespace rtc {
using namespace tc;

constexpr int BM = 128;  // tokens per tile (MMA M)
constexpr int BKF = 32;  // fp32 K elements per stage: one 128-byte swizzled row
constexpr int kChunkSlabs = 4;  // stages accumulated in TMEM before promotion to the fp32 running sum
constexpr int kMaxBlockExperts = 128;
constexpr int kProd = 8;  // A-producer warps
constexpr int kThreads = 32 * (2 + kProd + 4);  // 448
constexpr int kSmemLimit = 232448;

template <int NP>
struct RCfg {
    static_assert(NP % 16 == 0 && NP >= 32 && NP <= kMaxBlockExperts, "padded expert block");
    static constexpr int A_BYTES = BM * 128;
    static constexpr int B_BYTES = NP * 128;
    static constexpr int STAGE_BYTES = 2 * A_BYTES + 2 * B_BYTES;
    static constexpr int AUX_BYTES = 1024;
    static constexpr int ST = (kSmemLimit - 1024 - AUX_BYTES) / STAGE_BYTES;
    static constexpr int STAGES = ST > 4 ? 4 : ST;
    static_assert(STAGES >= 2, "pipeline depth");
    // columns [0, NP): running sum; [NP, 2NP) and [2NP, 3NP): chunk accumulators
    static constexpr int TMEM_COLS = (3 * NP <= 128) ? 128 : (3 * NP <= 256) ? 256 : 512;
    static constexpr int SMEM = 1024 + STAGES * STAGE_BYTES + AUX_BYTES;
};

struct RAux {
    uint64_t full[4];
    uint64_t empty[4];
    uint64_t cfull[2];   // chunk accumulator ready
    uint64_t cempty[2];  // chunk accumulator drained
    uint64_t drain;
    uint64_t never;      // completed by nothing: the injected stall waits on it
    uint32_t tmem_slot;
    int abort_flag;
};

struct RArgs {
    const void* a;       // x (NORM) or v, [T][d]
    const float* rstd;   // [T] (NORM only)
    const float* gamma;  // [d] (NORM only)
    float* partial;      // [ksplit][T][E]
    int T, d, E;
    int neb;             // expert blocks of NP
    int ksplit;
    int slabs_per_split;
    int32_t* status;
    // bounded waits: the limit of one wait, and (failure-path tests only) an extra wait on a barrier
    // that nothing completes, made by the epilogue warps before their first tile
    uint64_t wait_ns = kTimeoutNs;
    int stall = 0;
};

__global__ void __launch_bounds__(256) router_wsplit_kernel(const float* __restrict__ W, int64_t n,
                                                            float* __restrict__ hi, float* __restrict__ lo) {
    pdl_wait();
    pdl_trigger();
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
        const float w = W[i];
        const float h = to_tf32(w);
        hi[i] = h;
        lo[i] = to_tf32(w - h);
    }
}

template <int NP, bool NORM, int ADT>
__global__ void __launch_bounds__(kThreads, 1)
    router_tc_kernel(const __grid_constant__ CUtensorMap tm_whi, const __grid_constant__ CUtensorMap tm_wlo,
                     const RArgs p) {
    using C = RCfg<NP>;
    constexpr int STAGES = C::STAGES;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    RAux& aux = *reinterpret_cast<RAux*>(smem + STAGES * C::STAGE_BYTES);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    volatile int* abort_flag = &aux.abort_flag;
    const uint64_t wait_ns = p.wait_ns;

    if (warp == 0 && lane == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(smem_u32(&aux.full[s]), 1 + kProd);
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
        tma_prefetch(&tm_whi);
        tma_prefetch(&tm_wlo);
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
    const int kslabs = (p.d + BKF - 1) / BKF;
    auto raise_abort = [&]() {
        if (lane == 0) {
            *abort_flag = 1;
            set_status(p.status, DEV_TIMEOUT);
        }
    };

    if (warp == 0) {
        // ================= TMA: W_hi / W_lo slices
        int stage = 0;
        uint32_t phase = 0, used = 0, last_parity = 0;
        for (int u = blockIdx.x; u < units && !*abort_flag; u += gridDim.x) {
            const int rem = u % per_tile, eblk = rem / p.ksplit, split = rem % p.ksplit;
            const int kb0 = split * p.slabs_per_split, kb1 = min(kslabs, kb0 + p.slabs_per_split);
            bool ok = true;
            for (int kb = kb0; kb < kb1; ++kb) {
                if (!warp_wait(smem_u32(&aux.empty[stage]), phase ^ 1u, abort_flag, wait_ns)) {
                    ok = false;
                    break;
                }
                if (lane == 0) {
                    const uint32_t st = smem_u32(smem + stage * C::STAGE_BYTES);
                    const uint32_t full = smem_u32(&aux.full[stage]);
                    mbar_expect_tx(full, 2 * C::B_BYTES);
                    tma_load_2d(st + 2 * C::A_BYTES, &tm_whi, kb * BKF, eblk * NP, full);
                    tma_load_2d(st + 2 * C::A_BYTES + C::B_BYTES, &tm_wlo, kb * BKF, eblk * NP, full);
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
        // ================= MMA issuer: one chunk accumulator per kChunkSlabs stages, alternating
        int stage = 0;
        uint32_t phase = 0;
        int g = 0;  // chunks issued so far
        const uint32_t idesc = idesc_tf32(BM, NP);
        bool ok = true;
        for (int u = blockIdx.x; u < units && ok && !*abort_flag; u += gridDim.x) {
            const int split = (u % per_tile) % p.ksplit;
            const int kb0 = split * p.slabs_per_split, kb1 = min(kslabs, kb0 + p.slabs_per_split);
            for (int c0 = kb0; c0 < kb1 && ok; c0 += kChunkSlabs, ++g) {
                const int buf = g & 1;
                if (!warp_wait(smem_u32(&aux.cempty[buf]), ((uint32_t)(g >> 1) & 1u) ^ 1u, abort_flag, wait_ns)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)((1 + buf) * NP);
                const int c1 = min(kb1, c0 + kChunkSlabs);
                for (int kb = c0; kb < c1; ++kb) {
                    if (!warp_wait(smem_u32(&aux.full[stage]), phase, abort_flag, wait_ns)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    if (lane == 0) {
                        const uint32_t ahi = smem_u32(smem + stage * C::STAGE_BYTES);
                        const uint32_t alo = ahi + C::A_BYTES, bhi = ahi + 2 * C::A_BYTES, blo = bhi + C::B_BYTES;
#pragma unroll
                        for (int kk = 0; kk < BKF / 8; ++kk) {
                            const uint32_t o = kk * 32;
                            const uint32_t first = (kb == c0 && kk == 0) ? 0u : 1u;
                            tc_mma_tf32(d_tmem, sdesc_sw128(ahi + o), sdesc_sw128(bhi + o), idesc, first);
                            tc_mma_tf32(d_tmem, sdesc_sw128(ahi + o), sdesc_sw128(blo + o), idesc, 1u);
                            tc_mma_tf32(d_tmem, sdesc_sw128(alo + o), sdesc_sw128(bhi + o), idesc, 1u);
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
    } else if (warp < 2 + kProd) {
        // ================= A producers: 256 threads, thread -> (row, 16-column half) of the 128 x 32 slice
        const int pt = threadIdx.x - 64;
        const int row = pt >> 1, half = pt & 1;
        int stage = 0;
        uint32_t phase = 0;
        // no abort check in this loop: a stage whose slot was freed is always filled (so the TMA producer's
        // drain of that stage completes); after an abort the next wait for a slot that is not free fails
        for (int u = blockIdx.x; u < units; u += gridDim.x) {
            const int tile = u / per_tile, split = (u % per_tile) % p.ksplit;
            const int kb0 = split * p.slabs_per_split, kb1 = min(kslabs, kb0 + p.slabs_per_split);
            const int t = tile * BM + row;
            const bool row_ok = t < p.T;
            float rs = 1.f;
            if (NORM && row_ok) rs = p.rstd[t];
            bool ok = true;
            for (int kb = kb0; kb < kb1; ++kb) {
                // load before waiting for the slot: the global loads overlap the wait
                const int k0 = kb * BKF + half * 16;
                float v[16];
                if (row_ok && k0 < p.d) {  // d % 8 == 0: a 16-column group is all in, all out, or its first 8 in
                    load8<ADT>(p.a, (int64_t)t * p.d + k0, *reinterpret_cast<float(*)[8]>(&v[0]));
                    if (k0 + 8 < p.d)
                        load8<ADT>(p.a, (int64_t)t * p.d + k0 + 8, *reinterpret_cast<float(*)[8]>(&v[8]));
                    else
#pragma unroll
                        for (int i = 8; i < 16; ++i) v[i] = 0.f;
                    if (NORM) {
                        float g[16];
                        load8<DT_F32>(p.gamma, k0, *reinterpret_cast<float(*)[8]>(&g[0]));
                        if (k0 + 8 < p.d)
                            load8<DT_F32>(p.gamma, k0 + 8, *reinterpret_cast<float(*)[8]>(&g[8]));
                        else
#pragma unroll
                            for (int i = 8; i < 16; ++i) g[i] = 0.f;
#pragma unroll
                        for (int i = 0; i < 16; ++i) v[i] = (v[i] * rs) * g[i];
                    }
                } else {
#pragma unroll
                    for (int i = 0; i < 16; ++i) v[i] = 0.f;
                }
                if (!warp_wait(smem_u32(&aux.empty[stage]), phase ^ 1u, abort_flag, wait_ns)) {
                    ok = false;
                    break;
                }
                uint8_t* ahi = smem + stage * C::STAGE_BYTES;
                uint8_t* alo = ahi + C::A_BYTES;
                const int rbase = (row >> 3) * 1024 + (row & 7) * 128;
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const int chunk = half * 4 + c;
                    const int off = rbase + ((chunk ^ (row & 7)) << 4);
                    float h[4], l[4];
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        h[i] = to_tf32(v[4 * c + i]);
                        l[i] = to_tf32(v[4 * c + i] - h[i]);
                    }
                    *reinterpret_cast<float4*>(ahi + off) = make_float4(h[0], h[1], h[2], h[3]);
                    *reinterpret_cast<float4*>(alo + off) = make_float4(l[0], l[1], l[2], l[3]);
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_u32(&aux.full[stage]));
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
    } else {
        // ================= promotion + epilogue (warps 10..13 -> TMEM lane quarters 2,3,0,1)
        const int q = warp & 3;
        int g = 0;
        bool ok = true;
        if (p.stall && !warp_wait(smem_u32(&aux.never), 0, abort_flag, wait_ns)) ok = false;
        for (int u = blockIdx.x; u < units && ok && !*abort_flag; u += gridDim.x) {
            const int tile = u / per_tile, rem = u % per_tile, eblk = rem / p.ksplit, split = rem % p.ksplit;
            const int kb0 = split * p.slabs_per_split, kb1 = min(kslabs, kb0 + p.slabs_per_split);
            const int nch = (kb1 - kb0 + kChunkSlabs - 1) / kChunkSlabs;
            const int t = tile * BM + 32 * q + lane;
            const int e0 = eblk * NP;
            float* out = p.partial + ((int64_t)split * p.T + t) * p.E + e0;
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
                        const int ne = p.E - e0;  // columns of this block that exist
                        if ((p.E & 3) == 0 && c + 32 <= ne) {
#pragma unroll
                            for (int i = 0; i < 32; i += 4)
                                *reinterpret_cast<float4*>(out + c + i) = make_float4(
                                    __uint_as_float(r[i]), __uint_as_float(r[i + 1]), __uint_as_float(r[i + 2]),
                                    __uint_as_float(r[i + 3]));
                        } else {
#pragma unroll
                            for (int i = 0; i < 32; ++i)
                                if (c + i < ne) out[c + i] = __uint_as_float(r[i]);
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

// fp32 matrix [rows][inner], box = 32 x box_rows, 128-byte swizzle
static bool encode_f32(CUtensorMap* tm, const void* base, uint64_t inner, uint64_t rows, uint32_t box_rows) {
    EncodeTiledFn fn = encode_tiled_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {inner, rows};
    cuuint64_t strides[1] = {inner * 4};
    cuuint32_t box[2] = {(cuuint32_t)BKF, box_rows};
    cuuint32_t estr[2] = {1, 1};
    return fn(tm, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int NP, bool NORM, int ADT>
static cudaError_t run(const Ctx& c, const CUtensorMap& whi, const CUtensorMap& wlo, RArgs a, int units) {
    using C = RCfg<NP>;
    set_wait_args(a);
    auto kern = router_tc_kernel<NP, NORM, ADT>;
    static bool attr_done[64] = {};
    if (c.device < 0 || c.device >= 64) return cudaErrorInvalidDevice;
    if (!attr_done[c.device]) {
        cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
        if (err != cudaSuccess) return err;
        attr_done[c.device] = true;
    }
    const int grid = units < c.num_sms ? units : c.num_sms;
    return launch(kern, dim3(grid), dim3(kThreads), (size_t)C::SMEM, c, whi, wlo, a);
}

template <bool NORM, int ADT>
static cudaError_t run_np(int np, const Ctx& c, const CUtensorMap& whi, const CUtensorMap& wlo, const RArgs& a,
                          int units) {
    switch (np) {
        case 32: return run<32, NORM, ADT>(c, whi, wlo, a, units);
        case 64: return run<64, NORM, ADT>(c, whi, wlo, a, units);
        default: return run<128, NORM, ADT>(c, whi, wlo, a, units);
    }
}

}  // namespace rtc

// experts per block: the power of two >= E in [32, 128]; more experts take several blocks
static int block_experts(int E) {
    int np = 32;
    while (np < E && np < rtc::kMaxBlockExperts) np <<= 1;
    return np;
}

RouterPlan plan_router(int T, int d, int E, int num_sms) {
    RouterPlan p;
    const int tiles = ((T + rtc::BM - 1) / rtc::BM) * ((E + block_experts(E) - 1) / block_experts(E));
    const int kslabs = (d + rtc::BKF - 1) / rtc::BKF;
    int split = tiles > 0 ? num_sms / tiles : 1;
    const int max_split = kslabs / 4 > 1 ? kslabs / 4 : 1;  // at least 4 slabs (128 columns) per split
    if (split > max_split) split = max_split;
    if (split < 1) split = 1;
    const int per = (kslabs + split - 1) / split;
    p.splitk = (kslabs + per - 1) / per;
    p.kchunk = per * rtc::BKF;
    p.partial_bytes = (size_t)p.splitk * (size_t)T * (size_t)E * sizeof(float);
    p.wsplit_bytes = 2 * (size_t)E * (size_t)d * sizeof(float);
    return p;
}

cudaError_t launch_router_logits(const Ctx& c, const RouterPlan& p, const void* a, int a_dt, const float* rstd,
                                 const float* gamma, const float* W_r, int T, int d, int E, float* partial,
                                 float* wsplit, int32_t* status) {
    if (T == 0) return cudaSuccess;
    // bf16 rows with the normalisation folded in: three exact bf16 MMAs per K step on x itself
    if (rstd != nullptr && a_dt == DT_BF16 && d % 128 == 0)
        return launch_router_logits_x3(c, p, a, rstd, gamma, W_r, T, d, E, block_experts(E), partial, wsplit, status);
    float* whi = wsplit;
    float* wlo = wsplit + (size_t)E * d;
    const int64_t n = (int64_t)E * d;
    int64_t blocks = (n + 255) / 256;
    if (blocks > (int64_t)c.num_sms * 8) blocks = (int64_t)c.num_sms * 8;
    cudaError_t err = launch(rtc::router_wsplit_kernel, dim3((unsigned)blocks), dim3(256), 0, c, W_r, n, whi, wlo);
    if (err != cudaSuccess) return err;
    const int np = block_experts(E);
    const int neb = (E + np - 1) / np;
    CUtensorMap tm_hi, tm_lo;
    if (!rtc::encode_f32(&tm_hi, whi, (uint64_t)d, (uint64_t)E, (uint32_t)np) ||
        !rtc::encode_f32(&tm_lo, wlo, (uint64_t)d, (uint64_t)E, (uint32_t)np))
        return cudaErrorInvalidValue;
    rtc::RArgs args{a, rstd, gamma, partial, T, d, E, neb, p.splitk, p.kchunk / rtc::BKF, status};
    const int units = ((T + rtc::BM - 1) / rtc::BM) * neb * p.splitk;
    const bool norm = rstd != nullptr;
    if (norm && a_dt == DT_BF16) return rtc::run_np<true, DT_BF16>(np, c, tm_hi, tm_lo, args, units);
    if (norm) return rtc::run_np<true, DT_F32>(np, c, tm_hi, tm_lo, args, units);
    if (a_dt == DT_BF16) return rtc::run_np<false, DT_BF16>(np, c, tm_hi, tm_lo, args, units);
    return rtc::run_np<false, DT_F32>(np, c, tm_hi, tm_lo, args, units);
}

}  // namespace moe
