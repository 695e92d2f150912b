// Step 4, gate/up, for experts of ~256-767 rows: grouped GEMM tiles of two 128-row blocks of one expert
// sharing each staged weight slice.
//
// Same mathematics as expert_tc.cu ("推理计算流梳理", §实际 MLP 计算策略 and §EP 路径):
//   h = SiLU(xp W_gate^T) ⊙ (xp W_up^T)
// At the burst clock the one-CTA 128 x 256 tile is paced by delivering its operands into shared memory,
// two thirds of them weight bytes.  Here a tile is (expert e, row pair rp = rows [256 rp, 256 rp + 256),
// column block cb): two MMAs per K step, one per 128-row half, read the same staged weight slice into two
// accumulators, which halves the weight bytes per MMA.  Row padding stays 128 rows: a pair whose second half
// has no rows skips its loads and its MMAs.
//
// The two accumulators fill all 512 TMEM columns, so they are single-buffered.  Eight epilogue warps (one
// per TMEM lane quarter and half) read them one 32-column chunk ahead of their math and stores and release
// them as soon as their last chunk has landed; full 32-row pieces leave by TMA.
//
// Schedule: with a tile counter (moe_forward passes one, zeroed per call) the producer takes the next
// tile from it, so CTAs that drew light tiles (half-filled pairs) take more; without one, CTA i runs tiles
// i, i + gridDim.x, ...  The producer writes tile j's id to ring1[j % 8] before arming the tile's first
// stage (the barrier's arrive publishes it); the MMA warp reads it behind that stage's barrier and passes
// it on in ring2[j % 4] behind tidb[j % 4] to the epilogue.  An id of -1 (no more tiles) travels the same
// way on one stage armed with no data.
//
// Warp roles (1 CTA per SM, 320 threads):
//   warp 0      TMA producer: a 3-stage ring of 64-wide K slices (token rows of both halves, the weight
//               slice), 128-byte swizzle
//   warp 1      owns the TMEM allocation; lane 0 issues the MMAs and commits
//   warps 2..5  epilogue of the first half (TMEM lane quarters 2,3,0,1)
//   warps 6..9  epilogue of the second half
// Every wait is bounded; a wait that gives up raises DEV_TIMEOUT and all roles unwind as in expert_tc.cu
// (drains bounded by time only, TMEM freed last).
#include <cuda.h>
#include <math.h>

#include "common.cuh"
#include "kernels.h"
#include "tc_ptx.cuh"

namespace moe {
namespace tcd {
using namespace tc;

constexpr int BK = 64;
constexpr int RH = 128;  // token rows per half (MMA M)
constexpr int RP = 256;  // token rows per tile
constexpr int kThreads = 320;
constexpr int kSmemLimit = 232448;

template <bool SWIGLU>
struct DCfg {
    static constexpr int COLS = SWIGLU ? 128 : 256;  // output columns per tile (gate 128 | up 128, or 256)
    static constexpr int A_BYTES = RH * 128;
    static constexpr int B_BYTES = 256 * 128;
    static constexpr int STAGE_BYTES = 2 * A_BYTES + B_BYTES;
    static constexpr int AUX_BYTES = 4096;
    // per epilogue warp a 2 KB buffer: 32 rows x 32 bf16 columns, 64-byte swizzle, stored by TMA
    static constexpr int EPI_BYTES = 8 * 2048;
    static constexpr int ST = (kSmemLimit - 1024 - AUX_BYTES - EPI_BYTES) / STAGE_BYTES;
    static constexpr int STAGES = ST > 4 ? 4 : ST;
    static_assert(STAGES >= 3, "pipeline depth");
    static constexpr int SMEM = 1024 + STAGES * STAGE_BYTES + AUX_BYTES + EPI_BYTES;
};

struct DArgs {
    const int32_t* counts;
    const int32_t* offsets;
    int E;
    int K;      // reduction length (d for gate/up, d_ff for down)
    int n_out;  // weight rows per expert = output columns
    uint16_t* out;
    int64_t ldo;
    int32_t* status;
    int S;  // rows of the expert-contiguous buffers; a segment that does not fit is clamped and flagged
    // bounded waits: the limit of one wait, and (failure-path tests only) an extra wait on a barrier
    // that nothing completes, made by the epilogue warps before their first tile
    uint64_t wait_ns = kTimeoutNs;
    int stall = 0;
    // GEMM-core test form of gate/up: g in columns [0, n_out), u in [n_out, 2 n_out), no SwiGLU product
    int raw = 0;
    // dynamic schedule: tiles are taken in order from this counter (zero before the launch); null: CTA i
    // runs tiles i, i + gridDim.x, ...
    int32_t* tile_ctr = nullptr;
};

struct DAux {
    uint64_t full[4];
    uint64_t empty[4];
    uint64_t tfull;
    uint64_t tempty;
    uint64_t drain;
    uint64_t never;  // completed by nothing: the injected stall waits on it
    uint64_t tidb[4];  // the MMA warp has published ring2[j % 4] for the epilogue
    uint32_t tmem_slot;
    int abort_flag;
    int ring1[8];  // tile id of the producer's j-th tile (-1: no more), read by the MMA warp behind full[]
    int ring2[4];  // the same, passed on by the MMA warp to the epilogue behind tidb[]
    int tstart[kMaxExperts + 1];
    int cnt[kMaxExperts];
    int off[kMaxExperts];
};

__device__ __forceinline__ void decode_tile_d(const DAux& a, int E, int tile, int& e, int& rp, int& cb) {
    int lo = 0, hi = E - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (a.tstart[mid] <= tile) lo = mid; else hi = mid - 1;
    }
    e = lo;
    const int local = tile - a.tstart[e];
    const int nrp = (a.cnt[e] + RP - 1) / RP;
    cb = local / nrp;
    rp = local - cb * nrp;
}

// SiLU(g) * u with the hardware exp2 and reciprocal, as in expert_tc.cu
__device__ __forceinline__ float silu_mul_d(float g, float u) { return __fdividef(g, 1.0f + __expf(-g)) * u; }

template <bool SWIGLU>
__global__ void __launch_bounds__(kThreads, 1)
    grouped_gemm_dual_kernel(const __grid_constant__ CUtensorMap tm_act, const __grid_constant__ CUtensorMap tm_w1,
                             const __grid_constant__ CUtensorMap tm_w2, const __grid_constant__ CUtensorMap tm_out,
                             const DArgs p) {
    using C = DCfg<SWIGLU>;
    constexpr int STAGES = C::STAGES;
    constexpr int COLS = C::COLS;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    DAux& aux = *reinterpret_cast<DAux*>(smem + STAGES * C::STAGE_BYTES);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    volatile int* abort_flag = &aux.abort_flag;
    const uint64_t wait_ns = p.wait_ns;

    if (warp == 0 && lane == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(smem_u32(&aux.full[s]), 1);
            mbar_init(smem_u32(&aux.empty[s]), 1);
        }
        mbar_init(smem_u32(&aux.tfull), 1);
        mbar_init(smem_u32(&aux.tempty), 8);
        for (int s = 0; s < 4; ++s) mbar_init(smem_u32(&aux.tidb[s]), 1);
        mbar_init(smem_u32(&aux.drain), 1);
        mbar_init(smem_u32(&aux.never), 1);
        aux.abort_flag = 0;
        fence_mbar_init();
        tma_prefetch(&tm_act);
        tma_prefetch(&tm_w1);
        if (SWIGLU) tma_prefetch(&tm_w2);
        tma_prefetch(&tm_out);
    }
    if (warp == 1) tmem_alloc(smem_u32(&aux.tmem_slot), 512);

    pdl_wait();
    const int E = p.E;
    for (int e = threadIdx.x; e < E; e += (int)blockDim.x) {
        int o, n;
        if (!clamp_segment(p.offsets[e], p.counts[e], p.S, o, n)) set_status(p.status, DEV_BAD_COUNT);
        aux.cnt[e] = n;
        aux.off[e] = o;
    }
    __syncthreads();
    if (warp == 0) {
        // tile prefix over experts: lane owns experts 8*lane .. 8*lane+7
        const int ncb = p.n_out / COLS;
        int loc[8], sum = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int e = lane * 8 + i;
            loc[i] = (e < E) ? ((aux.cnt[e] + RP - 1) / RP) * ncb : 0;
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
    const int nk = p.K / BK;
    auto raise_abort = [&]() {
        if (lane == 0) {
            *abort_flag = 1;
            set_status(p.status, DEV_TIMEOUT);
        }
    };

    if (warp == 0) {
        // ================= TMA producer: takes tile j (from the counter, or CTA-strided), writes its id to
        // ring1[j % 8] before arming the tile's first stage; no more tiles: one stage armed with id -1 and
        // no data
        int stage = 0;
        uint32_t phase = 0, used = 0, last_parity = 0;
        bool ok = true;
        for (int j = 0; ok; ++j) {
            int tile = -1;
            if (lane == 0) {
                const int t = p.tile_ctr ? atomicAdd(p.tile_ctr, 1) : (int)blockIdx.x + j * (int)gridDim.x;
                tile = (t < total && !*abort_flag) ? t : -1;
            }
            tile = __shfl_sync(0xffffffffu, tile, 0);
            int row0 = 0, w_row = 0;
            bool two = false;
            if (tile >= 0) {
                int e, rp, cb;
                decode_tile_d(aux, E, tile, e, rp, cb);
                row0 = aux.off[e] + rp * RP;
                two = aux.cnt[e] - rp * RP > RH;  // the second half has rows
                w_row = e * p.n_out + cb * COLS;
            }
            const int steps = tile >= 0 ? nk : 1;
            for (int kb = 0; kb < steps; ++kb) {
                if (!warp_wait(smem_u32(&aux.empty[stage]), phase ^ 1u, abort_flag, wait_ns)) {
                    ok = false;
                    break;
                }
                if (lane == 0) {
                    const uint32_t full = smem_u32(&aux.full[stage]);
                    if (kb == 0) aux.ring1[j & 7] = tile;  // published by the arrive below (release)
                    if (tile < 0) {
                        mbar_arrive(full);
                    } else {
                        const uint32_t a0 = smem_u32(smem + stage * C::STAGE_BYTES);
                        const uint32_t b0 = a0 + 2 * C::A_BYTES;
                        mbar_expect_tx(full, (two ? 2 : 1) * C::A_BYTES + C::B_BYTES);
                        tma_load_2d(a0, &tm_act, kb * BK, row0, full);
                        if (two) tma_load_2d(a0 + C::A_BYTES, &tm_act, kb * BK, row0 + RH, full);
                        tma_load_2d(b0, &tm_w1, kb * BK, w_row, full);
                        if (SWIGLU) tma_load_2d(b0 + 128 * 128, &tm_w2, kb * BK, w_row, full);
                    }
                }
                used |= 1u << stage;
                last_parity = (last_parity & ~(1u << stage)) | (phase << stage);
                if (++stage == STAGES) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
            if (tile < 0) break;
        }
        if (!ok) raise_abort();
        {
            const uint64_t dl = drain_deadline();
            for (int s = 0; s < STAGES; ++s)
                if (used & (1u << s)) mbar_drain(smem_u32(&aux.full[s]), (last_parity >> s) & 1u, dl);
        }
    } else if (warp == 1) {
        // ================= MMA issuer: per K step the weight slice against both halves
        int stage = 0;
        uint32_t phase = 0;
        const uint32_t idesc = idesc_bf16(128, 256);
        bool ok = true;
        for (int j = 0;; ++j) {
            // the single accumulator pair is free once the epilogue has read the previous tile
            if (!warp_wait(smem_u32(&aux.tempty), ((uint32_t)j & 1u) ^ 1u, abort_flag, wait_ns) ||
                !warp_wait(smem_u32(&aux.full[stage]), phase, abort_flag, wait_ns)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const int tile = *reinterpret_cast<volatile int*>(&aux.ring1[j & 7]);
            if (lane == 0) {
                aux.ring2[j & 3] = tile;
                mbar_arrive(smem_u32(&aux.tidb[j & 3]));  // releases ring2[j % 4] to the epilogue
            }
            __syncwarp();
            if (tile < 0) break;  // the sentinel stage carries no data and is not released
            int e, rp, cb;
            decode_tile_d(aux, E, tile, e, rp, cb);
            const bool two = aux.cnt[e] - rp * RP > RH;
            for (int kb = 0; kb < nk; ++kb) {
                if (kb > 0) {
                    if (!warp_wait(smem_u32(&aux.full[stage]), phase, abort_flag, wait_ns)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                }
                if (lane == 0) {
                    const uint32_t a0 = smem_u32(smem + stage * C::STAGE_BYTES);
                    const uint32_t b0 = a0 + 2 * C::A_BYTES;
#pragma unroll
                    for (int kk = 0; kk < BK / 16; ++kk) {
                        const uint32_t acc = (kb | kk) ? 1u : 0u;
                        tc_mma(tmem_base, sdesc_sw128(a0 + kk * 32), sdesc_sw128(b0 + kk * 32), idesc, acc);
                        if (two)
                            tc_mma(tmem_base + 256, sdesc_sw128(a0 + C::A_BYTES + kk * 32), sdesc_sw128(b0 + kk * 32),
                                   idesc, acc);
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
            if (lane == 0) tc_commit(smem_u32(&aux.tfull));
            __syncwarp();
        }
        if (!ok) raise_abort();
        if (lane == 0) {
            tc_commit(smem_u32(&aux.drain));
            mbar_drain(smem_u32(&aux.drain), 0, drain_deadline());
        }
        __syncwarp();
    } else {
        // ================= epilogue: warps 2..5 the first half, 6..9 the second (TMEM lane quarters 2,3,0,1).
        // TMEM is read one 32-column chunk ahead of the math and stores; the accumulator pair is released
        // as soon as the warp's last chunk has been read.
        const int q = warp & 3, half = warp >= 6 ? 1 : 0;
        const uint32_t stg = smem_u32(smem) + STAGES * C::STAGE_BYTES + C::AUX_BYTES + 2048 * (warp - 2);
        bool ok = true;
        if (p.stall && !warp_wait(smem_u32(&aux.never), 0, abort_flag, wait_ns)) ok = false;
        for (int j = 0; ok; ++j) {
            if (!warp_wait(smem_u32(&aux.tidb[j & 3]), ((uint32_t)j >> 2) & 1u, abort_flag, wait_ns)) {
                ok = false;
                break;
            }
            const int tile = *reinterpret_cast<volatile int*>(&aux.ring2[j & 3]);
            if (tile < 0) break;
            if (!warp_wait(smem_u32(&aux.tfull), (uint32_t)j & 1u, abort_flag, wait_ns)) {
                ok = false;
                break;
            }
            tc_fence_after();
            int e, rp, cb;
            decode_tile_d(aux, E, tile, e, rp, cb);
            const int rows = min(RH, aux.cnt[e] - rp * RP - RH * half);  // this half's valid rows (may be <= 0)
            const int m = 32 * q + lane;
            const bool valid = m < rows;
            const int grow = aux.off[e] + rp * RP + RH * half + 32 * q;  // first output row of this warp
            uint16_t* orow = p.out + ((int64_t)grow + lane) * p.ldo + (int64_t)cb * COLS;
            const uint32_t tb = tmem_base + (uint32_t)(256 * half) + ((uint32_t)(32 * q) << 16);
            // a warp whose 32 rows are all valid writes them by TMA from its staging buffer; one with fewer
            // stores its valid rows directly
            const bool tma_rows = !p.raw && rows - 32 * q >= 32;
            auto release = [&]() {
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_u32(&aux.tempty));
            };
            if (rows <= 32 * q) {  // warp-uniform: nothing of this half's quarter to read
                release();
                continue;
            }
            // store one 32-column chunk of packed bf16 (16 registers) at column c
            auto store_chunk = [&](const uint32_t (&pk)[16], int c) {
                if (tma_rows) {
                    if (lane == 0) bulk_wait_read();  // the previous store from this buffer has read it
                    __syncwarp();
                    // row `lane`, 16-byte chunk v at lane * 64 + ((v ^ ((lane / 2) % 4)) * 16): the output tensor
                    // map's 64-byte swizzle; eight consecutive lanes cover all 32 banks
#pragma unroll
                    for (int v = 0; v < 4; ++v)
                        st_shared16(stg + lane * 64 + ((v ^ ((lane >> 1) & 3)) << 4),
                                    make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]));
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) {
                        tma_store_2d(&tm_out, stg, cb * COLS + c, grow);
                        bulk_commit();
                    }
                } else if (valid) {
#pragma unroll
                    for (int v = 0; v < 4; ++v)
                        st16(orow + c + 8 * v, make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]));
                }
            };
            if constexpr (SWIGLU) {
                // 4 chunks of gate and up columns; the raw test form stores g and u apart
                auto emit = [&](const uint32_t (&g)[32], const uint32_t (&u)[32], int c) {
                    if (p.raw) {
                        if (valid) {
#pragma unroll
                            for (int v = 0; v < 4; ++v) {
                                uint32_t a4[4], b4[4];
#pragma unroll
                                for (int i = 0; i < 4; ++i) {
                                    a4[i] = pack_bf16x2(__uint_as_float(g[8 * v + 2 * i]),
                                                        __uint_as_float(g[8 * v + 2 * i + 1]));
                                    b4[i] = pack_bf16x2(__uint_as_float(u[8 * v + 2 * i]),
                                                        __uint_as_float(u[8 * v + 2 * i + 1]));
                                }
                                st16(orow + c + 8 * v, make_uint4(a4[0], a4[1], a4[2], a4[3]));
                                st16(orow + p.n_out + c + 8 * v, make_uint4(b4[0], b4[1], b4[2], b4[3]));
                            }
                        }
                        return;
                    }
                    uint32_t pk[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        pk[i] = pack_bf16x2(silu_mul_d(__uint_as_float(g[2 * i]), __uint_as_float(u[2 * i])),
                                            silu_mul_d(__uint_as_float(g[2 * i + 1]), __uint_as_float(u[2 * i + 1])));
                    store_chunk(pk, c);
                };
                uint32_t g0[32], u0[32], g1[32], u1[32];
                tmem_ld32(tb + 0, g0);
                tmem_ld32(tb + 128, u0);
                tmem_wait_ld(g0);
                tmem_wait_ld(u0);
                tmem_ld32(tb + 32, g1);
                tmem_ld32(tb + 160, u1);
                emit(g0, u0, 0);
                tmem_wait_ld(g1);
                tmem_wait_ld(u1);
                tmem_ld32(tb + 64, g0);
                tmem_ld32(tb + 192, u0);
                emit(g1, u1, 32);
                tmem_wait_ld(g0);
                tmem_wait_ld(u0);
                tmem_ld32(tb + 96, g1);
                tmem_ld32(tb + 224, u1);
                emit(g0, u0, 64);
                tmem_wait_ld(g1);
                tmem_wait_ld(u1);
                release();  // every TMEM read of this warp has landed
                emit(g1, u1, 96);
            } else {
                // 8 chunks of 32 output columns
                auto emit = [&](const uint32_t (&g)[32], int c) {
                    uint32_t pk[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        pk[i] = pack_bf16x2(__uint_as_float(g[2 * i]), __uint_as_float(g[2 * i + 1]));
                    store_chunk(pk, c);
                };
                uint32_t g0[32], g1[32];
                tmem_ld32(tb + 0, g0);
                tmem_wait_ld(g0);
#pragma unroll
                for (int ci = 0; ci < 8; ci += 2) {
                    tmem_ld32(tb + 32 * (ci + 1), g1);
                    emit(g0, 32 * ci);
                    tmem_wait_ld(g1);
                    if (ci + 2 < 8) {
                        tmem_ld32(tb + 32 * (ci + 2), g0);
                        emit(g1, 32 * (ci + 1));
                        tmem_wait_ld(g0);
                    } else {
                        release();
                        emit(g1, 32 * (ci + 1));
                    }
                }
            }
        }
        if (!ok) raise_abort();
    }

    // ---- teardown: the epilogue's TMA stores are complete before the kernel ends
    if (warp >= 2 && lane == 0) bulk_wait_all();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem_base, 512);
}

// bf16 matrix [rows][inner], box = box_inner x box_rows, the given swizzle
static bool encode(CUtensorMap* tm, const void* base, uint64_t inner, uint64_t rows, uint32_t box_inner,
                   uint32_t box_rows, CUtensorMapSwizzle swz) {
    EncodeTiledFn fn = encode_tiled_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {inner, rows};
    cuuint64_t strides[1] = {inner * 2};
    cuuint32_t box[2] = {box_inner, box_rows};
    cuuint32_t estr[2] = {1, 1};
    return fn(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <bool SWIGLU>
static cudaError_t run_dual(const Ctx& c, const void* act, int S, const void* w1, const void* w2, DArgs a) {
    using C = DCfg<SWIGLU>;
    set_wait_args(a);
    auto kern = grouped_gemm_dual_kernel<SWIGLU>;
    static bool attr_done[64] = {};
    if (c.device < 0 || c.device >= 64) return cudaErrorInvalidDevice;
    if (!attr_done[c.device]) {
        cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
        if (err != cudaSuccess) return err;
        attr_done[c.device] = true;
    }
    CUtensorMap tm_act, tm_w1, tm_w2, tm_out;
    const uint64_t wrows = (uint64_t)a.E * a.n_out;
    if (!encode(&tm_act, act, (uint64_t)a.K, (uint64_t)S, BK, RH, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !encode(&tm_w1, w1, (uint64_t)a.K, wrows, BK, SWIGLU ? 128 : 256, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !encode(&tm_w2, SWIGLU ? w2 : w1, (uint64_t)a.K, wrows, BK, SWIGLU ? 128 : 256, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !encode(&tm_out, a.out, (uint64_t)a.ldo, (uint64_t)S, 32, 32, CU_TENSOR_MAP_SWIZZLE_64B))
        return cudaErrorInvalidValue;
    // upper bound on the tile count: sum_e ceil(cnt_e / 256) <= S / 256 + E
    const int64_t max_tiles = ((int64_t)S / RP + a.E) * (a.n_out / C::COLS);
    const int grid = (int)(max_tiles < c.num_sms ? max_tiles : c.num_sms);
    if (grid <= 0) return cudaSuccess;
    return launch(kern, dim3(grid), dim3(kThreads), (size_t)C::SMEM, c, tm_act, tm_w1, tm_w2, tm_out, a);
}

}  // namespace tcd

bool use_dual_gemm(int S, int E, int n_out) {
    const int avg = E > 0 ? S / E : 0;
    return avg >= 256 && !use_pair_gemm(S, E, n_out) && n_out % 256 == 0;
}

cudaError_t launch_gate_up_bf16_dual(const Ctx& c, const void* xp, const void* Wg, const void* Wu,
                                     const int32_t* counts, const int32_t* offsets, int S, int E, int d, int d_ff,
                                     void* h, int32_t* status, bool raw, int32_t* tile_ctr) {
    if (S == 0) return cudaSuccess;
    tcd::DArgs a{counts, offsets, E, d, d_ff, static_cast<uint16_t*>(h), (int64_t)d_ff * (raw ? 2 : 1), status, S};
    a.raw = raw ? 1 : 0;
    a.tile_ctr = tile_ctr;
    return tcd::run_dual<true>(c, xp, S, Wg, Wu, a);
}

}  // namespace moe
