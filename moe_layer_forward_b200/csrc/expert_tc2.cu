// Step 4 for many rows per expert: grouped GEMMs on CTA pairs (tcgen05 cta_group::2).
//
// Same mathematics as expert_tc.cu ("推理计算流梳理", §实际 MLP 计算策略 and §EP 路径):
//   gate/up: h = SiLU(xp W_gate^T) ⊙ (xp W_up^T)        down: y = h W_down^T
// but each work tile is computed by the two CTAs of a cluster with one 2-SM
// MMA: M = 256 token rows (128 per CTA), N = 256 weight rows (128 staged by
// each CTA), D = 128 x 256 in each CTA's tensor memory.  Each SM stages 32 KB
// per 64-wide K step instead of 48 KB for the one-CTA 128 x 256 tile, a third
// less L2 -> shared-memory traffic per FLOP; on B200 both shapes are limited by
// that delivery (in-kernel counters: the MMA waits for a filled stage 25-30% of
// the time with all stages in flight), and a mainloop probe with random bf16
// operands sustains ~1.5 PFLOP/s on the pair against ~1.3 on one CTA.
// The cost is padding: an expert's rows are rounded up to 256 rather than 128,
// so the host only picks this kernel when experts have many rows.
//
// Tile = (expert e, row block rb of 256, column block cb), run in the order
// (e, cb, rb) so the row blocks that share a weight block are computed back to
// back and read it from HBM once.  Column block:
//   gate/up: 128 features; CTA 0 stages the gate rows and CTA 1 the up rows,
//            so accumulator columns 0-127 hold gate and 128-255 up.
//   down:    256 output features; CTA r stages rows [128r, 128r+128).
//
// Roles per CTA (192 threads): warp 0 TMA producer (both CTAs load their own
// operands, completion counted on the leader CTA's stage barrier); warp 1 TMEM
// owner, and in the leader CTA the MMA issuer (commits multicast to both
// CTAs' barriers); warps 2..5 epilogue over the CTA's own 128 rows.  All waits
// are bounded.
#include <cuda.h>
#include <math.h>

#include "common.cuh"
#include "kernels.h"
#include "tc_ptx.cuh"

namespace moe {
namespace tc2 {
using namespace tc;

constexpr int BK = 64;
constexpr int kThreads = 192;
constexpr int kSmemLimit = 232448;
constexpr int RB = 256;              // token rows per tile (128 per CTA)
constexpr int STAGE_A = 128 * 128;   // 128 token rows x 128 B
constexpr int STAGE_B = 128 * 128;   // 128 weight rows x 128 B (half of N = 256)
constexpr int STAGE_BYTES = STAGE_A + STAGE_B;
constexpr int STAGES = 6;

struct Aux2 {
    uint64_t full[STAGES];   // leader CTA: both CTAs' loads of a stage landed
    uint64_t empty[STAGES];  // each CTA: the stage's MMAs finished
    uint64_t tfull[2];       // each CTA: accumulator ready
    uint64_t tempty[2];      // leader CTA: both CTAs' epilogues drained the accumulator
    uint64_t drain;
    uint64_t never;          // completed by nothing: the injected stall waits on it
    uint32_t tmem_slot;
    int abort_flag;
    int tstart[kMaxExperts + 1];
    int cnt[kMaxExperts];
    int off[kMaxExperts];
};
constexpr int AUX_BYTES = 4096;
static_assert((int)sizeof(Aux2) <= AUX_BYTES, "aux block");
// a 4 KB staging buffer per epilogue warp (32 rows x 64 bf16 columns, 128-byte swizzle) from which TMA stores
// the warp's output rows when all 32 are valid
constexpr int EPI_BYTES = 4 * 4096;
constexpr int SMEM = 1024 + STAGES * STAGE_BYTES + AUX_BYTES + EPI_BYTES;
static_assert(SMEM <= kSmemLimit, "shared memory budget");

struct Args2 {
    const int32_t* counts;
    const int32_t* offsets;
    int E;
    int K;      // reduction length
    int n_out;  // weight rows per expert (d_ff for gate/up, d for down)
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
};

__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// address of the same shared-memory location in CTA `rank` of the cluster
__device__ __forceinline__ uint32_t map_to_rank(uint32_t saddr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
    return r;
}
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}
// 2-D TMA load into this CTA's shared memory, completion counted on an mbarrier of either CTA of the pair
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap* tm, int x, int y, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, "
        "%3}], [%4];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(tm)), "r"(x), "r"(y), "r"(bar)
        : "memory");
}
__device__ __forceinline__ void tmem_alloc_pair(uint32_t slot, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(slot), "r"(ncols) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void mma_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(acc)
        : "memory");
}
// arrive on the barrier at this offset in both CTAs once this thread's MMAs are complete
__device__ __forceinline__ void commit_pair_multicast(uint32_t bar) {
    asm volatile(
        "{\n\t.reg .b16 m;\n\tmov.b16 m, 3;\n\t"
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], m;\n\t}" ::"r"(
            bar)
        : "memory");
}
__device__ __forceinline__ void commit_pair_local(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void decode_tile2(const Aux2& a, int E, int tile, int& e, int& rb, int& cb) {
    int lo = 0, hi = E - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (a.tstart[mid] <= tile) lo = mid; else hi = mid - 1;
    }
    e = lo;
    const int local = tile - a.tstart[e];
    const int nrb = (a.cnt[e] + RB - 1) / RB;
    cb = local / nrb;
    rb = local - cb * nrb;
}

template <bool SWIGLU>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    grouped_gemm_2sm_kernel(const __grid_constant__ CUtensorMap tm_act, const __grid_constant__ CUtensorMap tm_w1,
                            const __grid_constant__ CUtensorMap tm_w2, const __grid_constant__ CUtensorMap tm_out,
                            const Args2 p) {
    constexpr int WCOLS = SWIGLU ? 128 : 256;  // output columns of one weight block
    constexpr uint32_t TMEM_COLS = 512;          // two accumulators of up to 256 columns
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    Aux2& aux = *reinterpret_cast<Aux2*>(smem + STAGES * STAGE_BYTES);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_rank();
    const bool leader = rank == 0;
    volatile int* abort_flag = &aux.abort_flag;
    const uint64_t wait_ns = p.wait_ns;

    if (warp == 0 && lane == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(smem_u32(&aux.full[s]), 1);
            mbar_init(smem_u32(&aux.empty[s]), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(smem_u32(&aux.tfull[b]), 1);
            mbar_init(smem_u32(&aux.tempty[b]), 8);
        }
        mbar_init(smem_u32(&aux.drain), 1);
        mbar_init(smem_u32(&aux.never), 1);
        aux.abort_flag = 0;
        fence_mbar_init();
        tma_prefetch(&tm_act);
        tma_prefetch(&tm_w1);
        if (SWIGLU) tma_prefetch(&tm_w2);
        tma_prefetch(&tm_out);
    }
    cluster_sync();  // the peer's barriers exist before any remote arrive or copy completion
    if (warp == 1) tmem_alloc_pair(smem_u32(&aux.tmem_slot), TMEM_COLS);

    pdl_wait();
    const int E = p.E;
    for (int e = threadIdx.x; e < E; e += kThreads) {
        int o, n;
        if (!clamp_segment(p.offsets[e], p.counts[e], p.S, o, n) && leader) set_status(p.status, DEV_BAD_COUNT);
        aux.cnt[e] = n;
        aux.off[e] = o;
    }
    __syncthreads();
    const int ncb = p.n_out / WCOLS;
    if (warp == 0) {
        int loc[8], sum = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int e = lane * 8 + i;
            loc[i] = (e < E) ? ((aux.cnt[e] + RB - 1) / RB) * ncb : 0;
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
    const int cluster_id = blockIdx.x >> 1, nclusters = gridDim.x >> 1;
    auto raise_abort = [&]() {
        if (lane == 0) {
            *abort_flag = 1;
            set_status(p.status, DEV_TIMEOUT);
        }
    };

    if (warp == 0) {
        // ================= TMA producer (both CTAs)
        int stage = 0;
        uint32_t phase = 0;
        const int nk = p.K / BK;
        bool ok = true;
        uint64_t last_issue = 0;
        for (int tile = cluster_id; tile < total && ok && !*abort_flag; tile += nclusters) {
            int e, rb, cb;
            decode_tile2(aux, E, tile, e, rb, cb);
            const int act_row = aux.off[e] + rb * RB + 128 * (int)rank;
            const int w_row = e * p.n_out + cb * WCOLS + (SWIGLU ? 0 : 128 * (int)rank);
            const CUtensorMap* tm_w = (SWIGLU && rank == 1) ? &tm_w2 : &tm_w1;
            for (int kb = 0; kb < nk; ++kb) {
                if (!warp_wait(smem_u32(&aux.empty[stage]), phase ^ 1u, abort_flag, wait_ns)) {
                    ok = false;
                    break;
                }
                if (lane == 0) {
                    const uint32_t a0 = smem_u32(smem + stage * STAGE_BYTES);
                    const uint32_t full_leader = map_to_rank(smem_u32(&aux.full[stage]), 0);
                    if (leader) mbar_expect_tx(smem_u32(&aux.full[stage]), 2 * STAGE_BYTES);
                    tma_load_2d_pair(a0, &tm_act, kb * BK, act_row, full_leader);
                    tma_load_2d_pair(a0 + STAGE_A, tm_w, kb * BK, w_row, full_leader);
                    last_issue = globaltimer();
                }
                __syncwarp();
                if (++stage == STAGES) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
        }
        if (!ok) raise_abort();
        // Unwinding: this CTA's loads complete on the leader's barrier, which the other CTA cannot wait
        // on, so a producer that stopped early waits a fixed 200 us after its last load (a 32 KB copy
        // from valid memory lands within microseconds) before the CTA may reach its teardown.
        if (*abort_flag && lane == 0 && last_issue != 0)
            while (globaltimer() < last_issue + 200000ull) {
            }
        __syncwarp();
    } else if (warp == 1) {
        // ================= MMA issuer (leader CTA only)
        if (leader) {
            int stage = 0;
            uint32_t phase = 0;
            const int nk = p.K / BK;
            int j = 0;
            bool ok = true;
            for (int tile = cluster_id; tile < total && ok && !*abort_flag; tile += nclusters, ++j) {
                const uint32_t idesc = idesc_bf16(256, 256);
                const int buf = j & 1;
                if (!warp_wait(smem_u32(&aux.tempty[buf]), ((uint32_t)(j >> 1) & 1u) ^ 1u, abort_flag, wait_ns)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)(buf * 256);
                for (int kb = 0; kb < nk; ++kb) {
                    if (!warp_wait(smem_u32(&aux.full[stage]), phase, abort_flag, wait_ns)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    if (lane == 0) {
                        const uint32_t a0 = smem_u32(smem + stage * STAGE_BYTES);
#pragma unroll
                        for (int kk = 0; kk < BK / 16; ++kk)
                            mma_pair(d_tmem, sdesc_sw128(a0 + kk * 32), sdesc_sw128(a0 + STAGE_A + kk * 32), idesc,
                                     (kb | kk) ? 1u : 0u);
                        commit_pair_multicast(smem_u32(&aux.empty[stage]));
                    }
                    __syncwarp();
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok) break;
                if (lane == 0) commit_pair_multicast(smem_u32(&aux.tfull[buf]));
                __syncwarp();
            }
            if (!ok) raise_abort();
            if (lane == 0) {
                commit_pair_local(smem_u32(&aux.drain));
                mbar_drain(smem_u32(&aux.drain), 0, drain_deadline());
            }
            __syncwarp();
        }
    } else {
        // ================= epilogue (warps 2..5 -> TMEM lane quarters 2,3,0,1), both CTAs
        const int q = warp & 3;
        const uint32_t tempty_leader0 = map_to_rank(smem_u32(&aux.tempty[0]), 0);
        const uint32_t tempty_leader1 = map_to_rank(smem_u32(&aux.tempty[1]), 0);
        int j = 0;
        bool ok = true;
        if (p.stall && !warp_wait(smem_u32(&aux.never), 0, abort_flag, wait_ns)) ok = false;
        for (int tile = cluster_id; tile < total && ok && !*abort_flag; tile += nclusters, ++j) {
            const int buf = j & 1;
            if (!warp_wait(smem_u32(&aux.tfull[buf]), (uint32_t)(j >> 1) & 1u, abort_flag, wait_ns)) {
                ok = false;
                break;
            }
            tc_fence_after();
            int e, rb, cb;
            decode_tile2(aux, E, tile, e, rb, cb);
            const int rows = min(128, aux.cnt[e] - rb * RB - 128 * (int)rank);  // this CTA's valid rows (may be <= 0)
            const int m = 32 * q + lane;                                        // row inside this CTA's half
            const bool valid = m < rows;
            uint16_t* orow = p.out + ((int64_t)aux.off[e] + (int64_t)rb * RB + 128 * (int)rank + m) * p.ldo +
                             (int64_t)cb * WCOLS;
            const uint32_t tb_addr = tmem_base + (uint32_t)(buf * 256) + ((uint32_t)(32 * q) << 16);
            // a warp whose 32 rows are all valid writes them by TMA from its staging buffer (full 128-byte rows);
            // a warp with fewer stores its valid rows directly
            const bool tma_rows = !p.raw && rows - 32 * q >= 32;
            const uint32_t stg = smem_u32(smem) + STAGES * STAGE_BYTES + AUX_BYTES + 4096 * q;
            const int grow = aux.off[e] + rb * RB + 128 * (int)rank + 32 * q;  // first output row of this warp
            if (rows > 32 * q) {  // skip quarters without valid rows (warp-uniform)
#pragma unroll 1
                for (int c = 0; c < WCOLS; c += 64) {
                    uint32_t pk[32];  // 64 bf16 of this lane's row: columns c .. c + 63
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        uint32_t g[32];
                        tmem_ld32(tb_addr + c + 32 * hh, g);
                        if constexpr (SWIGLU) {
                            uint32_t u[32];
                            tmem_ld32(tb_addr + 128 + c + 32 * hh, u);
                            tmem_wait_ld(g);
                            tmem_wait_ld(u);
                            if (p.raw) {  // GEMM-core test form: g and u stored apart
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
                                        st16(orow + c + 32 * hh + 8 * v, make_uint4(a4[0], a4[1], a4[2], a4[3]));
                                        st16(orow + p.n_out + c + 32 * hh + 8 * v,
                                             make_uint4(b4[0], b4[1], b4[2], b4[3]));
                                    }
                                }
                                continue;
                            }
#pragma unroll
                            for (int i = 0; i < 16; ++i) {
                                const float g0 = __uint_as_float(g[2 * i]), g1 = __uint_as_float(g[2 * i + 1]);
                                pk[16 * hh + i] =
                                    pack_bf16x2(__fdividef(g0, 1.0f + __expf(-g0)) * __uint_as_float(u[2 * i]),
                                                __fdividef(g1, 1.0f + __expf(-g1)) * __uint_as_float(u[2 * i + 1]));
                            }
                        } else {
                            tmem_wait_ld(g);
#pragma unroll
                            for (int i = 0; i < 16; ++i)
                                pk[16 * hh + i] = pack_bf16x2(__uint_as_float(g[2 * i]), __uint_as_float(g[2 * i + 1]));
                        }
                    }
                    if (SWIGLU && p.raw) continue;
                    if (tma_rows) {
                        if (lane == 0) bulk_wait_read();  // the previous store from this buffer has read it
                        __syncwarp();
                        // row `lane`, 16-byte chunk v at lane * 128 + ((v ^ (lane % 8)) * 16): the output tensor
                        // map's 128-byte swizzle; eight consecutive lanes cover all 32 banks
#pragma unroll
                        for (int v = 0; v < 8; ++v)
                            st_shared16(stg + lane * 128 + ((v ^ (lane & 7)) << 4),
                                        make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]));
                        fence_proxy_async_smem();
                        __syncwarp();
                        if (lane == 0) {
                            tma_store_2d(&tm_out, stg, cb * WCOLS + c, grow);
                            bulk_commit();
                        }
                    } else if (valid) {
#pragma unroll
                        for (int v = 0; v < 8; ++v)
                            st16(orow + c + 8 * v, make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]));
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(buf ? tempty_leader1 : tempty_leader0);
        }
        if (!ok) raise_abort();
    }

    // ---- teardown: the epilogue's TMA stores are complete; the leader's MMAs read this CTA's shared memory
    // and write its tensor memory
    if (warp >= 2 && lane == 0) bulk_wait_all();
    tc_fence_before();
    __syncthreads();
    cluster_sync();
    tc_fence_after();
    if (warp == 1) tmem_dealloc_pair(tmem_base, TMEM_COLS);
}

// bf16 matrix [rows][inner], box = 64 x box_rows, 128-byte swizzle
static bool encode(CUtensorMap* tm, const void* base, uint64_t inner, uint64_t rows, uint32_t box_rows) {
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

template <bool SWIGLU>
static cudaError_t run2(const Ctx& c, const void* act, int S, const void* w1, const void* w2, Args2 a) {
    set_wait_args(a);
    auto kern = grouped_gemm_2sm_kernel<SWIGLU>;
    static bool attr_done[64] = {};
    if (c.device < 0 || c.device >= 64) return cudaErrorInvalidDevice;
    if (!attr_done[c.device]) {
        cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM);
        if (err != cudaSuccess) return err;
        attr_done[c.device] = true;
    }
    CUtensorMap tm_act, tm_w1, tm_w2, tm_out;
    if (!encode(&tm_act, act, (uint64_t)a.K, (uint64_t)S, 128)) return cudaErrorInvalidValue;
    // the output [S][ldo] in boxes of 64 columns x 32 rows (one epilogue warp's rows)
    if (!encode(&tm_out, a.out, (uint64_t)a.ldo, (uint64_t)S, 32)) return cudaErrorInvalidValue;
    if (!encode(&tm_w1, w1, (uint64_t)a.K, (uint64_t)a.E * a.n_out, 128)) return cudaErrorInvalidValue;
    if (!encode(&tm_w2, SWIGLU ? w2 : w1, (uint64_t)a.K, (uint64_t)a.E * a.n_out, 128)) return cudaErrorInvalidValue;
    static int max_clusters[64] = {};
    if (max_clusters[c.device] == 0) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(2 * (c.num_sms / 2));
        cfg.blockDim = dim3(kThreads);
        cfg.dynamicSmemBytes = SMEM;
        int n = 0;
        if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess || n <= 0) {
            cudaGetLastError();
            n = c.num_sms / 2;
        }
        max_clusters[c.device] = n;
    }
    const int wcols = SWIGLU ? 128 : 256;
    const int64_t max_tiles = ((int64_t)S / RB + a.E) * (a.n_out / wcols);
    int clusters = max_clusters[c.device];
    if (max_tiles < clusters) clusters = (int)max_tiles;
    if (clusters <= 0) return cudaSuccess;
    return launch(kern, dim3(2 * clusters), dim3(kThreads), (size_t)SMEM, c, tm_act, tm_w1, tm_w2, tm_out, a);
}

}  // namespace tc2

// The pair kernel rounds each expert's rows up to 256 (the one-CTA kernel to 128).  Measured on
// B200: at 512 rows per expert the extra padding outweighs its faster MMA rate (gate/up 1.55 vs
// 1.45 ms), at 1024 it wins (2.59 vs 2.75 ms).
bool use_pair_gemm(int S, int E, int n_out) {
    return E > 0 && S / E >= 768 && n_out % 256 == 0;
}

cudaError_t launch_gate_up_bf16_pair(const Ctx& c, const void* xp, const void* Wg, const void* Wu,
                                     const int32_t* counts, const int32_t* offsets, int S, int E, int d, int d_ff,
                                     void* h, int32_t* status, bool raw) {
    if (S == 0) return cudaSuccess;
    tc2::Args2 a{counts, offsets, E, d, d_ff, static_cast<uint16_t*>(h), (int64_t)d_ff * (raw ? 2 : 1), status, S};
    a.raw = raw ? 1 : 0;
    return tc2::run2<true>(c, xp, S, Wg, Wu, a);
}

cudaError_t launch_down_bf16_pair(const Ctx& c, const void* h, const void* Wd, const int32_t* counts,
                                  const int32_t* offsets, int S, int E, int d, int d_ff, void* y, int32_t* status) {
    if (S == 0) return cudaSuccess;
    tc2::Args2 a{counts, offsets, E, d_ff, d, static_cast<uint16_t*>(y), (int64_t)d, status, S};
    return tc2::run2<false>(c, h, S, Wd, nullptr, a);
}

}  // namespace moe
