// Step 4 for bf16 expert weights: grouped GEMMs on the 5th-generation tensor
// cores (tcgen05.mma, accumulators in tensor memory, operands staged by TMA).
//
// "推理计算流梳理" (huanyp.cn), §实际 MLP 计算策略: Y = (SiLU(X W_gate) ⊙ X W_up) W_down;
// §EP 路径: the active experts of a rank run as one grouped GEMM.  The Chitu MoE
// page (§专家计算实现) describes the prefill layout this kernel consumes: the rows
// of each expert are contiguous ("deepgemm_contiguous"); its FP8/Hopper kernels
// are prior art, not the design here.
//
// One persistent kernel template covers both halves of the expert MLP:
//   gate/up: h = SiLU(xp W_gate^T) ⊙ (xp W_up^T)   (SwiGLU fused in the epilogue)
//   down:    y = h W_down^T
// A work tile is (expert e, row block rb of R rows, column block cb).  Tiles
// are numbered expert-major, then column block, then row block, and CTAs take
// tiles tile = blockIdx.x + i * gridDim.x, so the row blocks that share a
// weight tile run side by side and read it from L2 once.  The per-expert row
// counts live only on the device; every CTA turns them into a tile prefix
// sum in shared memory (no host sync).
//
// On B200 an M = 128 MMA takes the same time (~86 ns per K = 16 on one SM)
// for every N from 16 to 256, and an M = 64 one as long as M = 128, so a
// tile's cost is set by its instruction count, not its useful rows.  Two
// operand arrangements:
//   rows-as-M: MMA M = 128 token rows x N = 256 weight rows (gate 128 | up
//     128 stacked, or 256 down rows).  Only R = 16/32/64/128 token rows are
//     staged per K slice; the rest of the M = 128 operand reads whatever
//     follows in shared memory and lands in accumulator rows that are never
//     stored.  With few rows per expert one MMA still consumes 8 KB of
//     weights, so the kernel streams weights at HBM speed.
//   weights-as-M (gate/up with few rows per expert): M = 128 gate rows and
//     128 up rows in two MMAs, N = the expert's rows rounded up to 16 (<= R).
//     Measured at 8 rows per expert it runs gate/up ~4% faster than
//     rows-as-M; for down, whose weight tile is one 128-row operand, it
//     leaves the tensor pipe co-limiting and rows-as-M is ~30% faster.
//
// Warp roles (1 CTA per SM; 192 threads, 320 for weights-as-M):
//   warp 0      TMA producer: a STAGES-deep ring of 64-wide K slices (128-byte
//               swizzled rows), one mbarrier pair (full/empty) per stage.
//   warp 1      owns the tensor-memory allocation; lane 0 issues tcgen05.mma
//               (4 x K=16 per stage) and tcgen05.commit to release each stage
//               and to publish a finished accumulator.
//   warps 2..5  epilogue: tcgen05.ld of the accumulator (each warp its 32 TMEM
//               lanes), SiLU(g)*u in fp32, bf16 stores.  Two accumulator
//               buffers let the epilogue of one tile overlap the next tile's MMAs.
//   warps 6..9  (weights-as-M with Args::gather) copy each stage's token rows
//               straight from V through the slot -> token map (cp.async).
// Masked layout (Args::cap > 0): expert e's rows start at e * cap.
// Every wait is bounded (globaltimer); a wait that gives up raises
// DEV_TIMEOUT in the status word and all roles unwind, drain in-flight copies
// and MMAs, free tensor memory and exit.
#include <cuda.h>
#include <math.h>

#include "common.cuh"
#include "kernels.h"
#include "tc_ptx.cuh"

namespace moe {
namespace tc {

constexpr int BK = 64;  // K elements per stage = one 128-byte swizzle row of bf16
// warps 0..5 as below; the weights-as-M form adds warps 6..9 that gather activation rows (Args::gather)
template <bool SWAP, bool SWIGLU, int R>
constexpr int threads_of() { return SWAP ? 320 : 192; }
constexpr int kSmemLimit = 232448;              // 227 KB opt-in per CTA

// SiLU(g) * u with the hardware exp2 and reciprocal (relative error ~1e-6, far below the bf16
// rounding of h that follows); the accurate library forms cost 2-3% of a prefill gate/up GEMM whose
// epilogue warps share issue slots with the producer and MMA warps.
__device__ __forceinline__ float silu_mul(float g, float u) { return __fdividef(g, 1.0f + __expf(-g)) * u; }

// ----------------------------------------------------------------------------- configuration
template <bool SWAP, bool SWIGLU, int R, int COLS>
struct Cfg {
    // SWAP = weights are the MMA's A operand (M = 128 weight rows), activations B (N <= R).
    static_assert(!SWAP || COLS == 128, "weights-as-M tiles cover 128 weight rows");
    static_assert(R == 16 || R == 32 || R == 64 || R == 128, "row block");
    static constexpr int MMA_N = SWAP ? R : (SWIGLU ? 2 * COLS : COLS);
    static_assert(MMA_N % 16 == 0 && MMA_N <= 256, "MMA N for M = 128");
    static constexpr int A_ROWS = SWAP ? 128 : R;
    static constexpr int NUM_A = (SWAP && SWIGLU) ? 2 : 1;
    static constexpr int B_ROWS = SWAP ? R : MMA_N;
    static constexpr int A_BYTES = A_ROWS * 128;
    static constexpr int B_BYTES = B_ROWS * 128;
    static constexpr int STAGE_BYTES = NUM_A * A_BYTES + B_BYTES;
    // the activation slice of a stage: A for rows-as-M, B for weights-as-M
    static constexpr int ACT_OFF = SWAP ? NUM_A * A_BYTES : 0;
    static constexpr int ACT_BYTES = R * 128;
    // rows-as-M reads 128 A rows from the stage start: they must stay inside the stage
    static_assert(SWAP || STAGE_BYTES >= 128 * 128, "M = 128 operand inside its stage");
    static constexpr int WBOX = SWAP ? 128 : (SWIGLU ? 128 : COLS);  // weight rows per TMA box
    // accumulator columns per buffer: SWAP+SWIGLU keeps gate and up side by side
    static constexpr int ACC = SWAP ? (SWIGLU ? 2 * R : R) : MMA_N;
    static constexpr int TMEM_COLS = (2 * ACC <= 32) ? 32 : (2 * ACC <= 64) ? 64 : (2 * ACC <= 128) ? 128 : (2 * ACC <= 256) ? 256 : 512;
    static_assert(2 * ACC <= 512, "two accumulator buffers must fit in 512 TMEM columns");
    static constexpr int AUX_BYTES = 4096;  // barriers, tile tables
    // rows-as-M with 128-row blocks: a 4 KB staging buffer per epilogue warp (32 rows x 64 bf16 columns,
    // 128-byte swizzle) from which TMA stores the warp's output rows when all 32 are valid
    static constexpr bool TMA_OUT = !SWAP && R == 128;
    static constexpr int EPI_BYTES = TMA_OUT ? 4 * 4096 : 0;
    static constexpr int STAGES_MAX = (kSmemLimit - 1024 - AUX_BYTES - EPI_BYTES) / STAGE_BYTES;
    static constexpr int STAGES = STAGES_MAX > 12 ? 12 : STAGES_MAX;
    static_assert(STAGES >= 2, "pipeline depth");
    static constexpr int SMEM = 1024 + STAGES * STAGE_BYTES + AUX_BYTES + EPI_BYTES;
    static constexpr int LDW = R < 32 ? R : 32;  // TMEM columns per tcgen05.ld in the weights-as-M epilogue
};

struct Args {
    const int32_t* counts;
    const int32_t* offsets;
    int E;
    int K;      // reduction length (d for gate/up, d_ff for down)
    int n_out;  // weight rows per expert = output columns
    uint16_t* out;
    int64_t ldo;
    int32_t* status;
    // Optional row gather: when set, activation row i of the expert-contiguous
    // order is row gather[i] of act (the permutation's slot -> token map), read
    // by the gather warps instead of a TMA load of a permuted copy.
    const int32_t* gather;
    const uint16_t* act;
    // Masked layout (cap > 0): expert e's rows are rows [e*cap, e*cap + counts[e]) of fixed
    // per-expert buffers, offsets is unused, and a count outside [0, cap] is clamped and flagged.
    int cap;
    // rows of the expert-contiguous buffers (the output's rows); a segment that does not fit is
    // clamped into it and flagged
    int S;
    int act_rows;  // rows of act when gather is set
    // bounded waits: the limit of one wait, and (failure-path tests only) an extra wait on a barrier
    // that nothing completes, made by the epilogue warps before their first tile
    uint64_t wait_ns = kTimeoutNs;
    int stall = 0;
    // GEMM-core test form of gate/up (SWIGLU only): g and u are stored apart as bf16, g in columns
    // [0, n_out) and u in [n_out, 2 n_out) of an output with ldo = 2 n_out; no SwiGLU product
    int raw = 0;
};

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }


struct Aux {  // lives after the stage ring in shared memory
    uint64_t full[12];
    uint64_t empty[12];
    uint64_t tfull[2];
    uint64_t tempty[2];
    uint64_t drain;
    uint64_t never;  // completed by nothing: the injected stall waits on it
    uint32_t tmem_slot;
    int abort_flag;
    int tstart[kMaxExperts + 1];
    int cnt[kMaxExperts];
    int off[kMaxExperts];
};

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

template <bool SWAP, bool SWIGLU, int R, int COLS>
__global__ void __launch_bounds__(threads_of<SWAP, SWIGLU, R>(), 1)
    grouped_gemm_kernel(const __grid_constant__ CUtensorMap tm_act, const __grid_constant__ CUtensorMap tm_w1,
                        const __grid_constant__ CUtensorMap tm_w2, const __grid_constant__ CUtensorMap tm_out,
                        const Args p) {
    using C = Cfg<SWAP, SWIGLU, R, COLS>;
    constexpr int STAGES = C::STAGES;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    Aux& aux = *reinterpret_cast<Aux*>(smem + STAGES * C::STAGE_BYTES);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    volatile int* abort_flag = &aux.abort_flag;
    const uint64_t wait_ns = p.wait_ns;

    // ---- prologue (overlaps the previous kernel's tail under PDL)
    if (warp == 0 && lane == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(smem_u32(&aux.full[s]), p.gather ? 2 : 1);  // + the gather warp's arrival
            mbar_init(smem_u32(&aux.empty[s]), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(smem_u32(&aux.tfull[b]), 1);
            mbar_init(smem_u32(&aux.tempty[b]), 4);
        }
        mbar_init(smem_u32(&aux.drain), 1);
        mbar_init(smem_u32(&aux.never), 1);
        aux.abort_flag = 0;
        fence_mbar_init();
        tma_prefetch(&tm_act);
        tma_prefetch(&tm_w1);
        if (SWIGLU) tma_prefetch(&tm_w2);
        if (C::TMA_OUT) tma_prefetch(&tm_out);
    }
    if (warp == 1) tmem_alloc(smem_u32(&aux.tmem_slot), C::TMEM_COLS);

    pdl_wait();
    const int E = p.E;
    for (int e = threadIdx.x; e < E; e += (int)blockDim.x) {
        if (p.cap > 0) {
            const int n = p.counts[e];
            if (n < 0 || n > p.cap) set_status(p.status, DEV_BAD_COUNT);
            aux.cnt[e] = n < 0 ? 0 : (n > p.cap ? p.cap : n);
            aux.off[e] = e * p.cap;
        } else {
            int o, n;
            if (!clamp_segment(p.offsets[e], p.counts[e], p.S, o, n)) set_status(p.status, DEV_BAD_COUNT);
            aux.cnt[e] = n;
            aux.off[e] = o;
        }
    }
    __syncthreads();
    if (warp == 0) {
        // tile prefix over experts: lane owns experts 8*lane .. 8*lane+7
        const int ncb = p.n_out / COLS;
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

    if (warp == 0) {
        // ================= TMA producer
        int stage = 0;
        uint32_t phase = 0;
        uint32_t used = 0, last_parity = 0;
        const int nk = p.K / BK;
        for (int tile = blockIdx.x; tile < total && !*abort_flag; tile += gridDim.x) {
            int e, rb, cb;
            decode_tile(aux, E, R, tile, e, rb, cb);
            const int act_row = aux.off[e] + rb * R;
            const int w_row = e * p.n_out + cb * COLS;
            for (int kb = 0; kb < nk; ++kb) {
                const uint32_t full = smem_u32(&aux.full[stage]), empty = smem_u32(&aux.empty[stage]);
                if (!warp_wait(empty, phase ^ 1u, abort_flag, wait_ns)) {
                    if (lane == 0) {
                        *abort_flag = 1;
                        set_status(p.status, DEV_TIMEOUT);
                    }
                    break;
                }
                if (lane == 0) {
                    uint8_t* st = smem + stage * C::STAGE_BYTES;
                    const uint32_t a0 = smem_u32(st);
                    const bool gath = p.gather != nullptr;
                    mbar_expect_tx(full, C::STAGE_BYTES - (gath ? C::ACT_BYTES : 0));
                    if constexpr (!SWAP) {
                        if (!gath) tma_load_2d(a0, &tm_act, kb * BK, act_row, full);
                        tma_load_2d(a0 + C::A_BYTES, &tm_w1, kb * BK, w_row, full);
                        if (SWIGLU) tma_load_2d(a0 + C::A_BYTES + 128 * 128, &tm_w2, kb * BK, w_row, full);
                    } else {
                        tma_load_2d(a0, &tm_w1, kb * BK, w_row, full);
                        if (SWIGLU) tma_load_2d(a0 + C::A_BYTES, &tm_w2, kb * BK, w_row, full);
                        if (!gath) tma_load_2d(a0 + C::NUM_A * C::A_BYTES, &tm_act, kb * BK, act_row, full);
                    }
                }
                used |= 1u << stage;
                last_parity = (last_parity & ~(1u << stage)) | (phase << stage);
                if (++stage == STAGES) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
        }
        // make sure no copy into this CTA's shared memory is still in flight
        {
            const uint64_t dl = drain_deadline();
            for (int s = 0; s < STAGES; ++s)
                if (used & (1u << s)) mbar_drain(smem_u32(&aux.full[s]), (last_parity >> s) & 1u, dl);
        }
    } else if (warp == 1) {
        // ================= MMA issuer
        int stage = 0;
        uint32_t phase = 0;
        const int nk = p.K / BK;
        int j = 0;
        for (int tile = blockIdx.x; tile < total && !*abort_flag; tile += gridDim.x, ++j) {
            const int buf = j & 1;
            const uint32_t use = (uint32_t)(j >> 1);
            if (!warp_wait(smem_u32(&aux.tempty[buf]), (use & 1u) ^ 1u, abort_flag, wait_ns)) {
                if (lane == 0) {
                    *abort_flag = 1;
                    set_status(p.status, DEV_TIMEOUT);
                }
                break;
            }
            tc_fence_after();
            uint32_t idesc;
            if constexpr (SWAP) {
                int e, rb, cb;
                decode_tile(aux, E, R, tile, e, rb, cb);
                const int rows = min(R, aux.cnt[e] - rb * R);
                idesc = idesc_bf16(128, (rows + 15) & ~15);
            } else {
                idesc = idesc_bf16(128, C::MMA_N);
            }
            const uint32_t d_tmem = tmem_base + (uint32_t)(buf * C::ACC);
            bool ok = true;
            for (int kb = 0; kb < nk; ++kb) {
                if (!warp_wait(smem_u32(&aux.full[stage]), phase, abort_flag, wait_ns)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                if (lane == 0) {
                    const uint32_t a0 = smem_u32(smem + stage * C::STAGE_BYTES);
#pragma unroll
                    for (int kk = 0; kk < BK / 16; ++kk) {
                        const uint32_t acc = (kb | kk) ? 1u : 0u;
                        if constexpr (!SWAP) {
                            tc_mma(d_tmem, sdesc_sw128(a0 + kk * 32), sdesc_sw128(a0 + C::A_BYTES + kk * 32), idesc,
                                   acc);
                        } else {
                            const uint32_t b0 = a0 + C::NUM_A * C::A_BYTES;
                            tc_mma(d_tmem, sdesc_sw128(a0 + kk * 32), sdesc_sw128(b0 + kk * 32), idesc, acc);
                            if (SWIGLU)
                                tc_mma(d_tmem + R, sdesc_sw128(a0 + C::A_BYTES + kk * 32), sdesc_sw128(b0 + kk * 32),
                                       idesc, acc);
                        }
                    }
                    tc_commit(smem_u32(&aux.empty[stage]));
                }
                __syncwarp();
                if (++stage == STAGES) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
            if (!ok) {
                if (lane == 0) {
                    *abort_flag = 1;
                    set_status(p.status, DEV_TIMEOUT);
                }
                break;
            }
            if (lane == 0) tc_commit(smem_u32(&aux.tfull[buf]));
            __syncwarp();
        }
        // all MMAs of this thread complete before tensor memory is freed
        if (lane == 0) {
            tc_commit(smem_u32(&aux.drain));
            mbar_drain(smem_u32(&aux.drain), 0, drain_deadline());
        }
        __syncwarp();
    } else if (SWAP && warp >= 6) {
        // ================= row gather (warps 6..9, only with p.gather): warp gw fills the stages
        // g = gw, gw + 4, ... with the tile's activation rows, 16-byte cp.async chunks into the
        // 128-byte-swizzled layout a TMA load would produce (chunk c of row r at r*128 + (c ^ r%8)*16).
        // It waits for its own copies and fences them into the async proxy before arriving on the
        // stage's full barrier, which the tensor cores' reads are ordered after.
        if (p.gather != nullptr) {  // weights-as-M only: the rows are the B operand, R <= 64
            constexpr int RPL = R / 4;    // rows per lane: lane covers rows (lane / 8) + 4 i
            const int gw = warp - 6;
            const int nk = p.K / BK;
            const int c = lane & 7, r0 = lane >> 3;
            int tok[RPL];
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
                        int tk = r < rows ? p.gather[base + r] : 0;
                        if (tk < 0 || tk >= p.act_rows) {  // a bad map entry reads row 0 instead and is flagged
                            if (c == 0) set_status(p.status, DEV_BAD_COUNT);
                            tk = 0;
                        }
                        tok[i] = tk;
                    }
                    cur = tile;
                }
                const int stage = g % STAGES;
                const uint32_t use = (uint32_t)(g / STAGES);
                if (!warp_wait(smem_u32(&aux.empty[stage]), (use & 1u) ^ 1u, abort_flag, wait_ns)) {
                    if (lane == 0) {
                        *abort_flag = 1;
                        set_status(p.status, DEV_TIMEOUT);
                    }
                    break;
                }
                const uint32_t dst = smem_u32(smem + stage * C::STAGE_BYTES) + C::ACT_OFF;
                const uint16_t* src = p.act + (int64_t)kb * BK + c * 8;
#pragma unroll
                for (int i = 0; i < RPL; ++i) {
                    const int r = r0 + 4 * i;
                    if (r < rows)  // rows past the tile's count feed only accumulator entries that are never stored
                        cp_async16(dst + r * 128 + ((c ^ (r & 7)) << 4), src + (int64_t)tok[i] * p.K);
                }
                cp_async_wait_all();
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_u32(&aux.full[stage]));
            }
        }
    } else {
        // ================= epilogue (warps 2..5 -> TMEM lane quarters 2,3,0,1)
        const int q = warp & 3;
        int j = 0;
        if (p.stall && !warp_wait(smem_u32(&aux.never), 0, abort_flag, wait_ns) && lane == 0) {
            *abort_flag = 1;
            set_status(p.status, DEV_TIMEOUT);
        }
        for (int tile = blockIdx.x; tile < total && !*abort_flag; tile += gridDim.x, ++j) {
            const int buf = j & 1;
            const uint32_t use = (uint32_t)(j >> 1);
            if (!warp_wait(smem_u32(&aux.tfull[buf]), use & 1u, abort_flag, wait_ns)) {
                if (lane == 0) {
                    *abort_flag = 1;
                    set_status(p.status, DEV_TIMEOUT);
                }
                break;
            }
            tc_fence_after();
            int e, rb, cb;
            decode_tile(aux, E, R, tile, e, rb, cb);
            const int rows = min(R, aux.cnt[e] - rb * R);
            const int64_t row0 = (int64_t)aux.off[e] + (int64_t)rb * R;
            const uint32_t tb = tmem_base + (uint32_t)(buf * C::ACC) + ((uint32_t)(32 * q) << 16);
            if constexpr (!SWAP) {
                const int m = 32 * q + lane;  // activation row inside the tile
                uint16_t* orow = p.out + (row0 + m) * p.ldo + (int64_t)cb * COLS;
                const bool valid = m < rows;
                // a warp whose 32 rows are all valid writes them by TMA from its staging buffer (full 128-byte
                // rows, no partial-line traffic); a warp with fewer stores its valid rows directly
                const bool tma_rows = C::TMA_OUT && !p.raw && rows - 32 * q >= 32;
                const uint32_t stg = smem_u32(smem) + STAGES * C::STAGE_BYTES + C::AUX_BYTES + 4096 * q;
                // warp-uniform: a lane quarter past the tile's rows holds nothing to store
#pragma unroll 1
                for (int c = 0; c < (32 * q < rows ? COLS : 0); c += 64) {
                    uint32_t pk[32];  // 64 bf16 of this lane's row: columns c .. c + 63
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        uint32_t g[32];
                        tmem_ld32(tb + c + 32 * hh, g);
                        if constexpr (SWIGLU) {
                            uint32_t u[32];
                            tmem_ld32(tb + COLS + c + 32 * hh, u);
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
                            for (int i = 0; i < 16; ++i)
                                pk[16 * hh + i] =
                                    pack_bf16x2(silu_mul(__uint_as_float(g[2 * i]), __uint_as_float(u[2 * i])),
                                                silu_mul(__uint_as_float(g[2 * i + 1]), __uint_as_float(u[2 * i + 1])));
                        } else {
                            tmem_wait_ld(g);
#pragma unroll
                            for (int i = 0; i < 16; ++i)
                                pk[16 * hh + i] = pack_bf16x2(__uint_as_float(g[2 * i]), __uint_as_float(g[2 * i + 1]));
                        }
                    }
                    if (SWIGLU && p.raw) continue;
                    if (tma_rows) {
                        // the staging buffer is free once the previous store from it has read it
                        if (lane == 0) bulk_wait_read();
                        __syncwarp();
                        // row `lane`, 16-byte chunk v at lane * 128 + ((v ^ (lane % 8)) * 16): the 128-byte swizzle
                        // of the output tensor map; eight consecutive lanes cover all 32 banks
#pragma unroll
                        for (int v = 0; v < 8; ++v)
                            st_shared16(stg + lane * 128 + ((v ^ (lane & 7)) << 4),
                                        make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]));
                        fence_proxy_async_smem();
                        __syncwarp();
                        if (lane == 0) {
                            tma_store_2d(&tm_out, stg, cb * COLS + c, (int)(row0 + 32 * q));
                            bulk_commit();
                        }
                    } else if (valid) {
#pragma unroll
                        for (int v = 0; v < 8; ++v)
                            st16(orow + c + 8 * v, make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]));
                    }
                }
            } else {
                const int f = 32 * q + lane;  // weight row (output column) inside the tile
                uint16_t* ocol = p.out + row0 * p.ldo + (int64_t)cb * 128 + f;
#pragma unroll 1
                for (int c = 0; c < rows; c += C::LDW) {
                    uint32_t g[C::LDW];
                    tmem_ld(tb + c, g);
                    if constexpr (SWIGLU) {
                        uint32_t u[C::LDW];
                        tmem_ld(tb + R + c, u);
                        tmem_wait_ld(g);
                        tmem_wait_ld(u);
                        if (p.raw) {  // GEMM-core test form: g and u stored apart
#pragma unroll
                            for (int i = 0; i < C::LDW; ++i)
                                if (c + i < rows) {
                                    ocol[(int64_t)(c + i) * p.ldo] = (uint16_t)f32_to_bf16_bits(__uint_as_float(g[i]));
                                    ocol[(int64_t)(c + i) * p.ldo + p.n_out] =
                                        (uint16_t)f32_to_bf16_bits(__uint_as_float(u[i]));
                                }
                            continue;
                        }
#pragma unroll
                        for (int i = 0; i < C::LDW; ++i)
                            if (c + i < rows)
                                ocol[(int64_t)(c + i) * p.ldo] = (uint16_t)f32_to_bf16_bits(
                                    silu_mul(__uint_as_float(g[i]), __uint_as_float(u[i])));
                    } else {
                        tmem_wait_ld(g);
#pragma unroll
                        for (int i = 0; i < C::LDW; ++i)
                            if (c + i < rows)
                                ocol[(int64_t)(c + i) * p.ldo] = (uint16_t)f32_to_bf16_bits(__uint_as_float(g[i]));
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&aux.tempty[buf]));
        }
    }

    // ---- teardown: the epilogue's TMA stores are complete before the kernel ends
    if (C::TMA_OUT && warp >= 2 && warp < 6 && lane == 0) bulk_wait_all();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem_base, C::TMEM_COLS);
}

// ----------------------------------------------------------------------------- host side
// bf16 matrix [rows][inner] (inner contiguous), box = 64 x box_rows, 128-byte swizzle
static bool encode_2d(CUtensorMap* tm, const void* base, uint64_t inner, uint64_t rows, uint32_t box_rows) {
    EncodeTiledFn fn = encode_tiled_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {inner, rows};
    cuuint64_t strides[1] = {inner * 2};
    cuuint32_t box[2] = {(cuuint32_t)BK, box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

template <bool SWAP, bool SWIGLU, int R, int COLS>
static cudaError_t run(const Ctx& c, const void* act, int S, const void* w1, const void* w2, Args a,
                       int act_rows = -1) {
    set_wait_args(a);
    using C = Cfg<SWAP, SWIGLU, R, COLS>;
    auto kern = grouped_gemm_kernel<SWAP, SWIGLU, R, COLS>;
    static bool attr_done[64] = {};
    if (c.device < 0 || c.device >= 64) return cudaErrorInvalidDevice;
    if (!attr_done[c.device]) {
        cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
        if (err != cudaSuccess) return err;
        attr_done[c.device] = true;
    }
    CUtensorMap tm_act, tm_w1, tm_w2, tm_out;
    // act holds S permuted rows, or (with a.gather) act_rows rows read through the slot -> row map
    const uint64_t arows = act_rows >= 0 ? (uint64_t)act_rows : (uint64_t)S;
    if (arows == 0) return cudaErrorInvalidValue;
    if (!encode_2d(&tm_act, act, (uint64_t)a.K, arows, (uint32_t)R)) return cudaErrorInvalidValue;
    if (!encode_2d(&tm_w1, w1, (uint64_t)a.K, (uint64_t)a.E * a.n_out, (uint32_t)C::WBOX)) return cudaErrorInvalidValue;
    if (!encode_2d(&tm_w2, SWIGLU ? w2 : w1, (uint64_t)a.K, (uint64_t)a.E * a.n_out, (uint32_t)C::WBOX))
        return cudaErrorInvalidValue;
    // the output [S][ldo] in boxes of 64 columns x 32 rows (one epilogue warp's rows), 128-byte swizzle
    if (!encode_2d(&tm_out, a.out, (uint64_t)a.ldo, (uint64_t)S, 32)) return cudaErrorInvalidValue;
    // upper bound on the tile count: sum_e ceil(cnt_e / R) <= S / R + E
    const int64_t max_tiles = ((int64_t)S / R + a.E) * (a.n_out / COLS);
    const int grid = (int)(max_tiles < c.num_sms ? max_tiles : c.num_sms);
    if (grid <= 0) return cudaSuccess;
    return launch(kern, dim3(grid), dim3(threads_of<SWAP, SWIGLU, R>()), (size_t)C::SMEM, c, tm_act, tm_w1, tm_w2,
                  tm_out, a);
}

// Token rows staged per rows-as-M tile: the smallest of 16/32/64/128 that
// holds about three times the average rows per expert, so nearly every
// expert takes one row block and reads each weight tile once.
static int pick_rows(int S, int E) {
    const int64_t want = E > 0 ? 3 * ((int64_t)S + E - 1) / E : 0;
    if (want <= 16) return 16;
    if (want <= 32) return 32;
    if (want <= 64) return 64;
    return 128;
}

// Row block of the weights-as-M gate/up tile (about twice the average), or 0
// when experts average more than 32 rows and rows-as-M is used.
static int pick_swap_rows(int S, int E) {
    const int avg = E > 0 ? S / E : 0;
    if (avg <= 8) return 16;
    if (avg <= 16) return 32;
    if (avg <= 32) return 64;
    return 0;
}

}  // namespace tc

// Only the weights-as-M gate/up form (few rows per expert) gathers its rows in place: there a tile
// stages at most 64 rows per K slice, which four gather warps copy well within a stage's time.  For
// 128-row tiles gathering measured slower than copying the rows once with the permutation and
// reading the copy by TMA: prefill 11% slower with one warp per stage, and still ~5% slower with all
// four warps filling every stage two cp.async groups ahead, so those read the permuted copy.
bool gate_up_needs_permuted_rows(int S, int E) { return use_pair_gemm(S, E, 256) || tc::pick_swap_rows(S, E) == 0; }

cudaError_t launch_gate_up_bf16(const Ctx& c, const void* xp, const void* Wg, const void* Wu, const int32_t* counts,
                                const int32_t* offsets, int S, int E, int d, int d_ff, void* h, int32_t* status,
                                const int32_t* gather, int act_rows, int cap, int S_sel, bool raw,
                                int32_t* tile_ctr) {
    if (S == 0) return cudaSuccess;
    const int Ss = S_sel > 0 ? S_sel : S;  // rows the tile form is chosen for
    if (gather && (cap > 0 || gate_up_needs_permuted_rows(Ss, E))) return cudaErrorInvalidValue;
    if (cap == 0 && use_pair_gemm(Ss, E, 256))
        return launch_gate_up_bf16_pair(c, xp, Wg, Wu, counts, offsets, S, E, d, d_ff, h, status, raw);
    if (cap == 0 && !gather && use_dual_gemm(Ss, E, 256))
        return launch_gate_up_bf16_dual(c, xp, Wg, Wu, counts, offsets, S, E, d, d_ff, h, status, raw, tile_ctr);
    tc::Args a{counts, offsets, E, d, d_ff, static_cast<uint16_t*>(h), (int64_t)d_ff * (raw ? 2 : 1), status, gather,
               static_cast<const uint16_t*>(xp), cap, S, gather ? act_rows : 0};
    a.raw = raw ? 1 : 0;
    const int ar = gather ? act_rows : -1;
    switch (tc::pick_swap_rows(Ss, E)) {
        case 16: return tc::run<true, true, 16, 128>(c, xp, S, Wg, Wu, a, ar);
        case 32: return tc::run<true, true, 32, 128>(c, xp, S, Wg, Wu, a, ar);
        case 64: return tc::run<true, true, 64, 128>(c, xp, S, Wg, Wu, a, ar);
        default: break;
    }
    return tc::run<false, true, 128, 128>(c, xp, S, Wg, Wu, a, ar);  // above 32 rows per expert pick_rows() is 128
}

cudaError_t launch_down_bf16(const Ctx& c, const void* h, const void* Wd, const int32_t* counts, const int32_t* offsets,
                             int S, int E, int d, int d_ff, void* y, int32_t* status, int cap, int S_sel) {
    if (S == 0) return cudaSuccess;
    const int Ss = S_sel > 0 ? S_sel : S;
    if (cap == 0 && use_pair_gemm(Ss, E, d))
        return launch_down_bf16_pair(c, h, Wd, counts, offsets, S, E, d, d_ff, y, status);
    tc::Args a{counts, offsets, E, d_ff, d, static_cast<uint16_t*>(y), (int64_t)d, status, nullptr, nullptr, cap, S, 0};
    const int ra = tc::pick_rows(Ss, E);
    if (d % 256 == 0) {
        switch (ra) {
            case 16: return tc::run<false, false, 16, 256>(c, h, S, Wd, nullptr, a);
            case 32: return tc::run<false, false, 32, 256>(c, h, S, Wd, nullptr, a);
            case 64: return tc::run<false, false, 64, 256>(c, h, S, Wd, nullptr, a);
            default: return tc::run<false, false, 128, 256>(c, h, S, Wd, nullptr, a);
        }
    }
    switch (ra) {
        case 16: return tc::run<false, false, 16, 128>(c, h, S, Wd, nullptr, a);
        case 32: return tc::run<false, false, 32, 128>(c, h, S, Wd, nullptr, a);
        case 64: return tc::run<false, false, 64, 128>(c, h, S, Wd, nullptr, a);
        default: return tc::run<false, false, 128, 128>(c, h, S, Wd, nullptr, a);
    }
}

}  // namespace moe
