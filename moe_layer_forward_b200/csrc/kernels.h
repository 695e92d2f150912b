// Host-side launchers of the MoE layer kernels (internal to libmoe.so).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <atomic>
#include <utility>

namespace moe {

// Kernels this library has enqueued in this process (successful launches only).
extern std::atomic<uint64_t> g_kernel_launches;

// Bounded waits of the tensor-core kernels, for launches queued from now on: the limit of one wait in
// ns (0 = the kernels' default), and the failure-path test switch that makes each kernel's epilogue wait
// once on a barrier that nothing completes (set through moe_set_wait_limit).
extern std::atomic<uint64_t> g_wait_limit_ns;
extern std::atomic<int> g_inject_stall;
template <typename A>
inline void set_wait_args(A& a) {
    const uint64_t ns = g_wait_limit_ns.load(std::memory_order_relaxed);
    if (ns != 0) a.wait_ns = ns;
    a.stall = g_inject_stall.load(std::memory_order_relaxed);
}

struct Ctx {
    cudaStream_t stream;
    int num_sms;
    int device;
};

// Every kernel is launched with programmatic stream serialisation; each one
// executes griddepcontrol.wait before it touches global memory, so it never
// reads a predecessor's output early, and triggers its dependents as soon as
// its own prologue is done.
template <typename... KArgs, typename... Args>
cudaError_t launch(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, const Ctx& c, Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = c.stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t err = cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
    if (err == cudaSuccess) g_kernel_launches.fetch_add(1, std::memory_order_relaxed);
    return err;
}

// ---- step 1: RMSNorm (norm_router.cu)
cudaError_t launch_rmsnorm(const Ctx& c, const void* x, int x_dt, const float* gamma, int T, int d, float eps, void* v,
                           int v_dt, float* rstd);

// ---- step 2: router (router_tc.cu: logits on tensor cores; norm_router.cu: top-k)
struct RouterPlan {
    int splitk;           // K split of the logits GEMM
    int kchunk;           // K extent of one split (multiple of 32)
    size_t partial_bytes; // [splitk][T][E] fp32 partial logits
    size_t wsplit_bytes;  // W_r split into tf32 hi / lo terms
};
RouterPlan plan_router(int T, int d, int E, int num_sms);
// A operand: v (a_dt) when rstd == nullptr, else x (a_dt) * rstd[t] * gamma[j]
cudaError_t launch_router_logits(const Ctx& c, const RouterPlan& p, const void* a, int a_dt, const float* rstd,
                                 const float* gamma, const float* W_r, int T, int d, int E, float* partial,
                                 float* wsplit, int32_t* status);
// bf16 x with rstd (d % 128 == 0): z = rstd * (x (gamma ⊙ W_r)^T) with gamma ⊙ W_r split exactly into three
// bf16 terms (router_x3.cu); ws holds the split weights (3 E d bf16, within wsplit_bytes)
cudaError_t launch_router_logits_x3(const Ctx& c, const RouterPlan& p, const void* x, const float* rstd,
                                    const float* gamma, const float* W_r, int T, int d, int E, int np,
                                    float* partial, void* ws, int32_t* status);
cudaError_t launch_router_topk(const Ctx& c, const RouterPlan& p, const float* partial, const float* b, int T, int E,
                               int k, int32_t* idx, float* w, float* logits, float* margin);

// ---- step 3: permutation (permute.cu)
constexpr int kPermuteChunk = 256;
inline size_t permute_ws_bytes(int T, int E) {
    size_t nchunks = (size_t)(T + kPermuteChunk - 1) / kPermuteChunk;
    return nchunks * (size_t)E * sizeof(int32_t);
}
// xp == nullptr: only the maps (counts, offsets, slot_token, token_slot), no row copy
cudaError_t launch_permute(const Ctx& c, const void* v, int v_dt, const int32_t* idx, int T, int d, int E, int k,
                           int32_t* counts, int32_t* offsets, int32_t* slot_token, int32_t* token_slot, void* xp,
                           int32_t* hist, int32_t* status);

// ---- steps 3 and 5 with expert parallelism over peer memory (ep_p2p.cu)
// table [N][E]: rows every rank routes to every expert; recv / y: device arrays of N peer pointers
cudaError_t launch_ep_dispatch(const Ctx& c, const void* v, int v_dt, const int32_t* idx, const int32_t* token_slot,
                               const int32_t* offsets, const int32_t* table, int rank, int N, int E, int T, int d,
                               int k, void* const* recv, int64_t recv_rows, int32_t* status);
cudaError_t launch_ep_layout(const Ctx& c, const int32_t* table, int rank, int N, int E, int32_t* counts_loc,
                             int32_t* offsets_loc);
cudaError_t launch_ep_combine(const Ctx& c, const void* const* y, int y_dt, const int32_t* idx,
                              const int32_t* token_slot, const int32_t* offsets, const int32_t* table, int rank, int N,
                              int E, const float* w, const void* res, int r_dt, int T, int d, int k, void* out,
                              int out_dt, int64_t recv_rows, int32_t* status);

// ---- step 4: expert MLP (expert_tc.cu: bf16 tensor cores; expert_simt.cu: fp32)
// gate/up: xp holds the S permuted rows; or, with gather, xp holds act_rows rows and slot i
// reads row gather[i] (the permutation's slot -> token map), so no permuted copy is made.
// The CTA-pair kernel needs the permuted copy (gate_up_needs_permuted_rows()).
bool gate_up_needs_permuted_rows(int S, int E);
// cap > 0 selects the masked layout: S = E * cap rows, expert e owns rows [e*cap, e*cap + counts[e])
// and offsets is ignored (one-CTA kernels only).  S_sel > 0: the tile form is chosen for S_sel rows
// while the buffers hold S (the row count on the device decides the work either way).
cudaError_t launch_gate_up_bf16(const Ctx& c, const void* xp, const void* Wg, const void* Wu, const int32_t* counts,
                                const int32_t* offsets, int S, int E, int d, int d_ff, void* h, int32_t* status,
                                const int32_t* gather = nullptr, int act_rows = 0, int cap = 0, int S_sel = 0,
                                bool raw = false, int32_t* tile_ctr = nullptr);
cudaError_t launch_down_bf16(const Ctx& c, const void* h, const void* Wd, const int32_t* counts, const int32_t* offsets,
                             int S, int E, int d, int d_ff, void* y, int32_t* status, int cap = 0, int S_sel = 0);
// CTA-pair (cta_group::2) variants for experts with many rows each (expert_tc2.cu)
bool use_pair_gemm(int S, int E, int n_out);
cudaError_t launch_gate_up_bf16_pair(const Ctx& c, const void* xp, const void* Wg, const void* Wu,
                                     const int32_t* counts, const int32_t* offsets, int S, int E, int d, int d_ff,
                                     void* h, int32_t* status, bool raw = false);
cudaError_t launch_down_bf16_pair(const Ctx& c, const void* h, const void* Wd, const int32_t* counts,
                                  const int32_t* offsets, int S, int E, int d, int d_ff, void* y, int32_t* status);
// Gate/up tiles of two 128-row blocks of one expert sharing each staged weight slice, one CTA
// (expert_tc_dual.cu), for experts averaging 256 rows up to the CTA-pair range.  tile_ctr (one int, zero
// before the launch) gives a dynamic schedule; null, CTA-strided tiles.
bool use_dual_gemm(int S, int E, int n_out);
cudaError_t launch_gate_up_bf16_dual(const Ctx& c, const void* xp, const void* Wg, const void* Wu,
                                     const int32_t* counts, const int32_t* offsets, int S, int E, int d, int d_ff,
                                     void* h, int32_t* status, bool raw, int32_t* tile_ctr);
// Block-FP8 experts (expert_fp8.cu): E4M3 codes, fp32 scales per 128 x 128 weight block and per
// (row, 128 columns) of a GEMM input
cudaError_t launch_quant_fp8(const Ctx& c, const void* x, int dt, int64_t rows, int64_t cols, int blk_rows,
                             uint8_t* q, float* s);
cudaError_t launch_rmsnorm_quant(const Ctx& c, const void* x, int x_dt, const float* gamma, int T, int d, float eps,
                                 uint8_t* q, float* s, float* rstd);
cudaError_t launch_gate_up_fp8(const Ctx& c, const uint8_t* xq, const float* xs, const int32_t* gather,
                               const uint8_t* Wg, const float* Wg_s, const uint8_t* Wu, const float* Wu_s,
                               const int32_t* counts, const int32_t* offsets, int S, int E, int d, int d_ff,
                               uint8_t* hq, float* hs, int32_t* status, int act_rows);
cudaError_t launch_down_fp8(const Ctx& c, const uint8_t* hq, const float* hs, const uint8_t* Wd, const float* Wd_s,
                            const int32_t* counts, const int32_t* offsets, int S, int E, int d, int d_ff, void* y,
                            int32_t* status);
cudaError_t launch_gate_up_f32(const Ctx& c, const float* xp, const float* Wg, const float* Wu, const int32_t* counts,
                               const int32_t* offsets, int S, int E, int d, int d_ff, float* h, int32_t* status);
cudaError_t launch_down_f32(const Ctx& c, const float* h, const float* Wd, const int32_t* counts,
                            const int32_t* offsets, int S, int E, int d, int d_ff, float* y, int32_t* status);

// ---- step 5: weighted un-permute + residual (combine.cu)
cudaError_t launch_combine(const Ctx& c, const void* y, int y_dt, const int32_t* token_slot, const float* w,
                           const void* res, int r_dt, int T, int d, int k, void* out, int out_dt);

}  // namespace moe
