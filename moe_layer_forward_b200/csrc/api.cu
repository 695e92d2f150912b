// C ABI of libmoe.so (declared in include/moe.h): argument checks, workspace
// layout and the launch sequence of the MoE layer forward.  No entry point
// allocates, synchronises with the host, throws or aborts.
#include <stdint.h>
#include <string.h>

#include "kernels.h"
#include "moe.h"

namespace moe {
std::atomic<uint64_t> g_kernel_launches{0};
std::atomic<uint64_t> g_wait_limit_ns{0};
std::atomic<int> g_inject_stall{0};
}  // namespace moe

using namespace moe;

namespace {

constexpr int kMaxDevices = 64;

struct DevCache {
    int sms = 0;
    int major = 0;
};
DevCache g_dev[kMaxDevices];

moe_status_t make_ctx(moe_stream_t stream, Ctx& c) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return MOE_ERR_CUDA;
    }
    if (dev < 0 || dev >= kMaxDevices) return MOE_ERR_DEVICE;
    DevCache& dc = g_dev[dev];
    if (dc.sms == 0) {
        int sms = 0, major = 0;
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) {
            cudaGetLastError();
            return MOE_ERR_CUDA;
        }
        dc.major = major;
        dc.sms = sms;
    }
    if (dc.major != 10) return MOE_ERR_DEVICE;
    c.stream = reinterpret_cast<cudaStream_t>(stream);
    c.num_sms = dc.sms;
    c.device = dev;
    return MOE_OK;
}

moe_status_t cuda_status(cudaError_t e) {
    if (e == cudaSuccess) return MOE_OK;
    cudaGetLastError();  // clear the non-sticky error so the caller's next call is not affected
    return MOE_ERR_CUDA;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool valid_dt(moe_dtype_t t) { return t == MOE_F32 || t == MOE_BF16; }
size_t esize(moe_dtype_t t) { return t == MOE_BF16 ? 2 : 4; }

// bump allocator over the caller's workspace; with base == nullptr it only measures
struct Carve {
    uint8_t* base;
    size_t off = 0;
    explicit Carve(void* b) : base(static_cast<uint8_t*>(b)) {}
    void* take(size_t bytes) {
        const size_t o = (off + 255) & ~size_t(255);
        off = o + bytes;
        return base ? base + o : nullptr;
    }
};

moe_status_t check_ws(void* ws, size_t* ws_bytes, size_t need, bool* query_only) {
    *query_only = false;
    if (!ws_bytes) return MOE_ERR_INVALID_ARG;
    if (!ws) {
        *ws_bytes = need;
        *query_only = true;
        return MOE_OK;
    }
    if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return MOE_ERR_INVALID_ARG;
    if (*ws_bytes < need) {
        *ws_bytes = need;
        return MOE_ERR_WORKSPACE;
    }
    return MOE_OK;
}

moe_status_t check_router_shape(int T, int d, int E, int k) {
    if (T < 0 || d <= 0 || E <= 0 || k <= 0) return MOE_ERR_INVALID_ARG;
    if (k > MOE_MAX_TOP_K || E > MOE_MAX_EXPERTS || k > E) return MOE_ERR_UNSUPPORTED;
    if (d % 8 != 0) return MOE_ERR_UNSUPPORTED;
    return MOE_OK;
}

moe_status_t check_expert_shape(moe_dtype_t dt, int S, int E, int d, int d_ff) {
    if (S < 0 || E <= 0 || d <= 0 || d_ff <= 0) return MOE_ERR_INVALID_ARG;
    if (E > MOE_MAX_EXPERTS) return MOE_ERR_UNSUPPORTED;
    if (dt == MOE_BF16) {
        if (d % 128 != 0 || d_ff % 128 != 0) return MOE_ERR_UNSUPPORTED;
    } else if (dt == MOE_F32) {
        if (d % 8 != 0 || d_ff % 8 != 0) return MOE_ERR_UNSUPPORTED;
    } else {
        return MOE_ERR_INVALID_ARG;
    }
    return MOE_OK;
}

}  // namespace

extern "C" {

const char* moe_status_string(moe_status_t s) {
    switch (s) {
        case MOE_OK: return "ok";
        case MOE_ERR_INVALID_ARG: return "invalid argument";
        case MOE_ERR_UNSUPPORTED: return "unsupported shape or dtype";
        case MOE_ERR_WORKSPACE: return "workspace too small";
        case MOE_ERR_CUDA: return "CUDA error";
        case MOE_ERR_DEVICE: return "device is not sm_100";
    }
    return "unknown status";
}

int32_t moe_abi_version(void) { return MOE_ABI_VERSION; }

uint64_t moe_kernel_launches(void) { return moe::g_kernel_launches.load(std::memory_order_relaxed); }

void moe_set_wait_limit(uint64_t limit_ns, int32_t inject_stall) {
    moe::g_wait_limit_ns.store(limit_ns, std::memory_order_relaxed);
    moe::g_inject_stall.store(inject_stall != 0, std::memory_order_relaxed);
}

moe_status_t moe_rmsnorm(const void* x, moe_dtype_t x_dt, const float* gamma, int32_t T, int32_t d, float eps,
                         void* v, moe_dtype_t v_dt, moe_stream_t stream) {
    if (T < 0 || d <= 0 || !valid_dt(x_dt) || !valid_dt(v_dt)) return MOE_ERR_INVALID_ARG;
    if (d % 8 != 0) return MOE_ERR_UNSUPPORTED;
    if (T == 0) return MOE_OK;
    if (!x || !gamma || !v || !aligned16(x) || !aligned16(v) || !aligned16(gamma)) return MOE_ERR_INVALID_ARG;
    Ctx c;
    moe_status_t st = make_ctx(stream, c);
    if (st != MOE_OK) return st;
    return cuda_status(launch_rmsnorm(c, x, x_dt, gamma, T, d, eps, v, v_dt, nullptr));
}

moe_status_t moe_router_topk(const void* v, moe_dtype_t v_dt, const float* W_r, const float* b, int32_t T,
                             int32_t d, int32_t E, int32_t k, int32_t* topk_idx, float* topk_w, float* logits,
                             float* margin, void* ws, size_t* ws_bytes, moe_stream_t stream) {
    moe_status_t st = check_router_shape(T, d, E, k);
    if (st != MOE_OK) return st;
    if (!valid_dt(v_dt)) return MOE_ERR_INVALID_ARG;
    Ctx c;
    st = make_ctx(stream, c);
    if (st != MOE_OK) return st;
    const RouterPlan plan = plan_router(T, d, E, c.num_sms);
    Carve cv(nullptr);
    cv.take(plan.partial_bytes);
    cv.take(plan.wsplit_bytes);
    bool query = false;
    st = check_ws(ws, ws_bytes, cv.off, &query);
    if (st != MOE_OK || query || T == 0) return st;
    if (!v || !W_r || !b || !topk_idx || !topk_w || !aligned16(v) || !aligned16(W_r)) return MOE_ERR_INVALID_ARG;
    Carve w(ws);
    float* partial = static_cast<float*>(w.take(plan.partial_bytes));
    float* wsplit = static_cast<float*>(w.take(plan.wsplit_bytes));
    st = cuda_status(launch_router_logits(c, plan, v, v_dt, nullptr, nullptr, W_r, T, d, E, partial, wsplit, nullptr));
    if (st != MOE_OK) return st;
    return cuda_status(launch_router_topk(c, plan, partial, b, T, E, k, topk_idx, topk_w, logits, margin));
}

moe_status_t moe_route(const void* x, moe_dtype_t x_dt, const float* gamma, const float* W_r, const float* b,
                       int32_t T, int32_t d, int32_t E, int32_t k, float eps, int32_t* topk_idx, float* topk_w,
                       float* logits, float* margin, void* ws, size_t* ws_bytes, moe_stream_t stream) {
    moe_status_t st = check_router_shape(T, d, E, k);
    if (st != MOE_OK) return st;
    if (!valid_dt(x_dt)) return MOE_ERR_INVALID_ARG;
    Ctx c;
    st = make_ctx(stream, c);
    if (st != MOE_OK) return st;
    const RouterPlan plan = plan_router(T, d, E, c.num_sms);
    Carve cv(nullptr);
    cv.take((size_t)T * sizeof(float));
    cv.take(plan.partial_bytes);
    cv.take(plan.wsplit_bytes);
    bool query = false;
    st = check_ws(ws, ws_bytes, cv.off, &query);
    if (st != MOE_OK || query || T == 0) return st;
    if (!x || !gamma || !W_r || !b || !topk_idx || !topk_w || !aligned16(x) || !aligned16(gamma) || !aligned16(W_r))
        return MOE_ERR_INVALID_ARG;
    Carve w(ws);
    float* rstd = static_cast<float*>(w.take((size_t)T * sizeof(float)));
    float* partial = static_cast<float*>(w.take(plan.partial_bytes));
    float* wsplit = static_cast<float*>(w.take(plan.wsplit_bytes));
    // the same kernels, in the same order, as steps 1-2 of moe_forward (1/rms only: no normalised copy)
    st = cuda_status(launch_rmsnorm(c, x, x_dt, gamma, T, d, eps, nullptr, MOE_F32, rstd));
    if (st != MOE_OK) return st;
    st = cuda_status(launch_router_logits(c, plan, x, x_dt, rstd, gamma, W_r, T, d, E, partial, wsplit, nullptr));
    if (st != MOE_OK) return st;
    return cuda_status(launch_router_topk(c, plan, partial, b, T, E, k, topk_idx, topk_w, logits, margin));
}

moe_status_t moe_permute(const void* v, moe_dtype_t v_dt, const int32_t* topk_idx, int32_t T, int32_t d, int32_t E,
                         int32_t k, int32_t* counts, int32_t* offsets, int32_t* slot_token, int32_t* token_slot,
                         void* xp, void* ws, size_t* ws_bytes, int32_t* dev_status, moe_stream_t stream) {
    moe_status_t st = check_router_shape(T, d, E, k);
    if (st != MOE_OK) return st;
    if (!valid_dt(v_dt)) return MOE_ERR_INVALID_ARG;
    Carve cv(nullptr);
    cv.take(permute_ws_bytes(T, E));
    bool query = false;
    st = check_ws(ws, ws_bytes, cv.off, &query);
    if (st != MOE_OK || query) return st;
    if (!counts || !offsets) return MOE_ERR_INVALID_ARG;
    // xp == NULL: the maps only (a caller that moves the rows itself, e.g. moe_ep_dispatch)
    if (T > 0 && (!v || !topk_idx || !slot_token || !token_slot || !aligned16(v) || (xp && !aligned16(xp))))
        return MOE_ERR_INVALID_ARG;
    Ctx c;
    st = make_ctx(stream, c);
    if (st != MOE_OK) return st;
    Carve w(ws);
    int32_t* hist = static_cast<int32_t*>(w.take(permute_ws_bytes(T, E)));
    return cuda_status(launch_permute(c, v, v_dt, topk_idx, T, d, E, k, counts, offsets, slot_token, token_slot, xp,
                                      hist, dev_status));
}

moe_status_t moe_expert_gate_up(const void* xp, const void* W_gate, const void* W_up, moe_dtype_t dt,
                                const int32_t* counts, const int32_t* offsets, int32_t S, int32_t E, int32_t d,
                                int32_t d_ff, void* h, int32_t* dev_status, moe_stream_t stream) {
    moe_status_t st = check_expert_shape(dt, S, E, d, d_ff);
    if (st != MOE_OK) return st;
    if (S == 0) return MOE_OK;
    if (!xp || !W_gate || !W_up || !counts || !offsets || !h) return MOE_ERR_INVALID_ARG;
    if (!aligned16(xp) || !aligned16(W_gate) || !aligned16(W_up) || !aligned16(h)) return MOE_ERR_INVALID_ARG;
    Ctx c;
    st = make_ctx(stream, c);
    if (st != MOE_OK) return st;
    if (dt == MOE_BF16)
        return cuda_status(launch_gate_up_bf16(c, xp, W_gate, W_up, counts, offsets, S, E, d, d_ff, h, dev_status));
    return cuda_status(launch_gate_up_f32(c, static_cast<const float*>(xp), static_cast<const float*>(W_gate),
                                          static_cast<const float*>(W_up), counts, offsets, S, E, d, d_ff,
                                          static_cast<float*>(h), dev_status));
}

moe_status_t moe_expert_gate_up_raw(const void* xp, const void* W_gate, const void* W_up, const int32_t* counts,
                                    const int32_t* offsets, int32_t S, int32_t E, int32_t d, int32_t d_ff, void* gu,
                                    int32_t* dev_status, moe_stream_t stream) {
    moe_status_t st = check_expert_shape(MOE_BF16, S, E, d, d_ff);
    if (st != MOE_OK) return st;
    if (S == 0) return MOE_OK;
    if (!xp || !W_gate || !W_up || !counts || !offsets || !gu) return MOE_ERR_INVALID_ARG;
    if (!aligned16(xp) || !aligned16(W_gate) || !aligned16(W_up) || !aligned16(gu)) return MOE_ERR_INVALID_ARG;
    Ctx c;
    st = make_ctx(stream, c);
    if (st != MOE_OK) return st;
    return cuda_status(launch_gate_up_bf16(c, xp, W_gate, W_up, counts, offsets, S, E, d, d_ff, gu, dev_status,
                                           nullptr, 0, 0, 0, true));
}

moe_status_t moe_expert_down(const void* h, const void* W_down, moe_dtype_t dt, const int32_t* counts,
                             const int32_t* offsets, int32_t S, int32_t E, int32_t d, int32_t d_ff, void* y,
                             int32_t* dev_status, moe_stream_t stream) {
    moe_status_t st = check_expert_shape(dt, S, E, d, d_ff);
    if (st != MOE_OK) return st;
    if (S == 0) return MOE_OK;
    if (!h || !W_down || !counts || !offsets || !y) return MOE_ERR_INVALID_ARG;
    if (!aligned16(h) || !aligned16(W_down) || !aligned16(y)) return MOE_ERR_INVALID_ARG;
    Ctx c;
    st = make_ctx(stream, c);
    if (st != MOE_OK) return st;
    if (dt == MOE_BF16) return cuda_status(launch_down_bf16(c, h, W_down, counts, offsets, S, E, d, d_ff, y, dev_status));
    return cuda_status(launch_down_f32(c, static_cast<const float*>(h), static_cast<const float*>(W_down), counts,
                                       offsets, S, E, d, d_ff, static_cast<float*>(y), dev_status));
}

moe_status_t moe_grouped_swiglu(const void* xp, const void* W_gate, const void* W_up, const void* W_down,
                                moe_dtype_t dt, const int32_t* counts, const int32_t* offsets, int32_t S, int32_t E,
                                int32_t d, int32_t d_ff, void* h, void* y, int32_t* dev_status, moe_stream_t stream) {
    moe_status_t st = check_expert_shape(dt, S, E, d, d_ff);
    if (st != MOE_OK) return st;
    if (S > 0 && !W_down) return MOE_ERR_INVALID_ARG;
    st = moe_expert_gate_up(xp, W_gate, W_up, dt, counts, offsets, S, E, d, d_ff, h, dev_status, stream);
    if (st != MOE_OK) return st;
    return moe_expert_down(h, W_down, dt, counts, offsets, S, E, d, d_ff, y, dev_status, stream);
}

moe_status_t moe_grouped_swiglu_sized(const void* xp, const void* W_gate, const void* W_up, const void* W_down,
                                      moe_dtype_t dt, const int32_t* counts, const int32_t* offsets, int32_t S_cap,
                                      int32_t S_expected, int32_t E, int32_t d, int32_t d_ff, void* h, void* y,
                                      int32_t* dev_status, moe_stream_t stream) {
    moe_status_t st = check_expert_shape(dt, S_cap, E, d, d_ff);
    if (st != MOE_OK) return st;
    if (S_expected <= 0 || S_expected > S_cap) return MOE_ERR_INVALID_ARG;
    if (!xp || !W_gate || !W_up || !W_down || !counts || !offsets || !h || !y) return MOE_ERR_INVALID_ARG;
    if (!aligned16(xp) || !aligned16(W_gate) || !aligned16(W_up) || !aligned16(W_down) || !aligned16(h) ||
        !aligned16(y))
        return MOE_ERR_INVALID_ARG;
    Ctx c;
    st = make_ctx(stream, c);
    if (st != MOE_OK) return st;
    if (dt == MOE_BF16) {
        st = cuda_status(launch_gate_up_bf16(c, xp, W_gate, W_up, counts, offsets, S_cap, E, d, d_ff, h, dev_status,
                                             nullptr, 0, 0, S_expected));
        if (st != MOE_OK) return st;
        return cuda_status(
            launch_down_bf16(c, h, W_down, counts, offsets, S_cap, E, d, d_ff, y, dev_status, 0, S_expected));
    }
    st = cuda_status(launch_gate_up_f32(c, static_cast<const float*>(xp), static_cast<const float*>(W_gate),
                                        static_cast<const float*>(W_up), counts, offsets, S_cap, E, d, d_ff,
                                        static_cast<float*>(h), dev_status));
    if (st != MOE_OK) return st;
    return cuda_status(launch_down_f32(c, static_cast<const float*>(h), static_cast<const float*>(W_down), counts,
                                       offsets, S_cap, E, d, d_ff, static_cast<float*>(y), dev_status));
}

moe_status_t moe_grouped_swiglu_masked(const void* x, const void* W_gate, const void* W_up, const void* W_down,
                                       moe_dtype_t dt, const int32_t* counts, int32_t E, int32_t cap, int32_t d,
                                       int32_t d_ff, void* h, void* y, int32_t* dev_status, moe_stream_t stream) {
    if (cap <= 0 || E <= 0 || (int64_t)E * cap >= (int64_t(1) << 30)) return MOE_ERR_INVALID_ARG;
    const int S = E * cap;
    moe_status_t st = check_expert_shape(dt, S, E, d, d_ff);
    if (st != MOE_OK) return st;
    if (dt != MOE_BF16) return MOE_ERR_UNSUPPORTED;
    if (!x || !W_gate || !W_up || !W_down || !counts || !h || !y) return MOE_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(W_gate) || !aligned16(W_up) || !aligned16(W_down) || !aligned16(h) ||
        !aligned16(y))
        return MOE_ERR_INVALID_ARG;
    Ctx c;
    st = make_ctx(stream, c);
    if (st != MOE_OK) return st;
    st = cuda_status(launch_gate_up_bf16(c, x, W_gate, W_up, counts, nullptr, S, E, d, d_ff, h, dev_status, nullptr, 0,
                                         cap));
    if (st != MOE_OK) return st;
    return cuda_status(launch_down_bf16(c, h, W_down, counts, nullptr, S, E, d, d_ff, y, dev_status, cap));
}

moe_status_t moe_unpermute_combine(const void* y, moe_dtype_t y_dt, const int32_t* token_slot, const float* topk_w,
                                   const void* residual, moe_dtype_t r_dt, int32_t T, int32_t d, int32_t k, void* out,
                                   moe_dtype_t out_dt, moe_stream_t stream) {
    if (T < 0 || d <= 0 || k <= 0 || !valid_dt(y_dt) || !valid_dt(r_dt) || !valid_dt(out_dt))
        return MOE_ERR_INVALID_ARG;
    if (k > MOE_MAX_TOP_K || d % 8 != 0) return MOE_ERR_UNSUPPORTED;
    if (T == 0) return MOE_OK;
    if (!y || !token_slot || !topk_w || !residual || !out) return MOE_ERR_INVALID_ARG;
    if (!aligned16(y) || !aligned16(residual) || !aligned16(out)) return MOE_ERR_INVALID_ARG;
    Ctx c;
    moe_status_t st = make_ctx(stream, c);
    if (st != MOE_OK) return st;
    return cuda_status(launch_combine(c, y, y_dt, token_slot, topk_w, residual, r_dt, T, d, k, out, out_dt));
}

// ----------------------------------------------------------------------------- expert parallelism over peer memory
namespace {
moe_status_t check_ep(int32_t rank, int32_t N, int32_t E, int32_t T, int32_t d, int32_t k, const int32_t* table) {
    if (N <= 0 || rank < 0 || rank >= N || E <= 0 || T < 0 || d <= 0 || k <= 0 || !table) return MOE_ERR_INVALID_ARG;
    if (E % N != 0 || E > MOE_MAX_EXPERTS || k > MOE_MAX_TOP_K || d % 8 != 0 || N > MOE_MAX_EP_RANKS)
        return MOE_ERR_UNSUPPORTED;
    return MOE_OK;
}
}  // namespace

moe_status_t moe_ep_dispatch(const void* v, moe_dtype_t v_dt, const int32_t* topk_idx, const int32_t* token_slot,
                             const int32_t* offsets, const int32_t* count_table, int32_t rank, int32_t N, int32_t E,
                             int32_t T, int32_t d, int32_t k, void* const* recv_bufs, int64_t recv_rows,
                             int32_t* dev_status, moe_stream_t stream) {
    if (!valid_dt(v_dt) || recv_rows < 0) return MOE_ERR_INVALID_ARG;
    moe_status_t st = check_ep(rank, N, E, T, d, k, count_table);
    if (st != MOE_OK) return st;
    if (T == 0) return MOE_OK;
    if (!v || !topk_idx || !token_slot || !offsets || !recv_bufs || !aligned16(v)) return MOE_ERR_INVALID_ARG;
    Ctx c;
    st = make_ctx(stream, c);
    if (st != MOE_OK) return st;
    return cuda_status(launch_ep_dispatch(c, v, v_dt, topk_idx, token_slot, offsets, count_table, rank, N, E, T, d, k,
                                          recv_bufs, recv_rows, dev_status));
}

moe_status_t moe_ep_layout(const int32_t* count_table, int32_t rank, int32_t N, int32_t E, int32_t* counts_loc,
                           int32_t* offsets_loc, moe_stream_t stream) {
    moe_status_t st = check_ep(rank, N, E, 0, 8, 1, count_table);
    if (st != MOE_OK) return st;
    if (!counts_loc || !offsets_loc) return MOE_ERR_INVALID_ARG;
    Ctx c;
    st = make_ctx(stream, c);
    if (st != MOE_OK) return st;
    return cuda_status(launch_ep_layout(c, count_table, rank, N, E, counts_loc, offsets_loc));
}

moe_status_t moe_ep_combine(const void* const* y_bufs, moe_dtype_t y_dt, const int32_t* topk_idx,
                            const int32_t* token_slot, const int32_t* offsets, const int32_t* count_table,
                            int32_t rank, int32_t N, int32_t E, const float* topk_w, const void* residual,
                            moe_dtype_t r_dt, int32_t T, int32_t d, int32_t k, void* out, moe_dtype_t out_dt,
                            int64_t recv_rows, int32_t* dev_status, moe_stream_t stream) {
    if (!valid_dt(y_dt) || !valid_dt(r_dt) || !valid_dt(out_dt) || recv_rows < 0) return MOE_ERR_INVALID_ARG;
    moe_status_t st = check_ep(rank, N, E, T, d, k, count_table);
    if (st != MOE_OK) return st;
    if (T == 0) return MOE_OK;
    if (!y_bufs || !topk_idx || !token_slot || !offsets || !topk_w || !residual || !out) return MOE_ERR_INVALID_ARG;
    if (!aligned16(residual) || !aligned16(out)) return MOE_ERR_INVALID_ARG;
    Ctx c;
    st = make_ctx(stream, c);
    if (st != MOE_OK) return st;
    return cuda_status(launch_ep_combine(c, y_bufs, y_dt, topk_idx, token_slot, offsets, count_table, rank, N, E,
                                         topk_w, residual, r_dt, T, d, k, out, out_dt, recv_rows, dev_status));
}

moe_status_t moe_forward(const moe_shape_t* shape, const moe_weights_t* wts, const void* x, void* out,
                         int32_t* topk_idx, float* topk_w, float* logits, void* ws, size_t* ws_bytes,
                         int32_t* dev_status, moe_stream_t stream) {
    if (!shape || !wts || !ws_bytes) return MOE_ERR_INVALID_ARG;
    const int T = shape->T, d = shape->d, E = shape->E, k = shape->top_k, d_ff = shape->d_ff;
    if (!valid_dt(shape->x_dtype) || !valid_dt(shape->w_dtype) || !valid_dt(shape->out_dtype))
        return MOE_ERR_INVALID_ARG;
    moe_status_t st = check_router_shape(T, d, E, k);
    if (st != MOE_OK) return st;
    const moe_dtype_t wdt = shape->w_dtype;
    if ((int64_t)T * k > INT32_MAX / 2) return MOE_ERR_UNSUPPORTED;
    const int S = T * k;
    st = check_expert_shape(wdt, S, E, d, d_ff);
    if (st != MOE_OK) return st;
    Ctx c;
    st = make_ctx(stream, c);
    if (st != MOE_OK) return st;
    const RouterPlan plan = plan_router(T, d, E, c.num_sms);
    const size_t es = esize(wdt);

    // workspace layout (each piece 256-byte aligned)
    Carve cv(ws);
    void* v = cv.take((size_t)T * d * es);
    float* rstd = static_cast<float*>(cv.take((size_t)T * sizeof(float)));
    float* partial = static_cast<float*>(cv.take(plan.partial_bytes));
    float* wsplit = static_cast<float*>(cv.take(plan.wsplit_bytes));
    // routing is kept in the workspace unless the caller asks for it (the size never depends on that)
    int32_t* idx_ws = static_cast<int32_t*>(cv.take((size_t)S * sizeof(int32_t)));
    float* wgt_ws = static_cast<float*>(cv.take((size_t)S * sizeof(float)));
    int32_t* idx = topk_idx ? topk_idx : idx_ws;
    float* wgt = topk_w ? topk_w : wgt_ws;
    int32_t* hist = static_cast<int32_t*>(cv.take(permute_ws_bytes(T, E)));
    int32_t* counts = static_cast<int32_t*>(cv.take((size_t)E * sizeof(int32_t)));
    int32_t* offsets = static_cast<int32_t*>(cv.take((size_t)(E + 1) * sizeof(int32_t)));
    int32_t* slot_token = static_cast<int32_t*>(cv.take((size_t)S * sizeof(int32_t)));
    int32_t* token_slot = static_cast<int32_t*>(cv.take((size_t)S * sizeof(int32_t)));
    // bf16 experts on one-CTA tiles read their rows straight from v through slot_token; only the
    // fp32 path and the CTA-pair tiles need the permuted copy Xp
    const bool fused_gather = wdt == MOE_BF16 && !gate_up_needs_permuted_rows(S, E);
    void* xp = fused_gather ? nullptr : cv.take((size_t)S * d * es);
    void* h = cv.take((size_t)S * d_ff * es);
    void* y = cv.take((size_t)S * d * es);
    // the tile counter of the gate/up GEMM's dynamic schedule (two-row-block tiles), zeroed per call
    int32_t* tile_ctr = static_cast<int32_t*>(cv.take(sizeof(int32_t)));
    bool query = false;
    st = check_ws(ws, ws_bytes, cv.off, &query);
    if (st != MOE_OK || query) return st;

    const bool need_w = T > 0;
    if (need_w && (!x || !out || !wts->gamma || !wts->W_r || !wts->b || !wts->W_gate || !wts->W_up || !wts->W_down))
        return MOE_ERR_INVALID_ARG;
    if (need_w && (!aligned16(x) || !aligned16(out) || !aligned16(wts->gamma) || !aligned16(wts->W_r) ||
                   !aligned16(wts->W_gate) || !aligned16(wts->W_up) || !aligned16(wts->W_down)))
        return MOE_ERR_INVALID_ARG;

    if (dev_status) {
        st = cuda_status(cudaMemsetAsync(dev_status, 0, sizeof(int32_t), c.stream));
        if (st != MOE_OK) return st;
    }
    if (T == 0) return MOE_OK;
    st = cuda_status(cudaMemsetAsync(tile_ctr, 0, sizeof(int32_t), c.stream));
    if (st != MOE_OK) return st;
    const int xdt = shape->x_dtype;
    // 1. RMSNorm: v rounded to the expert dtype, and 1/rms for the router
    st = cuda_status(launch_rmsnorm(c, x, xdt, wts->gamma, T, d, shape->eps, v, wdt, rstd));
    if (st != MOE_OK) return st;
    // 2. router on the unrounded fp32 normalised rows (x * rstd * gamma formed in the GEMM)
    st = cuda_status(
        launch_router_logits(c, plan, x, xdt, rstd, wts->gamma, wts->W_r, T, d, E, partial, wsplit, dev_status));
    if (st != MOE_OK) return st;
    st = cuda_status(launch_router_topk(c, plan, partial, wts->b, T, E, k, idx, wgt, logits, nullptr));
    if (st != MOE_OK) return st;
    // 3. permutation
    st = cuda_status(launch_permute(c, v, wdt, idx, T, d, E, k, counts, offsets, slot_token, token_slot, xp, hist,
                                    dev_status));
    if (st != MOE_OK) return st;
    // 4. grouped SwiGLU MLP
    if (wdt == MOE_BF16) {
        st = cuda_status(launch_gate_up_bf16(c, fused_gather ? v : xp, wts->W_gate, wts->W_up, counts, offsets, S, E,
                                             d, d_ff, h, dev_status, fused_gather ? slot_token : nullptr, T, 0, 0, false,
                                             tile_ctr));
        if (st != MOE_OK) return st;
        st = cuda_status(launch_down_bf16(c, h, wts->W_down, counts, offsets, S, E, d, d_ff, y, dev_status));
    } else {
        st = cuda_status(launch_gate_up_f32(c, static_cast<const float*>(xp), static_cast<const float*>(wts->W_gate),
                                            static_cast<const float*>(wts->W_up), counts, offsets, S, E, d, d_ff,
                                            static_cast<float*>(h), dev_status));
        if (st != MOE_OK) return st;
        st = cuda_status(launch_down_f32(c, static_cast<const float*>(h), static_cast<const float*>(wts->W_down),
                                         counts, offsets, S, E, d, d_ff, static_cast<float*>(y), dev_status));
    }
    if (st != MOE_OK) return st;
    // 5. weighted un-permute + residual
    return cuda_status(launch_combine(c, y, wdt, token_slot, wgt, x, xdt, T, d, k, out, shape->out_dtype));
}


// ----------------------------------------------------------------------------- block FP8
moe_status_t moe_quantize_fp8(const void* x, moe_dtype_t dt, int64_t rows, int64_t cols, int32_t blk_rows, uint8_t* q,
                              float* s, moe_stream_t stream) {
    if (!valid_dt(dt) || rows < 0 || cols <= 0 || (blk_rows != 1 && blk_rows != 128)) return MOE_ERR_INVALID_ARG;
    if (cols % 128 != 0 || rows * cols >= (int64_t(1) << 40)) return MOE_ERR_UNSUPPORTED;
    if (rows == 0) return MOE_OK;
    if (!x || !q || !s || !aligned16(x) || !aligned16(q)) return MOE_ERR_INVALID_ARG;
    Ctx c;
    moe_status_t st = make_ctx(stream, c);
    if (st != MOE_OK) return st;
    return cuda_status(launch_quant_fp8(c, x, dt, rows, cols, blk_rows, q, s));
}

namespace {
moe_status_t check_fp8_weights(const moe_weights_fp8_t* w) {
    if (!w || !w->W_gate_q || !w->W_gate_s || !w->W_up_q || !w->W_up_s || !w->W_down_q || !w->W_down_s)
        return MOE_ERR_INVALID_ARG;
    if (!aligned16(w->W_gate_q) || !aligned16(w->W_up_q) || !aligned16(w->W_down_q)) return MOE_ERR_INVALID_ARG;
    return MOE_OK;
}
}  // namespace

moe_status_t moe_grouped_swiglu_fp8(const uint8_t* xq, const float* xs, const moe_weights_fp8_t* w,
                                    const int32_t* counts, const int32_t* offsets, int32_t S, int32_t E, int32_t d,
                                    int32_t d_ff, uint8_t* hq, float* hs, void* y, int32_t* dev_status,
                                    moe_stream_t stream) {
    moe_status_t st = check_expert_shape(MOE_BF16, S, E, d, d_ff);
    if (st != MOE_OK) return st;
    if (S == 0) return MOE_OK;
    st = check_fp8_weights(w);
    if (st != MOE_OK) return st;
    if (!xq || !xs || !counts || !offsets || !hq || !hs || !y || !aligned16(xq) || !aligned16(hq) || !aligned16(y))
        return MOE_ERR_INVALID_ARG;
    Ctx c;
    st = make_ctx(stream, c);
    if (st != MOE_OK) return st;
    st = cuda_status(launch_gate_up_fp8(c, xq, xs, nullptr, w->W_gate_q, w->W_gate_s, w->W_up_q, w->W_up_s, counts,
                                        offsets, S, E, d, d_ff, hq, hs, dev_status, S));
    if (st != MOE_OK) return st;
    return cuda_status(
        launch_down_fp8(c, hq, hs, w->W_down_q, w->W_down_s, counts, offsets, S, E, d, d_ff, y, dev_status));
}

moe_status_t moe_forward_fp8(const moe_shape_t* shape, const moe_weights_fp8_t* w, const void* x, void* out,
                             int32_t* topk_idx, float* topk_w, float* logits, void* ws, size_t* ws_bytes,
                             int32_t* dev_status, moe_stream_t stream) {
    if (!shape || !w || !ws_bytes) return MOE_ERR_INVALID_ARG;
    const int T = shape->T, d = shape->d, E = shape->E, k = shape->top_k, d_ff = shape->d_ff;
    if (!valid_dt(shape->x_dtype) || !valid_dt(shape->out_dtype)) return MOE_ERR_INVALID_ARG;
    moe_status_t st = check_router_shape(T, d, E, k);
    if (st != MOE_OK) return st;
    if ((int64_t)T * k > INT32_MAX / 2) return MOE_ERR_UNSUPPORTED;
    const int S = T * k;
    st = check_expert_shape(MOE_BF16, S, E, d, d_ff);
    if (st != MOE_OK) return st;
    Ctx c;
    st = make_ctx(stream, c);
    if (st != MOE_OK) return st;
    const RouterPlan plan = plan_router(T, d, E, c.num_sms);

    Carve cv(ws);
    uint8_t* vq = static_cast<uint8_t*>(cv.take((size_t)T * d));
    float* vs = static_cast<float*>(cv.take((size_t)T * (d / 128) * sizeof(float)));
    float* rstd = static_cast<float*>(cv.take((size_t)T * sizeof(float)));
    float* partial = static_cast<float*>(cv.take(plan.partial_bytes));
    float* wsplit = static_cast<float*>(cv.take(plan.wsplit_bytes));
    int32_t* idx_ws = static_cast<int32_t*>(cv.take((size_t)S * sizeof(int32_t)));
    float* wgt_ws = static_cast<float*>(cv.take((size_t)S * sizeof(float)));
    int32_t* idx = topk_idx ? topk_idx : idx_ws;
    float* wgt = topk_w ? topk_w : wgt_ws;
    int32_t* hist = static_cast<int32_t*>(cv.take(permute_ws_bytes(T, E)));
    int32_t* counts = static_cast<int32_t*>(cv.take((size_t)E * sizeof(int32_t)));
    int32_t* offsets = static_cast<int32_t*>(cv.take((size_t)(E + 1) * sizeof(int32_t)));
    int32_t* slot_token = static_cast<int32_t*>(cv.take((size_t)S * sizeof(int32_t)));
    int32_t* token_slot = static_cast<int32_t*>(cv.take((size_t)S * sizeof(int32_t)));
    uint8_t* hq = static_cast<uint8_t*>(cv.take((size_t)S * d_ff));
    float* hs = static_cast<float*>(cv.take((size_t)S * (d_ff / 128) * sizeof(float)));
    void* y = cv.take((size_t)S * d * 2);
    bool query = false;
    st = check_ws(ws, ws_bytes, cv.off, &query);
    if (st != MOE_OK || query) return st;

    if (T > 0) {
        if (!x || !out || !w->gamma || !w->W_r || !w->b) return MOE_ERR_INVALID_ARG;
        if (!aligned16(x) || !aligned16(out) || !aligned16(w->gamma) || !aligned16(w->W_r)) return MOE_ERR_INVALID_ARG;
        st = check_fp8_weights(w);
        if (st != MOE_OK) return st;
    }
    if (dev_status) {
        st = cuda_status(cudaMemsetAsync(dev_status, 0, sizeof(int32_t), c.stream));
        if (st != MOE_OK) return st;
    }
    if (T == 0) return MOE_OK;
    const int xdt = shape->x_dtype;
    // 1. RMSNorm: codes of the normalised rows for the experts, 1/rms for the router
    st = cuda_status(launch_rmsnorm_quant(c, x, xdt, w->gamma, T, d, shape->eps, vq, vs, rstd));
    if (st != MOE_OK) return st;
    // 2. router on the unrounded fp32 normalised rows
    st = cuda_status(
        launch_router_logits(c, plan, x, xdt, rstd, w->gamma, w->W_r, T, d, E, partial, wsplit, dev_status));
    if (st != MOE_OK) return st;
    st = cuda_status(launch_router_topk(c, plan, partial, w->b, T, E, k, idx, wgt, logits, nullptr));
    if (st != MOE_OK) return st;
    // 3. permutation maps only: the gate/up GEMM reads the code rows in place
    st = cuda_status(launch_permute(c, nullptr, MOE_BF16, idx, T, d, E, k, counts, offsets, slot_token, token_slot,
                                    nullptr, hist, dev_status));
    if (st != MOE_OK) return st;
    // 4. block-FP8 SwiGLU MLP
    st = cuda_status(launch_gate_up_fp8(c, vq, vs, slot_token, w->W_gate_q, w->W_gate_s, w->W_up_q, w->W_up_s, counts,
                                        offsets, S, E, d, d_ff, hq, hs, dev_status, T));
    if (st != MOE_OK) return st;
    st = cuda_status(
        launch_down_fp8(c, hq, hs, w->W_down_q, w->W_down_s, counts, offsets, S, E, d, d_ff, y, dev_status));
    if (st != MOE_OK) return st;
    // 5. weighted un-permute + residual
    return cuda_status(launch_combine(c, y, MOE_BF16, token_slot, wgt, x, xdt, T, d, k, out, shape->out_dtype));
}

}  // extern "C"
