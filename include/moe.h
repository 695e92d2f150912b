/*
 * moe.h — C ABI of libmoe.so: forward pass of one Mixture-of-Experts
 * feed-forward layer on one NVIDIA B200 (sm_100a).
 *
 *   R = X + MoE(RMSNorm(X))
 *
 * Sources (web pages on MoE inference; each entry point cites its passage):
 *   [P1] "推理计算流梳理" (huanyp.cn) — §Norm&Residual, §实际 MLP 计算策略,
 *        §专家并行 / MoE Router 过程, §EP 路径.
 *   [P5] "「赤兔」Chitu 框架深度解读（七）：混合专家模型 (MoE) 的高效处理" —
 *        §Token 分发策略 (MoETokenDispatcher: token_permutation /
 *        token_unpermutation), §专家计算实现 (BatchedExperts; tokens laid out
 *        contiguously by expert id for the grouped GEMM).
 *
 * Conventions shared by every entry point
 *   - Pointers named as tensors are DEVICE pointers owned by the caller; the
 *     library never allocates, frees or keeps them.  Host pointers are only
 *     the small structs (moe_shape_t, moe_weights_t) and size_t* ws_bytes.
 *   - Layouts are row-major with the last index contiguous.  Weights are
 *     stored out x in: W_r [E][d], W_gate/W_up [E][d_ff][d], W_down [E][d][d_ff].
 *   - Work is queued on `stream` and never synchronised with the host.
 *   - Workspace: pass ws == NULL to have the size needed written to *ws_bytes
 *     (returns MOE_OK, queues nothing).  A buffer smaller than needed gives
 *     MOE_ERR_WORKSPACE with the needed size in *ws_bytes.  ws must be 256-byte
 *     aligned and must not be used by other work until the queued work ends.
 *   - Arguments are validated on the host before anything is queued; on any
 *     error nothing is queued.  No entry point throws, aborts or prints.
 *   - Errors found by kernels (bad expert ids, a bounded wait that gave up)
 *     are OR-ed as MOE_DEV_* bits into *dev_status when dev_status != NULL.
 *   - T == 0 is valid and queues nothing (moe_forward still clears dev_status).
 */
#ifndef MOE_H
#define MOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t (NULL = the legacy default stream). */
typedef struct CUstream_st* moe_stream_t;

typedef enum { MOE_F32 = 0, MOE_BF16 = 1 } moe_dtype_t;

typedef enum {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = 1, /* null pointer, negative or inconsistent size, misaligned pointer */
    MOE_ERR_UNSUPPORTED = 2, /* well-formed but outside what the kernels support (see each call) */
    MOE_ERR_WORKSPACE = 3,   /* workspace too small; *ws_bytes holds the size needed */
    MOE_ERR_CUDA = 4,        /* a CUDA runtime call or a kernel launch failed */
    MOE_ERR_DEVICE = 5       /* the current device is not sm_100 */
} moe_status_t;

/* bits OR-ed into *dev_status by kernels */
#define MOE_DEV_BAD_EXPERT_ID 1 /* topk_idx held an id outside [0, E); that pair was dropped */
#define MOE_DEV_TIMEOUT 2       /* a bounded in-kernel wait gave up; outputs are not valid */
#define MOE_DEV_BAD_COUNT 4     /* a row count or offset disagreed with the buffers; see each call */

#define MOE_MAX_EXPERTS 256
#define MOE_MAX_TOP_K 8

typedef struct {
    int32_t T;     /* tokens (rows of X) */
    int32_t d;     /* hidden size */
    int32_t E;     /* experts */
    int32_t top_k; /* experts per token, 1..8 */
    int32_t d_ff;  /* expert hidden size */
    float eps;     /* RMSNorm epsilon */
    moe_dtype_t x_dtype;   /* X and the residual */
    moe_dtype_t w_dtype;   /* expert weights (bf16: tensor-core path; f32: CUDA-core path) */
    moe_dtype_t out_dtype; /* R */
} moe_shape_t;

typedef struct {
    const float* gamma;  /* [d] RMSNorm scale */
    const float* W_r;    /* [E][d] router weights, z = v W_r^T */
    const float* b;      /* [E] selection bias */
    const void* W_gate;  /* [E][d_ff][d], w_dtype */
    const void* W_up;    /* [E][d_ff][d], w_dtype */
    const void* W_down;  /* [E][d][d_ff], w_dtype */
} moe_weights_t;

/* Block-FP8 expert weights (E4M3 codes + fp32 scales, see moe_quantize_fp8):
 * W_*_q [E][n][k] codes, W_*_s [E][n / 128][k / 128] scales, for W_gate and
 * W_up (n = d_ff, k = d) and W_down (n = d, k = d_ff).  gamma, W_r and b as in
 * moe_weights_t. */
typedef struct {
    const float* gamma;
    const float* W_r;
    const float* b;
    const uint8_t* W_gate_q;
    const float* W_gate_s;
    const uint8_t* W_up_q;
    const float* W_up_s;
    const uint8_t* W_down_q;
    const float* W_down_s;
} moe_weights_fp8_t;

/*
 * Step 1 — RMSNorm [P1 §Norm&Residual, RMSNorm equation]:
 *   v[t][j] = gamma[j] * x[t][j] / sqrt((1/d) * sum_k x[t][k]^2 + eps)
 * x [T][d] (x_dt), gamma [d] f32, v [T][d] (v_dt), fp32 arithmetic.
 * Requires d % 8 == 0; x and v 16-byte aligned.
 */
moe_status_t moe_rmsnorm(const void* x, moe_dtype_t x_dt, const float* gamma, int32_t T, int32_t d, float eps,
                         void* v, moe_dtype_t v_dt, moe_stream_t stream);

/*
 * Step 2 — router [P1 §专家并行 / MoE Router 过程]:
 *   z = v W_r^T (fp32),  s = sigmoid(z),  I = TopK(s + b),  w_i = s_i / sum_{j in I} s_j
 * The bias b only takes part in the choice of I, never in w.  The selection
 * score is fp32: sigmoid evaluated in double and rounded once, plus b in fp32.
 * Ties go to the lower expert index; I is written by descending score.
 * v [T][d] (v_dt), W_r [E][d] f32, b [E] f32.
 * Outputs: topk_idx [T][k] int32, topk_w [T][k] f32; optional (NULL to skip)
 * logits [T][E] f32 and margin [T] f32 = k-th score minus the best unpicked
 * score (+inf when E == k).  Workspace: split-K partial logits.
 * Requires 1 <= k <= 8, k <= E <= 256, d % 8 == 0.
 */
moe_status_t moe_router_topk(const void* v, moe_dtype_t v_dt, const float* W_r, const float* b, int32_t T,
                             int32_t d, int32_t E, int32_t k, int32_t* topk_idx, float* topk_w, float* logits,
                             float* margin, void* ws, size_t* ws_bytes, moe_stream_t stream);

/*
 * Steps 1-2 as the whole layer runs them [P1 §Norm&Residual and §MoE Router
 * 过程]: the router on the RMSNorm of x without materialising it,
 *   z = rstd * (x (gamma ⊙ W_r)^T),  rstd = 1 / sqrt((1/d) sum_k x_k^2 + eps),
 * then selection and weights as in moe_router_topk.  The same kernels as
 * moe_forward's first steps, so the routing is moe_forward's bit for bit
 * (a caller that runs the rest of the layer itself, e.g. with experts on
 * several ranks, routes exactly as the single-GPU layer).  With bf16 x and
 * d % 128 == 0 gamma ⊙ W_r is rounded once to fp32 and split exactly into
 * three bf16 terms, so the logits are fp32-accurate sums of exact products;
 * otherwise the normalised rows are formed in fp32 and multiplied in 3xTF32.
 * x [T][d] (x_dt), gamma [d], W_r [E][d], b [E]; outputs as moe_router_topk.
 * Workspace: 1/rms per token, the split-K partial logits and the split
 * weights.  Requires 1 <= k <= 8, k <= E <= 256, d % 8 == 0.
 */
moe_status_t moe_route(const void* x, moe_dtype_t x_dt, const float* gamma, const float* W_r, const float* b,
                       int32_t T, int32_t d, int32_t E, int32_t k, float eps, int32_t* topk_idx, float* topk_w,
                       float* logits, float* margin, void* ws, size_t* ws_bytes, moe_stream_t stream);

/*
 * Step 3 — token permutation into expert-contiguous rows
 * [P5 §Token 分发策略, token_permutation; §专家计算实现, contiguous layout]:
 *   counts[e]      = number of (t, i) with topk_idx[t][i] == e
 *   offsets[e]     = sum_{e' < e} counts[e'] (no padding), offsets[E] = T*k
 *   slot_token[r]  = source token of row r (r < T*k)
 *   token_slot[t][i] = row that holds pick i of token t (-1 if its id was bad)
 *   xp[r][:]       = v[slot_token[r]][:]   (dtype v_dt)
 * Rows inside a segment follow ascending token index, so the result is
 * deterministic.  Bad ids set MOE_DEV_BAD_EXPERT_ID and are dropped.
 * xp may be NULL: then only the maps are written (moe_ep_dispatch moves the
 * rows itself).
 * Requires d % 8 == 0, v and xp 16-byte aligned, 1 <= k <= 8, k <= E <= 256.
 */
moe_status_t moe_permute(const void* v, moe_dtype_t v_dt, const int32_t* topk_idx, int32_t T, int32_t d, int32_t E,
                         int32_t k, int32_t* counts, int32_t* offsets, int32_t* slot_token, int32_t* token_slot,
                         void* xp, void* ws, size_t* ws_bytes, int32_t* dev_status, moe_stream_t stream);

/*
 * moe_permute without a workspace, for callers that cannot allocate device
 * memory.  The pages have no counterpart: this is a convenience of this library.
 *
 * Some callers are handed only the tensors of the call and may not allocate on
 * the device while it runs (e.g. an inference engine's plugin execute hook that
 * owns a fixed memory pool, where an allocation would stall the stream or
 * fragment the pool).  This call computes exactly what moe_permute computes,
 * with the same kernels, but keeps their scratch (the per-chunk expert
 * histogram) in a 256 KiB array inside the library that each GPU loading it
 * holds until the process exits.  It calls no cudaMalloc/cudaFree.
 *   - T must be <= MOE_PERMUTE_STATIC_MAX_TOKENS (65536), else
 *     MOE_ERR_UNSUPPORTED; other arguments as for moe_permute.
 *   - The first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress) with that device current; make that first call
 *     before any stream capture.  A lookup that fails returns MOE_ERR_CUDA and
 *     is tried again by the next call.
 *   - All calls share the one array and nothing in it needs to start at zero
 *     (every entry read is written earlier in the same call), but calls whose
 *     work overlaps on the GPU (other streams, other host threads) race on it:
 *     order them on one stream.
 */
#define MOE_PERMUTE_STATIC_MAX_TOKENS 65536
moe_status_t moe_permute_static_ws(const void* v, moe_dtype_t v_dt, const int32_t* topk_idx, int32_t T, int32_t d,
                                   int32_t E, int32_t k, int32_t* counts, int32_t* offsets, int32_t* slot_token,
                                   int32_t* token_slot, void* xp, int32_t* dev_status, moe_stream_t stream);

/*
 * Step 4, first half — gate/up projections with the SwiGLU product
 * [P1 §实际 MLP 计算策略: SiLU(X W_gate) ⊙ X W_up; §EP 路径: grouped GEMM]:
 *   h[r][f] = SiLU(sum_j xp[r][j] W_gate[e][f][j]) * (sum_j xp[r][j] W_up[e][f][j])
 * for every row r of expert e's segment [offsets[e], offsets[e] + counts[e]).
 * SiLU(x) = x * sigmoid(x).  dt = MOE_BF16: tcgen05 tensor cores, fp32
 * accumulation in tensor memory, h rounded to bf16; dt = MOE_F32: fp32 CUDA cores.
 * xp [S][d], h [S][d_ff] (dtype dt); counts/offsets as written by moe_permute.
 * Rows outside every segment are not written.  A segment that does not fit the
 * S rows (negative count or offset, or offsets[e] + counts[e] > S) is clamped
 * into them and sets MOE_DEV_BAD_COUNT, so no row outside [0, S) is read or
 * written whatever the device-side counts hold.  (The same holds for
 * moe_expert_down, moe_grouped_swiglu, moe_grouped_swiglu_sized with S_cap
 * rows, and moe_grouped_swiglu_fp8.)
 * bf16 requires d % 64 == 0, d_ff % 128 == 0, 16-byte aligned pointers.
 */
moe_status_t moe_expert_gate_up(const void* xp, const void* W_gate, const void* W_up, moe_dtype_t dt,
                                const int32_t* counts, const int32_t* offsets, int32_t S, int32_t E, int32_t d,
                                int32_t d_ff, void* h, int32_t* dev_status, moe_stream_t stream);

/*
 * The gate/up GEMM core without its SwiGLU product, for testing the tensor-core
 * arithmetic on its own (the pages have no such step):
 *   gu[r][f]        = bf16(sum_j xp[r][j] W_gate[e][f][j])
 *   gu[r][d_ff + f] = bf16(sum_j xp[r][j] W_up[e][f][j])
 * for every row r of expert e's segment: the same kernels, tile forms and fp32
 * accumulation as moe_expert_gate_up (bf16 only), with the epilogue storing
 * the two sums instead of SiLU(g) * u.  gu [S][2 d_ff] bf16.
 */
moe_status_t moe_expert_gate_up_raw(const void* xp, const void* W_gate, const void* W_up, const int32_t* counts,
                                    const int32_t* offsets, int32_t S, int32_t E, int32_t d, int32_t d_ff, void* gu,
                                    int32_t* dev_status, moe_stream_t stream);

/*
 * Step 4, second half — down projection [P1 §实际 MLP 计算策略, "· W_down"]:
 *   y[r][o] = sum_f h[r][f] W_down[e][o][f]   for rows r of expert e's segment.
 * h [S][d_ff], y [S][d] (dtype dt).  bf16 requires d % 128 == 0, d_ff % 64 == 0.
 */
moe_status_t moe_expert_down(const void* h, const void* W_down, moe_dtype_t dt, const int32_t* counts,
                             const int32_t* offsets, int32_t S, int32_t E, int32_t d, int32_t d_ff, void* y,
                             int32_t* dev_status, moe_stream_t stream);

/*
 * Step 4 — grouped SwiGLU expert MLP [P1 §实际 MLP 计算策略; §EP 路径;
 * P5 §专家计算实现, BatchedExperts]: moe_expert_gate_up then moe_expert_down.
 * h is the caller's [S][d_ff] intermediate.
 */
moe_status_t moe_grouped_swiglu(const void* xp, const void* W_gate, const void* W_up, const void* W_down,
                                moe_dtype_t dt, const int32_t* counts, const int32_t* offsets, int32_t S, int32_t E,
                                int32_t d, int32_t d_ff, void* h, void* y, int32_t* dev_status, moe_stream_t stream);

/*
 * Step 4 for a caller that knows its buffer size but not its row count on the
 * host [same computation as moe_grouped_swiglu]: xp, h, y hold S_cap rows;
 * counts/offsets (device) decide which rows are computed, and the tile form is
 * chosen as if there were S_expected rows (1 <= S_expected <= S_cap), so the
 * call needs no device-to-host read.  With S_expected == S_cap it is
 * moe_grouped_swiglu.  Rows outside every segment are not written.
 */
moe_status_t moe_grouped_swiglu_sized(const void* xp, const void* W_gate, const void* W_up, const void* W_down,
                                      moe_dtype_t dt, const int32_t* counts, const int32_t* offsets, int32_t S_cap,
                                      int32_t S_expected, int32_t E, int32_t d, int32_t d_ff, void* h, void* y,
                                      int32_t* dev_status, moe_stream_t stream);

/*
 * Step 4 on the masked decode layout [P5 §专家计算实现: deepgemm_masked, the
 * decode-phase expert GEMM; the page names it without defining it, and this
 * follows the reading that its input is per-expert buffers of fixed capacity
 * with a valid-row count per expert, the form a low-latency token dispatch
 * writes]:
 *   for every expert e and row r < counts[e]:
 *     h[e][r][f] = SiLU(x[e][r] . W_gate[e][f]) * (x[e][r] . W_up[e][f])
 *     y[e][r][o] = h[e][r] . W_down[e][o]
 * x [E][cap][d], h [E][cap][d_ff], y [E][cap][d]; counts [E] on the device.
 * Rows r >= counts[e] are neither used for any stored result nor written, so
 * the buffers need no clearing and the call never reads counts on the host
 * (its launch configuration depends on E, cap, d, d_ff only, so one capture
 * into a CUDA graph serves any counts).  A count outside [0, cap] is clamped
 * and sets MOE_DEV_BAD_COUNT.  Same kernels and numerics as moe_grouped_swiglu
 * (one-CTA tiles); dt must be MOE_BF16; 1 <= cap, E * cap < 2^30; d % 128 == 0,
 * d_ff % 128 == 0; 16-byte aligned pointers.
 */
moe_status_t moe_grouped_swiglu_masked(const void* x, const void* W_gate, const void* W_up, const void* W_down,
                                       moe_dtype_t dt, const int32_t* counts, int32_t E, int32_t cap, int32_t d,
                                       int32_t d_ff, void* h, void* y, int32_t* dev_status, moe_stream_t stream);

/*
 * Step 5 — weighted un-permute and residual [P1 §EP 路径: weighted sum at the
 * source; §Norm&Residual: X' = R + FFN(V); P5 token_unpermutation]:
 *   out[t][j] = residual[t][j] + sum_{i<k} topk_w[t][i] * y[token_slot[t][i]][j]
 * fp32 accumulation in pick order.  Picks with a negative token_slot (moe_permute
 * writes -1 for a bad expert id) are skipped: their row is not read and their
 * weight takes no part.
 * y [T*k][d] (y_dt), residual [T][d] (r_dt), out [T][d] (out_dt).
 * Requires d % 8 == 0 and 16-byte aligned y, residual, out.
 */
moe_status_t moe_unpermute_combine(const void* y, moe_dtype_t y_dt, const int32_t* token_slot, const float* topk_w,
                                   const void* residual, moe_dtype_t r_dt, int32_t T, int32_t d, int32_t k, void* out,
                                   moe_dtype_t out_dt, moe_stream_t stream);

/*
 * The whole layer, steps 1-5 [P1 §Norm&Residual: X_{l+1} = R_l + FFN(RMSNorm(R_l))]:
 *   out = x + MoE(RMSNorm(x))
 * The router reads the unrounded fp32 normalised rows; the expert path reads
 * them rounded to w_dtype.  Optional outputs (NULL to keep them in the
 * workspace): topk_idx [T][k], topk_w [T][k], logits [T][E].
 * dev_status is cleared at the start and receives MOE_DEV_* bits.
 * Supported: x_dtype, out_dtype in {f32, bf16}; w_dtype bf16 (tensor cores,
 * needs d % 128 == 0, d_ff % 128 == 0) or f32 (CUDA cores, d % 8 == 0,
 * d_ff % 8 == 0); 1 <= top_k <= 8; top_k <= E <= 256.
 */
moe_status_t moe_forward(const moe_shape_t* shape, const moe_weights_t* weights, const void* x, void* out,
                         int32_t* topk_idx, float* topk_w, float* logits, void* ws, size_t* ws_bytes,
                         int32_t* dev_status, moe_stream_t stream);

/* Static text for a status code. */
const char* moe_status_string(moe_status_t status);

/*
 * Block-FP8 quantisation [P5 §专家计算实现: FP8 expert GEMMs (fp8_gemm_nt) and
 * the blockfp8 quantised experts; the page names the scheme without defining
 * it, and this follows the usual block-FP8 layout]:
 * x [rows][cols] (MOE_F32 or MOE_BF16, device) -> q [rows][cols] E4M3 codes and
 * s [ceil(rows / blk_rows)][cols / 128] fp32 scales, one per block of
 * blk_rows x 128 elements (blk_rows = 128 for weights, 1 for GEMM inputs).
 * For a block with largest magnitude a: s = a / 448 (1 if a == 0), and each
 * code is E4M3(x / s) rounded to nearest even, saturating at +-448 (E4M3: bias
 * 7, no infinities, S.1111.111 is NaN).  cols % 128 == 0; x, q 16-byte aligned.
 * A weight tensor [E][n][k] is quantised as rows = E * n (n % 128 == 0).
 */
moe_status_t moe_quantize_fp8(const void* x, moe_dtype_t dt, int64_t rows, int64_t cols, int32_t blk_rows, uint8_t* q,
                              float* s, moe_stream_t stream);

/*
 * Step 4 with block-FP8 experts: for every row r of expert e's segment
 *   g, u = dequant(xq[r]) . dequant(W_gate[e]), dequant(W_up[e])   (per feature)
 *   h    = SiLU(g) * u, quantised per (row, 128 features) -> hq [S][d_ff], hs [S][d_ff / 128]
 *   y[r] = dequant(hq[r]) . dequant(W_down[e])                      -> y [S][d] bf16
 * with dequant(code) = value(code) * scale of its block, fp32 accumulation per
 * 128-wide K block in tensor memory and fp32 promotion across blocks.  xq
 * [S][d] codes, xs [S][d / 128] scales (moe_quantize_fp8 with blk_rows 1);
 * w->gamma, W_r and b are not used.  d % 128 == 0, d_ff % 128 == 0.
 */
moe_status_t moe_grouped_swiglu_fp8(const uint8_t* xq, const float* xs, const moe_weights_fp8_t* w,
                                    const int32_t* counts, const int32_t* offsets, int32_t S, int32_t E, int32_t d,
                                    int32_t d_ff, uint8_t* hq, float* hs, void* y, int32_t* dev_status,
                                    moe_stream_t stream);

/*
 * The whole layer with block-FP8 experts: as moe_forward, except that the
 * expert path reads the normalised rows quantised per (row, 128 columns) from
 * their fp32 values, and the expert MLP is moe_grouped_swiglu_fp8 (rows read
 * in place through the permutation, no permuted copy).  The router is the
 * fp32 path of moe_forward.  shape->w_dtype is ignored (expert codes are
 * E4M3, y is bf16); x_dtype and out_dtype as in moe_forward.
 */
moe_status_t moe_forward_fp8(const moe_shape_t* shape, const moe_weights_fp8_t* w, const void* x, void* out,
                             int32_t* topk_idx, float* topk_w, float* logits, void* ws, size_t* ws_bytes,
                             int32_t* dev_status, moe_stream_t stream);

/*
 * Expert parallelism over peer memory (steps 3 and 5 fused with their
 * exchanges) [P5 §Token 分发策略: every (token, expert) row goes to the rank
 * that owns the expert and the results are summed back at the token's source;
 * P1 §EP 路径: the same exchange around the grouped GEMM].
 *
 * N ranks (one GPU each); rank j owns experts [j E/N, (j+1) E/N).  Every rank
 * first runs steps 1-3 on its own tokens (moe_permute with xp = NULL), then the
 * ranks exchange their counts so that each holds the same count_table
 * [N][E] (int32, device): count_table[s][e] = rows rank s routes to expert e.
 * Rank j's receive buffer then holds its experts' rows expert-major, within an
 * expert by source rank, within a source in that source's slot order:
 *   row(source r, expert e, i) = sum_{e' in [j E/N, e)} sum_s count_table[s][e']
 *                                + sum_{s < r} count_table[s][e] + i
 * which is the layout moe_grouped_swiglu takes, with counts and offsets from
 * moe_ep_layout.  recv_bufs / y_bufs are device arrays of N device pointers:
 * entry j is rank j's receive buffer / expert output buffer ([rows][d], dtype
 * of v / y, 16-byte aligned), mapped into this process (NVLink peer access or
 * the same GPU).  The calls only load and store through them: the caller
 * orders the ranks (all dispatches complete before any rank's expert MLP reads
 * its receive buffer; all expert MLPs complete before any combine reads their
 * outputs).  Requires E % N == 0, N <= MOE_MAX_EP_RANKS, d % 8 == 0.
 *
 * recv_rows is the row count of every rank's receive / output buffer (the
 * same on all ranks); no row at or past it is stored or loaded.
 *
 * moe_ep_dispatch: the permutation's row copy to the owners: for every pick
 *   (t, i) of this rank with expert e = topk_idx[t][i] and slot
 *   s = token_slot[t][i], recv_bufs[e / (E/N)][row(rank, e, s - offsets[e])] = v[t].
 *   topk_idx / token_slot / offsets as returned by moe_router_topk and
 *   moe_permute on this rank.  A pick with a bad expert id or slot sets
 *   MOE_DEV_BAD_EXPERT_ID; a pick whose index inside its segment is outside
 *   [0, count_table[rank][e]) or whose row falls outside [0, recv_rows) (a
 *   table that disagrees with the routing, or a short buffer) is not stored
 *   and sets MOE_DEV_BAD_COUNT.
 * moe_ep_layout: counts_loc[e] = sum_s count_table[s][rank E/N + e] and
 *   offsets_loc[0 .. E/N] its exclusive prefix (the receive buffer's segments).
 * moe_ep_combine: step 5 with each pick's expert output row read from its
 *   owner: out[t] = residual[t] + sum_{i<k} topk_w[t][i] * y_bufs[owner][row]
 *   in fp32, pick order; the same arithmetic as moe_unpermute_combine.  A
 *   pick that fails the dispatch's checks is left out of the sum (its row is
 *   not read) and sets the same status bit.
 */
#define MOE_MAX_EP_RANKS 64
moe_status_t moe_ep_dispatch(const void* v, moe_dtype_t v_dt, const int32_t* topk_idx, const int32_t* token_slot,
                             const int32_t* offsets, const int32_t* count_table, int32_t rank, int32_t N, int32_t E,
                             int32_t T, int32_t d, int32_t k, void* const* recv_bufs, int64_t recv_rows,
                             int32_t* dev_status, moe_stream_t stream);
moe_status_t moe_ep_layout(const int32_t* count_table, int32_t rank, int32_t N, int32_t E, int32_t* counts_loc,
                           int32_t* offsets_loc, moe_stream_t stream);
moe_status_t moe_ep_combine(const void* const* y_bufs, moe_dtype_t y_dt, const int32_t* topk_idx,
                            const int32_t* token_slot, const int32_t* offsets, const int32_t* count_table,
                            int32_t rank, int32_t N, int32_t E, const float* topk_w, const void* residual,
                            moe_dtype_t r_dt, int32_t T, int32_t d, int32_t k, void* out, moe_dtype_t out_dt,
                            int64_t recv_rows, int32_t* dev_status, moe_stream_t stream);

/* Number of kernels the library has enqueued in this process since it was
 * loaded, over all entry points, streams and threads (successful launches
 * only; a launch that returned an error is not counted).  Not part of any
 * method on the pages: it lets a caller check how many device launches a call
 * made, e.g. to count the kernels of a timed loop.  Never fails. */
uint64_t moe_kernel_launches(void);

/*
 * Limit of the bounded waits inside the tensor-core kernels (expert GEMMs,
 * router logits), for every launch this process queues after the call; not
 * part of any method on the pages.  Every wait of those kernels on another of
 * their roles (a filled stage, a drained accumulator) gives up after
 * limit_ns nanoseconds (0 restores the default, 2 s): the kernel then sets
 * MOE_DEV_TIMEOUT in dev_status, stops its other roles, waits (bounded by a
 * separate 2 s limit, never cut short) for the copies and MMAs it has already
 * issued, frees its tensor memory and returns, so the context stays usable.
 * inject_stall != 0 is for tests of that path only: each of those kernels
 * then also waits once, before its first output tile, on a barrier that
 * nothing completes, so the wait runs out and the unwinding above happens on
 * valid data.  Process-wide; not synchronised with work already queued.
 */
void moe_set_wait_limit(uint64_t limit_ns, int32_t inject_stall);

/* ABI version of this header (bumped on any incompatible change). */
#define MOE_ABI_VERSION 2
int32_t moe_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MOE_H */
