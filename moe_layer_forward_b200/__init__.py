"""MoE layer forward on one B200: Python binding of ``libmoe.so``.

Every function has the name of the C entry point it calls (``include/moe.h``)
and only marshals torch tensors into pointers, sizes and the current CUDA
stream.  All arithmetic runs in the library's sm_100a kernels.  Importing the
package fails loudly if ``libmoe.so`` has not been built.

    R = X + MoE(RMSNorm(X))   (see ``moe_forward``)
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with `python moe_layer_forward_b200/build.py` "
                      "(or __graft_entry__.build()); there is no fallback implementation")

_lib = ctypes.CDLL(LIB_PATH)

MOE_F32, MOE_BF16 = 0, 1
MOE_DEV_BAD_EXPERT_ID, MOE_DEV_TIMEOUT, MOE_DEV_BAD_COUNT = 1, 2, 4

_vp, _i32, _i64, _f32 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_float
_szp = ctypes.POINTER(ctypes.c_size_t)


class MoeShape(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int32), ("d", ctypes.c_int32), ("E", ctypes.c_int32), ("top_k", ctypes.c_int32),
                ("d_ff", ctypes.c_int32), ("eps", ctypes.c_float), ("x_dtype", ctypes.c_int),
                ("w_dtype", ctypes.c_int), ("out_dtype", ctypes.c_int)]


class MoeWeights(ctypes.Structure):
    _fields_ = [("gamma", _vp), ("W_r", _vp), ("b", _vp), ("W_gate", _vp), ("W_up", _vp), ("W_down", _vp)]


class MoeWeightsFP8(ctypes.Structure):
    _fields_ = [("gamma", _vp), ("W_r", _vp), ("b", _vp), ("W_gate_q", _vp), ("W_gate_s", _vp), ("W_up_q", _vp),
                ("W_up_s", _vp), ("W_down_q", _vp), ("W_down_s", _vp)]


_sig = {
    "moe_rmsnorm": [_vp, _i32, _vp, _i32, _i32, _f32, _vp, _i32, _vp],
    "moe_router_topk": [_vp, _i32, _vp, _vp, _i32, _i32, _i32, _i32, _vp, _vp, _vp, _vp, _vp, _szp, _vp],
    "moe_route": [_vp, _i32, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _f32, _vp, _vp, _vp, _vp, _vp, _szp, _vp],
    "moe_permute": [_vp, _i32, _vp, _i32, _i32, _i32, _i32, _vp, _vp, _vp, _vp, _vp, _vp, _szp, _vp, _vp],
    "moe_permute_static_ws": [_vp, _i32, _vp, _i32, _i32, _i32, _i32, _vp, _vp, _vp, _vp, _vp, _vp, _vp],
    "moe_expert_gate_up": [_vp, _vp, _vp, _i32, _vp, _vp, _i32, _i32, _i32, _i32, _vp, _vp, _vp],
    "moe_expert_down": [_vp, _vp, _i32, _vp, _vp, _i32, _i32, _i32, _i32, _vp, _vp, _vp],
    "moe_expert_gate_up_raw": [_vp, _vp, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _vp, _vp, _vp],
    "moe_grouped_swiglu": [_vp, _vp, _vp, _vp, _i32, _vp, _vp, _i32, _i32, _i32, _i32, _vp, _vp, _vp, _vp],
    "moe_grouped_swiglu_masked": [_vp, _vp, _vp, _vp, _i32, _vp, _i32, _i32, _i32, _i32, _vp, _vp, _vp, _vp],
    "moe_unpermute_combine": [_vp, _i32, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _vp, _i32, _vp],
    "moe_forward": [ctypes.POINTER(MoeShape), ctypes.POINTER(MoeWeights), _vp, _vp, _vp, _vp, _vp, _vp, _szp, _vp,
                    _vp],
    "moe_quantize_fp8": [_vp, _i32, _i64, _i64, _i32, _vp, _vp, _vp],
    "moe_grouped_swiglu_fp8": [_vp, _vp, ctypes.POINTER(MoeWeightsFP8), _vp, _vp, _i32, _i32, _i32, _i32, _vp, _vp,
                               _vp, _vp, _vp],
    "moe_forward_fp8": [ctypes.POINTER(MoeShape), ctypes.POINTER(MoeWeightsFP8), _vp, _vp, _vp, _vp, _vp, _vp, _szp,
                        _vp, _vp],
    "moe_grouped_swiglu_sized": [_vp, _vp, _vp, _vp, _i32, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _vp, _vp, _vp,
                                 _vp],
    "moe_ep_dispatch": [_vp, _i32, _vp, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _i32, _vp, _i64, _vp, _vp],
    "moe_ep_layout": [_vp, _i32, _i32, _i32, _vp, _vp, _vp],
    "moe_ep_combine": [_vp, _i32, _vp, _vp, _vp, _vp, _i32, _i32, _i32, _vp, _vp, _i32, _i32, _i32, _i32, _vp, _i32,
                       _i64, _vp, _vp],
}
for _name, _args in _sig.items():
    _fn = getattr(_lib, _name)
    _fn.argtypes = _args
    _fn.restype = ctypes.c_int
_lib.moe_status_string.argtypes = [ctypes.c_int]
_lib.moe_status_string.restype = ctypes.c_char_p
_lib.moe_abi_version.restype = ctypes.c_int32
_lib.moe_kernel_launches.restype = ctypes.c_uint64
_lib.moe_set_wait_limit.argtypes = [ctypes.c_uint64, ctypes.c_int32]
_lib.moe_set_wait_limit.restype = None


class MoEError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn}: {_lib.moe_status_string(status).decode()} (status {status})")


def _check(fn: str, status: int) -> None:
    if status != 0:
        raise MoEError(fn, status)


def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return MOE_F32
    if t.dtype == torch.bfloat16:
        return MOE_BF16
    raise TypeError(f"unsupported dtype {t.dtype}")


def _p(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensors passed to libmoe must live on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("tensors passed to libmoe must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(dev=None):
    return ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)


def _ws(query, device) -> torch.Tensor:
    n = ctypes.c_size_t(0)
    query(None, ctypes.byref(n))
    return torch.empty(max(int(n.value), 1), dtype=torch.uint8, device=device)


def abi_version() -> int:
    return int(_lib.moe_abi_version())


def set_wait_limit(limit_ns: int = 0, inject_stall: bool = False) -> None:
    """Limit (ns) of the tensor-core kernels' bounded waits for launches queued from now on (0: the default
    2 s); inject_stall makes each of them wait once on a barrier nothing completes (failure-path tests)."""
    _lib.moe_set_wait_limit(int(limit_ns), 1 if inject_stall else 0)


def kernel_launches() -> int:
    """Kernels the library has enqueued in this process so far (all entry points)."""
    return int(_lib.moe_kernel_launches())


def moe_rmsnorm(x: torch.Tensor, gamma: torch.Tensor, eps: float, v: torch.Tensor) -> None:
    T, d = x.shape
    _check("moe_rmsnorm", _lib.moe_rmsnorm(_p(x), _dt(x), _p(gamma), T, d, eps, _p(v), _dt(v), _stream(x.device)))


def moe_router_topk(v, W_r, b, topk_idx, topk_w, logits=None, margin=None, ws=None) -> None:
    T, d = v.shape
    E = W_r.shape[0]
    k = topk_idx.shape[1]

    def call(wsp, nbytes):
        return _lib.moe_router_topk(_p(v), _dt(v), _p(W_r), _p(b), T, d, E, k, _p(topk_idx), _p(topk_w), _p(logits),
                                    _p(margin), wsp, nbytes, _stream(v.device))

    if ws is None:
        ws = _ws(lambda w, n: _check("moe_router_topk", call(w, n)), v.device)
    n = ctypes.c_size_t(ws.numel())
    _check("moe_router_topk", call(_p(ws), ctypes.byref(n)))


def moe_route(x, gamma, W_r, b, topk_idx, topk_w, eps: float = 1e-5, logits=None, margin=None, ws=None) -> None:
    """RMSNorm + router top-k of x exactly as moe_forward runs them (the normalised rows are not materialised)."""
    T, d = x.shape
    E = W_r.shape[0]
    k = topk_idx.shape[1]

    def call(wsp, nbytes):
        return _lib.moe_route(_p(x), _dt(x), _p(gamma), _p(W_r), _p(b), T, d, E, k, eps, _p(topk_idx), _p(topk_w),
                              _p(logits), _p(margin), wsp, nbytes, _stream(x.device))

    if ws is None:
        ws = _ws(lambda w, n: _check("moe_route", call(w, n)), x.device)
    n = ctypes.c_size_t(ws.numel())
    _check("moe_route", call(_p(ws), ctypes.byref(n)))


def moe_permute(v, topk_idx, E: int, counts, offsets, slot_token, token_slot, xp, ws=None, dev_status=None) -> None:
    T, d = v.shape
    k = topk_idx.shape[1]

    def call(wsp, nbytes):
        return _lib.moe_permute(_p(v), _dt(v), _p(topk_idx), T, d, E, k, _p(counts), _p(offsets), _p(slot_token),
                                _p(token_slot), _p(xp), wsp, nbytes, _p(dev_status), _stream(v.device))

    if ws is None:
        ws = _ws(lambda w, n: _check("moe_permute", call(w, n)), v.device)
    n = ctypes.c_size_t(ws.numel())
    _check("moe_permute", call(_p(ws), ctypes.byref(n)))


def moe_permute_static_ws(v, topk_idx, E: int, counts, offsets, slot_token, token_slot, xp,
                          dev_status=None) -> None:
    """moe_permute for callers that cannot allocate: the library keeps the scratch itself.

    Same results as ``moe_permute``; needs no workspace (T <= 65536).  Calls that
    overlap on the GPU share that scratch and race, so keep them on one stream.
    """
    T, d = v.shape
    k = topk_idx.shape[1]
    _check("moe_permute_static_ws", _lib.moe_permute_static_ws(_p(v), _dt(v), _p(topk_idx), T, d, E, k, _p(counts),
                                                               _p(offsets), _p(slot_token), _p(token_slot), _p(xp),
                                                               _p(dev_status), _stream(v.device)))


def moe_expert_gate_up(xp, W_gate, W_up, counts, offsets, h, dev_status=None) -> None:
    S, d = xp.shape
    E, d_ff, _ = W_gate.shape
    _check("moe_expert_gate_up", _lib.moe_expert_gate_up(_p(xp), _p(W_gate), _p(W_up), _dt(W_gate), _p(counts),
                                                         _p(offsets), S, E, d, d_ff, _p(h), _p(dev_status),
                                                         _stream(xp.device)))


def moe_expert_gate_up_raw(xp, W_gate, W_up, counts, offsets, gu, dev_status=None) -> None:
    """The gate/up GEMMs without the SwiGLU product: gu [S][2 d_ff] = [xp W_gate^T | xp W_up^T] per segment (bf16)."""
    S, d = xp.shape
    E, d_ff, _ = W_gate.shape
    _check("moe_expert_gate_up_raw", _lib.moe_expert_gate_up_raw(_p(xp), _p(W_gate), _p(W_up), _p(counts),
                                                                 _p(offsets), S, E, d, d_ff, _p(gu), _p(dev_status),
                                                                 _stream(xp.device)))


def moe_expert_down(h, W_down, counts, offsets, y, dev_status=None) -> None:
    S, d_ff = h.shape
    E, d, _ = W_down.shape
    _check("moe_expert_down", _lib.moe_expert_down(_p(h), _p(W_down), _dt(W_down), _p(counts), _p(offsets), S, E, d,
                                                   d_ff, _p(y), _p(dev_status), _stream(h.device)))


def moe_grouped_swiglu(xp, W_gate, W_up, W_down, counts, offsets, h, y, dev_status=None) -> None:
    S, d = xp.shape
    E, d_ff, _ = W_gate.shape
    _check("moe_grouped_swiglu", _lib.moe_grouped_swiglu(_p(xp), _p(W_gate), _p(W_up), _p(W_down), _dt(W_gate),
                                                         _p(counts), _p(offsets), S, E, d, d_ff, _p(h), _p(y),
                                                         _p(dev_status), _stream(xp.device)))


def moe_grouped_swiglu_masked(x, W_gate, W_up, W_down, counts, h, y, dev_status=None) -> None:
    """Expert MLP on per-expert buffers x [E][cap][d] with counts [E] valid rows each (device)."""
    E, cap, d = x.shape
    d_ff = W_gate.shape[1]
    _check("moe_grouped_swiglu_masked",
           _lib.moe_grouped_swiglu_masked(_p(x), _p(W_gate), _p(W_up), _p(W_down), _dt(W_gate), _p(counts), E, cap,
                                          d, d_ff, _p(h), _p(y), _p(dev_status), _stream(x.device)))


def moe_unpermute_combine(y, token_slot, topk_w, residual, out) -> None:
    T, d = residual.shape
    k = token_slot.shape[1]
    _check("moe_unpermute_combine", _lib.moe_unpermute_combine(_p(y), _dt(y), _p(token_slot), _p(topk_w),
                                                               _p(residual), _dt(residual), T, d, k, _p(out),
                                                               _dt(out), _stream(residual.device)))


def moe_grouped_swiglu_sized(xp, W_gate, W_up, W_down, counts, offsets, h, y, S_expected: int,
                             dev_status=None) -> None:
    """moe_grouped_swiglu over buffers of S_cap = xp.shape[0] rows, tiles chosen for S_expected rows."""
    S, d = xp.shape
    E, d_ff, _ = W_gate.shape
    _check("moe_grouped_swiglu_sized",
           _lib.moe_grouped_swiglu_sized(_p(xp), _p(W_gate), _p(W_up), _p(W_down), _dt(W_gate), _p(counts),
                                         _p(offsets), S, S_expected, E, d, d_ff, _p(h), _p(y), _p(dev_status),
                                         _stream(xp.device)))


# --------------------------------------------------------------------------- expert parallelism over peer memory
def moe_ep_dispatch(v, topk_idx, token_slot, offsets, count_table, rank: int, recv_ptrs, recv_rows: int,
                    dev_status=None) -> None:
    """Store this rank's routed rows of v into their owners' receive buffers.

    count_table: int32 [N][E] on the device (every rank's counts); recv_ptrs: int64 [N] on the device, the
    receive buffers' addresses as mapped into this process; recv_rows: rows of every receive buffer."""
    T, d = v.shape
    k = topk_idx.shape[1]
    N, E = count_table.shape
    _check("moe_ep_dispatch", _lib.moe_ep_dispatch(_p(v), _dt(v), _p(topk_idx), _p(token_slot), _p(offsets),
                                                   _p(count_table), rank, N, E, T, d, k, _p(recv_ptrs), recv_rows,
                                                   _p(dev_status), _stream(v.device)))


def moe_ep_layout(count_table, rank: int, counts_loc, offsets_loc) -> None:
    """This rank's expert segments of its receive buffer: counts_loc [E/N], offsets_loc [E/N + 1]."""
    N, E = count_table.shape
    _check("moe_ep_layout", _lib.moe_ep_layout(_p(count_table), rank, N, E, _p(counts_loc), _p(offsets_loc),
                                               _stream(count_table.device)))


def moe_ep_combine(y_ptrs, y_dtype, topk_idx, token_slot, offsets, count_table, rank: int, topk_w, residual, out,
                   recv_rows: int, dev_status=None) -> None:
    """out = residual + sum_i w_i y_i with each pick's row y_i read from its owner's output buffer.

    y_ptrs: int64 [N] on the device, the expert output buffers' addresses; y_dtype their torch dtype;
    recv_rows: rows of every output buffer."""
    T, d = residual.shape
    k = topk_idx.shape[1]
    N, E = count_table.shape
    ydt = MOE_BF16 if y_dtype == torch.bfloat16 else MOE_F32
    _check("moe_ep_combine", _lib.moe_ep_combine(_p(y_ptrs), ydt, _p(topk_idx), _p(token_slot), _p(offsets),
                                                 _p(count_table), rank, N, E, _p(topk_w), _p(residual),
                                                 _dt(residual), T, d, k, _p(out), _dt(out), recv_rows,
                                                 _p(dev_status), _stream(residual.device)))


def _shape(x, W_gate, out, top_k, eps, E) -> MoeShape:
    T, d = x.shape
    _, d_ff, _ = W_gate.shape
    return MoeShape(T, d, E, top_k, d_ff, eps, _dt(x), _dt(W_gate), _dt(out))


def forward_workspace_bytes(x, W_r, W_gate, out, top_k: int = 8, eps: float = 1e-5) -> int:
    """Bytes of workspace ``moe_forward`` needs for these tensors (device query; queues nothing)."""
    shp = _shape(x, W_gate, out, top_k, eps, W_r.shape[0])
    wts = MoeWeights()
    n = ctypes.c_size_t(0)
    _check("moe_forward", _lib.moe_forward(ctypes.byref(shp), ctypes.byref(wts), None, None, None, None, None, None,
                                           ctypes.byref(n), None, _stream(x.device)))
    return int(n.value)


def moe_forward(x, gamma, W_r, b, W_gate, W_up, W_down, out, top_k: int = 8, eps: float = 1e-5, topk_idx=None,
                topk_w=None, logits=None, ws=None, dev_status=None) -> None:
    """out = x + MoE(RMSNorm(x)) on x's device and current stream (asynchronous)."""
    shp = _shape(x, W_gate, out, top_k, eps, W_r.shape[0])
    wts = MoeWeights(_p(gamma), _p(W_r), _p(b), _p(W_gate), _p(W_up), _p(W_down))
    if ws is None:
        ws = torch.empty(max(forward_workspace_bytes(x, W_r, W_gate, out, top_k, eps), 1), dtype=torch.uint8,
                         device=x.device)
    n = ctypes.c_size_t(ws.numel())
    _check("moe_forward", _lib.moe_forward(ctypes.byref(shp), ctypes.byref(wts), _p(x), _p(out), _p(topk_idx),
                                           _p(topk_w), _p(logits), _p(ws), ctypes.byref(n), _p(dev_status),
                                           _stream(x.device)))


# --------------------------------------------------------------------------- block FP8 experts
def quantize_fp8(x, blk_rows: int, q, s) -> None:
    """E4M3 codes q and fp32 scales s of x ([..., cols]) per blk_rows x 128 block (128: weights, 1: inputs)."""
    cols = x.shape[-1]
    rows = x.numel() // cols
    _check("moe_quantize_fp8", _lib.moe_quantize_fp8(_p(x), _dt(x), rows, cols, blk_rows, _p(q), _p(s),
                                                     _stream(x.device)))


def quantize_fp8_weights(W):
    """(codes uint8 [E][n][k], scales f32 [E][n/128][k/128]) of an expert weight tensor, on its device."""
    E, n, k = W.shape
    q = torch.empty((E, n, k), dtype=torch.uint8, device=W.device)
    s = torch.empty((E, n // 128, k // 128), dtype=torch.float32, device=W.device)
    quantize_fp8(W, 128, q, s)
    return q, s


def _fp8_weights(gamma, W_r, b, Wg, Wu, Wd) -> MoeWeightsFP8:
    return MoeWeightsFP8(_p(gamma), _p(W_r), _p(b), _p(Wg[0]), _p(Wg[1]), _p(Wu[0]), _p(Wu[1]), _p(Wd[0]),
                         _p(Wd[1]))


def moe_grouped_swiglu_fp8(xq, xs, Wg, Wu, Wd, counts, offsets, hq, hs, y, dev_status=None) -> None:
    """Block-FP8 expert MLP; Wg/Wu/Wd are (codes, scales) pairs, xq/xs the input rows' codes and scales."""
    S, d = xq.shape
    E, d_ff, _ = Wg[0].shape
    w = _fp8_weights(None, None, None, Wg, Wu, Wd)
    _check("moe_grouped_swiglu_fp8",
           _lib.moe_grouped_swiglu_fp8(_p(xq), _p(xs), ctypes.byref(w), _p(counts), _p(offsets), S, E, d, d_ff,
                                       _p(hq), _p(hs), _p(y), _p(dev_status), _stream(xq.device)))


def _shape_fp8(x, Wg_q, out, top_k, eps, E) -> MoeShape:
    T, d = x.shape
    return MoeShape(T, d, E, top_k, Wg_q.shape[1], eps, _dt(x), MOE_BF16, _dt(out))


def forward_fp8_workspace_bytes(x, W_r, Wg_q, out, top_k: int = 8, eps: float = 1e-5) -> int:
    shp = _shape_fp8(x, Wg_q, out, top_k, eps, W_r.shape[0])
    w = MoeWeightsFP8()
    n = ctypes.c_size_t(0)
    _check("moe_forward_fp8", _lib.moe_forward_fp8(ctypes.byref(shp), ctypes.byref(w), None, None, None, None, None,
                                                   None, ctypes.byref(n), None, _stream(x.device)))
    return int(n.value)


def moe_forward_fp8(x, gamma, W_r, b, Wg, Wu, Wd, out, top_k: int = 8, eps: float = 1e-5, topk_idx=None,
                    topk_w=None, logits=None, ws=None, dev_status=None) -> None:
    """out = x + MoE(RMSNorm(x)) with block-FP8 experts (Wg/Wu/Wd: (codes, scales) pairs)."""
    shp = _shape_fp8(x, Wg[0], out, top_k, eps, W_r.shape[0])
    w = _fp8_weights(gamma, W_r, b, Wg, Wu, Wd)
    if ws is None:
        ws = torch.empty(max(forward_fp8_workspace_bytes(x, W_r, Wg[0], out, top_k, eps), 1), dtype=torch.uint8,
                         device=x.device)
    n = ctypes.c_size_t(ws.numel())
    _check("moe_forward_fp8", _lib.moe_forward_fp8(ctypes.byref(shp), ctypes.byref(w), _p(x), _p(out), _p(topk_idx),
                                                   _p(topk_w), _p(logits), _p(ws), ctypes.byref(n), _p(dev_status),
                                                   _stream(x.device)))

