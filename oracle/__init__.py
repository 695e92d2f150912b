"""CPU oracle of the MoE layer forward (ctypes binding of ``oracle.c``).

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, ``__graft_entry__.smoke()``
and the CPU-baseline / reference legs of ``bench.py``.  The product package
never imports it.  It shares no code with the CUDA library.

All functions take CPU torch tensors (float32, bfloat16 or int32) and return
CPU tensors; floating results are float64.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_SO = os.path.join(_HERE, "liboracle.so")
_SRCS = [os.path.join(_HERE, "oracle.c"), os.path.join(_HERE, "oracle_fp8.c")]

F32, BF16 = 0, 1


def build(force: bool = False) -> str:
    """Compile ``liboracle.so`` with plain gcc (no fast-math, no OpenMP)."""
    if force or not os.path.exists(_SO) or any(os.path.getmtime(_SO) < os.path.getmtime(f) for f in _SRCS):
        tmp = _SO + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-std=c11", "-fno-fast-math",
                               "-ffp-contract=off", "-o", tmp, *_SRCS, "-lm"])
        os.replace(tmp, _SO)
    return _SO


_lib = None


def _L():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_SO)
        vp, i64, i32, dbl, flt = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_double, ctypes.c_float
        L.oracle_load.argtypes = [vp, i32, i64]
        L.oracle_load.restype = dbl
        L.oracle_sigmoid.argtypes = [dbl]
        L.oracle_sigmoid.restype = dbl
        L.oracle_silu.argtypes = [dbl]
        L.oracle_silu.restype = dbl
        L.oracle_selection_score.argtypes = [flt, flt]
        L.oracle_selection_score.restype = flt
        L.oracle_rmsnorm.argtypes = [vp, i32, vp, i64, i64, dbl, vp]
        L.oracle_linear.argtypes = [vp, vp, i32, i64, i64, vp]
        L.oracle_router_logits.argtypes = [vp, vp, i64, i64, i64, vp]
        L.oracle_select_topk.argtypes = [vp, vp, vp, i64, i64, i32, vp, vp, vp]
        L.oracle_select_topk.restype = i32
        L.oracle_expert_mlp.argtypes = [vp, vp, vp, vp, i32, i64, i64, i64, vp, vp]
        L.oracle_permute.argtypes = [vp, i64, i64, i32, vp, vp, vp, vp]
        L.oracle_permute.restype = i32
        L.oracle_gather.argtypes = [vp, i32, vp, i64, i64, vp]
        L.oracle_grouped_mlp.argtypes = [vp, i32, vp, vp, i64, i64, i64, vp, vp, vp, i32, vp, vp]
        L.oracle_combine.argtypes = [vp, i32, vp, vp, vp, i32, i64, i64, i32, vp]
        L.oracle_moe_layer.argtypes = [vp, i32, i64, vp, vp, vp, vp, vp, vp, i32, i64, i64, i32, i64, dbl,
                                       vp, vp, vp, vp, vp, vp, vp]
        L.oracle_moe_layer.restype = i32
        L.oracle_e4m3_decode.argtypes = [ctypes.c_uint8]
        L.oracle_e4m3_decode.restype = dbl
        L.oracle_e4m3_encode.argtypes = [flt]
        L.oracle_e4m3_encode.restype = ctypes.c_uint8
        L.oracle_quantize_blocks.argtypes = [vp, i32, i64, i64, i64, vp, vp]
        L.oracle_fp8_grouped_mlp.argtypes = [vp, vp, vp, vp, i64, i64, i64, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp,
                                             vp, vp]
        _lib = L
    return _lib


def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return F32
    if t.dtype == torch.bfloat16:
        return BF16
    raise TypeError(f"oracle takes float32 or bfloat16 tensors, not {t.dtype}")


def _c(t: torch.Tensor, dtype=None) -> torch.Tensor:
    t = t.detach().cpu()
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"expected {dtype}, got {t.dtype}")
    return t.contiguous()


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def sigmoid(z: float) -> float:
    return _L().oracle_sigmoid(z)


def silu(x: float) -> float:
    return _L().oracle_silu(x)


def selection_score(z: float, b: float) -> float:
    return _L().oracle_selection_score(z, b)


def rmsnorm(x: torch.Tensor, gamma: torch.Tensor, eps: float = 1e-5) -> torch.Tensor:
    x, gamma = _c(x), _c(gamma, torch.float32)
    T, d = x.shape
    v = torch.empty((T, d), dtype=torch.float64)
    _L().oracle_rmsnorm(_p(x), _dt(x), _p(gamma), T, d, eps, _p(v))
    return v


def linear(x: torch.Tensor, W: torch.Tensor) -> torch.Tensor:
    """y = W x for one fp64 row x [n_in]; W [n_out][n_in] (f32 or bf16)."""
    x, W = _c(x, torch.float64), _c(W)
    y = torch.empty(W.shape[0], dtype=torch.float64)
    _L().oracle_linear(_p(x), _p(W), _dt(W), W.shape[0], W.shape[1], _p(y))
    return y


def router_logits(v: torch.Tensor, W_r: torch.Tensor) -> torch.Tensor:
    v, W_r = _c(v, torch.float64), _c(W_r, torch.float32)
    T, d = v.shape
    E = W_r.shape[0]
    z = torch.empty((T, E), dtype=torch.float64)
    _L().oracle_router_logits(_p(v), _p(W_r), T, d, E, _p(z))
    return z


def select_topk(z_sel: torch.Tensor, b: torch.Tensor, k: int = 8, z_w: torch.Tensor | None = None):
    """(idx int32 [T][k], w f64 [T][k], margin f32 [T]) from fp32 logits ``z_sel``."""
    z_sel, b = _c(z_sel, torch.float32), _c(b, torch.float32)
    T, E = z_sel.shape
    if z_w is not None:
        z_w = _c(z_w, torch.float64)
    idx = torch.empty((T, k), dtype=torch.int32)
    w = torch.empty((T, k), dtype=torch.float64)
    margin = torch.empty(T, dtype=torch.float32)
    rc = _L().oracle_select_topk(_p(z_sel), _p(z_w), _p(b), T, E, k, _p(idx), _p(w), _p(margin))
    if rc != 0:
        raise ValueError("oracle_select_topk: bad arguments")
    return idx, w, margin


def expert_mlp(v: torch.Tensor, W_gate, W_up, W_down, e: int):
    """(h [d_ff], y [d]) of expert e on one fp64 row v [d]."""
    v = _c(v, torch.float64)
    W_gate, W_up, W_down = _c(W_gate), _c(W_up), _c(W_down)
    E, d_ff, d = W_gate.shape
    h = torch.empty(d_ff, dtype=torch.float64)
    y = torch.empty(d, dtype=torch.float64)
    _L().oracle_expert_mlp(_p(v), _p(W_gate), _p(W_up), _p(W_down), _dt(W_gate), e, d, d_ff, _p(h), _p(y))
    return h, y


def permute(idx: torch.Tensor, E: int):
    """(counts [E], offsets [E+1], slot_token [S], token_slot [T][k]) int32."""
    idx = _c(idx, torch.int32)
    T, k = idx.shape
    counts = torch.empty(E, dtype=torch.int32)
    offsets = torch.empty(E + 1, dtype=torch.int32)
    slot_token = torch.empty(T * k, dtype=torch.int32)
    token_slot = torch.empty((T, k), dtype=torch.int32)
    rc = _L().oracle_permute(_p(idx), T, E, k, _p(counts), _p(offsets), _p(slot_token), _p(token_slot))
    if rc != 0:
        raise ValueError("oracle_permute: expert id out of range")
    return counts, offsets, slot_token, token_slot


def gather(v: torch.Tensor, slot_token: torch.Tensor) -> torch.Tensor:
    v, slot_token = _c(v), _c(slot_token, torch.int32)
    S = slot_token.numel()
    d = v.shape[1]
    xp = torch.empty((S, d), dtype=torch.float64)
    _L().oracle_gather(_p(v), _dt(v), _p(slot_token), S, d, _p(xp))
    return xp


def grouped_mlp(xp: torch.Tensor, counts, offsets, W_gate, W_up, W_down):
    """(h [S][d_ff], y [S][d]) fp64; rows outside every segment are NaN."""
    xp = _c(xp)
    counts, offsets = _c(counts, torch.int32), _c(offsets, torch.int32)
    W_gate, W_up, W_down = _c(W_gate), _c(W_up), _c(W_down)
    E, d_ff, d = W_gate.shape
    S = xp.shape[0]
    h = torch.full((S, d_ff), float("nan"), dtype=torch.float64)
    y = torch.full((S, d), float("nan"), dtype=torch.float64)
    _L().oracle_grouped_mlp(_p(xp), _dt(xp), _p(counts), _p(offsets), E, d, d_ff, _p(W_gate), _p(W_up),
                            _p(W_down), _dt(W_gate), _p(h), _p(y))
    return h, y


def combine(y: torch.Tensor, token_slot, w, residual) -> torch.Tensor:
    y, residual = _c(y), _c(residual)
    token_slot, w = _c(token_slot, torch.int32), _c(w, torch.float32)
    T, k = token_slot.shape
    d = y.shape[1]
    out = torch.empty((T, d), dtype=torch.float64)
    _L().oracle_combine(_p(y), _dt(y), _p(token_slot), _p(w), _p(residual), _dt(residual), T, d, k, _p(out))
    return out


def moe_layer(x, gamma, W_r, b, W_gate, W_up, W_down, k: int = 8, eps: float = 1e-5, force_idx=None,
              force_w=None):
    """Whole layer on the rows of x, token by token.

    Returns dict(out f64 [n][d], idx int32 [n][k], w f64 [n][k], z32 f32 [n][E], margin f32 [n]).
    ``force_idx``/``force_w`` replace the oracle's routing for the expert part.
    """
    x = _c(x)
    gamma, W_r, b = _c(gamma, torch.float32), _c(W_r, torch.float32), _c(b, torch.float32)
    W_gate, W_up, W_down = _c(W_gate), _c(W_up), _c(W_down)
    n, d = x.shape
    E, d_ff, _ = W_gate.shape
    if force_idx is not None:
        force_idx, force_w = _c(force_idx, torch.int32), _c(force_w, torch.float32)
    out = torch.empty((n, d), dtype=torch.float64)
    idx = torch.empty((n, k), dtype=torch.int32)
    w = torch.empty((n, k), dtype=torch.float64)
    z32 = torch.empty((n, E), dtype=torch.float32)
    margin = torch.empty(n, dtype=torch.float32)
    rc = _L().oracle_moe_layer(_p(x), _dt(x), n, _p(gamma), _p(W_r), _p(b), _p(W_gate), _p(W_up), _p(W_down),
                               _dt(W_gate), d, E, k, d_ff, eps, _p(force_idx), _p(force_w), _p(out), _p(idx),
                               _p(w), _p(z32), _p(margin))
    if rc != 0:
        raise ValueError("oracle_moe_layer: bad arguments")
    return {"out": out, "idx": idx, "w": w, "z32": z32, "margin": margin}


# --------------------------------------------------------------------------- block FP8 (oracle_fp8.c)
def e4m3_decode(codes: torch.Tensor) -> torch.Tensor:
    """float64 value of every E4M3 code (uint8)."""
    c = codes.contiguous().to(torch.uint8).flatten()
    f = _L().oracle_e4m3_decode
    return torch.tensor([f(int(v)) for v in c.tolist()], dtype=torch.float64).reshape(codes.shape)


def e4m3_encode(x: torch.Tensor) -> torch.Tensor:
    """nearest E4M3 code (ties to even, saturating) of every fp32 value."""
    v = x.contiguous().to(torch.float32).flatten()
    f = _L().oracle_e4m3_encode
    return torch.tensor([f(float(a)) for a in v.tolist()], dtype=torch.uint8).reshape(x.shape)


def quantize_blocks(x: torch.Tensor, blk_rows: int):
    """(codes uint8 [rows][cols], scales f32 [ceil(rows/blk_rows)][cols/128]) of a 2-D f32/bf16 matrix."""
    x = _c(x)
    rows, cols = x.shape
    q = torch.empty((rows, cols), dtype=torch.uint8)
    s = torch.empty(((rows + blk_rows - 1) // blk_rows, cols // 128), dtype=torch.float32)
    _L().oracle_quantize_blocks(_p(x), _dt(x), rows, cols, blk_rows, _p(q), _p(s))
    return q, s


def fp8_grouped_mlp(xq, xs, counts, offsets, Wg_q, Wg_s, Wu_q, Wu_s, Wd_q, Wd_s, hq_in=None, hs_in=None):
    """Block-FP8 grouped SwiGLU MLP: dict(h f64, hq u8, hs f32, y f64); rows outside segments are NaN / 0."""
    xq, xs = xq.contiguous(), xs.contiguous()
    counts, offsets = _c(counts, torch.int32), _c(offsets, torch.int32)
    E, d_ff, d = Wg_q.shape
    S = xq.shape[0]
    h = torch.full((S, d_ff), float("nan"), dtype=torch.float64)
    y = torch.full((S, d), float("nan"), dtype=torch.float64)
    hq = torch.zeros((S, d_ff), dtype=torch.uint8)
    hs = torch.zeros((S, d_ff // 128), dtype=torch.float32)
    ins = [None if t is None else t.contiguous() for t in (hq_in, hs_in)]
    _L().oracle_fp8_grouped_mlp(_p(xq), _p(xs), _p(counts), _p(offsets), E, d, d_ff,
                                _p(Wg_q.contiguous()), _p(Wg_s.contiguous()), _p(Wu_q.contiguous()),
                                _p(Wu_s.contiguous()), _p(Wd_q.contiguous()), _p(Wd_s.contiguous()), _p(h), _p(hq),
                                _p(hs), _p(ins[0]), _p(ins[1]), _p(y))
    return {"h": h, "hq": hq, "hs": hs, "y": y}

