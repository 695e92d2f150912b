"""Seeded synthetic inputs for the MoE layer workloads.

This module only draws numbers (see ``gen.c``: a splitmix64 counter hash and
Box-Muller normals).  It holds none of the layer's arithmetic, and both the
CUDA path's tests/bench and the CPU oracle read the tensors it makes.

Workloads (the five MoE-layer cases; distributions read ``N(mu, v)`` with
``v`` a variance):

====  ======  ====  ===  =====  ==================================
name  T       d     E    d_ff   dtypes (x / experts / out)
====  ======  ====  ===  =====  ==================================
tiny  64      256   32   128    f32 / f32 / f32
decode 128    4096  128  1536   bf16 / bf16 / bf16
prefill 8192  4096  128  1536   bf16 / bf16 / bf16
skewed 16384  4096  128  1536   bf16 / bf16 / bf16 (Zipf(1.2) bias)
block  4096   4096  256  2048   f32 / bf16 / f32 (residual in f32)
====  ======  ====  ===  =====  ==================================

X ~ N(0,1); W_r ~ N(0, 1/d); gamma = 1 + N(0, 0.1); W_gate, W_up ~ N(0, 1/d);
W_down ~ N(0, 1/d_ff); b ~ U(-0.1, 0.1) (U(-0.01, 0.01) for ``decode``;
``0.5*ln(p_r)`` with Zipf(1.2) rank weights p_r, rank r = e+1, for ``skewed``).
Seed = the workload's index (tiny 0 ... block 4).
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess
from dataclasses import dataclass, replace

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_SO = os.path.join(_HERE, "libsynth.so")
_SRC = os.path.join(_HERE, "gen.c")

# tensor ids of the counter streams
TID_X, TID_WR, TID_B, TID_GAMMA, TID_WG, TID_WU, TID_WD = 1, 2, 3, 4, 5, 6, 7


def build(force: bool = False) -> str:
    """Compile ``libsynth.so`` (gcc, OpenMP, no fast-math) if missing or stale."""
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        tmp = _SO + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _SO)
    return _SO


_lib = None


def _L():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_SO)
        u64, i32, dbl, vp = ctypes.c_uint64, ctypes.c_int32, ctypes.c_double, ctypes.c_void_p
        for name in ("synth_normal_f32", "synth_normal_bf16"):
            getattr(lib, name).argtypes = [vp, u64, u64, u64, dbl, dbl]
        lib.synth_uniform_f32.argtypes = [vp, u64, u64, u64, dbl, dbl]
        lib.synth_uniform_i32.argtypes = [vp, u64, u64, u64, i32, i32]
        lib.synth_raw_u64.argtypes = [vp, u64, u64, u64]
        _lib = lib
    return _lib


def normal(shape, seed: int, tid: int, mean: float = 0.0, std: float = 1.0, dtype=torch.float32) -> torch.Tensor:
    """CPU tensor of ``mean + std * N(0,1)`` draws, as float32 or bfloat16."""
    n = math.prod(shape)
    if dtype == torch.float32:
        t = torch.empty(shape, dtype=torch.float32)
        _L().synth_normal_f32(t.data_ptr(), n, seed, tid, mean, std)
    elif dtype == torch.bfloat16:
        t = torch.empty(shape, dtype=torch.bfloat16)
        _L().synth_normal_bf16(t.data_ptr(), n, seed, tid, mean, std)
    else:
        raise ValueError(f"unsupported dtype {dtype}")
    return t


def uniform(shape, seed: int, tid: int, lo: float, hi: float) -> torch.Tensor:
    t = torch.empty(shape, dtype=torch.float32)
    _L().synth_uniform_f32(t.data_ptr(), math.prod(shape), seed, tid, lo, hi)
    return t


def randint(shape, seed: int, tid: int, lo: int, hi: int) -> torch.Tensor:
    """int32 draws, uniform on [lo, hi] inclusive."""
    t = torch.empty(shape, dtype=torch.int32)
    _L().synth_uniform_i32(t.data_ptr(), math.prod(shape), seed, tid, lo, hi)
    return t


def raw_u64(n: int, seed: int, tid: int) -> list:
    buf = (ctypes.c_uint64 * n)()
    _L().synth_raw_u64(ctypes.addressof(buf), n, seed, tid)
    return list(buf)


def distinct_topk(T: int, E: int, k: int, seed: int, tid: int = 11) -> torch.Tensor:
    """[T][k] int32 rows of k distinct experts in [0, E), drawn by partial shuffle."""
    raw = raw_u64(T * k, seed, tid)
    out = torch.empty((T, k), dtype=torch.int32)
    for t in range(T):
        pool = list(range(E))
        for i in range(k):
            j = i + raw[t * k + i] % (E - i)
            pool[i], pool[j] = pool[j], pool[i]
            out[t, i] = pool[i]
    return out


@dataclass(frozen=True)
class Workload:
    name: str
    T: int
    d: int
    E: int
    d_ff: int
    top_k: int = 8
    x_dtype: torch.dtype = torch.bfloat16
    w_dtype: torch.dtype = torch.bfloat16
    out_dtype: torch.dtype = torch.bfloat16
    bias: str = "u0.1"  # "u0.1" | "u0.01" | "zipf1.2"
    seed: int = 0
    eps: float = 1e-5

    def scaled(self, **kw) -> "Workload":
        return replace(self, **kw)

    @property
    def S(self) -> int:
        return self.T * self.top_k


WORKLOADS = {
    "tiny": Workload("tiny", 64, 256, 32, 128, x_dtype=torch.float32, w_dtype=torch.float32,
                     out_dtype=torch.float32, bias="u0.1", seed=0),
    "decode": Workload("decode", 128, 4096, 128, 1536, bias="u0.01", seed=1),
    "prefill": Workload("prefill", 8192, 4096, 128, 1536, bias="u0.1", seed=2),
    "skewed": Workload("skewed", 16384, 4096, 128, 1536, bias="zipf1.2", seed=3),
    "block": Workload("block", 4096, 4096, 256, 2048, x_dtype=torch.float32, out_dtype=torch.float32,
                      bias="u0.1", seed=4),
}


def zipf_bias(E: int, s: float = 1.2) -> torch.Tensor:
    """b_e = 0.5 * ln(p_{e+1}), p_r = r^-s / sum_q q^-s (expert 0 is the most popular)."""
    z = sum(q ** -s for q in range(1, E + 1))
    return torch.tensor([0.5 * math.log((r ** -s) / z) for r in range(1, E + 1)], dtype=torch.float32)


def make_layer_inputs(w: Workload, with_experts: bool = True) -> dict:
    """All layer inputs of workload ``w`` as CPU tensors.

    x [T][d]; gamma [d] f32; W_r [E][d] f32; b [E] f32;
    W_gate, W_up [E][d_ff][d]; W_down [E][d][d_ff] (out x in, K contiguous).
    """
    s = w.seed
    out = {
        "x": normal((w.T, w.d), s, TID_X, 0.0, 1.0, w.x_dtype),
        "gamma": normal((w.d,), s, TID_GAMMA, 1.0, math.sqrt(0.1), torch.float32),
        "W_r": normal((w.E, w.d), s, TID_WR, 0.0, 1.0 / math.sqrt(w.d), torch.float32),
    }
    if w.bias == "u0.1":
        out["b"] = uniform((w.E,), s, TID_B, -0.1, 0.1)
    elif w.bias == "u0.01":
        out["b"] = uniform((w.E,), s, TID_B, -0.01, 0.01)
    elif w.bias == "zipf1.2":
        out["b"] = zipf_bias(w.E, 1.2)
    elif w.bias == "zero":
        out["b"] = torch.zeros(w.E, dtype=torch.float32)
    else:
        raise ValueError(w.bias)
    if with_experts:
        out["W_gate"] = normal((w.E, w.d_ff, w.d), s, TID_WG, 0.0, 1.0 / math.sqrt(w.d), w.w_dtype)
        out["W_up"] = normal((w.E, w.d_ff, w.d), s, TID_WU, 0.0, 1.0 / math.sqrt(w.d), w.w_dtype)
        out["W_down"] = normal((w.E, w.d, w.d_ff), s, TID_WD, 0.0, 1.0 / math.sqrt(w.d_ff), w.w_dtype)
    return out
