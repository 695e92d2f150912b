"""Tensor-parallel experts: every expert's MLP split along d_ff across ranks.

"推理计算流梳理", §实际 MLP 计算策略: with tensor parallelism the gate and up
projections are split by columns (each rank holds a slice of the d_ff
features) and the down projection by rows (the matching slice of its input),
so each rank produces a partial sum of the output that one reduction
completes.  Applied here to every expert of the MoE layer.

Rank r of N holds W_gate[:, r*F:(r+1)*F, :], W_up[:, r*F:(r+1)*F, :] and
W_down[:, :, r*F:(r+1)*F] with F = d_ff / N (a multiple of 128).  Every rank
holds all tokens.  One step:

  1. RMSNorm, router top-k and the permutation, identical on every rank;
  2. the grouped SwiGLU MLP on the rank's d_ff slice: a partial y;
  3. the weighted combine of the partial y in fp32, with the residual added on
     rank 0 only, then one fp32 all-reduce (sum) across the ranks, and a cast
     to the output dtype.  With ``scatter=True`` the sum is a reduce-scatter
     over tokens instead: rank r receives tokens [r T/N, (r+1) T/N) (T
     divisible by N), the form that feeds a token-sharded next layer.

All arithmetic runs in the library's kernels (``ops``, as in ``ep``); the
reduction is ``torch.distributed.all_reduce`` (NCCL on GPUs).
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from .ep import CudaOps


def tp_forward(x, gamma, W_r, b, W_gate_slice, W_up_slice, W_down_slice, top_k: int = 8, eps: float = 1e-5,
               group=None, ops=None, out_dtype=None, scatter: bool = False):
    """out = x + MoE(RMSNorm(x)) with this rank's d_ff slice of every expert (collective over ``group``).

    scatter=False: every rank returns all T rows; scatter=True: rank r returns rows [r T/N, (r+1) T/N)."""
    ops = ops or CudaOps()
    rank = dist.get_rank(group)
    N = dist.get_world_size(group)
    if scatter and x.shape[0] % N != 0:
        raise ValueError(f"{x.shape[0]} tokens do not split over {N} ranks")
    E = W_gate_slice.shape[0]
    out_dtype = out_dtype or x.dtype
    if W_down_slice.shape[2] != W_gate_slice.shape[1]:
        raise ValueError("W_down's slice must match the gate/up feature slice")
    vx = ops.rmsnorm(x, gamma, eps, W_gate_slice.dtype)
    idx, w = ops.route(x, gamma, eps, W_r, b, top_k)
    counts, offsets, token_slot, xp = ops.permute(vx, idx, E)
    y_part = ops.grouped_swiglu(xp, W_gate_slice, W_up_slice, W_down_slice, counts, offsets)
    residual = x if rank == 0 else torch.zeros_like(x)
    part = ops.combine(y_part, token_slot, w, residual, torch.float32)
    if scatter:
        mine = torch.empty((x.shape[0] // N, part.shape[1]), dtype=part.dtype, device=part.device)
        dist.reduce_scatter_tensor(mine, part, op=dist.ReduceOp.SUM, group=group)
        return mine.to(out_dtype)
    dist.all_reduce(part, op=dist.ReduceOp.SUM, group=group)
    return part.to(out_dtype)


def tp_partials_emulated(x, gamma, W_r, b, W_gate, W_up, W_down, N: int, top_k: int = 8, eps: float = 1e-5,
                         ops=None):
    """All N ranks of tp_forward in this process, on one device: the N fp32 partial outputs, before the
    reduction.  Rank r runs the grouped MLP on the features [r F, (r+1) F) of every expert (F = d_ff / N,
    a multiple of 128) and the weighted combine of its partial y, with the residual on rank 0 only; their
    sum is the layer (the all-reduce), and rows [r T/N, (r+1) T/N) of the sum are rank r's block of the
    reduce-scatter.  The routing is computed once: it is identical on every rank."""
    ops = ops or CudaOps()
    E, d_ff, _ = W_gate.shape
    if d_ff % N != 0 or (d_ff // N) % 128 != 0:
        raise ValueError(f"d_ff = {d_ff} does not split over {N} ranks in multiples of 128")
    F = d_ff // N
    vx = ops.rmsnorm(x, gamma, eps, W_gate.dtype)
    idx, w = ops.route(x, gamma, eps, W_r, b, top_k)
    counts, offsets, token_slot, xp = ops.permute(vx, idx, E)
    parts = []
    for r in range(N):
        sl = slice(r * F, (r + 1) * F)
        y_part = ops.grouped_swiglu(xp, W_gate[:, sl].contiguous(), W_up[:, sl].contiguous(),
                                    W_down[:, :, sl].contiguous(), counts, offsets)
        residual = x if r == 0 else torch.zeros_like(x)
        parts.append(ops.combine(y_part, token_slot, w, residual, torch.float32))
    return parts, idx, w
