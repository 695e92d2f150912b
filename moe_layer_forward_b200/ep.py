"""Expert-parallel layer forward: the MoE layer with its experts split across ranks.

"「赤兔」Chitu 框架深度解读（七）", §Token 分发策略: with expert parallelism each
rank holds a subset of the experts; a dispatcher sends every (token, expert)
pair's row to the rank that owns the expert (All-to-All), the experts run
there, and the results travel back to be summed at the token's source
(token_unpermutation).  "推理计算流梳理", §EP 路径: the same exchange around the
grouped GEMM, weighted sum at the source.

Rank r of N owns experts [r * E/N, (r+1) * E/N) (E divisible by N) and the rows
of its own tokens.  One step:

  1. v = RMSNorm(x) in fp32 (for the router) and in the expert dtype;
  2. router top-k on the fp32 rows;
  3. permutation of the (token, k) pairs into expert order; experts are
     rank-contiguous, so this is also destination-rank order;
  4. All-to-All of the per-expert counts, then of the rows (counts reach the
     host here: they size the exchange);
  5. a second permutation of the received rows into local-expert order
     (stable: within an expert, source rank then source order);
  6. grouped SwiGLU MLP of the local experts;
  7. the k = 1 un-permutation back to arrival order, the reverse All-to-All,
     and the weighted combine with the residual at the source.

All arithmetic runs in the library's kernels (through ``ops``); the exchange is
``torch.distributed.all_to_all_single`` (NCCL on GPUs).  ``ops`` is a parameter
so that the orchestration can also be run on CPU ranks in tests.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch
import torch.distributed as dist


@dataclass
class EPStats:
    rows_sent: int
    rows_received: int


class CudaOps:
    """The library's kernels on CUDA tensors (asynchronous on the current stream)."""

    def __init__(self):
        import moe_layer_forward_b200 as m

        self.m = m

    def rmsnorm(self, x, gamma, eps, dtype):
        v = torch.empty(x.shape, dtype=dtype, device=x.device)
        self.m.moe_rmsnorm(x, gamma, eps, v)
        return v

    def route(self, x, gamma, eps, W_r, b, k):
        """the routing of moe_forward (RMSNorm folded into the router), bit for bit"""
        T = x.shape[0]
        idx = torch.empty((T, k), dtype=torch.int32, device=x.device)
        w = torch.empty((T, k), dtype=torch.float32, device=x.device)
        if T > 0:
            self.m.moe_route(x, gamma, W_r, b, idx, w, eps)
        return idx, w

    def router(self, v32, W_r, b, k):
        T = v32.shape[0]
        idx = torch.empty((T, k), dtype=torch.int32, device=v32.device)
        w = torch.empty((T, k), dtype=torch.float32, device=v32.device)
        self.m.moe_router_topk(v32, W_r, b, idx, w)
        return idx, w

    def permute(self, v, idx, E):
        T, k = idx.shape
        dev = v.device
        counts = torch.empty(E, dtype=torch.int32, device=dev)
        offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
        slot_token = torch.empty(T * k, dtype=torch.int32, device=dev)
        token_slot = torch.empty((T, k), dtype=torch.int32, device=dev)
        xp = torch.empty((T * k, v.shape[1]), dtype=v.dtype, device=dev)
        if T > 0:
            self.m.moe_permute(v, idx, E, counts, offsets, slot_token, token_slot, xp)
        else:
            counts.zero_()
            offsets.zero_()
        return counts, offsets, token_slot, xp

    def grouped_swiglu(self, xp, W_gate, W_up, W_down, counts, offsets):
        S, d = xp.shape
        h = torch.empty((S, W_gate.shape[1]), dtype=xp.dtype, device=xp.device)
        y = torch.empty((S, d), dtype=xp.dtype, device=xp.device)
        if S > 0:
            self.m.moe_grouped_swiglu(xp, W_gate, W_up, W_down, counts, offsets, h, y)
        return y

    def combine(self, y, token_slot, w, residual, out_dtype):
        out = torch.empty(residual.shape, dtype=out_dtype, device=residual.device)
        if residual.shape[0] > 0:
            self.m.moe_unpermute_combine(y, token_slot, w, residual, out)
        return out


def ep_forward(x, gamma, W_r, b, W_gate_local, W_up_local, W_down_local, E: int, top_k: int = 8,
               eps: float = 1e-5, group=None, ops=None, out_dtype=None):
    """out = x + MoE(RMSNorm(x)) for this rank's tokens, with this rank's slice of the experts.

    W_*_local hold the experts [rank * E/N, (rank+1) * E/N) of the full [E][...] tensors.
    Returns (out, EPStats).  Every rank of ``group`` must call it (collectives inside).
    """
    ops = ops or CudaOps()
    N = dist.get_world_size(group)
    rank = dist.get_rank(group)
    if E % N != 0:
        raise ValueError(f"{E} experts do not split over {N} ranks")
    E_loc = E // N
    if W_gate_local.shape[0] != E_loc:
        raise ValueError(f"rank {rank} holds {W_gate_local.shape[0]} experts, expected {E_loc}")
    dev = x.device
    out_dtype = out_dtype or x.dtype
    d = x.shape[1]

    # 1-3: local routing and dispatch order
    vx = ops.rmsnorm(x, gamma, eps, W_gate_local.dtype)
    idx, w = ops.route(x, gamma, eps, W_r, b, top_k)
    counts, _, token_slot, xp = ops.permute(vx, idx, E)

    # 4: counts, then rows
    recv_counts = torch.empty(E, dtype=torch.int32, device=dev)  # [source rank][local expert]
    dist.all_to_all_single(recv_counts, counts.contiguous(), group=group)
    send_splits = counts.view(N, E_loc).sum(1).tolist()
    rc = recv_counts.view(N, E_loc).cpu()
    recv_splits = rc.sum(1).tolist()
    R = int(sum(recv_splits))
    recv = torch.empty((R, d), dtype=xp.dtype, device=dev)
    dist.all_to_all_single(recv, xp, output_split_sizes=recv_splits, input_split_sizes=send_splits, group=group)

    # 5: local expert order of the received rows (source rank major in the arrival order)
    local_e = torch.repeat_interleave(torch.arange(E_loc, dtype=torch.int32).repeat(N), rc.flatten().long())
    idx_loc = local_e.to(dev).view(R, 1)
    counts_loc, offsets_loc, slot_of_arrival, xp_loc = ops.permute(recv, idx_loc, E_loc)

    # 6: the local experts
    y_loc = ops.grouped_swiglu(xp_loc, W_gate_local, W_up_local, W_down_local, counts_loc, offsets_loc)

    # 7: back to arrival order (k = 1, weight 1, zero residual: an exact copy), home, and combine
    ones = torch.ones((R, 1), dtype=torch.float32, device=dev)
    y_arrival = ops.combine(y_loc, slot_of_arrival, ones, torch.zeros((R, d), dtype=y_loc.dtype, device=dev),
                            y_loc.dtype)
    y_home = torch.empty((xp.shape[0], d), dtype=y_loc.dtype, device=dev)
    dist.all_to_all_single(y_home, y_arrival, output_split_sizes=send_splits, input_split_sizes=recv_splits,
                           group=group)
    out = ops.combine(y_home, token_slot, w, x, out_dtype)
    return out, EPStats(rows_sent=int(sum(send_splits)), rows_received=R)
