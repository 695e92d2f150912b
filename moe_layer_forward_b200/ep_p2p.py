"""Expert-parallel layer forward with the exchanges fused into the dispatch and
combine kernels (peer memory instead of All-to-All copies).

"「赤兔」Chitu 框架深度解读（七）", §Token 分发策略, and "推理计算流梳理", §EP 路径:
every routed (token, expert) row travels to the expert's rank, the experts run
there, and the outputs are summed with the router weights at the token's
source.  Here the travel is done by the kernels themselves:

  1-3. RMSNorm, router top-k and the permutation maps on the rank's own tokens
       (no local row copy);
  4.   the per-expert counts of every rank are gathered into one [N][E] table
       (a small all-gather);
  5.   ``moe_ep_dispatch``: the permutation's row copy stores each routed row
       straight into its owner's receive buffer, at the row the table fixes
       (expert-major, then source rank, then token order: the grouped GEMM's
       contiguous layout, so the receiver needs no second permutation);
  6.   barrier (every rank's rows have landed);
  7.   ``moe_ep_layout`` + ``moe_grouped_swiglu`` on the receive buffer, into the
       rank's expert output buffer;
  8.   barrier (every rank's outputs are ready);
  9.   ``moe_ep_combine``: step 5 reading each pick's output row from its owner
       (peer loads), weighted in pick order, plus the residual.

Rank r of N owns experts [r E/N, (r+1) E/N).  The buffers are sized for the
worst case, N * T_max * min(k, E/N) rows (a token's k picks are distinct
experts, at most E/N of them on one rank), and the expert MLP runs over the
whole buffer with its counts on the device (``moe_grouped_swiglu_sized``, tile
form chosen for the rank's own slot count, which is what a rank receives on
average), so no count ever reaches the host: the step has no host
synchronisation and can be captured in a CUDA graph.

``ops`` and ``peers`` are parameters: on GPUs the library's kernels and
peer-mapped buffers (``symmetric_peers`` over NVLink, or ``local_peers`` when
all ranks live in one process); the tests also run the same driver on CPU
ranks with shared-memory tensors standing in for peer memory.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch
import torch.distributed as dist

from .ep import CudaOps, EPStats


def capacity_rows(T_max: int, N: int, k: int, E: int) -> int:
    """Rows a rank's receive buffer needs when no rank has more than T_max tokens."""
    return N * T_max * min(k, E // N)


@dataclass
class Peers:
    """Every rank's receive and expert-output buffers, as this process sees them.

    recv / y: this rank's buffers ([rows][d]); recv_list / y_list: all ranks' buffers as tensors when they
    live in this process (emulation, CPU tests), else None; recv_ptrs / y_ptrs: int64 [N] device tensors of
    the buffers' addresses as mapped in this process (GPU kernels), else None."""
    recv: torch.Tensor
    y: torch.Tensor
    recv_list: list | None = None
    y_list: list | None = None
    recv_ptrs: torch.Tensor | None = None
    y_ptrs: torch.Tensor | None = None

    @property
    def rows(self) -> int:
        return self.recv.shape[0]


def local_peers(N: int, rows: int, d: int, dtype, device) -> list[Peers]:
    """All N ranks' buffers in this process (on one device): one Peers view per rank."""
    recv = [torch.empty((rows, d), dtype=dtype, device=device) for _ in range(N)]
    y = [torch.empty((rows, d), dtype=dtype, device=device) for _ in range(N)]
    rp = yp = None
    if torch.device(device).type == "cuda":
        rp = torch.tensor([t.data_ptr() for t in recv], dtype=torch.int64, device=device)
        yp = torch.tensor([t.data_ptr() for t in y], dtype=torch.int64, device=device)
    return [Peers(recv[r], y[r], recv, y, rp, yp) for r in range(N)]


def symmetric_peers(rows: int, d: int, dtype, device, group=None) -> Peers:
    """This rank's buffers in torch symmetric memory, with every peer's address mapped over NVLink.

    Collective over ``group``: every rank calls it with the same rows, d and dtype."""
    from torch.distributed import _symmetric_memory as symm_mem

    group = group or dist.group.WORLD
    name = group.group_name

    def one():
        t = symm_mem.empty((rows, d), dtype=dtype, device=device)
        h = symm_mem.rendezvous(t, name)
        base = h.buffer_ptrs[h.rank]
        ptrs = [p + (t.data_ptr() - base) for p in h.buffer_ptrs]  # same offset in every rank's allocation
        return t, torch.tensor(ptrs, dtype=torch.int64, device=device)

    recv, rp = one()
    y, yp = one()
    return Peers(recv, y, None, None, rp, yp)


class CudaP2POps(CudaOps):
    """The library's kernels for the peer-memory exchange (asynchronous on the current stream)."""

    def permute_maps(self, v, idx, E):
        T, k = idx.shape
        dev = v.device
        counts = torch.empty(E, dtype=torch.int32, device=dev)
        offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
        slot_token = torch.empty(T * k, dtype=torch.int32, device=dev)
        token_slot = torch.empty((T, k), dtype=torch.int32, device=dev)
        if T > 0:
            self.m.moe_permute(v, idx, E, counts, offsets, slot_token, token_slot, None)
        else:
            counts.zero_()
            offsets.zero_()
        return counts, offsets, token_slot

    def dispatch(self, v, idx, token_slot, offsets, table, rank, peers: Peers):
        self.m.moe_ep_dispatch(v, idx, token_slot, offsets, table, rank, peers.recv_ptrs, peers.rows)

    def layout(self, table, rank):
        N, E = table.shape
        counts_loc = torch.empty(E // N, dtype=torch.int32, device=table.device)
        offsets_loc = torch.empty(E // N + 1, dtype=torch.int32, device=table.device)
        self.m.moe_ep_layout(table, rank, counts_loc, offsets_loc)
        return counts_loc, offsets_loc

    def expert_mlp(self, xp, W_gate, W_up, W_down, counts, offsets, y, S_expected):
        """The grouped MLP over a whole receive buffer; counts/offsets on the device pick the rows."""
        S = xp.shape[0]
        if S > 0:
            h = torch.empty((S, W_gate.shape[1]), dtype=xp.dtype, device=xp.device)
            self.m.moe_grouped_swiglu_sized(xp, W_gate, W_up, W_down, counts, offsets, h, y,
                                            max(1, min(S_expected, S)))

    def combine_pull(self, peers: Peers, idx, token_slot, offsets, table, rank, w, residual, out_dtype):
        out = torch.empty(residual.shape, dtype=out_dtype, device=residual.device)
        if residual.shape[0] > 0:
            self.m.moe_ep_combine(peers.y_ptrs, peers.y.dtype, idx, token_slot, offsets, table, rank, w, residual,
                                  out, peers.rows)
        return out


@dataclass
class _Route:
    idx: torch.Tensor
    w: torch.Tensor
    vx: torch.Tensor
    counts: torch.Tensor
    offsets: torch.Tensor
    token_slot: torch.Tensor


def _route(ops, x, gamma, W_r, b, E, top_k, eps, dtype) -> _Route:
    vx = ops.rmsnorm(x, gamma, eps, dtype)
    idx, w = ops.route(x, gamma, eps, W_r, b, top_k)
    counts, offsets, token_slot = ops.permute_maps(vx, idx, E)
    return _Route(idx, w, vx, counts, offsets, token_slot)


def _barrier(group, device):
    # a one-element all-reduce: ordered on the stream after this rank's preceding kernels, complete on every
    # rank only once all ranks reached it (no host wait on GPUs)
    dist.all_reduce(torch.zeros(1, device=device), group=group)


def ep_p2p_forward(x, gamma, W_r, b, W_gate_local, W_up_local, W_down_local, E: int, peers: Peers, T_max: int,
                   top_k: int = 8, eps: float = 1e-5, group=None, ops=None, out_dtype=None, agree_checks=True):
    """out = x + MoE(RMSNorm(x)) for this rank's tokens (one process per rank; collectives inside).

    W_*_local hold experts [rank E/N, (rank+1) E/N); peers holds buffers of at least
    capacity_rows(T_max, N, top_k, E) rows on every rank.  Returns (out, EPStats); the stats' rows_received
    is a one-element device tensor.

    With agree_checks (the default) the ranks first combine their argument checks in one all-reduce (MIN of
    a pass flag) and read it on the host: if any rank fails a check, every rank raises ValueError together
    and none is left waiting in a collective that a failed rank never joins.  That read is the step's one
    host synchronisation; a caller that has validated its arguments once (e.g. before capturing the step in
    a CUDA graph) passes agree_checks=False, and then a rank that fails a check raises alone while the
    others' next collective ends with the process group's timeout error."""
    ops = ops or CudaP2POps()
    N = dist.get_world_size(group)
    rank = dist.get_rank(group)
    problem = None
    if E % N != 0:
        problem = f"{E} experts do not split over {N} ranks"
    elif W_gate_local.shape[0] != E // N:
        problem = f"rank {rank} holds {W_gate_local.shape[0]} experts, expected {E // N}"
    elif x.shape[0] > T_max:
        problem = f"rank {rank} has {x.shape[0]} tokens, more than T_max = {T_max}"
    elif peers.rows < capacity_rows(T_max, N, top_k, E):
        problem = f"peer buffers hold {peers.rows} rows, {capacity_rows(T_max, N, top_k, E)} needed"
    if agree_checks:
        ok = torch.tensor([0 if problem else 1], dtype=torch.int32, device=x.device)
        dist.all_reduce(ok, op=dist.ReduceOp.MIN, group=group)
        if problem is None and int(ok.item()) == 0:
            problem = "another rank failed its argument checks (T_max, buffer rows or expert split)"
    if problem is not None:
        raise ValueError(problem)
    E_loc = E // N
    dev = x.device
    rt = _route(ops, x, gamma, W_r, b, E, top_k, eps, W_gate_local.dtype)

    table = torch.empty((N, E), dtype=torch.int32, device=dev)
    dist.all_gather(list(table.unbind(0)), rt.counts, group=group)
    ops.dispatch(rt.vx, rt.idx, rt.token_slot, rt.offsets, table, rank, peers)
    _barrier(group, dev)

    counts_loc, offsets_loc = ops.layout(table, rank)
    ops.expert_mlp(peers.recv, W_gate_local, W_up_local, W_down_local, counts_loc, offsets_loc, peers.y,
                   int(x.shape[0]) * top_k)
    _barrier(group, dev)

    out = ops.combine_pull(peers, rt.idx, rt.token_slot, rt.offsets, table, rank, rt.w, x, out_dtype or x.dtype)
    return out, EPStats(rows_sent=int(x.shape[0]) * top_k, rows_received=offsets_loc[E_loc:])


def ep_p2p_forward_emulated(x_shards, gamma, W_r, b, W_gate, W_up, W_down, top_k: int = 8, eps: float = 1e-5,
                            ops=None, out_dtype=None, peers=None):
    """All N = len(x_shards) ranks in this process: the same steps as ep_p2p_forward, phase by phase.

    Rank r's tokens are x_shards[r]; it owns experts [r E/N, (r+1) E/N) of the full weights.  The phases
    follow one another in stream order, so no rank's kernel waits for another's.  Returns the N outputs."""
    ops = ops or CudaP2POps()
    N = len(x_shards)
    E, d = W_gate.shape[0], x_shards[0].shape[1]
    if E % N != 0:
        raise ValueError(f"{E} experts do not split over {N} ranks")
    E_loc = E // N
    dev = x_shards[0].device
    if peers is None:
        T_max = max(int(x.shape[0]) for x in x_shards)
        peers = local_peers(N, max(capacity_rows(T_max, N, top_k, E), 1), d, W_gate.dtype, dev)
    routes = [_route(ops, x, gamma, W_r, b, E, top_k, eps, W_gate.dtype) for x in x_shards]
    table = torch.stack([rt.counts for rt in routes])  # what the all-gather gives every rank
    for r, rt in enumerate(routes):
        ops.dispatch(rt.vx, rt.idx, rt.token_slot, rt.offsets, table, r, peers[r])
    for j in range(N):
        counts_loc, offsets_loc = ops.layout(table, j)
        sl = slice(j * E_loc, (j + 1) * E_loc)
        ops.expert_mlp(peers[j].recv, W_gate[sl], W_up[sl], W_down[sl], counts_loc, offsets_loc, peers[j].y,
                       int(x_shards[j].shape[0]) * top_k)
    return [ops.combine_pull(peers[r], rt.idx, rt.token_slot, rt.offsets, table, r, rt.w, x_shards[r],
                             out_dtype or x_shards[r].dtype) for r, rt in enumerate(routes)]
