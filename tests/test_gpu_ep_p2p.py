"""Expert parallelism over peer memory (moe_ep_dispatch, moe_ep_layout,
moe_ep_combine) on one GPU.

N ranks are emulated in one process, each with its own receive and output
buffers on the GPU, the phases run one after another (no kernel waits for
another).  Checks:
  - one rank: the layer equals moe_forward bit for bit (same routing, the
    receive buffer is the permutation's row order, same GEMM, same combine);
  - 2 and 4 ranks: every receive buffer holds exactly the rows the layout
    rule puts there (rebuilt here by enumerating (expert, source rank, row));
    every rank's output equals moe_unpermute_combine over the expert rows
    gathered by that layout, bit for bit; the layer is within the parity
    tolerances of the fp64 oracle on the GPU's routing;
  - the per-rank driver (NCCL group of one, spawned) equals moe_forward;
  - two emulated ranks replay from a CUDA graph (no host synchronisation).
"""
import os
import socket
import sys
import tempfile

import pytest
import torch
import torch.multiprocessing as mp

import oracle
import synth
from _layer_check import MAX_ABS, REL_L2, errors

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def moe():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import moe_layer_forward_b200 as m

    return m


def _inputs(shape, seed):
    T, d, E, d_ff = shape
    w = synth.Workload("ep_p2p", T, d, E, d_ff, seed=seed)
    I = synth.make_layer_inputs(w)
    return w, I, {n: t.to(DEV) for n, t in I.items()}


def _layout_start(table, j, E_loc):
    """(source rank, expert) -> first row of that segment on owner j, by enumeration."""
    N = table.shape[0]
    pos, start = 0, {}
    for e in range(j * E_loc, (j + 1) * E_loc):
        for r in range(N):
            start[(r, e)] = pos
            pos += int(table[r, e])
    return start, pos


@pytest.mark.parametrize("shape", [(96, 512, 64, 256), (1200, 256, 8, 256)])  # weights-as-M; CTA pairs
def test_one_rank_equals_moe_forward(moe, shape):
    from moe_layer_forward_b200 import ep_p2p

    w, I, D = _inputs(shape, 960)
    outs = ep_p2p.ep_p2p_forward_emulated([D["x"]], D["gamma"], D["W_r"], D["b"], D["W_gate"], D["W_up"],
                                          D["W_down"], top_k=w.top_k, eps=w.eps)
    ref = torch.empty_like(outs[0])
    moe.moe_forward(D["x"], D["gamma"], D["W_r"], D["b"], D["W_gate"], D["W_up"], D["W_down"], ref, top_k=w.top_k,
                    eps=w.eps)
    torch.cuda.synchronize()
    assert torch.equal(outs[0], ref)


@pytest.mark.parametrize("N", [2, 4])
@pytest.mark.parametrize("shape", [(96, 512, 64, 256), (300, 256, 16, 384)])
def test_ranks_exchange_exactly_and_match_the_oracle(moe, N, shape):
    from moe_layer_forward_b200 import ep_p2p

    w, I, D = _inputs(shape, 961)
    T, d, E, d_ff = shape
    E_loc = E // N
    shards = list(D["x"].chunk(N))
    ops = ep_p2p.CudaP2POps()
    T_max = max(x.shape[0] for x in shards)
    peers = ep_p2p.local_peers(N, ep_p2p.capacity_rows(T_max, N, w.top_k, E), d, D["W_gate"].dtype, DEV)
    outs = ep_p2p.ep_p2p_forward_emulated(shards, D["gamma"], D["W_r"], D["b"], D["W_gate"], D["W_up"], D["W_down"],
                                          top_k=w.top_k, eps=w.eps, ops=ops, peers=peers)
    # the same routing again (deterministic kernels) to rebuild what each buffer must hold
    routes = [ep_p2p._route(ops, x, D["gamma"], D["W_r"], D["b"], E, w.top_k, w.eps, D["W_gate"].dtype)
              for x in shards]
    torch.cuda.synchronize()
    table = torch.stack([rt.counts for rt in routes]).cpu()
    assert int(table.sum()) == T * w.top_k
    starts = [_layout_start(table, j, E_loc) for j in range(N)]
    for j in range(N):
        start, R = starts[j]
        want = torch.empty((R, d), dtype=D["W_gate"].dtype)
        for r, rt in enumerate(routes):
            idx, ts, off, vx = rt.idx.cpu(), rt.token_slot.cpu(), rt.offsets.cpu(), rt.vx.cpu()
            for t in range(idx.shape[0]):
                for i in range(w.top_k):
                    e = int(idx[t, i])
                    if e // E_loc == j:
                        want[start[(r, e)] + int(ts[t, i]) - int(off[e])] = vx[t]
        assert torch.equal(peers[j].recv[:R].cpu(), want), f"receive buffer of rank {j}"
    for r, rt in enumerate(routes):
        idx, ts, off = rt.idx.cpu(), rt.token_slot.cpu(), rt.offsets.cpu()
        rows = torch.empty(idx.shape[0] * w.top_k, d, dtype=D["W_gate"].dtype, device=DEV)
        for t in range(idx.shape[0]):
            for i in range(w.top_k):
                e, s = int(idx[t, i]), int(ts[t, i])
                j = e // E_loc
                rows[s] = peers[j].y[starts[j][0][(r, e)] + s - int(off[e])]
        ref = torch.empty_like(outs[r])
        moe.moe_unpermute_combine(rows, rt.token_slot, rt.w, shards[r], ref)
        torch.cuda.synchronize()
        assert torch.equal(outs[r], ref), f"output of rank {r}"
    # the layer: the oracle on the GPU's routing
    idx = torch.cat([rt.idx.cpu() for rt in routes])
    wt = torch.cat([rt.w.cpu() for rt in routes])
    args = (I["gamma"], I["W_r"], I["b"], I["W_gate"], I["W_up"], I["W_down"])
    forced = oracle.moe_layer(I["x"], *args, k=w.top_k, eps=w.eps, force_idx=idx, force_w=wt)
    max_abs, rel = errors(torch.cat([o.cpu() for o in outs]), forced["out"])
    assert max_abs <= MAX_ABS and rel <= REL_L2, (max_abs, rel)


def test_two_ranks_replay_from_a_cuda_graph(moe):
    # the step has no host synchronisation: captured once, a replay reproduces the eager result, also after a
    # replay on other inputs
    from moe_layer_forward_b200 import ep_p2p

    w, I, D = _inputs((96, 512, 64, 256), 980)
    N = 2
    shards = [s.contiguous() for s in D["x"].chunk(N)]  # views of D["x"]
    peers = ep_p2p.local_peers(N, ep_p2p.capacity_rows(48, N, 8, 64), 512, torch.bfloat16, DEV)
    args = (D["gamma"], D["W_r"], D["b"], D["W_gate"], D["W_up"], D["W_down"])
    eager = [o.clone() for o in ep_p2p.ep_p2p_forward_emulated(shards, *args, peers=peers)]
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        ep_p2p.ep_p2p_forward_emulated(shards, *args, peers=peers)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        outs = ep_p2p.ep_p2p_forward_emulated(shards, *args, peers=peers)
    saved = [x.clone() for x in shards]
    for x in shards:
        x.zero_()
    g.replay()
    for x, src in zip(shards, saved):
        x.copy_(src)
    g.replay()
    torch.cuda.synchronize()
    assert all(torch.equal(a, b) for a, b in zip(outs, eager))
    del g


def test_sized_grouped_mlp_equals_the_exact_call(moe):
    # a buffer of S_cap rows of which the counts use S: the same rows as moe_grouped_swiglu on exactly S rows,
    # and the rows past the segments are left as they were
    S, S_cap, d, d_ff = 200, 256, 256, 384
    counts = torch.tensor([30, 0, 7, 41, 12, 1, 50, 59], dtype=torch.int32)
    E = counts.numel()
    offsets = torch.zeros(E + 1, dtype=torch.int32)
    offsets[1:] = torch.cumsum(counts, 0)
    assert int(offsets[-1]) == S
    W = [synth.normal((E, n, kk), 970, 5 + i, 0.0, 1 / kk ** 0.5, torch.bfloat16).to(DEV)
         for i, (n, kk) in enumerate([(d_ff, d), (d_ff, d), (d, d_ff)])]
    xp = torch.full((S_cap, d), float("nan"), dtype=torch.bfloat16, device=DEV)
    xp[:S] = synth.normal((S, d), 970, 1, dtype=torch.bfloat16).to(DEV)
    c, o = counts.to(DEV), offsets.to(DEV)
    h_ref = torch.empty((S, d_ff), dtype=torch.bfloat16, device=DEV)
    y_ref = torch.empty((S, d), dtype=torch.bfloat16, device=DEV)
    moe.moe_grouped_swiglu(xp[:S].contiguous(), *W, c, o, h_ref, y_ref)
    h = torch.empty((S_cap, d_ff), dtype=torch.bfloat16, device=DEV)
    y = torch.full((S_cap, d), 7.0, dtype=torch.bfloat16, device=DEV)
    moe.moe_grouped_swiglu_sized(xp, *W, c, o, h, y, S)
    torch.cuda.synchronize()
    assert torch.equal(y[:S], y_ref)
    assert (y[S:] == 7.0).all()


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _driver_worker(rank, port, outdir, shape):
    sys.path.insert(0, ROOT)
    import datetime

    import torch.distributed as dist

    import moe_layer_forward_b200 as m
    from moe_layer_forward_b200 import ep_p2p

    torch.cuda.set_device(0)
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60), device_id=torch.device("cuda", 0))
    w, I, D = _inputs(shape, 962)
    T, d, E, d_ff = shape
    peers = ep_p2p.local_peers(1, ep_p2p.capacity_rows(T, 1, w.top_k, E), d, D["W_gate"].dtype, DEV)[0]
    out, stats = ep_p2p.ep_p2p_forward(D["x"], D["gamma"], D["W_r"], D["b"], D["W_gate"], D["W_up"], D["W_down"],
                                       E=E, peers=peers, T_max=T, top_k=w.top_k, eps=w.eps)
    ref = torch.empty_like(out)
    m.moe_forward(D["x"], D["gamma"], D["W_r"], D["b"], D["W_gate"], D["W_up"], D["W_down"], ref, top_k=w.top_k,
                  eps=w.eps)
    torch.cuda.synchronize()
    torch.save({"equal": torch.equal(out, ref), "rows": int(stats.rows_received)}, os.path.join(outdir, "r.pt"))
    dist.destroy_process_group()


def test_per_rank_driver_single_rank_equals_moe_forward(moe):
    shape = (96, 512, 64, 256)
    with tempfile.TemporaryDirectory() as d:
        mp.start_processes(_driver_worker, args=(_free_port(), d, shape), nprocs=1, join=True, start_method="spawn")
        r = torch.load(os.path.join(d, "r.pt"))
    assert r["equal"] and r["rows"] == shape[0] * 8
