"""The peer-memory expert-parallel driver (moe_layer_forward_b200.ep_p2p) on
CPU ranks.

ep_p2p_forward runs unchanged on 2 and 4 gloo ranks: the count all-gather and
the barriers are real collectives, and the "peer memory" is a set of
shared-memory CPU tensors that every rank process writes into (dispatch) and
reads from (combine).  The ops are the fp64 oracle's steps plus a dispatch and
a combine that place rows by enumerating the layout (expert, then source rank,
then the source's slot order), so the merged outputs must equal the
single-process layer exactly, and every row must land where the layout says.
"""
import os
import socket
import sys
import tempfile

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _inputs():
    sys.path.insert(0, ROOT)
    import synth

    w = synth.Workload("ep_p2p", 24, 256, 16, 128, x_dtype=torch.float32, w_dtype=torch.float32,
                       out_dtype=torch.float32, seed=47)
    return w, synth.make_layer_inputs(w)


def _start(table, j, E_loc):
    N = table.shape[0]
    pos, start = 0, {}
    for e in range(j * E_loc, (j + 1) * E_loc):
        for r in range(N):
            start[(r, e)] = pos
            pos += int(table[r, e])
    return start


def _p2p_ops():
    from test_ep_gloo import OracleOps

    class P2POracleOps(OracleOps):
        def permute_maps(self, v, idx, E):
            counts, offsets, _, token_slot = self.o.permute(idx, E)
            return counts.to(torch.int32), offsets.to(torch.int32), token_slot.to(torch.int32)

        def dispatch(self, v, idx, token_slot, offsets, table, rank, peers):
            E_loc = table.shape[1] // table.shape[0]
            for t in range(idx.shape[0]):
                for i in range(idx.shape[1]):
                    e, s = int(idx[t, i]), int(token_slot[t, i])
                    j = e // E_loc
                    peers.recv_list[j][_start(table, j, E_loc)[(rank, e)] + s - int(offsets[e])] = v[t]

        def layout(self, table, rank):
            N, E = table.shape
            E_loc = E // N
            counts = table[:, rank * E_loc:(rank + 1) * E_loc].sum(0).to(torch.int32)
            offsets = torch.zeros(E_loc + 1, dtype=torch.int32)
            offsets[1:] = torch.cumsum(counts, 0)
            return counts, offsets

        def expert_mlp(self, xp, W_gate, W_up, W_down, counts, offsets, y, S_expected):
            R = int(offsets[-1])
            if R:
                y[:R].copy_(self.grouped_swiglu(xp[:R], W_gate, W_up, W_down, counts, offsets))

        def combine_pull(self, peers, idx, token_slot, offsets, table, rank, w, residual, out_dtype):
            E_loc = table.shape[1] // table.shape[0]
            out = torch.empty(residual.shape, dtype=torch.float64)
            for t in range(idx.shape[0]):
                acc = torch.zeros(residual.shape[1], dtype=torch.float64)
                for i in range(idx.shape[1]):  # pick order
                    e, s = int(idx[t, i]), int(token_slot[t, i])
                    j = e // E_loc
                    acc = acc + float(w[t, i]) * peers.y_list[j][_start(table, j, E_loc)[(rank, e)] + s - int(offsets[e])]
                out[t] = residual[t].double() + acc
            return out.to(out_dtype)

    return P2POracleOps()


def _worker(rank, world, port, outdir, recv, y):
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import datetime

    import torch.distributed as dist

    from moe_layer_forward_b200 import ep_p2p

    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    w, I = _inputs()
    E_loc = w.E // world
    experts = slice(rank * E_loc, (rank + 1) * E_loc)
    x = I["x"].chunk(world)[rank].contiguous()
    T_max = max(c.shape[0] for c in I["x"].chunk(world))
    peers = ep_p2p.Peers(recv[rank], y[rank], recv, y)
    out, stats = ep_p2p.ep_p2p_forward(x, I["gamma"], I["W_r"], I["b"], I["W_gate"][experts], I["W_up"][experts],
                                       I["W_down"][experts], E=w.E, peers=peers, T_max=T_max, top_k=w.top_k,
                                       eps=w.eps, ops=_p2p_ops())
    torch.save({"out": out, "received": int(stats.rows_received)}, os.path.join(outdir, f"r{rank}.pt"))
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_peer_memory_expert_parallel_layer_equals_the_single_process_layer(world):
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    from moe_layer_forward_b200 import ep_p2p
    from test_ep_gloo import OracleOps

    w, I = _inputs()
    ops = OracleOps()
    v32 = ops.rmsnorm(I["x"], I["gamma"], w.eps, torch.float32)
    idx, wt = ops.router(v32, I["W_r"], I["b"], w.top_k)
    counts, offsets, token_slot, xp = ops.permute(v32, idx, w.E)
    ref = ops.combine(ops.grouped_swiglu(xp, I["W_gate"], I["W_up"], I["W_down"], counts, offsets), token_slot, wt,
                      I["x"], torch.float32)
    T_max = max(c.shape[0] for c in I["x"].chunk(world))
    rows = ep_p2p.capacity_rows(T_max, world, w.top_k, w.E)
    recv = [torch.full((rows, w.d), float("nan"), dtype=torch.float32).share_memory_() for _ in range(world)]
    y = [torch.full((rows, w.d), float("nan"), dtype=torch.float64).share_memory_() for _ in range(world)]
    with tempfile.TemporaryDirectory() as d:
        mp.start_processes(_worker, args=(world, _free_port(), d, recv, y), nprocs=world, join=True,
                           start_method="spawn")
        r = [torch.load(os.path.join(d, f"r{k}.pt")) for k in range(world)]
    assert torch.equal(torch.cat([x["out"] for x in r]), ref)
    assert sum(x["received"] for x in r) == w.T * w.top_k
    # every received row is the normalised row of its token; nothing past the received rows was written
    for j in range(world):
        R = r[j]["received"]
        assert not torch.isnan(recv[j][:R]).any() and torch.isnan(recv[j][R:]).all()


def test_capacity_covers_the_worst_case():
    from moe_layer_forward_b200 import ep_p2p

    # every token of every rank sends min(k, E/N) rows to one rank at most
    assert ep_p2p.capacity_rows(10, 4, 8, 16) == 4 * 10 * 4
    assert ep_p2p.capacity_rows(10, 2, 8, 64) == 2 * 10 * 8


def _failing_worker(rank, world, port, outdir, recv, y, agree):
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import datetime

    import torch.distributed as dist

    from moe_layer_forward_b200 import ep_p2p

    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=5))
    w, I = _inputs()
    E_loc = w.E // world
    experts = slice(rank * E_loc, (rank + 1) * E_loc)
    x = I["x"].chunk(world)[rank].contiguous()
    T_max = x.shape[0] - (1 if rank == 1 else 0)  # rank 1 holds one token more than the buffers were sized for
    outcome = "returned"
    try:
        ep_p2p.ep_p2p_forward(x, I["gamma"], I["W_r"], I["b"], I["W_gate"][experts], I["W_up"][experts],
                              I["W_down"][experts], E=w.E, peers=ep_p2p.Peers(recv[rank], y[rank], recv, y),
                              T_max=T_max, top_k=w.top_k, eps=w.eps, ops=_p2p_ops(), agree_checks=agree)
    except ValueError as e:
        outcome = "ValueError: " + str(e)
    except RuntimeError as e:  # the collective that the failed rank never joins
        outcome = "RuntimeError"
    torch.save({"outcome": outcome}, os.path.join(outdir, f"r{rank}.pt"))


@pytest.mark.parametrize("agree", [True, False])
def test_a_rank_that_fails_its_checks_stops_every_rank(agree):
    # with the checks agreed in one all-reduce every rank raises ValueError together; without it the
    # failing rank raises alone and the other's next collective ends with the group's timeout error
    from moe_layer_forward_b200 import ep_p2p

    world = 2
    w, I = _inputs()
    rows = ep_p2p.capacity_rows(w.T // world, world, w.top_k, w.E)
    recv = [torch.zeros((rows, w.d), dtype=torch.float32).share_memory_() for _ in range(world)]
    y = [torch.zeros((rows, w.d), dtype=torch.float64).share_memory_() for _ in range(world)]
    with tempfile.TemporaryDirectory() as d:
        mp.start_processes(_failing_worker, args=(world, _free_port(), d, recv, y, agree), nprocs=world,
                           join=True, start_method="spawn")
        r = [torch.load(os.path.join(d, f"r{k}.pt"))["outcome"] for k in range(world)]
    assert r[1].startswith("ValueError") and "T_max" in r[1]
    if agree:
        assert r[0].startswith("ValueError") and "another rank" in r[0]
    else:
        assert r[0] == "RuntimeError"
