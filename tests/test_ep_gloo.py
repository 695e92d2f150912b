"""Expert- and tensor-parallel orchestration (moe_layer_forward_b200.ep, .tp)
on CPU ranks.

Expert parallel: the exchange logic (count and row All-to-Alls, the local
re-permutation, the way back) runs on 2 and 4 gloo ranks, each with its share
of the tokens and of the experts.  The steps are the fp64 oracle's (ops on CPU
tensors): every row is computed by the same arithmetic with or without expert
parallelism, so the concatenated outputs must equal the single-process layer
exactly.  Tensor parallel: each rank holds a d_ff slice of every expert; the
all-reduced result must equal the single-process layer up to the regrouping
of the down projection's sum.
"""
import os
import socket
import sys
import tempfile

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


class OracleOps:
    """The layer's steps from the oracle, on CPU tensors (test infrastructure)."""

    def __init__(self):
        import oracle

        self.o = oracle

    def rmsnorm(self, x, gamma, eps, dtype):
        return self.o.rmsnorm(x, gamma, eps).to(dtype)

    def router(self, v32, W_r, b, k):
        z = self.o.router_logits(v32.double(), W_r) if v32.shape[0] else torch.zeros((0, W_r.shape[0]))
        idx, w, _ = self.o.select_topk(z.float(), b, k)
        return idx, w.float()

    def route(self, x, gamma, eps, W_r, b, k):
        return self.router(self.rmsnorm(x, gamma, eps, torch.float32), W_r, b, k)

    def permute(self, v, idx, E):
        counts, offsets, slot_token, token_slot = self.o.permute(idx, E)
        return counts, offsets, token_slot, v[slot_token.long()]

    def grouped_swiglu(self, xp, W_gate, W_up, W_down, counts, offsets):
        if xp.shape[0] == 0:
            return torch.zeros((0, W_down.shape[1]), dtype=torch.float64)
        _, y = self.o.grouped_mlp(xp, counts, offsets, W_gate, W_up, W_down)
        return y

    def combine(self, y, token_slot, w, residual, out_dtype):
        k = token_slot.shape[1]
        ys = y[token_slot.long().flatten()].view(residual.shape[0], k, -1).double()
        acc = torch.zeros(residual.shape, dtype=torch.float64)
        for i in range(k):  # pick order
            acc = acc + w[:, i:i + 1].double() * ys[:, i]
        return (residual.double() + acc).to(out_dtype)


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _inputs():
    sys.path.insert(0, ROOT)
    import synth

    w = synth.Workload("ep", 24, 256, 16, 128, x_dtype=torch.float32, w_dtype=torch.float32,
                       out_dtype=torch.float32, seed=41)
    return w, synth.make_layer_inputs(w)


def _worker(rank, world, port, outdir):
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import datetime

    import torch.distributed as dist

    from moe_layer_forward_b200 import ep

    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    w, I = _inputs()
    E_loc = w.E // world
    experts = slice(rank * E_loc, (rank + 1) * E_loc)
    x = I["x"][rank::world].contiguous()  # an uneven share of tokens when T % world != 0
    out, stats = ep.ep_forward(x, I["gamma"], I["W_r"], I["b"], I["W_gate"][experts], I["W_up"][experts],
                               I["W_down"][experts], E=w.E, top_k=w.top_k, eps=w.eps, ops=OracleOps())
    torch.save({"out": out, "sent": stats.rows_sent, "received": stats.rows_received},
               os.path.join(outdir, f"r{rank}.pt"))
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_expert_parallel_layer_equals_the_single_process_layer(world):
    sys.path.insert(0, ROOT)
    w, I = _inputs()
    ops = OracleOps()
    # the same steps without expert parallelism
    v32 = ops.rmsnorm(I["x"], I["gamma"], w.eps, torch.float32)
    idx, wt = ops.router(v32, I["W_r"], I["b"], w.top_k)
    counts, offsets, token_slot, xp = ops.permute(v32, idx, w.E)
    y = ops.grouped_swiglu(xp, I["W_gate"], I["W_up"], I["W_down"], counts, offsets)
    ref = ops.combine(y, token_slot, wt, I["x"], torch.float32)
    with tempfile.TemporaryDirectory() as d:
        mp.start_processes(_worker, args=(world, _free_port(), d), nprocs=world, join=True, start_method="spawn")
        r = [torch.load(os.path.join(d, f"r{k}.pt")) for k in range(world)]
    merged = torch.empty_like(ref)
    for k in range(world):
        merged[k::world] = r[k]["out"]
    assert torch.equal(merged, ref)
    # every routed row leaves and comes back once
    assert sum(x["sent"] for x in r) == sum(x["received"] for x in r) == w.T * w.top_k


# --------------------------------------------------------------------------- tensor-parallel experts
def _tp_inputs():
    sys.path.insert(0, ROOT)
    import synth

    w = synth.Workload("tp", 20, 256, 8, 512, x_dtype=torch.float32, w_dtype=torch.float32,
                       out_dtype=torch.float32, seed=43)
    return w, synth.make_layer_inputs(w)


def _tp_worker(rank, world, port, outdir):
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import datetime

    import torch.distributed as dist

    from moe_layer_forward_b200 import tp

    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    w, I = _tp_inputs()
    F = w.d_ff // world
    f = slice(rank * F, (rank + 1) * F)
    out = tp.tp_forward(I["x"], I["gamma"], I["W_r"], I["b"], I["W_gate"][:, f].contiguous(),
                        I["W_up"][:, f].contiguous(), I["W_down"][:, :, f].contiguous(), top_k=w.top_k, eps=w.eps,
                        ops=OracleOps())
    torch.save({"out": out}, os.path.join(outdir, f"r{rank}.pt"))
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_tensor_parallel_layer_equals_the_single_process_layer(world):
    sys.path.insert(0, ROOT)
    w, I = _tp_inputs()
    ops = OracleOps()
    v32 = ops.rmsnorm(I["x"], I["gamma"], w.eps, torch.float32)
    idx, wt = ops.router(v32, I["W_r"], I["b"], w.top_k)
    counts, offsets, token_slot, xp = ops.permute(v32, idx, w.E)
    y = ops.grouped_swiglu(xp, I["W_gate"], I["W_up"], I["W_down"], counts, offsets)
    ref = ops.combine(y, token_slot, wt, I["x"], torch.float64)
    with tempfile.TemporaryDirectory() as d:
        mp.start_processes(_tp_worker, args=(world, _free_port(), d), nprocs=world, join=True, start_method="spawn")
        r = [torch.load(os.path.join(d, f"r{k}.pt"))["out"] for k in range(world)]
    for k in range(world):  # every rank holds the whole result
        assert torch.equal(r[k], r[0])
    # the d_ff split only regroups the down projection's sum; fp32 partials add fp32 rounding
    assert torch.allclose(r[0].double(), ref, rtol=1e-5, atol=1e-5)


def _tp_scatter_worker(rank, world, port, outdir):
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import datetime

    import torch.distributed as dist

    from moe_layer_forward_b200 import tp

    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    w, I = _tp_inputs()
    F = w.d_ff // world
    f = slice(rank * F, (rank + 1) * F)
    out = tp.tp_forward(I["x"], I["gamma"], I["W_r"], I["b"], I["W_gate"][:, f].contiguous(),
                        I["W_up"][:, f].contiguous(), I["W_down"][:, :, f].contiguous(), top_k=w.top_k, eps=w.eps,
                        ops=OracleOps(), scatter=True)
    torch.save({"out": out}, os.path.join(outdir, f"r{rank}.pt"))
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_tensor_parallel_reduce_scatter_gives_each_rank_its_tokens(world):
    sys.path.insert(0, ROOT)
    w, I = _tp_inputs()
    ops = OracleOps()
    v32 = ops.rmsnorm(I["x"], I["gamma"], w.eps, torch.float32)
    idx, wt = ops.router(v32, I["W_r"], I["b"], w.top_k)
    counts, offsets, token_slot, xp = ops.permute(v32, idx, w.E)
    y = ops.grouped_swiglu(xp, I["W_gate"], I["W_up"], I["W_down"], counts, offsets)
    ref = ops.combine(y, token_slot, wt, I["x"], torch.float64)
    with tempfile.TemporaryDirectory() as d:
        mp.start_processes(_tp_scatter_worker, args=(world, _free_port(), d), nprocs=world, join=True,
                           start_method="spawn")
        r = [torch.load(os.path.join(d, f"r{k}.pt"))["out"] for k in range(world)]
    T_r = w.T // world
    for k in range(world):  # rank k holds tokens [k T/N, (k+1) T/N), the regrouped sum as in the all-reduce form
        assert r[k].shape[0] == T_r
        assert torch.allclose(r[k].double(), ref[k * T_r:(k + 1) * T_r], rtol=1e-5, atol=1e-5)


def _single_rank_group(port):
    import datetime

    import torch.distributed as dist

    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=30))
    return dist


def _check_arguments(port, outdir):
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    from moe_layer_forward_b200 import ep, tp

    dist = _single_rank_group(port)
    w, I = _inputs()
    msgs = []
    try:  # the rank holds fewer experts than E / N
        ep.ep_forward(I["x"], I["gamma"], I["W_r"], I["b"], I["W_gate"][:3], I["W_up"][:3], I["W_down"][:3], E=w.E,
                      ops=OracleOps())
    except ValueError as e:
        msgs.append(str(e))
    try:  # the down slice does not match the gate/up feature slice
        tp.tp_forward(I["x"], I["gamma"], I["W_r"], I["b"], I["W_gate"], I["W_up"], I["W_down"][:, :, :64],
                      ops=OracleOps())
    except ValueError as e:
        msgs.append(str(e))
    # one rank: both orchestrations reduce to the plain layer
    out, stats = ep.ep_forward(I["x"], I["gamma"], I["W_r"], I["b"], I["W_gate"], I["W_up"], I["W_down"], E=w.E,
                               top_k=w.top_k, eps=w.eps, ops=OracleOps())
    out_tp = tp.tp_forward(I["x"], I["gamma"], I["W_r"], I["b"], I["W_gate"], I["W_up"], I["W_down"], top_k=w.top_k,
                           eps=w.eps, ops=OracleOps())
    torch.save({"msgs": msgs, "out": out, "out_tp": out_tp, "rows": stats.rows_received},
               os.path.join(outdir, "r.pt"))
    dist.destroy_process_group()


def test_orchestration_argument_checks_and_single_rank():
    w, I = _inputs()
    with tempfile.TemporaryDirectory() as d:
        _spawn_one(_check_arguments, d)
        r = torch.load(os.path.join(d, "r.pt"))
    assert len(r["msgs"]) == 2 and "experts" in r["msgs"][0] and "slice" in r["msgs"][1]
    assert r["rows"] == w.T * w.top_k
    assert torch.allclose(r["out"].double(), r["out_tp"].double(), rtol=1e-6, atol=1e-6)


def _one(rank, fn, port, outdir):
    fn(port, outdir)


def _spawn_one(fn, outdir):
    mp.start_processes(_one, args=(fn, _free_port(), outdir), nprocs=1, join=True, start_method="spawn")
