"""Expert- and tensor-parallel forwards on the GPU with the library's kernels
and NCCL, one rank (the only GPU a test here has): with every expert and
feature local the exchange and the reduction are identities, and the result
must equal moe_forward bit for bit (same router arithmetic, same GEMM tiles,
same combine).  Runs in a spawned process so the NCCL group does not outlive
the test."""
import os
import socket
import sys
import tempfile

import pytest
import torch
import torch.multiprocessing as mp

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, port, outdir, shape):
    sys.path.insert(0, ROOT)
    import datetime

    import torch.distributed as dist

    import moe_layer_forward_b200 as moe
    import synth
    from moe_layer_forward_b200 import ep

    torch.cuda.set_device(0)
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60), device_id=torch.device("cuda", 0))
    T, d, E, d_ff = shape
    w = synth.Workload("ep1", T, d, E, d_ff, seed=950)
    D = {n: t.cuda() for n, t in synth.make_layer_inputs(w).items()}
    out_ep, stats = ep.ep_forward(D["x"], D["gamma"], D["W_r"], D["b"], D["W_gate"], D["W_up"], D["W_down"], E=E,
                                  top_k=w.top_k, eps=w.eps)
    out = torch.empty_like(out_ep)
    moe.moe_forward(D["x"], D["gamma"], D["W_r"], D["b"], D["W_gate"], D["W_up"], D["W_down"], out, top_k=w.top_k,
                    eps=w.eps)
    from moe_layer_forward_b200 import tp

    out_tp = tp.tp_forward(D["x"], D["gamma"], D["W_r"], D["b"], D["W_gate"], D["W_up"], D["W_down"], top_k=w.top_k,
                           eps=w.eps)
    out_tps = tp.tp_forward(D["x"], D["gamma"], D["W_r"], D["b"], D["W_gate"], D["W_up"], D["W_down"],
                            top_k=w.top_k, eps=w.eps, scatter=True)
    torch.cuda.synchronize()
    torch.save({"equal": torch.equal(out_ep, out), "tp_equal": torch.equal(out_tp, out) and torch.equal(out_tps, out),
                "rows": stats.rows_received}, os.path.join(outdir, "r.pt"))
    dist.destroy_process_group()


@pytest.mark.parametrize("shape", [(96, 512, 64, 256), (1200, 256, 8, 256)])  # weights-as-M; CTA pairs
def test_single_rank_expert_and_tensor_parallel_equal_moe_forward(shape):
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    with tempfile.TemporaryDirectory() as d:
        mp.start_processes(_worker, args=(_free_port(), d, shape), nprocs=1, join=True, start_method="spawn")
        r = torch.load(os.path.join(d, "r.pt"))
    assert r["equal"] and r["tp_equal"]
    assert r["rows"] == shape[0] * 8
