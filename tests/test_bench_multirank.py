"""The N > 1 path of the benchmark, on CPU with two gloo ranks.

The layer shards by tokens: every rank runs an independent replica on its own
tokens, so the only cross-rank operations are a barrier and the max over ranks
of the timed duration.  These tests run that logic in two spawned processes.
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


def _worker(rank: int, world: int, port: int, outdir: str):
    sys.path.insert(0, ROOT)
    import datetime

    import torch.distributed as dist

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import bench
    import oracle
    import synth

    # timing: rank r took 10 * (r + 1) ms for 5 steps of 128 tokens; the job time is the slowest rank's
    value, ms_per_step = bench.aggregate(10.0 * (rank + 1), 128, 5, world, bench.reduce_max_fn(dist, "cpu"))
    dist.barrier()
    # replicas: each rank computes the layer on its own shard of the tokens
    w = synth.Workload("shard", 12, 64, 16, 32, x_dtype=torch.float32, w_dtype=torch.float32,
                       out_dtype=torch.float32, seed=31)
    I = synth.make_layer_inputs(w)
    shard = I["x"][rank::world]
    out = oracle.moe_layer(shard, I["gamma"], I["W_r"], I["b"], I["W_gate"], I["W_up"], I["W_down"])["out"]
    torch.save({"value": value, "ms_per_step": ms_per_step, "out": out}, os.path.join(outdir, f"r{rank}.pt"))
    dist.barrier()
    dist.destroy_process_group()


def test_two_gloo_ranks_aggregate_with_the_slowest_rank_and_shard_tokens():
    world = 2
    with tempfile.TemporaryDirectory() as d:
        mp.start_processes(_worker, args=(world, _free_port(), d), nprocs=world, join=True, start_method="spawn")
        r = [torch.load(os.path.join(d, f"r{k}.pt")) for k in range(world)]
    for k in range(world):
        assert r[k]["value"] == pytest.approx(world * 128 * 5 / 0.020)  # slowest rank: 20 ms
        assert r[k]["ms_per_step"] == pytest.approx(4.0)
    # concatenating the ranks' shards reproduces the single-process layer (no data-path collective needed)
    sys.path.insert(0, ROOT)
    import oracle
    import synth

    w = synth.Workload("shard", 12, 64, 16, 32, x_dtype=torch.float32, w_dtype=torch.float32,
                       out_dtype=torch.float32, seed=31)
    I = synth.make_layer_inputs(w)
    full = oracle.moe_layer(I["x"], I["gamma"], I["W_r"], I["b"], I["W_gate"], I["W_up"], I["W_down"])["out"]
    merged = torch.empty_like(full)
    for k in range(world):
        merged[k::world] = r[k]["out"]
    assert torch.equal(merged, full)


def test_single_rank_aggregate_is_local():
    sys.path.insert(0, ROOT)
    import bench

    value, ms = bench.aggregate(8.0, 100, 4, 1, lambda v: v)
    assert value == pytest.approx(100 * 4 / 0.008) and ms == pytest.approx(2.0)


def test_reference_arm_runs_only_on_rank_zero(monkeypatch):
    sys.path.insert(0, ROOT)
    import argparse

    import bench
    import synth

    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    a = argparse.Namespace(steps=2, warmup=3, gpus=2)
    assert bench.run_reference(a, synth.WORKLOADS["decode"]) == 0  # returns at once, no inputs generated


def test_clock_summary_decodes_throttle_reasons():
    # the bench's clock record from NVML samples (SM MHz, clocks-event reason bits, W): the median clock, the
    # union of the reasons that reject or annotate a run, and how many samples it rests on
    sys.path.insert(0, ROOT)
    import bench

    c = bench.Clocks(0)
    c.thread = object()  # as if the NVML sampler had run
    c.max_mhz = 1965.0
    c.samples = [(1965, 0x0, 700.0), (1500, 0x4, 990.0), (1400, 0x4 | 0x1, 1000.0), (1800, 0x40, 950.0)]
    s = c.summary()
    assert s["sm_mhz"] == 1650.0 and s["sm_min_mhz"] == 1400 and s["sm_max_mhz"] == 1965.0
    assert s["reasons"] == ["hw_thermal_slowdown", "sw_power_cap"]
    assert s["samples"] == 4 and s["power_w"] == 970.0


def test_layer_roofline_binds_decode_to_hbm_and_prefill_to_the_tensor_peak():
    # the bench's layer fractions from the workloads' own sizes: decode streams the active experts' weights
    # (HBM-bound), prefill runs 6 S d d_ff flops (tensor-bound); recomputed here from the shapes by hand
    sys.path.insert(0, ROOT)
    import bench
    import synth

    pk = {"hbm_gbs": 6550.1, "bf16_tflops": 1640.7, "bf16_tflops_sustained": 1365.9, "source": "measured"}
    dec = synth.WORKLOADS["decode"]
    r = bench.layer_roofline(dec, 128, 0.7867, pk)
    weights = 128 * 3 * 4096 * 1536 * 2
    io = 128 * 4096 * (2 + 2) + 128 * 4096 * 4 + 4096 * 4 + 128 * 4
    assert r["algorithmic_bytes"] == weights + io == 4836049408
    assert r["bound"] == "hbm" and abs(r["frac"] - 4836049408 / 0.7867e-3 / 6550.1e9) < 1e-12
    pre = synth.WORKLOADS["prefill"]
    r = bench.layer_roofline(pre, 128, 2.5959, pk)
    assert r["expert_flops"] == 6.0 * 8192 * 8 * 4096 * 1536
    assert r["bound"] == "tensor" and abs(r["frac"] - 2.473901162496e12 / 2.5959e-3 / 1640.7e12) < 1e-12
    assert abs(r["frac_sustained"] - 2.473901162496e12 / 2.5959e-3 / 1365.9e12) < 1e-12
    assert abs(r["t_roof_ms"] - 2.473901162496e12 / 1640.7e12 * 1e3) < 1e-9


def test_dominant_kernel_label_follows_the_tile_form_selection():
    # the bench names the gate/up kernel the library selects by average rows per expert
    sys.path.insert(0, ROOT)
    import bench
    import synth

    want = {"decode": "weights-as-M", "block": "rows-as-M", "prefill": "two 128-row blocks", "skewed": "CTA pairs"}
    for name, form in want.items():
        w = synth.WORKLOADS[name]
        assert form in bench.gate_up_kernel_name(w.T * w.top_k, w.E), name
