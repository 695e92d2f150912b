#!/usr/bin/env python
"""MoE layer forward throughput on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload decode] [--impl ours|reference]

One step = one whole layer forward R = X + MoE(RMSNorm(X)) (RMSNorm, router,
permutation, grouped SwiGLU expert MLP, combine) over one batch of seeded
synthetic tokens, inputs resident in HBM.  Prints one JSON line (rank 0).

With N > 1 (torchrun) every rank runs an independent replica on its own GPU
(tokens are independent; there is no data-path collective) and the time is
the max over ranks.  ``--impl reference`` times the CPU oracle (the only
reference this layer has) on a bounded token sample per step.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MoE-layer tokens/s at 1 B200; % of HBM (decode) / BF16 tensor (prefill) roofline"
L2_BYTES = 126 * 1024 * 1024
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "roofline_traffic.json")
GEMM_SRC = [os.path.join(ROOT, "moe_layer_forward_b200", "csrc", f) for f in ("expert_tc.cu", "tc_ptx.cuh")]


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="decode", help="tiny | decode | prefill | skewed | block")
    ap.add_argument("--shrink", type=int, default=1,
                    help="divide T and E by this factor (same rows per expert, smaller device footprint); "
                         "for ncu captures of the same kernels, never for reported numbers")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-ep", action="store_true", help="skip the one-rank expert-parallel (peer memory) timing")
    ap.add_argument("--no-fp8", action="store_true",
                    help="skip the block-FP8 layer timing (run for bf16 workloads of <= 32 rows per expert)")
    ap.add_argument("--no-masked", action="store_true",
                    help="skip the masked-layout expert MLP timing (run for workloads of <= 32 rows per expert)")
    a = ap.parse_args()
    a.warmup = max(a.warmup, 3)
    return a


def dist_env():
    return int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")), int(
        os.environ.get("LOCAL_RANK", "0"))


def reduce_max_fn(dist, device):
    """max over ranks of a float (identity on one rank); the only cross-rank operation of a replica run"""
    import torch

    def reduce_max(v: float) -> float:
        if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
            return v
        t = torch.tensor([v], dtype=torch.float64, device=device)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return float(t.item())

    return reduce_max


def aggregate(local_ms: float, units_per_rank: int, steps: int, world: int, reduce_max):
    """(whole-job units/s, ms per step): every rank processed units_per_rank per step; time = slowest rank"""
    ms = reduce_max(local_ms)
    return world * units_per_rank * steps / (ms / 1000.0), ms / steps


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        j = json.load(open(p))
        return {"hbm_gbs": j["hbm_gbs"], "bf16_tflops": j["bf16_tflops"], "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "source": "fallback"}


class Clocks:
    """nvidia-smi samples of SM clock and throttle reasons while the timed region runs."""

    Q = ("index,clocks.sm,clocks.max.sm,clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                                          "-lms", "200", "-i", str(self.gpu)], stdout=subprocess.PIPE,
                                         stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            out, _ = self.proc.communicate(timeout=10)
            self.lines = [l for l in out.splitlines() if l.strip()]

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for l in self.lines:
            f = [x.strip() for x in l.split(",")]
            if len(f) < 7:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[3:7]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


def kernel_code_sha() -> str:
    """Hash of the dominant kernel's source code with comments and whitespace removed."""
    text = "".join(open(f, encoding="utf-8").read() for f in GEMM_SRC)
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    return hashlib.sha256(" ".join(text.split()).encode()).hexdigest()[:16]


def traffic_for(workload: str):
    """DRAM bytes per launch of the dominant kernel from the committed ncu summary, if its code is unchanged."""
    if not os.path.exists(TRAFFIC_FILE):
        return None
    j = json.load(open(TRAFFIC_FILE))
    sha = kernel_code_sha()
    e = j.get(workload)
    if not e or e.get("source_sha") != sha:
        return None
    return e.get("dram_bytes_per_launch")


# --------------------------------------------------------------------------- CPU oracle legs
def oracle_tokens_per_s(I, w, n_tokens: int, start: int = 0):
    import oracle

    sel = [(start + i * 7919) % w.T for i in range(n_tokens)]
    x = I["x"][sel].contiguous()
    t0 = time.perf_counter()
    oracle.moe_layer(x, I["gamma"], I["W_r"], I["b"], I["W_gate"], I["W_up"], I["W_down"], k=w.top_k, eps=w.eps)
    dt = time.perf_counter() - t0
    return n_tokens / dt, dt


def cpu_baseline(I, w):
    # one token first to size a sample of about 15 s of single-core work
    _, t1 = oracle_tokens_per_s(I, w, 1)
    n = int(max(1, min(256, 15.0 / max(t1, 1e-3))))
    v, dt = oracle_tokens_per_s(I, w, n, start=1)
    return {"value": v, "unit": "tokens/s", "cores": 1, "kind": "oracle",
            "sample": f"{n} token rows cycling through the {w.T} of the {w.name} workload, whole layer per "
                      f"token in fp64 (single-threaded C, {dt:.1f} s)"}


def run_reference(a, w):
    import synth

    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    I = synth.make_layer_inputs(w)
    _, t1 = oracle_tokens_per_s(I, w, 1)
    per_step = int(max(1, min(64, 2.0 / max(t1, 1e-3))))  # about 2 s of CPU work per step
    for i in range(a.warmup):
        oracle_tokens_per_s(I, w, 1, start=i)
    t0 = time.perf_counter()
    for i in range(a.steps):
        oracle_tokens_per_s(I, w, per_step, start=100 + i * per_step)
    dt = time.perf_counter() - t0
    value = a.steps * per_step / dt
    sample = f"{per_step} of {w.T} tokens per step, whole layer per token in fp64 (single-threaded C oracle)"
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": a.gpus,
            "steps": a.steps, "warmup": a.warmup, "ms_per_step": 1000.0 * dt / a.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_of(w, a.gpus),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": 1, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def config_of(w, n):
    return {"workload": w.name, "T": w.T, "d": w.d, "E": w.E, "top_k": w.top_k, "d_ff": w.d_ff,
            "x_dtype": str(w.x_dtype).replace("torch.", ""), "expert_dtype": str(w.w_dtype).replace("torch.", ""),
            "out_dtype": str(w.out_dtype).replace("torch.", ""), "global_batch_tokens": w.T * n,
            "parallelism": "replicas" if n > 1 else "single",
            "l2": "not flushed: every step streams the active experts' weights, many times the 126 MB L2"}


# --------------------------------------------------------------------------- GPU arm
def run_ours(a, w):
    import torch
    import torch.distributed as dist

    import moe_layer_forward_b200 as moe
    import synth

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=180), device_id=dev)

    I = synth.make_layer_inputs(w)
    D = {n: t.to(dev) for n, t in I.items()}
    T, k, E = w.T, w.top_k, w.E
    out = torch.empty((T, w.d), dtype=w.out_dtype, device=dev)
    idx = torch.empty((T, k), dtype=torch.int32, device=dev)
    wt = torch.empty((T, k), dtype=torch.float32, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    ws = torch.empty(moe.forward_workspace_bytes(D["x"], D["W_r"], D["W_gate"], out, k, w.eps), dtype=torch.uint8,
                     device=dev)

    def step(x=None, o=None):
        moe.moe_forward(D["x"] if x is None else x, D["gamma"], D["W_r"], D["b"], D["W_gate"], D["W_up"],
                        D["W_down"], out if o is None else o, top_k=k, eps=w.eps, topk_idx=idx, topk_w=wt, ws=ws,
                        dev_status=status)

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    max_over_ranks = reduce_max_fn(dist, dev)

    for _ in range(a.warmup):
        step()
    torch.cuda.synchronize()
    if status.item() != 0:
        raise RuntimeError(f"device status {status.item()} after warm-up")

    # ---- timed region: exactly K steps, device-resident inputs
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    with Clocks(local) as clk:
        n0 = moe.kernel_launches()
        e0.record()
        for _ in range(a.steps):
            step()
        e1.record()
        launches = moe.kernel_launches() - n0  # counted by the library itself
        barrier()
    value, ms_per_step = aggregate(e0.elapsed_time(e1), T, a.steps, world, max_over_ranks)
    if status.item() != 0:
        raise RuntimeError(f"device status {status.item()} in the timed region")

    # ---- dominant kernel (expert gate/up GEMM) timed per launch through the step-level entry points
    counts = torch.empty(E, dtype=torch.int32, device=dev)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
    slot_token = torch.empty(T * k, dtype=torch.int32, device=dev)
    token_slot = torch.empty((T, k), dtype=torch.int32, device=dev)
    v = torch.empty((T, w.d), dtype=w.w_dtype, device=dev)
    xp = torch.empty((T * k, w.d), dtype=w.w_dtype, device=dev)
    h = torch.empty((T * k, w.d_ff), dtype=w.w_dtype, device=dev)
    y = torch.empty((T * k, w.d), dtype=w.w_dtype, device=dev)
    names = ["rmsnorm", "router", "permute", "gate_up", "down", "combine"]
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(len(names) + 1)] for _ in range(a.steps)]

    def staged(ev=None):
        rec = (lambda i: ev[i].record()) if ev else (lambda i: None)
        rec(0)
        moe.moe_rmsnorm(D["x"], D["gamma"], w.eps, v)
        rec(1)
        moe.moe_router_topk(v, D["W_r"], D["b"], idx, wt)
        rec(2)
        moe.moe_permute(v, idx, E, counts, offsets, slot_token, token_slot, xp)
        rec(3)
        moe.moe_expert_gate_up(xp, D["W_gate"], D["W_up"], counts, offsets, h)
        rec(4)
        moe.moe_expert_down(h, D["W_down"], counts, offsets, y)
        rec(5)
        moe.moe_unpermute_combine(y, token_slot, wt, D["x"], out)
        rec(6)

    for _ in range(a.warmup):
        staged()
    barrier()
    for i in range(a.steps):
        staged(evs[i])
    torch.cuda.synchronize()
    stage_ms = {n: statistics.mean(evs[i][j].elapsed_time(evs[i][j + 1]) for i in range(a.steps))
                for j, n in enumerate(names)}
    active = int((counts > 0).sum().item())
    S = T * k
    esz = 2 if w.w_dtype == torch.bfloat16 else 4
    gate_up_bytes = active * 2 * w.d_ff * w.d * esz + S * w.d * esz + S * w.d_ff * esz
    gate_up_flops = 2.0 * S * w.d * 2 * w.d_ff
    pk = peaks()
    t_s = stage_ms["gate_up"] / 1000.0
    hbm_bound = gate_up_bytes / (pk["hbm_gbs"] * 1e9) >= gate_up_flops / (pk["bf16_tflops"] * 1e12)
    if hbm_bound:
        roof = {"bound": "hbm", "achieved": gate_up_bytes / t_s / 1e9, "peak": pk["hbm_gbs"], "unit": "GB/s"}
    else:
        roof = {"bound": "tensor", "achieved": gate_up_flops / t_s / 1e12, "peak": pk["bf16_tflops"],
                "unit": "TFLOP/s"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["traffic"] = traffic_for(w.name)
    roof["kernel"] = "grouped_gemm_kernel (expert gate/up + SwiGLU)"
    roof["algorithmic_bytes_per_launch"] = gate_up_bytes
    roof["algorithmic_flops_per_launch"] = gate_up_flops
    roof["launch_ms"] = stage_ms["gate_up"]
    roof["peak_source"] = f"{pk['source']} (burst, kernel timed alone)"

    # ---- the expert MLP on the masked layout ([E][cap][d] buffers + counts), same routing
    masked = None
    if not a.no_masked and w.w_dtype == torch.bfloat16 and S // E <= 32:
        cn, of = counts.cpu(), offsets.cpu()
        cap = int((int(cn.max()) + 15) // 16 * 16)
        xm = torch.zeros((E, cap, w.d), dtype=w.w_dtype, device=dev)
        for e in range(E):  # input preparation, outside the timed region
            xm[e, :int(cn[e])] = xp[int(of[e]):int(of[e]) + int(cn[e])]
        hm = torch.empty((E, cap, w.d_ff), dtype=w.w_dtype, device=dev)
        ym = torch.empty((E, cap, w.d), dtype=w.w_dtype, device=dev)

        def mstep():
            moe.moe_grouped_swiglu_masked(xm, D["W_gate"], D["W_up"], D["W_down"], counts, hm, ym, dev_status=status)

        for _ in range(a.warmup):
            mstep()
        barrier()
        m0, m1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        m0.record()
        for _ in range(a.steps):
            mstep()
        m1.record()
        torch.cuda.synchronize()
        if status.item() != 0:
            raise RuntimeError(f"device status {status.item()} in the masked-layout timing")
        mms = m0.elapsed_time(m1) / a.steps
        mbytes = active * 3 * w.d_ff * w.d * esz + S * (2 * w.d + 2 * w.d_ff) * esz
        masked = {"expert_mlp_ms": mms, "tokens_per_s": T / (mms / 1000.0), "cap": cap,
                  "hbm_achieved_gbs": mbytes / (mms / 1000.0) / 1e9,
                  "hbm_frac": mbytes / (mms / 1000.0) / 1e9 / pk["hbm_gbs"], "algorithmic_bytes": mbytes,
                  "contiguous_expert_mlp_ms": stage_ms["gate_up"] + stage_ms["down"]}

    # ---- the layer with block-FP8 experts (weights quantised on the device beforehand)
    fp8 = None
    if not a.no_fp8 and w.w_dtype == torch.bfloat16 and S // E <= 32:
        Wq = [moe.quantize_fp8_weights(D[n]) for n in ("W_gate", "W_up", "W_down")]
        out8 = torch.empty_like(out)
        ws8 = torch.empty(moe.forward_fp8_workspace_bytes(D["x"], D["W_r"], Wq[0][0], out8, k, w.eps),
                          dtype=torch.uint8, device=dev)

        def fstep():
            moe.moe_forward_fp8(D["x"], D["gamma"], D["W_r"], D["b"], *Wq, out8, top_k=k, eps=w.eps, ws=ws8,
                                dev_status=status)

        for _ in range(a.warmup):
            fstep()
        barrier()
        g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        g0.record()
        for _ in range(a.steps):
            fstep()
        g1.record()
        torch.cuda.synchronize()
        if status.item() != 0:
            raise RuntimeError(f"device status {status.item()} in the FP8 timing")
        fms = g0.elapsed_time(g1) / a.steps
        # algorithmic bytes: active experts' codes and scales, the input, the output and the router weights
        fbytes = active * 3 * w.d_ff * w.d * (1 + 4 / (128 * 128)) + T * w.d * (D["x"].element_size() +
                                                                                 out.element_size()) + E * w.d * 4
        fp8 = {"ms_per_step": fms, "tokens_per_s": T / (fms / 1000.0), "dtype": "e4m3 experts, fp32 router",
               "algorithmic_bytes": fbytes, "hbm_achieved_gbs": fbytes / (fms / 1000.0) / 1e9,
               "hbm_frac": fbytes / (fms / 1000.0) / 1e9 / pk["hbm_gbs"],
               "vs_bf16_layer": ms_per_step / fms}
        del Wq

    # ---- expert parallelism with the exchange fused into the dispatch and combine kernels: one rank's step
    epp = None
    if not a.no_ep and world == 1 and w.w_dtype == torch.bfloat16:
        from moe_layer_forward_b200 import ep_p2p

        peers = ep_p2p.local_peers(1, ep_p2p.capacity_rows(T, 1, k, E), w.d, w.w_dtype, dev)

        def estep():
            return ep_p2p.ep_p2p_forward_emulated([D["x"]], D["gamma"], D["W_r"], D["b"], D["W_gate"], D["W_up"],
                                                  D["W_down"], top_k=k, eps=w.eps, peers=peers)

        for _ in range(a.warmup):
            estep()
        barrier()
        p0, p1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        p0.record()
        for _ in range(a.steps):
            estep()
        p1.record()
        torch.cuda.synchronize()
        ems = p0.elapsed_time(p1) / a.steps
        epp = {"ranks": 1, "ms_per_step": ems, "tokens_per_s": T / (ems / 1000.0), "vs_moe_forward": ms_per_step / ems,
               "steps": "routing, permutation maps, dispatch into the receive buffer, layout, grouped MLP over "
                        "the whole buffer, pull combine; no host synchronisation",
               "multi_gpu": "not measured (one GPU per call here)"}
        del peers

    # ---- end to end through the public API with host buffers
    e2e = None
    if not a.no_e2e:
        x_host = I["x"].pin_memory()
        out_host = torch.empty(out.shape, dtype=out.dtype).pin_memory()
        x_dev = torch.empty_like(D["x"])
        for _ in range(a.warmup):
            x_dev.copy_(x_host, non_blocking=True)
            step(x_dev)
            out_host.copy_(out, non_blocking=True)
            torch.cuda.current_stream().synchronize()
        barrier()
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        f0.record()
        for _ in range(a.steps):
            x_dev.copy_(x_host, non_blocking=True)
            step(x_dev)
            out_host.copy_(out, non_blocking=True)
            torch.cuda.current_stream().synchronize()  # the host reads this step's result
        f1.record()
        barrier()
        e2e_value, _ = aggregate(f0.elapsed_time(f1), T, a.steps, world, max_over_ranks)
        e2e = {"value": e2e_value, "unit": "tokens/s",
               "h2d_bytes_per_step": x_host.numel() * x_host.element_size(),
               "d2h_bytes_per_step": out_host.numel() * out_host.element_size()}

    cpu = None
    if rank == 0 and world == 1 and not a.no_cpu_baseline:
        cpu = cpu_baseline(I, w)

    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": a.steps,
                "warmup": a.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "bf16" if w.w_dtype == torch.bfloat16 else "f32",
                "data": "synthetic", "config": config_of(w, world), "roofline": roof, "cpu_baseline": cpu,
                "e2e": e2e, "gpu_launches": launches, "clocks": clk.summary(),
                "stages_ms": stage_ms, "active_experts": active, "masked_layout": masked, "fp8_layer": fp8,
                "ep_p2p": epp}
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main():
    a = parse()
    import synth

    w = synth.WORKLOADS[a.workload]
    if a.shrink > 1:
        w = w.scaled(name=f"{w.name}/shrink{a.shrink}", T=max(1, w.T // a.shrink), E=max(w.top_k, w.E // a.shrink))
    if a.impl == "reference":
        return run_reference(a, w)
    return run_ours(a, w)


if __name__ == "__main__":
    sys.exit(main())
