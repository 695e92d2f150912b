#!/usr/bin/env python
"""MoE layer forward throughput on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload decode] [--impl ours|reference]

One step = one whole layer forward R = X + MoE(RMSNorm(X)) (RMSNorm, router,
permutation, grouped SwiGLU expert MLP, combine) over one batch of seeded
synthetic tokens, inputs resident in HBM.  Prints one JSON line (rank 0): the
headline workload (decode by default) at the top level and, at one GPU, all
five workloads (tiny, decode, prefill, skewed, block) under "workloads", each
with tokens/s, the layer's fraction of its roofline, the dominant kernel's
fraction, the near-tie token count, end-to-end throughput and a CPU oracle
sample.

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
    ap.add_argument("--workload", default="decode", help="headline workload: tiny | decode | prefill | skewed | block")
    ap.add_argument("--workloads", choices=["all", "one"], default="all",
                    help="all: at one GPU, also measure the other four workloads (reported under 'workloads'); "
                         "one: the headline workload only")
    ap.add_argument("--shrink", type=int, default=1,
                    help="divide T and E by this factor (same rows per expert, smaller device footprint); "
                         "for ncu captures of the same kernels, never for reported numbers")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-anchor", action="store_true",
                    help="skip the comparison of the expert GEMMs with a vendor grouped GEMM (bf16 workloads)")
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
        return {"hbm_gbs": j["hbm_gbs"], "bf16_tflops": j["bf16_tflops"],
                "bf16_tflops_sustained": j.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


class Clocks:
    """SM clock and throttle reasons while the timed region runs: NVML every 5 ms from a thread (the device
    found by its PCI bus id), else nvidia-smi every 200 ms."""

    Q = ("index,clocks.sm,clocks.max.sm,clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    # NVML clocks-event reason bits
    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown"}

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.thread = None
        self.samples = []  # (sm MHz, reason bits, power W)
        self.max_mhz = None
        self.lines = []

    def _nvml_handle(self):
        import pynvml
        import torch

        pynvml.nvmlInit()
        props = torch.cuda.get_device_properties(self.gpu)
        bus = getattr(props, "pci_bus_id", None)
        if bus is not None:
            pci = f"{getattr(props, 'pci_domain_id', 0):08x}:{bus:02x}:{getattr(props, 'pci_device_id', 0):02x}.0"
            try:
                return pynvml, pynvml.nvmlDeviceGetHandleByPciBusId(pci.encode())
            except pynvml.NVMLError:
                pass
        return pynvml, pynvml.nvmlDeviceGetHandleByIndex(self.gpu)

    def __enter__(self):
        import threading

        try:
            nv, h = self._nvml_handle()
            self.max_mhz = float(nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM))
            self.stop = threading.Event()

            def run():
                while not self.stop.is_set():
                    try:
                        self.samples.append((nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM),
                                             nv.nvmlDeviceGetCurrentClocksEventReasons(h),
                                             nv.nvmlDeviceGetPowerUsage(h) / 1000.0))
                    except nv.NVMLError:
                        pass
                    self.stop.wait(0.005)

            self.thread = threading.Thread(target=run, daemon=True)
            self.thread.start()
            return self
        except Exception:
            self.thread = None
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                                          "-lms", "200", "-i", str(self.gpu)], stdout=subprocess.PIPE,
                                         stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.thread is not None:
            self.stop.set()
            self.thread.join(timeout=5)
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            out, _ = self.proc.communicate(timeout=10)
            self.lines = [l for l in out.splitlines() if l.strip()]

    def summary(self):
        if self.thread is not None:
            if not self.samples:
                return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0, "source": "nvml"}
            reasons = sorted({n for _, bits, _ in self.samples for b, n in self.REASONS.items() if bits & b})
            sm = [c for c, _, _ in self.samples]
            return {"sm_mhz": statistics.median(sm), "sm_min_mhz": min(sm), "sm_max_mhz": self.max_mhz,
                    "power_w": round(statistics.median(p for _, _, p in self.samples), 1), "reasons": reasons,
                    "samples": len(sm), "source": "nvml, 5 ms"}
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
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": [], "samples": 0, "source": "nvidia-smi, 200 ms"}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm),
                "source": "nvidia-smi, 200 ms"}


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


def cpu_baseline(I, w, seconds: float = 15.0):
    # one token first to size a sample of about `seconds` of single-core work
    _, t1 = oracle_tokens_per_s(I, w, 1)
    n = int(max(1, min(256, seconds / max(t1, 1e-3))))
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


def active_weight_bytes(w) -> int:
    esz = 2 if str(w.w_dtype).endswith("bfloat16") else 4
    return w.E * 3 * w.d * w.d_ff * esz


def config_of(w, n):
    return {"workload": w.name, "T": w.T, "d": w.d, "E": w.E, "top_k": w.top_k, "d_ff": w.d_ff,
            "x_dtype": str(w.x_dtype).replace("torch.", ""), "expert_dtype": str(w.w_dtype).replace("torch.", ""),
            "out_dtype": str(w.out_dtype).replace("torch.", ""), "global_batch_tokens": w.T * n,
            "parallelism": "replicas" if n > 1 else "single",
            "l2": "not flushed: inputs larger than L2 (every step streams the active experts' weights, "
                  f"{active_weight_bytes(w) / 1e9:.1f} GB at most, against the 126 MB L2)"}


# --------------------------------------------------------------------------- GPU arm
def _timed(fn, steps: int, warmup: int, barrier, clocks_gpu=None):
    """(device ms over exactly `steps` calls of fn, clock summary or None, launches): CUDA events on the
    current stream, a barrier and a device synchronisation on both sides, after `warmup` untimed calls."""
    import torch

    import moe_layer_forward_b200 as moe

    for _ in range(warmup):
        fn()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clk = Clocks(clocks_gpu) if clocks_gpu is not None else None
    if clk:
        clk.__enter__()
    n0 = moe.kernel_launches()
    e0.record()
    for _ in range(steps):
        fn()
    e1.record()
    launches = moe.kernel_launches() - n0
    barrier()
    if clk:
        clk.__exit__(None, None, None)
    return e0.elapsed_time(e1), (clk.summary() if clk else None), launches


def gate_up_kernel_name(S: int, E: int) -> str:
    """The gate/up GEMM form the library picks for S routed rows over E experts (the host's selection by
    average rows per expert: weights-as-M up to 32, rows-as-M up to 255, two-row-block tiles up to 767, CTA
    pairs above)."""
    avg = S // E if E > 0 else 0
    if avg >= 768:
        return "grouped_gemm_2sm_kernel (expert gate/up + SwiGLU, CTA pairs)"
    if avg >= 256:
        return "grouped_gemm_dual_kernel (expert gate/up + SwiGLU, two 128-row blocks per tile)"
    if avg > 32:
        return "grouped_gemm_kernel (expert gate/up + SwiGLU, rows-as-M)"
    return "grouped_gemm_kernel (expert gate/up + SwiGLU, weights-as-M)"


def layer_roofline(w, active: int, ms: float, pk: dict) -> dict:
    """The whole layer against its binding roofline: algorithmic bytes (active experts' weights, X, R, W_r,
    gamma, b) over the measured copy peak, or expert-GEMM flops (6 S d d_ff) over the measured bf16 peak."""
    esz = 2 if str(w.w_dtype).endswith("bfloat16") else 4
    xsz = 2 if str(w.x_dtype).endswith("bfloat16") else 4
    osz = 2 if str(w.out_dtype).endswith("bfloat16") else 4
    nbytes = active * 3 * w.d * w.d_ff * esz + w.T * w.d * (xsz + osz) + w.E * w.d * 4 + w.d * 4 + w.E * 4
    flops = 6.0 * w.T * w.top_k * w.d * w.d_ff
    t = ms / 1000.0
    t_hbm = nbytes / (pk["hbm_gbs"] * 1e9)
    t_tc = flops / (pk["bf16_tflops"] * 1e12)
    r = {"algorithmic_bytes": nbytes, "expert_flops": flops,
         "hbm_gbs": nbytes / t / 1e9, "hbm_frac": nbytes / t / 1e9 / pk["hbm_gbs"],
         "tensor_tflops": flops / t / 1e12, "tensor_frac": flops / t / 1e12 / pk["bf16_tflops"],
         "t_roof_ms": 1000.0 * max(t_hbm, t_tc)}
    if t_hbm >= t_tc:
        r.update(bound="hbm", frac=r["hbm_frac"], peak=pk["hbm_gbs"], unit="GB/s", achieved=r["hbm_gbs"])
    else:
        r.update(bound="tensor", frac=r["tensor_frac"], peak=pk["bf16_tflops"], unit="TFLOP/s",
                 achieved=r["tensor_tflops"])
        if pk.get("bf16_tflops_sustained"):
            r["frac_sustained"] = r["tensor_tflops"] / pk["bf16_tflops_sustained"]
    r["peak_source"] = pk["source"]
    return r


class Layer:
    """One workload's inputs, outputs and workspace on the device, and its step through moe_forward."""

    def __init__(self, w, dev):
        import torch

        import moe_layer_forward_b200 as moe
        import synth

        self.w, self.dev = w, dev
        self.I = synth.make_layer_inputs(w)
        self.D = {n: t.to(dev) for n, t in self.I.items()}
        T, k, E = w.T, w.top_k, w.E
        self.out = torch.empty((T, w.d), dtype=w.out_dtype, device=dev)
        self.idx = torch.empty((T, k), dtype=torch.int32, device=dev)
        self.wt = torch.empty((T, k), dtype=torch.float32, device=dev)
        self.status = torch.zeros(1, dtype=torch.int32, device=dev)
        self.ws = torch.empty(moe.forward_workspace_bytes(self.D["x"], self.D["W_r"], self.D["W_gate"], self.out, k,
                                                          w.eps), dtype=torch.uint8, device=dev)

    def step(self, x=None, out=None):
        import moe_layer_forward_b200 as moe

        D, w = self.D, self.w
        moe.moe_forward(D["x"] if x is None else x, D["gamma"], D["W_r"], D["b"], D["W_gate"], D["W_up"],
                        D["W_down"], self.out if out is None else out, top_k=w.top_k, eps=w.eps, topk_idx=self.idx,
                        topk_w=self.wt, ws=self.ws, dev_status=self.status)

    def check_status(self, where: str):
        if self.status.item() != 0:
            raise RuntimeError(f"{self.w.name}: device status {self.status.item()} {where}")


def near_ties(L) -> dict:
    """Tokens whose 8th-to-9th selection-score margin is below 1e-5, from the library's routing of the layer
    (moe_route: the forward's own router, bit for bit); a diagnostic, outside every timed region."""
    import torch

    import moe_layer_forward_b200 as moe

    w, D, dev = L.w, L.D, L.dev
    if w.E <= w.top_k:
        return {"count": 0, "threshold": 1e-5, "tokens": w.T}
    idx = torch.empty((w.T, w.top_k), dtype=torch.int32, device=dev)
    wt = torch.empty((w.T, w.top_k), dtype=torch.float32, device=dev)
    margin = torch.empty(w.T, dtype=torch.float32, device=dev)
    moe.moe_route(D["x"], D["gamma"], D["W_r"], D["b"], idx, wt, w.eps, margin=margin)
    n = int((margin < 1e-5).sum().item())
    return {"count": n, "threshold": 1e-5, "tokens": w.T, "routing_equals_forward": bool(torch.equal(idx, L.idx))}


def staged(L, a, barrier, pk) -> tuple:
    """Per-step CUDA-event times of the six step-level entry points (a permuted copy feeds the GEMMs), and the
    dominant kernel's (the gate/up GEMM's) roofline object."""
    import torch

    import moe_layer_forward_b200 as moe

    w, D, dev = L.w, L.D, L.dev
    T, k, E = w.T, w.top_k, w.E
    counts = torch.empty(E, dtype=torch.int32, device=dev)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
    slot_token = torch.empty(T * k, dtype=torch.int32, device=dev)
    token_slot = torch.empty((T, k), dtype=torch.int32, device=dev)
    v = torch.empty((T, w.d), dtype=w.w_dtype, device=dev)
    xp = torch.empty((T * k, w.d), dtype=w.w_dtype, device=dev)
    h = torch.empty((T * k, w.d_ff), dtype=w.w_dtype, device=dev)
    y = torch.empty((T * k, w.d), dtype=w.w_dtype, device=dev)
    idx, wt, out = torch.empty_like(L.idx), torch.empty_like(L.wt), torch.empty_like(L.out)
    names = ["rmsnorm", "router", "permute", "gate_up", "down", "combine"]
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(len(names) + 1)] for _ in range(a.steps)]

    def run(ev=None):
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
        run()
    barrier()
    for i in range(a.steps):
        run(evs[i])
    torch.cuda.synchronize()
    stage_ms = {n: statistics.mean(evs[i][j].elapsed_time(evs[i][j + 1]) for i in range(a.steps))
                for j, n in enumerate(names)}
    active = int((counts > 0).sum().item())
    S = T * k
    esz = 2 if w.w_dtype == torch.bfloat16 else 4
    gate_up_bytes = active * 2 * w.d_ff * w.d * esz + S * w.d * esz + S * w.d_ff * esz
    gate_up_flops = 2.0 * S * w.d * 2 * w.d_ff
    t_s = stage_ms["gate_up"] / 1000.0
    hbm_bound = gate_up_bytes / (pk["hbm_gbs"] * 1e9) >= gate_up_flops / (pk["bf16_tflops"] * 1e12)
    if hbm_bound:
        roof = {"bound": "hbm", "achieved": gate_up_bytes / t_s / 1e9, "peak": pk["hbm_gbs"], "unit": "GB/s"}
    else:
        roof = {"bound": "tensor", "achieved": gate_up_flops / t_s / 1e12, "peak": pk["bf16_tflops"],
                "unit": "TFLOP/s"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["traffic"] = traffic_for(w.name)
    if roof["traffic"] is not None:
        roof["traffic_note"] = ("DRAM bytes of the same kernel template as run by moe_forward, which gathers the "
                                "token rows from V instead of reading the permuted copy Xp timed here (S*d*2 - "
                                "T*d*2 fewer algorithmic bytes)")
    roof["kernel"] = (gate_up_kernel_name(S, E) if w.w_dtype == torch.bfloat16
                      else "fp32 expert kernel (expert_simt.cu, gate/up + SwiGLU)")
    roof["algorithmic_bytes_per_launch"] = gate_up_bytes
    roof["algorithmic_flops_per_launch"] = gate_up_flops
    roof["launch_ms"] = stage_ms["gate_up"]
    roof["peak_source"] = f"{pk['source']} (burst, kernel timed alone)"
    return stage_ms, roof, active, (counts, offsets, xp)


def e2e_of(L, a, barrier, world, max_over_ranks) -> dict:
    """The same layer through moe_forward with every step's input copied from pinned host memory and every
    step's output copied back to pinned host memory and waited for by the host, inside the timed region.
    The copies run on two copy streams with double-buffered device input and output, so step i+1's input
    copy and step i-1's output copy overlap step i's layer; the host waits for each step's output one step
    later, and the region ends when the last output has reached the host."""
    import torch

    w = L.w
    x_host = L.I["x"].pin_memory()
    out_host = [torch.empty(L.out.shape, dtype=L.out.dtype).pin_memory() for _ in range(2)]
    x_dev = [torch.empty_like(L.D["x"]) for _ in range(2)]
    out_dev = [L.out, torch.empty_like(L.out)]
    comp = torch.cuda.current_stream()
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    ev = lambda: torch.cuda.Event()
    in_done, comp_done, out_done = [ev(), ev()], [ev(), ev()], [ev(), ev()]
    for e in comp_done + out_done:  # every buffer starts free
        e.record(comp)

    def run(n: int, start_event=None):
        for i in range(n):
            b = i % 2
            s_in.wait_event(comp_done[b])  # the layer of step i-2 has read x_dev[b]
            if start_event is not None and i == 0:
                s_in.wait_event(start_event)
            with torch.cuda.stream(s_in):
                x_dev[b].copy_(x_host, non_blocking=True)
            in_done[b].record(s_in)
            comp.wait_event(in_done[b])
            comp.wait_event(out_done[b])  # the output copy of step i-2 has read out_dev[b]
            L.step(x_dev[b], out_dev[b])
            comp_done[b].record(comp)
            s_out.wait_event(comp_done[b])
            with torch.cuda.stream(s_out):
                out_host[b].copy_(out_dev[b], non_blocking=True)
            out_done[b].record(s_out)
            if i >= 1:
                out_done[(i - 1) % 2].synchronize()  # the host has step i-1's result
        comp.wait_event(out_done[(n - 1) % 2])

    run(a.warmup)
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(comp)
    run(a.steps, start_event=e0)
    e1.record(comp)
    barrier()
    ms = e0.elapsed_time(e1)
    L.check_status("in the end-to-end timing")
    value, _ = aggregate(ms, w.T, a.steps, world, max_over_ranks)
    return {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": x_host.numel() * x_host.element_size(),
            "d2h_bytes_per_step": out_host[0].numel() * out_host[0].element_size(),
            "copies": "pinned host memory, two copy streams, double-buffered; the host waits for every output"}


def headline_extras(L, a, barrier, pk, ms_per_step, staged_bufs, active) -> dict:
    """Next-row measurements on the headline workload: the masked layout, block-FP8 experts, and one rank of
    the peer-memory expert-parallel step."""
    import torch

    import moe_layer_forward_b200 as moe

    w, D, dev, status = L.w, L.D, L.dev, L.status
    T, k, E = w.T, w.top_k, w.E
    S = T * k
    esz = 2 if w.w_dtype == torch.bfloat16 else 4
    counts, offsets, xp = staged_bufs
    res = {"masked_layout": None, "fp8_layer": None, "ep_p2p": None}

    if not a.no_masked and w.w_dtype == torch.bfloat16 and S // E <= 32:
        cn, of = counts.cpu(), offsets.cpu()
        cap = int((int(cn.max()) + 15) // 16 * 16)
        xm = torch.zeros((E, cap, w.d), dtype=w.w_dtype, device=dev)
        for e in range(E):  # input preparation, outside the timed region
            xm[e, :int(cn[e])] = xp[int(of[e]):int(of[e]) + int(cn[e])]
        hm = torch.empty((E, cap, w.d_ff), dtype=w.w_dtype, device=dev)
        ym = torch.empty((E, cap, w.d), dtype=w.w_dtype, device=dev)
        ms, _, _ = _timed(lambda: moe.moe_grouped_swiglu_masked(xm, D["W_gate"], D["W_up"], D["W_down"], counts, hm,
                                                                ym, dev_status=status), a.steps, a.warmup, barrier)
        L.check_status("in the masked-layout timing")
        mms = ms / a.steps
        mbytes = active * 3 * w.d_ff * w.d * esz + S * (2 * w.d + 2 * w.d_ff) * esz
        res["masked_layout"] = {"expert_mlp_ms": mms, "tokens_per_s": T / (mms / 1000.0), "cap": cap,
                                "hbm_achieved_gbs": mbytes / (mms / 1000.0) / 1e9,
                                "hbm_frac": mbytes / (mms / 1000.0) / 1e9 / pk["hbm_gbs"],
                                "algorithmic_bytes": mbytes}
        del xm, hm, ym

    if not a.no_fp8 and w.w_dtype == torch.bfloat16 and S // E <= 32:
        Wq = [moe.quantize_fp8_weights(D[n]) for n in ("W_gate", "W_up", "W_down")]
        out8 = torch.empty_like(L.out)
        ws8 = torch.empty(moe.forward_fp8_workspace_bytes(D["x"], D["W_r"], Wq[0][0], out8, k, w.eps),
                          dtype=torch.uint8, device=dev)
        ms, _, _ = _timed(lambda: moe.moe_forward_fp8(D["x"], D["gamma"], D["W_r"], D["b"], *Wq, out8, top_k=k,
                                                      eps=w.eps, ws=ws8, dev_status=status),
                          a.steps, a.warmup, barrier)
        L.check_status("in the FP8 timing")
        fms = ms / a.steps
        # algorithmic bytes: active experts' codes and scales, the input, the output and the router weights
        fbytes = active * 3 * w.d_ff * w.d * (1 + 4 / (128 * 128)) + T * w.d * (D["x"].element_size() +
                                                                                 L.out.element_size()) + E * w.d * 4
        res["fp8_layer"] = {"ms_per_step": fms, "tokens_per_s": T / (fms / 1000.0),
                            "dtype": "e4m3 experts, fp32 router", "algorithmic_bytes": fbytes,
                            "hbm_achieved_gbs": fbytes / (fms / 1000.0) / 1e9,
                            "hbm_frac": fbytes / (fms / 1000.0) / 1e9 / pk["hbm_gbs"],
                            "vs_bf16_layer": ms_per_step / fms}
        del Wq, ws8

    if not a.no_ep and w.w_dtype == torch.bfloat16:
        from moe_layer_forward_b200 import ep_p2p

        peers = ep_p2p.local_peers(1, ep_p2p.capacity_rows(T, 1, k, E), w.d, w.w_dtype, dev)
        ms, _, _ = _timed(lambda: ep_p2p.ep_p2p_forward_emulated([D["x"]], D["gamma"], D["W_r"], D["b"], D["W_gate"],
                                                                 D["W_up"], D["W_down"], top_k=k, eps=w.eps,
                                                                 peers=peers), a.steps, a.warmup, barrier)
        ems = ms / a.steps
        res["ep_p2p"] = {"ranks": 1, "ms_per_step": ems, "tokens_per_s": T / (ems / 1000.0),
                         "vs_moe_forward": ms_per_step / ems,
                         "steps": "routing, permutation maps, dispatch into the receive buffer, layout, grouped MLP "
                                  "over the whole buffer, pull combine; no host synchronisation",
                         "multi_gpu": "not measured (one GPU per call here)"}
        del peers
    return res


def vendor_anchor(L, a, bufs, local) -> dict | None:
    """The expert GEMMs of this library against a vendor grouped GEMM (torch.nn.functional.grouped_mm, a CUTLASS
    kernel) on the same permuted rows, weights and expert segments. Each timing is 3 untimed and 10 timed calls
    after a 0.5 s idle gap, so both run at the burst clock; medians over 3 interleaved rounds. The vendor call
    multiplies the gate and up weights as one fused N = 2 d_ff operand and applies no SwiGLU. Outside the
    timed region; a comparison only, nothing of the layer runs through it."""
    import torch

    import moe_layer_forward_b200 as moe

    w, D, dev = L.w, L.D, L.dev
    F = torch.nn.functional
    if w.w_dtype != torch.bfloat16 or not hasattr(F, "grouped_mm"):
        return None
    counts, offsets, xp = bufs
    S = w.T * w.top_k
    ends = offsets[1:].contiguous()
    wgu = torch.cat([D["W_gate"], D["W_up"]], 1)
    h = torch.empty((S, w.d_ff), dtype=w.w_dtype, device=dev)
    y = torch.empty((S, w.d), dtype=w.w_dtype, device=dev)
    fns = {"ours": (lambda: moe.moe_expert_gate_up(xp, D["W_gate"], D["W_up"], counts, offsets, h),
                    lambda: moe.moe_expert_down(h, D["W_down"], counts, offsets, y)),
           "grouped_mm": (lambda: F.grouped_mm(xp, wgu.transpose(1, 2), offs=ends),
                          lambda: F.grouped_mm(h, D["W_down"].transpose(1, 2), offs=ends))}
    try:
        for f in fns["grouped_mm"]:
            f()
        torch.cuda.synchronize()
    except Exception as e:  # a torch build without the grouped GEMM for this device
        return {"unavailable": f"{type(e).__name__}: {str(e)[:120]}"}
    times = {n: ([], []) for n in fns}
    clk = Clocks(local)
    clk.__enter__()
    for _ in range(3):
        for n, pair in fns.items():
            for j, f in enumerate(pair):
                time.sleep(0.5)
                for _ in range(3):
                    f()
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record()
                for _ in range(10):
                    f()
                e1.record()
                torch.cuda.synchronize()
                times[n][j].append(e0.elapsed_time(e1) / 10)
    clk.__exit__(None, None, None)
    med = {n: {"gate_up_ms": statistics.median(t[0]), "down_ms": statistics.median(t[1])} for n, t in times.items()}
    del wgu, h, y
    return {"vendor": "torch.nn.functional.grouped_mm", **med,
            "ours_over_vendor_time": (med["ours"]["gate_up_ms"] + med["ours"]["down_ms"]) /
                                     (med["grouped_mm"]["gate_up_ms"] + med["grouped_mm"]["down_ms"]),
            "clocks": clk.summary(),
            "note": "vendor gate/up writes g|u (2 d_ff columns) without the SwiGLU product"}


def measure_workload(a, w, dev, world, rank, local, barrier, max_over_ranks, headline: bool) -> dict:
    """Everything the bench reports for one workload: the timed layer, its roofline fractions, the stage
    breakdown and dominant kernel, near-tie tokens, end-to-end throughput and the CPU oracle sample."""
    import torch

    pk = peaks()
    L = Layer(w, dev)
    L.step()
    torch.cuda.synchronize()
    L.check_status("after the first step")
    ms, clk, launches = _timed(L.step, a.steps, a.warmup, barrier, clocks_gpu=local)
    value, ms_per_step = aggregate(ms, w.T, a.steps, world, max_over_ranks)
    L.check_status("in the timed region")
    stage_ms, kroof, active, bufs = staged(L, a, barrier, pk)
    r = {"workload": w.name, "ms_per_step": ms_per_step, "tokens_per_s": value, "steps": a.steps,
         "warmup": a.warmup, "gpu_launches": launches, "clocks": clk, "active_experts": active,
         "layer_roofline": layer_roofline(w, active, ms_per_step, pk), "dominant_kernel": kroof,
         "stages_ms": stage_ms, "near_ties": near_ties(L), "config": config_of(w, world)}
    r["e2e"] = None if a.no_e2e else e2e_of(L, a, barrier, world, max_over_ranks)
    r["vendor_anchor"] = None if (a.no_anchor or world > 1) else vendor_anchor(L, a, bufs, local)
    if headline:
        r.update(headline_extras(L, a, barrier, pk, ms_per_step, bufs, active))
    r["cpu_baseline"] = None
    if rank == 0 and world == 1 and not a.no_cpu_baseline:
        r["cpu_baseline"] = cpu_baseline(L.I, w, seconds=15.0 if headline else 10.0)
    del L, bufs
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return r


def run_ours(a, w):
    import torch
    import torch.distributed as dist

    import synth

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=180), device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    max_over_ranks = reduce_max_fn(dist, dev)
    # the headline workload first; at one GPU the other four workloads follow, one at a time (each freed
    # before the next is built); under torchrun every rank measures the headline workload only
    names = [w.name]
    if world == 1 and a.workloads == "all" and a.shrink == 1:
        names += [n for n in synth.WORKLOADS if n != w.name]
    results = {}
    for n in names:
        wl = w if n == w.name else synth.WORKLOADS[n]
        results[n] = measure_workload(a, wl, dev, world, rank, local, barrier, max_over_ranks, headline=(n == w.name))
    h = results[w.name]

    if rank == 0:
        line = {"metric": METRIC, "value": h["tokens_per_s"], "unit": "tokens/s", "n_gpus": world,
                "steps": a.steps, "warmup": a.warmup, "ms_per_step": h["ms_per_step"], "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "bf16" if w.w_dtype == torch.bfloat16 else "f32",
                "data": "synthetic", "config": h["config"], "roofline": h["dominant_kernel"],
                "layer_roofline": h["layer_roofline"], "cpu_baseline": h["cpu_baseline"], "e2e": h["e2e"],
                "gpu_launches": h["gpu_launches"], "clocks": h["clocks"], "stages_ms": h["stages_ms"],
                "active_experts": h["active_experts"], "near_ties": h["near_ties"],
                "vendor_anchor": h.get("vendor_anchor"), "masked_layout": h.get("masked_layout"), "fp8_layer": h.get("fp8_layer"), "ep_p2p": h.get("ep_p2p")}
        if len(results) > 1:
            keep = ("ms_per_step", "tokens_per_s", "layer_roofline", "dominant_kernel", "stages_ms", "near_ties",
                    "active_experts", "clocks", "gpu_launches", "e2e", "cpu_baseline", "vendor_anchor", "config")
            line["workloads"] = {n: {k: r[k] for k in keep} for n, r in results.items()}
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
