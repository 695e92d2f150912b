"""The tensor-core kernels' failure path, on the GPU, without a fault or a hang.

Every wait of those kernels on another of their roles is bounded.  Here the
library's test switch (moe_set_wait_limit with inject_stall) makes each kernel
wait once on a barrier that nothing completes, with a short limit, on valid
inputs.  The wait must run out; the call must then return with MOE_DEV_TIMEOUT
in the status word, after its kernels have drained the copies and MMAs they had
issued; and the next call on the same stream, with the switch off, must give
exactly the result of a call made before (which itself matches the oracle).
"""
import math

import pytest
import torch

import synth
from test_gpu_parity import SMALL, _check_layer

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
LIMIT_NS = 2_000_000  # 2 ms


@pytest.fixture(scope="module")
def moe():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import moe_layer_forward_b200 as m

    return m


def _stalled(moe, fn):
    """Run fn() with every tensor-core kernel stalling once under a short wait limit; return its status."""
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    torch.cuda.synchronize()
    moe.set_wait_limit(LIMIT_NS, inject_stall=True)
    try:
        fn(status)
    finally:
        moe.set_wait_limit(0, inject_stall=False)
    torch.cuda.synchronize()
    return status.item()


# (E, rows per expert, d, d_ff): each average picks one GEMM form
GEMM_CASES = {
    "weights_as_m": (16, 4, 512, 256),
    "rows_as_m": (4, 100, 512, 256),
    "row_block_pairs": (4, 300, 512, 256),
    "cta_pairs": (2, 800, 256, 256),
}


@pytest.mark.parametrize("case", list(GEMM_CASES))
def test_expert_gemms_time_out_and_recover(moe, case):
    E, per, d, d_ff = GEMM_CASES[case]
    S = E * per
    xp = synth.normal((S, d), 830, 1, dtype=torch.bfloat16).to(DEV)
    Wg = synth.normal((E, d_ff, d), 830, 2, 0.0, 1 / math.sqrt(d), torch.bfloat16).to(DEV)
    Wu = synth.normal((E, d_ff, d), 830, 3, 0.0, 1 / math.sqrt(d), torch.bfloat16).to(DEV)
    Wd = synth.normal((E, d, d_ff), 830, 4, 0.0, 1 / math.sqrt(d_ff), torch.bfloat16).to(DEV)
    counts = torch.full((E,), per, dtype=torch.int32, device=DEV)
    offsets = (torch.arange(E + 1, dtype=torch.int32) * per).to(DEV)

    def call(status=None):
        h = torch.empty((S, d_ff), dtype=torch.bfloat16, device=DEV)
        y = torch.empty((S, d), dtype=torch.bfloat16, device=DEV)
        moe.moe_grouped_swiglu(xp, Wg, Wu, Wd, counts, offsets, h, y, dev_status=status)
        return h, y

    h0, y0 = call()
    st = _stalled(moe, call)
    assert st & moe.MOE_DEV_TIMEOUT
    h1, y1 = call()
    torch.cuda.synchronize()
    assert torch.equal(h1, h0) and torch.equal(y1, y0)


def test_fp8_expert_gemms_time_out_and_recover(moe):
    E, per, d, d_ff = 16, 4, 512, 256
    S = E * per
    x = synth.normal((S, d), 831, 1, dtype=torch.bfloat16).to(DEV)
    xq = torch.empty((S, d), dtype=torch.uint8, device=DEV)
    xs = torch.empty((S, d // 128), dtype=torch.float32, device=DEV)
    moe.quantize_fp8(x, 1, xq, xs)
    Wq = [moe.quantize_fp8_weights(synth.normal(shape, 831, 2 + i, 0.0, 0.05, torch.bfloat16).to(DEV))
          for i, shape in enumerate([(E, d_ff, d), (E, d_ff, d), (E, d, d_ff)])]
    counts = torch.full((E,), per, dtype=torch.int32, device=DEV)
    offsets = (torch.arange(E + 1, dtype=torch.int32) * per).to(DEV)

    def call(status=None):
        hq = torch.empty((S, d_ff), dtype=torch.uint8, device=DEV)
        hs = torch.empty((S, d_ff // 128), dtype=torch.float32, device=DEV)
        y = torch.empty((S, d), dtype=torch.bfloat16, device=DEV)
        moe.moe_grouped_swiglu_fp8(xq, xs, *Wq, counts, offsets, hq, hs, y, dev_status=status)
        return hq, hs, y

    r0 = call()
    st = _stalled(moe, call)
    assert st & moe.MOE_DEV_TIMEOUT
    r1 = call()
    torch.cuda.synchronize()
    for a, b in zip(r0, r1):
        assert torch.equal(a, b)


@pytest.mark.parametrize("name", ["decode_like", "prefill_like", "dual_like"])
def test_layer_times_out_and_the_next_call_matches_the_oracle(moe, name):
    # the whole layer: router logits and both expert GEMMs stall (with few rows per expert the gate/up GEMM
    # gathers its rows in place; with ~300 it runs two-row-block tiles on a dynamic schedule; with many, CTA pairs)
    T, d, E, d_ff, xd, wd, od = SMALL[name]
    dt = {"bf16": torch.bfloat16, "f32": torch.float32}
    w = synth.Workload(name, T, d, E, d_ff, x_dtype=dt[xd], w_dtype=dt[wd], out_dtype=dt[od], seed=832)
    I = synth.make_layer_inputs(w)
    D = {n: t.to(DEV) for n, t in I.items()}

    def call(status=None):
        out = torch.empty((T, d), dtype=w.out_dtype, device=DEV)
        idx = torch.empty((T, w.top_k), dtype=torch.int32, device=DEV)
        wt = torch.empty((T, w.top_k), dtype=torch.float32, device=DEV)
        logits = torch.empty((T, E), dtype=torch.float32, device=DEV)
        moe.moe_forward(D["x"], D["gamma"], D["W_r"], D["b"], D["W_gate"], D["W_up"], D["W_down"], out,
                        top_k=w.top_k, eps=w.eps, topk_idx=idx, topk_w=wt, logits=logits, dev_status=status)
        return out, idx, wt, logits

    first = call()
    st = _stalled(moe, call)
    assert st & moe.MOE_DEV_TIMEOUT
    again = call()
    torch.cuda.synchronize()
    for a, b in zip(first, again):
        assert torch.equal(a, b)
    _check_layer(moe, w, I, result=again)
