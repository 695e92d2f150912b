"""Tensor-parallel experts sliced on one GPU: N = 2 and 4 ranks emulated in one
process.  Each rank runs the library's grouped MLP on its d_ff slice of every
expert and the weighted combine of its partial output (residual on rank 0);
the sum of the partials (what the all-reduce computes) must match the fp64
oracle layer on the GPU's routing within the parity tolerances, and each
reduce-scatter block (rows [r T/N, (r+1) T/N) of that sum) must equal those
rows.  The partial outputs differ from rank to rank (each holds other
features), so this checks the column/row split itself, which a one-rank
group cannot."""
import pytest
import torch

import oracle
import synth
from _layer_check import MAX_ABS, REL_L2, check_routing, errors

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


@pytest.fixture(scope="module")
def moe():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import moe_layer_forward_b200 as m

    return m


@pytest.mark.parametrize("N", [2, 4])
@pytest.mark.parametrize("shape", [(96, 512, 64, 512), (1200, 256, 8, 512), (256, 256, 16, 1024)])
def test_sliced_tensor_parallel_partials_sum_to_the_layer(moe, N, shape):
    from moe_layer_forward_b200 import tp

    T, d, E, d_ff = shape
    w = synth.Workload("tp_sliced", T, d, E, d_ff, seed=970 + N)
    I = synth.make_layer_inputs(w)
    D = {n: t.to(DEV) for n, t in I.items()}
    parts, idx, wt = tp.tp_partials_emulated(D["x"], D["gamma"], D["W_r"], D["b"], D["W_gate"], D["W_up"],
                                             D["W_down"], N, top_k=w.top_k, eps=w.eps)
    torch.cuda.synchronize()
    # the ranks hold different features: no partial is the layer, each carries a share of the MoE output
    moe_parts = [p - (D["x"].float() if r == 0 else 0) for r, p in enumerate(parts)]
    assert all(mp.abs().max().item() > 0 for mp in moe_parts)
    total = torch.stack(parts).sum(0)
    ref = oracle.moe_layer(I["x"], I["gamma"], I["W_r"], I["b"], I["W_gate"], I["W_up"], I["W_down"], k=w.top_k,
                           eps=w.eps, force_idx=idx.cpu(), force_w=wt.cpu())["out"]
    max_abs, rel = errors(total.to(w.out_dtype), ref)
    assert max_abs <= MAX_ABS and rel <= REL_L2, (max_abs, rel)
    # the split itself, without the residual: the MoE part of the sum against the oracle's
    m_abs, m_rel = errors(total - D["x"].float(), ref - I["x"].double())
    assert m_rel <= 2e-2, m_rel
    # reduce-scatter blocks: rank r receives the sum over ranks of rows [r T/N, (r+1) T/N) of the partials
    for r in range(N):
        rows = slice(r * T // N, (r + 1) * T // N)
        block = torch.stack([p[rows] for p in parts]).sum(0)
        b_abs, b_rel = errors(block.to(w.out_dtype), ref[rows])
        assert b_abs <= MAX_ABS and b_rel <= REL_L2, (r, b_abs, b_rel)
    # the routing is the single-GPU layer's (moe_route), bit-exact given its logits
    logits = torch.empty((T, E), dtype=torch.float32, device=DEV)
    i2, w2 = torch.empty_like(idx), torch.empty_like(wt)
    moe.moe_route(D["x"], D["gamma"], D["W_r"], D["b"], i2, w2, w.eps, logits=logits)
    assert torch.equal(i2, idx) and torch.equal(w2, wt)
    check_routing(oracle, logits, I["b"], idx, wt, w.top_k)
