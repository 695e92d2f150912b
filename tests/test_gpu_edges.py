"""Edge cases of the layer on the GPU, against the fp64 oracle: a single token,
the smallest hidden sizes the tensor-core path takes, the largest expert count
with about one row per expert, and the same shapes through the block-FP8
layer, plus a CUDA-graph replay of the FP8 layer."""
import pytest
import torch

import oracle
import synth
from _layer_check import MAX_ABS, REL_L2, errors, oracle_fp8_weights
from test_gpu_parity import _check_layer

pytestmark = pytest.mark.gpu
DEV = "cuda:0"

EDGES = {
    # (T, d, E, d_ff)
    "one_token": (1, 512, 16, 256),
    "smallest_dims": (70, 128, 8, 128),
    "max_experts": (40, 256, 256, 128),
    "max_experts_more_rows": (300, 128, 256, 256),
}


@pytest.fixture(scope="module")
def moe():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import moe_layer_forward_b200 as m

    return m


def cuda(t):
    return t.contiguous().to(DEV)


@pytest.mark.parametrize("name", list(EDGES))
def test_forward_edge_shapes(moe, name):
    T, d, E, d_ff = EDGES[name]
    w = synth.Workload(name, T, d, E, d_ff, seed=900)
    _check_layer(moe, w, synth.make_layer_inputs(w))


def _fp8_layer(moe, w, I):
    D = {n: cuda(t) for n, t in I.items()}
    Wq = [oracle_fp8_weights(oracle, I[n], DEV) for n in ("W_gate", "W_up", "W_down")]
    out = torch.empty((w.T, w.d), dtype=w.out_dtype, device=DEV)
    idx = torch.empty((w.T, w.top_k), dtype=torch.int32, device=DEV)
    wt = torch.empty((w.T, w.top_k), dtype=torch.float32, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    return D, Wq, out, idx, wt, status


def _fp8_reference(w, I, Wq, idx, wt):
    v = oracle.rmsnorm(I["x"], I["gamma"], w.eps).float()
    vq, vs = oracle.quantize_blocks(v, 1)
    counts, offsets, slot_token, token_slot = oracle.permute(idx.cpu(), w.E)
    Wc = [(q.cpu(), s.cpu()) for q, s in Wq]
    r = oracle.fp8_grouped_mlp(vq[slot_token.long()], vs[slot_token.long()], counts, offsets, *Wc[0], *Wc[1], *Wc[2])
    return I["x"].double() + (wt.cpu().double().unsqueeze(-1) * r["y"][token_slot.long()]).sum(1)


@pytest.mark.parametrize("name", ["one_token", "smallest_dims", "max_experts"])
def test_fp8_forward_edge_shapes(moe, name):
    T, d, E, d_ff = EDGES[name]
    w = synth.Workload(name, T, d, E, d_ff, seed=910)
    I = synth.make_layer_inputs(w)
    D, Wq, out, idx, wt, status = _fp8_layer(moe, w, I)
    moe.moe_forward_fp8(D["x"], D["gamma"], D["W_r"], D["b"], *Wq, out, topk_idx=idx, topk_w=wt, dev_status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    max_abs, rel = errors(out, _fp8_reference(w, I, Wq, idx, wt))
    assert rel < REL_L2 and max_abs < MAX_ABS, (max_abs, rel)


def test_fp8_forward_replays_from_a_cuda_graph(moe):
    T, d, E, d_ff = 96, 512, 64, 256
    w = synth.Workload("fp8_graph", T, d, E, d_ff, seed=920)
    I = synth.make_layer_inputs(w)
    D, Wq, out, idx, wt, status = _fp8_layer(moe, w, I)
    x2 = cuda(synth.make_layer_inputs(w.scaled(seed=921))["x"])
    ws = torch.empty(moe.forward_fp8_workspace_bytes(D["x"], D["W_r"], Wq[0][0], out), dtype=torch.uint8, device=DEV)
    args = (D["gamma"], D["W_r"], D["b"], *Wq)
    eager = [torch.empty_like(out) for _ in range(2)]
    moe.moe_forward_fp8(D["x"], *args, eager[0], ws=ws)
    moe.moe_forward_fp8(x2, *args, eager[1], ws=ws)
    torch.cuda.synchronize()
    x_in = D["x"].clone()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        moe.moe_forward_fp8(x_in, *args, out, ws=ws)
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(out, eager[0])
    x_in.copy_(x2)
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(out, eager[1])
    del g
