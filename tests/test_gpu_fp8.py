"""GPU parity of the block-FP8 expert path through the C ABI.

Quantisation: codes and scales bit-exact against the oracle (both decide in fp32).
Expert MLP: h codes against the fp64 oracle within half a code step (a code may
differ where the fp32 and fp64 h straddle a rounding boundary), y against the
oracle evaluated on the GPU's own h codes (so only fp32 accumulation and bf16
output rounding remain).  Layer: against the oracle's composition of the same
steps, with the GPU's routing (the bf16 path's experts, weights within 1e-6).
"""
import math

import pytest
import torch

import oracle
import synth
from _layer_check import MAX_ABS, REL_L2, errors, oracle_fp8_weights

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


@pytest.fixture(scope="module")
def moe():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import moe_layer_forward_b200 as m

    return m


def cuda(t):
    return t.contiguous().to(DEV)


def deq(q, s, blk_rows):
    v = q.cpu().view(torch.float8_e4m3fn).to(torch.float64)
    sc = s.cpu().double().repeat_interleave(blk_rows, 0)[:q.shape[0]].repeat_interleave(128, 1)
    return v * sc


@pytest.mark.parametrize("rows,cols,blk", [(300, 384, 1), (300, 384, 128), (256, 4096, 128), (5, 128, 1)])
@pytest.mark.parametrize("dt", [torch.bfloat16, torch.float32])
def test_quantize_matches_oracle_bit_for_bit(moe, rows, cols, blk, dt):
    x = synth.normal((rows, cols), 800 + rows, blk, dtype=dt)
    x[3, :128] = 0  # an all-zero input block
    x[min(rows - 1, 200), 5] = 300.0  # an outlier
    q = torch.empty((rows, cols), dtype=torch.uint8, device=DEV)
    s = torch.empty(((rows + blk - 1) // blk, cols // 128), dtype=torch.float32, device=DEV)
    moe.quantize_fp8(cuda(x), blk, q, s)
    torch.cuda.synchronize()
    q_ref, s_ref = oracle.quantize_blocks(x, blk)
    assert torch.equal(s.cpu(), s_ref)
    assert torch.equal(q.cpu(), q_ref)


COUNTS = {
    "r16": [0, 1, 3, 8, 16, 17, 5, 0, 2, 9, 7, 4],       # avg <= 8: 16 token columns per tile
    "r32": [12, 0, 33, 31, 70, 9, 20, 1],                # avg > 8: 32 columns, several row blocks
}


def _expert_inputs(counts, d, d_ff, seed):
    E, S = len(counts), sum(counts)
    ct = torch.tensor(counts, dtype=torch.int32)
    offs = torch.zeros(E + 1, dtype=torch.int32)
    offs[1:] = torch.cumsum(ct, 0)
    x = synth.normal((S, d), seed, 1, dtype=torch.bfloat16)
    xq, xs = oracle.quantize_blocks(x, 1)
    W = [synth.normal((E, n, k), seed, 5 + i, 0.0, 1 / math.sqrt(k), torch.bfloat16)
         for i, (n, k) in enumerate([(d_ff, d), (d_ff, d), (d, d_ff)])]
    Wq = []
    for w in W:
        q, s = oracle.quantize_blocks(w.reshape(-1, w.shape[2]), 128)
        Wq.append((q.reshape(w.shape), s.reshape(w.shape[0], w.shape[1] // 128, w.shape[2] // 128)))
    return ct, offs, xq, xs, Wq


@pytest.mark.parametrize("case", list(COUNTS))
@pytest.mark.parametrize("d,d_ff", [(256, 256), (512, 384), (384, 256)])  # down tiles of 256 / 256 / 128 features
def test_fp8_grouped_swiglu_matches_oracle(moe, case, d, d_ff):
    counts = COUNTS[case]
    ct, offs, xq, xs, Wq = _expert_inputs(counts, d, d_ff, seed=810)
    S = sum(counts)
    hq = torch.zeros((S, d_ff), dtype=torch.uint8, device=DEV)
    hs = torch.zeros((S, d_ff // 128), dtype=torch.float32, device=DEV)
    y = torch.empty((S, d), dtype=torch.bfloat16, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    dev_w = [(cuda(q), cuda(s)) for q, s in Wq]
    moe.moe_grouped_swiglu_fp8(cuda(xq), cuda(xs), *dev_w, cuda(ct), cuda(offs), hq, hs, y, dev_status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    r = oracle.fp8_grouped_mlp(xq, xs, ct, offs, *Wq[0], *Wq[1], *Wq[2], hq_in=hq.cpu(), hs_in=hs.cpu())
    h_ref = r["h"]
    # h: the GPU's codes dequantise to the fp64 h within half a code step (plus fp32 accumulation)
    h_gpu = deq(hq, hs, 1)
    rms = h_ref.pow(2).mean().sqrt().item()
    sc = hs.cpu().double().repeat_interleave(128, 1)
    assert ((h_gpu - h_ref).abs() <= h_ref.abs() * 2.0 ** -4 + sc * 2.0 ** -10 + 1e-5 * rms).all()
    assert ((hs.cpu().double() - r["hs"].double()).abs() <= 1e-5 * r["hs"].double()).all()
    assert (hq.cpu() != r["hq"]).float().mean().item() < 2e-3  # codes differ only at rounding boundaries
    # y from the GPU's own h codes: fp32 accumulation and bf16 rounding only
    y_ref = r["y"]
    yr = y.cpu().double()
    rms_y = y_ref.pow(2).mean().sqrt().item()
    assert ((yr - y_ref).abs() <= 2.0 ** -8 * y_ref.abs() + 1e-4 * rms_y).all()


SMALL = {
    # (T, d, E, d_ff, x dtype, out dtype)
    "decode_like": (96, 512, 64, 256, torch.bfloat16, torch.bfloat16),
    "wider": (200, 256, 16, 384, torch.float32, torch.float32),
}


@pytest.mark.parametrize("name", list(SMALL))
def test_fp8_forward_matches_oracle_composition(moe, name):
    T, d, E, d_ff, xd, od = SMALL[name]
    w = synth.Workload(name, T, d, E, d_ff, x_dtype=xd, out_dtype=od, seed=820)
    I = synth.make_layer_inputs(w)
    D = {n: cuda(t) for n, t in I.items()}
    Wq = [oracle_fp8_weights(oracle, I[n], DEV) for n in ("W_gate", "W_up", "W_down")]
    out = torch.empty((T, d), dtype=od, device=DEV)
    idx = torch.empty((T, 8), dtype=torch.int32, device=DEV)
    wt = torch.empty((T, 8), dtype=torch.float32, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    moe.moe_forward_fp8(D["x"], D["gamma"], D["W_r"], D["b"], *Wq, out, topk_idx=idx, topk_w=wt, dev_status=status)
    # the router is the bf16 path's, on the same 1/rms (both sum the squares per CTA for small batches):
    # the same experts and weights to the bit
    out_bf = torch.empty_like(out)
    idx_bf, wt_bf = torch.empty_like(idx), torch.empty_like(wt)
    moe.moe_forward(D["x"], D["gamma"], D["W_r"], D["b"], D["W_gate"], D["W_up"], D["W_down"], out_bf,
                    topk_idx=idx_bf, topk_w=wt_bf)
    torch.cuda.synchronize()
    assert status.item() == 0
    assert torch.equal(idx, idx_bf) and torch.equal(wt, wt_bf)
    # the oracle's composition of the same steps on the GPU's routing
    v = oracle.rmsnorm(I["x"], I["gamma"], w.eps).float()
    vq, vs = oracle.quantize_blocks(v, 1)
    counts, offsets, slot_token, token_slot = oracle.permute(idx.cpu(), E)
    Wq_cpu = [(q.cpu(), s.cpu()) for q, s in Wq]
    r = oracle.fp8_grouped_mlp(vq[slot_token.long()], vs[slot_token.long()], counts, offsets, *Wq_cpu[0],
                               *Wq_cpu[1], *Wq_cpu[2])
    yk = r["y"][token_slot.long()]  # [T][k][d]
    ref = I["x"].double() + (wt.cpu().double().unsqueeze(-1) * yk).sum(1)
    max_abs, rel = errors(out, ref)
    assert rel < REL_L2 and max_abs < MAX_ABS, (max_abs, rel)


def test_fp8_forward_full_decode_size_sampled(moe):
    # the decode workload's full sizes (T=128, d=4096, E=128, d_ff=1536) through the FP8 layer; the oracle
    # evaluates the expert MLP only for the slots of a sample of tokens
    w = synth.WORKLOADS["decode"]
    I = synth.make_layer_inputs(w)
    D = {n: cuda(t) for n, t in I.items()}
    Wq = [oracle_fp8_weights(oracle, I[n], DEV) for n in ("W_gate", "W_up", "W_down")]
    out = torch.empty((w.T, w.d), dtype=w.out_dtype, device=DEV)
    idx = torch.empty((w.T, 8), dtype=torch.int32, device=DEV)
    wt = torch.empty((w.T, 8), dtype=torch.float32, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    moe.moe_forward_fp8(D["x"], D["gamma"], D["W_r"], D["b"], *Wq, out, topk_idx=idx, topk_w=wt, dev_status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    tokens = [0, 1, 37, 64, 99, w.T - 1]
    v = oracle.rmsnorm(I["x"][tokens], I["gamma"], w.eps).float()
    vq, vs = oracle.quantize_blocks(v, 1)
    sub_idx = idx.cpu()[tokens]
    counts, offsets, slot_token, token_slot = oracle.permute(sub_idx, w.E)
    Wq_cpu = [(q.cpu(), s.cpu()) for q, s in Wq]
    r = oracle.fp8_grouped_mlp(vq[slot_token.long()], vs[slot_token.long()], counts, offsets, *Wq_cpu[0],
                               *Wq_cpu[1], *Wq_cpu[2])
    ref = I["x"][tokens].double() + (wt.cpu()[tokens].double().unsqueeze(-1) * r["y"][token_slot.long()]).sum(1)
    max_abs, rel = errors(out.cpu()[tokens], ref)
    assert rel < REL_L2 and max_abs < MAX_ABS, (max_abs, rel)
