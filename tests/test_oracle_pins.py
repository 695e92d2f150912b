"""Pins of the CPU oracle to facts the pages and the mathematics fix.

None of these re-types the oracle's formula: each checks a closed form, an
invariant, a brute-force search or a split identity printed on the pages, so
that a dropped term, a wrong sign or index or a transposed operand in
``oracle/oracle.c`` fails at least one of them.
"""
import itertools
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _bf16_exact(x: torch.Tensor) -> torch.Tensor:
    return x.to(torch.bfloat16)


# --------------------------------------------------------------------------- RMSNorm
# 推理计算流梳理 §Norm&Residual: v_j = gamma_j x_j / sqrt(mean(x^2) + eps)

@pytest.mark.parametrize("c", [1.0, 1e-3, -2.5, 37.0])
def test_rmsnorm_constant_row_closed_form(c):
    d = 256
    gamma = synth.normal((d,), 0, 4, 1.0, math.sqrt(0.1))
    x = torch.full((1, d), c, dtype=torch.float32)
    v = oracle.rmsnorm(x, gamma, 1e-5)
    cf = float(np.float32(c))
    expect = gamma.double() * cf / math.sqrt(cf * cf + 1e-5)
    assert torch.allclose(v[0], expect, rtol=1e-14, atol=0)


def test_rmsnorm_unit_rms_and_scale_invariance():
    d = 512
    x = synth.normal((3, d), 1, 1)
    gamma = synth.normal((d,), 1, 4, 1.0, 0.3)
    v = oracle.rmsnorm(x, gamma, 0.0)
    # with eps = 0 the row v/gamma has mean square exactly 1
    ms = ((v / gamma.double()) ** 2).mean(dim=1)
    assert torch.allclose(ms, torch.ones(3, dtype=torch.float64), rtol=1e-13, atol=0)
    # and the map is invariant to scaling x by a power of two
    v8 = oracle.rmsnorm(x * 8.0, gamma, 0.0)
    assert torch.allclose(v8, v, rtol=1e-14, atol=0)
    # eps enters inside the root: for tiny x it pulls the norm below unit rms
    tiny = oracle.rmsnorm(x * 1e-4, gamma, 1e-5)
    assert ((tiny / gamma.double()) ** 2).mean() < 1e-2


def test_rmsnorm_reads_bf16_exactly():
    d = 128
    x = synth.normal((2, d), 2, 1, dtype=torch.bfloat16)
    gamma = torch.ones(d)
    assert torch.equal(oracle.rmsnorm(x, gamma), oracle.rmsnorm(x.float(), gamma))


# --------------------------------------------------------------------------- linear / splits
# Megatron张量并行 (aiqz.cc) column/row-parallel example; LLM 推理并行 §1.1 场景一 (column split)

def test_linear_page_example_and_tp_splits():
    g = json.load(open(os.path.join(GOLDEN, "tp_split_4x4.json")))
    W = torch.tensor(g["W"], dtype=torch.float32)  # [d][f], Y = X W
    X = torch.tensor(g["X"], dtype=torch.float64)
    Wt = W.t().contiguous()  # the oracle stores out x in
    Y = oracle.linear(X, Wt)
    assert Y.tolist() == g["Y"]
    halves = [oracle.linear(X, W[:, :2].t().contiguous()), oracle.linear(X, W[:, 2:].t().contiguous())]
    assert [h.tolist() for h in halves] == g["Y_col_halves"]
    parts = [oracle.linear(X[:2].contiguous(), W[:2, :].t().contiguous()),
             oracle.linear(X[2:].contiguous(), W[2:, :].t().contiguous())]
    assert [p.tolist() for p in parts] == g["Y_row_partials"]
    assert (parts[0] + parts[1]).tolist() == g["Y"]


def test_linear_integer_column_split_exact():
    # scenario 1 of the split analysis: A [3x4], B [4x6] random integers in [0, 10), 3 column blocks
    A = synth.randint((3, 4), 7, 20, 0, 9).double()
    B = synth.randint((4, 6), 7, 21, 0, 9).float()
    full = torch.stack([oracle.linear(A[m], B.t().contiguous()) for m in range(3)])
    blocks = []
    for j in range(3):
        Bj = B[:, 2 * j:2 * j + 2].t().contiguous()
        blocks.append(torch.stack([oracle.linear(A[m], Bj) for m in range(3)]))
    assert torch.equal(torch.cat(blocks, dim=1), full)
    # and the integer product equals numpy's exact integer matmul
    assert np.array_equal(full.numpy().astype(np.int64), A.numpy().astype(np.int64) @ B.numpy().astype(np.int64))


def test_router_logits_one_hot_rows_pick_coordinates():
    d, E = 16, 8
    v = synth.normal((2, d), 3, 1).double()
    W_r = torch.zeros(E, d)
    cols = [3, 0, 15, 7, 7, 1, 9, 2]
    for e, j in enumerate(cols):
        W_r[e, j] = 1.0
    z = oracle.router_logits(v, W_r)
    assert torch.equal(z, v[:, cols])


# --------------------------------------------------------------------------- sigmoid / SiLU

def test_sigmoid_and_silu_identities():
    assert oracle.sigmoid(0.0) == 0.5
    for z in [0.1, 1.0, 3.7, 20.0]:
        assert abs(oracle.sigmoid(-z) + oracle.sigmoid(z) - 1.0) < 2e-16
        assert oracle.sigmoid(z) > oracle.sigmoid(z - 0.05)
    assert oracle.silu(0.0) == 0.0
    for x in [0.3, 1.0, 2.0, 6.5]:
        # SiLU(-x) = SiLU(x) - x
        assert abs(oracle.silu(-x) - (oracle.silu(x) - x)) < 1e-15
    assert abs(oracle.silu(40.0) - 40.0) < 1e-15
    assert 0 > oracle.silu(-40.0) > -1e-15


def test_selection_score_is_one_fp32_rounding():
    # sigmoid(0) + 0 and sigmoid(0) + 0.25 are exact in fp32
    assert oracle.selection_score(0.0, 0.0) == 0.5
    assert oracle.selection_score(0.0, 0.25) == 0.75
    for z, b in [(0.37, -0.05), (-2.0, 0.013), (5.0, 0.1)]:
        s = oracle.selection_score(z, b)
        assert s == float(np.float32(s))  # representable in fp32
        ref = 1.0 / (1.0 + math.exp(-float(np.float32(z)))) + float(np.float32(b))
        assert abs(s - ref) <= 2 * np.spacing(np.float32(abs(ref)))


# --------------------------------------------------------------------------- top-8 selection
# 推理计算流梳理 §MoE Router 过程: I = Top8(s + b), w_i = s_i / sum_I s_j, bias only selects

def test_all_equal_scores_pick_lowest_indices_with_equal_weights():
    for E in (8, 9, 32, 256):
        z = torch.zeros((3, E))
        b = torch.zeros(E)
        idx, w, margin = oracle.select_topk(z, b, 8)
        assert idx.tolist() == [list(range(8))] * 3
        assert torch.equal(w, torch.full((3, 8), 0.125, dtype=torch.float64))
        if E > 8:
            assert margin.tolist() == [0.0] * 3


@pytest.mark.parametrize("E", [8, 9, 12, 16])
def test_topk_matches_brute_force_subset_search(E):
    T, k = 6, 8
    z = synth.normal((T, E), 10 + E, 30, 0.0, 1.0)
    b = synth.uniform((E,), 10 + E, 31, -0.1, 0.1)
    # plant exact ties: equal logits and biases on experts 1, 3 (and 0, E-1 on some tokens)
    z[:, 3] = z[:, 1]
    b[3] = b[1]
    z[::2, E - 1] = z[::2, 0]
    b[E - 1] = b[0]
    idx, w, _ = oracle.select_topk(z, b, k)
    for t in range(T):
        sc = [Fraction(oracle.selection_score(float(z[t, e]), float(b[e]))) for e in range(E)]
        best = None
        for sub in itertools.combinations(range(E), k):  # lexicographic order
            s = sum(sc[e] for e in sub)
            if best is None or s > best[0]:
                best = (s, sub)
        assert sorted(idx[t].tolist()) == list(best[1])
        # listed by descending score, ties by ascending index
        order = sorted(best[1], key=lambda e: (-sc[e], e))
        assert idx[t].tolist() == order


def test_weights_sum_to_one_and_follow_sigmoid_ratios():
    T, E = 50, 64
    z = synth.normal((T, E), 5, 30)
    b = synth.uniform((E,), 5, 31, -0.1, 0.1)
    idx, w, _ = oracle.select_topk(z, b, 8)
    assert torch.all((w.sum(1) - 1.0).abs() <= 8 * 2.0 ** -52)
    # w_i / w_j = sigmoid(z_i) / sigmoid(z_j) (the bias never enters the weights)
    for t in range(0, T, 7):
        s = [oracle.sigmoid(float(z[t, e])) for e in idx[t].tolist()]
        for i in range(1, 8):
            assert abs(w[t, i] / w[t, 0] - s[i] / s[0]) < 1e-14


def test_bias_changes_selection_not_weights():
    T, E = 40, 32
    z = synth.normal((T, E), 6, 30)
    b = synth.uniform((E,), 6, 31, -0.1, 0.1)
    idx, w, margin = oracle.select_topk(z, b, 8)
    # (1) a perturbation far smaller than every margin keeps I and leaves w bit-identical
    eps = float(margin.min()) / 8
    b2 = b + synth.uniform((E,), 6, 32, -eps, eps)
    idx2, w2, _ = oracle.select_topk(z, b2, 8)
    same = [sorted(a) == sorted(c) for a, c in zip(idx.tolist(), idx2.tolist())]
    assert all(same)
    for t in range(T):
        m1 = dict(zip(idx[t].tolist(), w[t].tolist()))
        m2 = dict(zip(idx2[t].tolist(), w2[t].tolist()))
        assert m1 == m2
    # (2) a large bias on one expert forces it first into every I, yet its weight is its sigmoid share
    b3 = b.clone()
    b3[5] = 10.0
    idx3, w3, _ = oracle.select_topk(z, b3, 8)
    assert all(r[0] == 5 for r in idx3.tolist())
    # same selection with the bias moved to another in-set expert gives the same weights
    for t in range(T):
        s = [oracle.sigmoid(float(z[t, e])) for e in idx3[t].tolist()]
        assert abs(w3[t, 0] - s[0] / math.fsum(s)) < 1e-15


def test_margin_is_kth_minus_next_score():
    E = 12
    z = torch.zeros((1, E))
    b = torch.tensor([0.4, 0.3, 0.2, 0.1, 0.0, -0.1, -0.2, -0.25, -0.375, -0.5, -0.6, -0.7])
    idx, _, margin = oracle.select_topk(z, b, 8)
    assert idx[0].tolist() == list(range(8))
    s8 = oracle.selection_score(0.0, float(b[7]))
    s9 = oracle.selection_score(0.0, float(b[8]))
    assert margin[0].item() == float(np.float32(np.float32(s8) - np.float32(s9)))
    assert abs(margin[0].item() - 0.125) < 1e-7


def test_nan_logit_never_selected_before_numbers():
    E = 16
    z = synth.normal((1, E), 8, 30)
    z[0, 2] = float("nan")
    idx, _, _ = oracle.select_topk(z, torch.zeros(E), 8)
    assert 2 not in idx[0].tolist()


# --------------------------------------------------------------------------- expert MLP
# 推理计算流梳理 §实际 MLP 计算策略: y = (SiLU(x W_gate) ⊙ x W_up) W_down

def _experts(E, d, d_ff, seed, dtype=torch.float32):
    Wg = synth.normal((E, d_ff, d), seed, 5, 0.0, 1 / math.sqrt(d), dtype)
    Wu = synth.normal((E, d_ff, d), seed, 6, 0.0, 1 / math.sqrt(d), dtype)
    Wd = synth.normal((E, d, d_ff), seed, 7, 0.0, 1 / math.sqrt(d_ff), dtype)
    return Wg, Wu, Wd


def test_expert_mlp_one_dim_gate_vs_up():
    # d = d_ff = 1: gate weight 1, up weight -1, down weight 3, input 2
    Wg = torch.ones((1, 1, 1))
    Wu = -torch.ones((1, 1, 1))
    Wd = 3 * torch.ones((1, 1, 1))
    h, y = oracle.expert_mlp(torch.tensor([2.0], dtype=torch.float64), Wg, Wu, Wd, 0)
    # SiLU acts on the gate (2), not on the up projection (-2)
    assert h.item() == pytest.approx(-2.0 * oracle.silu(2.0), rel=1e-15)
    assert h.item() != pytest.approx(2.0 * oracle.silu(-2.0), rel=1e-3)
    assert y.item() == pytest.approx(3.0 * h.item(), rel=1e-15)


@pytest.mark.parametrize("p", [2, 4])
def test_expert_mlp_megatron_split_identity(p):
    # gate/up column split, pointwise SiLU, down row split: summing the p partial outputs gives the full MLP
    E, d, d_ff = 3, 64, 128
    Wg, Wu, Wd = _experts(E, d, d_ff, 9)
    v = synth.normal((d,), 9, 1).double()
    for e in range(E):
        h, y = oracle.expert_mlp(v, Wg, Wu, Wd, e)
        c = d_ff // p
        acc = torch.zeros(d, dtype=torch.float64)
        hs = []
        for j in range(p):
            sl = slice(j * c, (j + 1) * c)
            hj, yj = oracle.expert_mlp(v, Wg[:, sl].contiguous(), Wu[:, sl].contiguous(),
                                       Wd[:, :, sl].contiguous(), e)
            hs.append(hj)
            acc += yj
        assert torch.equal(torch.cat(hs), h)  # column split: identical per element
        assert torch.allclose(acc, y, rtol=1e-12, atol=1e-14)  # row split: equal up to summation order


def test_expert_mlp_zero_and_scaling():
    E, d, d_ff = 2, 32, 64
    Wg, Wu, Wd = _experts(E, d, d_ff, 11)
    v = synth.normal((d,), 11, 1).double()
    _, y = oracle.expert_mlp(v, Wg, torch.zeros_like(Wu), Wd, 1)
    assert torch.equal(y, torch.zeros(d, dtype=torch.float64))
    _, y1 = oracle.expert_mlp(v, Wg, Wu, Wd, 1)
    _, y2 = oracle.expert_mlp(v, Wg, Wu, Wd * 2, 1)
    assert torch.equal(y2, 2 * y1)
    # the expert index selects the weights: expert 0 and 1 differ
    _, y0 = oracle.expert_mlp(v, Wg, Wu, Wd, 0)
    assert not torch.allclose(y0, y1)


# --------------------------------------------------------------------------- permutation
# Chitu §Token 分发策略 (token_permutation) and §专家计算实现 (tokens contiguous by expert id)

def test_permute_matches_brute_force_stable_sort():
    T, E, k = 37, 16, 8
    idx = synth.distinct_topk(T, E, k, 12)
    counts, offsets, slot_token, token_slot = oracle.permute(idx, E)
    pairs = sorted(((idx[t, i].item(), t, i) for t in range(T) for i in range(k)))
    assert slot_token.tolist() == [t for _, t, _ in pairs]
    for s, (_, t, i) in enumerate(pairs):
        assert token_slot[t, i].item() == s
    bc = np.bincount(idx.flatten().numpy(), minlength=E)
    assert counts.tolist() == bc.tolist()
    assert offsets.tolist() == [0] + np.cumsum(bc).tolist()


def test_permute_invariants_and_bad_id():
    T, E, k = 100, 64, 8
    idx = synth.distinct_topk(T, E, k, 13)
    counts, offsets, slot_token, token_slot = oracle.permute(idx, E)
    assert counts.sum().item() == T * k
    # every (t, i) owns exactly one row, and the row's token is t
    assert sorted(token_slot.flatten().tolist()) == list(range(T * k))
    for t in range(T):
        for i in range(k):
            assert slot_token[token_slot[t, i]].item() == t
    # rows of one expert are in ascending token order
    for e in range(E):
        seg = slot_token[offsets[e]:offsets[e + 1]].tolist()
        assert seg == sorted(seg) and len(set(seg)) == len(seg)
    bad = idx.clone()
    bad[3, 2] = E
    with pytest.raises(ValueError):
        oracle.permute(bad, E)


def test_permute_then_unpermute_is_identity():
    # with the expert MLP replaced by the identity (y = xp), the weighted un-permute gives
    # sum_i w_i v_t + x_t = v_t + x_t, since the weights sum to one
    T, E, k, d = 24, 16, 8, 32
    idx = synth.distinct_topk(T, E, k, 14)
    v = synth.normal((T, d), 14, 1)
    x = synth.normal((T, d), 14, 2)
    _, _, slot_token, token_slot = oracle.permute(idx, E)
    xp = oracle.gather(v, slot_token)
    onehot = torch.zeros((T, k))
    onehot[:, 3] = 1.0
    out = oracle.combine(xp.float(), token_slot, onehot, x)
    assert torch.equal(out, v.double() + x.double())
    w = torch.full((T, k), 0.125)
    out = oracle.combine(xp.float(), token_slot, w, x)
    assert torch.allclose(out, v.double() + x.double(), rtol=0, atol=1e-6)


# --------------------------------------------------------------------------- whole layer

def _layer_inputs(T, d, E, d_ff, seed, bias="u0.1", wdt=torch.float32, xdt=torch.float32):
    w = synth.Workload("t", T, d, E, d_ff, x_dtype=xdt, w_dtype=wdt, out_dtype=torch.float32, bias=bias, seed=seed)
    return synth.make_layer_inputs(w)


def test_layer_with_identical_experts_is_a_dense_swiglu_mlp():
    T, d, E, d_ff = 6, 32, 12, 48
    I = _layer_inputs(T, d, E, d_ff, 21)
    for name in ("W_gate", "W_up", "W_down"):
        I[name] = I[name][:1].repeat(E, 1, 1).contiguous()
    r = oracle.moe_layer(I["x"], I["gamma"], I["W_r"], I["b"], I["W_gate"], I["W_up"], I["W_down"])
    # dense reference with numpy's matmul: mean-square normalisation, then the gated MLP
    x = I["x"].double().numpy()
    g = I["gamma"].double().numpy()
    v = g * x / np.sqrt((x * x).mean(1, keepdims=True) + 1e-5)
    a = v @ I["W_gate"][0].double().numpy().T
    u = v @ I["W_up"][0].double().numpy().T
    hid = a / (1 + np.exp(-a)) * u
    dense = x + hid @ I["W_down"][0].double().numpy().T
    assert np.allclose(r["out"].numpy(), dense, rtol=1e-12, atol=1e-12)


def test_layer_rows_are_independent_and_forced_routing_reproduces():
    T, d, E, d_ff = 10, 32, 16, 32
    I = _layer_inputs(T, d, E, d_ff, 22)
    args = (I["gamma"], I["W_r"], I["b"], I["W_gate"], I["W_up"], I["W_down"])
    full = oracle.moe_layer(I["x"], *args)
    part = oracle.moe_layer(I["x"][3:7], *args)
    assert torch.equal(part["out"], full["out"][3:7])
    forced = oracle.moe_layer(I["x"], *args, force_idx=full["idx"], force_w=full["w"].float())
    assert torch.allclose(forced["out"], full["out"], rtol=0, atol=1e-6)


def test_layer_is_equivariant_under_expert_relabelling():
    T, d, E, d_ff = 8, 32, 16, 32
    I = _layer_inputs(T, d, E, d_ff, 23)
    args = (I["gamma"], I["W_r"], I["b"], I["W_gate"], I["W_up"], I["W_down"])
    ref = oracle.moe_layer(I["x"], *args)
    perm = torch.tensor(synth.distinct_topk(1, E, E, 23)[0].tolist(), dtype=torch.long)
    pargs = (I["gamma"], I["W_r"][perm].contiguous(), I["b"][perm].contiguous(), I["W_gate"][perm].contiguous(),
             I["W_up"][perm].contiguous(), I["W_down"][perm].contiguous())
    got = oracle.moe_layer(I["x"], *pargs)
    assert torch.equal(got["out"], ref["out"])
    inv = torch.argsort(perm)
    assert torch.equal(perm[got["idx"].long()], ref["idx"].long())
    assert torch.equal(inv[ref["idx"].long()], got["idx"].long())


def test_layer_routes_by_biased_score_but_weights_by_sigmoid():
    # E == k: every expert is chosen, so the output is x + sum_e (s_e / sum s) MLP_e(v)
    T, d, E, d_ff = 3, 16, 8, 16
    I = _layer_inputs(T, d, E, d_ff, 24)
    args = (I["gamma"], I["W_r"], I["b"], I["W_gate"], I["W_up"], I["W_down"])
    r = oracle.moe_layer(I["x"], *args)
    assert sorted(r["idx"][0].tolist()) == list(range(E))
    b2 = I["b"] + 5.0 * synth.uniform((E,), 24, 40, -1, 1)
    r2 = oracle.moe_layer(I["x"], I["gamma"], I["W_r"], b2, I["W_gate"], I["W_up"], I["W_down"])
    assert torch.allclose(r2["out"], r["out"], rtol=0, atol=1e-12)


def test_layer_bf16_inputs_are_read_exactly():
    T, d, E, d_ff = 4, 64, 16, 64
    I = _layer_inputs(T, d, E, d_ff, 25, wdt=torch.bfloat16, xdt=torch.bfloat16)
    args = (I["gamma"], I["W_r"], I["b"])
    a = oracle.moe_layer(I["x"], *args, I["W_gate"], I["W_up"], I["W_down"])
    c = oracle.moe_layer(I["x"].float(), *args, I["W_gate"].float(), I["W_up"].float(), I["W_down"].float())
    assert torch.equal(a["out"], c["out"])


# --------------------------------------------------------------------------- grouped expert MLP (segments)
def _labelled_experts(E, d):
    """Experts whose MLP is y = (e + 1) * x exactly, for rows with x[0] == 1 and integer entries.

    W_gate[e] maps every feature to 64 * x[0] = 64, where SiLU(64) = 64 exactly in fp64 (sigmoid(64)
    rounds to 1); W_up[e] = (e + 1) * I; W_down[e] = I / 64 (a power of two).  So h = 64 (e + 1) x and
    y = (e + 1) x, both exact: a row sent through the wrong expert, or left out, shows at once."""
    Wg = torch.zeros((E, d, d))
    Wg[:, :, 0] = 64.0
    Wu = torch.stack([(e + 1) * torch.eye(d) for e in range(E)])
    Wd = torch.stack([torch.eye(d) / 64.0 for _ in range(E)])
    return Wg, Wu, Wd


def _labelled_rows(S, d, seed):
    x = synth.randint((S, d), seed, 1, -3, 3).double()
    x[:, 0] = 1.0
    return x.float()


def _expected_grouped(x, counts, offsets, E):
    """Row r of expert e's segment -> (e + 1) * x[r]; rows in no segment stay NaN (test-side restatement)."""
    S, d = x.shape
    h = torch.full((S, d), float("nan"), dtype=torch.float64)
    y = torch.full((S, d), float("nan"), dtype=torch.float64)
    for e in range(E):
        lo, n = int(offsets[e]), int(counts[e])
        y[lo:lo + n] = (e + 1) * x[lo:lo + n].double()
        h[lo:lo + n] = 64.0 * (e + 1) * x[lo:lo + n].double()
    return h, y


@pytest.mark.parametrize("counts", [
    [0, 3, 0, 1, 5, 0, 2],        # empty experts first, between and last-but-one; single-row segment
    [4, 0, 0, 0, 0, 0, 1],        # the last expert owns the last row
    [1, 1, 1, 1, 1, 1, 1, 1],     # every segment one row
    [0, 0, 0, 9],                 # only the last expert has rows
])
def test_grouped_mlp_sends_each_segment_through_its_own_expert(counts):
    E, d = len(counts), 8
    c = torch.tensor(counts, dtype=torch.int32)
    o = torch.zeros(E + 1, dtype=torch.int32)
    o[1:] = torch.cumsum(c, 0)
    x = _labelled_rows(int(c.sum()), d, 700 + E)
    Wg, Wu, Wd = _labelled_experts(E, d)
    h, y = oracle.grouped_mlp(x, c, o, Wg, Wu, Wd)
    h_ref, y_ref = _expected_grouped(x, c, o, E)
    assert torch.equal(y, y_ref) and torch.equal(h, h_ref)


def test_grouped_mlp_leaves_rows_outside_every_segment_untouched():
    # segments with gaps between them and rows past the last one: those rows keep their NaN fill
    E, d, S = 4, 8, 20
    c = torch.tensor([2, 0, 3, 4], dtype=torch.int32)
    o = torch.tensor([1, 5, 6, 12, 16], dtype=torch.int32)  # rows 0, 3-5, 9-11 and 16-19 belong to no segment
    x = _labelled_rows(S, d, 710)
    Wg, Wu, Wd = _labelled_experts(E, d)
    _, y = oracle.grouped_mlp(x, c, o, Wg, Wu, Wd)
    _, y_ref = _expected_grouped(x, c, o, E)
    covered = torch.zeros(S, dtype=torch.bool)
    for e in range(E):
        covered[int(o[e]):int(o[e]) + int(c[e])] = True
    assert torch.isnan(y[~covered]).all()
    assert torch.equal(y[covered], y_ref[covered])


def test_grouped_mlp_over_the_permutation_reproduces_each_pick():
    # real routing through oracle.permute and oracle.gather: the row that holds pick i of token t must
    # come out as (idx[t][i] + 1) * v[t], the pick's own expert applied to its own token
    T, E, k, d = 40, 6, 3, 8
    idx = synth.distinct_topk(T, E, k, 720)
    v = _labelled_rows(T, d, 721)
    counts, offsets, slot_token, token_slot = oracle.permute(idx, E)
    xp = oracle.gather(v, slot_token).float()
    Wg, Wu, Wd = _labelled_experts(E, d)
    _, y = oracle.grouped_mlp(xp, counts, offsets, Wg, Wu, Wd)
    for t in range(T):
        for i in range(k):
            r = int(token_slot[t, i])
            assert torch.equal(y[r], (int(idx[t, i]) + 1) * v[t].double())
