"""GPU parity: every step of the CUDA path, called through the C ABI, against
the fp64 oracle on the same seeded inputs.  Integer and index results must be
bit-exact; floating results within the stated tolerances."""
import math

import pytest
import torch

import oracle
import synth
from _layer_check import MAX_ABS, REL_L2, check_routing, errors

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def moe():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import moe_layer_forward_b200 as m

    return m


DEV = "cuda:0"
DT = {"f32": torch.float32, "bf16": torch.bfloat16}


def cuda(t):
    return t.contiguous().to(DEV)


# bf16 rounding of a result: at most half an ulp (2^-9 relative); 2^-8 leaves room for fp32 sums
def assert_close_rounded(got, ref, rel=2.0 ** -8, rms_frac=1e-4):
    got = got.double().cpu()
    ref = ref.double().cpu()
    rms = ref.pow(2).mean().sqrt().item()
    bound = rel * ref.abs() + rms_frac * rms
    bad = (got - ref).abs() > bound
    assert not bad.any(), f"{bad.sum().item()} of {bad.numel()} outside tolerance; worst " \
                          f"{((got - ref).abs() - bound).max().item():.3g}"


# --------------------------------------------------------------------------- step 1: RMSNorm
@pytest.mark.parametrize("T,d", [(37, 4096), (5, 256), (300, 1024)])
@pytest.mark.parametrize("xdt,vdt", [("bf16", "bf16"), ("f32", "f32"), ("f32", "bf16"), ("bf16", "f32")])
def test_rmsnorm(moe, T, d, xdt, vdt):
    x = synth.normal((T, d), 100 + T, 1, dtype=DT[xdt])
    gamma = synth.normal((d,), 100 + T, 4, 1.0, math.sqrt(0.1))
    v = torch.empty((T, d), dtype=DT[vdt], device=DEV)
    moe.moe_rmsnorm(cuda(x), cuda(gamma), 1e-5, v)
    ref = oracle.rmsnorm(x, gamma, 1e-5)
    if vdt == "f32":
        assert_close_rounded(v, ref, rel=1e-5, rms_frac=1e-6)
    else:
        assert_close_rounded(v, ref)


# --------------------------------------------------------------------------- step 2: router
@pytest.mark.parametrize("T,d,E,k", [(300, 512, 32, 8), (129, 4096, 128, 8), (64, 256, 256, 8), (70, 512, 16, 2),
                                     (33, 256, 8, 8), (45, 256, 9, 1)])
@pytest.mark.parametrize("vdt", ["f32", "bf16"])
def test_router_topk(moe, T, d, E, k, vdt):
    v = synth.normal((T, d), 200 + E, 1, dtype=DT[vdt])
    W_r = synth.normal((E, d), 200 + E, 2, 0.0, 1 / math.sqrt(d))
    b = synth.uniform((E,), 200 + E, 3, -0.1, 0.1)
    idx = torch.empty((T, k), dtype=torch.int32, device=DEV)
    w = torch.empty((T, k), dtype=torch.float32, device=DEV)
    logits = torch.empty((T, E), dtype=torch.float32, device=DEV)
    margin = torch.empty(T, dtype=torch.float32, device=DEV)
    moe.moe_router_topk(cuda(v), cuda(W_r), cuda(b), idx, w, logits, margin)
    z_ref = oracle.router_logits(v.double(), W_r)
    assert (logits.cpu().double() - z_ref).abs().max().item() < 1e-4
    check_routing(oracle, logits, b, idx, w, k)
    _, _, m_ref = oracle.select_topk(logits.cpu(), b, k)
    if E > k:
        assert torch.equal(margin.cpu(), m_ref)
    else:
        assert torch.isinf(margin.cpu()).all()


# bf16 cases cover an expert count that is not a multiple of the 64-expert block (E = 40) and, with T = 640 at
# d = 4096, K splits of two 128-column chunks each of which the last ten are empty (their partial sums are zero)
@pytest.mark.parametrize("T,d,E,k,xdt", [(300, 512, 32, 8, "bf16"), (129, 4096, 128, 8, "bf16"), (64, 256, 256, 8, "bf16"),
                                         (70, 264, 16, 2, "bf16"), (90, 512, 64, 8, "f32"), (1, 1024, 128, 8, "bf16"),
                                         (50, 256, 40, 8, "bf16"), (640, 4096, 128, 8, "bf16")])
def test_route_is_the_forward_routing_and_matches_the_oracle(moe, T, d, E, k, xdt):
    # moe_route: RMSNorm folded into the router (bf16 x with d % 128 == 0: three exact bf16 products per
    # step; otherwise normalised rows in 3xTF32); logits within 1e-4 of the fp64 oracle, routing bit-exact
    # given them, and identical to what moe_forward routes
    x = synth.normal((T, d), 250 + E, 1, dtype=DT[xdt])
    gamma = synth.normal((d,), 250 + E, 4, 1.0, math.sqrt(0.1))
    W_r = synth.normal((E, d), 250 + E, 2, 0.0, 1 / math.sqrt(d))
    b = synth.uniform((E,), 250 + E, 3, -0.1, 0.1)
    idx = torch.empty((T, k), dtype=torch.int32, device=DEV)
    w = torch.empty((T, k), dtype=torch.float32, device=DEV)
    logits = torch.empty((T, E), dtype=torch.float32, device=DEV)
    margin = torch.empty(T, dtype=torch.float32, device=DEV)
    moe.moe_route(cuda(x), cuda(gamma), cuda(W_r), cuda(b), idx, w, 1e-5, logits=logits, margin=margin)
    z_ref = oracle.router_logits(oracle.rmsnorm(x, gamma, 1e-5), W_r)
    assert (logits.cpu().double() - z_ref).abs().max().item() < 1e-4
    check_routing(oracle, logits, b, idx, w, k)
    _, _, m_ref = oracle.select_topk(logits.cpu(), b, k)
    assert torch.equal(margin.cpu(), m_ref)
    if d % 128 == 0:  # the layer itself (bf16 experts need d % 128 == 0)
        d_ff = 128
        Wg = cuda(synth.normal((E, d_ff, d), 251, 5, 0.0, 1 / math.sqrt(d), torch.bfloat16))
        Wd = cuda(synth.normal((E, d, d_ff), 251, 7, 0.0, 1 / math.sqrt(d_ff), torch.bfloat16))
        out = torch.empty((T, d), dtype=DT[xdt], device=DEV)
        i2, w2 = torch.empty_like(idx), torch.empty_like(w)
        moe.moe_forward(cuda(x), cuda(gamma), cuda(W_r), cuda(b), Wg, Wg, Wd, out, top_k=k, topk_idx=i2, topk_w=w2)
        torch.cuda.synchronize()
        assert torch.equal(i2, idx) and torch.equal(w2, w)


def test_router_all_equal_scores_pick_lowest_indices(moe):
    T, d, E = 20, 256, 64
    v = torch.zeros((T, d), device=DEV)
    W_r = cuda(synth.normal((E, d), 1, 2))
    b = torch.zeros(E, device=DEV)
    idx = torch.empty((T, 8), dtype=torch.int32, device=DEV)
    w = torch.empty((T, 8), dtype=torch.float32, device=DEV)
    moe.moe_router_topk(v, W_r, b, idx, w)
    assert idx.cpu().tolist() == [list(range(8))] * T
    assert torch.equal(w.cpu(), torch.full((T, 8), 0.125))


# --------------------------------------------------------------------------- step 3: permute
def _idx(T, E, k, kind, seed):
    if kind == "uniform":
        return synth.distinct_topk(T, E, k, seed)
    if kind == "hot":  # every token picks experts 0..k-1 (in a shuffled order)
        base = synth.distinct_topk(T, k, k, seed)
        return base.clone()
    raise ValueError(kind)


@pytest.mark.parametrize("T,E,k,kind", [(1, 16, 8, "uniform"), (255, 64, 8, "uniform"), (256, 64, 8, "uniform"),
                                        (257, 64, 8, "uniform"), (1000, 128, 8, "uniform"), (700, 256, 8, "hot"),
                                        (513, 8, 8, "uniform"), (300, 32, 1, "uniform"), (200, 256, 8, "hot")])
@pytest.mark.parametrize("vdt", ["bf16", "f32"])
def test_permute_bit_exact(moe, T, E, k, kind, vdt):
    d = 64
    idx = _idx(T, E, k, kind, T + E)
    v = synth.normal((T, d), T, 1, dtype=DT[vdt])
    S = T * k
    counts = torch.empty(E, dtype=torch.int32, device=DEV)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=DEV)
    slot_token = torch.empty(S, dtype=torch.int32, device=DEV)
    token_slot = torch.empty((T, k), dtype=torch.int32, device=DEV)
    xp = torch.empty((S, d), dtype=DT[vdt], device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    moe.moe_permute(cuda(v), cuda(idx), E, counts, offsets, slot_token, token_slot, xp, dev_status=status)
    c_ref, o_ref, st_ref, ts_ref = oracle.permute(idx, E)
    assert torch.equal(counts.cpu(), c_ref)
    assert torch.equal(offsets.cpu(), o_ref)
    assert torch.equal(slot_token.cpu(), st_ref)
    assert torch.equal(token_slot.cpu(), ts_ref)
    assert torch.equal(xp.cpu(), v[st_ref.long()])
    assert status.item() == 0


def test_permute_bad_expert_id_sets_status(moe):
    T, E, k, d = 40, 16, 4, 64
    idx = synth.distinct_topk(T, E, k, 5)
    idx[7, 2] = E  # out of range
    idx[9, 0] = -3
    v = cuda(synth.normal((T, d), 5, 1, dtype=torch.bfloat16))
    counts = torch.empty(E, dtype=torch.int32, device=DEV)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=DEV)
    slot_token = torch.full((T * k,), -7, dtype=torch.int32, device=DEV)
    token_slot = torch.empty((T, k), dtype=torch.int32, device=DEV)
    xp = torch.empty((T * k, d), dtype=torch.bfloat16, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    moe.moe_permute(v, cuda(idx), E, counts, offsets, slot_token, token_slot, xp, dev_status=status)
    assert status.item() & moe.MOE_DEV_BAD_EXPERT_ID
    ts = token_slot.cpu()
    assert ts[7, 2].item() == -1 and ts[9, 0].item() == -1
    assert counts.sum().item() == T * k - 2
    assert offsets[E].item() == T * k - 2


def test_permute_zero_tokens(moe):
    E = 32
    counts = torch.full((E,), 5, dtype=torch.int32, device=DEV)
    offsets = torch.full((E + 1,), 5, dtype=torch.int32, device=DEV)
    e = torch.empty(0, dtype=torch.int32, device=DEV)
    v = torch.empty((0, 64), dtype=torch.bfloat16, device=DEV)
    moe.moe_permute(v, torch.empty((0, 8), dtype=torch.int32, device=DEV), E, counts, offsets, e, e.view(0, 8),
                    v.view(0, 64))
    assert counts.cpu().tolist() == [0] * E and offsets.cpu().tolist() == [0] * (E + 1)


# --------------------------------------------------------------------------- step 4: expert MLP
def _segments(counts):
    counts = torch.tensor(counts, dtype=torch.int32)
    offsets = torch.zeros(len(counts) + 1, dtype=torch.int32)
    offsets[1:] = torch.cumsum(counts, 0)
    return counts, offsets


# row counts per expert chosen to reach each tile arrangement (average rows per expert decides it):
#   weights-as-M with 16/32/64/128-row blocks, rows-as-M on one CTA, and rows-as-M on CTA pairs
#   (256-row blocks, including a block whose second CTA has one row or none); each has empty experts
#   and ragged tails
# Per-expert row counts.  The name says which GEMM arrangement the average selects: token rows
# staged per tile (16/32/64/128, about 3x the average) on one CTA, or CTA pairs with 256-row
# blocks ("pairs", from 768 rows per expert).
COUNT_CASES = {
    "ra16": [0, 1, 3, 8, 16, 17, 5, 0, 2, 2, 7, 4, 1, 1, 2, 3],            # avg 4.5
    "ra32": [0, 1, 3, 8, 16, 17, 33, 5, 0, 9, 2, 7, 4, 6, 10, 7],         # avg 8
    "ra64": [12, 0, 16, 31, 33, 9, 20, 15, 4, 14, 18, 2, 16, 11, 13, 10],  # avg 14
    "ra128": [0, 64, 65, 20, 1, 40, 30, 37],                              # avg 32
    "ra128b": [129, 0, 60, 45, 33, 90, 7, 100],                           # avg 58
    "rows": [0, 1, 127, 128, 129, 300, 0, 290],                           # avg 122
    "rows256": [0, 1, 128, 129, 256, 257, 384, 511, 512, 640, 0, 300],    # avg 260: remainders 0/1/128/129/255
    "pairs": [0, 255, 256, 257, 2900, 1024, 1, 1513],                     # avg 775
}


def _expert_inputs(name, d, d_ff, dtype=torch.bfloat16, seed=300):
    counts, offsets = _segments(COUNT_CASES[name])
    E, S = len(counts), int(counts.sum())
    xp = synth.normal((S, d), seed, 1, dtype=dtype)
    Wg = synth.normal((E, d_ff, d), seed, 5, 0.0, 1 / math.sqrt(d), dtype)
    Wu = synth.normal((E, d_ff, d), seed, 6, 0.0, 1 / math.sqrt(d), dtype)
    Wd = synth.normal((E, d, d_ff), seed, 7, 0.0, 1 / math.sqrt(d_ff), dtype)
    return counts, offsets, xp, Wg, Wu, Wd


@pytest.mark.parametrize("case", list(COUNT_CASES))
@pytest.mark.parametrize("d,d_ff", [(256, 256), (1024, 384)])
def test_expert_gate_up_bf16(moe, case, d, d_ff):
    counts, offsets, xp, Wg, Wu, _ = _expert_inputs(case, d, d_ff)
    S = xp.shape[0]
    h = torch.full((S, d_ff), float("nan"), dtype=torch.bfloat16, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    moe.moe_expert_gate_up(cuda(xp), cuda(Wg), cuda(Wu), cuda(counts), cuda(offsets), h, dev_status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    h_ref, _ = oracle.grouped_mlp(xp, counts, offsets, Wg, Wu, torch.zeros((Wg.shape[0], d, d_ff)).to(Wg.dtype))
    assert_close_rounded(h, h_ref)


@pytest.mark.parametrize("case", list(COUNT_CASES))
@pytest.mark.parametrize("d,d_ff", [(256, 256), (512, 1024)])
def test_expert_down_bf16(moe, case, d, d_ff):
    counts, offsets, _, _, _, Wd = _expert_inputs(case, d, d_ff)
    S = int(counts.sum())
    h = synth.normal((S, d_ff), 301, 1, dtype=torch.bfloat16)
    y = torch.full((S, d), float("nan"), dtype=torch.bfloat16, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    moe.moe_expert_down(cuda(h), cuda(Wd), cuda(counts), cuda(offsets), y, dev_status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    # y = h W_down^T per segment: the oracle's row map with the gate/up stage replaced by the identity is
    # exactly oracle.linear on each row
    ref = torch.empty((S, d), dtype=torch.float64)
    for e in range(len(counts)):
        for r in range(int(offsets[e]), int(offsets[e + 1])):
            ref[r] = oracle.linear(h[r].double(), Wd[e])
    assert_close_rounded(y, ref)


@pytest.mark.parametrize("case", ["ra16", "ra128", "rows", "rows256", "pairs"])
def test_expert_down_integer_inputs_bit_exact(moe, case):
    # entries in {-1, 0, 1}: every fp32 partial sum is an integer below 2^24 and |y| <= d_ff = 256, so the
    # tensor-core result rounds to bf16 exactly and must equal the oracle bit for bit
    d, d_ff = 256, 256
    counts, offsets = _segments(COUNT_CASES[case])
    E, S = len(counts), int(counts.sum())
    h = synth.randint((S, d_ff), 302, 1, -1, 1).to(torch.bfloat16)
    Wd = synth.randint((E, d, d_ff), 302, 2, -1, 1).to(torch.bfloat16)
    y = torch.empty((S, d), dtype=torch.bfloat16, device=DEV)
    moe.moe_expert_down(cuda(h), cuda(Wd), cuda(counts), cuda(offsets), y)
    ref = torch.empty((S, d), dtype=torch.float64)
    for e in range(E):
        for r in range(int(offsets[e]), int(offsets[e + 1])):
            ref[r] = oracle.linear(h[r].double(), Wd[e])
    assert torch.equal(y.cpu().double(), ref)


@pytest.mark.parametrize("case", list(COUNT_CASES))
def test_expert_gate_up_core_integer_inputs_bit_exact(moe, case):
    # the gate/up GEMMs with the SwiGLU product left out (moe_expert_gate_up_raw), every tile form: weights-as-M
    # with 16/32/64 staged rows (ra16 .. ra128), rows-as-M one-CTA (ra128b, rows, rows256) and CTA pairs (pairs).
    # Entries in {-1, 0, 1}: every fp32 partial sum is an integer and |g|, |u| <= d = 256, so both round to bf16
    # exactly and must equal the oracle's linear map bit for bit
    d, d_ff = 256, 256
    counts, offsets = _segments(COUNT_CASES[case])
    E, S = len(counts), int(counts.sum())
    xp = synth.randint((S, d), 305, 1, -1, 1).to(torch.bfloat16)
    Wg = synth.randint((E, d_ff, d), 305, 2, -1, 1).to(torch.bfloat16)
    Wu = synth.randint((E, d_ff, d), 305, 3, -1, 1).to(torch.bfloat16)
    gu = torch.full((S, 2 * d_ff), float("nan"), dtype=torch.bfloat16, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    moe.moe_expert_gate_up_raw(cuda(xp), cuda(Wg), cuda(Wu), cuda(counts), cuda(offsets), gu, dev_status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    ref = torch.empty((S, 2 * d_ff), dtype=torch.float64)
    for e in range(E):
        for r in range(int(offsets[e]), int(offsets[e + 1])):
            ref[r, :d_ff] = oracle.linear(xp[r].double(), Wg[e])
            ref[r, d_ff:] = oracle.linear(xp[r].double(), Wu[e])
    assert torch.equal(gu.cpu().double(), ref)


@pytest.mark.parametrize("case", ["ra32", "rows"])
def test_expert_mlp_f32(moe, case):
    d, d_ff = 64, 96
    counts, offsets, xp, Wg, Wu, Wd = _expert_inputs(case, d, d_ff, torch.float32, 303)
    S = xp.shape[0]
    h = torch.empty((S, d_ff), device=DEV)
    y = torch.empty((S, d), device=DEV)
    moe.moe_grouped_swiglu(cuda(xp), cuda(Wg), cuda(Wu), cuda(Wd), cuda(counts), cuda(offsets), h, y)
    h_ref, y_ref = oracle.grouped_mlp(xp, counts, offsets, Wg, Wu, Wd)
    assert_close_rounded(h, h_ref, rel=1e-5, rms_frac=1e-5)
    assert_close_rounded(y, y_ref, rel=1e-4, rms_frac=1e-5)


@pytest.mark.parametrize("case", ["ra32", "ra64", "rows", "rows256", "pairs"])
def test_grouped_swiglu_bf16_matches_oracle(moe, case):
    d, d_ff = 256, 256
    counts, offsets, xp, Wg, Wu, Wd = _expert_inputs(case, d, d_ff, seed=304)
    S = xp.shape[0]
    h = torch.empty((S, d_ff), dtype=torch.bfloat16, device=DEV)
    y = torch.empty((S, d), dtype=torch.bfloat16, device=DEV)
    moe.moe_grouped_swiglu(cuda(xp), cuda(Wg), cuda(Wu), cuda(Wd), cuda(counts), cuda(offsets), h, y)
    _, y_ref = oracle.grouped_mlp(xp, counts, offsets, Wg, Wu, Wd)
    max_abs, rel = errors(y, y_ref)
    assert rel < REL_L2 and max_abs < MAX_ABS, (max_abs, rel)


# --------------------------------------------------------------------------- step 5: combine
@pytest.mark.parametrize("ydt,rdt,odt", [("bf16", "bf16", "bf16"), ("bf16", "f32", "f32"), ("f32", "f32", "f32"),
                                         ("f32", "bf16", "bf16")])
@pytest.mark.parametrize("T,E,k,d", [(300, 64, 8, 256), (17, 16, 1, 4096), (5, 8, 8, 64)])
def test_unpermute_combine(moe, ydt, rdt, odt, T, E, k, d):
    idx = synth.distinct_topk(T, E, k, 400 + T)
    _, _, _, token_slot = oracle.permute(idx, E)
    y = synth.normal((T * k, d), 400, 1, dtype=DT[ydt])
    w = synth.uniform((T, k), 400, 2, 0.0, 0.3)
    res = synth.normal((T, d), 400, 3, dtype=DT[rdt])
    out = torch.empty((T, d), dtype=DT[odt], device=DEV)
    moe.moe_unpermute_combine(cuda(y), cuda(token_slot), cuda(w), cuda(res), out)
    ref = oracle.combine(y, token_slot, w, res)
    if odt == "f32":
        assert_close_rounded(out, ref, rel=1e-6, rms_frac=1e-6)
    else:
        assert_close_rounded(out, ref)


# --------------------------------------------------------------------------- whole layer
def _run_forward(moe, w: synth.Workload, I: dict):
    T, E, k = w.T, w.E, w.top_k
    dev = {n: cuda(t) for n, t in I.items()}
    out = torch.empty((T, w.d), dtype=w.out_dtype, device=DEV)
    idx = torch.empty((T, k), dtype=torch.int32, device=DEV)
    wt = torch.empty((T, k), dtype=torch.float32, device=DEV)
    logits = torch.empty((T, E), dtype=torch.float32, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    moe.moe_forward(dev["x"], dev["gamma"], dev["W_r"], dev["b"], dev["W_gate"], dev["W_up"], dev["W_down"], out,
                    top_k=k, eps=w.eps, topk_idx=idx, topk_w=wt, logits=logits, dev_status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    return out, idx, wt, logits


def _assert_rounding_bound(got, ref, x):
    # For shapes outside the top-8 workloads, where the bf16 roundings are not averaged over 8 picks:
    # the output's own rounding (2^-9 |R|), the rounding of y (2^-7 |R - X|), and the roundings of v and h,
    # whose effect on an output element scales with the row's expert-output RMS, not with that element
    # (2^-5 rms_t(R - X): a few half-ulps of bf16 at 4 sigma).
    got, ref, x = got.double(), ref.double(), x.double()
    part = ref - x
    rms = part.pow(2).mean(dim=1, keepdim=True).sqrt()
    bound = 2.0 ** -9 * ref.abs() + 2.0 ** -7 * part.abs() + 2.0 ** -5 * rms + 1e-4
    assert ((got - ref).abs() <= bound).all(), ((got - ref).abs() - bound).max().item()


def _oracle_layer(x, *args, **kw):
    """oracle.moe_layer on the rows of x, in chunks on parallel threads (the C oracle releases the GIL; each
    row is computed independently, so the result is the same as one call)."""
    import os
    from concurrent.futures import ThreadPoolExecutor

    n = x.shape[0]
    workers = max(1, min(32, os.cpu_count() or 1, n // 4))
    if workers == 1:
        return oracle.moe_layer(x, *args, **kw)
    bounds = [n * i // workers for i in range(workers + 1)]

    def part(i):
        lo, hi = bounds[i], bounds[i + 1]
        kk = dict(kw)
        if kk.get("force_idx") is not None:
            kk["force_idx"], kk["force_w"] = kk["force_idx"][lo:hi], kk["force_w"][lo:hi]
        return oracle.moe_layer(x[lo:hi], *args, **kk)

    with ThreadPoolExecutor(max_workers=workers) as ex:
        parts = list(ex.map(part, range(workers)))
    return {k: torch.cat([p[k] for p in parts]) for k in parts[0]}


def _check_layer(moe, w, I, tokens=None, result=None, spec_tolerance=True):
    out, idx, wt, logits = result if result is not None else _run_forward(moe, w, I)
    args = (I["gamma"], I["W_r"], I["b"], I["W_gate"], I["W_up"], I["W_down"])
    # routing: bit-exact on the GPU's logits for every token
    check_routing(oracle, logits, I["b"], idx, wt, w.top_k)
    sel = torch.arange(w.T) if tokens is None else torch.tensor(tokens)
    x = I["x"][sel]
    ref = _oracle_layer(x, *args, k=w.top_k, eps=w.eps)
    z_err = (logits.cpu()[sel].double() - ref["z32"].double()).abs().max().item()
    assert z_err < 1e-4, z_err
    differs = check_routing(oracle, logits.cpu()[sel], I["b"], idx.cpu()[sel], wt.cpu()[sel], w.top_k,
                            ref_idx=ref["idx"], ref_margin=ref["margin"], ref_z32=ref["z32"])
    keep = [i for i in range(len(sel)) if i not in set(differs)]
    got = out.cpu()[sel]
    max_abs, rel = errors(got[keep], ref["out"][keep])
    if spec_tolerance:
        assert max_abs <= MAX_ABS and rel <= REL_L2, (max_abs, rel)
    else:
        assert rel <= REL_L2, rel
        _assert_rounding_bound(got[keep], ref["out"][keep], x[keep])
    # the MoE part alone (R - X), so that the residual cannot hide an error
    moe_abs, moe_rel = errors(got[keep].double() - x[keep].double(), ref["out"][keep] - x[keep].double())
    assert moe_rel <= 2e-2, moe_rel
    # forced routing: the oracle follows the GPU's experts and weights, every token compared
    forced = _oracle_layer(x, *args, k=w.top_k, eps=w.eps, force_idx=idx.cpu()[sel], force_w=wt.cpu()[sel])
    f_abs, f_rel = errors(got, forced["out"])
    if spec_tolerance:
        assert f_abs <= MAX_ABS and f_rel <= REL_L2, (f_abs, f_rel)
    else:
        assert f_rel <= REL_L2, f_rel
        _assert_rounding_bound(got, forced["out"], x)
    return {"max_abs": max_abs, "rel_l2": rel, "moe_rel": moe_rel, "near_tie_set_diffs": len(differs)}


def test_forward_tiny_workload_every_token(moe):
    w = synth.WORKLOADS["tiny"]
    I = synth.make_layer_inputs(w)
    r = _check_layer(moe, w, I)
    assert r["max_abs"] < 1e-4  # all-fp32 path: only fp32 vs fp64 rounding separates them


SMALL = {
    # (T, d, E, d_ff, x, w, out): weights-as-M (few rows per expert) and rows-as-M (many)
    "decode_like": (96, 512, 64, 256, "bf16", "bf16", "bf16"),
    "prefill_like": (1200, 256, 8, 256, "bf16", "bf16", "bf16"),
    "dual_like": (600, 256, 16, 256, "bf16", "bf16", "bf16"),  # ~300 rows per expert: two-row-block gate/up
    "block_like": (160, 256, 32, 384, "f32", "bf16", "f32"),
    "mixed_out": (50, 256, 16, 128, "f32", "bf16", "bf16"),
    "f32_experts": (40, 64, 16, 48, "bf16", "f32", "f32"),
}


@pytest.mark.parametrize("name", list(SMALL))
def test_forward_small(moe, name):
    T, d, E, d_ff, xd, wd, od = SMALL[name]
    w = synth.Workload(name, T, d, E, d_ff, x_dtype=DT[xd], w_dtype=DT[wd], out_dtype=DT[od], seed=500)
    I = synth.make_layer_inputs(w)
    _check_layer(moe, w, I)


def test_forward_top1_and_all_experts(moe):
    for (E, k) in [(8, 8), (16, 1)]:
        w = synth.Workload("edge", 70, 256, E, 128, seed=501 + E, top_k=k)
        _check_layer(moe, w, synth.make_layer_inputs(w), spec_tolerance=(k == 8))


def test_forward_zero_tokens_clears_status(moe):
    w = synth.Workload("empty", 0, 256, 16, 128)
    I = {n: cuda(t) for n, t in synth.make_layer_inputs(w).items()}
    out = torch.empty((0, 256), dtype=torch.bfloat16, device=DEV)
    status = torch.full((1,), 9, dtype=torch.int32, device=DEV)
    moe.moe_forward(I["x"], I["gamma"], I["W_r"], I["b"], I["W_gate"], I["W_up"], I["W_down"], out, dev_status=status)
    torch.cuda.synchronize()
    assert status.item() == 0


def test_forward_workspace_too_small_is_rejected(moe):
    w = synth.Workload("ws", 32, 256, 16, 128)
    I = {n: cuda(t) for n, t in synth.make_layer_inputs(w).items()}
    out = torch.empty((32, 256), dtype=torch.bfloat16, device=DEV)
    need = moe.forward_workspace_bytes(I["x"], I["W_r"], I["W_gate"], out)
    ws = torch.empty(need - 256, dtype=torch.uint8, device=DEV)
    with pytest.raises(moe.MoEError) as ei:
        moe.moe_forward(I["x"], I["gamma"], I["W_r"], I["b"], I["W_gate"], I["W_up"], I["W_down"], out, ws=ws)
    assert ei.value.status == 3


@pytest.mark.parametrize("name", ["decode_like", "block_like", "prefill_like", "dual_like"])
def test_forward_replays_from_a_cuda_graph(moe, name):
    # the whole layer is capturable (no host sync, shape-only grids, caller-owned workspace): a graph
    # captured once replays the eager result bit for bit, and follows new data written into its input
    T, d, E, d_ff, xd, wd, od = SMALL[name]
    w = synth.Workload(name, T, d, E, d_ff, x_dtype=DT[xd], w_dtype=DT[wd], out_dtype=DT[od], seed=510)
    I = {n: cuda(t) for n, t in synth.make_layer_inputs(w).items()}
    x2 = cuda(synth.make_layer_inputs(w.scaled(seed=511))["x"])
    args = (I["gamma"], I["W_r"], I["b"], I["W_gate"], I["W_up"], I["W_down"])
    eager = [torch.empty((T, d), dtype=DT[od], device=DEV) for _ in range(2)]
    ws = torch.empty(moe.forward_workspace_bytes(I["x"], I["W_r"], I["W_gate"], eager[0]), dtype=torch.uint8,
                     device=DEV)
    moe.moe_forward(I["x"], *args, eager[0], ws=ws)
    moe.moe_forward(x2, *args, eager[1], ws=ws)
    torch.cuda.synchronize()
    x_in = I["x"].clone()
    out = torch.empty_like(eager[0])
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        moe.moe_forward(x_in, *args, out, ws=ws)
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(out, eager[0])
    x_in.copy_(x2)
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(out, eager[1])
    del g


def test_forward_launch_count_is_reported_and_stable(moe):
    # the library's own launch counter: one forward enqueues the same nonzero number of kernels each time
    w = synth.Workload("count", 32, 256, 16, 128)
    I = {n: cuda(t) for n, t in synth.make_layer_inputs(w).items()}
    out = torch.empty((32, 256), dtype=torch.bfloat16, device=DEV)
    n = []
    for _ in range(3):
        n0 = moe.kernel_launches()
        moe.moe_forward(I["x"], I["gamma"], I["W_r"], I["b"], I["W_gate"], I["W_up"], I["W_down"], out)
        n.append(moe.kernel_launches() - n0)
    torch.cuda.synchronize()
    assert n[0] > 0 and n[0] == n[1] == n[2]


# --------------------------------------------------------------------------- full-size workloads (sampled)
def _tile_covering_tokens(idx, E):
    """Tokens whose rows include the first row of every 128-row block of every active expert's segment and
    its last row, so that every row block the kernels use (16 to 256 rows, all aligned to the segment start)
    holds a checked row; with the number of 128-row blocks covered out of all of them."""
    counts, offsets, slot_token, _ = oracle.permute(idx.cpu(), E)
    slots = set()
    for e in range(E):
        c, o = int(counts[e]), int(offsets[e])
        if c:
            slots.update(range(o, o + c, 128))
            slots.add(o + c - 1)
    tokens = sorted({int(slot_token[r]) for r in slots})
    # the 128-row blocks of each expert that the chosen tokens' rows reach
    tok = torch.zeros(idx.shape[0], dtype=torch.bool)
    tok[tokens] = True
    covered, total = 0, 0
    for e in range(E):
        c, o = int(counts[e]), int(offsets[e])
        for b in range((c + 127) // 128):
            total += 1
            rows = slot_token[o + 128 * b:o + min(c, 128 * (b + 1))].long()
            covered += int(tok[rows].any())
    return tokens, covered, total


@pytest.mark.parametrize("name", ["decode", "prefill", "skewed", "block"])
def test_forward_full_size_sampled(moe, name):
    w = synth.WORKLOADS[name]
    I = synth.make_layer_inputs(w)
    res = _run_forward(moe, w, I)
    out, idx, wt, logits = res
    # every token: routing bit-exact given the GPU's logits; the permutation's counts follow from it
    check_routing(oracle, logits, I["b"], idx, wt, w.top_k)
    counts = torch.bincount(idx.cpu().flatten().long(), minlength=w.E)
    assert counts.sum().item() == w.T * w.top_k
    assert torch.isfinite(out).all()
    # the layer output for tokens that reach every 128-row block and the last row of every active expert
    # (every token of the decode workload), against the oracle
    tokens, covered, total = _tile_covering_tokens(idx, w.E)
    if w.T <= 256:
        tokens = list(range(w.T))
    print(f"{name}: {len(tokens)} tokens checked; they reach {covered} of {total} 128-row expert blocks of the "
          f"{int((counts > 0).sum())} active experts")
    assert covered == total
    _check_layer(moe, w, I, tokens, result=res)
