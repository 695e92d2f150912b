"""Device-side guards against inconsistent maps, on the GPU, through the C ABI.

Each kernel that follows a row map or a segment table must stay inside the
buffers it is given when the map disagrees with them, skip the bad part and
report it in the status word:
  - the combine skips picks whose slot is negative (the permutation's mark
    for a bad expert id): their row is not read and their weight not used;
  - the expert GEMMs cut a segment that runs past the S rows of their buffers
    (or starts before them) to the part inside and set MOE_DEV_BAD_COUNT; the
    rows inside come out exactly as from a call with the cut segment;
  - the expert-parallel dispatch and combine never store or load a row past
    the receive buffer's recv_rows, and flag the picks they leave out.
Every access stays inside allocated memory in these tests, even one that a
missing guard would make: each buffer sits in the middle of a larger
allocation whose margins (64 rows before and after, more than any planted
overrun) hold canary values that must be left untouched.
"""
import math

import pytest
import torch

import synth

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
CANARY = 7.0


@pytest.fixture(scope="module")
def moe():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import moe_layer_forward_b200 as m

    return m


PAD = 64  # rows of margin on each side of a buffer: more than any overrun planted below


def _padded(rows, cols, dtype, fill=CANARY):
    """(view of `rows` rows in the middle of a larger allocation, the whole allocation), all set to `fill`."""
    big = torch.full((PAD + rows + PAD, cols), fill, dtype=dtype, device=DEV)
    return big[PAD:PAD + rows], big


def _margins(big, fill=CANARY):
    return torch.cat([big[:PAD], big[-PAD:]]).eq(fill).all().item()


def _padded_copy(t):
    view, big = _padded(t.shape[0], t.shape[1], t.dtype, fill=0)
    view.copy_(t)
    return view


# --------------------------------------------------------------------------- combine
@pytest.mark.parametrize("ydt,odt", [(torch.bfloat16, torch.bfloat16), (torch.float32, torch.float32)])
def test_combine_skips_picks_with_a_negative_slot(moe, ydt, odt):
    # small integers and power-of-two weights: every sum is exact, so the result is compared bit for bit
    T, k, d = 64, 8, 256
    S = T * k
    big = torch.full((S + 1, d), 1000.0, dtype=ydt, device=DEV)  # row 0 would be read for slot -1
    y = big[1:]
    y.copy_(synth.randint((S, d), 800, 1, -8, 8).to(ydt).to(DEV))
    token_slot = torch.randperm(S, generator=torch.Generator().manual_seed(0)).to(torch.int32).view(T, k)
    drop = synth.randint((T, k), 800, 2, 0, 3) == 0
    drop[0] = True  # one token with no valid pick at all
    token_slot[drop] = -1
    w = torch.tensor([0.5, 0.25, 0.125, 0.0625, 1.0, 2.0, 0.5, 0.25]).repeat(T, 1)
    res = synth.randint((T, d), 800, 3, -4, 4).to(odt)
    out = torch.empty((T, d), dtype=odt, device=DEV)
    moe.moe_unpermute_combine(y, token_slot.to(DEV), w.to(DEV), res.to(DEV), out)
    torch.cuda.synchronize()
    yc = y.cpu().double()
    ref = res.double().clone()
    for t in range(T):
        for i in range(k):
            s = int(token_slot[t, i])
            if s >= 0:
                ref[t] += float(w[t, i]) * yc[s]
    # the fp32 sum is exact; the only rounding is the store to the output dtype
    assert torch.equal(out.cpu(), ref.to(odt))
    assert torch.equal(out[0].cpu(), res[0])


# --------------------------------------------------------------------------- expert GEMMs
# (E, rows per expert, d, d_ff, dtype): each picks one kernel form through the average rows per expert
GEMM_CASES = {
    "weights_as_m": (16, 4, 256, 256, torch.bfloat16),
    "rows_as_m": (4, 100, 256, 256, torch.bfloat16),
    "cta_pairs": (2, 800, 256, 256, torch.bfloat16),
    "fp32": (4, 16, 64, 96, torch.float32),
}


def _gemm_inputs(E, per, d, d_ff, dtype, seed):
    S = E * per
    xp = _padded_copy(synth.normal((S, d), seed, 1, dtype=dtype).to(DEV))
    Wg = synth.normal((E, d_ff, d), seed, 2, 0.0, 1 / math.sqrt(d), dtype).to(DEV)
    Wu = synth.normal((E, d_ff, d), seed, 3, 0.0, 1 / math.sqrt(d), dtype).to(DEV)
    Wd = synth.normal((E, d, d_ff), seed, 4, 0.0, 1 / math.sqrt(d_ff), dtype).to(DEV)
    return S, xp, Wg, Wu, Wd


def _bad_segments(E, per, S):
    """Counts and offsets whose last segment runs 40 rows past S and whose first starts at -3, plus the
    same segments cut to [0, S)."""
    counts = torch.full((E,), per, dtype=torch.int32)
    offsets = torch.arange(E + 1, dtype=torch.int32) * per
    counts[-1] = per + 40
    offsets[0], counts[0] = -3, per + 3
    cut_c, cut_o = counts.clone(), offsets.clone()
    cut_c[-1] = S - int(offsets[E - 1])
    cut_o[0], cut_c[0] = 0, per
    return counts, offsets, cut_c, cut_o


@pytest.mark.parametrize("case", list(GEMM_CASES))
def test_expert_mlp_cuts_segments_to_its_buffers(moe, case):
    E, per, d, d_ff, dt = GEMM_CASES[case]
    S, xp, Wg, Wu, Wd = _gemm_inputs(E, per, d, d_ff, dt, 810)
    counts, offsets, cut_c, cut_o = _bad_segments(E, per, S)
    outs = []
    for c, o in [(cut_c, cut_o), (counts, offsets)]:
        h, hbig = _padded(S, d_ff, dt)
        y, ybig = _padded(S, d, dt)
        status = torch.zeros(1, dtype=torch.int32, device=DEV)
        moe.moe_grouped_swiglu(xp, Wg, Wu, Wd, c.to(DEV), o.to(DEV), h, y, dev_status=status)
        torch.cuda.synchronize()
        outs.append((hbig.cpu(), ybig.cpu(), status.item()))
    (h0, y0, s0), (h1, y1, s1) = outs
    assert s0 == 0 and s1 == moe.MOE_DEV_BAD_COUNT
    assert torch.equal(h1, h0) and torch.equal(y1, y0)  # the rows inside, and the untouched margins
    assert _margins(h1) and _margins(y1)


def test_fp8_expert_mlp_cuts_segments_to_its_buffers(moe):
    E, per, d, d_ff = 16, 4, 256, 256
    S, xp, Wg, Wu, Wd = _gemm_inputs(E, per, d, d_ff, torch.bfloat16, 811)
    xq = _padded(S, d, torch.uint8, fill=0)[0]
    xs = _padded(S, d // 128, torch.float32, fill=0)[0]
    moe.quantize_fp8(xp, 1, xq, xs)
    Wq = [moe.quantize_fp8_weights(W) for W in (Wg, Wu, Wd)]
    counts, offsets, cut_c, cut_o = _bad_segments(E, per, S)
    outs = []
    for c, o in [(cut_c, cut_o), (counts, offsets)]:
        hq, hqbig = _padded(S, d_ff, torch.uint8, fill=0x11)
        hs, hsbig = _padded(S, d_ff // 128, torch.float32)
        y, ybig = _padded(S, d, torch.bfloat16)
        status = torch.zeros(1, dtype=torch.int32, device=DEV)
        moe.moe_grouped_swiglu_fp8(xq, xs, *Wq, c.to(DEV), o.to(DEV), hq, hs, y, dev_status=status)
        torch.cuda.synchronize()
        outs.append((hqbig.cpu(), hsbig.cpu(), ybig.cpu(), status.item()))
    assert outs[0][3] == 0 and outs[1][3] == moe.MOE_DEV_BAD_COUNT
    for a, b in zip(outs[0][:3], outs[1][:3]):
        assert torch.equal(a, b)
    assert _margins(outs[1][0], 0x11) and _margins(outs[1][1]) and _margins(outs[1][2])


# --------------------------------------------------------------------------- expert parallelism
def test_ep_dispatch_and_combine_stay_inside_a_short_receive_buffer(moe):
    from moe_layer_forward_b200 import ep_p2p
    from test_gpu_ep_p2p import _layout_start

    N, T, d, E, d_ff = 2, 64, 256, 16, 128
    E_loc = E // N
    w = synth.Workload("ep_short", T, d, E, d_ff, seed=820)
    D = {n: t.to(DEV) for n, t in synth.make_layer_inputs(w).items()}
    ops = ep_p2p.CudaP2POps()
    shards = list(D["x"].chunk(N))
    routes = [ep_p2p._route(ops, x, D["gamma"], D["W_r"], D["b"], E, w.top_k, w.eps, torch.bfloat16)
              for x in shards]
    table = torch.stack([rt.counts for rt in routes])
    tab = table.cpu()
    need = int(tab.sum(0).view(N, E_loc).sum(1).max())  # rows the fullest owner receives
    rows = need - 37  # that owner's buffer is 37 rows short (less than the margin PAD)
    starts = [_layout_start(tab, j, E_loc)[0] for j in range(N)]

    def placement(r, rt):
        """(t, i) -> (owner, row) of every pick of rank r, by the layout rule"""
        idx, ts, off = rt.idx.cpu(), rt.token_slot.cpu(), rt.offsets.cpu()
        return {(t, i): (int(idx[t, i]) // E_loc,
                         starts[int(idx[t, i]) // E_loc][(r, int(idx[t, i]))] + int(ts[t, i]) - int(off[idx[t, i]]))
                for t in range(idx.shape[0]) for i in range(w.top_k)}

    places = [placement(r, rt) for r, rt in enumerate(routes)]
    recv = [_padded(rows, d, torch.bfloat16) for _ in range(N)]
    ys = [_padded(rows, d, torch.bfloat16) for _ in range(N)]
    for j in range(N):
        ys[j][0].copy_(synth.normal((rows, d), 821 + j, 1, dtype=torch.bfloat16).to(DEV))
    rp = torch.tensor([r[0].data_ptr() for r in recv], dtype=torch.int64, device=DEV)
    yp = torch.tensor([y[0].data_ptr() for y in ys], dtype=torch.int64, device=DEV)
    for r, rt in enumerate(routes):
        status = torch.zeros(1, dtype=torch.int32, device=DEV)
        moe.moe_ep_dispatch(rt.vx, rt.idx, rt.token_slot, rt.offsets, table, r, rp, rows, dev_status=status)
        torch.cuda.synchronize()
        lost = sum(1 for (_, row) in places[r].values() if row >= rows)
        assert status.item() == (moe.MOE_DEV_BAD_COUNT if lost else 0)
    assert any(row >= rows for pl in places for (_, row) in pl.values())
    for j in range(N):  # rows inside the buffers are where the layout puts them; the canary tail is intact
        assert _margins(recv[j][1])
        for r, rt in enumerate(routes):
            vx = rt.vx.cpu()
            for (t, i), (owner, row) in places[r].items():
                if owner == j and row < rows:
                    assert torch.equal(recv[j][0][row].cpu(), vx[t])
    # the combine sums exactly the picks whose row lies inside the owner's buffer
    for r, rt in enumerate(routes):
        status = torch.zeros(1, dtype=torch.int32, device=DEV)
        out = torch.empty_like(shards[r])
        moe.moe_ep_combine(yp, torch.bfloat16, rt.idx, rt.token_slot, rt.offsets, table, r, rt.w, shards[r], out,
                           rows, dev_status=status)
        ts = rt.token_slot.cpu()
        gathered = torch.zeros((ts.numel(), d), dtype=torch.bfloat16, device=DEV)
        slot = ts.clone()
        for (t, i), (owner, row) in places[r].items():
            if row < rows:
                gathered[int(ts[t, i])] = ys[owner][0][row]
            else:
                slot[t, i] = -1
        ref = torch.empty_like(out)
        moe.moe_unpermute_combine(gathered, slot.to(DEV), rt.w, shards[r], ref)
        torch.cuda.synchronize()
        assert torch.equal(out, ref)
        lost = int((slot < 0).sum())
        assert status.item() == (moe.MOE_DEV_BAD_COUNT if lost else 0)
