"""GPU parity of the masked decode layout: per-expert buffers [E][cap][.] with a
valid-row count per expert, through moe_grouped_swiglu_masked, against the
fp64 oracle's grouped MLP on the same rows (segments at offsets e * cap)."""
import math

import pytest
import torch

import oracle
import synth
from _layer_check import MAX_ABS, REL_L2, errors

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
SENTINEL = 0x7FA5  # a bf16 NaN pattern no kernel produces: rows that must stay unwritten keep it


@pytest.fixture(scope="module")
def moe():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import moe_layer_forward_b200 as m

    return m


def _inputs(E, cap, d, d_ff, counts, seed):
    x = synth.normal((E, cap, d), seed, 1, dtype=torch.bfloat16)
    for e, n in enumerate(counts):  # rows past the count hold NaN: none may reach a stored result
        x[e, max(n, 0):] = float("nan")
    Wg = synth.normal((E, d_ff, d), seed, 5, 0.0, 1 / math.sqrt(d), torch.bfloat16)
    Wu = synth.normal((E, d_ff, d), seed, 6, 0.0, 1 / math.sqrt(d), torch.bfloat16)
    Wd = synth.normal((E, d, d_ff), seed, 7, 0.0, 1 / math.sqrt(d_ff), torch.bfloat16)
    return x, Wg, Wu, Wd


def _sentinel(shape):
    return torch.full(shape, SENTINEL, dtype=torch.int16, device=DEV).view(torch.bfloat16)


def _run(moe, x, Wg, Wu, Wd, counts):
    E, cap, d = x.shape
    d_ff = Wg.shape[1]
    h, y = _sentinel((E, cap, d_ff)), _sentinel((E, cap, d))
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    moe.moe_grouped_swiglu_masked(x.to(DEV), Wg.to(DEV), Wu.to(DEV), Wd.to(DEV),
                                  torch.tensor(counts, dtype=torch.int32, device=DEV), h, y, dev_status=status)
    torch.cuda.synchronize()
    return h.cpu(), y.cpu(), status.item()


# caps that select each tile arrangement: weights-as-M gate/up with 16/32/64 token columns and
# rows-as-M down with 32/64/128 staged rows; then rows-as-M for both with several row blocks
@pytest.mark.parametrize("cap,counts", [
    (8, [0, 1, 8, 3, 7, 5, 2, 8]),
    (16, [16, 0, 9, 15, 1, 16, 4, 11]),
    (24, [24, 1, 0, 13, 23, 7, 19, 2]),
    (160, [0, 1, 127, 128, 129, 160, 40, 97]),
])
def test_masked_swiglu_matches_oracle_and_leaves_padding_rows_unwritten(moe, cap, counts):
    E, d, d_ff = len(counts), 256, 384
    x, Wg, Wu, Wd = _inputs(E, cap, d, d_ff, counts, seed=700 + cap)
    h, y, status = _run(moe, x, Wg, Wu, Wd, counts)
    assert status == 0
    ct = torch.tensor(counts, dtype=torch.int32)
    offs = torch.arange(E + 1, dtype=torch.int32) * cap
    h_ref, y_ref = oracle.grouped_mlp(x.reshape(E * cap, d), ct, offs, Wg, Wu, Wd)
    valid = torch.zeros(E * cap, dtype=torch.bool)
    for e, n in enumerate(counts):
        valid[e * cap:e * cap + n] = True
    hf, yf = h.reshape(E * cap, d_ff), y.reshape(E * cap, d)
    # valid rows: h within bf16 rounding of the fp64 oracle, y within the layer tolerance
    hv, hr = hf[valid].double(), h_ref[valid]
    rms = hr.pow(2).mean().sqrt().item()
    assert ((hv - hr).abs() <= 2.0 ** -8 * hr.abs() + 1e-4 * rms).all()
    max_abs, rel = errors(yf[valid], y_ref[valid])
    assert rel < REL_L2 and max_abs < MAX_ABS, (max_abs, rel)
    # padding rows: untouched bit for bit
    assert (hf[~valid].view(torch.int16) == SENTINEL).all()
    assert (yf[~valid].view(torch.int16) == SENTINEL).all()


def test_masked_count_above_capacity_is_clamped_and_flagged(moe):
    E, cap, d, d_ff = 4, 16, 256, 256
    counts = [3, 20, -2, 16]
    clamped = [3, 16, 0, 16]
    x, Wg, Wu, Wd = _inputs(E, cap, d, d_ff, clamped, seed=720)
    h, y, status = _run(moe, x, Wg, Wu, Wd, counts)
    assert status & 4  # MOE_DEV_BAD_COUNT
    offs = torch.arange(E + 1, dtype=torch.int32) * cap
    _, y_ref = oracle.grouped_mlp(x.reshape(E * cap, d), torch.tensor(clamped, dtype=torch.int32), offs, Wg, Wu, Wd)
    yf = y.reshape(E * cap, d)
    for e, n in enumerate(clamped):
        rows = slice(e * cap, e * cap + n)
        if n:
            max_abs, rel = errors(yf[rows], y_ref[rows])
            assert rel < REL_L2 and max_abs < MAX_ABS
        assert (yf[e * cap + n:(e + 1) * cap].view(torch.int16) == SENTINEL).all()


def test_masked_matches_the_contiguous_entry_point_bit_for_bit(moe):
    # same rows, same kernels: the masked call and the contiguous call on the packed rows agree exactly
    E, cap, d, d_ff = 8, 24, 256, 256
    counts = [24, 1, 0, 13, 23, 7, 19, 2]
    x, Wg, Wu, Wd = _inputs(E, cap, d, d_ff, counts, seed=730)
    h, y, _ = _run(moe, x, Wg, Wu, Wd, counts)
    packed = torch.cat([x[e, :n] for e, n in enumerate(counts)])
    S = packed.shape[0]
    ct = torch.tensor(counts, dtype=torch.int32)
    offs = torch.zeros(E + 1, dtype=torch.int32)
    offs[1:] = torch.cumsum(ct, 0)
    hp = torch.empty((S, d_ff), dtype=torch.bfloat16, device=DEV)
    yp = torch.empty((S, d), dtype=torch.bfloat16, device=DEV)
    moe.moe_grouped_swiglu(packed.to(DEV), Wg.to(DEV), Wu.to(DEV), Wd.to(DEV), ct.to(DEV), offs.to(DEV), hp, yp)
    torch.cuda.synchronize()
    # every tile accumulates over K in the same order (64-wide stages of four K = 16 steps) and its MMA
    # shape follows from its own row count, so both layouts give identical bits
    h_masked = torch.cat([h[e, :n] for e, n in enumerate(counts)])
    y_masked = torch.cat([y[e, :n] for e, n in enumerate(counts)])
    assert torch.equal(h_masked.view(torch.int16), hp.cpu().view(torch.int16))
    assert torch.equal(y_masked.view(torch.int16), yp.cpu().view(torch.int16))
