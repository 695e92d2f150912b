"""Pins of the block-FP8 oracle against facts that do not come from it: an
independent library decoder (torch.float8_e4m3fn), the E4M3 format's own
definition (exhaustive round trips, ties, saturation), quantisation bounds,
and a brute-force GEMM on tiny inputs built from library-decoded values."""
import math

import pytest
import torch

import oracle
import synth

F8 = torch.float8_e4m3fn


def lib_decode(codes):
    return codes.view(F8).to(torch.float64)


def test_decode_matches_library_for_all_codes():
    c = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ours, ref = oracle.e4m3_decode(c), lib_decode(c)
    nan = ref.isnan()
    assert torch.equal(nan, ours.isnan())
    assert torch.equal(ours[~nan], ref[~nan])
    assert nan.sum() == 2  # S.1111.111 only
    assert ours[0x7E] == 448.0 and ours[0x01] == 2.0 ** -9 and ours[0x08] == 2.0 ** -6


def test_every_finite_code_round_trips_and_signed_zero_keeps_its_sign():
    c = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    v = oracle.e4m3_decode(c)
    fin = ~v.isnan()
    assert torch.equal(oracle.e4m3_encode(v[fin].float()), c[fin])
    assert oracle.e4m3_encode(torch.tensor([0.0, -0.0])).tolist() == [0x00, 0x80]


def test_encode_matches_library_rounding_in_range():
    x = synth.normal((40000,), 11, 1, 0.0, 60.0).clamp(-448, 448)
    x = torch.cat([x, synth.normal((4000,), 11, 2, 0.0, 0.01)])  # subnormals and small normals
    assert torch.equal(oracle.e4m3_encode(x), x.to(F8).view(torch.uint8))


def test_midpoints_round_to_the_even_mantissa():
    pos = torch.arange(0, 0x7E, dtype=torch.int32)  # adjacent finite positive codes c, c + 1
    lo = oracle.e4m3_decode(pos.to(torch.uint8))
    hi = oracle.e4m3_decode((pos + 1).to(torch.uint8))
    mid = ((lo + hi) / 2).float()  # exactly representable in fp32
    assert torch.equal(mid.double(), (lo + hi) / 2)
    got = oracle.e4m3_encode(mid).to(torch.int32)
    even = torch.where(pos % 2 == 0, pos, pos + 1)
    assert torch.equal(got, even)


def test_finite_overflow_saturates_and_nan_stays_nan():
    x = torch.tensor([448.0, 463.9, 464.0, 464.1, 479.9, 480.0, 1e6, 3.0e38, -500.0, float("nan")])
    assert oracle.e4m3_encode(x).tolist() == [0x7E, 0x7E, 0x7E, 0x7E, 0x7E, 0x7E, 0x7E, 0x7E, 0xFE, 0x7F]


@pytest.mark.parametrize("blk_rows", [1, 128])
def test_block_quantisation_bounds(blk_rows):
    rows, cols = 256, 384
    x = synth.normal((rows, cols), 12, blk_rows, dtype=torch.bfloat16)
    x[5, 130] = 20.0  # one outlier: its block's scale follows it
    x[128:, 256:] = 0  # zero blocks get scale 1 and zero codes
    q, s = oracle.quantize_blocks(x, blk_rows)
    xf = x.double()
    deq = lib_decode(q) * s.double().repeat_interleave(blk_rows, 0)[:rows].repeat_interleave(128, 1)
    assert not deq.isnan().any()
    blocks = xf.abs().reshape(rows // blk_rows, blk_rows, cols // 128, 128).amax(dim=(1, 3))
    # each block's largest element gets the largest code, +-448
    for br in range(rows // blk_rows):
        for bc in range(cols // 128):
            blk = xf[br * blk_rows:(br + 1) * blk_rows, bc * 128:(bc + 1) * 128]
            qb = q[br * blk_rows:(br + 1) * blk_rows, bc * 128:(bc + 1) * 128]
            if blocks[br, bc] == 0:
                assert s[br, bc] == 1.0 and (qb == 0).all()
            else:
                i = blk.abs().argmax()
                assert int(qb.flatten()[i]) & 0x7F == 0x7E
    # half a code step at most: 2^-4 relative for normal codes, 2^-10 * s below them
    sc = s.double().repeat_interleave(blk_rows, 0)[:rows].repeat_interleave(128, 1)
    assert ((deq - xf).abs() <= xf.abs() * 2.0 ** -4 + sc * 2.0 ** -10).all()


def test_fp8_grouped_mlp_equals_brute_force_on_library_decoded_operands():
    E, d, d_ff = 3, 256, 256
    counts = torch.tensor([2, 0, 3], dtype=torch.int32)
    offsets = torch.tensor([0, 2, 2, 5], dtype=torch.int32)
    S = 5
    x = synth.normal((S, d), 13, 1, dtype=torch.bfloat16)
    Wg = synth.normal((E, d_ff, d), 13, 2, 0.0, 1 / 16, torch.bfloat16)
    Wu = synth.normal((E, d_ff, d), 13, 3, 0.0, 1 / 16, torch.bfloat16)
    Wd = synth.normal((E, d, d_ff), 13, 4, 0.0, 1 / 16, torch.bfloat16)
    xq, xs = oracle.quantize_blocks(x, 1)
    qs = [oracle.quantize_blocks(W.reshape(-1, W.shape[2]), 128) for W in (Wg, Wu, Wd)]
    (gq, gs), (uq, us), (dq, ds) = qs
    r = oracle.fp8_grouped_mlp(xq, xs, counts, offsets, gq.reshape(E, d_ff, d), gs.reshape(E, -1, d // 128),
                               uq.reshape(E, d_ff, d), us.reshape(E, -1, d // 128), dq.reshape(E, d, d_ff),
                               ds.reshape(E, -1, d_ff // 128))

    def deq2(q, s, blk):
        return lib_decode(q) * s.double().repeat_interleave(blk, 0)[:q.shape[0]].repeat_interleave(128, 1)

    a = deq2(xq, xs, 1)
    G, U, D = deq2(gq, gs, 128), deq2(uq, us, 128), deq2(dq, ds, 128)
    for e in range(E):
        for row in range(int(offsets[e]), int(offsets[e] + counts[e])):
            g = G[e * d_ff:(e + 1) * d_ff] @ a[row]
            u = U[e * d_ff:(e + 1) * d_ff] @ a[row]
            h = g * torch.sigmoid(g) * u
            assert torch.allclose(r["h"][row], h, rtol=1e-12, atol=1e-12)
            hq, hs = oracle.quantize_blocks(r["h"][row:row + 1].float(), 1)
            assert torch.equal(r["hq"][row], hq[0]) and torch.equal(r["hs"][row], hs[0])
            y = D[e * d:(e + 1) * d] @ deq2(hq, hs, 1)[0]
            assert torch.allclose(r["y"][row], y, rtol=1e-12, atol=1e-12)
    # with no rows in any segment nothing is computed (NaN everywhere); given codes replace the oracle's own
    empty = oracle.fp8_grouped_mlp(xq, xs, torch.zeros(E, dtype=torch.int32), offsets, gq.reshape(E, d_ff, d),
                                   gs.reshape(E, -1, d // 128), uq.reshape(E, d_ff, d), us.reshape(E, -1, d // 128),
                                   dq.reshape(E, d, d_ff), ds.reshape(E, -1, d_ff // 128))
    assert torch.isnan(empty["y"]).all()
    zq, zs = torch.zeros_like(r["hq"]), torch.ones_like(r["hs"])
    r0 = oracle.fp8_grouped_mlp(xq, xs, counts, offsets, gq.reshape(E, d_ff, d), gs.reshape(E, -1, d // 128),
                                uq.reshape(E, d_ff, d), us.reshape(E, -1, d // 128), dq.reshape(E, d, d_ff),
                                ds.reshape(E, -1, d_ff // 128), hq_in=zq, hs_in=zs)
    valid = torch.tensor([0, 1, 2, 3, 4])
    assert (r0["y"][valid] == 0).all()
