"""Comparison rules of the parity tests (test-side helpers; no layer arithmetic).

Layer outputs: max-abs <= 2e-2 and rel-L2 <= 5e-3 against the fp64 oracle.
Routing: given the GPU's own fp32 logits the oracle's choice must be
bit-identical; where the oracle's own routing (from its fp64 logits) differs,
the token must be a near-tie (margin < 1e-5) and is reported.
"""
from __future__ import annotations

import torch

MAX_ABS = 2e-2
REL_L2 = 5e-3
NEAR_TIE = 1e-5
W_TOL = 1e-6


def errors(got: torch.Tensor, ref: torch.Tensor) -> tuple[float, float]:
    got = got.double().cpu()
    ref = ref.double().cpu()
    d = got - ref
    max_abs = d.abs().max().item() if d.numel() else 0.0
    den = ref.norm().item()
    rel = d.norm().item() / den if den > 0 else d.norm().item()
    return max_abs, rel


def check_routing(oracle_mod, logits, b, idx, w, k, ref_idx=None, ref_margin=None, ref_z32=None):
    """Check the GPU's routing; return the tokens whose oracle expert SET differs (near-ties).

    Given the GPU's fp32 logits the oracle must pick bit-identical experts in
    the same order.  Against the oracle's own routing (fp64 logits) a token may
    differ only where scores are within NEAR_TIE: a different set needs the
    8th-9th margin below it, a different order needs the swapped scores within it.
    """
    sel_idx, sel_w, sel_margin = oracle_mod.select_topk(logits.cpu(), b.cpu(), k)
    assert torch.equal(sel_idx, idx.cpu()), "top-k differs from the oracle on identical fp32 logits"
    assert (sel_w - w.cpu().double()).abs().max().item() <= W_TOL
    set_differs = []
    if ref_idx is not None:
        gi, ri = idx.cpu(), ref_idx.cpu()
        for t in (ri != gi).any(dim=1).nonzero().flatten().tolist():
            if sorted(ri[t].tolist()) != sorted(gi[t].tolist()):
                assert ref_margin[t].item() < NEAR_TIE or sel_margin[t].item() < NEAR_TIE, \
                    f"token {t} routes to other experts with margin {ref_margin[t].item()}"
                set_differs.append(t)
            else:
                sc = {e: oracle_mod.selection_score(float(ref_z32[t, e]), float(b[e])) for e in ri[t].tolist()}
                for a, c in zip(ri[t].tolist(), gi[t].tolist()):
                    assert abs(sc[a] - sc[c]) < NEAR_TIE, f"token {t}: pick order differs beyond a near-tie"
    return set_differs


def oracle_fp8_weights(oracle_mod, W: torch.Tensor, device):
    """Block-FP8 codes and scales of an expert weight tensor [E][n][k], quantised by the CPU oracle (so no
    GPU value feeds the reference) and uploaded to `device` for the layer under test.  The experts are
    quantised in parallel threads (the oracle's C calls release the GIL)."""
    from concurrent.futures import ThreadPoolExecutor

    E, n, k = W.shape
    W = W.detach().cpu().contiguous()
    with ThreadPoolExecutor(max_workers=16) as ex:
        parts = list(ex.map(lambda e: oracle_mod.quantize_blocks(W[e], 128), range(E)))
    q = torch.stack([p[0] for p in parts])
    s = torch.stack([p[1] for p in parts])
    return q.to(device), s.to(device)
