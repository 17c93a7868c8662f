"""Algorithmic byte counts of the decode path (the roofline numerators).

Algorithmic bytes are what one call must move at minimum: the resident codes,
the fp16 step/offset pairs, the refinement bits of the selected channels or
tokens, and the activations in and results out.  Workspaces (stored logits,
selection candidates, split partials) are overhead and are not counted.

The bits-per-weight model reproduces the worked example of "StrataFlux --
Selective precision streaming -- What does it mean?": with k of every C input
channels refined by r extra bits over a b-bit resident base, each weight costs
b + r*k/C bits per step.
"""
from __future__ import annotations


def fetched_share(k: int, chunk: int) -> float:
    """Fraction of input channels refined per step (k per chunk)."""
    return k / chunk


def extra_bits_per_weight(r: int, k: int, chunk: int) -> float:
    return r * fetched_share(k, chunk)


def bits_touched_per_weight(b: int, r: int, k: int, chunk: int) -> float:
    """Resident bits plus fetched refinement bits per weight (scales excluded)."""
    return b + extra_bits_per_weight(r, k, chunk)


def gemv_bytes(n: int, k: int, b: int, r: int, group: int, kch: int, chunk: int,
               batch: int = 1) -> int:
    """One refined GEMV: base codes + step/offset + selected refinement rows
    (one row of n*r/8 bytes per selected channel and batch row) + x (fp16) +
    the selected indices (int32) + y (fp32)."""
    codes = n * k * b // 8
    sz = n * (k // group) * 4
    n_sel = (k // chunk) * kch
    refine = batch * n_sel * n * r // 8
    io = batch * (k * 2 + n_sel * 4 + n * 4)
    return codes + sz + refine + io


def kv_attention_bytes(t: int, h_kv: int, h_q: int, d: int, b: int, r: int, group: int,
                       k_tok: int, batch: int = 1) -> int:
    """Score + select + refined attention over t cached tokens: K and V base codes
    and step/offset once, the selected tokens' K and V refinements, q in (fp16)
    and out (fp32)."""
    per_token = 2 * (d * b // 8 + (d // group) * 4)
    refine = 2 * k_tok * d * r // 8
    io = h_q * d * (2 + 4)
    return batch * (h_kv * (t * per_token + refine) + io)
