"""Seeded synthetic inputs shaped like the StrataFlux evaluation workloads.

This module holds random-number generation only: no quantisation, selection or
attention arithmetic.  It is the one module that both the CUDA path's tests and
benchmark and the CPU oracle's tests draw their inputs from.

The pages evaluate on real Llama-3.1-8B / Qwen3-8B checkpoints and text datasets
(abstract of "StrataFlux: Memory-Hierarchy-Native Low-Bit LLM Inference"); none
of those is used.  These generators stand in for them with the same shapes:
Llama-3.1-8B projections (hidden 4096, intermediate 14336, 32 query / 8 KV heads,
head_dim 128) and 8K-128K token contexts.  Weights are N(0, 0.02); activations
are N(0, 1) with 1 % of channels scaled by 20 (outlier channels); keys and values
are N(0, 1) with 4 key channels per KV head scaled by 10.  Every array is drawn
from numpy's PCG64 in a fixed order and converted to fp16 with numpy's
round-to-nearest-even cast.
"""
from __future__ import annotations

import numpy as np

HIDDEN = 4096
INTER = 14336
N_HEADS = 32
N_KV_HEADS = 8
HEAD_DIM = 128
VOCAB = 128256

# (name, out features, in features, activation group) of one decoder layer.
LAYER_PROJECTIONS = (
    ("q", HIDDEN, HIDDEN, "attn"),
    ("k", N_KV_HEADS * HEAD_DIM, HIDDEN, "attn"),
    ("v", N_KV_HEADS * HEAD_DIM, HIDDEN, "attn"),
    ("o", HIDDEN, HIDDEN, "o"),
    ("gate", INTER, HIDDEN, "mlp"),
    ("up", INTER, HIDDEN, "mlp"),
    ("down", HIDDEN, INTER, "down"),
)


def weight(rng: np.random.Generator, n: int, k: int, std: float = 0.02) -> np.ndarray:
    """W[n][k] fp32 ~ N(0, std)."""
    return rng.normal(0.0, std, size=(n, k)).astype(np.float32)


def activation(rng: np.random.Generator, k: int, batch: int = 1, outlier_frac: float = 0.01,
               outlier_scale: float = 20.0) -> np.ndarray:
    """x[batch][k] fp16: N(0, 1) with round(outlier_frac * k) channels per row scaled."""
    out = np.empty((batch, k), np.float16)
    n_out = int(round(outlier_frac * k))
    for b in range(batch):
        x = rng.normal(0.0, 1.0, size=k)
        idx = rng.choice(k, n_out, replace=False)
        x[idx] *= outlier_scale
        out[b] = x.astype(np.float16)
    return out


def calibration_activations(n: int, k: int, seed: int, structure_seed: int = 1000, rank: int = 16,
                            noise: float = 0.5, outlier_frac: float = 0.01,
                            outlier_scale: float = 20.0) -> np.ndarray:
    """x[n][k] fp16 rows for fitting and checking refinement values: a rank-`rank`
    factor part F L^T (F[n][rank] ~ N(0, 1), L[k][rank] ~ N(0, 1/rank), so each
    channel's factor part has unit variance) plus N(0, noise) per element, with
    the same round(outlier_frac * k) channels scaled by outlier_scale in every
    row.  L and the outlier channels come from structure_seed, the rows from
    seed: a calibration set and a held-out set share the structure and differ
    in their rows."""
    gs = np.random.default_rng(structure_seed)
    L = gs.normal(0.0, 1.0, size=(k, rank)) / np.sqrt(rank)
    out_ch = gs.choice(k, int(round(outlier_frac * k)), replace=False)
    g = np.random.default_rng(seed)
    x = g.normal(0.0, 1.0, size=(n, rank)) @ L.T + noise * g.normal(0.0, 1.0, size=(n, k))
    x[:, out_ch] *= outlier_scale
    return x.astype(np.float16)


def kv_values(rng: np.random.Generator, h_kv: int, t: int, d: int, batch: int = 1,
              n_key_outliers: int = 4, key_scale: float = 10.0):
    """(k, v) each [batch][h_kv][t][d] fp16; per KV head n_key_outliers key channels scaled."""
    k = np.empty((batch, h_kv, t, d), np.float16)
    v = np.empty((batch, h_kv, t, d), np.float16)
    for b in range(batch):
        kk = rng.normal(0.0, 1.0, size=(h_kv, t, d))
        vv = rng.normal(0.0, 1.0, size=(h_kv, t, d))
        for h in range(h_kv):
            ch = rng.choice(d, n_key_outliers, replace=False)
            kk[h][:, ch] *= key_scale
        k[b] = kk.astype(np.float16)
        v[b] = vv.astype(np.float16)
    return k, v


def query(rng: np.random.Generator, h_q: int, d: int, batch: int = 1) -> np.ndarray:
    return rng.normal(0.0, 1.0, size=(batch, h_q, d)).astype(np.float16)


# ---------------------------------------------------------------------------
# the five workloads


def gemv_case(seed: int = 0, n: int = 4096, k: int = 4096, batch: int = 1):
    """Single GEMV: W[n][k] fp32 and x[batch][k] fp16 (4096 x 4096 at seed 0)."""
    rng = np.random.default_rng(seed)
    w = weight(rng, n, k)
    x = activation(rng, k, batch)
    return w, x


def layer_case(seed: int = 1, batch: int = 1, hidden: int = HIDDEN, inter: int = INTER,
               kv_dim: int = N_KV_HEADS * HEAD_DIM):
    """One decoder layer's projections.  Projection p draws its weight from seed
    seed + p (p = 0..6 in LAYER_PROJECTIONS order); the four activations (attn,
    o, mlp, down) come from seed seed + 100 in that order.  Projections that
    read the same activation (q/k/v, gate/up) are returned concatenated along
    the output dimension, in that order."""
    shapes = {"q": (hidden, hidden), "k": (kv_dim, hidden), "v": (kv_dim, hidden),
              "o": (hidden, hidden), "gate": (inter, hidden), "up": (inter, hidden),
              "down": (hidden, inter)}
    ws = {}
    for p, (name, _, _, _) in enumerate(LAYER_PROJECTIONS):
        n, k = shapes[name]
        ws[name] = weight(np.random.default_rng(seed + p), n, k)
    rng = np.random.default_rng(seed + 100)
    xs = {
        "attn": activation(rng, hidden, batch),
        "o": activation(rng, hidden, batch),
        "mlp": activation(rng, hidden, batch),
        "down": activation(rng, inter, batch),
    }
    fused = {
        "qkv": (np.concatenate([ws["q"], ws["k"], ws["v"]], 0), xs["attn"]),
        "o": (ws["o"], xs["o"]),
        "gate_up": (np.concatenate([ws["gate"], ws["up"]], 0), xs["mlp"]),
        "down": (ws["down"], xs["down"]),
    }
    return fused


def kv_case(seed: int = 2, t: int = 8192, h_kv: int = N_KV_HEADS, h_q: int = N_HEADS,
            d: int = HEAD_DIM, batch: int = 1):
    """KV attention: (k, v, q) with k, v [batch][h_kv][t][d] and q [batch][h_q][d], fp16."""
    rng = np.random.default_rng(seed)
    k, v = kv_values(rng, h_kv, t, d, batch)
    q = query(rng, h_q, d, batch)
    return k, v, q


# ---------------------------------------------------------------------------
# a Llama-shaped decoder (the full decode-step workload)

def decoder_layer_weights(seed: int, layer: int, hidden: int = HIDDEN, inter: int = INTER,
                          h_q: int = N_HEADS, h_kv: int = N_KV_HEADS, d: int = HEAD_DIM):
    """fp32 weights of one layer, projections sharing an input concatenated:
    qkv [(h_q + 2 h_kv) d][hidden], o [hidden][h_q d], gate_up [2 inter][hidden],
    down [hidden][inter].  Seed: seed * 1000 + layer."""
    rng = np.random.default_rng(seed * 1000 + layer)
    return {
        "qkv": weight(rng, (h_q + 2 * h_kv) * d, hidden),
        "o": weight(rng, hidden, h_q * d),
        "gate_up": weight(rng, 2 * inter, hidden),
        "down": weight(rng, hidden, inter),
    }


def decoder_layer_kv(seed: int, layer: int, t: int, batch: int = 1, h_kv: int = N_KV_HEADS,
                     d: int = HEAD_DIM):
    """The layer's cached keys and values (fp16 [batch][h_kv][t][d]), drawn as
    for the KV workloads.  Seed: seed * 1000 + 500 + layer."""
    rng = np.random.default_rng(seed * 1000 + 500 + layer)
    return kv_values(rng, h_kv, t, d, batch)


def decoder_io(seed: int, batch: int = 1, hidden: int = HIDDEN, vocab: int = VOCAB):
    """(input hidden state fp16 [batch][hidden], LM head fp16 [vocab][hidden])."""
    rng = np.random.default_rng(seed * 1000 + 999)
    h = rng.normal(0.0, 1.0, size=(batch, hidden)).astype(np.float16)
    lm = rng.normal(0.0, 0.02, size=(vocab, hidden)).astype(np.float16)
    return h, lm


def torch_normal(shape, std: float, seed: int, device="cuda", dtype=None):
    """Seeded N(0, std) drawn on the device with torch's Philox generator (used
    where a workload is too large to draw on the host in reasonable time)."""
    import torch

    g = torch.Generator(device=device)
    g.manual_seed(seed)
    t = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    t.mul_(std)
    return t if dtype is None else t.to(dtype)


def decoder_hidden_pool(seed: int, n: int, batch: int = 1, hidden: int = HIDDEN, outlier_frac: float = 0.01,
                        outlier_scale: float = 20.0, device="cuda"):
    """n decode-step inputs fp16 [n][batch][hidden], one per step of a
    multi-step run: N(0, 1) per channel, with the same round(outlier_frac *
    hidden) channels scaled by outlier_scale in every input (outlier channels
    that persist from token to token, as the activation recipe's 1 % outliers
    but fixed), drawn on the device with torch's seeded Philox generator."""
    import torch

    g = torch.Generator(device=device)
    g.manual_seed(seed)
    h = torch.randn((n, batch, hidden), generator=g, device=device, dtype=torch.float32)
    gc = torch.Generator(device="cpu").manual_seed(seed)
    ch = torch.randperm(hidden, generator=gc)[: int(round(outlier_frac * hidden))].to(device)
    h[:, :, ch] *= outlier_scale
    return h.to(torch.float16)
