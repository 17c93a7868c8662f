"""Synthetic accuracy ablation of the KV refinement.

"StrataFlux -- Selective precision streaming -- What does it mean?", nested
quantization paragraph and the comparison table under it: at matched key+value
bit budgets, nested refinement of the selected tokens (4 or 8 extra bits per
element in the paper's measurement) gives a lower KL divergence than fetching
complete 16-bit entries for selected tokens (SpeCache-style, the rest stay at
the low-bit value) and than sparse attention (only the selected tokens, at 16
bits, attended at all).  The paper measures this on real models; here the
ranking is reproduced on the seeded synthetic KV workload, no dataset.

Model: one GQA attention layer (8 KV heads, 4 query heads each, head dim 128)
followed by a fixed random projection to a 512-way softmax; the divergence is
KL(p_exact || p_method) of that softmax, p_exact from the fp16 keys and values.
Every method keeps the 2-bit base of every token resident (except sparse
attention, which has none) and spends the same extra bits per element over
the cache:
  nested  : r refinement bits on the k_tok highest-scoring tokens (2 + r k/T);
  fetch16 : 16-bit entries for the k_tok r / 16 highest-scoring tokens;
  sparse  : 16-bit entries for (2 T + r k_tok) / 16 tokens, nothing else.
Tokens are ranked by the method's score (the sum over the group's query heads
of each head's softmax probability, from the base keys).  The quantisation is
the oracle's; the small attention model is written out here.
"""
import numpy as np
import pytest

import oracle
from bit_decode_selective_b200 import inputs

H, GQ, D, GROUP, B_BITS = 8, 4, 128, 32, 2
T, K_TOK, VOCAB = 2048, 128, 512


def dequant(x, refine_rows, r):
    """Keys or values [H][T][D] after nested quantisation (b = 2, r bits),
    refined on the tokens of refine_rows [H][T]."""
    qb, rho, sz = oracle.quant_kv(x[None], B_BITS, r, GROUP)
    n = H * T
    mask = np.repeat(refine_rows.reshape(n, 1), D, 1)
    return oracle.dequant_weights(qb.reshape(n, D), rho.reshape(n, D), sz.reshape(n, D // GROUP, 2),
                                  r, GROUP, mask).reshape(H, T, D)


def ablation(seed, r):
    k, v, q = inputs.kv_case(seed=seed, t=T, h_kv=H, h_q=H * GQ, batch=1)
    kf, vf, qf = k[0].astype(np.float64), v[0].astype(np.float64), q[0].astype(np.float64)
    w_out = np.random.default_rng(seed + 7).standard_normal((H * GQ * D, VOCAB)) / np.sqrt(H * GQ * D)

    def model(keys, vals, keep=None):
        outs = []
        for h in range(H * GQ):
            g = h // GQ
            l = keys[g] @ qf[h] / np.sqrt(D)
            if keep is not None:
                l = np.where(keep[g], l, -np.inf)
            p = np.exp(l - l.max())
            outs.append((p / p.sum()) @ vals[g])
        z = np.concatenate(outs) @ w_out
        e = np.exp(z - z.max())
        return e / e.sum()

    p_ref = model(kf, vf)

    def kl(p):
        return float(np.sum(p_ref * np.log(p_ref / p)))

    none = np.zeros((H, T), bool)
    kb, vb = dequant(k[0], none, r), dequant(v[0], none, r)

    def top(n):
        sel = np.zeros((H, T), bool)
        for g in range(H):
            s = np.zeros(T)
            for h in range(g * GQ, (g + 1) * GQ):
                l = kb[g] @ qf[h] / np.sqrt(D)
                p = np.exp(l - l.max())
                s += p / p.sum()
            sel[g, np.argsort(-s, kind="stable")[:n]] = True
        return sel

    sel = top(K_TOK)
    out = {"base": kl(model(kb, vb)),
           "nested": kl(model(dequant(k[0], sel, r), dequant(v[0], sel, r)))}
    s16 = top(K_TOK * r // 16)
    out["fetch16"] = kl(model(np.where(s16[..., None], kf, kb), np.where(s16[..., None], vf, vb)))
    out["sparse"] = kl(model(kf, vf, keep=top((T * B_BITS + K_TOK * r) // 16)))
    return out


@pytest.fixture(scope="module", autouse=True)
def threads():
    oracle.set_threads(0)


@pytest.mark.parametrize("r", [2, 4])
@pytest.mark.parametrize("seed", [0, 1, 2, 3])
def test_nested_refinement_beats_16bit_fetch_and_sparse_attention(seed, r):
    kl = ablation(seed, r)
    assert kl["nested"] < kl["base"] / 5, kl
    assert kl["nested"] < kl["fetch16"], kl
    assert kl["nested"] < kl["sparse"], kl
