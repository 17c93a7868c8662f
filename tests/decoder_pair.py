"""Helpers of the decode-step parity tests: run the CUDA step and the fp64
oracle step on the same seeded model, with the oracle taking the GPU's
selections after checking that each differs from the oracle's own choice only
at near-ties.

Why teacher forcing: the GPU carries the residual stream in fp32 and the oracle
in fp64, and both hand fp16 activations between operations.  An fp16 rounding
can land on the other side of a midpoint, so a channel whose |x| ties the k-th
largest of its chunk (to an fp16 step), or a token whose score ties the k-th
score, can be selected on one side and not the other.  Such a flip is a valid
outcome on both sides (the selection is only defined up to those ties), but it
changes the output by far more than rounding.  So the oracle is run with the
GPU's selections, each checked to differ from the oracle's own only at
near-ties, and the logits are then compared at the benchmark spec's bar.
"""
import numpy as np
import torch

import oracle
from oracle.decoder import OracleDecoder
from bit_decode_selective_b200 import inputs
from bit_decode_selective_b200.decoder import Decoder

# a differing channel's |x| must lie within W_TOL (relative) of its chunk's k-th
# largest |x|: four fp16 steps, the reach of activations that differ by the
# rounding of an fp32 against an fp64 residual stream
W_TOL = 2.0 ** -8
# a differing token's oracle score must lie within TOK_TOL (relative) of the
# k-th score.  The two sides' q differ by the fp16 rounding of each component
# (relative 2^-11), so a logit moves by up to 2^-11 sum_d |q_d k_d| / sqrt(d),
# about 5e-3 for logits of a few units; a score (a sum of softmax
# probabilities, each moved through its logit and its head's normaliser) by
# up to about twice that
TOK_TOL = 1e-2


def cu(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def rel_l2(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30))


def check_near_ties(checks, chunk, kch, k_tok):
    """Every forced selection is well formed and differs from the oracle's own
    only at near-ties.  Returns (channel flips, token flips)."""
    wf = tf = 0
    for kind, l, name, b, own, forced, vals in checks:
        if kind == "w":
            own = np.asarray(own).reshape(-1, kch)
            forced = np.asarray(forced).reshape(-1, kch)
            forced = np.where(forced < 0, -1 - forced, forced)  # skipped entries name their channel too
            xv = np.asarray(vals)
            if xv.dtype != np.float16:  # fp16 bit patterns
                xv = xv.astype(np.uint16).view(np.float16)
            mag = np.abs(xv.astype(np.float64).reshape(-1))
            for c in range(own.shape[0]):
                f = forced[c]
                assert np.all(np.diff(f) > 0) and f[0] >= c * chunk and f[-1] < (c + 1) * chunk, (l, name, b, c)
                d = set(own[c].tolist()) ^ set(f.tolist())
                if not d:
                    continue
                kth = np.sort(mag[c * chunk:(c + 1) * chunk])[::-1][kch - 1]
                for ch in d:
                    assert abs(mag[ch] - kth) <= W_TOL * kth, (l, name, b, ch, mag[ch], kth)
                wf += len(d) // 2
        else:
            own = np.asarray(own)
            forced = np.asarray(forced)
            for g in range(own.shape[0]):
                f = forced[g]
                assert np.all(np.diff(f) > 0) and f[0] >= 0 and f[-1] < vals.shape[-1], (l, b, g)
                d = set(own[g].tolist()) ^ set(f.tolist())
                if not d:
                    continue
                kth = np.sort(vals[g])[::-1][k_tok - 1]
                for t in d:
                    assert abs(vals[g][t] - kth) <= TOK_TOL * kth, (l, b, g, t, vals[g][t], kth)
                tf += len(d) // 2
    return wf, tf


def run_step_pair(cfg, T: int, batch: int = 1, seed: int = 4, warm: int = 0):
    """The GPU step (with its selections traced) and the oracle step forced to
    those selections.  warm > 0: the GPU decoder first runs `warm` steps on
    other inputs (whose state, e.g. cached refinement rows, the compared step
    inherits; the KV caches are the same, since every step writes the new token
    to the same position).  Returns (rel-L2 of the logits, channel flips,
    token flips)."""
    oracle.set_threads(0)
    h16, lm = inputs.decoder_io(seed, batch, cfg.hidden, cfg.vocab)
    dec = Decoder(cfg, batch, T)
    layers = []
    for l in range(cfg.n_layers):
        W = inputs.decoder_layer_weights(seed, l, cfg.hidden, cfg.inter, cfg.h_q, cfg.h_kv, cfg.d)
        k, v = inputs.decoder_layer_kv(seed, l, T, batch, cfg.h_kv, cfg.d)
        dec.load_layer({n: cu(w) for n, w in W.items()}, cu(k.view(np.uint16)), cu(v.view(np.uint16)))
        del W, k, v
    dec.set_lm_head(cu(lm.view(np.uint16)))
    for i in range(warm):
        other, _ = inputs.decoder_io(seed + 100 + i, batch, cfg.hidden, 8)
        mix = other.astype(np.float32) * 0.5 + h16.astype(np.float32) * 0.5  # inputs that share some channels
        dec.step(cu(mix.astype(np.float16).view(np.uint16)))
    torch.cuda.synchronize()
    dec.trace = []
    logits = dec.step(cu(h16.view(np.uint16)))
    torch.cuda.synchronize()
    got = logits.cpu().numpy()
    force = {key: t.cpu().numpy() for key, t in dec.trace}
    del dec
    torch.cuda.empty_cache()
    ref = OracleDecoder(h16, h_q=cfg.h_q, h_kv=cfg.h_kv, d=cfg.d, r=cfg.w_refine, G=cfg.group,
                        chunk=cfg.chunk, kch=cfg.kch, kv_b=cfg.kv_bits, kv_r=cfg.kv_refine, k_tok=cfg.k_tok,
                        lead=cfg.lead, lag=cfg.lag, eps=cfg.eps, theta=cfg.theta, force=force)
    for l in range(cfg.n_layers):
        W = inputs.decoder_layer_weights(seed, l, cfg.hidden, cfg.inter, cfg.h_q, cfg.h_kv, cfg.d)
        Q = {n: oracle.quant_weights(w, cfg.w_bits, cfg.w_refine, cfg.group) for n, w in W.items()}
        del W
        k, v = inputs.decoder_layer_kv(seed, l, T, batch, cfg.h_kv, cfg.d)
        ref.layer(Q, k, v, T)
        del Q, k, v
    want = ref.finish(lm)
    wf, tf = check_near_ties(ref.checks, cfg.chunk, cfg.kch, cfg.k_tok)
    return rel_l2(got, want), wf, tf
