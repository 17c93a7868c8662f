"""fp64 oracle of one decode step of a Llama-shaped decoder whose projections
and KV attention are refined selectively (TEST INFRASTRUCTURE).

The step follows the StrataFlux pages ("StrataFlux -- Selective precision
streaming -- What does it mean?"):
  which-tiles-count paragraph -- per projection, the k channels with the
    largest |x| in each 1,024-channel chunk are refined; per KV head the
    highest-scoring tokens are refined;
  the-map-app-also-loads-tiles paragraph -- fetch lead picks the channels one
    layer early, from an earlier activation; fetch lag adds the correction one
    layer later.
Readings (the pages describe lead/lag only in prose):
  lead = 1: the selection used by a projection of layer l is made from the same
    projection input one layer earlier (layer l-1); layer 0 uses its own input.
    The correction always uses the current layer's activation values.
  lag = 1: only the residual-writing projections (o, down) defer their
    correction: it is added to the residual stream at the start of the next
    layer (after the last layer: before the final norm).  q/k/v and gate/up
    correct in place, because a nonlinearity follows them.
  The new token's key/value are appended at position T (quantised like the
  cache) and attention runs over T + 1 tokens.  Activations handed between
  operations are fp16; the residual stream and all arithmetic are fp64.

The layers are fed one at a time (layer(...)), so a caller can generate,
quantise and discard each layer's weights in turn.
"""
from __future__ import annotations

import math

import numpy as np

from . import (gemv_correction, gemv_f16, gemv_refined, kv_attention, kv_logits, kv_scores,
               kv_select, quant_kv, rmsnorm_f16, rope, select_chunks, silu_mul_f16)


class OracleDecoder:
    def __init__(self, hidden_f16, *, h_q=32, h_kv=8, d=128, r=2, G=128, chunk=1024, kch=32,
                 kv_b=2, kv_r=2, k_tok=512, lead=1, lag=1, eps=1e-5, theta=500000.0, force=None):
        """force (optional): selections to use instead of the oracle's own,
        {("w", layer, name): int32 [B][n_sel], ("tok", layer): int32 [B][h_kv][k_tok]}.
        The oracle still makes its own choice at every point and records it,
        with the values it was made from, in self.checks, so a caller can check
        that a forced selection differs from it only at near-ties."""
        self.force = force
        self.checks = []                       # (kind, layer, name, b, own, forced, values)
        self.h = np.asarray(hidden_f16, np.float16).astype(np.float64).copy()  # [B][H]
        self.B = self.h.shape[0]
        self.h_q, self.h_kv, self.d = h_q, h_kv, d
        self.r, self.G, self.chunk, self.kch = r, G, chunk, kch
        self.kv_b, self.kv_r, self.k_tok = kv_b, kv_r, k_tok
        self.lead, self.lag, self.eps, self.theta = lead, lag, eps, theta
        self.pending = np.zeros_like(self.h)   # lagged corrections
        self.prev_sel = None                   # lead selections from the layer before
        self.prev_x = None                     # and the activations they were made from
        self.l = 0
        self.trace = []                        # per layer: selections used

    def _select(self, name, x16, b):
        """Selection used by projection `name` of the current layer for row b."""
        if self.lead and self.prev_sel is not None:
            own, src = self.prev_sel[name][b], self.prev_x[name][b]
        else:
            own, src = select_chunks(x16, self.chunk, self.kch)[0], x16
        if self.force is not None and self.kch > 0:
            forced = np.asarray(self.force[("w", self.l, name)][b]).reshape(own.shape)
            self.checks.append(("w", self.l, name, b, own, forced, src))
            return forced
        return own

    def _proj(self, w, x16, sel):
        qb, rho, sz = w
        sel = np.asarray(sel)
        if (sel < 0).any():
            # a forced selection may mark a channel -1 - c: selected, but its
            # refinement did not arrive in this step, so it stays at base
            # precision (the map-app paragraph's skip on a miss)
            y = gemv_refined(qb, rho, sz, self.r, self.G, x16, None, self.chunk, 0)[0]
            return y + gemv_correction(qb, rho, sz, self.r, self.G, x16, sel[sel >= 0])
        return gemv_refined(qb, rho, sz, self.r, self.G, x16, sel[None], self.chunk, self.kch)[0]

    def layer(self, W, k_cache, v_cache, pos):
        """W: {'qkv','o','gate_up','down'} -> (qb, rho, sz) from quant_weights.
        k_cache, v_cache: fp16 [B][h_kv][pos][d] (the cached tokens); the new
        token goes to position pos."""
        B, H = self.h.shape
        hq, hk, d = self.h_q, self.h_kv, self.d
        next_sel = {n: [None] * B for n in ("qkv", "o", "gate_up", "down")}
        next_x = {n: [None] * B for n in ("qkv", "o", "gate_up", "down")}
        used = {n: [None] * B for n in ("qkv", "o", "gate_up", "down")}
        sel_tok = []
        for b in range(B):
            self.h[b] += self.pending[b]
            self.pending[b] = 0.0
            x_attn = rmsnorm_f16(self.h[b], self.eps)
            s = self._select("qkv", x_attn, b)
            used["qkv"][b] = s
            next_sel["qkv"][b] = select_chunks(x_attn, self.chunk, self.kch)[0]
            next_x["qkv"][b] = x_attn
            qkv = self._proj(W["qkv"], x_attn, s)
            q = rope(qkv[: hq * d].reshape(hq, d), pos, self.theta)
            k = rope(qkv[hq * d:(hq + hk) * d].reshape(hk, d), pos, self.theta)
            v = qkv[(hq + hk) * d:].reshape(hk, d)
            q16 = q.astype(np.float16)
            k16 = k.astype(np.float16)
            v16 = v.astype(np.float16)
            K = np.concatenate([k_cache[b], k16[:, None, :]], axis=1)[None]  # [1][hk][T+1][d]
            V = np.concatenate([v_cache[b], v16[:, None, :]], axis=1)[None]
            kc = quant_kv(K, self.kv_b, self.kv_r)
            vc = quant_kv(V, self.kv_b, self.kv_r)
            lg = kv_logits(kc[0], kc[2], q16[None])
            sc = kv_scores(lg, hk)
            st = kv_select(sc, self.k_tok)
            if self.force is not None:
                forced = np.asarray(self.force[("tok", self.l)][b])[None]
                self.checks.append(("tok", self.l, None, b, st[0], forced[0], sc[0]))
                st = forced
            sel_tok.append(st[0])
            att = kv_attention(kc, vc, q16[None], st, self.k_tok, self.kv_r)[0]  # [hq][d]
            x_o = att.reshape(-1).astype(np.float16)
            s = self._select("o", x_o, b)
            used["o"][b] = s
            next_sel["o"][b] = select_chunks(x_o, self.chunk, self.kch)[0]
            next_x["o"][b] = x_o
            if self.lag:
                qb, rho, sz = W["o"]
                o = gemv_refined(qb, rho, sz, self.r, self.G, x_o, None, self.chunk, 0)[0]
                self.pending[b] += gemv_correction(qb, rho, sz, self.r, self.G, x_o, np.asarray(s)[np.asarray(s) >= 0])
            else:
                o = self._proj(W["o"], x_o, s)
            self.h[b] += o
            x_mlp = rmsnorm_f16(self.h[b], self.eps)
            s = self._select("gate_up", x_mlp, b)
            used["gate_up"][b] = s
            next_sel["gate_up"][b] = select_chunks(x_mlp, self.chunk, self.kch)[0]
            next_x["gate_up"][b] = x_mlp
            gu = self._proj(W["gate_up"], x_mlp, s)
            x_down = silu_mul_f16(gu)
            s = self._select("down", x_down, b)
            used["down"][b] = s
            next_sel["down"][b] = select_chunks(x_down, self.chunk, self.kch)[0]
            next_x["down"][b] = x_down
            if self.lag:
                qb, rho, sz = W["down"]
                dn = gemv_refined(qb, rho, sz, self.r, self.G, x_down, None, self.chunk, 0)[0]
                self.pending[b] += gemv_correction(qb, rho, sz, self.r, self.G, x_down,
                                                   np.asarray(s)[np.asarray(s) >= 0])
            else:
                dn = self._proj(W["down"], x_down, s)
            self.h[b] += dn
        self.prev_sel = next_sel
        self.prev_x = next_x
        self.trace.append({"weights": used, "tokens": sel_tok})
        self.l += 1

    def finish(self, lm_head_f16):
        """Final norm (after the last lagged corrections) and the fp16 LM head."""
        out = []
        for b in range(self.B):
            self.h[b] += self.pending[b]
            self.pending[b] = 0.0
            x = rmsnorm_f16(self.h[b], self.eps)
            out.append(gemv_f16(lm_head_f16, x))
        return np.stack(out)
