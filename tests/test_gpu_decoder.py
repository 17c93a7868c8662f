"""Decode-step parity: the CUDA decode step (bit_decode_selective_b200.decoder)
against the fp64 oracle step (oracle/decoder.py), same seeded weights, caches
and input.

Activations are handed between operations in fp16 on both sides, but the GPU
keeps the residual stream in fp32 and the oracle in fp64, so an fp16 rounding
can land on the other side of a tie and flip one channel of a selection; the
bar is therefore on the final logits (relative L2 <= 1e-3), with the share of
identical selections reported.
"""
import numpy as np
import pytest
import torch

import oracle
from oracle.decoder import OracleDecoder
from bit_decode_selective_b200 import inputs
from bit_decode_selective_b200.decoder import Decoder, DecoderConfig

pytestmark = pytest.mark.gpu


def cu(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def run_pair(cfg: DecoderConfig, T: int, batch: int = 1, seed: int = 4):
    oracle.set_threads(0)
    h16, lm = inputs.decoder_io(seed, batch, cfg.hidden, cfg.vocab)
    dec = Decoder(cfg, batch, T)
    ref = OracleDecoder(h16, h_q=cfg.h_q, h_kv=cfg.h_kv, d=cfg.d, r=cfg.w_refine, G=cfg.group,
                        chunk=cfg.chunk, kch=cfg.kch, kv_b=cfg.kv_bits, kv_r=cfg.kv_refine, k_tok=cfg.k_tok,
                        lead=cfg.lead, lag=cfg.lag, eps=cfg.eps, theta=cfg.theta)
    for l in range(cfg.n_layers):
        W = inputs.decoder_layer_weights(seed, l, cfg.hidden, cfg.inter, cfg.h_q, cfg.h_kv, cfg.d)
        k, v = inputs.decoder_layer_kv(seed, l, T, batch, cfg.h_kv, cfg.d)
        dec.load_layer({n: cu(w) for n, w in W.items()}, cu(k.view(np.uint16)), cu(v.view(np.uint16)))
        Q = {n: oracle.quant_weights(w, cfg.w_bits, cfg.w_refine, cfg.group) for n, w in W.items()}
        ref.layer(Q, k, v, T)
        del W, Q
    dec.set_lm_head(cu(lm.view(np.uint16)))
    logits = dec.step(cu(h16.view(np.uint16)))
    torch.cuda.synchronize()
    got = logits.cpu().numpy()
    want = ref.finish(lm)
    err = float(np.linalg.norm(got - want) / np.linalg.norm(want))
    return err, got, want, dec, ref


SMALL = dict(n_layers=3, hidden=1024, inter=2048, h_q=8, h_kv=2, d=128, vocab=1000, k_tok=16)


@pytest.mark.parametrize("lead,lag,host", [(0, 0, False), (1, 1, False), (1, 1, True), (1, 0, True)])
def test_decode_step_small(lead, lag, host):
    cfg = DecoderConfig(**SMALL, lead=lead, lag=lag, host_refine=host)
    err, got, want, _, _ = run_pair(cfg, T=100)
    assert err <= 1e-3, err


def test_decode_step_batch():
    cfg = DecoderConfig(**SMALL, lead=1, lag=1, host_refine=True)
    err, got, want, _, _ = run_pair(cfg, T=64, batch=3)
    assert err <= 1e-3, err


def test_decode_step_base_only():
    """No refinement anywhere (k = 0): the base-only path of every kernel."""
    cfg = DecoderConfig(**SMALL, kch=0, lead=0, lag=0, host_refine=False)
    err, *_ = run_pair(cfg, T=50)
    assert err <= 1e-3, err
