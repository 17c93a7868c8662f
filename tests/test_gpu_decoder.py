"""Decode-step parity: the CUDA decode step (bit_decode_selective_b200.decoder)
against the fp64 oracle step (oracle/decoder.py), same seeded weights, caches
and input, with the oracle taking the GPU's selections after checking that
they differ from its own only at near-ties (tests/decoder_pair.py says why);
the bar is the benchmark spec's relative L2 1e-3 on the final logits.
"""
import pytest

from bit_decode_selective_b200.decoder import DecoderConfig
from decoder_pair import run_step_pair

pytestmark = pytest.mark.gpu


SMALL = dict(n_layers=3, hidden=1024, inter=2048, h_q=8, h_kv=2, d=128, vocab=1000, k_tok=16)


@pytest.mark.parametrize("lead,lag,host", [(0, 0, False), (1, 1, False), (1, 1, True), (1, 0, True)])
def test_decode_step_small(lead, lag, host):
    cfg = DecoderConfig(**SMALL, lead=lead, lag=lag, host_refine=host)
    err, wf, tf = run_step_pair(cfg, T=100)
    assert err <= 1e-3, (err, wf, tf)


def test_decode_step_batch():
    cfg = DecoderConfig(**SMALL, lead=1, lag=1, host_refine=True)
    err, wf, tf = run_step_pair(cfg, T=64, batch=3)
    assert err <= 1e-3, (err, wf, tf)


def test_decode_step_base_only():
    """No refinement anywhere (k = 0): the base-only path of every kernel."""
    cfg = DecoderConfig(**SMALL, kch=0, lead=0, lag=0, host_refine=False)
    err, wf, tf = run_step_pair(cfg, T=50)
    assert err <= 1e-3, (err, wf, tf)


@pytest.mark.parametrize("skip", [False, True])
def test_decode_step_row_cache(skip):
    """The step with refinement rows cached across steps, after two steps on
    other inputs (so some rows are hits, some misses); with skip, the missing
    channels stay at base precision in this step (the oracle applies exactly
    the channels the GPU refined)."""
    cfg = DecoderConfig(**SMALL, lead=1, lag=1, host_refine=True, cache_rows=2.0, skip_missing=skip)
    err, wf, tf = run_step_pair(cfg, T=100, warm=2)
    assert err <= 1e-3, (err, wf, tf)
