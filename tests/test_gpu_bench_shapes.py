"""Parity at exactly the shapes and launch forms the benchmark times.

The decode-step benchmark runs the refined GEMV with a 2-bit base and 2
refinement bits, k = 32 of every 1,024 channels, on the four fused projections
of a Llama-3.1-8B-shaped layer (qkv 6,144 x 4,096, o 4,096 x 4,096, gate/up
28,672 x 4,096, down 4,096 x 14,336), with the selection given (fetch lead),
the refinement rows staged, and o in the split form (fetch lag); and it runs
the whole step at hidden 4,096, intermediate 14,336, 32/8 heads, vocab 128,256,
T = 32,768 cached tokens and top-512 tokens per KV head.  Every one of those
launches is compared with the oracle here, and the step itself on two layers
(the lead/lag hand-off between layers included) at batch 1 and batch 8.
"""
import numpy as np
import pytest
import torch

import oracle
from bit_decode_selective_b200 import inputs
from bit_decode_selective_b200.decoder import DecoderConfig
from bit_decode_selective_b200.ops import QuantWeights
from decoder_pair import run_step_pair

pytestmark = pytest.mark.gpu

RTOL_L2 = 1e-3


def cu(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def rel_l2(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30))


@pytest.fixture(scope="module", autouse=True)
def threads():
    oracle.set_threads(0)


STEP_SHAPES = [("qkv", 6144, 4096), ("o", 4096, 4096), ("gate_up", 28672, 4096), ("down", 4096, 14336)]


@pytest.mark.parametrize("name,n,k", STEP_SHAPES)
def test_gemv_step_shapes_b2r2(name, n, k):
    """Self-selected, lead-selected with staged rows, and the split form, at a
    decode-step projection's full shape (b = 2, r = 2, k = 32 per 1,024)."""
    rng = np.random.default_rng(1000 + n + k)
    w = inputs.weight(rng, n, k)
    x = inputs.activation(rng, k, batch=1)
    qb, rho, sz = oracle.quant_weights(w, 2, 2, 128)
    qw = QuantWeights.pack(cu(w), 2, 2, 128)
    del w
    xd = cu(x.view(np.uint16))
    sel_o = oracle.select_chunks(x, 1024, 32)
    want = oracle.gemv_refined(qb, rho, sz, 2, 128, x, sel_o, 1024, 32)
    # the call selects from x itself
    y, sel = qw.gemv(xd, 1024, 32)
    torch.cuda.synchronize()
    assert np.array_equal(sel.cpu().numpy(), sel_o)
    assert rel_l2(y.cpu().numpy(), want) <= RTOL_L2
    # fetch lead: selection given, rows staged in the order of the selection
    sel_d = cu(sel_o)
    rows = qw.refine_rows()[sel_d.view(1, -1).long()].contiguous()
    y2, _ = qw.gemv(xd, 1024, 32, sel_in=sel_d, refine_rows=rows)
    # fetch lag: base product and correction to separate outputs
    yb, yc = qw.gemv_split(xd, sel_d, 1024, 32, refine_rows=rows)
    torch.cuda.synchronize()
    assert rel_l2(y2.cpu().numpy(), want) <= RTOL_L2
    base_o = oracle.gemv_refined(qb, rho, sz, 2, 128, x, None, 1024, 0)
    corr_o = oracle.gemv_correction(qb, rho, sz, 2, 128, x[0], sel_o[0])
    assert rel_l2(yb.cpu().numpy(), base_o) <= RTOL_L2
    assert rel_l2(yc.cpu().numpy()[0], corr_o) <= RTOL_L2
    assert rel_l2(yb.cpu().numpy() + yc.cpu().numpy(), want) <= RTOL_L2


@pytest.mark.slow
@pytest.mark.parametrize("batch", [1, 8])
def test_decode_step_full_shape(batch):
    """Two layers of the benchmarked step at full width (hidden 4,096, inter
    14,336, vocab 128,256), T = 32,768, top-512 tokens, lead = lag = 1,
    refinement rows in pinned host memory staged per layer."""
    cfg = DecoderConfig(n_layers=2, lead=1, lag=1, host_refine=True)
    err, wf, tf = run_step_pair(cfg, T=32768, batch=batch)
    assert err <= RTOL_L2, (err, wf, tf)
