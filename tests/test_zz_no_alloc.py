"""sf_kv_attend_selective_static (library-owned scratch) against
sf_kv_attend_selective (caller workspace), both called through the C ABI.

The two run the same kernels, so the static-scratch call must give the same
selection and an output within the attention bar (relative L2 1e-3, max-abs
2e-3) of the workspace call, on every call: two calls in a row with different
queries share the one scratch array.  This file is collected last so that it
also runs after every other GPU test in the same process.
"""
import ctypes

import numpy as np
import pytest
import torch

from bit_decode_selective_b200 import abi, inputs
from bit_decode_selective_b200.ops import KVCache, _p

pytestmark = pytest.mark.gpu

RTOL_L2 = 1e-3
ATTN_MAX_ABS = 2e-3


def rel_l2(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30))


def f16(x):
    return torch.from_numpy(np.ascontiguousarray(x).view(np.uint16)).cuda()


def static_call(cache, q, t, k_tok, logits=None):
    B, h_q = q.shape[0], q.shape[1]
    out = torch.full((B, h_q, 128), float("nan"), dtype=torch.float32, device="cuda")
    sel = torch.full((B, cache.h_kv, k_tok), -1, dtype=torch.int32, device="cuda")
    st = abi.sf_kv_attend_selective_static(ctypes.byref(cache.desc), t, _p(q), h_q, k_tok, _p(sel),
                                           _p(logits), _p(out),
                                           ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    abi.check(st, "sf_kv_attend_selective_static")
    return out, sel


def workspace_call(cache, q, t, k_tok, logits=None):
    B, h_q = q.shape[0], q.shape[1]
    out = torch.empty((B, h_q, 128), dtype=torch.float32, device="cuda")
    sel = torch.empty((B, cache.h_kv, k_tok), dtype=torch.int32, device="cuda")
    need = abi.sf_kv_attend_selective_workspace_bytes(ctypes.byref(cache.desc), t, h_q, k_tok,
                                                      int(logits is not None))
    ws = torch.empty(max(need, 16), dtype=torch.uint8, device="cuda")
    st = abi.sf_kv_attend_selective(ctypes.byref(cache.desc), t, _p(q), h_q, k_tok, _p(sel), _p(logits),
                                    _p(out), _p(ws), ws.numel(),
                                    ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    abi.check(st, "sf_kv_attend_selective")
    return out, sel


@pytest.mark.parametrize("T,k_tok,batch", [(8192, 256, 1), (2049, 300, 2)])
def test_static_scratch_matches_workspace_call(T, k_tok, batch):
    assert torch.cuda.is_available(), "the gpu tests need a CUDA device"
    k, v, _ = inputs.kv_case(seed=21, t=T, batch=batch)
    cache = KVCache(batch, 8, (T + 15) // 16 * 16)
    cache.pack_tokens(f16(k), f16(v), 0)
    rng = np.random.default_rng(22)
    queries = [f16(inputs.query(rng, 32, 128, batch)) for _ in range(2)]
    for q in queries:  # two calls in a row on the one scratch array
        want, want_sel = workspace_call(cache, q, T, k_tok)
        got, got_sel = static_call(cache, q, T, k_tok)
        torch.cuda.synchronize()
        g, w = got.cpu().numpy(), want.cpu().numpy()
        assert np.array_equal(got_sel.cpu().numpy(), want_sel.cpu().numpy())
        assert np.isfinite(g).all()
        assert rel_l2(g, w) <= RTOL_L2, rel_l2(g, w)
        assert np.abs(g - w).max() <= ATTN_MAX_ABS


def test_static_scratch_rejects_oversize_request():
    """A request whose workspace exceeds the 32 MiB array fails with
    SF_ERR_WORKSPACE before anything is enqueued."""
    B, T = 2, 133000  # 2 x 32 query heads x T x 4-byte logits = 34.0 MB > 32 MiB
    cache = KVCache(B, 8, (T + 15) // 16 * 16)
    need = abi.sf_kv_attend_selective_workspace_bytes(ctypes.byref(cache.desc), T, 32, 64, 0)
    assert need > abi.SF_KV_STATIC_WS_BYTES
    q = torch.zeros((B, 32, 128), dtype=torch.float16, device="cuda")
    out = torch.zeros((B, 32, 128), dtype=torch.float32, device="cuda")
    sel = torch.zeros((B, 8, 64), dtype=torch.int32, device="cuda")
    st = abi.sf_kv_attend_selective_static(ctypes.byref(cache.desc), T, _p(q), 32, 64, _p(sel), None, _p(out),
                                           ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == abi.SF_ERR_WORKSPACE
    assert b"static scratch" in abi.sf_last_error()
    torch.cuda.synchronize()
    assert not out.any().item() and not sel.any().item()
    # with the logits supplied by the caller the same request fits
    assert abi.sf_kv_attend_selective_workspace_bytes(ctypes.byref(cache.desc), T, 32, 64, 1) \
        <= abi.SF_KV_STATIC_WS_BYTES
