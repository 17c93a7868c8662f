"""CPU oracle for the selective-precision decode path (TEST INFRASTRUCTURE).

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg
(and its ``--impl reference`` arm) may import this package.  The product path
(``bit_decode_selective_b200``) never imports it, and the two share no code: the
oracle is plain C in fp64 (``sf_oracle.c``), this module only marshals numpy
arrays into it.  The one exception is ``fit.py``, the least-squares fit of
weight refinement values, written in numpy fp64 with matrix products and a
linear solve as its library steps.

Each function cites the passage of the StrataFlux pages it follows; the C file
states every reading taken where the pages are silent.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from .build import build_oracle

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = build_oracle()
        _lib = ctypes.CDLL(path)
        _declare(_lib)
    return _lib


def _p(a):
    return a.ctypes.data_as(ctypes.c_void_p)


def _declare(L):
    i, d, vp, u16 = ctypes.c_int, ctypes.c_double, ctypes.c_void_p, ctypes.c_uint16
    sig = {
        "or_set_threads": ([i], i),
        "or_f16_to_f64": ([u16], d),
        "or_f16_from_f64": ([d], u16),
        "or_quant_group": ([vp, i, i, i, vp, vp, vp, vp], None),
        "or_dequant_base": ([u16, u16, i], d),
        "or_dequant_refined": ([u16, u16, i, i, i], d),
        "or_quant_weights": ([vp, i, i, i, i, i, vp, vp, vp], None),
        "or_quant_kv": ([vp, i, i, i, i, i, i, i, vp, vp, vp], None),
        "or_pack_weights": ([vp, vp, i, i, i, i, vp, vp], None),
        "or_pack_kv": ([vp, vp, i, i, i, i, i, i, i, i, vp, vp], None),
        "or_select_chunks": ([vp, i, i, i, i, vp], None),
        "or_gemv_refined": ([vp, vp, vp, i, i, i, i, vp, i, vp, i, i, vp], None),
        "or_kv_logits": ([vp, vp, i, i, i, i, i, vp, i, vp], None),
        "or_kv_scores": ([vp, i, i, i, i, vp], None),
        "or_kv_select": ([vp, i, i, i, i, vp], None),
        "or_kv_attention": ([vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, vp, i, vp, i, vp], None),
        "or_rmsnorm_f16": ([vp, i, d, vp], None),
        "or_rope": ([vp, i, i, i, d], None),
        "or_silu_mul_f16": ([vp, i, vp], None),
        "or_gemv_f16": ([vp, vp, i, i, vp], None),
        "or_gemv_correction": ([vp, vp, vp, i, i, i, i, vp, vp, i, vp], None),
    }
    for name, (args, res) in sig.items():
        fn = getattr(L, name)
        fn.argtypes = args
        fn.restype = res


def set_threads(n: int = 0) -> int:
    """Set the OpenMP thread count (0 keeps the current one); returns it."""
    return lib().or_set_threads(n)


# --------------------------------------------------------------------------
# fp16


def f16_to_f64(bits: int) -> float:
    return lib().or_f16_to_f64(bits)


def f16_from_f64(x: float) -> int:
    return lib().or_f16_from_f64(x)


def _as_f16_bits(x) -> np.ndarray:
    x = np.asarray(x)
    if x.dtype == np.float16:
        return np.ascontiguousarray(x).view(np.uint16)
    assert x.dtype == np.uint16, x.dtype
    return np.ascontiguousarray(x)


# --------------------------------------------------------------------------
# nested quantisation ("nested quantization" paragraph of the explainer)


def quant_group(w, b: int, r: int):
    """One group -> (step fp16 bits, offset fp16 bits, base codes, refinement codes)."""
    w = np.ascontiguousarray(w, dtype=np.float64)
    n = w.size
    s = np.zeros(1, np.uint16)
    m = np.zeros(1, np.uint16)
    qb = np.zeros(n, np.uint8)
    rho = np.zeros(n, np.uint8)
    lib().or_quant_group(_p(w), n, b, r, _p(s), _p(m), _p(qb), _p(rho))
    return int(s[0]), int(m[0]), qb, rho


def dequant_base(s: int, m: int, q: int) -> float:
    return lib().or_dequant_base(s, m, q)


def dequant_refined(s: int, m: int, q: int, rho: int, r: int) -> float:
    return lib().or_dequant_refined(s, m, q, rho, r)


def quant_weights(w: np.ndarray, b: int, r: int, G: int = 128):
    """W[N][K] fp32 -> qb[N][K] u8, rho[N][K] u8, sz[N][K/G][2] fp16 bits."""
    w = np.ascontiguousarray(w, dtype=np.float32)
    N, K = w.shape
    qb = np.empty((N, K), np.uint8)
    rho = np.empty((N, K), np.uint8)
    sz = np.empty((N, K // G, 2), np.uint16)
    lib().or_quant_weights(_p(w), N, K, b, r, G, _p(qb), _p(rho), _p(sz))
    return qb, rho, sz


def quant_kv(x, b: int, r: int, G: int = 32):
    """x[B][H][T][D] fp16 -> qb, rho [B][H][T][D] u8 and sz[B][H][T][D/G][2] fp16 bits."""
    xb = _as_f16_bits(x)
    B, H, T, D = xb.shape
    qb = np.empty((B, H, T, D), np.uint8)
    rho = np.empty((B, H, T, D), np.uint8)
    sz = np.empty((B, H, T, D // G, 2), np.uint16)
    lib().or_quant_kv(_p(xb), B, H, T, D, b, r, G, _p(qb), _p(rho), _p(sz))
    return qb, rho, sz


def dequant_weights(qb, rho, sz, r: int, G: int, refined_mask=None) -> np.ndarray:
    """Dense fp64 reconstruction; refined where refined_mask[N][K] (or a [K] mask) is set."""
    N, K = qb.shape
    f16 = lambda a: np.asarray(a, np.uint16).view(np.float16).astype(np.float64)
    S = np.repeat(f16(sz[:, :, 0]), G, axis=1)
    M = np.repeat(f16(sz[:, :, 1]), G, axis=1)
    val = qb.astype(np.float64)
    if refined_mask is not None:
        mask = np.broadcast_to(refined_mask, (N, K))
        sub = (2.0 * rho.astype(np.float64) + 1.0 - (1 << r)) / float(1 << (r + 1))
        val = val + np.where(mask, sub, 0.0)
    return M + S * val


def pack_weights(qb, rho, b: int, r: int):
    N, K = qb.shape
    # the format permutes 16-byte units inside 128-byte blocks of every row:
    # rows of whole blocks only (the library's k % 1024 rule)
    assert K % 1024 == 0, "k must be a multiple of 1024"
    qb = np.ascontiguousarray(qb, np.uint8)
    rho = np.ascontiguousarray(rho, np.uint8)
    base = np.empty(N * K * b // 8, np.uint8)
    refine = np.empty(K * N * r // 8, np.uint8)
    lib().or_pack_weights(_p(qb), _p(rho), N, K, b, r, _p(base), _p(refine))
    return base, refine


def pack_kv(qb, rho, which: int, b: int, r: int, t_max: int | None = None):
    """Packed bytes of keys (which=0) or values (which=1) in the pair-slot layout."""
    B, H, T, D = qb.shape
    t_max = T if t_max is None else t_max
    assert D == 128 and t_max % 16 == 0
    qb = np.ascontiguousarray(qb, np.uint8)
    rho = np.ascontiguousarray(rho, np.uint8)
    base = np.empty(B * H * t_max * D * b // 8, np.uint8)
    refine = np.empty(B * H * t_max * D * r // 8, np.uint8)
    lib().or_pack_kv(_p(qb), _p(rho), which, B, H, T, t_max, D, b, r, _p(base), _p(refine))
    return base, refine


# --------------------------------------------------------------------------
# selection and the refined GEMV ("which tiles count" paragraph)


def select_chunks(x, C: int, k: int) -> np.ndarray:
    xb = _as_f16_bits(x)
    if xb.ndim == 1:
        xb = xb[None]
    B, K = xb.shape
    sel = np.zeros((B, K // C, k), np.int32)
    if k > 0:
        lib().or_select_chunks(_p(xb), B, K, C, k, _p(sel))
    return sel


def gemv_refined(qb, rho, sz, r: int, G: int, x, sel, C: int, k: int) -> np.ndarray:
    xb = _as_f16_bits(x)
    if xb.ndim == 1:
        xb = xb[None]
    B, K = xb.shape
    N = qb.shape[0]
    y = np.empty((B, N), np.float64)
    sel = np.ascontiguousarray(np.zeros((B, K // C, max(k, 1)), np.int32) if sel is None else sel, np.int32)
    lib().or_gemv_refined(_p(np.ascontiguousarray(qb)), _p(np.ascontiguousarray(rho)),
                          _p(np.ascontiguousarray(sz)), N, K, r, G, _p(xb), B, _p(sel), C, k, _p(y))
    return y


# --------------------------------------------------------------------------
# KV scoring, selection and refined attention


def kv_logits(kqb, ksz, q, G: int = 32) -> np.ndarray:
    B, H, T, D = kqb.shape
    qb16 = _as_f16_bits(q)
    Hq = qb16.shape[1]
    out = np.empty((B, Hq, T), np.float64)
    lib().or_kv_logits(_p(np.ascontiguousarray(kqb)), _p(np.ascontiguousarray(ksz)), B, H, T, D, G,
                       _p(qb16), Hq, _p(out))
    return out


def kv_scores(logits, H: int) -> np.ndarray:
    logits = np.ascontiguousarray(logits, np.float64)
    B, Hq, T = logits.shape
    out = np.empty((B, H, T), np.float64)
    lib().or_kv_scores(_p(logits), B, Hq, H, T, _p(out))
    return out


def kv_select(score, k_tok: int) -> np.ndarray:
    score = np.ascontiguousarray(score, np.float64)
    B, H, T = score.shape
    sel = np.zeros((B, H, k_tok), np.int32)
    if k_tok > 0:
        lib().or_kv_select(_p(score), B, H, T, k_tok, _p(sel))
    return sel


def kv_attention(k_codes, v_codes, q, sel, k_tok: int, r: int, G: int = 32) -> np.ndarray:
    """k_codes, v_codes: (qb, rho, sz) from quant_kv.  Returns out[B][Hq][D] fp64."""
    kqb, krho, ksz = (np.ascontiguousarray(a) for a in k_codes)
    vqb, vrho, vsz = (np.ascontiguousarray(a) for a in v_codes)
    B, H, T, D = kqb.shape
    qb16 = _as_f16_bits(q)
    Hq = qb16.shape[1]
    out = np.empty((B, Hq, D), np.float64)
    sel = np.ascontiguousarray(np.zeros((B, H, 1), np.int32) if sel is None or k_tok == 0 else sel, np.int32)
    lib().or_kv_attention(_p(kqb), _p(krho), _p(ksz), _p(vqb), _p(vrho), _p(vsz), B, H, T, D, G, r,
                          _p(qb16), Hq, _p(sel), k_tok, _p(out))
    return out


# --------------------------------------------------------------------------
# decoder-step glue (standard Llama operations; readings in sf_oracle.c)


def rmsnorm_f16(h, eps: float = 1e-5) -> np.ndarray:
    h = np.ascontiguousarray(h, np.float64)
    x = np.empty(h.size, np.uint16)
    lib().or_rmsnorm_f16(_p(h), h.size, eps, _p(x))
    return x


def rope(v, pos: int, theta: float = 500000.0) -> np.ndarray:
    """v[heads][d] (fp64), rotated in a copy."""
    v = np.array(v, np.float64, copy=True, order="C")
    lib().or_rope(_p(v), v.shape[0], v.shape[1], pos, theta)
    return v


def silu_mul_f16(gu) -> np.ndarray:
    gu = np.ascontiguousarray(gu, np.float64)
    out = np.empty(gu.size // 2, np.uint16)
    lib().or_silu_mul_f16(_p(gu), gu.size // 2, _p(out))
    return out


def gemv_f16(w, x) -> np.ndarray:
    w16 = _as_f16_bits(w)
    x16 = _as_f16_bits(x).ravel()
    N, K = w16.shape
    y = np.empty(N, np.float64)
    lib().or_gemv_f16(_p(w16), _p(x16), N, K, _p(y))
    return y


def gemv_correction(qb, rho, sz, r: int, G: int, x, sel) -> np.ndarray:
    """y = sum over sel of x_c (w~ - w^)[:, c] for one activation row x."""
    x16 = _as_f16_bits(x).ravel()
    sel = np.ascontiguousarray(np.asarray(sel, np.int32).ravel())
    N, K = qb.shape
    y = np.empty(N, np.float64)
    lib().or_gemv_correction(_p(np.ascontiguousarray(qb)), _p(np.ascontiguousarray(rho)),
                             _p(np.ascontiguousarray(sz)), N, K, r, G, _p(x16), _p(sel), sel.size, _p(y))
    return y
