"""ctypes binding of the C ABI in include/sf.h (libsf.so).

Same names as the C entry points; this module only marshals arguments.  Every
step of the decode path runs in the CUDA library: if libsf.so is missing this
module raises on import of the library, there is no CPU fallback.
"""
from __future__ import annotations

import ctypes
import os
from ctypes import POINTER, c_char_p, c_int, c_int32, c_size_t, c_void_p

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "_lib", "libsf.so")

SF_KV_STATIC_WS_BYTES = 32 << 20  # include/sf.h

SF_OK, SF_ERR_INVALID_ARG, SF_ERR_UNSUPPORTED, SF_ERR_CUDA, SF_ERR_TIMEOUT, SF_ERR_WORKSPACE = range(6)


class SFError(RuntimeError):
    def __init__(self, status: int, where: str, message: str):
        super().__init__(f"{where}: status {status} ({message})")
        self.status = status


class sf_wq(ctypes.Structure):
    _fields_ = [("n", c_int32), ("k", c_int32), ("b", c_int32), ("r", c_int32),
                ("group", c_int32), ("base", c_void_p), ("refine", c_void_p), ("sz", c_void_p)]


class sf_row_cache(ctypes.Structure):
    _fields_ = [("capacity", c_int32), ("n_channels", c_int32), ("row_bytes", c_int32),
                ("slot_of", c_void_p), ("channel_of", c_void_p), ("stamp", c_void_p), ("state", c_void_p),
                ("work", c_void_p), ("max_sel", c_int32), ("rows", c_void_p)]


class sf_kv(ctypes.Structure):
    _fields_ = [("batch", c_int32), ("h_kv", c_int32), ("d", c_int32), ("t_max", c_int32),
                ("b", c_int32), ("r", c_int32), ("group", c_int32),
                ("kb", c_void_p), ("kr", c_void_p), ("vb", c_void_p), ("vr", c_void_p),
                ("ksz", c_void_p), ("vsz", c_void_p)]


_SIGNATURES = {
    "sf_abi_version": ([], c_int),
    "sf_status_string": ([c_int], c_char_p),
    "sf_last_error": ([], c_char_p),
    "sf_wq_bytes": ([c_int] * 5 + [POINTER(c_size_t)] * 3, c_int),
    "sf_pack_nested": ([c_void_p, POINTER(sf_wq), c_void_p], c_int),
    "sf_unpack_codes": ([POINTER(sf_wq), c_void_p, c_void_p, c_void_p], c_int),
    "sf_select_channels": ([c_void_p, c_int, c_int, c_int, c_int, c_void_p, c_void_p], c_int),
    "sf_fit_refinements": ([c_void_p, POINTER(sf_wq), c_void_p, c_int, c_int, c_int, ctypes.c_double, c_void_p,
                            c_void_p, c_size_t, c_void_p], c_int),
    "sf_fit_refinements_workspace_bytes": ([c_int] * 5, c_size_t),
    "sf_gemv_refined": ([POINTER(sf_wq), c_void_p, c_int, c_int, c_int, c_void_p, c_void_p,
                         c_void_p, c_void_p, c_void_p, c_size_t, c_void_p], c_int),
    "sf_gemv_workspace_bytes": ([POINTER(sf_wq), c_int, c_int, c_int], c_size_t),
    "sf_gemv_correction": ([POINTER(sf_wq), c_void_p, c_int, c_int, c_int, c_void_p, c_void_p,
                            c_void_p, c_void_p], c_int),
    "sf_gemv_refined_split": ([POINTER(sf_wq), c_void_p, c_int, c_int, c_int, c_void_p, c_void_p,
                               c_void_p, c_void_p, c_void_p], c_int),
    "sf_device_wait_timeouts": ([POINTER(ctypes.c_uint), c_int], c_int),
    "sf_kv_bytes": ([c_int] * 7 + [POINTER(c_size_t)] * 3, c_int),
    "sf_kv_pack_tokens": ([POINTER(sf_kv), c_void_p, c_void_p, c_int, c_int, c_void_p], c_int),
    "sf_kv_append_rope": ([POINTER(sf_kv), c_void_p, c_int, c_int, ctypes.c_float, c_int, c_void_p, c_void_p],
                          c_int),
    "sf_kv_unpack_codes": ([POINTER(sf_kv), c_int, c_int, c_void_p, c_void_p, c_void_p], c_int),
    "sf_kv_score_select": ([POINTER(sf_kv), c_int, c_void_p, c_int, c_int, c_void_p, c_void_p,
                            c_void_p, c_void_p, c_size_t, c_void_p], c_int),
    "sf_kv_score_select_workspace_bytes": ([POINTER(sf_kv), c_int, c_int, c_int, c_int], c_size_t),
    "sf_kv_logits_fma": ([POINTER(sf_kv), c_int, c_void_p, c_int, c_void_p, c_void_p, c_size_t, c_void_p], c_int),
    "sf_kv_logits_fma_workspace_bytes": ([POINTER(sf_kv), c_int, c_int], c_size_t),
    "sf_kv_attn_refined": ([POINTER(sf_kv), c_int, c_void_p, c_int, c_void_p, c_int, c_int,
                            c_void_p, c_void_p, c_size_t, c_void_p], c_int),
    "sf_kv_attn_workspace_bytes": ([POINTER(sf_kv), c_int, c_int, c_int, c_int], c_size_t),
    "sf_kv_attend_selective": ([POINTER(sf_kv), c_int, c_void_p, c_int, c_int, c_void_p, c_void_p,
                                c_void_p, c_void_p, c_size_t, c_void_p], c_int),
    "sf_kv_attend_selective_f16": ([POINTER(sf_kv), c_int, c_void_p, c_int, c_int, c_void_p, c_void_p, c_void_p,
                                    c_void_p, c_size_t, c_void_p], c_int),
    "sf_kv_attend_selective_workspace_bytes": ([POINTER(sf_kv), c_int, c_int, c_int, c_int], c_size_t),
    "sf_kv_attend_selective_static": ([POINTER(sf_kv), c_int, c_void_p, c_int, c_int, c_void_p, c_void_p,
                                       c_void_p, c_void_p], c_int),
    "sf_rmsnorm_residual": ([c_void_p, c_void_p, c_void_p, c_int, c_int, ctypes.c_float, c_void_p,
                             c_void_p], c_int),
    "sf_rope_split": ([c_void_p, c_int, c_int, c_int, c_int, c_int, ctypes.c_float, c_void_p, c_void_p,
                       c_void_p, c_void_p], c_int),
    "sf_silu_mul": ([c_void_p, c_int, c_int, c_void_p, c_void_p], c_int),
    "sf_cast_f16": ([c_void_p, c_size_t, c_void_p, c_void_p], c_int),
    "sf_widen_f16": ([c_void_p, c_size_t, c_void_p, c_void_p], c_int),
    "sf_gemv_f16": ([c_void_p, c_void_p, c_int, c_int, c_int, c_void_p, c_void_p], c_int),
    "sf_stage_refinements": ([c_void_p, c_size_t, c_int, c_void_p, c_int, c_void_p, c_void_p, c_void_p,
                              c_void_p], c_int),
    "sf_stage_refinements_host": ([c_void_p, c_size_t, c_int, c_void_p, c_int, c_void_p, c_void_p,
                                   c_void_p], c_int),
    "sf_row_cache_reset": ([POINTER(sf_row_cache), c_void_p], c_int),
    "sf_stage_refinements_cached": ([c_void_p, c_size_t, c_int, c_void_p, c_int, c_int, POINTER(sf_row_cache),
                                     c_int, c_void_p, c_void_p, c_void_p, c_void_p], c_int),
}

# Symbols every build must export (the header's declarations).
EXPORTED = tuple(_SIGNATURES)

_lib = None


def lib() -> ctypes.CDLL:
    """Load libsf.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise OSError(f"{LIB_PATH} is missing: build it with "
                          "`python -m bit_decode_selective_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (args, res) in _SIGNATURES.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = res
        _lib = L
    return _lib


def check(status: int, where: str) -> None:
    if status != SF_OK:
        msg = lib().sf_last_error().decode(errors="replace")
        raise SFError(status, where, msg)


def _call(name):
    def f(*args):
        return getattr(lib(), name)(*args)

    f.__name__ = name
    return f


# Same-named thin wrappers over the raw entry points.
sf_abi_version = _call("sf_abi_version")
sf_status_string = _call("sf_status_string")
sf_last_error = _call("sf_last_error")
sf_wq_bytes = _call("sf_wq_bytes")
sf_pack_nested = _call("sf_pack_nested")
sf_unpack_codes = _call("sf_unpack_codes")
sf_select_channels = _call("sf_select_channels")
sf_fit_refinements = _call("sf_fit_refinements")
sf_fit_refinements_workspace_bytes = _call("sf_fit_refinements_workspace_bytes")
sf_gemv_refined = _call("sf_gemv_refined")
sf_gemv_workspace_bytes = _call("sf_gemv_workspace_bytes")
sf_gemv_correction = _call("sf_gemv_correction")
sf_gemv_refined_split = _call("sf_gemv_refined_split")
sf_device_wait_timeouts = _call("sf_device_wait_timeouts")
sf_kv_bytes = _call("sf_kv_bytes")
sf_kv_pack_tokens = _call("sf_kv_pack_tokens")
sf_kv_unpack_codes = _call("sf_kv_unpack_codes")
sf_kv_append_rope = _call("sf_kv_append_rope")
sf_kv_score_select = _call("sf_kv_score_select")
sf_kv_score_select_workspace_bytes = _call("sf_kv_score_select_workspace_bytes")
sf_kv_logits_fma = _call("sf_kv_logits_fma")
sf_kv_logits_fma_workspace_bytes = _call("sf_kv_logits_fma_workspace_bytes")
sf_kv_attn_refined = _call("sf_kv_attn_refined")
sf_kv_attn_workspace_bytes = _call("sf_kv_attn_workspace_bytes")
sf_kv_attend_selective = _call("sf_kv_attend_selective")
sf_kv_attend_selective_f16 = _call("sf_kv_attend_selective_f16")
sf_kv_attend_selective_workspace_bytes = _call("sf_kv_attend_selective_workspace_bytes")
sf_kv_attend_selective_static = _call("sf_kv_attend_selective_static")
sf_rmsnorm_residual = _call("sf_rmsnorm_residual")
sf_rope_split = _call("sf_rope_split")
sf_silu_mul = _call("sf_silu_mul")
sf_cast_f16 = _call("sf_cast_f16")
sf_widen_f16 = _call("sf_widen_f16")
sf_gemv_f16 = _call("sf_gemv_f16")
sf_stage_refinements = _call("sf_stage_refinements")
sf_stage_refinements_host = _call("sf_stage_refinements_host")
sf_row_cache_reset = _call("sf_row_cache_reset")
sf_stage_refinements_cached = _call("sf_stage_refinements_cached")
