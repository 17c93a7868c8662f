"""Host-only checks of the C ABI (no GPU needed): the library loads, exports
every entry point include/sf.h declares, and rejects bad arguments on the host
before touching the device."""
import ctypes
import os
import re

import pytest

from bit_decode_selective_b200 import abi

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    text = open(os.path.join(ROOT, "include", "sf.h")).read()
    return set(re.findall(r"^SF_API\s+[\w\s\*]+?\b(sf_\w+)\s*\(", text, flags=re.M))


@pytest.fixture(scope="module")
def L():
    from bit_decode_selective_b200.build import build_library

    build_library()
    return abi.lib()


def test_exports_every_declared_symbol(L):
    names = declared_symbols()
    assert len(names) >= 18
    for name in names:
        assert hasattr(L, name), name
    assert names == set(abi.EXPORTED)


def test_version_and_status_strings(L):
    assert abi.sf_abi_version() == 1
    assert abi.sf_status_string(0) == b"ok"
    assert abi.sf_status_string(abi.SF_ERR_WORKSPACE) == b"workspace too small"


def test_byte_sizes(L):
    s = [ctypes.c_size_t() for _ in range(3)]
    assert abi.sf_wq_bytes(4096, 4096, 2, 2, 128, *[ctypes.byref(x) for x in s]) == 0
    assert [x.value for x in s] == [4096 * 4096 // 4, 4096 * 4096 // 4, 4096 * 32 * 4]
    assert abi.sf_wq_bytes(4096, 4096, 5, 2, 128, *[ctypes.byref(x) for x in s]) == abi.SF_ERR_INVALID_ARG
    assert abi.sf_kv_bytes(1, 8, 128, 8192, 2, 2, 32, *[ctypes.byref(x) for x in s]) == 0
    assert [x.value for x in s] == [8 * 8192 * 32, 8 * 8192 * 32, 8 * 8192 * 16]


def test_validation_rejects_before_launch(L):
    # null pointers / unsupported shapes are refused on the host
    wq = abi.sf_wq(4096, 4096, 2, 2, 128, None, None, None)
    assert abi.sf_pack_nested(None, ctypes.byref(wq), None) == abi.SF_ERR_INVALID_ARG
    assert b"base" in abi.sf_last_error()
    wq = abi.sf_wq(4096, 4000, 2, 2, 128, 16, 16, 16)
    assert abi.sf_pack_nested(ctypes.c_void_p(16), ctypes.byref(wq), None) == abi.SF_ERR_UNSUPPORTED
    wq = abi.sf_wq(4096, 4096, 2, 2, 128, 17, 16, 16)  # misaligned
    assert abi.sf_pack_nested(ctypes.c_void_p(16), ctypes.byref(wq), None) == abi.SF_ERR_INVALID_ARG
    assert abi.sf_select_channels(None, 1, 4096, 1024, 32, None, None) == abi.SF_ERR_INVALID_ARG
    assert abi.sf_select_channels(ctypes.c_void_p(16), 1, 4096, 1000, 32, ctypes.c_void_p(16), None) \
        == abi.SF_ERR_UNSUPPORTED
    assert abi.sf_select_channels(ctypes.c_void_p(16), 1, 4096, 1024, 0, ctypes.c_void_p(16), None) \
        == abi.SF_ERR_INVALID_ARG
    kv = abi.sf_kv(1, 8, 128, 8192, 2, 2, 32, 16, 16, 16, 16, 16, 16)
    # k_tok > t
    assert abi.sf_kv_score_select(ctypes.byref(kv), 10, ctypes.c_void_p(16), 32, 11, ctypes.c_void_p(16),
                                  None, None, None, 0, None) == abi.SF_ERR_INVALID_ARG
    # 5-bit KV bases are not built; 3-bit ones size as 48 bytes per key token
    kv5 = abi.sf_kv(1, 8, 128, 8192, 5, 2, 32, 16, 16, 16, 16, 16, 16)
    assert abi.sf_kv_pack_tokens(ctypes.byref(kv5), ctypes.c_void_p(16), None, 0, 1, None) \
        == abi.SF_ERR_UNSUPPORTED
    s3 = [ctypes.c_size_t() for _ in range(3)]
    assert abi.sf_kv_bytes(1, 8, 128, 16, 3, 2, 32, *[ctypes.byref(x) for x in s3]) == 0
    assert s3[0].value == 8 * 16 * 48
    # too little workspace is reported, not overrun
    assert abi.sf_kv_attn_refined(ctypes.byref(kv), 100, ctypes.c_void_p(16), 32, None, 0, 4,
                                  ctypes.c_void_p(16), ctypes.c_void_p(16), 8, None) == abi.SF_ERR_WORKSPACE
    assert abi.sf_kv_attend_selective(ctypes.byref(kv), 100, ctypes.c_void_p(16), 32, 0, ctypes.c_void_p(16),
                                      None, ctypes.c_void_p(16), None, 0, None) == abi.SF_ERR_INVALID_ARG
    assert abi.sf_stage_refinements_host(None, 16, 4, None, 1, None, None, None) == abi.SF_ERR_INVALID_ARG


def test_ktok_cap_every_attention_entry_point(L):
    """k_tok above 4,096 is refused on the host by every attention call (each
    of a head's 8 cluster CTAs holds at most 512 selected tokens), before any
    launch or workspace lookup; 4,096 itself passes the k_tok check."""
    p16 = ctypes.c_void_p(16)
    kv = abi.sf_kv(1, 8, 128, 8192, 2, 2, 32, 16, 16, 16, 16, 16, 16)
    t = 8000
    assert abi.sf_kv_score_select(ctypes.byref(kv), t, p16, 32, 4097, p16, None, None, None, 0, None) \
        == abi.SF_ERR_UNSUPPORTED
    assert b"4097" in abi.sf_last_error()
    assert abi.sf_kv_attn_refined(ctypes.byref(kv), t, p16, 32, p16, 4097, 0, p16, None, 0, None) \
        == abi.SF_ERR_UNSUPPORTED
    assert abi.sf_kv_attend_selective(ctypes.byref(kv), t, p16, 32, 4097, p16, None, p16, None, 0, None) \
        == abi.SF_ERR_UNSUPPORTED
    assert abi.sf_kv_attend_selective_f16(ctypes.byref(kv), t, p16, 32, 4097, p16, None, p16, None, 0, None) \
        == abi.SF_ERR_UNSUPPORTED
    assert abi.sf_kv_attend_selective_static(ctypes.byref(kv), t, p16, 32, 4097, p16, None, p16, None) \
        == abi.SF_ERR_UNSUPPORTED
    # at the cap the k_tok check passes and the call stops at the missing workspace instead
    assert abi.sf_kv_attend_selective(ctypes.byref(kv), t, p16, 32, 4096, p16, None, p16, None, 0, None) \
        == abi.SF_ERR_WORKSPACE


def test_context_cap(L):
    """t above 262,144 tokens is refused (the selection keeps a bitmap of a
    head's tokens in shared memory); 262,144 itself passes the check and stops
    at the missing workspace."""
    p16 = ctypes.c_void_p(16)
    kv = abi.sf_kv(1, 8, 128, 270000, 2, 2, 32, 16, 16, 16, 16, 16, 16)
    assert abi.sf_kv_attend_selective(ctypes.byref(kv), 262145, p16, 32, 64, p16, None, p16, None, 0, None) \
        == abi.SF_ERR_UNSUPPORTED
    assert abi.sf_kv_attend_selective(ctypes.byref(kv), 262144, p16, 32, 64, p16, None, p16, None, 0, None) \
        == abi.SF_ERR_WORKSPACE


def test_stage_host_index_out_of_range(L):
    """The host-index staging checks every index against n_rows before it enqueues a copy."""
    p16 = ctypes.c_void_p(16)
    sel = (ctypes.c_int32 * 3)(0, 2, 4)
    assert abi.sf_stage_refinements_host(p16, 16, 4, sel, 3, p16, None, None) == abi.SF_ERR_INVALID_ARG
    assert b"outside" in abi.sf_last_error()
    sel = (ctypes.c_int32 * 2)(-1, 2)
    assert abi.sf_stage_refinements_host(p16, 16, 4, sel, 2, p16, None, None) == abi.SF_ERR_INVALID_ARG
    # the device-index form needs a row count
    assert abi.sf_stage_refinements(p16, 16, 0, p16, 2, p16, None, None, None) == abi.SF_ERR_INVALID_ARG


def test_split_gemv_checks(L):
    wq = abi.sf_wq(4096, 4096, 2, 2, 128, 16, 16, 16)
    p16 = ctypes.c_void_p(16)
    # the split form needs a correction, a selection and a separate output
    assert abi.sf_gemv_refined_split(ctypes.byref(wq), p16, 1, 1024, 0, p16, None, p16, p16, None) \
        == abi.SF_ERR_INVALID_ARG
    assert abi.sf_gemv_refined_split(ctypes.byref(wq), p16, 1, 1024, 32, None, None, p16, p16, None) \
        == abi.SF_ERR_INVALID_ARG
    assert abi.sf_gemv_refined_split(ctypes.byref(wq), p16, 1, 1024, 32, p16, None, p16, None, None) \
        == abi.SF_ERR_INVALID_ARG
    assert abi.sf_gemv_refined_split(ctypes.byref(wq), p16, 1, 1024, 32, p16, None, ctypes.c_void_p(4096),
                                     ctypes.c_void_p(4096 + 1024), None) == abi.SF_ERR_INVALID_ARG
    assert b"overlap" in abi.sf_last_error()


def test_decode_step_forms_reject_before_launch(L):
    p16 = ctypes.c_void_p(16)
    kv = abi.sf_kv(1, 8, 128, 8192, 2, 2, 32, 16, 16, 16, 16, 16, 16)
    # the new token's slot must lie inside the cache, h_q a multiple of h_kv, pointers aligned
    assert abi.sf_kv_append_rope(ctypes.byref(kv), p16, 32, 0, 500000.0, 8192, p16, None) == abi.SF_ERR_INVALID_ARG
    assert abi.sf_kv_append_rope(ctypes.byref(kv), p16, 30, 0, 500000.0, 5, p16, None) == abi.SF_ERR_INVALID_ARG
    assert abi.sf_kv_append_rope(ctypes.byref(kv), ctypes.c_void_p(20), 32, 0, 500000.0, 5, p16, None) \
        == abi.SF_ERR_INVALID_ARG
    assert abi.sf_kv_append_rope(ctypes.byref(kv), p16, 32, -1, 500000.0, 5, p16, None) == abi.SF_ERR_INVALID_ARG
    # the fp16-output attention needs its output
    assert abi.sf_kv_attend_selective_f16(ctypes.byref(kv), 100, p16, 32, 8, p16, None, None, p16, 1 << 20,
                                          None) == abi.SF_ERR_INVALID_ARG
    # the correction alone: nothing to do without a selection budget, a selection otherwise
    wq = abi.sf_wq(4096, 4096, 2, 2, 128, 16, 16, 16)
    assert abi.sf_gemv_correction(ctypes.byref(wq), p16, 1, 1024, 0, None, None, p16, None) == 0
    assert abi.sf_gemv_correction(ctypes.byref(wq), p16, 1, 1024, 32, None, None, p16, None) \
        == abi.SF_ERR_INVALID_ARG
    assert abi.sf_gemv_correction(ctypes.byref(wq), p16, 1, 1024, 32, p16, None, None, None) \
        == abi.SF_ERR_INVALID_ARG


def test_fit_refinements_checks(L):
    # every refusal happens on the host, before any launch
    p16 = ctypes.c_void_p(16)
    wq = abi.sf_wq(4096, 4096, 2, 2, 128, 16, 16, 16)
    need = abi.sf_fit_refinements_workspace_bytes(4096, 4096, 512, 1024, 32)
    assert need > 2 * 4096 * 4096 * 8  # the base errors and the fitted corrections, fp64
    assert abi.sf_fit_refinements_workspace_bytes(4096, 4096, 0, 1024, 32) == 0
    fit = lambda **kw: abi.sf_fit_refinements(
        kw.get("wf", p16), ctypes.byref(kw.get("wq", wq)), kw.get("x", p16), kw.get("n_cal", 512),
        kw.get("chunk", 1024), kw.get("kch", 32), ctypes.c_double(kw.get("alpha", 0.01)), None,
        kw.get("ws", p16), kw.get("ws_bytes", need), None)
    assert fit(alpha=0.0) == abi.SF_ERR_INVALID_ARG
    assert fit(alpha=float("nan")) == abi.SF_ERR_INVALID_ARG
    assert fit(n_cal=0) == abi.SF_ERR_INVALID_ARG
    assert fit(wf=None) == abi.SF_ERR_INVALID_ARG
    assert fit(chunk=1000) == abi.SF_ERR_UNSUPPORTED
    assert fit(kch=0) == abi.SF_ERR_INVALID_ARG
    assert fit(ws_bytes=need - 1) == abi.SF_ERR_WORKSPACE
    assert fit(wq=abi.sf_wq(4096, 4096, 2, 2, 128, 16, None, 16)) == abi.SF_ERR_INVALID_ARG  # no refine buffer


def test_logits_cuda_core_form_refusals(L):
    p16 = ctypes.c_void_p(16)
    kv2 = abi.sf_kv(1, 8, 128, 8192, 2, 2, 32, 16, 16, 16, 16, 16, 16)
    kv3 = abi.sf_kv(1, 8, 128, 8192, 3, 2, 32, 16, 16, 16, 16, 16, 16)
    need = abi.sf_kv_logits_fma_workspace_bytes(ctypes.byref(kv2), 4096, 32)
    assert need > 0
    # 3-bit keys and groups of 8 query heads are outside the comparison form
    assert abi.sf_kv_logits_fma(ctypes.byref(kv3), 4096, p16, 32, p16, p16, need, None) == abi.SF_ERR_UNSUPPORTED
    assert abi.sf_kv_logits_fma(ctypes.byref(kv2), 4096, p16, 64, p16, p16, need, None) == abi.SF_ERR_UNSUPPORTED
    assert abi.sf_kv_logits_fma(ctypes.byref(kv2), 4096, p16, 32, None, p16, need, None) == abi.SF_ERR_INVALID_ARG
    assert abi.sf_kv_logits_fma(ctypes.byref(kv2), 4096, p16, 32, p16, p16, need - 1, None) == abi.SF_ERR_WORKSPACE
