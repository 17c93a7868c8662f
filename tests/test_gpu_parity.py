"""Parity of the CUDA path (through the C ABI) with the CPU oracle.

Bar (from the method's pass criteria): packed bytes, codes and channel indices
bit-exact; KV token sets equal except tokens whose oracle score is within 1e-5
(relative) of the k-th score; outputs within relative L2 1e-3, attention also
within max-abs 2e-3.
"""
import numpy as np
import pytest
import torch

import oracle
import ctypes

from bit_decode_selective_b200 import abi, inputs
from bit_decode_selective_b200.ops import KVCache, QuantWeights, _p, select_channels

pytestmark = pytest.mark.gpu

RTOL_L2 = 1e-3
ATTN_MAX_ABS = 2e-3
SEL_RTOL = 1e-5


@pytest.fixture(scope="module", autouse=True)
def dev():
    assert torch.cuda.is_available(), "the gpu tests need a CUDA device"
    oracle.set_threads(0)
    return torch.device("cuda")


def cu(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def host(t):
    return t.cpu().numpy()


def rel_l2(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30))


def f16bits(x):
    return np.ascontiguousarray(x).view(np.uint16)


# ---------------------------------------------------------------------------
# weight packing


def special_weights(rng, n, k):
    w = inputs.weight(rng, n, k)
    w[0, :128] = 0.25                      # constant group: step 0
    w[1, :64] = 0.0
    w[1, 64:128] = -0.0                    # signed zeros
    w[2, 128:256] = rng.normal(0, 30, 128)  # wide range
    w[3, :128] = np.linspace(-1, 1, 128)   # many exact bin edges
    return w


def check_packed(qw, w, b, r, G):
    qb, rho, sz = oracle.quant_weights(w, b, r, G)
    base, refine = oracle.pack_weights(qb, rho, b, r)
    gq, grho = qw.unpack()
    torch.cuda.synchronize()
    assert np.array_equal(host(qw.sz).view(np.uint16).reshape(sz.shape), sz)
    assert np.array_equal(host(gq), qb)
    assert np.array_equal(host(grho), rho)
    assert np.array_equal(host(qw.base), base)
    assert np.array_equal(host(qw.refine), refine)
    return qb, rho, sz


@pytest.mark.parametrize("b,r,G", [(2, 2, 128), (2, 1, 64), (3, 1, 128), (3, 2, 32), (4, 2, 128), (4, 1, 256)])
def test_pack_weights_bit_exact(b, r, G):
    rng = np.random.default_rng(100 + 10 * b + r)
    w = special_weights(rng, 256, 2048)
    qw = QuantWeights.pack(cu(w), b, r, G)
    check_packed(qw, w, b, r, G)


def test_pack_weights_gemv_workload_full_size():
    w, _ = inputs.gemv_case(seed=0)
    qw = QuantWeights.pack(cu(w), 2, 2, 128)
    check_packed(qw, w, 2, 2, 128)


# ---------------------------------------------------------------------------
# channel selection


@pytest.mark.parametrize("chunk,kch", [(1024, 32), (1024, 1), (1024, 1024), (256, 7), (2048, 100), (512, 512)])
def test_select_channels_bit_exact(chunk, kch):
    rng = np.random.default_rng(chunk + kch)
    x = inputs.activation(rng, 4096, batch=3)
    x[0, ::9] = np.float16(1.5)      # ties of both signs
    x[0, 1::13] = np.float16(-1.5)
    x[1, :50] = np.float16(0.0)
    x[1, 50:80] = np.float16(-0.0)
    x[2, :] = np.float16(2.0)        # a row of equal magnitudes
    sel = select_channels(cu(f16bits(x)), chunk, kch)
    torch.cuda.synchronize()
    assert np.array_equal(host(sel), oracle.select_chunks(x, chunk, kch))


# ---------------------------------------------------------------------------
# refined GEMV


def gemv_check(w, x, b, r, G, chunk, kch, staged=False, give_sel=False):
    qb, rho, sz = oracle.quant_weights(w, b, r, G)
    qw = QuantWeights.pack(cu(w), b, r, G)
    xd = cu(f16bits(x))
    sel_o = oracle.select_chunks(x, chunk, kch) if kch else None
    if staged or give_sel:
        sel_d = cu(sel_o)
        rows = qw.refine_rows()[sel_d.view(x.shape[0], -1).long()].contiguous() if staged else None
        y, sel = qw.gemv(xd, chunk, kch, sel_in=sel_d, refine_rows=rows)
    else:
        y, sel = qw.gemv(xd, chunk, kch)
    torch.cuda.synchronize()
    if kch:
        assert np.array_equal(host(sel), sel_o)
    yo = oracle.gemv_refined(qb, rho, sz, r, G, x, sel_o, chunk, kch)
    err = rel_l2(host(y), yo)
    assert err <= RTOL_L2, err
    return err


def fixed_point_bound(qb, rho, sz, r, G, x):
    """Elementwise bound on |y_gpu - y| for the GEMV's arithmetic: the base
    product takes x in fixed point per 64-channel block, x_fix =
    round(x * 2^(19 - ilogb(max |x| of the block))), so each x_c moves by at most
    half a step, 2^(ilogb - 20) (every x_c within 2^9 of the block's largest is
    exact); the correction uses x_c as is.  Plus fp32 rounding of the partial
    sums (a few ulps of the sum of |terms|)."""
    f16 = lambda a: np.asarray(a, np.uint16).view(np.float16).astype(np.float64)
    SQ = np.abs(np.repeat(f16(sz[:, :, 0]), G, axis=1) * qb)   # |s q|, the terms that take x_fix
    M = np.abs(np.repeat(f16(sz[:, :, 1]), G, axis=1))
    xb = x.astype(np.float64).reshape(x.shape[0], -1, 64)
    mx = np.abs(xb).max(-1)
    half = np.where(mx > 0, 2.0 ** (np.floor(np.log2(np.where(mx > 0, mx, 1))) - 20), 0.0)
    h = np.repeat(half, 64, axis=-1)                        # [batch][k]
    ax = np.abs(x.astype(np.float64))
    return SQ @ h.T + 1e-5 * ((SQ + M) @ ax.T)              # [n][batch]


@pytest.mark.parametrize("b,r", [(2, 2), (2, 1), (3, 1), (3, 2), (4, 2)])
@pytest.mark.parametrize("kch", [0, 32, 1024])
def test_gemv_parity(b, r, kch):
    rng = np.random.default_rng(7 * b + r + kch)
    # k = 3072: one full 2048-channel segment plus a half one (ragged lane tail)
    w = inputs.weight(rng, 384, 3072)
    x = inputs.activation(rng, 3072, batch=1)
    gemv_check(w, x, b, r, 128, 1024, kch)
    # elementwise, within the bound the fixed-point activations allow
    qb, rho, sz = oracle.quant_weights(w, b, r, 128)
    qw = QuantWeights.pack(cu(w), b, r, 128)
    y, _ = qw.gemv(cu(f16bits(x)), 1024, kch)
    torch.cuda.synchronize()
    sel_o = oracle.select_chunks(x, 1024, kch) if kch else None
    yo = oracle.gemv_refined(qb, rho, sz, r, 128, x, sel_o, 1024, kch)
    bound = fixed_point_bound(qb, rho, sz, r, 128, x).T
    assert np.all(np.abs(host(y) - yo) <= bound)


@pytest.mark.parametrize("batch", [2, 5])
def test_gemv_batch_and_staged_rows(batch):
    rng = np.random.default_rng(50 + batch)
    w = inputs.weight(rng, 256, 4096)
    x = inputs.activation(rng, 4096, batch=batch)
    gemv_check(w, x, 2, 2, 128, 1024, 32)
    gemv_check(w, x, 2, 2, 128, 1024, 32, give_sel=True)
    gemv_check(w, x, 2, 2, 128, 1024, 32, staged=True)


@pytest.mark.parametrize("b,r,staged", [(2, 2, False), (3, 1, True), (4, 2, False)])
def test_gemv_correction_only_equals_fused(b, r, staged):
    """Fetch-lag form: base product (kch = 0) plus the correction on its own."""
    rng = np.random.default_rng(70 + b)
    w = inputs.weight(rng, 512, 4096)
    x = inputs.activation(rng, 4096, batch=2)
    qb, rho, sz = oracle.quant_weights(w, b, r, 128)
    qw = QuantWeights.pack(cu(w), b, r, 128)
    xd = cu(f16bits(x))
    sel_o = oracle.select_chunks(x, 1024, 32)
    sel_d = cu(sel_o)
    rows = qw.refine_rows()[sel_d.view(2, -1).long()].contiguous() if staged else None
    y, _ = qw.gemv(xd, 1024, 0)
    qw.correction(xd, sel_d, y, 1024, 32, refine_rows=rows)
    torch.cuda.synchronize()
    yo = oracle.gemv_refined(qb, rho, sz, r, 128, x, sel_o, 1024, 32)
    assert rel_l2(host(y), yo) < 1e-5


@pytest.mark.parametrize("b,r,staged,n", [(2, 2, True, 6144), (3, 1, False, 512), (4, 2, True, 1152)])
def test_gemv_split_outputs(b, r, staged, n):
    """Base product and correction to separate outputs in one launch: the base
    against the oracle's kch = 0 product, the correction against the oracle's
    correction on its own (6,144 rows: 1,536 four-row units over the 148-CTA
    grid, ragged; 1,152 rows: 288 units, most CTAs two, some one)."""
    rng = np.random.default_rng(90 + b + n)
    w = inputs.weight(rng, n, 4096)
    x = inputs.activation(rng, 4096, batch=2)
    qb, rho, sz = oracle.quant_weights(w, b, r, 128)
    qw = QuantWeights.pack(cu(w), b, r, 128)
    xd = cu(f16bits(x))
    sel_o = oracle.select_chunks(x, 1024, 32)
    sel_d = cu(sel_o)
    rows = qw.refine_rows()[sel_d.view(2, -1).long()].contiguous() if staged else None
    yb, yc = qw.gemv_split(xd, sel_d, 1024, 32, refine_rows=rows)
    torch.cuda.synchronize()
    base_o = oracle.gemv_refined(qb, rho, sz, r, 128, x, None, 1024, 0)
    assert rel_l2(host(yb), base_o) < 1e-5
    for bb in range(2):
        corr_o = oracle.gemv_correction(qb, rho, sz, r, 128, x[bb], sel_o[bb])
        assert rel_l2(host(yc)[bb], corr_o) < 1e-5


@pytest.mark.parametrize("G", [32, 64, 256])
def test_gemv_group_sizes(G):
    rng = np.random.default_rng(G)
    w = inputs.weight(rng, 128, 1024)
    x = inputs.activation(rng, 1024)
    gemv_check(w, x, 3, 2, G, 1024, 16)
    gemv_check(w, x, 2, 2, G, 256, 5)


def test_gemv_single_workload_full_size():
    """4096 x 4096, 2-bit base + 2 refinement bits, k = 32 per 1,024 (seed 0)."""
    w, x = inputs.gemv_case(seed=0)
    gemv_check(w, x, 2, 2, 128, 1024, 32)


def test_gemv_layer_workload_full_size():
    """One Llama-3.1-8B-shaped layer's projections, 3-bit base + 1 refinement bit."""
    for name, (w, x) in inputs.layer_case(seed=1).items():
        gemv_check(w, x, 3, 1, 128, 1024, 32)


# ---------------------------------------------------------------------------
# KV cache


def kv_setup(T, b=2, r=2, t_max=None, seed=2, batch=1, h_kv=8, h_q=32, split_pack=False):
    k, v, q = inputs.kv_case(seed=seed, t=T, h_kv=h_kv, h_q=h_q, batch=batch)
    t_max = t_max or ((T + 15) // 16) * 16
    cache = KVCache(batch, h_kv, t_max, b, r)
    if split_pack and T > 1:
        h = T // 2
        cache.pack_tokens(cu(f16bits(k[:, :, :h])), cu(f16bits(v[:, :, :h])), 0)
        cache.pack_tokens(cu(f16bits(k[:, :, h:])), cu(f16bits(v[:, :, h:])), h)
    else:
        cache.pack_tokens(cu(f16bits(k)), cu(f16bits(v)), 0)
    kc = oracle.quant_kv(k, b, r)
    vc = oracle.quant_kv(v, b, r)
    return cache, kc, vc, q


def check_selection(sel, score, k_tok):
    B, H, T = score.shape
    for bb in range(B):
        for g in range(H):
            s = sel[bb, g]
            assert len(s) == k_tok and np.all(np.diff(s) > 0) and s[0] >= 0 and s[-1] < T
            order = np.lexsort((np.arange(T), -score[bb, g]))
            kth = score[bb, g, order[k_tok - 1]]
            diff = set(s.tolist()) ^ set(order[:k_tok].tolist())
            for t in diff:
                assert abs(score[bb, g, t] - kth) <= SEL_RTOL * kth, (bb, g, t, score[bb, g, t], kth)


@pytest.mark.parametrize("b,r", [(2, 2), (2, 1), (3, 2), (3, 1), (4, 2), (4, 1)])
def test_kv_pack_bit_exact(b, r):
    cache, kc, vc, q = kv_setup(37, b, r, t_max=48, split_pack=True, batch=2, h_kv=2, h_q=8)
    torch.cuda.synchronize()
    for which, (qb, rho, sz) in ((0, kc), (1, vc)):
        gq, grho = cache.unpack(which, 37)
        assert np.array_equal(host(gq), qb) and np.array_equal(host(grho), rho)
        gsz = host(cache.ksz if which == 0 else cache.vsz).view(np.uint16).reshape(2, 2, 48, 4, 2)[:, :, :37]
        assert np.array_equal(gsz, sz)
        base, refine = oracle.pack_kv(qb, rho, which, b, r, t_max=48)
        # the cache buffers start zeroed, so unwritten slots compare equal too
        assert np.array_equal(host(cache.kb if which == 0 else cache.vb), base)
        assert np.array_equal(host(cache.kr if which == 0 else cache.vr), refine)


def kv_parity(T, k_tok, splits=(0,), b=2, r=2, batch=1, h_kv=8, h_q=32, seed=2):
    cache, kc, vc, q = kv_setup(T, b, r, batch=batch, h_kv=h_kv, h_q=h_q, seed=seed)
    qd = cu(f16bits(q))
    sel, logits, scores = cache.score_select(qd, T, k_tok, want_scores=True)
    torch.cuda.synchronize()
    lo = oracle.kv_logits(kc[0], kc[2], q)
    assert rel_l2(host(logits), lo) < 1e-5
    so = oracle.kv_scores(lo, h_kv)
    assert rel_l2(host(scores), so) < 1e-5
    gsel = host(sel)
    check_selection(gsel, so, k_tok)
    ref = oracle.kv_attention(kc, vc, q, gsel, k_tok, r)
    for ns in splits:
        out = cache.attn_refined(qd, T, sel, k_tok, n_splits=ns)
        torch.cuda.synchronize()
        o = host(out)
        assert rel_l2(o, ref) <= RTOL_L2
        assert np.abs(o - ref).max() <= ATTN_MAX_ABS
    # the fused score-select-attend call: same selection, same output
    lg2 = torch.empty_like(logits)
    out2, sel2 = cache.attend_selective(qd, T, k_tok, logits=lg2)
    torch.cuda.synchronize()
    assert np.array_equal(host(sel2), gsel)
    assert np.array_equal(host(lg2), host(logits))
    o2 = host(out2)
    assert rel_l2(o2, ref) <= RTOL_L2 and np.abs(o2 - ref).max() <= ATTN_MAX_ABS
    return cache, kc, vc, q, qd


@pytest.mark.parametrize("T,k_tok", [(1, 1), (37, 1), (37, 37), (100, 10), (1000, 64), (2049, 300)])
def test_kv_parity_small(T, k_tok):
    kv_parity(T, k_tok, splits=(0, 1, 7))


def test_kv_parity_batch_and_head_groups():
    kv_parity(777, 50, splits=(0, 3), batch=2, h_kv=4, h_q=32, seed=9)   # 8 query heads per KV head
    kv_parity(500, 20, splits=(0,), b=4, r=1, h_kv=2, h_q=4, seed=10)    # 2 per KV head, 4-bit base
    kv_parity(300, 30, splits=(0, 5), h_kv=4, h_q=4, seed=12)            # 1 per KV head
    # 3 caches x 8 heads x 16 refinement CTAs: more than one wave, two CTAs per SM
    kv_parity(2000, 512, splits=(0,), batch=3, h_kv=8, h_q=32, seed=13)


@pytest.mark.parametrize("T,k_tok,r,batch,h_kv,h_q,seed", [
    (37, 5, 2, 1, 8, 32, 20),      # one partial tile, 4 query heads per KV head
    (1000, 64, 2, 2, 4, 32, 21),   # 8 per KV head, two caches
    (2049, 300, 1, 1, 2, 4, 22),   # ragged last tile, 2 per KV head, 1 refinement bit
])
def test_kv_parity_3bit_base(T, k_tok, r, batch, h_kv, h_q, seed):
    kv_parity(T, k_tok, splits=(0, 3), b=3, r=r, batch=batch, h_kv=h_kv, h_q=h_q, seed=seed)


@pytest.mark.parametrize("T,batch,h_kv,h_q", [(37, 1, 8, 32), (2049, 2, 4, 16), (32768, 1, 8, 32)])
def test_kv_logits_cuda_core_form(T, batch, h_kv, h_q):
    # the CUDA-core form of the key contraction: the oracle's logits, and the
    # tensor-core form's within fp32 summation order
    cache, kc, vc, q = kv_setup(T, 2, 2, batch=batch, h_kv=h_kv, h_q=h_q, seed=14)
    qd = cu(f16bits(q))
    lf = cache.logits_fma(qd, T)
    _, lt, _ = cache.score_select(qd, T, 1)
    torch.cuda.synchronize()
    lo = oracle.kv_logits(kc[0], kc[2], q)
    assert rel_l2(host(lf), lo) < 1e-5
    assert np.abs(host(lf) - host(lt)).max() <= 1e-4 * np.abs(lo).max()


def test_kv_base_only_and_all_selected():
    cache, kc, vc, q = kv_setup(300, batch=1, h_kv=8, h_q=32, seed=11)
    qd = cu(f16bits(q))
    out0 = cache.attn_refined(qd, 300, None, 0)
    all_sel = torch.arange(300, dtype=torch.int32, device="cuda").repeat(1, 8, 1).contiguous()
    outT = cache.attn_refined(qd, 300, all_sel, 300)
    torch.cuda.synchronize()
    ref0 = oracle.kv_attention(kc, vc, q, None, 0, 2)
    refT = oracle.kv_attention(kc, vc, q, host(all_sel), 300, 2)
    assert np.abs(host(out0) - ref0).max() <= ATTN_MAX_ABS and rel_l2(host(out0), ref0) <= RTOL_L2
    assert np.abs(host(outT) - refT).max() <= ATTN_MAX_ABS and rel_l2(host(outT), refT) <= RTOL_L2


@pytest.mark.parametrize("b,r,batch,t", [(2, 2, 1, 37), (4, 1, 2, 0), (2, 1, 3, 47), (3, 2, 2, 21)])
def test_kv_append_rope_equals_rope_then_pack(b, r, batch, t):
    """The fused rotary embedding + append of the decode step's token stores
    the same codes, refinements and steps/offsets, and the same rotated q, as
    the rotary embedding followed by the token pack (bit-exact)."""
    h_q, h_kv, theta, pos = 32, 8, 500000.0, 32768 + t
    rng = np.random.default_rng(300 + 10 * b + batch)
    qkv = cu((rng.standard_normal((batch, (h_q + 2 * h_kv) * 128)) * 3).astype(np.float32))
    s = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    c1, c2 = KVCache(batch, h_kv, 48, b, r), KVCache(batch, h_kv, 48, b, r)
    q1 = torch.empty((batch, h_q, 128), dtype=torch.float16, device="cuda")
    k1 = torch.empty((batch, h_kv, 1, 128), dtype=torch.float16, device="cuda")
    v1 = torch.empty_like(k1)
    abi.check(abi.sf_rope_split(_p(qkv), batch, h_q, h_kv, 128, pos, theta, _p(q1), _p(k1), _p(v1), s),
              "sf_rope_split")
    abi.check(abi.sf_kv_pack_tokens(ctypes.byref(c1.desc), _p(k1), _p(v1), t, 1, s), "sf_kv_pack_tokens")
    q2 = torch.empty_like(q1)
    abi.check(abi.sf_kv_append_rope(ctypes.byref(c2.desc), _p(qkv), h_q, pos, theta, t, _p(q2), s),
              "sf_kv_append_rope")
    torch.cuda.synchronize()
    assert torch.equal(q1.view(torch.int16), q2.view(torch.int16))
    for name in ("kb", "kr", "vb", "vr", "ksz", "vsz"):
        assert torch.equal(getattr(c1, name), getattr(c2, name)), name
    assert getattr(c2, "ksz").abs().sum().item() > 0  # the token was written


def test_kv_attend_selective_f16_output():
    """The fp16-output form equals the fp32 output rounded to fp16 (same kernels)."""
    T, k_tok = 3000, 128
    k, v, _ = inputs.kv_case(seed=31, t=T)
    cache = KVCache(1, 8, (T + 15) // 16 * 16)
    cache.pack_tokens(cu(f16bits(k)), cu(f16bits(v)), 0)
    q = cu(f16bits(inputs.query(np.random.default_rng(32), 32, 128, 1)))
    s = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    need = abi.sf_kv_attend_selective_workspace_bytes(ctypes.byref(cache.desc), T, 32, k_tok, 0)
    ws = torch.empty(max(need, 16), dtype=torch.uint8, device="cuda")
    sel = torch.empty((1, 8, k_tok), dtype=torch.int32, device="cuda")
    out = torch.empty((1, 32, 128), dtype=torch.float32, device="cuda")
    out16 = torch.empty((1, 32, 128), dtype=torch.float16, device="cuda")
    abi.check(abi.sf_kv_attend_selective(ctypes.byref(cache.desc), T, _p(q), 32, k_tok, _p(sel), None, _p(out),
                                         _p(ws), ws.numel(), s), "sf_kv_attend_selective")
    abi.check(abi.sf_kv_attend_selective_f16(ctypes.byref(cache.desc), T, _p(q), 32, k_tok, _p(sel), None,
                                             _p(out16), _p(ws), ws.numel(), s), "sf_kv_attend_selective_f16")
    torch.cuda.synchronize()
    assert torch.equal(out.half().view(torch.int16), out16.view(torch.int16))


def test_kv_attention_8k_workload():
    """32 query / 8 KV heads, d 128, T = 8,192, 2+2 bits, top-256 tokens per KV head."""
    kv_parity(8192, 256, splits=(0, 1, 7), seed=2)


def test_kv_attention_128k_workload():
    """T = 131,072, top-1,024 tokens per KV head, split-K merged by log-sum-exp."""
    kv_parity(131072, 1024, splits=(0,), seed=3)


def test_kv_attention_3bit_32k_workload():
    """The benchmarked 3-bit base: T = 32,768, 3+2 bits, top-512 tokens per KV head."""
    kv_parity(32768, 512, splits=(0,), b=3, r=2, seed=6)


# ---------------------------------------------------------------------------
# decoder glue


@pytest.mark.parametrize("n,adds", [(4096, 2), (8192, 1), (14336, 0), (1000, 2), (20000, 1)])
def test_rmsnorm_residual(n, adds):
    """h += add0 + add1 in fp32 (bit-exact with the same fp32 sums) and x =
    fp16(h / rms(h)) within one fp16 step of the oracle's fp64 RMSNorm of the
    same h (n = 1,000 and 20,000 take the looping kernel, the others the
    register-resident one)."""
    batch = 2
    rng = np.random.default_rng(400 + n + adds)
    h0 = (rng.standard_normal((batch, n)) * 3).astype(np.float32)
    a0 = (rng.standard_normal((batch, n))).astype(np.float32)
    a1 = (rng.standard_normal((batch, n)) * 0.5).astype(np.float32)
    h = cu(h0)
    x = torch.empty((batch, n), dtype=torch.float16, device="cuda")
    d0, d1 = (cu(a0) if adds >= 1 else None), (cu(a1) if adds >= 2 else None)
    s = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    abi.check(abi.sf_rmsnorm_residual(_p(h), _p(d0), _p(d1), batch, n, 1e-5, _p(x), s), "sf_rmsnorm_residual")
    torch.cuda.synchronize()
    want_h = h0.copy()
    if adds >= 1:
        want_h = want_h + a0
    if adds >= 2:
        want_h = want_h + a1
    assert np.array_equal(host(h), want_h)
    for b in range(batch):
        ref = oracle.rmsnorm_f16(want_h[b].astype(np.float64)).view(np.float16).astype(np.float64)
        got = host(x)[b].astype(np.float64)
        assert np.all(np.abs(got - ref) <= np.abs(ref) * 2.0 ** -10 + 2.0 ** -24)


# ---------------------------------------------------------------------------
# refinement staging


@pytest.mark.parametrize("rows,row_bytes,n_sel", [(4096, 7168, 128), (14336, 1024, 448), (1024, 16, 1000),
                                                  (512, 1536, 3)])
def test_stage_refinements_bit_exact(rows, row_bytes, n_sel):
    """Rows named by a device index array, read from mapped pinned host memory,
    land in order in the device slot (duplicates and unsorted indices too);
    the host-index form (one copy per run of consecutive rows) gives the same."""
    rng = np.random.default_rng(rows + n_sel)
    host_rows = torch.from_numpy(rng.integers(0, 256, rows * row_bytes, dtype=np.uint8)).pin_memory()
    sel_h = rng.integers(0, rows, n_sel).astype(np.int32)
    sel_h[: n_sel // 2] = np.sort(sel_h[: n_sel // 2])  # runs of consecutive rows for the host form
    sel = cu(sel_h)
    dst = torch.empty(n_sel * row_bytes, dtype=torch.uint8, device="cuda")
    s = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    bad = torch.zeros(4, dtype=torch.int32, device="cuda")
    abi.check(abi.sf_stage_refinements(ctypes.c_void_p(host_rows.data_ptr()), row_bytes, rows, _p(sel), n_sel,
                                       _p(dst), _p(bad), s, None), "sf_stage_refinements")
    dst2 = torch.empty_like(dst)
    sel_c = np.ascontiguousarray(sel_h)
    abi.check(abi.sf_stage_refinements_host(ctypes.c_void_p(host_rows.data_ptr()), row_bytes, rows,
                                            sel_c.ctypes.data_as(ctypes.c_void_p), n_sel, _p(dst2), s, None),
              "sf_stage_refinements_host")
    torch.cuda.synchronize()
    want = host_rows.view(rows, row_bytes)[torch.from_numpy(sel_h).long()].reshape(-1)
    assert torch.equal(dst.cpu(), want)
    assert torch.equal(dst2.cpu(), want)
    assert bad[0].item() == 0


def test_stage_refinements_out_of_range_index():
    """Indices outside [0, n_rows) in the device array are not read: their rows
    are zero-filled and counted in the error word; the valid ones still land."""
    rows, row_bytes = 64, 256
    rng = np.random.default_rng(5)
    host_rows = torch.from_numpy(rng.integers(1, 256, rows * row_bytes, dtype=np.uint8)).pin_memory()
    sel_h = np.array([3, 64, 10, -1, 63, 1 << 30], dtype=np.int32)
    dst = torch.full((len(sel_h) * row_bytes,), 7, dtype=torch.uint8, device="cuda")
    bad = torch.zeros(4, dtype=torch.int32, device="cuda")
    s = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    abi.check(abi.sf_stage_refinements(ctypes.c_void_p(host_rows.data_ptr()), row_bytes, rows, _p(cu(sel_h)),
                                       len(sel_h), _p(dst), _p(bad), s, None), "sf_stage_refinements")
    torch.cuda.synchronize()
    got = dst.cpu().view(len(sel_h), row_bytes)
    src = host_rows.view(rows, row_bytes)
    for j, i in enumerate(sel_h):
        if 0 <= i < rows:
            assert torch.equal(got[j], src[i])
        else:
            assert int(got[j].sum()) == 0
    assert bad[0].item() == 3


# ---------------------------------------------------------------------------
# refinement rows cached across steps


class CachePolicy:
    """The row cache's replacement rule, restated: a selected channel the cache
    holds is a hit (its slot is marked used in this step); each missing channel,
    in entry order, takes the next slot not used in this step, in clock order
    from the hand, and the hand moves past the last slot taken."""

    def __init__(self, cap):
        self.cap, self.slot_of, self.channel_of = cap, {}, [-1] * cap
        self.stamp, self.now, self.hand = [0] * cap, 0, 0

    def call(self, sel):
        self.now += 1
        hit = [c in self.slot_of for c in sel]
        for c, h in zip(sel, hit):
            if h:
                self.stamp[self.slot_of[c]] = self.now
        free = [(self.hand + i) % self.cap for i in range(self.cap)
                if self.stamp[(self.hand + i) % self.cap] != self.now]
        misses = [c for c, h in zip(sel, hit) if not h]
        for c, v in zip(misses, free):
            old = self.channel_of[v]
            if old >= 0:
                del self.slot_of[old]
            self.channel_of[v], self.slot_of[c], self.stamp[v] = c, v, self.now
        if misses:
            self.hand = (free[len(misses) - 1] + 1) % self.cap
        return hit


def make_caches(batch, cap, n_ch, row_bytes, n_sel):
    i32 = lambda n: torch.empty(n, dtype=torch.int32, device="cuda")
    arr = (abi.sf_row_cache * batch)()
    keep = []
    s = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for b in range(batch):
        t = dict(slot_of=i32(n_ch), channel_of=i32(cap), stamp=i32(cap), state=i32(4), work=i32(n_sel),
                 rows=torch.empty(cap * row_bytes, dtype=torch.uint8, device="cuda"))
        keep.append(t)
        arr[b] = abi.sf_row_cache(cap, n_ch, row_bytes, t["slot_of"].data_ptr(), t["channel_of"].data_ptr(),
                                  t["stamp"].data_ptr(), t["state"].data_ptr(), t["work"].data_ptr(), n_sel,
                                  t["rows"].data_ptr())
        abi.check(abi.sf_row_cache_reset(ctypes.byref(arr[b]), s), "sf_row_cache_reset")
    return arr, keep


@pytest.mark.parametrize("skip", [0, 1])
def test_stage_refinements_cached(skip):
    """Six steps of selections that partly repeat, two batch rows with a cache
    each: staged rows equal the host rows of the entries the GEMV will refine;
    hits and misses follow the replacement rule exactly; with skip, missing
    channels are marked -1 - c in the effective selection and their rows are in
    the cache (a hit) when the same channel comes again."""
    n_ch, row_bytes, n_sel, cap, batch = 1000, 256, 64, 96, 2
    rng = np.random.default_rng(80 + skip)
    host_rows = torch.from_numpy(rng.integers(0, 256, n_ch * row_bytes, dtype=np.uint8)).pin_memory()
    src = host_rows.view(n_ch, row_bytes)
    arr, keep = make_caches(batch, cap, n_ch, row_bytes, n_sel)
    models = [CachePolicy(cap) for _ in range(batch)]
    prev = [rng.choice(n_ch, n_sel, replace=False) for _ in range(batch)]
    dst = torch.empty(batch * n_sel * row_bytes, dtype=torch.uint8, device="cuda")
    eff = torch.empty((batch, n_sel), dtype=torch.int32, device="cuda")
    s = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for step in range(6):
        sels = []
        for b in range(batch):
            keepn = int(rng.integers(0, n_sel + 1))
            old = rng.permutation(prev[b])[:keepn]
            pool = np.setdiff1d(np.arange(n_ch), old)
            sels.append(np.concatenate([old, rng.choice(pool, n_sel - keepn, replace=False)]).astype(np.int32))
        prev = sels
        sel_d = cu(np.stack(sels))
        dst.fill_(0)
        abi.check(abi.sf_stage_refinements_cached(ctypes.c_void_p(host_rows.data_ptr()), row_bytes, n_ch,
                                                  _p(sel_d), n_sel, batch, arr, skip, _p(dst), _p(eff), s, None),
                  "sf_stage_refinements_cached")
        torch.cuda.synchronize()
        got = dst.cpu().view(batch, n_sel, row_bytes)
        e = host(eff)
        for b in range(batch):
            hit = models[b].call(sels[b].tolist())
            for j, c in enumerate(sels[b]):
                if skip and not hit[j]:
                    assert e[b, j] == -1 - c
                else:
                    assert e[b, j] == c
                    assert torch.equal(got[b, j], src[c]), (step, b, j)
            st = host(keep[b]["state"]).view(np.uint32)
            assert st[0] == step + 1
    # every cached slot holds its channel's row
    for b in range(batch):
        ch = host(keep[b]["channel_of"])
        rows = keep[b]["rows"].cpu().view(cap, row_bytes)
        for slot in range(cap):
            if ch[slot] >= 0:
                assert torch.equal(rows[slot], src[ch[slot]])


def test_gemv_skipped_entries_get_no_correction():
    """An entry -1 - c of the selection leaves channel c at base precision: the
    GEMV equals the base product plus the correction of the other entries."""
    rng = np.random.default_rng(91)
    w = inputs.weight(rng, 512, 4096)
    x = inputs.activation(rng, 4096, batch=1)
    qb, rho, sz = oracle.quant_weights(w, 2, 2, 128)
    qw = QuantWeights.pack(cu(w), 2, 2, 128)
    sel_o = oracle.select_chunks(x, 1024, 32)
    flat = sel_o.reshape(-1).copy()
    skip = rng.random(flat.size) < 0.4
    eff = np.where(skip, -1 - flat, flat).astype(np.int32).reshape(sel_o.shape)
    rows = qw.refine_rows()[cu(flat).long()].contiguous()
    y, _ = qw.gemv(cu(f16bits(x)), 1024, 32, sel_in=cu(eff), refine_rows=rows)
    yb, yc = qw.gemv_split(cu(f16bits(x)), cu(eff), 1024, 32, refine_rows=rows)
    y2 = torch.zeros_like(y)
    qw.correction(cu(f16bits(x)), cu(eff), y2, 1024, 32, refine_rows=rows)
    torch.cuda.synchronize()
    base = oracle.gemv_refined(qb, rho, sz, 2, 128, x, None, 1024, 0)
    corr = oracle.gemv_correction(qb, rho, sz, 2, 128, x[0], flat[~skip])
    assert rel_l2(host(y)[0], base[0] + corr) < 1e-5
    assert rel_l2(host(yc)[0], corr) < 1e-5
    assert rel_l2(host(y2)[0], corr) < 1e-5
