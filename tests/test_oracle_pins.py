"""Pins of the CPU oracle against what the pages and the mathematics fix.

Each test checks the oracle against something other than itself: values the
explainer page works out, closed forms, invariants of nested quantisation,
brute force on tiny inputs, and textbook routines (numpy's fp16 cast, dense
matrix-vector products, softmax attention).  A dropped term, a wrong sign or
index, or a transposed operand in the oracle fails at least one of them.

Source pages: "StrataFlux -- Selective precision streaming -- What does it
mean?" (nested-quantization, which-tiles-count and worked-example paragraphs).
"""
import math

import numpy as np
import pytest

from conftest import read_golden
from bit_decode_selective_b200 import bytemodel


def f16(bits):
    return np.asarray(bits, np.uint16).view(np.float16).astype(np.float64)


# ---------------------------------------------------------------------------
# IEEE binary16 conversion: exhaustive against numpy's cast


def test_f16_decode_all_patterns(orc):
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = bits.view(np.float16).astype(np.float64)
    got = np.array([orc.f16_to_f64(int(b)) for b in bits])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])
    # sign of zero
    assert math.copysign(1.0, orc.f16_to_f64(0x8000)) == -1.0


def test_f16_encode_roundtrip_and_midpoints(orc):
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    vals = bits.view(np.float16).astype(np.float64)
    finite = np.isfinite(vals)
    for b, v in zip(bits[finite], vals[finite]):
        assert orc.f16_from_f64(float(v)) == int(b)
    # midpoints between consecutive finite positive values (ties -> even) and
    # points a hair either side of each midpoint
    pos = np.sort(np.unique(vals[finite & (vals >= 0)]))
    mids = (pos[:-1] + pos[1:]) / 2
    with np.errstate(over="ignore"):
        for m in mids:
            for x in (m, np.nextafter(m, 0.0), np.nextafter(m, np.inf)):
                assert orc.f16_from_f64(float(x)) == int(np.float64(x).astype(np.float16).view(np.uint16))
                assert orc.f16_from_f64(float(-x)) == int(np.float64(-x).astype(np.float16).view(np.uint16))
        # overflow boundary: 65504 + 16 ties to the even neighbour 2^16 = inf
        for x in (65504.0, 65519.99, 65520.0, 1e6):
            assert orc.f16_from_f64(x) == int(np.float64(x).astype(np.float16).view(np.uint16))


def test_f16_encode_random_doubles(orc):
    rng = np.random.default_rng(7)
    xs = np.concatenate([rng.normal(0, 1, 20000), rng.normal(0, 1e-5, 5000),
                         rng.uniform(-7e4, 7e4, 5000), rng.normal(0, 1e-7, 5000)])
    with np.errstate(over="ignore"):
        ref = xs.astype(np.float16).view(np.uint16)
    for x, r in zip(xs, ref):
        assert orc.f16_from_f64(float(x)) == int(r)


# ---------------------------------------------------------------------------
# nested quantisation of a group


def test_nested_worked_example(orc):
    """Page values: 2-bit base, 2 fetched bits split each of the 4 bins into 4."""
    rows = read_golden("nested_2bit_plus_2.txt")
    w = np.array([float(r[0]) for r in rows])
    s, m, qb, rho = orc.quant_group(w, 2, 2)
    assert f16(s) == 1.0 and f16(m) == 0.0
    for i, r in enumerate(rows):
        assert qb[i] == int(r[1]) and rho[i] == int(r[2]), (r, qb[i], rho[i])
        assert orc.dequant_base(s, m, int(qb[i])) == float(r[3])
        assert orc.dequant_refined(s, m, int(qb[i]), int(rho[i]), 2) == float(r[4])


@pytest.mark.parametrize("b,r", [(2, 1), (2, 2), (3, 1), (3, 2), (4, 1), (4, 2)])
def test_nested_levels_closed_form(orc, b, r):
    """2^(b+r) refined levels, equally spaced by s/2^r; each base level is the
    mean of its 2^r sub-levels (the 4 x 4 subdivision of the explainer)."""
    s, m = 0x3A00, 0xB800  # 0.75, -0.5
    S, M = f16(s), f16(m)
    levels = []
    for q in range(1 << b):
        sub = [orc.dequant_refined(s, m, q, p, r) for p in range(1 << r)]
        assert np.isclose(np.mean(sub), orc.dequant_base(s, m, q), rtol=0, atol=1e-15)
        levels += sub
    levels = np.array(levels)
    assert len(levels) == 1 << (b + r)
    assert np.allclose(np.diff(levels), S / (1 << r), rtol=0, atol=1e-15)
    # the fine grid is the (b+r)-bit grid with step S/2^r and offset M + S(1-2^r)/2^(r+1)
    M2 = M + S * (1 - (1 << r)) / (1 << (r + 1))
    assert np.allclose(levels, M2 + (S / (1 << r)) * np.arange(1 << (b + r)), rtol=0, atol=1e-15)


@pytest.mark.parametrize("b,r", [(2, 1), (2, 2), (3, 1), (3, 2), (4, 1), (4, 2)])
def test_nested_equals_direct_fine_quantisation(orc, b, r):
    """Invariant: (base code, refinement) concatenated equals direct (b+r)-bit
    round-to-nearest on the same step and offset (S' = S/2^r,
    M' = M + S(1-2^r)/2^(r+1)), computed here as a separate procedure."""
    rng = np.random.default_rng(11 + 10 * b + r)
    near_boundary = 0
    for trial in range(400):
        w = rng.normal(0, rng.uniform(0.01, 3), size=128) + rng.normal(0, 1)
        s, m, qb, rho = orc.quant_group(w, b, r)
        S, M = f16(s), f16(m)
        S2 = S / (1 << r)
        M2 = M + S * (1 - (1 << r)) / (1 << (r + 1))
        arg = (w - M2) / S2 + 0.5
        frac = arg - np.floor(arg)
        ok = (frac > 1e-12) & (frac < 1 - 1e-12)
        near_boundary += int((~ok).sum())
        direct = np.clip(np.floor(arg), 0, (1 << (b + r)) - 1).astype(int)
        both = (qb.astype(int) << r) | rho.astype(int)
        assert np.array_equal(both[ok], direct[ok])
        # base code alone is ordinary b-bit round-to-nearest
        base = np.clip(np.floor((w - M) / S + 0.5), 0, (1 << b) - 1).astype(int)
        fb = (w - M) / S + 0.5
        okb = np.abs(fb - np.round(fb)) > 1e-12
        assert np.array_equal(qb.astype(int)[okb], base[okb])
    assert near_boundary == 0


@pytest.mark.parametrize("b,r", [(2, 2), (3, 1), (4, 2)])
def test_nested_brute_force_nearest(orc, b, r):
    """Brute force on tiny groups: the base code is a nearest base level over all
    2^b levels, and the refinement picks a nearest sub-level among the 2^r
    children of that base code."""
    rng = np.random.default_rng(5 + b)
    for trial in range(300):
        w = rng.normal(0, 1, size=rng.integers(2, 9))
        s, m, qb, rho = orc.quant_group(w, b, r)
        for i, wi in enumerate(w):
            dist_base = [abs(wi - orc.dequant_base(s, m, q)) for q in range(1 << b)]
            assert abs(wi - orc.dequant_base(s, m, int(qb[i]))) <= min(dist_base) + 1e-12
            dist_sub = [abs(wi - orc.dequant_refined(s, m, int(qb[i]), p, r)) for p in range(1 << r)]
            assert abs(wi - orc.dequant_refined(s, m, int(qb[i]), int(rho[i]), r)) <= min(dist_sub) + 1e-12
            # the refined error is at most half a sub-bin (the group's extremes
            # may sit up to one fp16 rounding of the step outside the grid)
            S = f16(s)
            assert abs(wi - orc.dequant_refined(s, m, int(qb[i]), int(rho[i]), r)) <= \
                S / (2 << r) + 4e-3 * S + 1e-12


def test_nested_scale_offset_and_degenerate(orc):
    w = np.array([0.1, -0.7, 0.35, 1.9, 0.0])
    s, m, qb, rho = orc.quant_group(w, 3, 2)
    # step and offset are the fp16 roundings of (hi - lo)/(2^b - 1) and lo
    assert s == int(np.float16((1.9 + 0.7) / 7).view(np.uint16))
    assert m == int(np.float16(-0.7).view(np.uint16))
    assert qb[1] == 0 and qb[3] == 7
    # constant group: step rounds to zero, every code 0, value = offset
    s, m, qb, rho = orc.quant_group(np.full(32, 0.3), 2, 2)
    assert s == 0 and (qb == 0).all() and (rho == 0).all()
    assert orc.dequant_base(s, m, 0) == f16(m) == orc.dequant_refined(s, m, 0, 0, 2) + f16(s)
    # range too small for an fp16 step: also all zero
    s, m, qb, rho = orc.quant_group(np.array([1.0, 1.0 + 1e-9]), 2, 2)
    assert s == 0 and (qb == 0).all()


def test_quant_weights_rows_and_groups(orc):
    """Row/group addressing of the matrix quantiser against per-group calls."""
    rng = np.random.default_rng(3)
    W = rng.normal(0, 0.02, (8, 512)).astype(np.float32)
    qb, rho, sz = orc.quant_weights(W, 3, 1, 128)
    for n in (0, 5, 7):
        for j in (0, 3):
            s, m, q1, r1 = orc.quant_group(W[n, j * 128:(j + 1) * 128].astype(np.float64), 3, 1)
            assert (s, m) == (sz[n, j, 0], sz[n, j, 1])
            assert np.array_equal(q1, qb[n, j * 128:(j + 1) * 128])
            assert np.array_equal(r1, rho[n, j * 128:(j + 1) * 128])


def test_quant_kv_addressing(orc):
    rng = np.random.default_rng(4)
    x = rng.normal(0, 1, (2, 3, 5, 64)).astype(np.float16)
    qb, rho, sz = orc.quant_kv(x, 2, 2, 32)
    s, m, q1, r1 = orc.quant_group(x[1, 2, 4, 32:64].astype(np.float64), 2, 2)
    assert (s, m) == (sz[1, 2, 4, 1, 0], sz[1, 2, 4, 1, 1])
    assert np.array_equal(q1, qb[1, 2, 4, 32:64]) and np.array_equal(r1, rho[1, 2, 4, 32:64])


# ---------------------------------------------------------------------------
# packed formats (this project's definition, pinned by hand-computed bytes)


def test_pack_weights_2bit_by_hand(orc):
    N, K = 64, 1024  # 256 bytes per row: 16 units of 16 bytes
    qb = np.repeat(np.array([[0, 1, 2, 3, 3, 2, 1, 0] * 128], np.uint8), N, 0)
    rho = np.zeros_like(qb)
    rho[:, 0] = 1
    base, refine = orc.pack_weights(qb, rho, 2, 1)
    # channel c at bits 2c: codes 0,1,2,3 -> 0b11_10_01_00 = 0xE4; 3,2,1,0 -> 0x1B
    assert base[0] == 0xE4 and base[1] == 0x1B and base[256] == 0xE4
    # refinement: channel-major, row n at bit n (r=1): channel 0 has all 64 rows set
    assert (refine[:8] == 0xFF).all() and (refine[8:] == 0).all()


def test_pack_weights_unit_permutation_by_hand(orc):
    N, K = 16, 1024
    qb = np.zeros((N, K), np.uint8)
    qb[1, 0] = 1      # row 1, unit 0 -> unit 0 ^ 1 = 1: byte 16 of the row, bits 0-1
    qb[9, 64] = 2     # row 9 (9 mod 8 = 1), channel 64 = bit 128 = unit 1 -> unit 0
    qb[7, 1023] = 3   # row 7, bit 2046 = byte 255 (unit 15, bits 6-7) -> unit 8, byte 15
    qb[12, 100] = 1   # row 12 (mod 8 = 4): bit 200 = byte 25 = unit 1, byte 9 -> unit 5
    base, _ = orc.pack_weights(qb, np.zeros_like(qb), 2, 1)
    rows = base.reshape(N, 256)
    assert rows[1, 16] == 1 and rows[9, 0] == 2 << 0 and rows[7, 8 * 16 + 15] == 3 << 6
    assert rows[12, 5 * 16 + 9] == 1 << 0
    assert int(base.astype(np.int64).sum()) == 1 + 2 + (3 << 6) + 1


def test_pack_weights_3bit_high_plane_by_hand(orc):
    N, K = 64, 1024
    qb = np.zeros((N, K), np.uint8)
    qb[0, 5] = 4     # high bit only; channel 5 -> word 0 bit 8*1+1 = 9
    qb[0, 20] = 7    # channel 20 -> 16+4 -> bit 8*1+4+0 = 12; low bits 3
    qb[0, 32 + 31] = 4  # block 1, channel 31 -> 15 -> bit 8*3+4+3 = 31
    qb[3, 5] = 4     # row 3: word 0 of its high plane is unit 0 -> unit 3
    base, _ = orc.pack_weights(qb, np.zeros_like(qb), 3, 1)
    lo, hi = base[:N * K // 4], base[N * K // 4:]
    word0 = int.from_bytes(hi[0:4].tobytes(), "little")
    word1 = int.from_bytes(hi[4:8].tobytes(), "little")
    assert word0 == (1 << 9) | (1 << 12)
    assert word1 == (1 << 31)
    assert lo[20 // 4] == 3 << (2 * (20 % 4))
    row3 = hi[3 * 128:4 * 128]
    assert int.from_bytes(row3[48:52].tobytes(), "little") == 1 << 9
    assert int(hi[8:].astype(np.int64).sum()) == (1 << 1)  # only row 3's bit 9 (byte 49, bit 1)


def test_pack_kv_by_hand(orc):
    qb = np.zeros((1, 2, 3, 128), np.uint8)
    rho = np.zeros_like(qb)
    qb[0, 1, 2, 3] = 2
    rho[0, 0, 1, 31] = 3
    # keys, 2-bit codes, 32 bytes per token, t_max 16.  Dim 3: s=0, e=0, chunk
    # c=1 (bytes 8..15 of the token), pair 0, second code -> bit 16 -> byte 2.
    kb, kr = orc.pack_kv(qb, rho, 0, 2, 2, t_max=16)
    assert kb[(1 * 16 + 2) * 32 + 8 + 2] == 2 and kb.sum() == 2
    # dim 31: s=1, e=1, chunk 3, pair 3, second -> bit 22 -> byte 2, bits 6-7
    assert kr[(0 * 16 + 1) * 32 + 24 + 2] == 3 << 6 and kr.sum() == 3 << 6
    # values, 512-byte tiles of 16 tokens.  Token 2 of its tile: c=1, h=0,
    # first code; dim 3: g=3, m=0, e=0 -> chunk 4*3+1 = 13 (16 bytes each),
    # pair 0 -> bit 0.
    vb, vr = orc.pack_kv(qb, rho, 1, 2, 2, t_max=16)
    assert vb[1 * 512 + 13 * 16] == 2 and vb.sum() == 2
    # 1-bit refinements: 16 pairs per word; token 1, dim 31: c=0, h=0,
    # second; g=7, m=1, e=1 -> chunk 28 (8 bytes), pair 16*0+2+1 = 3 -> bit 16+3
    vb1, vr1 = orc.pack_kv(qb, np.minimum(rho, 1), 1, 2, 1, t_max=16)
    assert vr1[28 * 8 + 2] == 1 << 3 and vr1.sum() == 1 << 3


def test_pack_kv_3bit_planes_by_hand(orc):
    # 3-bit codes: a plane of the low two bits (2-bit layout) followed by a
    # plane of the high bits (1-bit layout); 48 bytes per key token, 768 per
    # value tile.
    qb = np.zeros((1, 2, 3, 128), np.uint8)
    rho = np.zeros_like(qb)
    qb[0, 1, 2, 3] = 6   # low bits 2, high bit 1
    qb[0, 0, 1, 31] = 5  # low bits 1, high bit 1
    kb, _ = orc.pack_kv(qb, rho, 0, 3, 2, t_max=16)
    assert kb.size == 2 * 16 * 48
    # token slot 18, dim 3: chunk 1, pair 0, second code.  Low plane: chunk at
    # byte 8, bit 16; high plane: byte 32 + 4, bit 16.
    assert kb[18 * 48 + 8 + 2] == 2 and kb[18 * 48 + 32 + 4 + 2] == 1
    # token slot 1, dim 31: chunk 3, pair 3, second.  Low: byte 24, bit 16 + 6;
    # high: byte 32 + 12, bit 16 + 3.
    assert kb[48 + 24 + 2] == 1 << 6 and kb[48 + 44 + 2] == 1 << 3
    assert int(kb.astype(np.int64).sum()) == 2 + 1 + 64 + 8
    vb, _ = orc.pack_kv(qb, rho, 1, 3, 2, t_max=16)
    assert vb.size == 2 * 768
    # head 1 tile, token 2, dim 3: chunk 13, pair 0, first code.  Low plane:
    # 16-byte chunks; high plane at byte 512, 8-byte chunks.
    assert vb[768 + 13 * 16] == 2 and vb[768 + 512 + 13 * 8] == 1
    # head 0 tile, token 1, dim 31: chunk 28, pair 3, second code
    assert vb[28 * 16 + 2] == 1 << 6 and vb[512 + 28 * 8 + 2] == 1 << 3
    assert int(vb.astype(np.int64).sum()) == 2 + 1 + 64 + 8


# ---------------------------------------------------------------------------
# chunked channel selection: brute force with forced ties


def brute_select(x16, C, k):
    B, K = x16.shape
    out = np.zeros((B, K // C, k), np.int32)
    for b in range(B):
        for c in range(K // C):
            idx = list(range(c * C, (c + 1) * C))
            idx.sort(key=lambda i: (-(int(x16[b, i]) & 0x7FFF), i))
            out[b, c] = sorted(idx[:k])
    return out


@pytest.mark.parametrize("C,k", [(16, 1), (16, 5), (16, 16), (32, 7), (64, 3)])
def test_select_chunks_brute_force(orc, C, k):
    rng = np.random.default_rng(C + k)
    for trial in range(20):
        x = rng.normal(0, 1, (3, 4 * C)).astype(np.float16)
        # forced ties: repeated magnitudes of both signs and signed zeros
        x[:, ::5] = np.float16(0.5)
        x[:, 1::7] = np.float16(-0.5)
        x[0, :3] = np.float16(0.0)
        x[0, 3:5] = np.float16(-0.0)
        x16 = x.view(np.uint16)
        assert np.array_equal(orc.select_chunks(x16, C, k), brute_select(x16, C, k))


# ---------------------------------------------------------------------------
# refined GEMV against dense matrix-vector products


@pytest.fixture(scope="module")
def small_gemv(orc):
    rng = np.random.default_rng(21)
    N, K, G, C = 96, 512, 128, 128
    W = rng.normal(0, 0.02, (N, K)).astype(np.float32)
    x = rng.normal(0, 1, (2, K))
    x[:, rng.choice(K, 5, replace=False)] *= 20
    x = x.astype(np.float16)
    return W, x, N, K, G, C


@pytest.mark.parametrize("b,r", [(2, 2), (3, 1), (4, 2)])
def test_gemv_k0_is_dense_base(orc, small_gemv, b, r):
    W, x, N, K, G, C = small_gemv
    qb, rho, sz = orc.quant_weights(W, b, r, G)
    y = orc.gemv_refined(qb, rho, sz, r, G, x, None, C, 0)
    Wb = orc.dequant_weights(qb, rho, sz, r, G)
    assert np.allclose(y, x.astype(np.float64) @ Wb.T, rtol=1e-12, atol=1e-12)
    # and the base grid really is the b-bit quantisation of W (error <= s/2)
    S = np.repeat(f16(sz[:, :, 0]), G, axis=1)
    assert (np.abs(Wb - W) <= S / 2 * (1 + 1e-3) + 1e-6).all()


@pytest.mark.parametrize("b,r", [(2, 2), (3, 1), (4, 2)])
def test_gemv_all_selected_is_dense_refined(orc, small_gemv, b, r):
    W, x, N, K, G, C = small_gemv
    qb, rho, sz = orc.quant_weights(W, b, r, G)
    sel = orc.select_chunks(x, C, C)
    y = orc.gemv_refined(qb, rho, sz, r, G, x, sel, C, C)
    Wf = orc.dequant_weights(qb, rho, sz, r, G, refined_mask=np.ones((N, K), bool))
    assert np.allclose(y, x.astype(np.float64) @ Wf.T, rtol=1e-12, atol=1e-12)
    # the refined grid halves the error bound per extra bit
    S = np.repeat(f16(sz[:, :, 0]), G, axis=1)
    assert (np.abs(Wf - W) <= S / (2 << r) * (1 + 1e-3) + 1e-6).all()


def test_gemv_linearity_of_the_correction(orc, small_gemv):
    """Error model of the "which tiles count" paragraph: the output changes by
    sum over selected i of x_i * (w~ - w^)_i, exactly (fp64)."""
    W, x, N, K, G, C = small_gemv
    b, r, k = 2, 2, 9
    qb, rho, sz = orc.quant_weights(W, b, r, G)
    sel = orc.select_chunks(x, C, k)
    y0 = orc.gemv_refined(qb, rho, sz, r, G, x, None, C, 0)
    yk = orc.gemv_refined(qb, rho, sz, r, G, x, sel, C, k)
    Wb = orc.dequant_weights(qb, rho, sz, r, G)
    Wf = orc.dequant_weights(qb, rho, sz, r, G, refined_mask=np.ones((N, K), bool))
    for bb in range(x.shape[0]):
        idx = sel[bb].ravel()
        delta = (Wf - Wb)[:, idx] @ x[bb, idx].astype(np.float64)
        assert np.allclose(yk[bb] - y0[bb], delta, rtol=1e-10, atol=1e-12)
        # refining the largest-|x| channels reduces the error against W more than
        # refining nothing, on average over rows
        yt = W.astype(np.float64) @ x[bb].astype(np.float64)
        assert np.linalg.norm(yk[bb] - yt) < np.linalg.norm(y0[bb] - yt)


# ---------------------------------------------------------------------------
# KV scoring, selection and refined attention against numpy attention


@pytest.fixture(scope="module")
def small_kv(orc):
    rng = np.random.default_rng(31)
    B, H, Hq, T, D = 2, 2, 8, 37, 64
    k = rng.normal(0, 1, (B, H, T, D))
    k[:, :, :, [3, 17]] *= 10
    v = rng.normal(0, 1, (B, H, T, D))
    q = rng.normal(0, 1, (B, Hq, D)).astype(np.float16)
    kc = orc.quant_kv(k.astype(np.float16), 2, 2, 32)
    vc = orc.quant_kv(v.astype(np.float16), 2, 2, 32)
    return kc, vc, q, B, H, Hq, T, D


def kv_dense(codes, refined):
    qb, rho, sz = codes
    f = lambda a: np.asarray(a, np.uint16).view(np.float16).astype(np.float64)
    S = np.repeat(f(sz[..., 0]), 32, axis=-1)
    M = np.repeat(f(sz[..., 1]), 32, axis=-1)
    val = qb.astype(np.float64)
    if refined is not None:
        val = val + np.where(refined[..., None], (2.0 * rho + 1 - 4) / 8, 0.0)
    return M + S * val


def np_attention(q, K, V, grp):
    B, Hq, D = q.shape
    out = np.zeros((B, Hq, D))
    for b in range(B):
        for h in range(Hq):
            l = K[b, h // grp] @ q[b, h].astype(np.float64) / math.sqrt(D)
            p = np.exp(l - l.max())
            p /= p.sum()
            out[b, h] = p @ V[b, h // grp]
    return out


def test_kv_logits_and_scores(orc, small_kv):
    kc, vc, q, B, H, Hq, T, D = small_kv
    logits = orc.kv_logits(kc[0], kc[2], q)
    Kb = kv_dense(kc, None)
    for b in range(B):
        for h in range(Hq):
            assert np.allclose(logits[b, h], Kb[b, h // 4] @ q[b, h].astype(np.float64) / 8.0,
                               rtol=1e-12, atol=1e-12)
    score = orc.kv_scores(logits, H)
    assert np.allclose(score.sum(-1), Hq // H, rtol=1e-12)
    assert (score > 0).all()


def test_kv_scores_head_grouping_closed_form(orc):
    """Query head h belongs to KV head h // (h_q / h_kv) ("which tiles count":
    a KV head's score sums the attention of the query heads that share it).
    Head h puts logit L on token h and 0 on every other token, so its softmax is
    p_hot = e^L / (e^L + T - 1) on token h and p_cold = 1 / (e^L + T - 1)
    elsewhere; KV head g's score is then, in closed form,
    grp * p_cold + (p_hot - p_cold) on each of its own query heads' tokens.
    A grouping by h % h_kv (or any other) puts the hot tokens elsewhere and fails."""
    B, Hq, H, T, L = 2, 32, 8, 40, 3.0
    grp = Hq // H
    logits = np.zeros((B, Hq, T))
    for b in range(B):
        for h in range(Hq):
            logits[b, h, h] = L
    score = orc.kv_scores(logits, H)
    den = np.exp(L) + (T - 1)
    p_hot, p_cold = np.exp(L) / den, 1.0 / den
    want = np.full((B, H, T), grp * p_cold)
    for g in range(H):
        for h in range(g * grp, (g + 1) * grp):
            want[:, g, h] += p_hot - p_cold
    assert np.allclose(score, want, rtol=1e-13, atol=1e-15)
    # and the selection of each KV head's top grp tokens is exactly its own query heads' hot tokens
    sel = orc.kv_select(score, grp)
    for g in range(H):
        assert list(sel[0, g]) == list(range(g * grp, (g + 1) * grp))


def test_kv_select_brute_force(orc):
    rng = np.random.default_rng(41)
    for trial in range(30):
        T = int(rng.integers(1, 40))
        score = rng.integers(0, 6, size=(1, 3, T)).astype(np.float64) / 7  # many ties
        k = int(rng.integers(1, T + 1))
        sel = orc.kv_select(score, k)
        for h in range(3):
            order = sorted(range(T), key=lambda t: (-score[0, h, t], t))
            assert list(sel[0, h]) == sorted(order[:k])


def test_kv_attention_special_cases(orc, small_kv):
    kc, vc, q, B, H, Hq, T, D = small_kv
    # k_tok = 0: base attention
    out0 = orc.kv_attention(kc, vc, q, None, 0, 2)
    ref0 = np_attention(q, kv_dense(kc, None), kv_dense(vc, None), Hq // H)
    assert np.allclose(out0, ref0, rtol=1e-11, atol=1e-12)
    # every token selected: full (b+r)-bit attention
    sel = np.tile(np.arange(T, dtype=np.int32), (B, H, 1))
    outT = orc.kv_attention(kc, vc, q, sel, T, 2)
    allsel = np.ones((B, H, T), bool)
    refT = np_attention(q, kv_dense(kc, allsel), kv_dense(vc, allsel), Hq // H)
    assert np.allclose(outT, refT, rtol=1e-11, atol=1e-12)
    # a proper subset: refined exactly where selected
    logits = orc.kv_logits(kc[0], kc[2], q)
    sel5 = orc.kv_select(orc.kv_scores(logits, H), 5)
    mask = np.zeros((B, H, T), bool)
    for b in range(B):
        for h in range(H):
            mask[b, h, sel5[b, h]] = True
    out5 = orc.kv_attention(kc, vc, q, sel5, 5, 2)
    ref5 = np_attention(q, kv_dense(kc, mask), kv_dense(vc, mask), Hq // H)
    assert np.allclose(out5, ref5, rtol=1e-11, atol=1e-12)
    assert not np.allclose(out5, out0, rtol=1e-6)


def test_kv_attention_single_token(orc, small_kv):
    """T = 1: the output is the (refined) value of the only token, for any q."""
    kc, vc, q, B, H, Hq, T, D = small_kv
    k1 = tuple(a[:, :, :1] for a in kc)
    v1 = tuple(a[:, :, :1] for a in vc)
    sel = np.zeros((B, H, 1), np.int32)
    out = orc.kv_attention(k1, v1, q, sel, 1, 2)
    V = kv_dense(v1, np.ones((B, H, 1), bool))
    for h in range(Hq):
        assert np.allclose(out[:, h], V[:, h // 4, 0], rtol=1e-13, atol=1e-13)


# ---------------------------------------------------------------------------
# byte model: the explainer's worked example


def test_worked_example_bits():
    g = {r[0]: float(r[1]) for r in read_golden("worked_example_bits.txt")}
    b, r, k, C = int(g["base_bits"]), int(g["refine_bits"]), int(g["k"]), int(g["chunk"])
    assert bytemodel.fetched_share(k, C) == g["fetched_share"]
    assert bytemodel.extra_bits_per_weight(r, k, C) == g["extra_bits"]
    assert bytemodel.bits_touched_per_weight(b, r, k, C) == g["bits_touched"]
    assert 16 / bytemodel.extra_bits_per_weight(r, k, C) == g["bf16_over_payload"]
    assert math.isclose(100 * bytemodel.extra_bits_per_weight(r, k, C) / b, g["increase_percent"])


def test_byte_model_configs():
    # single 4096 x 4096 GEMV, 2+2 bits, k = 32 of 1024
    assert bytemodel.gemv_bytes(4096, 4096, 2, 2, 128, 32, 1024) == 4_874_752
    assert bytemodel.kv_attention_bytes(8192, 8, 32, 128, 2, 2, 32, 256) == 6_447_104
    assert bytemodel.kv_attention_bytes(131072, 8, 32, 128, 2, 2, 32, 1024) == 101_212_160


# ---------------------------------------------------------------------------
# decoder-step glue: closed forms and library routines


def test_rmsnorm_closed_form(orc):
    rng = np.random.default_rng(51)
    h = rng.normal(0, 3, 4096)
    x = f16(orc.rmsnorm_f16(h))
    ref = h / np.sqrt(np.mean(h * h) + 1e-5)
    assert np.array_equal(orc.rmsnorm_f16(h), ref.astype(np.float16).view(np.uint16))
    assert abs(np.mean(x * x) - 1.0) < 1e-3
    # scale invariance (eps aside)
    assert np.abs(f16(orc.rmsnorm_f16(h * 7.0)) - x).max() <= 2 ** -9


def test_rope_is_a_rotation_by_the_stated_angle(orc):
    rng = np.random.default_rng(52)
    v = rng.normal(0, 1, (3, 128))
    assert np.allclose(orc.rope(v, 0), v)
    pos, theta = 32768, 500000.0
    out = orc.rope(v, pos, theta)
    # complex multiplication of (x_i + i x_{i+64}) by e^{i pos theta^(-2i/128)}
    z = v[:, :64] + 1j * v[:, 64:]
    ang = pos * theta ** (-2.0 * np.arange(64) / 128)
    w = z * np.exp(1j * ang)
    assert np.allclose(out[:, :64], w.real, atol=1e-9) and np.allclose(out[:, 64:], w.imag, atol=1e-9)
    assert np.allclose(np.linalg.norm(out, axis=1), np.linalg.norm(v, axis=1))


def test_silu_mul_and_f16_gemv(orc):
    rng = np.random.default_rng(53)
    gu = rng.normal(0, 2, 2 * 300)
    g, u = gu[:300], gu[300:]
    ref = (g / (1 + np.exp(-g)) * u).astype(np.float16).view(np.uint16)
    assert np.array_equal(orc.silu_mul_f16(gu), ref)
    w = rng.normal(0, 0.02, (70, 256)).astype(np.float16)
    x = rng.normal(0, 1, 256).astype(np.float16)
    assert np.allclose(orc.gemv_f16(w, x), w.astype(np.float64) @ x.astype(np.float64), rtol=1e-12, atol=1e-12)


def test_correction_is_the_difference_of_refined_and_base(orc, small_gemv):
    W, x, N, K, G, C = small_gemv
    qb, rho, sz = orc.quant_weights(W, 2, 2, G)
    sel = orc.select_chunks(x, C, 9)
    y0 = orc.gemv_refined(qb, rho, sz, 2, G, x, None, C, 0)
    yk = orc.gemv_refined(qb, rho, sz, 2, G, x, sel, C, 9)
    for b in range(x.shape[0]):
        corr = orc.gemv_correction(qb, rho, sz, 2, G, x[b], sel[b])
        assert np.allclose(y0[b] + corr, yk[b], rtol=1e-12, atol=1e-12)


def _dense_decoder(h16, layers, lm16, pos, h_q, h_kv, d, theta=500000.0, eps=1e-5):
    """Textbook fp64 Llama step with dense weights/KV (every value refined)."""
    f = lambda a: np.asarray(a, np.float16).astype(np.float64)
    h = f(h16)[0].copy()

    def norm(v):
        return (v / np.sqrt(np.mean(v * v) + eps)).astype(np.float16).astype(np.float64)

    def rot(v):
        z = v[:, : d // 2] + 1j * v[:, d // 2:]
        z = z * np.exp(1j * pos * theta ** (-2.0 * np.arange(d // 2) / d))
        return np.concatenate([z.real, z.imag], axis=1)

    for L in layers:
        x = norm(h)
        qkv = L["qkv"] @ x
        q = rot(qkv[: h_q * d].reshape(h_q, d)).astype(np.float16).astype(np.float64)
        k = rot(qkv[h_q * d:(h_q + h_kv) * d].reshape(h_kv, d)).astype(np.float16)
        v = qkv[(h_q + h_kv) * d:].reshape(h_kv, d).astype(np.float16)
        K = L["K"](k)  # dense refined keys [h_kv][T+1][d]
        V = L["V"](v)
        att = np.zeros((h_q, d))
        for hh in range(h_q):
            g = hh // (h_q // h_kv)
            lg = K[g] @ q[hh] / math.sqrt(d)
            p = np.exp(lg - lg.max())
            att[hh] = (p / p.sum()) @ V[g]
        h = h + L["o"] @ att.reshape(-1).astype(np.float16).astype(np.float64)
        x = norm(h)
        gu = L["gate_up"] @ x
        I = gu.size // 2
        xd = (gu[:I] / (1 + np.exp(-gu[:I])) * gu[I:]).astype(np.float16).astype(np.float64)
        h = h + L["down"] @ xd
    return f(lm16) @ norm(h)


def test_oracle_decoder_all_refined_equals_dense_decoder(orc):
    """lead = lag = 0, every channel and token refined: the step is a plain
    decoder with (b+r)-bit weights and KV (textbook fp64 reference)."""
    from oracle.decoder import OracleDecoder

    rng = np.random.default_rng(61)
    H, I, h_q, h_kv, d, T, C = 512, 1024, 4, 2, 128, 20, 256
    h16 = rng.normal(0, 1, (1, H)).astype(np.float16)
    dec = OracleDecoder(h16, h_q=h_q, h_kv=h_kv, d=d, r=2, G=128, chunk=C, kch=C, kv_b=2, kv_r=2,
                        k_tok=T + 1, lead=0, lag=0)
    dense_layers = []
    for layer in range(2):
        Ws = {"qkv": rng.normal(0, 0.02, ((h_q + 2 * h_kv) * d, H)), "o": rng.normal(0, 0.02, (H, h_q * d)),
              "gate_up": rng.normal(0, 0.02, (2 * I, H)), "down": rng.normal(0, 0.02, (H, I))}
        Q, D = {}, {}
        for n, w in Ws.items():
            qb, rho, sz = orc.quant_weights(w.astype(np.float32), 2, 2, 128)
            Q[n] = (qb, rho, sz)
            D[n] = orc.dequant_weights(qb, rho, sz, 2, 128, refined_mask=np.ones(qb.shape, bool))
        kc = rng.normal(0, 1, (1, h_kv, T, d)).astype(np.float16)
        vc = rng.normal(0, 1, (1, h_kv, T, d)).astype(np.float16)

        def dense_kv(new, cache):
            full = np.concatenate([cache[0], np.asarray(new)[:, None, :]], axis=1)[None]
            qb, rho, sz = orc.quant_kv(full, 2, 2)
            Sv = np.repeat(f16(sz[..., 0]), 32, -1)
            Mv = np.repeat(f16(sz[..., 1]), 32, -1)
            return (Mv + Sv * (qb + (2.0 * rho + 1 - 4) / 8))[0]

        D["K"] = lambda new, cache=kc: dense_kv(new, cache)
        D["V"] = lambda new, cache=vc: dense_kv(new, cache)
        dense_layers.append(D)
        dec.layer(Q, kc, vc, T)
    lm = rng.normal(0, 0.02, (300, H)).astype(np.float16)
    got = dec.finish(lm)[0]
    ref = _dense_decoder(h16, dense_layers, lm, T, h_q, h_kv, d)
    assert np.allclose(got, ref, rtol=1e-9, atol=1e-9), np.abs(got - ref).max()


def test_oracle_decoder_lag_without_refinement_is_a_no_op(orc):
    from oracle.decoder import OracleDecoder

    rng = np.random.default_rng(62)
    H, I, h_q, h_kv, d, T = 512, 1024, 4, 2, 128, 9
    h16 = rng.normal(0, 1, (1, H)).astype(np.float16)
    W = {n: orc.quant_weights(rng.normal(0, 0.02, s).astype(np.float32), 2, 2, 128)
         for n, s in {"qkv": ((h_q + 2 * h_kv) * d, H), "o": (H, h_q * d), "gate_up": (2 * I, H),
                      "down": (H, I)}.items()}
    kc = rng.normal(0, 1, (1, h_kv, T, d)).astype(np.float16)
    vc = rng.normal(0, 1, (1, h_kv, T, d)).astype(np.float16)
    lm = rng.normal(0, 0.02, (50, H)).astype(np.float16)
    outs = []
    for lag in (0, 1):
        dec = OracleDecoder(h16, h_q=h_q, h_kv=h_kv, d=d, chunk=256, kch=0, k_tok=3, lead=1, lag=lag)
        dec.layer(W, kc, vc, T)
        outs.append(dec.finish(lm))
    assert np.array_equal(outs[0], outs[1])


def _lag_case(orc, seed, zero):
    """One small model (2 layers) with the projections in `zero` set to zero
    weights; the final logits at lag 0 and lag 1 (lead 0, channels refined)."""
    from oracle.decoder import OracleDecoder

    rng = np.random.default_rng(seed)
    H, I, h_q, h_kv, d, T = 512, 1024, 4, 2, 128, 9
    h16 = rng.normal(0, 1, (1, H)).astype(np.float16)
    shapes = {"qkv": ((h_q + 2 * h_kv) * d, H), "o": (H, h_q * d), "gate_up": (2 * I, H), "down": (H, I)}
    layers = []
    for _ in range(2):
        W = {}
        for n, s in shapes.items():
            w = np.zeros(s, np.float32) if n in zero else rng.normal(0, 0.05, s).astype(np.float32)
            W[n] = orc.quant_weights(w, 2, 2, 128)
        layers.append((W, rng.normal(0, 1, (1, h_kv, T, d)).astype(np.float16),
                       rng.normal(0, 1, (1, h_kv, T, d)).astype(np.float16)))
    lm = rng.normal(0, 0.02, (50, H)).astype(np.float16)
    outs = []
    for lag in (0, 1):
        dec = OracleDecoder(h16, h_q=h_q, h_kv=h_kv, d=d, chunk=256, kch=16, k_tok=3, lead=0, lag=lag)
        for W, kc, vc in layers:
            dec.layer(W, kc, vc, T)
        outs.append(dec.finish(lm)[0])
    return outs


def test_oracle_decoder_lag_moves_o_correction_past_the_mlp(orc):
    """Lag 1 holds o's correction back from the MLP input of its layer and adds
    it to the residual before the next layer: with a zero MLP nothing reads the
    residual in between, so lag 1 equals lag 0 (up to the order of the sums);
    with a working MLP it does not (the MLP input differs)."""
    same = _lag_case(orc, 71, zero=("gate_up", "down"))
    assert np.allclose(same[0], same[1], rtol=1e-10, atol=1e-12)
    differ = _lag_case(orc, 71, zero=())
    assert not np.allclose(differ[0], differ[1], rtol=1e-6, atol=1e-9)


def test_oracle_decoder_down_lag_lands_with_down(orc):
    """Down's lagged correction enters the residual where down's own output
    does (the next layer's start, or the final norm): with o zero (no o
    correction to hold back), lag 1 equals lag 0 up to the order of the sums."""
    outs = _lag_case(orc, 72, zero=("o",))
    assert np.allclose(outs[0], outs[1], rtol=1e-10, atol=1e-12)


def test_oracle_decoder_forced_selections_are_its_own(orc):
    """Teacher forcing (used by the decode-step parity tests) is plumbing only:
    forcing the oracle to the selections it would make itself leaves every
    output bit unchanged, and every recorded own choice equals the forced one;
    forcing one channel swap changes the output."""
    from oracle.decoder import OracleDecoder

    rng = np.random.default_rng(73)
    H, I, h_q, h_kv, d, T = 512, 1024, 4, 2, 128, 20
    h16 = rng.normal(0, 1, (2, H)).astype(np.float16)
    shapes = {"qkv": ((h_q + 2 * h_kv) * d, H), "o": (H, h_q * d), "gate_up": (2 * I, H), "down": (H, I)}
    layers = []
    for _ in range(2):
        W = {n: orc.quant_weights(rng.normal(0, 0.05, s).astype(np.float32), 2, 2, 128) for n, s in shapes.items()}
        layers.append((W, rng.normal(0, 1, (2, h_kv, T, d)).astype(np.float16),
                       rng.normal(0, 1, (2, h_kv, T, d)).astype(np.float16)))
    lm = rng.normal(0, 0.02, (50, H)).astype(np.float16)
    kw = dict(h_q=h_q, h_kv=h_kv, d=d, chunk=256, kch=16, k_tok=5, lead=1, lag=1)

    def run(force):
        dec = OracleDecoder(h16, force=force, **kw)
        for W, kc, vc in layers:
            dec.layer(W, kc, vc, T)
        return dec, dec.finish(lm)

    free, out0 = run(None)
    force = {}
    for l, tr in enumerate(free.trace):
        for name, per_b in tr["weights"].items():
            force[("w", l, name)] = np.stack([np.asarray(s).reshape(-1) for s in per_b])
        force[("tok", l)] = np.stack(tr["tokens"])
    forced, out1 = run(force)
    assert np.array_equal(out0, out1)
    assert len(forced.checks) == 2 * 2 * 5
    for kind, l, name, b, own, f, vals in forced.checks:
        assert np.array_equal(np.asarray(own).reshape(-1), np.asarray(f).reshape(-1))
    # swap one selected channel of layer 1's gate_up for an unselected one
    f2 = {k: v.copy() for k, v in force.items()}
    row = f2[("w", 1, "gate_up")][0]
    chunk0 = set(row[:16].tolist())
    row[0] = next(c for c in range(256) if c not in chunk0)
    row[:16] = np.sort(row[:16])
    _, out2 = run(f2)
    assert not np.array_equal(out0, out2)
