"""Pins for the CPU oracle, checked against things other than the oracle itself:
numpy's IEEE binary16 conversions, the worked examples of the pages
(tests/golden), numpy's bit unpacking, exact rational arithmetic (brute force),
integer dot products and closed forms.

Sources: the ZSE wiki article "ZSE - open-source движок для запуска LLM локально
на GPU - 2026", section "Формат модели .zse" (quantizer formula, INT4 packing,
fp16 scale/zero) and "ZSE: A Memory-Efficient LLM Inference Engine with Smart
Resource Orchestration", section "Technical Architecture" (INT2-8 per tensor).
"""
import os
from fractions import Fraction

import numpy as np
import pytest

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
BITS = (2, 3, 4, 8)


# ----------------------------------------------------------------- binary16 --

def test_f16_decode_exhaustive(orc):
    """Every one of the 65536 bit patterns decodes like numpy's float16."""
    pats = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = pats.view(np.float16).astype(np.float64)
    got = np.array([orc.f16_to_f64(int(h)) for h in pats])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])
    # signed zeros keep their sign
    assert np.signbit(got[0x8000]) and not np.signbit(got[0])


def test_f16_encode_roundtrip_all_finite(orc):
    for h in range(65536):
        e = (h >> 10) & 0x1F
        if e == 31:
            continue
        assert orc.f64_to_f16(orc.f16_to_f64(h)) == h


def test_f16_encode_matches_numpy_random(orc):
    rng = np.random.default_rng(1)
    vals = np.concatenate([
        rng.normal(0, 1, 20000),
        rng.normal(0, 1e-5, 5000),            # subnormal range
        rng.normal(0, 3e4, 5000),             # near overflow
        rng.uniform(-70000, 70000, 2000),
    ])
    ref = vals.astype(np.float16).view(np.uint16)
    got = np.array([orc.f64_to_f16(float(v)) for v in vals], np.uint16)
    assert np.array_equal(got, ref)


def test_f16_ties_to_even_and_overflow(orc):
    """Midpoints between neighbouring halves go to the even code; one ulp of
    fp64 above goes up; 65520 (midpoint past the max) overflows."""
    rng = np.random.default_rng(2)
    hs = rng.integers(0, 0x7BFF, 3000)
    for h in hs:
        a = orc.f16_to_f64(int(h))
        b = orc.f16_to_f64(int(h) + 1)
        mid = (a + b) / 2                     # exact in fp64
        even = int(h) if (int(h) & 1) == 0 else int(h) + 1
        assert orc.f64_to_f16(mid) == even
        assert orc.f64_to_f16(np.nextafter(mid, np.inf)) == int(h) + 1
        assert orc.f64_to_f16(np.nextafter(mid, -np.inf)) == int(h)
        assert orc.f64_to_f16(-mid) == (even | 0x8000)
    assert orc.f64_to_f16(65504.0) == 0x7BFF
    assert orc.f64_to_f16(65519.999) == 0x7BFF
    assert orc.f64_to_f16(65520.0) == 0x7C00
    assert orc.f64_to_f16(-1e9) == 0xFC00
    assert orc.f64_to_f16(2.0 ** -25) == 0x0000          # tie to even (0)
    assert orc.f64_to_f16(3 * 2.0 ** -25) == 0x0002      # tie to even (2)


# ------------------------------------------------------------------ packing --

def _read_pack_golden():
    rows = []
    with open(os.path.join(GOLDEN, "pack_examples.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            b, codes, words = [p.strip() for p in line.split("|")]
            rows.append((int(b), [int(c) for c in codes.split()],
                         [int(w, 16) for w in words.split()]))
    return rows


@pytest.mark.parametrize("case", _read_pack_golden())
def test_pack_worked_examples(orc, case):
    bits, codes, words = case
    got = orc.pack_row(np.array(codes, np.uint8), bits)
    assert [int(w) for w in got] == words
    back = orc.unpack_row(np.array(words, np.uint32), len(codes), bits)
    assert list(back) == codes


def _stream_codes_numpy(words, K, bits):
    """Independent unpack: numpy little-endian bit order over the row bytes."""
    stream = np.unpackbits(np.asarray(words, "<u4").view(np.uint8), bitorder="little")
    chunks = stream[:K * bits].reshape(K, bits).astype(np.int64)
    return (chunks << np.arange(bits)).sum(axis=1)


@pytest.mark.parametrize("bits", BITS)
def test_pack_matches_numpy_bitstream(orc, bits):
    rng = np.random.default_rng(10 + bits)
    for K in (128, 256, 1024, 3584):
        codes = rng.integers(0, 1 << bits, K).astype(np.uint8)
        words = orc.pack_row(codes, bits)
        assert words.size == K * bits // 32
        assert np.array_equal(_stream_codes_numpy(words, K, bits), codes)
        assert np.array_equal(orc.unpack_row(words, K, bits), codes)


def test_pack_int4_low_nibble_first(orc):
    """The page's byte rule: byte j holds code 2j in the low nibble, 2j+1 high."""
    rng = np.random.default_rng(3)
    codes = rng.integers(0, 16, 4096).astype(np.uint8)
    by = orc.pack_row(codes, 4).astype("<u4").view(np.uint8)
    assert np.array_equal(by, codes[0::2] | (codes[1::2] << 4))


def test_pack_int8_and_int2_bytes(orc):
    rng = np.random.default_rng(4)
    c8 = rng.integers(0, 256, 512).astype(np.uint8)
    assert np.array_equal(orc.pack_row(c8, 8).astype("<u4").view(np.uint8), c8)
    c2 = rng.integers(0, 4, 512).astype(np.uint8)
    by = orc.pack_row(c2, 2).astype("<u4").view(np.uint8)
    exp = c2[0::4] | (c2[1::4] << 2) | (c2[2::4] << 4) | (c2[3::4] << 6)
    assert np.array_equal(by, exp)


@pytest.mark.parametrize("bits", BITS)
def test_unpack_whole_tensor(orc, bits):
    rng = np.random.default_rng(20 + bits)
    N, K = 7, 384
    codes = rng.integers(0, 1 << bits, (N, K)).astype(np.uint8)
    packed = np.stack([orc.pack_row(c, bits) for c in codes])
    assert np.array_equal(orc.unpack(packed, N, K, bits), codes)


# ---------------------------------------------------------------- quantizer --

def test_quantizer_page_example(orc):
    with open(os.path.join(GOLDEN, "quant_int4_example.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            sz, ws, qs = [p.strip() for p in line.split("|")]
            s_bits, z_bits = [int(v, 16) for v in sz.split()]
            w = np.array([float(v) for v in ws.split()], np.float32)
            q_exp = [int(v) for v in qs.split()]
            s, z, q = orc.quantize_group(w, 4)
            assert (s, z) == (s_bits, z_bits)
            assert list(q) == q_exp


def _f16(v):
    return float(np.float16(v))


@pytest.mark.parametrize("bits", BITS)
def test_quantizer_scale_zero_are_fp16_of_minmax(orc, bits):
    """s16 = fp16((max-min)/L), z16 = fp16(min), checked with numpy's fp16."""
    rng = np.random.default_rng(30 + bits)
    L = (1 << bits) - 1
    for _ in range(200):
        w = (rng.normal(0, 0.02, 128) * rng.choice([1, 20], 128, p=[.99, .01])).astype(np.float32)
        s, z, q = orc.quantize_group(w, bits)
        mn, mx = float(w.min()), float(w.max())
        assert s == np.float16((mx - mn) / L).view(np.uint16)
        assert z == np.float16(mn).view(np.uint16)


@pytest.mark.parametrize("bits", BITS)
def test_quantizer_error_bound_and_range(orc, bits):
    """|w - w_hat| <= s16/2 for unclamped elements, q in [0, L], min -> 0,
    max -> L (the config distributions: N(0, 0.02) with x20 outliers)."""
    rng = np.random.default_rng(40 + bits)
    L = (1 << bits) - 1
    for _ in range(300):
        w = rng.normal(0, 0.02, 128)
        w[rng.random(128) < 0.01] *= 20
        w = w.astype(np.float32)
        s_b, z_b, q = orc.quantize_group(w, bits)
        s = float(np.uint16(s_b).view(np.float16))
        z = float(np.uint16(z_b).view(np.float16))
        assert q.max() <= L
        w_hat = q.astype(np.float64) * s + z
        err = np.abs(w.astype(np.float64) - w_hat)
        unclamped = (q > 0) & (q < L)
        assert np.all(err[unclamped] <= s / 2 * (1 + 1e-12))
        # clamped ends: bounded by the fp16 rounding of zero and scale
        lo_gap = abs(float(w.min()) - z)
        hi_gap = abs(float(w.max()) - (L * s + z))
        assert np.all(err[~unclamped] <= max(lo_gap, hi_gap) + s / 2)
        assert q[np.argmin(w)] == 0
        assert q[np.argmax(w)] == L


@pytest.mark.parametrize("bits", BITS)
def test_quantizer_constant_group(orc, bits):
    for v in (0.0, 0.0123, -3.5, 1e-6):
        w = np.full(128, v, np.float32)
        s, z, q = orc.quantize_group(w, bits)
        assert s == 0
        assert z == np.float16(v).view(np.uint16)
        assert not q.any()
    # scale underflow in fp16: max - min tiny -> s16 == 0, w_hat = z16
    w = np.zeros(128, np.float32)
    w[5] = 1e-9
    s, z, q = orc.quantize_group(w, bits)
    assert s == 0 and not q.any()


def test_quantizer_ties_round_half_even(orc):
    """Group with min 0 and max 15/16: s16 = 1/16, z16 = 0 exactly; elements at
    (j + 1/2)/16 are exact ties and must go to the even code."""
    base = np.zeros(128, np.float32)
    base[0] = 0.0
    base[1] = 15.0 / 16
    for j in range(15):
        base[2 + j] = (j + 0.5) / 16
    s, z, q = orc.quantize_group(base, 4)
    assert s == np.float16(1 / 16).view(np.uint16) and z == 0
    for j in range(15):
        exp = j if j % 2 == 0 else j + 1
        assert q[2 + j] == exp, (j, q[2 + j])


@pytest.mark.parametrize("bits", BITS)
def test_quantizer_brute_force_exact(orc, bits):
    """Exhaustive search over q in [0, L] with exact rational arithmetic: the
    oracle's code minimises |w - (q*s16 + z16)|, ties to the even code."""
    rng = np.random.default_rng(50 + bits)
    L = (1 << bits) - 1
    for trial in range(40):
        n = int(rng.integers(2, 24))
        w = (rng.normal(0, 0.02, n) * (20 if trial % 7 == 0 else 1)).astype(np.float32)
        s_b, z_b, q = orc.quantize_group(w, bits)
        s = Fraction(float(np.uint16(s_b).view(np.float16)))
        z = Fraction(float(np.uint16(z_b).view(np.float16)))
        for i in range(n):
            wi = Fraction(float(w[i]))
            best = None
            for cand in range(L + 1):
                d = abs(wi - (cand * s + z))
                if best is None or d < best[0] or (d == best[0] and cand % 2 == 0):
                    best = (d, cand)
            assert q[i] == best[1], (trial, i, q[i], best)


def test_quantizer_rejects_nonfinite(orc):
    for bad in (np.nan, np.inf, -np.inf, 65505.0, -70000.0):
        w = np.zeros(128, np.float32)
        w[3] = bad
        with pytest.raises(orc.OracleError) as e:
            orc.quantize_group(w, 4)
        assert e.value.status == orc.NONFINITE
    w = np.zeros(128, np.float32)
    w[3] = 65504.0
    orc.quantize_group(w, 4)        # the largest half is accepted


@pytest.mark.parametrize("bits", BITS)
def test_quantize_pack_tensor_consistent_with_groups(orc, bits):
    rng = np.random.default_rng(60 + bits)
    N, K = 5, 512
    w = rng.normal(0, 0.02, (N, K)).astype(np.float32)
    packed, scales, zeros = orc.quantize_pack(w, bits)
    assert packed.shape == (N, K * bits // 32) and scales.shape == (N, K // 128)
    codes = orc.unpack(packed, N, K, bits)
    for n in range(N):
        for g in range(K // 128):
            s, z, q = orc.quantize_group(w[n, g * 128:(g + 1) * 128], bits)
            assert scales[n, g] == s and zeros[n, g] == z
            assert np.array_equal(codes[n, g * 128:(g + 1) * 128], q)


def test_quantize_pack_rejects_bad_format(orc):
    w = np.zeros((2, 256), np.float32)
    for bits in (1, 5, 6, 7, 16):
        with pytest.raises(orc.OracleError) as e:
            orc.quantize_pack(w, bits)
        assert e.value.status == orc.UNSUPPORTED
    with pytest.raises(orc.OracleError) as e:
        orc.quantize_pack(np.zeros((2, 200), np.float32), 4)
    assert e.value.status == orc.INVALID


# ------------------------------------------------------- symmetric quantizer --
# The wiki section "Формат модели .zse" lists symmetric INT8 quantization
# without a formula; the reading (Q = 2^(b-1) - 1, scale = fp16(max|w|/Q),
# q = clamp(round(w/scale), -Q, Q), stored code = q + 2^(b-1), zero =
# -2^(b-1)*scale) is pinned here by hand-derived examples, numpy's fp16, exact
# rational brute force, odd symmetry and the dequantized values.

def test_symmetric_worked_examples(orc):
    n_lines = 0
    with open(os.path.join(GOLDEN, "quant_symmetric_examples.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            head, ws, qs = [p.strip() for p in line.split("|")]
            bits, s_bits, z_bits = head.split()
            w = np.array([float(v) for v in ws.split()], np.float32)
            s, z, q = orc.quantize_group_symmetric(w, int(bits))
            assert (s, z) == (int(s_bits, 16), int(z_bits, 16))
            assert list(q) == [int(v) for v in qs.split()]
            n_lines += 1
    assert n_lines == 2


@pytest.mark.parametrize("bits", BITS)
def test_symmetric_scale_zero_and_range(orc, bits):
    """s16 = numpy fp16(max|w| / Q), z16 = numpy fp16(-2^(b-1) * s16) (exact),
    codes in [1, 2^b - 1], |w - q*s16| <= s16/2 unless clamped at +-Q."""
    rng = np.random.default_rng(70 + bits)
    half, Q = 1 << (bits - 1), (1 << (bits - 1)) - 1
    for _ in range(200):
        w = (rng.normal(0, 0.02, 128) * rng.choice([1, 20], 128, p=[.99, .01])).astype(np.float32)
        s_b, z_b, codes = orc.quantize_group_symmetric(w, bits)
        amax = np.abs(w.astype(np.float64)).max()
        assert s_b == np.float16(amax / Q).view(np.uint16)
        s = float(np.uint16(s_b).view(np.float16))
        assert float(np.uint16(z_b).view(np.float16)) == -half * s
        q = codes.astype(np.int64) - half
        assert codes.min() >= 1 and codes.max() <= (1 << bits) - 1
        err = np.abs(w.astype(np.float64) - q * s)
        inside = np.abs(q) < Q
        assert np.all(err[inside] <= s / 2)
        assert np.all(err[~inside] <= max(s / 2, amax - Q * s) + 1e-300)


@pytest.mark.parametrize("bits", BITS)
def test_symmetric_odd_symmetry(orc, bits):
    """Negating the group negates every q and keeps the scale (round half to
    even is symmetric about zero)."""
    rng = np.random.default_rng(80 + bits)
    half = 1 << (bits - 1)
    for _ in range(50):
        w = rng.normal(0, 0.02, 128).astype(np.float32)
        s1, z1, c1 = orc.quantize_group_symmetric(w, bits)
        s2, z2, c2 = orc.quantize_group_symmetric(-w, bits)
        assert (s1, z1) == (s2, z2)
        assert np.array_equal(c1.astype(int) - half, -(c2.astype(int) - half))


@pytest.mark.parametrize("bits", BITS)
def test_symmetric_brute_force_exact(orc, bits):
    """Exhaustive search over q in [-Q, Q] with exact rationals: the chosen q
    minimises |w - q*s16|, ties to the even q."""
    rng = np.random.default_rng(90 + bits)
    half, Q = 1 << (bits - 1), (1 << (bits - 1)) - 1
    for trial in range(40):
        n = int(rng.integers(2, 24))
        w = (rng.normal(0, 0.02, n) * (20 if trial % 7 == 0 else 1)).astype(np.float32)
        s_b, _, codes = orc.quantize_group_symmetric(w, bits)
        s = Fraction(float(np.uint16(s_b).view(np.float16)))
        for i in range(n):
            wi = Fraction(float(w[i]))
            best = None
            for cand in range(-Q, Q + 1):
                d = abs(wi - cand * s)
                if best is None or d < best[0] or (d == best[0] and cand % 2 == 0):
                    best = (d, cand)
            assert int(codes[i]) - half == best[1], (trial, i, codes[i], best)


@pytest.mark.parametrize("bits", BITS)
def test_symmetric_dequant_is_q_times_scale(orc, bits):
    """Through the ordinary dequantizer (code*s16 + z16) a symmetric tensor
    gives exactly q*s16, computed here in numpy from the bit fields."""
    rng = np.random.default_rng(100 + bits)
    N, K = 4, 384
    half = 1 << (bits - 1)
    w = rng.normal(0, 0.02, (N, K)).astype(np.float32)
    w[1, 128:256] = 0.0                                   # an all-zero group
    packed, scales, zeros = orc.quantize_pack_symmetric(w, bits)
    codes = np.stack([_stream_codes_numpy(packed[n], K, bits) for n in range(N)]).astype(np.int64)
    s = scales.view(np.float16).astype(np.float64).repeat(128, axis=1)
    assert np.array_equal(orc.dequant(packed, scales, zeros, bits, N, K), (codes - half) * s)
    assert scales[1, 1] == 0 and np.all(codes[1, 128:256] == half)
    for n in range(N):
        for g in range(K // 128):
            sg, zg, cg = orc.quantize_group_symmetric(w[n, g * 128:(g + 1) * 128], bits)
            assert scales[n, g] == sg and zeros[n, g] == zg
            assert np.array_equal(codes[n, g * 128:(g + 1) * 128], cg)


def test_symmetric_rejects(orc):
    for bad in (np.nan, np.inf, 65505.0):
        w = np.zeros(128, np.float32)
        w[5] = bad
        with pytest.raises(orc.OracleError) as e:
            orc.quantize_group_symmetric(w, 8)
        assert e.value.status == orc.NONFINITE
    # zero = -2^(b-1)*scale must be a finite fp16: 65400/127 -> 515, 128*515 > 65504
    for bits, big in ((8, 65400.0), (2, 40000.0)):
        w = np.zeros(128, np.float32)
        w[0] = big
        with pytest.raises(orc.OracleError) as e:
            orc.quantize_group_symmetric(w, bits)
        assert e.value.status == orc.NONFINITE
    w = np.zeros(128, np.float32)
    w[0] = 32000.0                     # 128 * fp16(32000/127) = 32256: storable
    orc.quantize_group_symmetric(w, 8)
    with pytest.raises(orc.OracleError) as e:
        orc.quantize_pack_symmetric(np.zeros((2, 256), np.float32), 5)
    assert e.value.status == orc.UNSUPPORTED


# ------------------------------------------------------------ dequant/linear --

def _numpy_dequant(packed, scales, zeros, bits, N, K):
    codes = np.stack([_stream_codes_numpy(packed[n], K, bits) for n in range(N)])
    s = scales.view(np.float16).astype(np.float64).repeat(128, axis=1)
    z = zeros.view(np.float16).astype(np.float64).repeat(128, axis=1)
    return codes * s + z


@pytest.mark.parametrize("bits", BITS)
def test_dequant_matches_numpy_decode(orc, bits):
    rng = np.random.default_rng(70 + bits)
    N, K = 6, 384
    w = rng.normal(0, 0.02, (N, K)).astype(np.float32)
    packed, scales, zeros = orc.quantize_pack(w, bits)
    ref = _numpy_dequant(packed, scales, zeros, bits, N, K)
    assert np.array_equal(orc.dequant(packed, scales, zeros, bits, N, K), ref)


def _pack_codes(orc, codes, bits):
    return np.stack([orc.pack_row(c, bits) for c in codes])


@pytest.mark.parametrize("bits", BITS)
def test_linear_brute_force_integer(orc, bits):
    """s = 1, z = 0 and integer-valued x: y is an exact integer dot product."""
    rng = np.random.default_rng(80 + bits)
    for M in (1, 2, 3):
        for N in (1, 2, 3):
            K = 128
            codes = rng.integers(0, 1 << bits, (N, K)).astype(np.uint8)
            xi = rng.integers(-8, 9, (M, K))
            x16 = xi.astype(np.float16).view(np.uint16)
            scales = np.full((N, 1), 0x3C00, np.uint16)     # 1.0
            zeros = np.zeros((N, 1), np.uint16)
            y, bound = orc.linear(x16, _pack_codes(orc, codes, bits), scales, zeros, bits, N, K)
            for m in range(M):
                for n in range(N):
                    exact = sum(int(xi[m, k]) * int(codes[n, k]) for k in range(K))
                    assert y[m, n] == exact
                    assert bound[m, n] == sum(abs(int(xi[m, k])) * int(codes[n, k]) for k in range(K))


def test_linear_zero_scale_rows(orc):
    """With s16 = 0 in every group the row reduces to z16 * sum(x) per group."""
    rng = np.random.default_rng(90)
    M, N, K = 3, 4, 256
    codes = rng.integers(0, 16, (N, K)).astype(np.uint8)
    zeros_f = rng.normal(0, 0.05, (N, 2)).astype(np.float16)
    scales = np.zeros((N, 2), np.uint16)
    x = rng.normal(0, 1, (M, K)).astype(np.float16)
    y, _ = orc.linear(x.view(np.uint16), _pack_codes(orc, codes, 4), scales,
                      zeros_f.view(np.uint16), 4, N, K)
    xd = x.astype(np.float64)
    for m in range(M):
        for n in range(N):
            exp = zeros_f[n, 0] * xd[m, :128].sum() + zeros_f[n, 1] * xd[m, 128:].sum()
            assert abs(y[m, n] - float(exp)) <= 1e-12 * (1 + abs(float(exp)))


@pytest.mark.parametrize("bits", BITS)
def test_linear_matches_numpy_matmul(orc, bits):
    """Oracle linear vs numpy fp64 matmul of an independently decoded W."""
    rng = np.random.default_rng(100 + bits)
    M, N, K = 5, 19, 640
    w = rng.normal(0, 0.02, (N, K)).astype(np.float32)
    packed, scales, zeros = orc.quantize_pack(w, bits)
    x = rng.normal(0, 1, (M, K)).astype(np.float16)
    y, bound = orc.linear(x.view(np.uint16), packed, scales, zeros, bits, N, K)
    wd = _numpy_dequant(packed, scales, zeros, bits, N, K)
    xd = x.astype(np.float64)
    ref = xd @ wd.T
    refb = np.abs(xd) @ np.abs(wd).T
    assert np.allclose(y, ref, rtol=1e-12, atol=1e-12)
    assert np.allclose(bound, refb, rtol=1e-12, atol=1e-12)
    assert np.all(bound >= np.abs(y))
    # row subset selects the same columns
    rows = np.array([18, 0, 7, 7], np.int64)
    ys, bs = orc.linear(x.view(np.uint16), packed, scales, zeros, bits, N, K, rows=rows)
    assert np.array_equal(ys, y[:, rows]) and np.array_equal(bs, bound[:, rows])


def test_linear_is_linear_in_x(orc):
    rng = np.random.default_rng(110)
    M, N, K = 2, 5, 256
    w = rng.normal(0, 0.02, (N, K)).astype(np.float32)
    packed, scales, zeros = orc.quantize_pack(w, 4)
    x1 = rng.integers(-4, 5, (M, K)).astype(np.float16)
    x2 = rng.integers(-4, 5, (M, K)).astype(np.float16)
    y1, _ = orc.linear(x1.view(np.uint16), packed, scales, zeros, 4, N, K)
    y2, _ = orc.linear(x2.view(np.uint16), packed, scales, zeros, 4, N, K)
    y12, _ = orc.linear((x1 + x2).view(np.uint16), packed, scales, zeros, 4, N, K)
    assert np.allclose(y12, y1 + y2, rtol=0, atol=1e-12)
    # W-side: transposing x and W is a plausible slip; y[m][n] uses row n of W
    e = np.zeros((1, K), np.float16)
    e[0, 3] = 1.0
    ye, _ = orc.linear(e.view(np.uint16), packed, scales, zeros, 4, N, K)
    wd = orc.dequant(packed, scales, zeros, 4, N, K)
    assert np.array_equal(ye[0], wd[:, 3])


def test_size_closed_form(orc):
    """Bytes per weight = b/8 + 4/128 (codes + fp16 scale + fp16 zero per 128)."""
    for bits in BITS:
        N, K = 3, 1024
        packed, scales, zeros = orc.quantize_pack(np.zeros((N, K), np.float32), bits)
        nbytes = packed.nbytes + scales.nbytes + zeros.nbytes
        assert nbytes == N * K * (bits / 8 + 4 / 128)
