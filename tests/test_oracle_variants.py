"""Pins for the oracle's encoding variants, checked against things other than
the oracle itself: numpy's float16 and torch's bfloat16 conversions, exact
rational brute force, integer and power-of-two closed forms, and numpy fp64
matmuls of independently decoded operands.

Variants (the .zse format section of "ZSE - open-source движок для запуска LLM
локально на GPU - 2026" keeps some tensors as fp16 and lists other encodings):
  * group sizes 32 and 64 besides 128: the same min/max quantizer per group;
  * fp16 passthrough: bits = 16, the weights used as their fp16 values;
  * bf16 activations: x given as bfloat16, decoded exactly.
"""
from fractions import Fraction

import numpy as np
import pytest
import torch

BITS = (2, 3, 4, 8)
GROUPS = (32, 64)


# --------------------------------------------------------------- bfloat16 --

def test_bf16_decode_exhaustive(orc):
    """Every bfloat16 pattern decodes to the binary32 whose top half it is."""
    pats = np.arange(65536, dtype=np.uint32)
    with np.errstate(invalid="ignore"):
        ref = (pats << 16).astype(np.uint32).view(np.float32).astype(np.float64)
    got = np.array([orc.bf16_to_f64(int(b)) for b in pats])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])


def test_bf16_encode_matches_torch(orc):
    """Round to nearest even, as torch converts float32 to bfloat16: random
    values over the whole range, exact midpoints, subnormals, the overflow edge."""
    rng = np.random.default_rng(3)
    vals = np.concatenate([rng.normal(0, 1, 2000), rng.normal(0, 1e-3, 500) * 10.0 ** rng.integers(-30, 30, 500),
                           np.ldexp(rng.uniform(1, 2, 300), rng.integers(-140, -120, 300))]).astype(np.float32)
    # midpoints between neighbouring bfloat16 values (ties to even)
    base = (np.arange(1, 400, dtype=np.uint32) * 97 + 0x3F80).astype(np.uint32)
    mids = ((base << 16) | 0x8000).view(np.float32)
    big = np.array([3.3895314e38, 3.3961775e38, -3.3961775e38], np.float32)  # max, midpoint above it
    vals = np.concatenate([vals, mids[np.isfinite(mids)], big])
    ref = torch.from_numpy(vals).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = np.array([orc.f64_to_bf16(float(v)) for v in vals], np.uint16)
    assert np.array_equal(got, ref)


# ----------------------------------------------------------- group 32, 64 --

@pytest.mark.parametrize("bits", BITS)
@pytest.mark.parametrize("group", GROUPS)
def test_small_groups_reshape_invariance(orc, bits, group):
    """A group never straddles words (group*bits is a multiple of 32), so
    quantizing W with groups of g gives the same bytes as quantizing the
    N*K/g rows of g weights of W.reshape(-1, g)."""
    rng = np.random.default_rng(bits * 7 + group)
    N, K = 6, 384
    w = (rng.normal(0, 0.02, (N, K)) * np.where(rng.random((N, K)) < 0.01, 20, 1)).astype(np.float32)
    p, s, z = orc.quantize_pack(w, bits, group=group)
    assert p.shape == (N, K * bits // 32) and s.shape == (N, K // group)
    p2, s2, z2 = orc.quantize_pack(w.reshape(-1, group), bits, group=group)
    assert np.array_equal(p.reshape(-1), p2.reshape(-1))
    assert np.array_equal(s.reshape(-1), s2.reshape(-1)) and np.array_equal(z.reshape(-1), z2.reshape(-1))


@pytest.mark.parametrize("bits", BITS)
@pytest.mark.parametrize("group", GROUPS)
def test_small_groups_brute_force_exact(orc, bits, group):
    """Each stored code minimises |w - (q*s16 + z16)| over q in [0, L] (exact
    rationals, ties to even), with s16 and z16 the fp16 of (max-min)/L and min
    of ITS group of g weights."""
    rng = np.random.default_rng(200 + bits + group)
    L = (1 << bits) - 1
    N, K = 2, 2 * group
    w = rng.normal(0, 0.02, (N, K)).astype(np.float32)
    p, s, z = orc.quantize_pack(w, bits, group=group)
    codes = orc.unpack(p, N, K, bits)
    for n in range(N):
        for g in range(K // group):
            seg = w[n, g * group:(g + 1) * group].astype(np.float64)
            assert s[n, g] == np.float16((seg.max() - seg.min()) / L).view(np.uint16)
            assert z[n, g] == np.float16(seg.min()).view(np.uint16)
            sf = Fraction(float(np.uint16(s[n, g]).view(np.float16)))
            zf = Fraction(float(np.uint16(z[n, g]).view(np.float16)))
            for i in range(0, group, 5):  # a sample of each group
                wi = Fraction(float(seg[i]))
                best = min(range(L + 1), key=lambda c: (abs(wi - (c * sf + zf)), c % 2))
                assert codes[n, g * group + i] == best


@pytest.mark.parametrize("group", GROUPS + (128,))
def test_small_groups_linear_power_of_two_scales(orc, group):
    """Codes 1, zero 0, and scale 2^(g mod 7) in group g: y = sum over groups of
    2^(g mod 7) * (sum of that group's x), exact -- pins which scale each k uses."""
    rng = np.random.default_rng(group)
    M, N, K, bits = 3, 2, 512, 4
    G = K // group
    codes = np.ones((N, K), np.uint8)
    packed = np.stack([orc.pack_row(c, bits) for c in codes])
    sc = np.array([[np.float16(2.0 ** (g % 7)) for g in range(G)]] * N).view(np.uint16)
    zr = np.zeros((N, G), np.uint16)
    xi = rng.integers(-8, 9, (M, K))
    y, _ = orc.linear(xi.astype(np.float16).view(np.uint16), packed, sc, zr, bits, N, K, group=group)
    for m in range(M):
        exact = sum(2 ** (g % 7) * int(xi[m, g * group:(g + 1) * group].sum()) for g in range(G))
        assert np.all(y[m] == exact)


@pytest.mark.parametrize("group", GROUPS)
def test_small_groups_linear_matches_numpy(orc, group):
    rng = np.random.default_rng(300 + group)
    M, N, K = 4, 9, 640
    for bits in BITS:
        w = rng.normal(0, 0.02, (N, K)).astype(np.float32)
        p, s, z = orc.quantize_pack(w, bits, group=group)
        codes = orc.unpack(p, N, K, bits).astype(np.float64)
        sd = np.repeat(s.view(np.float16).astype(np.float64), group, axis=1)
        zd = np.repeat(z.view(np.float16).astype(np.float64), group, axis=1)
        wd = codes * sd + zd
        x = rng.normal(0, 1, (M, K)).astype(np.float16)
        y, bound = orc.linear(x.view(np.uint16), p, s, z, bits, N, K, group=group)
        assert np.allclose(y, x.astype(np.float64) @ wd.T, rtol=1e-12, atol=1e-12)
        assert np.allclose(bound, np.abs(x.astype(np.float64)) @ np.abs(wd).T, rtol=1e-12, atol=1e-12)


def test_group_sizes_rejected(orc):
    w = np.zeros((2, 256), np.float32)
    for g in (16, 48, 256):
        with pytest.raises(orc.OracleError) as e:
            orc.quantize_pack(w, 4, group=g)
        assert e.value.status == orc.UNSUPPORTED


# ------------------------------------------------- fp16 weights, bf16 x --

def test_fp16_weights_match_numpy(orc):
    """bits = 16: y = x W^T with W's fp16 values (numpy decodes both)."""
    rng = np.random.default_rng(7)
    M, N, K = 5, 13, 384  # K need not be a multiple of 128 for fp16 weights
    for K in (384, 200):
        w = (rng.normal(0, 0.05, (N, K))).astype(np.float16)
        x = rng.normal(0, 1, (M, K)).astype(np.float16)
        y, bound = orc.linear(x.view(np.uint16), w.view(np.uint16), None, None, 16, N, K)
        xd, wd = x.astype(np.float64), w.astype(np.float64)
        assert np.allclose(y, xd @ wd.T, rtol=1e-12, atol=1e-12)
        assert np.allclose(bound, np.abs(xd) @ np.abs(wd).T, rtol=1e-12, atol=1e-12)


def test_bf16_activations_match_numpy(orc):
    rng = np.random.default_rng(8)
    M, N, K, bits = 4, 11, 512, 4
    w = rng.normal(0, 0.02, (N, K)).astype(np.float32)
    p, s, z = orc.quantize_pack(w, bits)
    xt = torch.from_numpy(rng.normal(0, 3, (M, K)).astype(np.float32)).to(torch.bfloat16)
    xb = xt.view(torch.int16).numpy().view(np.uint16)
    y, _ = orc.linear(xb, p, s, z, bits, N, K, xfmt="bf16")
    y16, _ = orc.linear(np.zeros_like(xb), p, s, z, bits, N, K)
    wd = orc.dequant(p, s, z, bits, N, K)
    assert np.allclose(y, xt.double().numpy() @ wd.T, rtol=1e-12, atol=1e-12)
    assert np.all(y16 == 0)
