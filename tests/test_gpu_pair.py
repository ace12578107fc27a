"""GPU parity of the tile kernel's CTA-pair plan (tcgen05.mma.cta_group::2:
a cluster of two CTAs computes a 512-token x 256-row tile, each CTA
dequantizing its own 128 weight rows), which runs every launch of b-bit codes
with some M >= 512, against the fp64 oracle at the tolerance
|y - y_ref| <= 2e-3 * sum|x||w_hat| + 1e-3.

Cases: ragged token tiles (a last tile whose second 256-token half is empty,
and one where it holds a few tokens), ragged weight-row tiles (N not a multiple
of 256, nor of 8), several ops of different K in one launch, groups of 32 and
64, bfloat16 activations, and fp32 partial sums.
"""
import numpy as np
import pytest
import torch

import zq_inputs as zi
from zq_testutil import assert_linear_close, u16, u32

pytestmark = pytest.mark.gpu

BITS = (2, 3, 4, 8)


@pytest.fixture(scope="module")
def zq():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import weight_only_quantized_zq_b200 as m
    return m


def _quantize(zq, orc, N, K, bits, seed, group=128):
    w = zi.weight(N, K, seed=seed, device="cuda", outliers=True)
    q = zq.quantize(w, bits, group=group)
    torch.cuda.synchronize()
    ref = orc.quantize_pack(w.cpu().numpy(), bits, group=group)
    assert np.array_equal(u32(q[0]).reshape(N, -1), ref[0]), "packed codes differ"
    return q, ref


@pytest.mark.parametrize("bits", BITS)
def test_pair_ragged_tiles(zq, orc, bits):
    # M = 520: tiles at t0 = 0 (both halves) and t0 = 512 (first half, 8 tokens);
    # M = 780: second tile's second half holds 12 tokens; N ragged by 8 and by 1
    for i, (M, N, K) in enumerate(((520, 264, 640), (780, 257, 384), (512, 512, 1152), (600, 100, 256))):
        q, ref = _quantize(zq, orc, N, K, bits, 9100 + 10 * bits + i)
        x = zi.activations(M, K, seed=9200 + i, device="cuda")
        y = zq.linear(x, *q, bits, N)
        torch.cuda.synchronize()
        y_ref, bound = orc.linear(u16(x), *ref, bits, N, K)
        assert_linear_close(y, y_ref, bound, f"pair bits={bits} M={M} N={N} K={K}")


def test_pair_stack_of_different_k(zq, orc):
    """One launch over ops whose K differ (tiles of unequal length, assigned
    to the pairs in turn) and whose M differ (one below 512 in a pair launch)."""
    specs = [(640, 300, 1280), (520, 264, 384), (300, 130, 640), (700, 520, 3584)]
    layers = [_quantize(zq, orc, N, K, 4, 9300 + i) for i, (M, N, K) in enumerate(specs)]
    xs = [zi.activations(M, K, seed=9400 + i, device="cuda") for i, (M, N, K) in enumerate(specs)]
    outs = [torch.empty(M, N, dtype=torch.float16, device="cuda") for (M, N, K) in specs]
    zq.linear_stack([(xs[i], *layers[i][0], outs[i], 4, 128, M, N, K) for i, (M, N, K) in enumerate(specs)])
    torch.cuda.synchronize()
    for i, (M, N, K) in enumerate(specs):
        y_ref, bound = orc.linear(u16(xs[i]), *layers[i][1], 4, N, K)
        assert_linear_close(outs[i], y_ref, bound, f"pair stack op {i} M={M} N={N} K={K}")


@pytest.mark.parametrize("group", (32, 64))
def test_pair_small_groups(zq, orc, group):
    for bits in BITS:
        M, N, K = 530, 270, 512
        q, ref = _quantize(zq, orc, N, K, bits, 9500 + bits + group, group=group)
        x = zi.activations(M, K, seed=9600 + bits, device="cuda")
        y = zq.linear(x, *q, bits, N, group=group)
        torch.cuda.synchronize()
        y_ref, bound = orc.linear(u16(x), *ref, bits, N, K, group=group)
        assert_linear_close(y, y_ref, bound, f"pair group={group} bits={bits}")


def test_pair_bf16_activations(zq, orc):
    M, N, K = 600, 264, 768
    q, ref = _quantize(zq, orc, N, K, 4, 9700)
    for scale in (1.0, 1e-6, 1e4):
        g = torch.Generator().manual_seed(9701)
        x = (torch.randn(M, K, generator=g) * scale).to(torch.bfloat16).cuda()
        y = zq.linear(x, *q, 4, N)
        torch.cuda.synchronize()
        assert y.dtype == torch.bfloat16
        y_ref, bound = orc.linear(u16(x), *ref, 4, N, K, xfmt="bf16")
        yg = y.float().cpu().numpy().astype(np.float64)
        lim = 2e-3 * bound + 1e-3 + 2.0 ** -9 * np.abs(y_ref)
        assert np.all(np.abs(yg - y_ref) <= lim), f"pair bf16 scale={scale}"


def test_pair_partial_sums(zq, orc):
    """fp32 partial sums (out32) from the pair epilogue, unrounded."""
    M, N, K = 700, 300, 640
    q, ref = _quantize(zq, orc, N, K, 3, 9800)
    x = zi.activations(M, K, seed=9801, device="cuda")
    y = zq.linear_partial(x, *q, 3, N)
    torch.cuda.synchronize()
    assert y.dtype == torch.float32
    y_ref, bound = orc.linear(u16(x), *ref, 3, N, K)
    assert_linear_close(y, y_ref, bound, "pair fp32 partial sums")
