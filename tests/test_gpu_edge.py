"""GPU parity on the method's edge cases, through both linear kernel families
(decode kernel for M <= 32, tcgen05 tile kernel above) against the fp64 oracle
at the tolerance |y_gpu - y_ref| <= 2e-3 * sum|x||w_hat| + 1e-3.

The quantizer of "ZSE - open-source движок для запуска LLM локально на GPU -
2026", section "Формат модели .zse" (scale = (max - min) / L, zero = min) has
degenerate groups where the two kernel families part ways: the decode kernel
applies scale and zero once per group in fp32 (s * sum q x + z * sum x), the
tile kernel rounds every weight to fp16(q * s + z).  These tests put whole
groups of each kind through both:

  * constant groups (scale 0, every weight equal to the zero);
  * groups whose fp16 scale is subnormal (range about 1e-6);
  * a large zero with a tiny scale (|z| >> s * L);
  * a single outlier with every other code 0;
  * groups spanning the whole fp16 range (+-65504, where the top code's
    q * s + z rounds past the largest fp16);
mixed with ordinary groups in the same rows, and activations whose magnitudes
run from about 1e-6 (fp16 subnormals) to 1e2.
"""
import numpy as np
import pytest
import torch

import zq_inputs as zi
from zq_testutil import assert_linear_close, u16, u32

pytestmark = pytest.mark.gpu

BITS = (2, 3, 4, 8)
G = 128


@pytest.fixture(scope="module")
def zq():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import weight_only_quantized_zq_b200 as m
    return m


def _edge_weights(N, K, seed, scale=1.0):
    """fp32 N x K: every row cycles through the edge-group kinds, one group
    each, starting at a row-dependent kind so every kind meets every column of
    groups; `scale` multiplies the ordinary and outlier groups."""
    g = torch.Generator().manual_seed(seed)
    w = torch.randn(N, K, generator=g) * 0.02 * scale
    kinds = 6
    for n in range(N):
        for j in range(K // G):
            kind = (n + j) % kinds
            sl = slice(j * G, (j + 1) * G)
            if kind == 0:    # constant group: scale 0
                w[n, sl] = 0.0123 * scale
            elif kind == 1:  # subnormal fp16 scale
                w[n, sl] = torch.rand(G, generator=g) * 1e-6
            elif kind == 2:  # large zero, tiny scale
                w[n, sl] = -3.0 * scale + torch.rand(G, generator=g) * 1e-3 * scale
            elif kind == 3:  # one outlier, every other code 0
                w[n, sl] = 0.0
                w[n, j * G + (n * 7 + j) % G] = 5.0 * scale
            # kinds 4, 5: ordinary N(0, 0.02 * scale) groups
    return w.contiguous()


def _x_mixed(M, K, seed):
    """Token m has magnitude 10^e with e cycling through 0, -4, -6, 2, -2, -5:
    rows whose x * 2^-s would sit in fp16's subnormal range or flush to 0."""
    g = torch.Generator().manual_seed(seed)
    mags = (1.0, 1e-4, 1e-6, 1e2, 1e-2, 1e-5)
    x = torch.randn(M, K, generator=g)
    for m in range(M):
        x[m] *= mags[m % len(mags)]
    return x.to(torch.float16)


def _run(zq, orc, w, x, bits, what):
    N, K = w.shape
    M = x.shape[0]
    w = w.cuda()
    packed, scales, zeros = zq.quantize(w, bits)
    torch.cuda.synchronize()
    p_ref, s_ref, z_ref = orc.quantize_pack(w.cpu().numpy(), bits)
    assert np.array_equal(u32(packed).reshape(N, -1), p_ref), f"{what}: packed codes differ"
    assert np.array_equal(u16(scales).reshape(N, -1), s_ref), f"{what}: scales differ"
    assert np.array_equal(u16(zeros).reshape(N, -1), z_ref), f"{what}: zeros differ"
    xd = x.cuda()
    y = zq.linear(xd, packed, scales, zeros, bits, N)
    torch.cuda.synchronize()
    y_ref, bound = orc.linear(u16(xd), p_ref, s_ref, z_ref, bits, N, K)
    assert_linear_close(y, y_ref, bound, what)


@pytest.mark.parametrize("bits", BITS)
@pytest.mark.parametrize("M", (1, 8, 16, 24, 40, 300))
def test_edge_groups_mixed_activations(zq, orc, bits, M):
    """Edge groups of ordinary magnitude with activations from 1e-6 to 1e2."""
    N, K = 96, 768
    w = _edge_weights(N, K, seed=800 + bits)
    x = _x_mixed(M, K, seed=900 + M)
    _run(zq, orc, w, x, bits, f"edge groups bits={bits} M={M}")


@pytest.mark.parametrize("bits", BITS)
@pytest.mark.parametrize("M", (1, 8, 16, 24, 40, 300))
def test_edge_groups_full_fp16_range(zq, orc, bits, M):
    """Large weights (ordinary groups N(0, 200), outliers 5e3, groups spanning
    -65504..65504) with tiny activations (|x| about 1e-5, many fp16 subnormals),
    so y stays finite while the bound sum |x||w_hat| is far above 1: the
    tolerance is then relative, and losing the small activations' bits (decode)
    or rounding a weight to +inf (tile) would fail it."""
    N, K = 64, 640
    w = _edge_weights(N, K, seed=1800 + bits, scale=1e4)
    for n in range(0, N, 3):  # one full-range group per third row
        j = (n // 3) % (K // G)
        w[n, j * G:(j + 1) * G] = torch.linspace(-65504.0, 65504.0, G)
    w.clamp_(-65504.0, 65504.0)
    g = torch.Generator().manual_seed(1900 + M)
    x = (torch.randn(M, K, generator=g) * 1e-5).to(torch.float16)
    _run(zq, orc, w, x, bits, f"full fp16 range bits={bits} M={M}")


@pytest.mark.parametrize("bits", BITS)
def test_tiny_activations_ordinary_weights(zq, orc, bits):
    """Whole rows of tiny activations (1e-4 .. 1e-6) with weights scaled so
    the bound is well above the absolute tolerance: the decode kernel's
    pre-scaled activations must keep their precision."""
    N, K = 200, 1024
    w = zi.weight(N, K, seed=2100 + bits) * 5e4
    w.clamp_(-65504.0, 65504.0)
    for M, mag in ((1, 1e-4), (4, 1e-5), (9, 1e-6), (24, 1e-6), (40, 1e-6)):
        g = torch.Generator().manual_seed(2200 + M)
        x = (torch.randn(M, K, generator=g) * mag).to(torch.float16)
        _run(zq, orc, w, x, bits, f"tiny x bits={bits} M={M} |x|~{mag}")


def test_constant_rows_reduce_to_zero_times_sum_x(zq, orc):
    """Rows made only of constant groups: w_hat = z, so y = z * sum(x) (the
    oracle's closed form), on both families."""
    N, K = 33, 512
    w = torch.zeros(N, K)
    for n in range(N):
        w[n] = (n - 16) * 0.37
    for M in (1, 16, 17, 40, 130):
        x = zi.activations(M, K, seed=2300 + M)
        _run(zq, orc, w, x, 4, f"constant rows M={M}")
