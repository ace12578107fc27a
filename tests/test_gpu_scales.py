"""GPU parity of the tile kernel's scale/zero loading against the fp64 oracle,
|y - y_ref| <= 2e-3 * sum|x||w_hat| + 1e-3.

With groups of 128 the one-token-half plan loads the scales (and zeros) of
two consecutive groups with one 4-byte load when a row holds an even number of
groups, and one group at a time when it holds an odd number; every plan keeps
the loaded values unpacked until their block is used.  The cases cover each
plan (M = 40 and 100: one token half with 64- and 128-token x stages; M = 200:
two token halves; M = 520: CTA pairs) with an odd and an even number of groups
per row, and launches whose ops mix the two, so that consecutive tiles of one
CTA switch between the loading modes.
"""
import pytest
import torch

import zq_inputs as zi
from zq_testutil import assert_linear_close, u16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def zq():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import weight_only_quantized_zq_b200 as m
    return m


def _layer(zq, orc, N, K, bits, seed):
    w = zi.weight(N, K, seed=seed, device="cuda", outliers=True)
    q = zq.quantize(w, bits)
    torch.cuda.synchronize()
    return q, orc.quantize_pack(w.cpu().numpy(), bits)


@pytest.mark.parametrize("bits", (2, 3, 4, 8))
@pytest.mark.parametrize("M", (40, 100, 200, 520))
@pytest.mark.parametrize("K", (384, 1024, 1408))
def test_scale_loading_modes(zq, orc, bits, M, K):
    # K = 384 and 1408: 3 and 11 groups per row (one group per load); K = 1024: 8 (pairs)
    N = 264
    q, ref = _layer(zq, orc, N, K, bits, 9900 + 7 * bits + K)
    x = zi.activations(M, K, seed=9950 + M, device="cuda")
    y = zq.linear(x, *q, bits, N)
    torch.cuda.synchronize()
    y_ref, bound = orc.linear(u16(x), *ref, bits, N, K)
    assert_linear_close(y, y_ref, bound, f"bits={bits} M={M} K={K}")


@pytest.mark.parametrize("M", (60, 120, 300))
def test_mixed_modes_in_one_launch(zq, orc, M):
    """Ops with odd and even group counts in one launch."""
    specs = [(300, 640), (264, 1024), (130, 384), (520, 2048), (257, 1152)]
    layers = [_layer(zq, orc, N, K, 4, 9970 + i) for i, (N, K) in enumerate(specs)]
    xs = [zi.activations(M, K, seed=9980 + i, device="cuda") for i, (N, K) in enumerate(specs)]
    outs = [torch.empty(M, N, dtype=torch.float16, device="cuda") for (N, K) in specs]
    zq.linear_stack([(xs[i], *layers[i][0], outs[i], 4, 128, M, N, K) for i, (N, K) in enumerate(specs)])
    torch.cuda.synchronize()
    for i, (N, K) in enumerate(specs):
        y_ref, bound = orc.linear(u16(xs[i]), *layers[i][1], 4, N, K)
        assert_linear_close(outs[i], y_ref, bound, f"op {i} N={N} K={K}")
