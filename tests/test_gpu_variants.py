"""GPU parity of the encoding variants against the fp64 oracle:

  * group sizes 32 and 64 (besides 128): zq_quantize_pack and its symmetric
    variant bit-exact, the linear (tcgen05 tile kernel at every M) within
    |y - y_ref| <= 2e-3 * sum|x||w_hat| + 1e-3;
  * fp16 passthrough (bits = 16, the .zse format's unquantized tensors):
    the linear on both kernel families, alone and inside a stack with
    quantized ops, at the same tolerance;
  * bfloat16 activations and outputs (zq_linear_bf16, zq_linear_stack_bf16),
    at that tolerance plus the bf16 rounding of the output.
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


def _quantize_both(zq, orc, w, bits, group, symmetric=False):
    N, K = w.shape
    q = zq.quantize(w, bits, symmetric=symmetric, group=group)
    torch.cuda.synchronize()
    fn = orc.quantize_pack_symmetric if symmetric else orc.quantize_pack
    ref = fn(w.cpu().numpy(), bits, group=group)
    assert np.array_equal(u32(q[0]).reshape(N, -1), ref[0]), "packed codes differ"
    assert np.array_equal(u16(q[1]).reshape(N, -1), ref[1]), "scales differ"
    assert np.array_equal(u16(q[2]).reshape(N, -1), ref[2]), "zeros differ"
    return q, ref


@pytest.mark.parametrize("bits", BITS)
@pytest.mark.parametrize("group", (32, 64))
def test_small_groups_quantize_bit_exact(zq, orc, bits, group):
    for i, (N, K, outl) in enumerate(((1, 128, False), (37, 512, True), (5, 3584, True))):
        w = zi.weight(N, K, seed=8000 + 10 * bits + group + i, device="cuda", outliers=outl)
        _quantize_both(zq, orc, w, bits, group)
        _quantize_both(zq, orc, w, bits, group, symmetric=True)
    # edge groups: constant, ties, subnormal scales, one-signed
    K = 512
    w = torch.zeros(4, K)
    w[0] = 0.0123
    w[1] = torch.linspace(0, 1e-6, K)
    w[2] = torch.randn(K) * 1e-3 - 3.0
    w[3, ::3] = 1.0
    _quantize_both(zq, orc, w.cuda().contiguous(), bits, group)


@pytest.mark.parametrize("bits", BITS)
@pytest.mark.parametrize("group", (32, 64))
def test_small_groups_linear(zq, orc, bits, group):
    for i, (M, N, K) in enumerate(((1, 300, 512), (8, 257, 1280), (16, 64, 384), (40, 520, 640),
                                   (300, 264, 1024))):
        w = zi.weight(N, K, seed=8100 + 10 * bits + group + i, device="cuda", outliers=(i % 2 == 0))
        q, ref = _quantize_both(zq, orc, w, bits, group)
        x = zi.activations(M, K, seed=8200 + i, device="cuda")
        y = zq.linear(x, *q, bits, N, group=group)
        torch.cuda.synchronize()
        y_ref, bound = orc.linear(u16(x), *ref, bits, N, K, group=group)
        assert_linear_close(y, y_ref, bound, f"group={group} bits={bits} M={M} N={N} K={K}")


def _fp16_weights(N, K, seed):
    return (zi.weight(N, K, seed=seed, device="cuda", outliers=True) * 4).to(torch.float16).contiguous()


@pytest.mark.parametrize("M", (1, 3, 8, 9, 16, 17, 32, 33, 64, 130, 300))
def test_fp16_weights_linear(zq, orc, M):
    """bits = 16: decode kernel for M <= 32, tile kernel above (TMA-fed W)."""
    for i, (N, K) in enumerate(((1, 128), (130, 512), (520, 1280), (64, 3584))):
        w = _fp16_weights(N, K, 8300 + i)
        x = zi.activations(M, K, seed=8400 + i, device="cuda")
        y = zq.linear(x, w, None, None, 16, N)
        torch.cuda.synchronize()
        y_ref, bound = orc.linear(u16(x), u16(w), None, None, 16, N, K)
        assert_linear_close(y, y_ref, bound, f"fp16 weights M={M} N={N} K={K}")


def test_fp16_weights_in_a_stack(zq, orc):
    """Quantized ops, small-group ops and fp16-weight ops in one stack call,
    with a dependent chain through an fp16-weight op."""
    K = 512
    w16 = _fp16_weights(256, K, 8500)
    wq = zi.weight(384, K, seed=8501, device="cuda")
    q4, r4 = _quantize_both(zq, orc, wq, 4, 128)
    q3, r3 = _quantize_both(zq, orc, zi.weight(200, 256, seed=8502, device="cuda"), 3, 64)
    x = zi.activations(4, K, seed=8503, device="cuda")
    x40 = zi.activations(40, K, seed=8504, device="cuda")
    y16 = torch.empty(4, 256, dtype=torch.float16, device="cuda")
    y4 = torch.empty(4, 384, dtype=torch.float16, device="cuda")
    y16b = torch.empty(40, 256, dtype=torch.float16, device="cuda")
    y3 = torch.empty(4, 200, dtype=torch.float16, device="cuda")  # consumes y16 (K = 256)
    ops = [(x, w16, None, None, y16, 16, 128, 4, 256, K), (x, *q4, y4, 4, 128, 4, 384, K),
           (x40, w16, None, None, y16b, 16, 128, 40, 256, K), (y16, *q3, y3, 3, 64, 4, 200, 256)]
    zq.linear_stack(ops)
    torch.cuda.synchronize()
    for xin, y, args, N, KK, what in ((x, y16, (u16(w16), None, None, 16), 256, K, "fp16 M=4"),
                                      (x, y4, (*r4, 4), 384, K, "int4 M=4"),
                                      (x40, y16b, (u16(w16), None, None, 16), 256, K, "fp16 M=40"),
                                      (y16, y3, (*r3, 3), 200, 256, "int3 g64 after fp16")):
        group = 64 if what.startswith("int3") else 128
        y_ref, bound = orc.linear(u16(xin), *args, N, KK, group=group)
        assert_linear_close(y, y_ref, bound, f"stack {what}")


# ---------------------------------------------------- bf16 activations --
# The output is rounded to bfloat16 (8 significant bits) instead of fp16 (11):
# the fp16 tolerance 2e-3 * bound + 1e-3 already covers the fp16 rounding of
# the output (<= 2^-11 |y|), so bf16 adds at most 2^-9 |y_ref| on top of it.

def _assert_bf16_close(y, y_ref, bound, what):
    yg = y.float().cpu().numpy().astype(np.float64)
    assert np.all(np.isfinite(yg)), what
    lim = 2e-3 * bound + 1e-3 + 2.0 ** -9 * np.abs(y_ref)
    err = np.abs(yg - y_ref)
    assert np.all(err <= lim), f"{what}: worst {float((err / lim).max()):.3f} of the limit"


def _bf16_x(M, K, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(M, K, generator=g) * scale).to(torch.bfloat16).cuda()


@pytest.mark.parametrize("bits", BITS + (16,))
@pytest.mark.parametrize("M", (1, 8, 16, 24, 40, 300))
def test_bf16_activations(zq, orc, bits, M):
    """Both families; activation scales from 1e-6 to 1e4 per token block (bf16's
    range is fp32's, wider than fp16's)."""
    N, K = 264, 768
    if bits == 16:
        w = _fp16_weights(N, K, 8600 + M)
        q, ref = (w, None, None), (u16(w), None, None)
    else:
        q, ref = _quantize_both(zq, orc, zi.weight(N, K, seed=8600 + bits + M, device="cuda", outliers=True),
                                bits, 128)
    for scale in (1.0, 1e-6, 1e4):
        x = _bf16_x(M, K, 8700 + M, scale)
        y = zq.linear(x, *q, bits, N)
        torch.cuda.synchronize()
        assert y.dtype == torch.bfloat16
        y_ref, bound = orc.linear(u16(x), *ref, bits, N, K, xfmt="bf16")
        _assert_bf16_close(y, y_ref, bound, f"bf16 x bits={bits} M={M} scale={scale}")


def test_bf16_stack_matches_single_calls(zq, orc):
    """zq_linear_stack_bf16 over decode and tile ops, one chained."""
    K = 512
    q4, r4 = _quantize_both(zq, orc, zi.weight(384, K, seed=8800, device="cuda"), 4, 128)
    q8, r8 = _quantize_both(zq, orc, zi.weight(256, 384, seed=8801, device="cuda"), 8, 128)
    x1, x2 = _bf16_x(3, K, 8802), _bf16_x(70, K, 8803)
    y1 = torch.empty(3, 384, dtype=torch.bfloat16, device="cuda")
    y2 = torch.empty(70, 384, dtype=torch.bfloat16, device="cuda")
    y3 = torch.empty(3, 256, dtype=torch.bfloat16, device="cuda")  # from y1
    ops = [(x1, *q4, y1, 4, 128, 3, 384, K), (x2, *q4, y2, 4, 128, 70, 384, K), (y1, *q8, y3, 8, 128, 3, 256, 384)]
    arr, n = zq.make_descs(ops)
    zq.ensure_workspace(zq.zq_linear_stack_bf16_workspace_bytes(arr, n))
    zq.zq_linear_stack_bf16(arr, n)
    torch.cuda.synchronize()
    for xin, y, r, bits, N, KK in ((x1, y1, r4, 4, 384, K), (x2, y2, r4, 4, 384, K), (y1, y3, r8, 8, 256, 384)):
        y_ref, bound = orc.linear(u16(xin), *r, bits, N, KK, xfmt="bf16")
        _assert_bf16_close(y, y_ref, bound, f"bf16 stack bits={bits} M={xin.shape[0]}")
