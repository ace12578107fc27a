"""zq_linear_noalloc: the allocation-free variant of zq_linear for callers that
cannot allocate device memory (inside a stream capture, under a fixed memory
budget, or on paths that must not risk the synchronisation of cudaMalloc).

On two calls in a row (the fixed scratch array keeps the previous call's
contents) its output must meet the fp64 oracle's tolerance, and match
zq_linear's output within the same tolerance, whether this file runs alone in
a fresh process or after every other test.
"""
import numpy as np
import pytest
import torch

import zq_inputs as zi
from zq_testutil import assert_linear_close, u16, u32

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def zq():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import weight_only_quantized_zq_b200 as m
    return m


@pytest.mark.parametrize("bits", (2, 3, 4, 8))
def test_noalloc_matches_zq_linear(zq, orc, bits):
    cases = [(1, 512, 512), (3, 4608, 3584), (8, 257, 1280), (1, 3584, 18944)]
    for i, (M, N, K) in enumerate(cases):
        w = zi.weight(N, K, seed=7000 + 10 * bits + i, device="cuda")
        packed, scales, zeros = zq.quantize(w, bits)
        x = zi.activations(M, K, seed=7100 + i, device="cuda")
        ref = zq.linear(x, packed, scales, zeros, bits, N)
        torch.cuda.synchronize()
        p_ref = u32(packed).reshape(N, -1)
        y_ref, bound = orc.linear(u16(x), p_ref, u16(scales).reshape(N, -1), u16(zeros).reshape(N, -1),
                                  bits, N, K)
        lin64 = ref.float().cpu().numpy().astype(np.float64)
        for call in range(2):  # two calls in a row share the scratch array
            out = torch.full((M, N), float("nan"), dtype=torch.float16, device="cuda")
            zq.zq_linear_noalloc(x, packed, scales, zeros, bits, 128, M, N, K, out)
            torch.cuda.synchronize()
            what = f"noalloc call {call} bits={bits} M={M} N={N} K={K}"
            assert_linear_close(out, y_ref, bound, what + " vs the oracle")
            assert_linear_close(out, lin64, bound, what + " vs zq_linear")
    zq.zq_check_device()


def test_noalloc_rejects_beyond_limit(zq):
    w = zi.weight(64, 256, seed=1, device="cuda")
    packed, scales, zeros = zq.quantize(w, 4)
    x = zi.activations(9, 256, seed=2, device="cuda")
    out = torch.empty(9, 64, dtype=torch.float16, device="cuda")
    with pytest.raises(zq.ZQError) as e:
        zq.zq_linear_noalloc(x, packed, scales, zeros, 4, 128, 9, 64, 256, out)
    assert e.value.status == zq.ZQ_ERR_UNSUPPORTED
    assert "M <= 8" in str(e.value)
