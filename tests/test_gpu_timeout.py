"""Failure detection without a fault: the kernels' bounded waits.

Every spin-wait of the decode and tile kernels is bounded; a wait that runs
out makes the kernel stop, drain the copies and MMAs it already issued, free
its tensor memory and return, and zq_check_device reports ZQ_ERR_TIMEOUT.
The test makes the waits run out with the test hook zq_set_wait_limit_ns (a
zero limit: any wait not satisfied at its first poll gives up), then checks
that the device answers, the timeout is reported once, and the next ordinary
calls on the same streams (whose split-K counters the aborted decode launch may
have left set) match the fp64 oracle again.
"""
import pytest
import torch

import zq_inputs as zi
from zq_testutil import assert_linear_close, u16

pytestmark = pytest.mark.gpu

DEFAULT_LIMIT_NS = 2_000_000_000


@pytest.fixture(scope="module")
def zq():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import weight_only_quantized_zq_b200 as m
    return m


def test_wait_timeout_is_reported_and_recovered(zq, orc):
    # decode x2, tile kernel one-half and two-half plans, CTA-pair plan
    cases = [(1, 3584, 3584), (4, 1024, 2560), (64, 768, 1280), (300, 512, 1024), (600, 520, 1024)]
    data = []
    for i, (M, N, K) in enumerate(cases):
        w = zi.weight(N, K, seed=9600 + i, device="cuda")
        q = zq.quantize(w, 4)
        torch.cuda.synchronize()
        ref = orc.quantize_pack(w.cpu().numpy(), 4)
        x = zi.activations(M, K, seed=9700 + i, device="cuda")
        data.append((M, N, K, q, ref, x))
    zq.zq_check_device()  # nothing pending
    for (M, N, K, q, ref, x) in data:  # reserve outside the aborted region
        zq.linear(x, *q, 4, N)
    zq.zq_check_device()
    try:
        zq.zq_set_wait_limit_ns(0)
        for (M, N, K, q, ref, x) in data:
            zq.linear(x, *q, 4, N)
        with pytest.raises(zq.ZQError) as e:
            zq.zq_check_device()
        assert e.value.status == zq.ZQ_ERR_TIMEOUT
    finally:
        zq.zq_set_wait_limit_ns(DEFAULT_LIMIT_NS)
    zq.zq_check_device()  # the record was cleared; the device still answers
    for _ in range(2):
        for (M, N, K, q, ref, x) in data:
            y = zq.linear(x, *q, 4, N)
            torch.cuda.synchronize()
            y_ref, bound = orc.linear(u16(x), *ref, 4, N, K)
            assert_linear_close(y, y_ref, bound, f"after the timeout M={M} N={N} K={K}")
    zq.zq_check_device()
