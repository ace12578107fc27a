"""GPU checks of the workspace contract of zq_linear / zq_linear_stack:

  * a call on a stream without (enough) workspace returns ZQ_ERR_INVALID_ARG
    and enqueues nothing;
  * with the workspace reserved at exactly zq_linear_workspace_bytes (or the
    stack's size), the calls run and match the fp64 oracle;
  * the calls themselves allocate nothing: the device's free memory is the
    same before and after a run of calls on two streams with growing shapes;
  * a caller-owned buffer can be attached instead, and workspaces released.
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


def _layer(zq, orc, N, K, bits, seed):
    w = zi.weight(N, K, seed, device="cuda")
    q = zq.quantize(w, bits)
    torch.cuda.synchronize()
    return q, orc.quantize_pack(w.cpu().numpy(), bits)


def test_call_without_workspace_is_rejected_and_enqueues_nothing(zq, orc):
    q, ref = _layer(zq, orc, 256, 512, 4, 9100)
    x = zi.activations(2, 512, 9101, device="cuda")
    s = torch.cuda.Stream()
    for M, xx in ((2, x), (40, zi.activations(40, 512, 9102, device="cuda"))):
        out = torch.full((M, 256), 7.0, dtype=torch.float16, device="cuda")
        with pytest.raises(zq.ZQError) as e:
            zq.zq_linear(xx, *q, 4, 128, M, 256, 512, out, s)
        assert e.value.status == zq.ZQ_ERR_INVALID_ARG
        assert "zq_reserve_workspace" in str(e.value)
        s.synchronize()
        assert torch.all(out == 7.0)
    # a reservation one byte short is still rejected; the exact size works
    need = zq.zq_linear_workspace_bytes(4, 2, 256, 512)
    assert need > 256 * 1024
    zq.zq_reserve_workspace(need - 1, s)
    out = torch.full((2, 256), 7.0, dtype=torch.float16, device="cuda")
    with pytest.raises(zq.ZQError) as e:
        zq.zq_linear(x, *q, 4, 128, 2, 256, 512, out, s)
    assert e.value.status == zq.ZQ_ERR_INVALID_ARG
    s.synchronize()
    assert torch.all(out == 7.0)
    zq.zq_reserve_workspace(need, s)
    zq.zq_linear(x, *q, 4, 128, 2, 256, 512, out, s)
    s.synchronize()
    y_ref, bound = orc.linear(u16(x), *ref, 4, 256, 512)
    assert_linear_close(out, y_ref, bound, "exact reservation")
    big = zi.activations(16, 512, 9103, device="cuda")
    if zq.zq_linear_workspace_bytes(4, 16, 256, 512) > need:
        out16 = torch.full((16, 256), 7.0, dtype=torch.float16, device="cuda")
        with pytest.raises(zq.ZQError) as e:
            zq.zq_linear(big, *q, 4, 128, 16, 256, 512, out16, s)
        assert e.value.status == zq.ZQ_ERR_INVALID_ARG
        s.synchronize()
        assert torch.all(out16 == 7.0)
    zq.zq_release_workspace(s)
    with pytest.raises(zq.ZQError):
        zq.zq_linear(x, *q, 4, 128, 2, 256, 512, out, s)


def test_two_streams_growing_shapes_allocate_nothing(zq, orc):
    shapes = [(1, 512, 512), (4, 1024, 1280), (9, 3584, 3584), (16, 4608, 3584), (40, 1024, 1280),
              (1, 3584, 18944)]
    layers = [_layer(zq, orc, N, K, 4, 9200 + i) for i, (M, N, K) in enumerate(shapes)]
    xs = [zi.activations(M, K, 9300 + i, device="cuda") for i, (M, N, K) in enumerate(shapes)]
    outs = {(si, i): torch.empty(M, N, dtype=torch.float16, device="cuda")
            for si in range(2) for i, (M, N, K) in enumerate(shapes)}
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    for s in streams:
        zq.zq_reserve_workspace(max(zq.zq_linear_workspace_bytes(4, M, N, K) for (M, N, K) in shapes), s)
    for rep in range(2):  # the first pass also loads every kernel module (lazy loading)
        torch.cuda.synchronize()
        free0 = torch.cuda.mem_get_info()[0]
        for i, (M, N, K) in enumerate(shapes):  # growing shapes, interleaved on two streams
            for si, s in enumerate(streams):
                zq.zq_linear(xs[i], *layers[i][0], 4, 128, M, N, K, outs[(si, i)], s)
        torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free0, "zq_linear allocated device memory"
    for i, (M, N, K) in enumerate(shapes):
        y_ref, bound = orc.linear(u16(xs[i]), *layers[i][1], 4, N, K)
        for si in range(2):
            assert_linear_close(outs[(si, i)], y_ref, bound, f"stream {si} M={M} N={N} K={K}")
    for s in streams:
        zq.zq_release_workspace(s)


def test_attached_caller_buffer_and_stack_size(zq, orc):
    specs = [(1, 512, 512), (1, 256, 512), (12, 1024, 512), (40, 128, 384)]
    layers = [_layer(zq, orc, N, K, 4, 9400 + i) for i, (M, N, K) in enumerate(specs)]
    xs = [zi.activations(M, K, 9500 + i, device="cuda") for i, (M, N, K) in enumerate(specs)]
    outs = [torch.empty(M, N, dtype=torch.float16, device="cuda") for (M, N, K) in specs]
    ops = [(xs[i], *layers[i][0], outs[i], 4, 128, M, N, K) for i, (M, N, K) in enumerate(specs)]
    arr, n = zq.make_descs(ops)
    need = zq.zq_linear_stack_workspace_bytes(arr, n)
    assert need >= 256 * 1024
    s = torch.cuda.Stream()
    buf = torch.empty(need, dtype=torch.uint8, device="cuda")
    zq.zq_attach_workspace(buf, need, s)
    for rep in range(2):  # the first pass also loads every kernel module (lazy loading)
        s.synchronize()
        free0 = torch.cuda.mem_get_info()[0]
        zq.zq_linear_stack(arr, n, s)
        s.synchronize()
    assert torch.cuda.mem_get_info()[0] == free0
    for i, (M, N, K) in enumerate(specs):
        y_ref, bound = orc.linear(u16(xs[i]), *layers[i][1], 4, N, K)
        assert_linear_close(outs[i], y_ref, bound, f"attached op {i}")
    zq.zq_release_workspace(s)
    with pytest.raises(zq.ZQError) as e:
        zq.zq_attach_workspace(buf[1:], need - 1, s)  # not 256-byte aligned
    assert e.value.status == zq.ZQ_ERR_INVALID_ARG
