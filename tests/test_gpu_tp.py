"""GPU parity of the tensor-parallel quantized linear ("Тензорный параллелизм"
of the ZSE wiki page: column-parallel QKV/Gate/Up, row-parallel O/Down), with
P = 2 and P = 4 shards run one after another on one GPU and their results
combined as the ranks would combine them, against the fp64 oracle on the
unsharded layer at the tolerance |y - y_ref| <= 2e-3 * sum|x||w_hat| + 1e-3.
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
    w = zi.weight(N, K, seed, device="cuda", outliers=True)
    q = zq.quantize(w, bits)
    torch.cuda.synchronize()
    ref = orc.quantize_pack(w.cpu().numpy(), bits)
    assert np.array_equal(u32(q[0]).reshape(N, -1), ref[0])
    return q, ref


@pytest.mark.parametrize("P", (2, 4))
def test_column_parallel(zq, orc, P):
    from weight_only_quantized_zq_b200 import tp
    for i, (M, N, K, bits) in enumerate(((1, 4608, 3584, 4), (16, 1000, 512, 3), (24, 600, 1024, 4),
                                         (40, 777, 640, 8), (300, 520, 384, 2))):
        q, ref = _layer(zq, orc, N, K, bits, 9800 + i)
        x = zi.activations(M, K, 9900 + i, device="cuda")
        slices = [tp.ColumnParallelLinear(*q, N, K, bits, r, P).forward(x) for r in range(P)]
        torch.cuda.synchronize()
        y = torch.cat(slices, dim=1)
        y_ref, bound = orc.linear(u16(x), *ref, bits, N, K)
        assert_linear_close(y, y_ref, bound, f"column-parallel P={P} M={M} N={N} K={K} b={bits}")


@pytest.mark.parametrize("P", (2, 4))
def test_row_parallel_partial_sums(zq, orc, P):
    """Each shard's fp32 partial sums, added in rank order by
    zq_reduce_partials; K = 640 gives 5 groups, an uneven split over 4."""
    from weight_only_quantized_zq_b200 import tp
    for i, (M, N, K, bits) in enumerate(((1, 3584, 18944, 4), (4, 512, 3584, 2), (9, 300, 640, 8),
                                         (24, 600, 1152, 2), (40, 300, 1280, 3), (300, 256, 640, 4))):
        q, ref = _layer(zq, orc, N, K, bits, 9810 + i)
        x = zi.activations(M, K, 9910 + i, device="cuda")
        shards = [tp.RowParallelLinear(*q, N, K, bits, r, P) for r in range(P)]
        parts = [s.partial(x[:, s.k0:s.k1].contiguous()) for s in shards]
        y = torch.empty(M, N, dtype=torch.float16, device="cuda")
        zq.zq_reduce_partials(parts, M * N, y)
        torch.cuda.synchronize()
        y_ref, bound = orc.linear(u16(x), *ref, bits, N, K)
        assert_linear_close(y, y_ref, bound, f"row-parallel P={P} M={M} N={N} K={K} b={bits}")
        # each fp32 partial is its shard's own product (oracle on the shard's groups)
        k0, k1 = shards[-1].k0, shards[-1].k1
        g0, g1 = k0 // 128, k1 // 128
        w0, w1 = k0 * bits // 32, k1 * bits // 32
        p_ref, bnd = orc.linear(u16(x[:, k0:k1]), ref[0][:, w0:w1], ref[1][:, g0:g1], ref[2][:, g0:g1],
                                bits, N, k1 - k0)
        assert_linear_close(parts[-1], p_ref, bnd, f"last shard's partial P={P} M={M}")


@pytest.mark.parametrize("P", (2, 4))
def test_row_parallel_owner_slices(zq, orc, P):
    """The reduce-scatter layout: in ONE zq_linear_partial_stack launch per
    shard, shard r writes its partial sums for the output rows each rank s owns
    straight into receive buffer [s][r] (on several GPUs that is rank s's
    memory, written over NVLink); rank s then adds its P buffers in rank order.
    On one GPU all buffers are local, the kernels and the order the same."""
    from weight_only_quantized_zq_b200 import tp
    M, N, K, bits = 2, 3584, 3584, 4
    q, ref = _layer(zq, orc, N, K, bits, 9830)
    x = zi.activations(M, K, 9930, device="cuda")
    owners = [tp.row_shard(N, P, s) for s in range(P)]
    recv = [[torch.empty(M, n1 - n0, dtype=torch.float32, device="cuda") for _ in range(P)] for (n0, n1) in owners]
    for r in range(P):
        sh = tp.RowParallelLinear(*q, N, K, bits, r, P)
        xs = x[:, sh.k0:sh.k1].contiguous()
        Kr = sh.k1 - sh.k0
        ops = []
        for s, (n0, n1) in enumerate(owners):
            p = sh.packed[n0:n1]
            ops.append((xs, p, sh.scales[n0:n1], sh.zeros[n0:n1], recv[s][r], bits, 128, M, n1 - n0, Kr))
        arr, n = zq.make_partial_descs(ops)
        zq.ensure_workspace(zq.zq_linear_partial_stack_workspace_bytes(arr, n))
        zq.zq_linear_partial_stack(arr, n)
    y_ref, bound = orc.linear(u16(x), *ref, bits, N, K)
    for s, (n0, n1) in enumerate(owners):
        ys = torch.empty(M, n1 - n0, dtype=torch.float16, device="cuda")
        zq.zq_reduce_partials(recv[s], M * (n1 - n0), ys)
        torch.cuda.synchronize()
        assert_linear_close(ys, y_ref[:, n0:n1], bound[:, n0:n1], f"owner {s} of {P}")


def test_reduce_partials_order_and_conversion(zq):
    """Fixed-order fp32 sum then one fp16 rounding, against numpy; odd counts
    take the scalar path, counts divisible by 4 the vector path."""
    g = np.random.default_rng(5)
    for count, P in ((1, 1), (7, 3), (4096, 4), (1001, 16)):
        parts = [g.normal(0, 100, count).astype(np.float32) for _ in range(P)]
        ref = parts[0].copy()
        for p in parts[1:]:
            ref = (ref + p).astype(np.float32)  # fp32 adds in order
        dev = [torch.from_numpy(p).cuda() for p in parts]
        out = torch.empty(count, dtype=torch.float16, device="cuda")
        zq.zq_reduce_partials(dev, count, out)
        torch.cuda.synchronize()
        assert np.array_equal(out.cpu().numpy(), ref.astype(np.float16)), (count, P)
