"""Host logic of the tensor-parallel layer, on the CPU: the shard planner, the
group-aligned slicing of packed tensors, and the exchange of fp32 partial sums
between world_size-2 gloo ranks (each rank's partial sums come from the fp64
oracle on its shard; the kernels themselves are covered by tests/test_gpu_tp.py).
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def tp():
    sys.path.insert(0, ROOT)
    from weight_only_quantized_zq_b200 import tp as m
    return m


def test_shard_planner_covers_exactly(tp):
    for N in (1, 63, 64, 65, 512, 3584, 4608, 37888):
        for P in (1, 2, 3, 4, 8):
            rows = [tp.row_shard(N, P, r) for r in range(P)]
            assert rows[0][0] == 0 and rows[-1][1] == N
            for (a0, a1), (b0, b1) in zip(rows, rows[1:]):
                assert a1 == b0 and a0 <= a1
            assert all(n0 % 64 == 0 for n0, _ in rows)
    for K in (128, 640, 3584, 18944):
        for P in (1, 2, 3, 4, 8):
            cols = [tp.group_shard(K, P, r) for r in range(P)]
            assert cols[0][0] == 0 and cols[-1][1] == K
            for (a0, a1), (b0, b1) in zip(cols, cols[1:]):
                assert a1 == b0
            assert all(k0 % 128 == 0 and k1 % 128 == 0 for k0, k1 in cols)
            sizes = [k1 - k0 for k0, k1 in cols]
            assert max(sizes) - min(sizes) <= 128  # whole groups, as even as possible
    with pytest.raises(Exception):
        tp.group_shard(100, 2, 0)


@pytest.mark.parametrize("bits", (2, 3, 4, 8))
def test_k_shard_equals_packing_the_shard(tp, orc, bits):
    """Slicing whole groups of packed words gives exactly the packing of the
    sliced weights: groups never straddle words, at every width."""
    N, K, P = 5, 640, 3
    w = np.random.default_rng(bits).normal(0, 0.02, (N, K)).astype(np.float32)
    p, s, z = orc.quantize_pack(w, bits)
    for r in range(P):
        (ps, ss, zs), (k0, k1) = tp.k_shard(torch.from_numpy(p.view(np.int32)), torch.from_numpy(s.view(np.int16)),
                                             torch.from_numpy(z.view(np.int16)), N, K, bits, P, r)
        p2, s2, z2 = orc.quantize_pack(w[:, k0:k1], bits)
        assert np.array_equal(ps.numpy().view(np.uint32), p2)
        assert np.array_equal(ss.numpy().view(np.uint16), s2) and np.array_equal(zs.numpy().view(np.uint16), z2)
    (pc, sc, zc), (n0, n1) = tp.column_shard(torch.from_numpy(p.view(np.int32)), torch.from_numpy(s.view(np.int16)),
                                             torch.from_numpy(z.view(np.int16)), N, K, bits, 1, 0)
    assert (n0, n1) == (0, N) and np.array_equal(pc.numpy().view(np.uint32), p)


def _free_port():
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        return sk.getsockname()[1]


def _rank(rank, world, port, out_dir):
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    sys.path.insert(0, ROOT)
    import datetime
    import torch.distributed as dist
    import oracle as orc
    from weight_only_quantized_zq_b200 import tp
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    M, N, K, bits = 3, 70, 640, 4
    g = np.random.default_rng(11)
    w = g.normal(0, 0.02, (N, K)).astype(np.float32)
    x = g.normal(0, 1, (M, K)).astype(np.float16).view(np.uint16)
    p, s, z = orc.quantize_pack(w, bits)
    k0, k1 = tp.group_shard(K, world, rank)
    g0, g1, w0, w1 = k0 // 128, k1 // 128, k0 * bits // 32, k1 * bits // 32
    part64, _ = orc.linear(x[:, k0:k1], p[:, w0:w1], s[:, g0:g1], z[:, g0:g1], bits, N, k1 - k0)
    part = torch.from_numpy(part64.astype(np.float32))
    parts = tp.gather_partials(part)
    summed = tp.all_reduce_partials(part.clone())
    dist.barrier()
    dist.destroy_process_group()
    np.savez(os.path.join(out_dir, f"rank{rank}.npz"), parts=np.stack([q.numpy() for q in parts]),
             summed=summed.numpy(), mine=part.numpy())


def test_exchange_gloo_world2(tmp_path, orc):
    world = 2
    mp.start_processes(_rank, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    got = [np.load(tmp_path / f"rank{r}.npz") for r in range(world)]
    # all-gather order is rank order, on every rank
    for r in range(world):
        for q in range(world):
            assert np.array_equal(got[r]["parts"][q], got[q]["mine"])
    # the rank-order sum of the shards' partial sums is the unsharded product
    M, N, K, bits = 3, 70, 640, 4
    g = np.random.default_rng(11)
    w = g.normal(0, 0.02, (N, K)).astype(np.float32)
    x = g.normal(0, 1, (M, K)).astype(np.float16).view(np.uint16)
    y_ref, bound = orc.linear(x, *orc.quantize_pack(w, bits), bits, N, K)
    ordered = got[0]["parts"][0].astype(np.float32)
    for q in range(1, world):
        ordered = (ordered + got[0]["parts"][q]).astype(np.float32)
    assert np.array_equal(ordered, got[1]["parts"][0] + got[1]["parts"][1])  # same bits on every rank
    assert np.all(np.abs(ordered.astype(np.float16).astype(np.float64) - y_ref) <= 2e-3 * bound + 1e-3)
    for r in range(world):
        assert np.allclose(got[r]["summed"], ordered, rtol=1e-6, atol=1e-6)
