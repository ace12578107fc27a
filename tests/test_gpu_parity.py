"""GPU parity: the CUDA path through the C ABI against the fp64 CPU oracle.

Bit-exact: quantize_pack and quantize_pack_symmetric (codes, scales, zeros)
and unpack.
Tolerance (the linear): |y_gpu - y_ref| <= 2e-3 * sum|x||w_hat| + 1e-3 per element.
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


def _quantize_both(zq, orc, w, bits):
    """Quantize on the GPU and with the oracle; assert bit-exact; return GPU buffers."""
    N, K = w.shape
    packed, scales, zeros = zq.quantize(w, bits)
    torch.cuda.synchronize()
    p_ref, s_ref, z_ref = orc.quantize_pack(w.cpu().numpy(), bits)
    assert np.array_equal(u16(scales).reshape(N, -1), s_ref), "scales differ"
    assert np.array_equal(u16(zeros).reshape(N, -1), z_ref), "zeros differ"
    assert np.array_equal(u32(packed).reshape(N, -1), p_ref), "packed codes differ"
    return packed, scales, zeros, (p_ref, s_ref, z_ref)


CANARY = 0x5A5A  # fp16 bit pattern of the guard regions around an output
GUARD = 64       # guard halves on each side (128 bytes keeps the output 16-byte aligned)


def _check_linear(zq, orc, x, qbufs, ref_bufs, bits, N, what, rows=None):
    M, K = x.shape
    packed, scales, zeros = qbufs
    # the output sits between two guard regions: a kernel writing outside the
    # M x N result would change them
    buf = torch.full((GUARD + M * N + GUARD,), CANARY, dtype=torch.int16, device=x.device)
    out = buf[GUARD:GUARD + M * N].view(torch.float16).view(M, N)
    zq.linear(x, packed, scales, zeros, bits, N, out=out)
    torch.cuda.synchronize()
    guards = torch.cat([buf[:GUARD], buf[GUARD + M * N:]])
    assert bool((guards == CANARY).all()), f"{what}: write outside the output"
    p_ref, s_ref, z_ref = ref_bufs
    y_ref, bound = orc.linear(u16(x), p_ref, s_ref, z_ref, bits, N, K, rows=rows)
    got = out if rows is None else out[:, torch.as_tensor(rows, device=out.device)]
    return assert_linear_close(got, y_ref, bound, what)


# ------------------------------------------------------------- bit-exact --

@pytest.mark.parametrize("bits", BITS)
def test_quantize_pack_bit_exact(zq, orc, bits):
    for N, K, seed, outl in ((1, 128, 1, False), (37, 512, 2, True), (64, 3584, 3, False),
                             (5, 27648, 4, True)):
        w = zi.weight(N, K, seed + 100 * bits, device="cuda", outliers=outl)
        _quantize_both(zq, orc, w, bits)


@pytest.mark.parametrize("bits", BITS)
def test_quantize_pack_edge_groups(zq, orc, bits):
    """Constant groups (scale 0), exact ties, fp16-range extremes, subnormal scales."""
    K = 1024
    w = torch.zeros(6, K)
    w[0] = 0.0123                                  # constant group everywhere
    w[1, :128] = torch.arange(128) % 16 / 16.0     # ties at (j+1/2)/16 below
    w[1, 2:17] = (torch.arange(15) + 0.5) / 16
    w[1, 0], w[1, 1] = 0.0, 15.0 / 16
    w[2] = torch.linspace(-65504, 65504, K)        # largest magnitudes
    w[3] = torch.linspace(0, 1e-6, K)              # fp16 subnormal scales
    w[4] = torch.randn(K) * 1e-3 - 3.0
    w[5, ::2] = 1.0
    _quantize_both(zq, orc, w.cuda().contiguous(), bits)


def test_quantize_pack_rejects_nonfinite(zq):
    for bad in (float("nan"), float("inf"), 70000.0):
        w = torch.zeros(4, 256, device="cuda")
        w[2, 77] = bad
        with pytest.raises(zq.ZQError) as e:
            zq.quantize(w, 4)
        assert e.value.status == zq.ZQ_ERR_NONFINITE
    zq.quantize(torch.zeros(4, 256, device="cuda"), 4)  # next call is clean


def _quantize_both_symmetric(zq, orc, w, bits):
    N, K = w.shape
    packed, scales, zeros = zq.quantize(w, bits, symmetric=True)
    torch.cuda.synchronize()
    p_ref, s_ref, z_ref = orc.quantize_pack_symmetric(w.cpu().numpy(), bits)
    assert np.array_equal(u16(scales).reshape(N, -1), s_ref), "scales differ"
    assert np.array_equal(u16(zeros).reshape(N, -1), z_ref), "zeros differ"
    assert np.array_equal(u32(packed).reshape(N, -1), p_ref), "packed codes differ"
    return packed, scales, zeros, (p_ref, s_ref, z_ref)


@pytest.mark.parametrize("bits", BITS)
def test_quantize_pack_symmetric_bit_exact(zq, orc, bits):
    """The symmetric quantizer (INT8-symmetric of the .zse format section, at
    every width) against the oracle, bit for bit, including edge groups."""
    for N, K, seed, outl in ((1, 128, 11, False), (37, 512, 12, True), (5, 27648, 14, True)):
        w = zi.weight(N, K, seed + 100 * bits, device="cuda", outliers=outl)
        _quantize_both_symmetric(zq, orc, w, bits)
    Q = (1 << (bits - 1)) - 1
    K = 768
    w = torch.zeros(6, K)                          # row 0: all-zero groups (scale 0)
    w[1, 0] = Q / 128.0                            # scale exactly 2^-7 ...
    j = torch.arange(Q, dtype=torch.float32)
    w[1, 1:1 + Q] = (j + 0.5) / 128                # ... so these are exact ties
    w[1, 64:64 + Q] = -(j + 0.5) / 128
    w[2] = torch.linspace(-32000, 32000, K)        # large, still storable zeros
    w[3] = torch.linspace(0, 1e-6, K)              # fp16 subnormal scales
    w[4] = torch.randn(K) * 1e-3 - 3.0             # one-signed groups
    w[5, ::2] = 1.0
    _quantize_both_symmetric(zq, orc, w.cuda().contiguous(), bits)


def test_quantize_pack_symmetric_rejects(zq):
    for bits, bad in ((8, float("nan")), (8, 70000.0), (8, 65400.0), (2, 40000.0)):
        w = torch.zeros(4, 256, device="cuda")
        w[1, 200] = bad
        with pytest.raises(zq.ZQError) as e:
            zq.quantize(w, bits, symmetric=True)
        assert e.value.status == zq.ZQ_ERR_NONFINITE
    zq.quantize(torch.zeros(4, 256, device="cuda"), 8, symmetric=True)  # next call is clean


@pytest.mark.parametrize("bits", BITS)
def test_linear_symmetric_weights(zq, orc, bits):
    """Symmetric tensors run through the unchanged linear kernels (decode and
    tile) and meet the oracle tolerance."""
    for i, (M, N, K) in enumerate(((1, 130, 512), (7, 64, 1280), (16, 33, 384), (40, 264, 640))):
        w = zi.weight(N, K, seed=5000 + 10 * bits + i, device="cuda", outliers=(i % 2 == 1))
        q = _quantize_both_symmetric(zq, orc, w, bits)
        x = zi.activations(M, K, seed=5100 + i, device="cuda")
        _check_linear(zq, orc, x, q[:3], q[3], bits, N, f"symmetric bits={bits} M={M} N={N} K={K}")


@pytest.mark.parametrize("bits", BITS)
def test_unpack_bit_exact(zq, orc, bits):
    for N, K in ((1, 128), (19, 640), (8, 27648)):
        codes = zi.codes(N, K, bits, seed=7 + bits).numpy()
        packed_np = np.stack([orc.pack_row(c, bits) for c in codes])
        packed = torch.from_numpy(packed_np.view(np.int32)).cuda()
        out = torch.empty(N, K, dtype=torch.uint8, device="cuda")
        zq.zq_unpack(packed, N, K, bits, out)
        torch.cuda.synchronize()
        assert np.array_equal(out.cpu().numpy(), orc.unpack(packed_np, N, K, bits))


@pytest.mark.parametrize("bits", BITS)
@pytest.mark.parametrize("group", (32, 64, 128))
def test_dequant_bit_exact(zq, orc, bits, group):
    """The tile kernel's dequantization (zq_dequant runs its routine) gives
    fp16_rne(q * s16 + z16) of the oracle's exact w_hat, bit for bit; where that
    rounds past the fp16 range the kernel holds 65504."""
    N, K = 40, 1024
    w = zi.weight(N, K, seed=9990 + bits + group, outliers=True)
    w[3] = torch.linspace(-65504.0, 65504.0, group).repeat(K // group)  # top codes round past 65504
    w[4] = 0.0123                                  # scale 0
    w[5] = torch.linspace(0, 1e-6, K)              # subnormal scales
    w[6] = w[6] * 1e3 - 3e3                        # large zero, small scale
    wd = w.contiguous().cuda()
    packed, scales, zeros = zq.quantize(wd, bits, group=group)
    out = torch.empty(N, K, dtype=torch.float16, device="cuda")
    zq.zq_dequant(packed, scales, zeros, bits, group, N, K, out)
    torch.cuda.synchronize()
    p_ref, s_ref, z_ref = orc.quantize_pack(w.numpy(), bits, group=group)
    exact = orc.dequant(p_ref, s_ref, z_ref, bits, N, K, group=group)
    with np.errstate(over="ignore"):
        h = exact.astype(np.float16)  # numpy's round-to-nearest-even, pinned against the oracle's encoder
    want = h.view(np.uint16).copy()
    want[np.isinf(h)] = 0x7BFF  # held at the largest finite fp16
    got = u16(out)
    bad = got != want
    assert not bad.any(), (int(bad.sum()), np.argwhere(bad)[:5], got[bad][:5], want[bad][:5])
    assert (want == 0x7BFF).any()  # the overflow case occurs


# ---------------------------------------------------------------- linear --

@pytest.mark.parametrize("bits", BITS)
def test_linear_shapes(zq, orc, bits):
    """Ragged N, every decode token tile, split-K and the multi-piece path."""
    cases = [(1, 1, 128), (1, 17, 512), (2, 100, 384), (3, 33, 1024), (5, 512, 512),
             (8, 257, 1280), (9, 64, 512), (16, 130, 256), (17, 48, 640), (32, 96, 512),
             (24, 257, 1152), (31, 64, 384), (20, 300, 3584),
             (33, 40, 384), (64, 200, 768), (65, 31, 256), (130, 70, 512)]
    for i, (M, N, K) in enumerate(cases):
        w = zi.weight(N, K, seed=1000 + 10 * bits + i, device="cuda", outliers=(i % 3 == 0))
        q = _quantize_both(zq, orc, w, bits)
        x = zi.activations(M, K, seed=2000 + i, device="cuda")
        _check_linear(zq, orc, x, q[:3], q[3], bits, N, f"bits={bits} M={M} N={N} K={K}")


@pytest.mark.parametrize("bits", BITS)
def test_prefill_shapes(zq, orc, bits):
    """M > 32 runs the tcgen05 tile kernel: ragged token tiles (TMA zero
    fill), ragged weight-row tiles, N not a multiple of 8 (scalar stores)."""
    cases = [(65, 31, 256), (130, 70, 512), (256, 256, 128), (300, 520, 1024), (257, 264, 384),
             (512, 256, 3584), (1000, 1000, 640)]
    for i, (M, N, K) in enumerate(cases):
        w = zi.weight(N, K, seed=3000 + 10 * bits + i, device="cuda", outliers=(i % 2 == 0))
        q = _quantize_both(zq, orc, w, bits)
        x = zi.activations(M, K, seed=4000 + i, device="cuda")
        _check_linear(zq, orc, x, q[:3], q[3], bits, N, f"prefill bits={bits} M={M} N={N} K={K}")
    zq.zq_check_device()


def test_linear_adversarial_all_positive(zq, orc):
    """All-positive x and weights: errors cannot cancel (worst case of fp32
    accumulation against the bound)."""
    for bits in BITS:
        N, K = 64, 18944
        w = zi.weight(N, K, seed=31 + bits, device="cuda").abs()
        q = _quantize_both(zq, orc, w, bits)
        for M in (4, 300):
            x = zi.activations(M, K, seed=32, device="cuda").abs()
            _check_linear(zq, orc, x, q[:3], q[3], bits, N, f"all-positive bits={bits} M={M}")


def test_config1_single_layer(zq, orc):
    """M=1, N=K=512 INT4; W ~ N(0,0.02) seed 0 quantized by the oracle; x seed
    0 (the benchmark's draw) and seed 15 (the per-tensor seed recipe)."""
    N = K = 512
    w = zi.weight(N, K, seed=0)  # CPU draw, as the oracle gets it
    p_ref, s_ref, z_ref = orc.quantize_pack(w.numpy(), 4)
    packed = torch.from_numpy(p_ref.view(np.int32).reshape(-1)).cuda()
    scales = torch.from_numpy(s_ref.view(np.int16)).cuda()
    zeros = torch.from_numpy(z_ref.view(np.int16)).cuda()
    for xs in (0, zi.X_SEED):
        x = zi.activations(1, K, seed=xs).cuda()
        _check_linear(zq, orc, x, (packed, scales, zeros), (p_ref, s_ref, z_ref), 4, N, f"config1 x seed {xs}")


def test_config2_7b_decode_projections(zq, orc):
    for t, (name, N, K) in enumerate(zi.QWEN7B):
        w = zi.weight(N, K, zi.seed_for(0, t), device="cuda")
        q = _quantize_both(zq, orc, w, 4)
        del w
        x = zi.activations(1, K, zi.seed_for(0, zi.X_SEED), device="cuda")
        _check_linear(zq, orc, x, q[:3], q[3], 4, N, f"7b {name}")


def test_config4_32b_mixed_precision(zq, orc):
    for t, (name, N, K, bits) in enumerate(zi.QWEN32B_MIXED):
        w = zi.weight(N, K, zi.seed_for(0, t), device="cuda", outliers=True)
        q = _quantize_both(zq, orc, w, bits)
        del w
        x = zi.activations(1, K, zi.seed_for(0, zi.X_SEED), device="cuda")
        _check_linear(zq, orc, x, q[:3], q[3], bits, N, f"32b {name} int{bits}")


# ----------------------------------------------------------------- stack --

def _layer(zq, orc, N, K, bits, seed):
    w = zi.weight(N, K, seed, device="cuda")
    q = zq.quantize(w, bits)
    torch.cuda.synchronize()
    ref = orc.quantize_pack(w.cpu().numpy(), bits)
    return q, ref


def test_stack_against_oracle(zq, orc):
    """Independent ops of mixed bits and batch sizes (fused into shared
    launches) and a dependent chain (x of an op is the out of the previous
    one), all through one zq_linear_stack call."""
    specs = [(4, 512, 512, 4), (4, 256, 512, 3), (4, 512, 256, 8), (4, 1024, 512, 2),
             (12, 512, 512, 4), (1, 384, 512, 4), (40, 128, 384, 4)]
    layers = [_layer(zq, orc, N, K, b, 50 + i) for i, (M, N, K, b) in enumerate(specs)]
    xs = [zi.activations(M, K, 60 + i, device="cuda") for i, (M, N, K, b) in enumerate(specs)]
    outs = [torch.empty(M, N, dtype=torch.float16, device="cuda") for (M, N, K, b) in specs]
    ops = [(xs[i], *layers[i][0], outs[i], b, 128, M, N, K) for i, (M, N, K, b) in enumerate(specs)]
    # chain: A (K=512 -> N=512) feeds B (K=512 -> N=256), which feeds C (K=256)
    qa, ra = _layer(zq, orc, 512, 512, 4, 70)
    qb, rb = _layer(zq, orc, 256, 512, 3, 71)
    qc, rc = _layer(zq, orc, 384, 256, 8, 73)
    xa = zi.activations(2, 512, 72, device="cuda")
    ya = torch.empty(2, 512, dtype=torch.float16, device="cuda")
    yb = torch.empty(2, 256, dtype=torch.float16, device="cuda")
    yc = torch.empty(2, 384, dtype=torch.float16, device="cuda")
    ops += [(xa, *qa, ya, 4, 128, 2, 512, 512), (ya, *qb, yb, 3, 128, 2, 256, 512),
            (yb, *qc, yc, 8, 128, 2, 384, 256)]
    zq.linear_stack(ops)
    torch.cuda.synchronize()
    for i, (M, N, K, b) in enumerate(specs):
        p, s, z = layers[i][1]
        y_ref, bound = orc.linear(u16(xs[i]), p, s, z, b, N, K)
        assert_linear_close(outs[i], y_ref, bound, f"stack op {i}")
    for x_in, y_out, ref, b, N, K in ((xa, ya, ra, 4, 512, 512), (ya, yb, rb, 3, 256, 512),
                                       (yb, yc, rc, 8, 384, 256)):
        y_ref, bound = orc.linear(u16(x_in), *ref, b, N, K)
        assert_linear_close(y_out, y_ref, bound, "stack chain")


def test_stack_every_route_with_a_chain(zq, orc):
    """One zq_linear_stack call over every route of the library: the decode
    kernel with one, two and four token tiles (M = 1, 12, 24), the tile
    kernel's one-half plan (M = 40), two-half plan (M = 200) and CTA-pair plan
    (M = 600); plus a chain of three ops at M = 24, each reading the previous
    op's output: INT4 and INT3 on the decode kernel, then INT2 with groups of
    64 on the tile kernel."""
    specs = [(1, 520, 640, 4), (12, 264, 1152, 3), (24, 600, 1024, 2), (40, 300, 640, 8),
             (200, 264, 384, 4), (600, 520, 512, 3)]
    layers = [_layer(zq, orc, N, K, b, 110 + i) for i, (M, N, K, b) in enumerate(specs)]
    xs = [zi.activations(M, K, 120 + i, device="cuda") for i, (M, N, K, b) in enumerate(specs)]
    outs = [torch.empty(M, N, dtype=torch.float16, device="cuda") for (M, N, K, b) in specs]
    ops = [(xs[i], *layers[i][0], outs[i], b, 128, M, N, K) for i, (M, N, K, b) in enumerate(specs)]
    # chain at M = 24: INT4 (K=512 -> 384), then INT3 (384 -> 640), then INT2 with groups of 64 (640 -> 256)
    qa, ra = _layer(zq, orc, 384, 512, 4, 130)
    qb, rb = _layer(zq, orc, 640, 384, 3, 131)
    wc = zi.weight(256, 640, seed=132, device="cuda")
    qc = zq.quantize(wc, 2, group=64)
    torch.cuda.synchronize()
    rc = orc.quantize_pack(wc.cpu().numpy(), 2, group=64)
    xa = zi.activations(24, 512, 133, device="cuda")
    ya = torch.empty(24, 384, dtype=torch.float16, device="cuda")
    yb = torch.empty(24, 640, dtype=torch.float16, device="cuda")
    yc = torch.empty(24, 256, dtype=torch.float16, device="cuda")
    ops += [(xa, *qa, ya, 4, 128, 24, 384, 512), (ya, *qb, yb, 3, 128, 24, 640, 384),
            (yb, *qc, yc, 2, 64, 24, 256, 640)]
    zq.linear_stack(ops)
    torch.cuda.synchronize()
    for i, (M, N, K, b) in enumerate(specs):
        y_ref, bound = orc.linear(u16(xs[i]), *layers[i][1], b, N, K)
        assert_linear_close(outs[i], y_ref, bound, f"every-route stack op {i} M={M} b={b}")
    for x_in, y_out, ref, b, N, K, g in ((xa, ya, ra, 4, 384, 512, 128), (ya, yb, rb, 3, 640, 384, 128),
                                          (yb, yc, rc, 2, 256, 640, 64)):
        y_ref, bound = orc.linear(u16(x_in), *ref, b, N, K, group=g)
        assert_linear_close(y_out, y_ref, bound, f"every-route chain b={b} group={g}")
    zq.zq_check_device()


@pytest.mark.parametrize("bits", BITS)
def test_prefill_grouped_plans(zq, orc, bits):
    """Grouped tile-kernel launches of independent ops: one whose ops all have
    17..128 tokens (one-token-half plan: 128-token x boxes, cp.async code ring;
    several row tiles per op, ops of different K so tiles of different group
    counts follow each other in a CTA), and one that mixes such ops with a
    larger M (two-half plan)."""
    for specs in ([(17, 520, 640), (100, 264, 1280), (128, 256, 384), (64, 300, 3584)],
                  [(40, 264, 640), (200, 130, 384), (128, 512, 512)]):
        layers = [_layer(zq, orc, N, K, bits, 90 + 7 * i + bits) for i, (M, N, K) in enumerate(specs)]
        xs = [zi.activations(M, K, 95 + i, device="cuda") for i, (M, N, K) in enumerate(specs)]
        outs = [torch.empty(M, N, dtype=torch.float16, device="cuda") for (M, N, K) in specs]
        zq.linear_stack([(xs[i], *layers[i][0], outs[i], bits, 128, M, N, K)
                            for i, (M, N, K) in enumerate(specs)])
        torch.cuda.synchronize()
        for i, (M, N, K) in enumerate(specs):
            p, s, z = layers[i][1]
            y_ref, bound = orc.linear(u16(xs[i]), p, s, z, bits, N, K)
            assert_linear_close(outs[i], y_ref, bound, f"grouped bits={bits} M={M} N={N} K={K}")


@pytest.mark.parametrize("bits", (2, 8))
def test_prefill_one_half_many_short_tiles(zq, orc, bits):
    """One-half plan with more row tiles than SMs and one group per tile
    (K = 128): the code-ring issue cursor runs whole tiles ahead of the
    consumer (INT2: 5 groups in flight, INT8: 2)."""
    M, N, K = 40, 157 * 256 - 13, 128
    w = zi.weight(N, K, seed=6100 + bits, device="cuda")
    q = _quantize_both(zq, orc, w, bits)
    x = zi.activations(M, K, seed=6200, device="cuda")
    _check_linear(zq, orc, x, q[:3], q[3], bits, N, f"many short tiles bits={bits}")


def test_stack_validation_enqueues_nothing(zq, orc):
    q, _ = _layer(zq, orc, 64, 256, 4, 80)
    x = zi.activations(1, 256, 81, device="cuda")
    out = torch.full((1, 64), 7.0, dtype=torch.float16, device="cuda")
    bad = (x, *q, out, 5, 128, 1, 64, 256)
    good = (x, *q, out, 4, 128, 1, 64, 256)
    with pytest.raises(zq.ZQError) as e:
        zq.zq_linear_stack([good, bad])
    assert e.value.status == zq.ZQ_ERR_UNSUPPORTED
    torch.cuda.synchronize()
    assert torch.all(out == 7.0)
