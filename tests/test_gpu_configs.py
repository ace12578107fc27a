"""GPU parity at the full workload sizes, in the launch configuration the
benchmark uses (one zq_linear_stack call over the whole stack).

Config 3: 28 Qwen2.5-7B-shaped layers x (qkv, o, gate_up, down), INT4 g128,
M in {1, 4, 16, 64}; layers 0 and 27 are quantized on the GPU AND by the oracle
(bit-exact) and every output of their projections is checked.
Config 4 (stack): 64 Qwen2.5-32B-shaped layers, INT8 qkv / INT4 o / INT3
gate_up / INT2 down with 0.1% outliers, M = 1 (the benchmark's 32b-mixed
workload: one decode launch per bit width); layers 0 and 63 checked in full.
Config 5: M = 2048 prefill, INT4 g128, the four projections of layers 0 and 27;
all M rows x 256 sampled output columns per projection are checked.
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


def _layer_weights(zq, orc, layer, check_layers):
    out = []
    for t, (name, N, K) in enumerate(zi.QWEN7B):
        w = zi.weight(N, K, zi.seed_for(layer, t), device="cuda")
        q = zq.quantize(w, 4)
        ref = None
        if layer in check_layers:
            torch.cuda.synchronize()
            ref = orc.quantize_pack(w.cpu().numpy(), 4)
            assert np.array_equal(u32(q[0]).reshape(N, -1), ref[0]), f"layer {layer} {name} codes"
            assert np.array_equal(u16(q[1]).reshape(N, -1), ref[1]), f"layer {layer} {name} scales"
            assert np.array_equal(u16(q[2]).reshape(N, -1), ref[2]), f"layer {layer} {name} zeros"
        del w
        out.append((name, N, K, q, ref))
    return out


def test_config3_decode_stack_28_layers(zq, orc):
    check = (0, 27)
    layers = [_layer_weights(zq, orc, l, check) for l in range(zi.QWEN7B_LAYERS)]
    Ms = (1, 4, 16, 64)
    xs = {(M, K): zi.activations(M, K, zi.seed_for(0, zi.X_SEED), device="cuda")
          for M in Ms for K in (3584, 18944)}
    for M in Ms:
        ops, outs = [], []
        for l, lw in enumerate(layers):
            for (name, N, K, q, ref) in lw:
                out = torch.empty(M, N, dtype=torch.float16, device="cuda")
                ops.append((xs[(M, K)], *q, out, 4, 128, M, N, K))
                outs.append((l, name, N, K, out, ref))
        zq.linear_stack(ops)
        torch.cuda.synchronize()
        for (l, name, N, K, out, ref) in outs:
            if l in check:
                y_ref, bound = orc.linear(u16(xs[(M, K)]), *ref, 4, N, K)
                assert_linear_close(out, y_ref, bound, f"config3 M={M} layer {l} {name}")


def test_config4_mixed_stack_64_layers(zq, orc):
    check = (0, zi.QWEN32B_LAYERS - 1)
    xs = {K: zi.activations(1, K, zi.seed_for(0, zi.X_SEED), device="cuda") for K in (5120, 27648)}
    ops, outs = [], []
    for layer in range(zi.QWEN32B_LAYERS):
        for t, (name, N, K, bits) in enumerate(zi.QWEN32B_MIXED):
            w = zi.weight(N, K, zi.seed_for(layer, t), device="cuda", outliers=True)
            q = zq.quantize(w, bits)
            ref = None
            if layer in check:
                torch.cuda.synchronize()
                ref = orc.quantize_pack(w.cpu().numpy(), bits)
                assert np.array_equal(u32(q[0]).reshape(N, -1), ref[0]), f"layer {layer} {name} codes"
            del w
            out = torch.empty(1, N, dtype=torch.float16, device="cuda")
            ops.append((xs[K], *q, out, bits, 128, 1, N, K))
            outs.append((layer, name, N, K, bits, out, ref))
    zq.linear_stack(ops)
    torch.cuda.synchronize()
    zq.zq_check_device()
    for (layer, name, N, K, bits, out, ref) in outs:
        if layer in check:
            y_ref, bound = orc.linear(u16(xs[K]), *ref, bits, N, K)
            assert_linear_close(out, y_ref, bound, f"config4 stack layer {layer} {name} int{bits}")


def test_config5_prefill_m2048(zq, orc):
    M = 2048
    check = (0, 27)
    xs = {K: zi.activations(M, K, zi.seed_for(0, zi.X_SEED), device="cuda") for K in (3584, 18944)}
    rng = np.random.default_rng(5)
    for l in check:
        lw = _layer_weights(zq, orc, l, check)
        ops, outs = [], []
        for (name, N, K, q, ref) in lw:
            out = torch.empty(M, N, dtype=torch.float16, device="cuda")
            ops.append((xs[K], *q, out, 4, 128, M, N, K))
            outs.append((name, N, K, out, ref))
        zq.linear_stack(ops)
        torch.cuda.synchronize()
        zq.zq_check_device()
        for (name, N, K, out, ref) in outs:
            cols = np.sort(rng.choice(N, 256, replace=False)).astype(np.int64)
            cols[0], cols[-1] = 0, N - 1      # edges of the first and last tiles
            y_ref, bound = orc.linear(u16(xs[K]), *ref, 4, N, K, rows=cols)
            got = out[:, torch.as_tensor(cols, device="cuda")]
            assert_linear_close(got, y_ref, bound, f"config5 layer {l} {name}")
