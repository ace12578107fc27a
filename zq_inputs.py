"""Seeded synthetic inputs and workload shapes, shared by the tests, the smoke
check and the benchmark.

This module holds none of the quantization or matmul arithmetic: it only draws
random tensors and names the layer shapes. The CPU oracle and the CUDA library
both receive the tensors it produces as inputs.

Workloads are synthetic stand-ins for Qwen2.5-7B / Qwen2.5-32B shaped linear
layers (hidden 3584 / 5120, intermediate 18944 / 27648, fused qkv of
hidden + 2*512 / hidden + 2*1024 rows, 28 / 64 layers). No checkpoint is used.

Recipe:
  * weights: fp32 N(0, 0.02) from a torch generator seeded per tensor
    (seed = 16*layer + t, t = 0 qkv, 1 o, 2 gate_up, 3 down);
    optional outliers: each element independently with probability 0.001 is
    multiplied by 20 (drawn from the same generator);
  * activations: fp32 N(0, 1) rounded to fp16 (round to nearest even), seed
    16*layer + 15 (one buffer per distinct (M, K)).
"""
import torch

STD = 0.02
OUTLIER_P = 0.001
OUTLIER_MUL = 20.0
X_SEED = 15
PROJ = ("qkv", "o", "gate_up", "down")

# 7B-shaped decode/prefill projections: (name, N, K)
QWEN7B = (("qkv", 4608, 3584), ("o", 3584, 3584),
          ("gate_up", 37888, 3584), ("down", 3584, 18944))
QWEN7B_LAYERS = 28

# 32B-shaped mixed-precision layer: (name, N, K, bits)
QWEN32B_MIXED = (("qkv", 7168, 5120, 8), ("o", 5120, 5120, 4),
                 ("gate_up", 55296, 5120, 3), ("down", 5120, 27648, 2))
QWEN32B_LAYERS = 64


def seed_for(layer, t):
    return 16 * layer + t


def _gen(seed, device):
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def weight(N, K, seed, device="cpu", outliers=False, std=STD):
    """fp32 N x K weight ~ N(0, std), optional 0.1% x20 outliers."""
    g = _gen(seed, device)
    w = torch.randn(N, K, generator=g, device=device, dtype=torch.float32)
    w.mul_(std)
    if outliers:
        mask = torch.rand(N, K, generator=g, device=device) < OUTLIER_P
        w[mask] *= OUTLIER_MUL
    return w


def activations(M, K, seed, device="cpu"):
    """fp16 M x K activations ~ N(0, 1), fp32 draw rounded to fp16 (RNE)."""
    g = _gen(seed, device)
    return torch.randn(M, K, generator=g, device=device,
                       dtype=torch.float32).to(torch.float16)


def codes(N, K, bits, seed, device="cpu"):
    """Uniform random b-bit codes (uint8 N x K), for pack/unpack tests."""
    g = _gen(seed, device)
    return torch.randint(0, 1 << bits, (N, K), generator=g, device=device,
                         dtype=torch.int32).to(torch.uint8)
