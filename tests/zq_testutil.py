"""Helpers for the GPU parity tests: tensor <-> numpy views and the tolerance
check of the quantized linear.

Tolerance: |y_gpu - y_ref| <= 2e-3 * bound + 1e-3 per output element, where
y_ref = sum_k x*w_hat in fp64 and bound = sum_k |x|*|w_hat| (the oracle's).
"""
import numpy as np
import torch

REL_TOL = 2e-3
ABS_TOL = 1e-3


def u16(t):
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def u32(t):
    return t.detach().contiguous().view(torch.int32).cpu().numpy().view(np.uint32)


def assert_linear_close(y_gpu, y_ref, bound, what=""):
    yg = y_gpu.detach().float().cpu().numpy().astype(np.float64)
    assert yg.shape == y_ref.shape, (yg.shape, y_ref.shape)
    assert np.all(np.isfinite(yg)), f"{what}: non-finite output"
    err = np.abs(yg - y_ref)
    lim = REL_TOL * bound + ABS_TOL
    bad = err > lim
    if bad.any():
        i = np.unravel_index(np.argmax(err - lim), err.shape)
        raise AssertionError(
            f"{what}: {int(bad.sum())}/{bad.size} elements out of tolerance; worst at {i}: "
            f"gpu={yg[i]!r} ref={y_ref[i]!r} err={err[i]:.3e} lim={lim[i]:.3e}")
    return float((err / lim).max()) if err.size else 0.0
