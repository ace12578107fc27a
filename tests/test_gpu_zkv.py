"""GPU: zKV (quantized KV cache with sliding precision) through the C ABI
against the oracle of oracle/zkv_oracle.py, bit for bit: the store (codes,
scales, zeros) of every token older than the window, the ring slots of the
window, and gathered fp16 rows, after every append of uneven sequences of
chunk sizes (single tokens, fewer than, exactly and more than one window)."""
import time

import numpy as np
import pytest
import torch

from oracle import zkv_oracle as zk

pytestmark = pytest.mark.gpu

BITS = (2, 3, 4, 8)


@pytest.fixture(scope="module")
def zq():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import weight_only_quantized_zq_b200 as m
    return m


def _rows(n, heads, dim, seed, scale=1.0):
    rng = np.random.default_rng(seed)
    return rng.normal(0, scale, (n, heads, dim)).astype(np.float16).view(np.uint16)


def _dev(rows16):
    return torch.from_numpy(np.ascontiguousarray(rows16).view(np.int16)).cuda().view(torch.float16)


def _u16(t):
    return t.cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def _compare(pl, ref, what):
    T, W = ref.tokens, ref.window
    ns = max(T - W, 0)
    assert pl.tokens == T
    assert np.array_equal(pl.packed[:ns].cpu().numpy().view(np.uint32), ref.packed[:ns]), f"{what}: codes"
    assert np.array_equal(_u16(pl.scales[:ns]), ref.scales[:ns]), f"{what}: scales"
    assert np.array_equal(_u16(pl.zeros[:ns]), ref.zeros[:ns]), f"{what}: zeros"
    ring = _u16(pl.ring)
    for s in range(W):
        if ref.slot_token[s] >= 0:
            assert np.array_equal(ring[s], ref.ring[s]), f"{what}: ring slot {s}"
    got = _u16(pl.gather(0, T))
    assert np.array_equal(got, ref.gather(0, T)), f"{what}: gather"
    if T > 2:
        assert np.array_equal(_u16(pl.gather(1, T - 1)), got[1:T - 1]), f"{what}: partial gather"


@pytest.mark.parametrize("bits", BITS)
def test_append_and_gather_match_oracle(zq, bits):
    cases = [(1, 1, 128, [1, 1, 3, 2]),
             (16, 3, 256, [5, 11, 16, 1, 40, 7]),
             (64, 2, 128, [64, 64, 200, 1, 0, 63])]
    for k, (window, heads, dim, chunks) in enumerate(cases):
        cap = sum(chunks) + 5
        pl = zq.KVPlane(window, cap, heads, dim, bits)
        ref = zk.Plane(window, cap, heads, dim, bits)
        rows = _rows(sum(chunks), heads, dim, seed=700 + 10 * bits + k)
        t = 0
        for c in chunks:
            pl.append(_dev(rows[t:t + c]))
            ref.append(rows[t:t + c])
            t += c
            torch.cuda.synchronize()
            _compare(pl, ref, f"bits={bits} window={window} after {t} tokens")


def test_nonfinite_row_is_reported(zq):
    pl = zq.KVPlane(2, 8, 1, 128, 4)
    rows = _rows(5, 1, 128, 1)
    rows[0, 0, 17] = np.float16(np.nan).view(np.uint16)
    pl.append(_dev(rows))
    with pytest.raises(zq.ZQError) as e:
        zq.zq_check_device()
    assert e.value.status == zq.ZQ_ERR_NONFINITE
    zq.zq_check_device()  # the record was cleared


def test_decode_shaped_plane(zq, capsys):
    """A 7B-shaped plane (4 KV heads x 128): a 4096-token prompt in chunks of
    512, then 64 single-token decode steps; every stored token checked
    against the oracle on a sample, the gather of the whole plane on all."""
    window, heads, dim, bits = 256, 4, 128, 4
    T0, steps = 4096, 64
    pl = zq.KVPlane(window, T0 + steps, heads, dim, bits)
    ref = zk.Plane(window, T0 + steps, heads, dim, bits)
    rows = _rows(T0 + steps, heads, dim, seed=9)
    dev = _dev(rows)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    for a in range(0, T0, 512):
        pl.append(dev[a:a + 512])
    for t in range(T0, T0 + steps):
        pl.append(dev[t:t + 1])
    torch.cuda.synchronize()
    dt = time.perf_counter() - t0
    ref.append(rows)
    _compare(pl, ref, "7B-shaped plane")
    fp16 = (T0 + steps) * heads * dim * 2
    store = (T0 + steps - window) * heads * zk.bytes_per_group(bits) * dim // 128
    with capsys.disabled():
        print(f"\nzKV 7B-shaped plane: {T0 + steps} tokens appended in {dt * 1e3:.2f} ms "
              f"(72 calls); store {store / 1e6:.2f} MB vs fp16 {fp16 / 1e6:.2f} MB")
