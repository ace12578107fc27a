"""Pins for the zKV oracle (quantized KV cache with sliding precision), on the
CPU: the state after any number of appends against its closed form, the
gathered values against an independent numpy decode of the bit fields, and
the memory saving against the pages' "about 4x".

Sources: "ZSE: Motor de inferência de LLM de código aberto com inicializações
a frio de 3,9 segundos", section "Componentes da arquitetura" (zKV), and the
ZSE wiki article, section "Формат модели .zse" (the group codec)."""
import numpy as np
import pytest

from oracle import zkv_oracle as zk

BITS = (2, 3, 4, 8)


def _rows(n, heads, dim, seed, scale=1.0):
    rng = np.random.default_rng(seed)
    return (rng.normal(0, scale, (n, heads, dim))).astype(np.float16).view(np.uint16)


def _codes_numpy(words, K, bits):
    """Independent unpack: numpy little-endian bit order over the row bytes."""
    stream = np.unpackbits(np.asarray(words, "<u4").view(np.uint8), bitorder="little")
    return (stream[:K * bits].reshape(K, bits).astype(np.int64) << np.arange(bits)).sum(axis=1)


@pytest.mark.parametrize("window,T", [(1, 5), (4, 3), (4, 4), (4, 11), (16, 40)])
@pytest.mark.parametrize("bits", BITS)
def test_state_matches_closed_form(orc, window, T, bits):
    """Ring slot s holds the newest token t < T with t = s (mod window); every
    token older than the window is in the store as the quantizer's output."""
    heads, dim = 2, 256
    rows = _rows(T, heads, dim, seed=window * 100 + T + bits)
    pl = zk.Plane(window, T + 3, heads, dim, bits)
    # uneven chunks: the oracle's state must not depend on them
    cuts = sorted({0, T, *[c for c in (1, 2, window, window + 1) if c < T]})
    for a, b in zip(cuts[:-1], cuts[1:]):
        pl.append(rows[a:b])
    assert pl.tokens == T
    for s in range(window):
        newest = [t for t in range(T) if t % window == s]
        if newest:
            assert pl.slot_token[s] == newest[-1]
            assert np.array_equal(pl.ring[s], rows[newest[-1]])
        else:
            assert pl.slot_token[s] == -1
    for t in range(max(T - window, 0)):
        w = rows[t].view(np.float16).astype(np.float32)
        p, sc, z = orc.quantize_pack(w, bits)
        assert np.array_equal(pl.packed[t], p) and np.array_equal(pl.scales[t], sc)
        assert np.array_equal(pl.zeros[t], z)


@pytest.mark.parametrize("bits", BITS)
def test_gather_window_exact_store_decoded(orc, bits):
    """Window tokens come back bit for bit; older tokens equal fp16(q*s + z)
    decoded here from the stored bit fields with numpy, and lie within half a
    quantization step (plus the fp16 rounding) of what was appended."""
    window, T, heads, dim = 8, 29, 3, 256
    rows = _rows(T, heads, dim, seed=500 + bits, scale=0.5)
    pl = zk.Plane(window, 64, heads, dim, bits)
    pl.append(rows[:13])
    pl.append(rows[13:])
    got = pl.gather(0, T)
    assert np.array_equal(got[T - window:], rows[T - window:])
    for t in range(T - window):
        for h in range(heads):
            q = _codes_numpy(pl.packed[t, h], dim, bits)
            s = pl.scales[t, h].view(np.float16).astype(np.float64).repeat(128)
            z = pl.zeros[t, h].view(np.float16).astype(np.float64).repeat(128)
            ref = (q * s + z).astype(np.float16)
            assert np.array_equal(got[t, h], ref.view(np.uint16))
            x = rows[t, h].view(np.float16).astype(np.float64)
            err = np.abs(ref.astype(np.float64) - x)
            assert np.all(err <= s / 2 + np.abs(x) * 2.0 ** -11 + 2.0 ** -24)
    assert np.array_equal(pl.gather(5, 23), got[5:23])


def test_memory_saving_closed_form():
    """Store bytes per 128 fp16 values (256 bytes): 16*b codes + 4 bytes of
    scale and zero; INT4 gives 256/68 = 3.76x, the pages' 'about 4x'."""
    assert [zk.bytes_per_group(b) for b in BITS] == [36, 52, 68, 132]
    assert abs(256 / zk.bytes_per_group(4) - 3.7647) < 1e-4
    pl = zk.Plane(16, 100, 4, 128, 4)
    store = pl.packed.nbytes + pl.scales.nbytes + pl.zeros.nbytes
    assert store == 100 * 4 * zk.bytes_per_group(4)


def test_capacity_is_enforced():
    pl = zk.Plane(4, 6, 1, 128, 4)
    pl.append(_rows(6, 1, 128, 1))
    with pytest.raises(AssertionError):
        pl.append(_rows(1, 1, 128, 2))
