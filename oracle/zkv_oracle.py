"""CPU oracle of zKV, the quantized KV cache with sliding precision.

TEST INFRASTRUCTURE: only the tests and ``__graft_entry__.smoke()`` import
this module.  It shares no code with the CUDA library.

Sources: "ZSE: Motor de inferência de LLM de código aberto com inicializações
a frio de 3,9 segundos", section "Componentes da arquitetura", and "ZSE: A
Memory-Efficient LLM Inference Engine with Smart Resource Orchestration",
section "Technical Architecture": zKV, a KV cache quantized with "sliding
precision" that saves about 4x of memory.  The pages give no formula; the
reading taken is:

- a plane holds one fp16 row (heads x dim) per token;
- the newest `window` tokens stay exact, token t in ring slot t % window;
- a token that leaves the window is quantized with the weights' group codec
  (the asymmetric min/max quantizer of the wiki section "Формат модели .zse",
  groups of 128 along dim, L = 2^bits - 1), into store row t;
- reading a stored token gives fp16(q * scale + zero), rounded once.

The append below follows that definition literally, one token at a time:
token t enters slot t % window, and token t - window, which held the slot,
moves to the store.  Quantization and dequantization are the oracle's own
(``oracle.quantize_pack`` and ``oracle.dequant``, fp64); the final fp16
rounding of a dequantized value is numpy's float64 -> float16 cast (round to
nearest even), the same rounding the oracle's binary16 encoder is pinned to.
"""
import numpy as np

from . import dequant, quantize_pack

GROUP = 128


class Plane:
    """The state of one plane: ring (fp16 bits), which token each ring slot
    holds, and the store (packed codes, scales, zeros)."""

    def __init__(self, window, capacity, heads, dim, bits):
        assert window >= 1 and capacity >= 1 and heads >= 1 and dim % GROUP == 0
        self.window, self.capacity, self.heads, self.dim, self.bits = window, capacity, heads, dim, bits
        self.ring = np.zeros((window, heads, dim), np.uint16)
        self.slot_token = np.full(window, -1, np.int64)
        self.packed = np.zeros((capacity, heads, dim * bits // 32), np.uint32)
        self.scales = np.zeros((capacity, heads, dim // GROUP), np.uint16)
        self.zeros = np.zeros((capacity, heads, dim // GROUP), np.uint16)
        self.tokens = 0

    def _store(self, t, row16):
        """Quantize one token's row (heads x dim fp16 bits) into store row t."""
        w = row16.view(np.float16).astype(np.float32)  # exact
        p, s, z = quantize_pack(w.reshape(self.heads, self.dim), self.bits)
        self.packed[t] = p
        self.scales[t] = s
        self.zeros[t] = z

    def append(self, rows16):
        """rows16: uint16 (n, heads, dim), fp16 bit patterns."""
        rows16 = np.asarray(rows16, np.uint16)
        assert self.tokens + rows16.shape[0] <= self.capacity
        for row in rows16:
            t = self.tokens
            slot = t % self.window
            leaving = t - self.window
            if leaving >= 0:
                assert self.slot_token[slot] == leaving
                self._store(leaving, self.ring[slot])
            self.ring[slot] = row
            self.slot_token[slot] = t
            self.tokens += 1

    def stored_values(self, t):
        """Dequantized store row t, fp64 (heads x dim): q * scale + zero, exact."""
        return dequant(self.packed[t], self.scales[t], self.zeros[t], self.bits, self.heads, self.dim)

    def gather(self, a, b):
        """Tokens [a, b) as fp16 bits (b - a, heads, dim)."""
        assert 0 <= a <= b <= self.tokens
        out = np.zeros((b - a, self.heads, self.dim), np.uint16)
        for t in range(a, b):
            if t >= self.tokens - self.window:
                assert self.slot_token[t % self.window] == t
                out[t - a] = self.ring[t % self.window]
            else:
                out[t - a] = self.stored_values(t).astype(np.float16).view(np.uint16)
        return out


def bytes_per_group(bits):
    """Store bytes per 128 values: codes plus one fp16 scale and zero."""
    return GROUP * bits // 8 + 4
