"""CPU oracle for the weight-only quantized linear layer (fp64, plain C).

TEST INFRASTRUCTURE: only the tests, ``__graft_entry__.smoke()`` and the
benchmark's ``cpu_baseline`` leg may import this package. It shares no code
with the CUDA library and never imports it.

What it computes follows the ZSE wiki article "ZSE - open-source движок для
запуска LLM локально на GPU - 2026", section "Формат модели .zse" (group-wise
asymmetric min/max quantizer, low-nibble-first packing, fp16 scale/zero),
generalised to b in {2,3,4,8} per the per-tensor INT2-8 scheme of "ZSE: A
Memory-Efficient LLM Inference Engine with Smart Resource Orchestration",
section "Technical Architecture". The same section's symmetric INT8 variant
(listed without a formula) is ``quantize_group_symmetric`` /
``quantize_pack_symmetric``; ``zkv_oracle`` holds the quantized KV cache. The C
source states every reading taken where the pages are silent.

Arrays are numpy; fp16 values travel as uint16 bit patterns.
"""
import ctypes
import os

import numpy as np

from .build import LIB, build

OK, INVALID, UNSUPPORTED, NONFINITE = 0, 1, 2, 3
GROUP = 128

_lib = None


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(LIB)
        P = ctypes.c_void_p
        I = ctypes.c_int
        lib.zo_f16_to_f64.argtypes = [ctypes.c_uint16]
        lib.zo_f16_to_f64.restype = ctypes.c_double
        lib.zo_f64_to_f16.argtypes = [ctypes.c_double]
        lib.zo_f64_to_f16.restype = ctypes.c_uint16
        lib.zo_quantize_group.argtypes = [P, I, I, P, P, P]
        lib.zo_quantize_group.restype = I
        lib.zo_pack_row.argtypes = [P, I, I, P]
        lib.zo_pack_row.restype = None
        lib.zo_unpack_row.argtypes = [P, I, I, P]
        lib.zo_unpack_row.restype = None
        lib.zo_quantize_pack.argtypes = [P, I, I, I, I, P, P, P]
        lib.zo_quantize_pack.restype = I
        lib.zo_quantize_group_symmetric.argtypes = [P, I, I, P, P, P]
        lib.zo_quantize_group_symmetric.restype = I
        lib.zo_quantize_pack_symmetric.argtypes = [P, I, I, I, I, P, P, P]
        lib.zo_quantize_pack_symmetric.restype = I
        lib.zo_unpack.argtypes = [P, I, I, I, P]
        lib.zo_unpack.restype = I
        lib.zo_dequant.argtypes = [P, P, P, I, I, I, I, P]
        lib.zo_dequant.restype = I
        lib.zo_linear_rows.argtypes = [P, I, I, P, P, P, I, I, I, P, I, P, P]
        lib.zo_linear_rows.restype = I
        lib.zo_linear_rows_ex.argtypes = [P, I, I, I, P, P, P, I, I, I, P, I, P, P]
        lib.zo_linear_rows_ex.restype = I
        lib.zo_bf16_to_f64.argtypes = [ctypes.c_uint16]
        lib.zo_bf16_to_f64.restype = ctypes.c_double
        lib.zo_f64_to_bf16.argtypes = [ctypes.c_double]
        lib.zo_f64_to_bf16.restype = ctypes.c_uint16
        lib.zo_set_threads.argtypes = [I]
        lib.zo_set_threads.restype = None
        lib.zo_get_threads.argtypes = []
        lib.zo_get_threads.restype = I
        _lib = lib
    return _lib


class OracleError(RuntimeError):
    def __init__(self, status):
        super().__init__(f"oracle status {status}")
        self.status = status


def _ptr(a):
    return ctypes.c_void_p(a.ctypes.data)


def _c(a, dtype):
    a = np.ascontiguousarray(a, dtype=dtype)
    return a


def words_per_row(K, bits):
    return K * bits // 32


def f16_to_f64(h):
    return _load().zo_f16_to_f64(int(h))


def f64_to_f16(v):
    return _load().zo_f64_to_f16(float(v))


def bf16_to_f64(b):
    return _load().zo_bf16_to_f64(int(b))


def f64_to_bf16(v):
    return _load().zo_f64_to_bf16(float(v))


def quantize_group(w, bits):
    """Quantize one group; returns (s16_bits, z16_bits, q uint8 array)."""
    w = _c(w, np.float32)
    q = np.zeros(w.size, np.uint8)
    s = ctypes.c_uint16()
    z = ctypes.c_uint16()
    st = _load().zo_quantize_group(_ptr(w), w.size, (1 << bits) - 1,
                                   ctypes.byref(s), ctypes.byref(z), _ptr(q))
    if st != OK:
        raise OracleError(st)
    return s.value, z.value, q


def quantize_group_symmetric(w, bits):
    """Symmetric quantizer, one group; returns (s16_bits, z16_bits, stored
    codes uint8 array, code = q + 2^(bits-1))."""
    w = _c(w, np.float32)
    q = np.zeros(w.size, np.uint8)
    s = ctypes.c_uint16()
    z = ctypes.c_uint16()
    st = _load().zo_quantize_group_symmetric(_ptr(w), w.size, bits,
                                             ctypes.byref(s), ctypes.byref(z), _ptr(q))
    if st != OK:
        raise OracleError(st)
    return s.value, z.value, q


def pack_row(codes, bits):
    codes = _c(codes, np.uint8)
    K = codes.size
    words = np.zeros(K * bits // 32, np.uint32)
    _load().zo_pack_row(_ptr(codes), K, bits, _ptr(words))
    return words


def unpack_row(words, K, bits):
    words = _c(words, np.uint32)
    codes = np.zeros(K, np.uint8)
    _load().zo_unpack_row(_ptr(words), K, bits, _ptr(codes))
    return codes


def quantize_pack(w, bits, group=GROUP):
    """W (N x K fp32) -> (packed uint32 N x K*b/32, scales u16 N x G, zeros u16 N x G)."""
    w = _c(w, np.float32)
    N, K = w.shape
    G = max(K // group, 1)
    packed = np.zeros((N, max(K * bits // 32, 1)), np.uint32)
    scales = np.zeros((N, G), np.uint16)
    zeros = np.zeros((N, G), np.uint16)
    st = _load().zo_quantize_pack(_ptr(w), N, K, bits, group,
                                  _ptr(packed), _ptr(scales), _ptr(zeros))
    if st != OK:
        raise OracleError(st)
    return packed, scales, zeros


def quantize_pack_symmetric(w, bits, group=GROUP):
    """Symmetric quantizer over W (N x K fp32); same outputs as quantize_pack."""
    w = _c(w, np.float32)
    N, K = w.shape
    G = max(K // group, 1)
    packed = np.zeros((N, max(K * bits // 32, 1)), np.uint32)
    scales = np.zeros((N, G), np.uint16)
    zeros = np.zeros((N, G), np.uint16)
    st = _load().zo_quantize_pack_symmetric(_ptr(w), N, K, bits, group,
                                            _ptr(packed), _ptr(scales), _ptr(zeros))
    if st != OK:
        raise OracleError(st)
    return packed, scales, zeros


def unpack(packed, N, K, bits):
    packed = _c(packed, np.uint32)
    codes = np.zeros((N, K), np.uint8)
    st = _load().zo_unpack(_ptr(packed), N, K, bits, _ptr(codes))
    if st != OK:
        raise OracleError(st)
    return codes


def dequant(packed, scales, zeros, bits, N, K, group=GROUP):
    packed = _c(packed, np.uint32)
    scales = _c(scales, np.uint16)
    zeros = _c(zeros, np.uint16)
    w_hat = np.zeros((N, K), np.float64)
    st = _load().zo_dequant(_ptr(packed), _ptr(scales), _ptr(zeros),
                            bits, group, N, K, _ptr(w_hat))
    if st != OK:
        raise OracleError(st)
    return w_hat


def linear(x16, packed, scales, zeros, bits, N, K, rows=None, group=GROUP, xfmt="f16"):
    """x16: M x K uint16 (fp16 bits, or bf16 bits with xfmt="bf16"). Returns
    (y, bound), each M x len(rows) (or M x N when rows is None), fp64.
    bits=16: `packed` is the N x K fp16 weights (uint16 bits) and scales/zeros
    are not used (pass None)."""
    x16 = _c(x16, np.uint16)
    M = x16.shape[0]
    if bits == 16:
        packed = _c(packed, np.uint16)
        scales = np.zeros(1, np.uint16) if scales is None else _c(scales, np.uint16)
        zeros = np.zeros(1, np.uint16) if zeros is None else _c(zeros, np.uint16)
    else:
        packed = _c(packed, np.uint32)
        scales = _c(scales, np.uint16)
        zeros = _c(zeros, np.uint16)
    if rows is None:
        nrows = N
        rows_p = None
    else:
        rows = _c(rows, np.int64)
        nrows = rows.size
        rows_p = _ptr(rows)
    y = np.zeros((M, nrows), np.float64)
    bound = np.zeros((M, nrows), np.float64)
    st = _load().zo_linear_rows_ex(_ptr(x16), {"f16": 0, "bf16": 1}[xfmt], M, K, _ptr(packed),
                                   _ptr(scales), _ptr(zeros), bits, group, N, rows_p, nrows,
                                   _ptr(y), _ptr(bound))
    if st != OK:
        raise OracleError(st)
    return y, bound


def set_threads(n):
    _load().zo_set_threads(int(n))


def get_threads():
    return _load().zo_get_threads()
