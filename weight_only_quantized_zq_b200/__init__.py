"""Python binding of libzq, the B200 (sm_100a) weight-only quantized linear.

Argument marshalling only: every step of the computation runs in the CUDA
kernels behind the C ABI of ``include/zq.h``; the .zse container reader and
loader of ``include/zq_zse.h`` run in the library's native code.  The functions carry the C names;
tensor arguments are torch CUDA tensors (their device pointers are passed), and
``stream`` defaults to torch's current stream on the tensor's device.

There is no CPU fallback: importing this package raises if ``libzq.so`` has
not been built (``python weight_only_quantized_zq_b200/build.py``).
"""
import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libzq.so")

ZQ_OK = 0
ZQ_ERR_INVALID_ARG = 1
ZQ_ERR_UNSUPPORTED = 2
ZQ_ERR_NONFINITE = 3
ZQ_ERR_CUDA = 4
ZQ_ERR_TIMEOUT = 5
GROUP = 128

# Every symbol the headers declare (checked by the CPU test suite).
EXPORTS = ("zq_packed_words", "zq_quantize_pack", "zq_quantize_pack_symmetric", "zq_linear", "zq_linear_noalloc", "zq_linear_stack",
           "zq_unpack", "zq_reserve_workspace", "zq_attach_workspace", "zq_release_workspace",
           "zq_release_all_workspaces", "zq_linear_workspace_bytes", "zq_linear_stack_workspace_bytes",
           "zq_set_wait_limit_ns", "zq_status_string", "zq_last_error", "zq_check_device", "zq_kernel_launches",
           "zq_version",
           "zq_zse_open", "zq_zse_close", "zq_zse_flags", "zq_zse_tensor_count", "zq_zse_tensor_info",
           "zq_zse_find", "zq_zse_section", "zq_zse_weight_bytes", "zq_zse_verify", "zq_zse_load_weights",
           "zq_kv_plane_bytes", "zq_kv_append", "zq_kv_gather",
           "zq_linear_partial", "zq_linear_partial_stack", "zq_linear_partial_stack_workspace_bytes",
           "zq_reduce_partials", "zq_linear_bf16", "zq_linear_bf16_workspace_bytes", "zq_linear_stack_bf16",
           "zq_linear_stack_bf16_workspace_bytes", "zq_dequant")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing; build it with "
                      "`python weight_only_quantized_zq_b200/build.py`")

_lib = ctypes.CDLL(LIB_PATH)
_P = ctypes.c_void_p
_I = ctypes.c_int
_S = ctypes.c_size_t

_lib.zq_packed_words.argtypes = [_I, _I, _I]
_lib.zq_packed_words.restype = _S
_lib.zq_quantize_pack.argtypes = [_P, _I, _I, _I, _I, _P, _P, _P, _P]
_lib.zq_quantize_pack.restype = _I
_lib.zq_quantize_pack_symmetric.argtypes = [_P, _I, _I, _I, _I, _P, _P, _P, _P]
_lib.zq_quantize_pack_symmetric.restype = _I
_lib.zq_linear.argtypes = [_P, _P, _P, _P, _I, _I, _I, _I, _I, _P, _P]
_lib.zq_linear.restype = _I
_lib.zq_linear_noalloc.argtypes = [_P, _P, _P, _P, _I, _I, _I, _I, _I, _P, _P]
_lib.zq_linear_noalloc.restype = _I
_lib.zq_linear_stack.argtypes = [_P, _I, _P]
_lib.zq_linear_stack.restype = _I
_lib.zq_unpack.argtypes = [_P, _I, _I, _I, _P, _P]
_lib.zq_unpack.restype = _I
_lib.zq_dequant.argtypes = [_P, _P, _P, _I, _I, _I, _I, _P, _P]
_lib.zq_dequant.restype = _I
_lib.zq_reserve_workspace.argtypes = [_S, _P]
_lib.zq_reserve_workspace.restype = _I
_lib.zq_attach_workspace.argtypes = [_P, _S, _P]
_lib.zq_attach_workspace.restype = _I
_lib.zq_release_workspace.argtypes = [_P]
_lib.zq_release_workspace.restype = _I
_lib.zq_release_all_workspaces.argtypes = []
_lib.zq_release_all_workspaces.restype = _I
_lib.zq_linear_workspace_bytes.argtypes = [_I, _I, _I, _I]
_lib.zq_linear_workspace_bytes.restype = _S
_lib.zq_set_wait_limit_ns.argtypes = [ctypes.c_uint64]
_lib.zq_set_wait_limit_ns.restype = _I
_lib.zq_status_string.argtypes = [_I]
_lib.zq_status_string.restype = ctypes.c_char_p
_lib.zq_last_error.argtypes = []
_lib.zq_last_error.restype = ctypes.c_char_p
_lib.zq_check_device.argtypes = []
_lib.zq_check_device.restype = _I
_lib.zq_kernel_launches.argtypes = []
_lib.zq_kernel_launches.restype = ctypes.c_uint64
_lib.zq_version.argtypes = []
_lib.zq_version.restype = _I
_U64 = ctypes.c_uint64
_lib.zq_zse_open.argtypes = [ctypes.c_char_p, ctypes.POINTER(_P)]
_lib.zq_zse_open.restype = _I
_lib.zq_zse_close.argtypes = [_P]
_lib.zq_zse_close.restype = None
_lib.zq_zse_flags.argtypes = [_P]
_lib.zq_zse_flags.restype = ctypes.c_uint32
_lib.zq_zse_tensor_count.argtypes = [_P]
_lib.zq_zse_tensor_count.restype = _I
_lib.zq_zse_find.argtypes = [_P, ctypes.c_char_p]
_lib.zq_zse_find.restype = _I
_lib.zq_zse_section.argtypes = [_P, _I, ctypes.POINTER(_U64)]
_lib.zq_zse_section.restype = _P
_lib.zq_zse_weight_bytes.argtypes = [_P]
_lib.zq_zse_weight_bytes.restype = _U64
_lib.zq_zse_verify.argtypes = [_P]
_lib.zq_zse_verify.restype = _I
_lib.zq_zse_load_weights.argtypes = [_P, _P, _U64, _P]
_lib.zq_zse_load_weights.restype = _I


class ZQError(RuntimeError):
    def __init__(self, status, message):
        super().__init__(f"{zq_status_string(status)}: {message}")
        self.status = status


class zq_zse_tensor(ctypes.Structure):
    _fields_ = [("name", ctypes.c_char * 64), ("kind", _I), ("bits", _I), ("group", _I),
                ("rows", _U64), ("cols", _U64), ("data_offset", _U64), ("data_bytes", _U64),
                ("scales_offset", _U64), ("zeros_offset", _U64)]


_lib.zq_zse_tensor_info.argtypes = [_P, _I, ctypes.POINTER(zq_zse_tensor)]
_lib.zq_zse_tensor_info.restype = _I


class zq_kv_plane(ctypes.Structure):
    _fields_ = [("ring", _P), ("packed", _P), ("scales", _P), ("zeros", _P), ("window", _I),
                ("capacity", _I), ("heads", _I), ("dim", _I), ("bits", _I)]


_lib.zq_kv_plane_bytes.argtypes = [_I, _I, _I, _I, _I]
_lib.zq_kv_plane_bytes.restype = _S
_lib.zq_kv_append.argtypes = [ctypes.POINTER(zq_kv_plane), _I, _P, _I, _P]
_lib.zq_kv_append.restype = _I
_lib.zq_kv_gather.argtypes = [ctypes.POINTER(zq_kv_plane), _I, _I, _I, _P, _P]
_lib.zq_kv_gather.restype = _I


class zq_linear_desc(ctypes.Structure):
    _fields_ = [("x", _P), ("packed", _P), ("scales", _P), ("zeros", _P), ("out", _P),
                ("bits", _I), ("group", _I), ("M", _I), ("N", _I), ("K", _I)]


_lib.zq_linear_stack_workspace_bytes.argtypes = [_P, _I]
_lib.zq_linear_stack_workspace_bytes.restype = _S


class zq_partial_desc(ctypes.Structure):
    _fields_ = [("x", _P), ("packed", _P), ("scales", _P), ("zeros", _P), ("out", _P),
                ("bits", _I), ("group", _I), ("M", _I), ("N", _I), ("K", _I)]


_lib.zq_linear_partial.argtypes = [_P, _P, _P, _P, _I, _I, _I, _I, _I, _P, _P]
_lib.zq_linear_partial.restype = _I
_lib.zq_linear_partial_stack.argtypes = [_P, _I, _P]
_lib.zq_linear_partial_stack.restype = _I
_lib.zq_linear_partial_stack_workspace_bytes.argtypes = [_P, _I]
_lib.zq_linear_partial_stack_workspace_bytes.restype = _S
_lib.zq_reduce_partials.argtypes = [ctypes.POINTER(_P), _I, _S, _P, _P]
_lib.zq_reduce_partials.restype = _I
_lib.zq_linear_bf16.argtypes = [_P, _P, _P, _P, _I, _I, _I, _I, _I, _P, _P]
_lib.zq_linear_bf16.restype = _I
_lib.zq_linear_bf16_workspace_bytes.argtypes = [_I, _I, _I, _I]
_lib.zq_linear_bf16_workspace_bytes.restype = _S
_lib.zq_linear_stack_bf16.argtypes = [_P, _I, _P]
_lib.zq_linear_stack_bf16.restype = _I
_lib.zq_linear_stack_bf16_workspace_bytes.argtypes = [_P, _I]
_lib.zq_linear_stack_bf16_workspace_bytes.restype = _S


def _check(status):
    if status != ZQ_OK:
        raise ZQError(status, zq_last_error())


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream, like=None):
    if stream is None:
        dev = like.device if isinstance(like, torch.Tensor) else None
        return torch.cuda.current_stream(dev).cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def zq_status_string(status):
    return _lib.zq_status_string(int(status)).decode()


def zq_last_error():
    return _lib.zq_last_error().decode()


def zq_version():
    return _lib.zq_version()


def zq_kv_plane_bytes(window, capacity, heads, dim, bits):
    return _lib.zq_kv_plane_bytes(window, capacity, heads, dim, bits)


def zq_check_device():
    _check(_lib.zq_check_device())


def zq_kernel_launches():
    return _lib.zq_kernel_launches()


def zq_packed_words(N, K, bits):
    return _lib.zq_packed_words(N, K, bits)


def zq_linear_workspace_bytes(bits, M, N, K):
    return _lib.zq_linear_workspace_bytes(bits, M, N, K)


def zq_reserve_workspace(nbytes, stream=None):
    _check(_lib.zq_reserve_workspace(nbytes, _stream(stream)))


def zq_attach_workspace(buffer, nbytes, stream=None):
    _check(_lib.zq_attach_workspace(_ptr(buffer), nbytes, _stream(stream, buffer)))


def zq_release_workspace(stream=None):
    _check(_lib.zq_release_workspace(_stream(stream)))


def zq_release_all_workspaces():
    _check(_lib.zq_release_all_workspaces())


def zq_linear_stack_workspace_bytes(ops, n_ops=None):
    """ops: a ctypes array from make_descs(), or an iterable accepted by it."""
    if not isinstance(ops, ctypes.Array):
        ops, n = make_descs(ops)
        n_ops = n if n_ops is None else n_ops
    return _lib.zq_linear_stack_workspace_bytes(ops, n_ops)


def zq_set_wait_limit_ns(ns):
    _check(_lib.zq_set_wait_limit_ns(int(ns)))


def zq_quantize_pack(w, N, K, bits, group, packed, scales, zeros, stream=None):
    _check(_lib.zq_quantize_pack(_ptr(w), N, K, bits, group, _ptr(packed), _ptr(scales),
                                 _ptr(zeros), _stream(stream, w)))


def zq_quantize_pack_symmetric(w, N, K, bits, group, packed, scales, zeros, stream=None):
    _check(_lib.zq_quantize_pack_symmetric(_ptr(w), N, K, bits, group, _ptr(packed), _ptr(scales),
                                           _ptr(zeros), _stream(stream, w)))


def zq_linear(x, packed, scales, zeros, bits, group, M, N, K, out, stream=None):
    _check(_lib.zq_linear(_ptr(x), _ptr(packed), _ptr(scales), _ptr(zeros), bits, group,
                          M, N, K, _ptr(out), _stream(stream, x)))


def zq_linear_noalloc(x, packed, scales, zeros, bits, group, M, N, K, out, stream=None):
    _check(_lib.zq_linear_noalloc(_ptr(x), _ptr(packed), _ptr(scales), _ptr(zeros), bits, group,
                                  M, N, K, _ptr(out), _stream(stream, x)))


def make_descs(ops):
    """ops: iterable of dicts/tuples (x, packed, scales, zeros, out, bits, group, M, N, K)."""
    ops = list(ops)
    arr = (zq_linear_desc * max(len(ops), 1))()
    for i, o in enumerate(ops):
        if isinstance(o, dict):
            o = (o["x"], o["packed"], o["scales"], o["zeros"], o["out"], o["bits"],
                 o.get("group", GROUP), o["M"], o["N"], o["K"])
        x, packed, scales, zeros, out, bits, group, M, N, K = o
        arr[i] = zq_linear_desc(_ptr(x), _ptr(packed), _ptr(scales), _ptr(zeros), _ptr(out),
                                bits, group, M, N, K)
    return arr, len(ops)


def zq_linear_stack(ops, n_ops=None, stream=None):
    """ops: a ctypes array from make_descs(), or an iterable accepted by it."""
    if not isinstance(ops, ctypes.Array):
        ops, n = make_descs(ops)
        n_ops = n if n_ops is None else n_ops
    _check(_lib.zq_linear_stack(ops, n_ops, _stream(stream)))


def zq_linear_partial(x, packed, scales, zeros, bits, group, M, N, K, out, stream=None):
    _check(_lib.zq_linear_partial(_ptr(x), _ptr(packed), _ptr(scales), _ptr(zeros), bits, group,
                                  M, N, K, _ptr(out), _stream(stream, x)))


def make_partial_descs(ops):
    """ops: iterable of tuples (x, packed, scales, zeros, out_fp32, bits, group, M, N, K)."""
    ops = list(ops)
    arr = (zq_partial_desc * max(len(ops), 1))()
    for i, (x, packed, scales, zeros, out, bits, group, M, N, K) in enumerate(ops):
        arr[i] = zq_partial_desc(_ptr(x), _ptr(packed), _ptr(scales), _ptr(zeros), _ptr(out),
                                 bits, group, M, N, K)
    return arr, len(ops)


def zq_linear_partial_stack(ops, n_ops=None, stream=None):
    """ops: a ctypes array from make_partial_descs(), or an iterable accepted by it."""
    if not isinstance(ops, ctypes.Array):
        ops, n = make_partial_descs(ops)
        n_ops = n if n_ops is None else n_ops
    _check(_lib.zq_linear_partial_stack(ops, n_ops, _stream(stream)))


def zq_linear_partial_stack_workspace_bytes(ops, n_ops=None):
    if not isinstance(ops, ctypes.Array):
        ops, n = make_partial_descs(ops)
        n_ops = n if n_ops is None else n_ops
    return _lib.zq_linear_partial_stack_workspace_bytes(ops, n_ops)


def zq_reduce_partials(parts, count, out, stream=None):
    """parts: sequence of fp32 device buffers (tensors or addresses), summed in order."""
    arr = (_P * len(parts))(*[_ptr(p) for p in parts])
    _check(_lib.zq_reduce_partials(arr, len(parts), count, _ptr(out),
                                   _stream(stream, out if isinstance(out, torch.Tensor) else None)))


def zq_linear_bf16(x, packed, scales, zeros, bits, group, M, N, K, out, stream=None):
    _check(_lib.zq_linear_bf16(_ptr(x), _ptr(packed), _ptr(scales), _ptr(zeros), bits, group,
                               M, N, K, _ptr(out), _stream(stream, x)))


def zq_linear_bf16_workspace_bytes(bits, M, N, K):
    return _lib.zq_linear_bf16_workspace_bytes(bits, M, N, K)


def zq_linear_stack_bf16(ops, n_ops=None, stream=None):
    if not isinstance(ops, ctypes.Array):
        ops, n = make_descs(ops)
        n_ops = n if n_ops is None else n_ops
    _check(_lib.zq_linear_stack_bf16(ops, n_ops, _stream(stream)))


def zq_linear_stack_bf16_workspace_bytes(ops, n_ops=None):
    if not isinstance(ops, ctypes.Array):
        ops, n = make_descs(ops)
        n_ops = n if n_ops is None else n_ops
    return _lib.zq_linear_stack_bf16_workspace_bytes(ops, n_ops)


def zq_dequant(packed, scales, zeros, bits, group, N, K, w_hat, stream=None):
    _check(_lib.zq_dequant(_ptr(packed), _ptr(scales), _ptr(zeros), bits, group, N, K, _ptr(w_hat),
                           _stream(stream, packed)))


def zq_unpack(packed, N, K, bits, codes, stream=None):
    _check(_lib.zq_unpack(_ptr(packed), N, K, bits, _ptr(codes), _stream(stream, packed)))


# ------------------------------------------------------------ conveniences --

def alloc_quantized(N, K, bits, device="cuda", group=GROUP):
    """Empty (packed, scales, zeros) buffers for an N x K tensor."""
    packed = torch.empty(N * K * bits // 32, dtype=torch.int32, device=device)
    scales = torch.empty(N, K // group, dtype=torch.int16, device=device)
    zeros = torch.empty(N, K // group, dtype=torch.int16, device=device)
    return packed, scales, zeros


def _need(t, nbytes, dtype, what, device):
    if (not isinstance(t, torch.Tensor) or t.dtype != dtype or not t.is_contiguous()
            or t.numel() * t.element_size() != nbytes or t.device != device):
        raise ZQError(ZQ_ERR_INVALID_ARG, f"{what}: need a contiguous {dtype} tensor of {nbytes} bytes on "
                      f"{device}, got {getattr(t, 'dtype', type(t))} of "
                      f"{t.numel() * t.element_size() if isinstance(t, torch.Tensor) else '?'} bytes")


def quantize(w, bits, stream=None, symmetric=False, group=GROUP):
    """fp32 CUDA tensor N x K -> (packed, scales, zeros) via zq_quantize_pack
    (or zq_quantize_pack_symmetric); both give the same storage format.
    group: 128 (default), 64 or 32 weights per scale and zero."""
    if w.dim() != 2:
        raise ZQError(ZQ_ERR_INVALID_ARG, f"w must be 2-D (N x K), got shape {tuple(w.shape)}")
    N, K = w.shape
    _need(w, N * K * 4, torch.float32, "w", w.device)
    if group not in (32, 64, 128) or K % 128:
        raise ZQError(ZQ_ERR_UNSUPPORTED if group not in (32, 64, 128) else ZQ_ERR_INVALID_ARG,
                      f"group={group} (32, 64 or 128) and K={K} (a multiple of 128)")
    packed, scales, zeros = alloc_quantized(N, K, bits, w.device, group)
    fn = zq_quantize_pack_symmetric if symmetric else zq_quantize_pack
    fn(w, N, K, bits, group, packed, scales, zeros, stream)
    return packed, scales, zeros


def ensure_workspace(nbytes, stream=None):
    """Reserves a workspace of at least `nbytes` on `stream` (default: torch's
    current stream) unless it already holds that much.  A reservation that
    grows the buffer waits for the stream; this happens here, between calls,
    never inside zq_linear or zq_linear_stack."""
    if nbytes > 0:
        zq_reserve_workspace(nbytes, stream)


def linear_stack(ops, stream=None):
    """zq_linear_stack over `ops` (see make_descs) after making sure the
    stream's workspace covers it."""
    arr, n = ops if isinstance(ops, tuple) and isinstance(ops[0], ctypes.Array) else make_descs(ops)
    ensure_workspace(zq_linear_stack_workspace_bytes(arr, n), stream)
    zq_linear_stack(arr, n, stream)


def linear_partial(x, packed, scales, zeros, bits, N, out=None, stream=None):
    """fp16 CUDA x (M x K) -> fp32 partial sums (M x N) via zq_linear_partial."""
    M, K = x.shape
    _need(x, M * K * 2, torch.float16, "x", x.device)
    if out is None:
        out = torch.empty(M, N, dtype=torch.float32, device=x.device)
    _need(out, M * N * 4, torch.float32, "out", x.device)
    ensure_workspace(zq_linear_workspace_bytes(bits, M, N, K), stream if stream is not None else
                     torch.cuda.current_stream(x.device))
    zq_linear_partial(x, packed, scales, zeros, bits, GROUP, M, N, K, out, stream)
    return out


def linear(x, packed, scales, zeros, bits, N, out=None, stream=None, group=GROUP):
    """fp16 (or bfloat16) CUDA x (M x K) -> out (M x N) of the same type via
    zq_linear (zq_linear_bf16), reserving the workspace it needs on the stream
    first.  bits=16: `packed` is the fp16 weights (N x K) and scales/zeros may
    be None."""
    if x.dim() != 2:
        raise ZQError(ZQ_ERR_INVALID_ARG, f"x must be 2-D (M x K), got shape {tuple(x.shape)}")
    M, K = x.shape
    bf16 = x.dtype == torch.bfloat16
    xt = torch.bfloat16 if bf16 else torch.float16
    _need(x, M * K * 2, xt, "x", x.device)
    if K % 128 == 0 and bits in (2, 3, 4, 8, 16) and group in (32, 64, 128):  # else the library reports it
        _need(packed, N * K * bits // 8, packed.dtype, "packed", x.device)
        if bits != 16:
            _need(scales, N * (K // group) * 2, scales.dtype, "scales", x.device)
            _need(zeros, N * (K // group) * 2, zeros.dtype, "zeros", x.device)
    if out is None:
        out = torch.empty(M, N, dtype=xt, device=x.device)
    _need(out, M * N * 2, xt, "out", x.device)
    ws = zq_linear_bf16_workspace_bytes if bf16 else zq_linear_workspace_bytes
    ensure_workspace(ws(bits, M, N, K), stream if stream is not None else torch.cuda.current_stream(x.device))
    (zq_linear_bf16 if bf16 else zq_linear)(x, packed, scales, zeros, bits, group, M, N, K, out, stream)
    return out


# ------------------------------------------------------------ .zse reader --

ZSE_CONFIG, ZSE_TOKENIZER, ZSE_WEIGHT_INDEX, ZSE_WEIGHT_DATA, ZSE_KERNELS = 1, 2, 3, 4, 5


class KVPlane:
    """One K or V plane of the quantized KV cache (zq_kv.h): the newest
    `window` tokens in an fp16 ring, older ones quantized at `bits` in the
    store.  Owns its device buffers; `tokens` counts what it holds."""

    def __init__(self, window, capacity, heads, dim, bits=4, device="cuda"):
        if zq_kv_plane_bytes(window, capacity, heads, dim, bits) == 0:
            raise ZQError(ZQ_ERR_INVALID_ARG, f"bad plane shape {(window, capacity, heads, dim, bits)}")
        self.ring = torch.empty(window, heads, dim, dtype=torch.float16, device=device)
        self.packed = torch.empty(capacity, heads, dim * bits // 32, dtype=torch.int32, device=device)
        self.scales = torch.empty(capacity, heads, dim // GROUP, dtype=torch.int16, device=device)
        self.zeros = torch.empty(capacity, heads, dim // GROUP, dtype=torch.int16, device=device)
        self.desc = zq_kv_plane(_ptr(self.ring), _ptr(self.packed), _ptr(self.scales), _ptr(self.zeros),
                                window, capacity, heads, dim, bits)
        self.window, self.capacity, self.heads, self.dim, self.bits = window, capacity, heads, dim, bits
        self.tokens = 0

    def _rows_ok(self, t, n, what):
        if (t.dtype != torch.float16 or not t.is_contiguous() or tuple(t.shape) != (n, self.heads, self.dim)
                or t.device != self.ring.device):
            raise ZQError(ZQ_ERR_INVALID_ARG, f"{what} must be a contiguous fp16 tensor of shape "
                          f"{(n, self.heads, self.dim)} on {self.ring.device}, got {tuple(t.shape)} "
                          f"{t.dtype} on {t.device}")

    def append(self, rows, stream=None):
        """rows: fp16 CUDA tensor (n, heads, dim)."""
        n = rows.shape[0]
        self._rows_ok(rows, n, "rows")
        _check(_lib.zq_kv_append(ctypes.byref(self.desc), self.tokens, _ptr(rows), n, _stream(stream, rows)))
        self.tokens += n

    def gather(self, a=0, b=None, out=None, stream=None):
        """Tokens [a, b) as an fp16 tensor (b - a, heads, dim)."""
        b = self.tokens if b is None else b
        if out is None:
            out = torch.empty(max(b - a, 0), self.heads, self.dim, dtype=torch.float16, device=self.ring.device)
        self._rows_ok(out, max(b - a, 0), "out")
        _check(_lib.zq_kv_gather(ctypes.byref(self.desc), self.tokens, a, b, _ptr(out), _stream(stream, out)))
        return out


class ZseFile:
    """An open .zse file (``zq_zse_open``); close() or use as a context manager."""

    def __init__(self, path):
        h = _P()
        _check(_lib.zq_zse_open(os.fsencode(path), ctypes.byref(h)))
        self._h = h

    def close(self):
        if self._h:
            _lib.zq_zse_close(self._h)
            self._h = None

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.close()

    @property
    def flags(self):
        return _lib.zq_zse_flags(self._h)

    @property
    def weight_bytes(self):
        return _lib.zq_zse_weight_bytes(self._h)

    def tensors(self):
        out = []
        for i in range(_lib.zq_zse_tensor_count(self._h)):
            t = zq_zse_tensor()
            _check(_lib.zq_zse_tensor_info(self._h, i, ctypes.byref(t)))
            out.append({"name": t.name.decode(), "kind": t.kind, "bits": t.bits, "group": t.group,
                        "rows": t.rows, "cols": t.cols, "data_offset": t.data_offset,
                        "data_bytes": t.data_bytes, "scales_offset": t.scales_offset,
                        "zeros_offset": t.zeros_offset})
        return out

    def find(self, name):
        return _lib.zq_zse_find(self._h, name.encode())

    def section(self, kind):
        """Bytes of a section (a copy), or None."""
        n = _U64()
        p = _lib.zq_zse_section(self._h, kind, ctypes.byref(n))
        return None if not p else ctypes.string_at(p, n.value)

    def verify(self):
        _check(_lib.zq_zse_verify(self._h))

    def load_weights(self, dst, stream=None):
        """Copies WEIGHT_DATA into the uint8 CUDA tensor dst (synchronous)."""
        _check(_lib.zq_zse_load_weights(self._h, _ptr(dst), dst.numel() * dst.element_size(),
                                        _stream(stream, dst)))

    def views(self, weights):
        """Per-tensor views into `weights`, a uint8 tensor holding WEIGHT_DATA
        (as filled by load_weights): name -> {"bits", "rows", "cols", and
        "packed" (int32 rows x cols*bits/32), "scales", "zeros" (int16 rows x
        cols/128) for a quantized tensor, or "data" (fp16 rows x cols)}.  No
        copy: the views share the buffer, ready for zq_linear / zq_linear_stack."""
        if weights.dtype != torch.uint8 or weights.dim() != 1 or weights.numel() < self.weight_bytes:
            raise ZQError(ZQ_ERR_INVALID_ARG, "weights must be a 1-D uint8 tensor of at least "
                          f"{self.weight_bytes} bytes")
        out = {}
        for t in self.tensors():
            rows, cols = t["rows"], t["cols"]

            def view(off, nbytes, dtype, shape):
                return weights[off:off + nbytes].view(dtype).view(*shape)

            if t["kind"] == 1:
                G = cols // t["group"]
                out[t["name"]] = {
                    "bits": t["bits"], "rows": rows, "cols": cols,
                    "packed": view(t["data_offset"], t["data_bytes"], torch.int32, (rows, cols * t["bits"] // 32)),
                    "scales": view(t["scales_offset"], rows * G * 2, torch.int16, (rows, G)),
                    "zeros": view(t["zeros_offset"], rows * G * 2, torch.int16, (rows, G))}
            else:
                out[t["name"]] = {"bits": 16, "rows": rows, "cols": cols,
                                  "data": view(t["data_offset"], t["data_bytes"], torch.float16, (rows, cols))}
        return out
