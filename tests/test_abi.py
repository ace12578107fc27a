"""CPU-only checks of the C ABI: the library loads, exports every function the
header declares, and its host-side validation rejects bad arguments before any
CUDA call (these calls never touch a GPU)."""
import ctypes
import glob
import os
import re
import shutil
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADERS = sorted(glob.glob(os.path.join(ROOT, "include", "*.h")))


def _build_library():
    import importlib.util
    path = os.path.join(ROOT, "weight_only_quantized_zq_b200", "build.py")
    spec = importlib.util.spec_from_file_location("zq_build", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod.build()


@pytest.fixture(scope="module")
def zq():
    _build_library()
    import weight_only_quantized_zq_b200 as m
    return m


def _declared_functions():
    text = "".join(open(h).read() for h in HEADERS)
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(zq_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_expected_entry_points(zq):
    decl = _declared_functions()
    for name in ("zq_quantize_pack", "zq_linear", "zq_linear_stack", "zq_unpack"):
        assert name in decl
    assert set(decl) == set(zq.EXPORTS), (decl, zq.EXPORTS)


def test_library_exports_every_declared_symbol(zq):
    lib = ctypes.CDLL(zq.LIB_PATH)
    for name in _declared_functions():
        assert hasattr(lib, name), name
    out = subprocess.run(["nm", "-D", "--defined-only", zq.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r" T (zq_\w+)", out))
    assert set(_declared_functions()) <= exported
    # nothing else of ours leaks out of the shared object
    assert not [s for s in exported if s not in _declared_functions()]


def test_status_strings_and_version(zq):
    assert zq.zq_status_string(zq.ZQ_OK) == "ZQ_OK"
    assert zq.zq_status_string(zq.ZQ_ERR_NONFINITE) == "ZQ_ERR_NONFINITE"
    assert zq.zq_status_string(99) == "ZQ_UNKNOWN_STATUS"
    assert zq.zq_version() >= 100


def test_packed_words_closed_form(zq):
    assert zq.zq_packed_words(4608, 3584, 4) == 4608 * 3584 * 4 // 32
    assert zq.zq_packed_words(55296, 5120, 3) == 55296 * 5120 * 3 // 32
    assert zq.zq_packed_words(1, 128, 2) == 8
    assert zq.zq_packed_words(1, 100, 4) == 0
    assert zq.zq_packed_words(1, 128, 5) == 0
    assert zq.zq_packed_words(0, 128, 4) == 0


A = 1 << 20  # a fake, 16-byte aligned address: validation fails before any use


def _lin(zq, **kw):
    args = dict(x=A, packed=A, scales=A, zeros=A, bits=4, group=128, M=1, N=16, K=128, out=A)
    args.update(kw)
    return zq._lib.zq_linear(args["x"], args["packed"], args["scales"], args["zeros"],
                             args["bits"], args["group"], args["M"], args["N"], args["K"],
                             args["out"], None)


@pytest.mark.parametrize("kw,status", [
    (dict(bits=5), 2), (dict(bits=1), 2), (dict(bits=12), 2), (dict(group=48), 2), (dict(group=256), 2),
    (dict(group=16), 2), (dict(bits=16, K=100), 1), (dict(bits=16, x=0), 1),
    (dict(K=100), 1), (dict(K=0), 1), (dict(N=0), 1), (dict(M=0), 1), (dict(M=-3), 1),
    (dict(x=0), 1), (dict(packed=0), 1), (dict(scales=0), 1), (dict(zeros=0), 1),
    (dict(out=0), 1), (dict(x=A + 8), 1), (dict(out=A + 2), 1), (dict(packed=A + 4), 1),
])
def test_linear_rejects(zq, kw, status):
    assert _lin(zq, **kw) == status
    assert zq.zq_last_error() != ""


@pytest.mark.parametrize("name", ["zq_quantize_pack", "zq_quantize_pack_symmetric"])
def test_quantize_rejects(zq, name):
    q = getattr(zq._lib, name)
    assert q(A, 4, 256, 5, 128, A, A, A, None) == zq.ZQ_ERR_UNSUPPORTED
    assert q(A, 4, 256, 4, 16, A, A, A, None) == zq.ZQ_ERR_UNSUPPORTED
    assert q(A, 4, 256, 16, 128, A, A, A, None) == zq.ZQ_ERR_UNSUPPORTED  # fp16 weights are not quantized
    assert q(A, 4, 200, 4, 128, A, A, A, None) == zq.ZQ_ERR_INVALID_ARG
    assert q(0, 4, 256, 4, 128, A, A, A, None) == zq.ZQ_ERR_INVALID_ARG
    assert q(A, 4, 256, 4, 128, A + 1, A, A, None) == zq.ZQ_ERR_INVALID_ARG
    assert q(A, 4, 256, 4, 128, A, A, 0, None) == zq.ZQ_ERR_INVALID_ARG


def test_kv_plane_bytes_and_rejects(zq):
    # ring 256 x 4 x 128 fp16 + store 4096 x 4 x (64 code bytes) + 2 x 4096 x 4 x 2 (scales, zeros)
    assert zq.zq_kv_plane_bytes(256, 4096, 4, 128, 4) == 262144 + 1048576 + 2 * 32768
    assert zq.zq_kv_plane_bytes(256, 4096, 4, 100, 4) == 0
    assert zq.zq_kv_plane_bytes(256, 4096, 4, 128, 5) == 0
    pl = zq.zq_kv_plane(A, A, A, A, 8, 8, 1, 128, 4)
    assert zq._lib.zq_kv_append(ctypes.byref(pl), 5, A, 4, None) == zq.ZQ_ERR_INVALID_ARG  # past capacity
    assert zq._lib.zq_kv_append(ctypes.byref(pl), 0, A + 2, 1, None) == zq.ZQ_ERR_INVALID_ARG  # misaligned
    assert zq._lib.zq_kv_append(ctypes.byref(pl), 0, A, 0, None) == zq.ZQ_OK  # nothing to do
    assert zq._lib.zq_kv_gather(ctypes.byref(pl), 4, 3, 5, A, None) == zq.ZQ_ERR_INVALID_ARG
    assert zq._lib.zq_kv_gather(ctypes.byref(pl), 4, 2, 2, A, None) == zq.ZQ_OK
    bad = zq.zq_kv_plane(A, A, A, A, 8, 8, 1, 128, 6)
    assert zq._lib.zq_kv_append(ctypes.byref(bad), 0, A, 1, None) == zq.ZQ_ERR_UNSUPPORTED
    assert zq._lib.zq_kv_append(None, 0, A, 1, None) == zq.ZQ_ERR_INVALID_ARG


def test_unpack_rejects(zq):
    u = zq._lib.zq_unpack
    assert u(A, 4, 256, 6, A, None) == zq.ZQ_ERR_UNSUPPORTED
    assert u(A, 4, 96, 4, A, None) == zq.ZQ_ERR_INVALID_ARG
    assert u(0, 4, 256, 4, A, None) == zq.ZQ_ERR_INVALID_ARG


def test_stack_validates_every_op_first(zq):
    good = (A, A, A, A, A, 4, 128, 1, 16, 128)
    bad = (A, A, A, A, A, 4, 128, 1, 16, 130)
    arr, n = zq.make_descs([good, good, bad])
    assert zq._lib.zq_linear_stack(arr, n, None) == zq.ZQ_ERR_INVALID_ARG
    assert "op 2" in zq.zq_last_error()
    assert zq._lib.zq_linear_stack(None, 3, None) == zq.ZQ_ERR_INVALID_ARG
    assert zq._lib.zq_linear_stack(None, -1, None) == zq.ZQ_ERR_INVALID_ARG
    assert zq._lib.zq_linear_stack(None, 0, None) == zq.ZQ_OK


def test_import_fails_loudly_without_library(tmp_path):
    pkg = os.path.join(ROOT, "weight_only_quantized_zq_b200")
    dst = tmp_path / "weight_only_quantized_zq_b200"
    shutil.copytree(pkg, dst, ignore=shutil.ignore_patterns("*.so", "_build", "__pycache__"))
    code = "import weight_only_quantized_zq_b200"
    r = subprocess.run([sys.executable, "-c", code], cwd=tmp_path, capture_output=True, text=True)
    assert r.returncode != 0 and "libzq.so" in r.stderr


def test_kv_plane_binding_checks_shapes(zq):
    """The Python plane rejects mis-shaped or mistyped rows before any call
    into the library (a wrong shape would make the kernel read out of bounds)."""
    import torch
    pl = zq.KVPlane(4, 16, 2, 128, 4, device="cpu")
    for bad in (torch.zeros(3, 2, 64, dtype=torch.float16), torch.zeros(3, 2, 128, dtype=torch.float32),
                torch.zeros(2, 3, 128, dtype=torch.float16).transpose(0, 1)):
        with pytest.raises(zq.ZQError) as e:
            pl.append(bad)
        assert e.value.status == zq.ZQ_ERR_INVALID_ARG
    assert pl.tokens == 0
    with pytest.raises(zq.ZQError):
        pl.gather(0, 0, out=torch.zeros(1, 2, 128, dtype=torch.float16))


def test_linear_and_quantize_wrappers_check_buffers(zq):
    """The convenience wrappers size every buffer against (M, N, K, bits)
    before calling the library, which sees only pointers."""
    import torch
    x = torch.zeros(2, 256, dtype=torch.float16)
    p, s, z = zq.alloc_quantized(64, 256, 4, device="cpu")
    for args in ((x, p[:-1], s, z), (x, p, s[:-1], z), (x, p, s, z[:, :1]), (x.float(), p, s, z),
                 (x[:, :128], p, s, z)):
        with pytest.raises(zq.ZQError) as e:
            zq.linear(*args, 4, 64)
        assert e.value.status == zq.ZQ_ERR_INVALID_ARG
    with pytest.raises(zq.ZQError):
        zq.linear(x, p, s, z, 4, 64, out=torch.zeros(2, 63, dtype=torch.float16))
    with pytest.raises(zq.ZQError):
        zq.quantize(torch.zeros(4, 256, dtype=torch.float16), 4)
    with pytest.raises(zq.ZQError):
        zq.quantize(torch.zeros(256, 4).t(), 4)  # not contiguous
