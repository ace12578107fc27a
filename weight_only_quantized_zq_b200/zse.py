"""Writer of .zse container files (the layout of ``include/zq_zse.h``).

The pages' converter (quantizing a Hugging Face checkpoint) is out of scope;
this writer packs tensors that are already quantized (``zq_quantize_pack``
output, or any arrays in that format) and fp16 tensors into one mmap-ready
file, together with an opaque configuration (JSON), tokenizer and kernel
cache.  Reading and loading is native (``ZseFile`` in the package).

[wiki] "ZSE - open-source движок для запуска LLM локально на GPU - 2026",
section "Формат модели .zse": signature ZSE\\x01, version 1, a 64-byte header,
a CRC32 and 32-byte section entries; weights page-aligned, tensors aligned to
256 bytes.
"""
import json
import struct
import zlib

import numpy as np

MAGIC = b"ZSE\x01"
VERSION = 1
CONFIG, TOKENIZER, WEIGHT_INDEX, WEIGHT_DATA, KERNELS = 1, 2, 3, 4, 5
HAS_TOKENIZER, HAS_KERNELS, MMAP_READY = 1, 2, 4
PAGE = 4096
TENSOR_ALIGN = 256
GROUP = 128


# Tensors that stay fp16 ([wiki] "Формат модели .zse": embeddings, layer
# norms and every bias are kept unquantized, through an exclusion list of name
# patterns).  Matched against Hugging Face-style tensor names.
NO_QUANTIZE_PATTERNS = (
    r"(^|\.)embed",        # token / position embeddings
    r"norm(\.|_|$)",       # layernorm, rmsnorm, input_layernorm, ...
    r"(^|\.)ln_?\w*\.",   # GPT-style ln_1., ln_f.
    r"\.bias$",            # every bias
)


def keep_fp16(name, shape=None):
    """True if the tensor `name` stays fp16: it matches NO_QUANTIZE_PATTERNS,
    or it cannot be stored in the quantized format (not 2-D, or the number of
    columns is not a multiple of the group of 128)."""
    import re
    if any(re.search(p, name) for p in NO_QUANTIZE_PATTERNS):
        return True
    if shape is not None and (len(shape) != 2 or shape[1] % GROUP != 0):
        return True
    return False


def _bytes(a):
    """A flat read-only byte view of a numpy array, torch CPU tensor or bytes."""
    if isinstance(a, (bytes, bytearray, memoryview)):
        return memoryview(a).cast("B")
    if hasattr(a, "numpy"):  # torch tensor
        a = a.detach().cpu().numpy()
    return memoryview(np.ascontiguousarray(a)).cast("B")


def _align(x, a):
    return (x + a - 1) // a * a


def write_zse(path, tensors, config=None, tokenizer=None, kernels=None):
    """Writes a .zse file.

    tensors: list of dicts, each either
      quantized: {"name", "bits", "rows", "cols", "packed", "scales", "zeros"}
                 (packed: uint32 rows x cols*bits/32; scales, zeros: fp16 bit
                 patterns rows x cols/128), or
      fp16:      {"name", "rows", "cols", "data"} (fp16 rows x cols).
    Returns the layout: {"weight_offset", "weight_bytes", "tensors": [entry dicts]}.
    """
    entries, arrays, woff = [], [], 0

    def place(buf):
        nonlocal woff
        off = _align(woff, TENSOR_ALIGN)
        arrays.append((off, buf))
        woff = off + len(buf)
        return off

    layout = []
    for t in tensors:
        name = t["name"].encode()
        if not 0 < len(name) < 64:
            raise ValueError(f"tensor name {t['name']!r} must be 1..63 bytes")
        rows, cols = int(t["rows"]), int(t["cols"])
        if "packed" in t:
            bits = int(t["bits"])
            if bits not in (2, 3, 4, 8) or cols % GROUP:
                raise ValueError(f"{t['name']}: bits {bits}, cols {cols}")
            data = _bytes(t["packed"])
            sz = rows * (cols // GROUP) * 2
            if len(data) != rows * cols * bits // 8:
                raise ValueError(f"{t['name']}: packed size {len(data)}")
            s, z = _bytes(t["scales"]), _bytes(t["zeros"])
            if len(s) != sz or len(z) != sz:
                raise ValueError(f"{t['name']}: scales/zeros size")
            e = (1, bits, GROUP, place(data), len(data), place(s), place(z))
        else:
            data = _bytes(t["data"])
            if len(data) != rows * cols * 2:
                raise ValueError(f"{t['name']}: fp16 size {len(data)}")
            e = (0, 16, 0, place(data), len(data), 0, 0)
        kind, bits, group, d_off, d_len, s_off, z_off = e
        entries.append(name.ljust(64, b"\0") + struct.pack("<IIIIQQQQQQ", kind, bits, group, 0, rows, cols,
                                                           d_off, d_len, s_off, z_off))
        layout.append({"name": t["name"], "kind": kind, "bits": bits, "group": group, "rows": rows,
                       "cols": cols, "data_offset": d_off, "data_bytes": d_len, "scales_offset": s_off,
                       "zeros_offset": z_off})
    wsize = _align(woff, TENSOR_ALIGN)

    blobs = {CONFIG: json.dumps(config or {}, sort_keys=True).encode(),
             WEIGHT_INDEX: struct.pack("<II", len(entries), 128) + b"".join(entries)}
    if tokenizer is not None:
        blobs[TOKENIZER] = bytes(tokenizer)
    if kernels is not None:
        blobs[KERNELS] = bytes(kernels)
    n_sec = len(blobs) + 1
    table_end = 68 + 32 * n_sec
    off, place_at = _align(table_end, 64), {}
    for typ in sorted(blobs):
        place_at[typ] = off
        off = _align(off + len(blobs[typ]), 64)
    w_at = _align(off, PAGE)
    file_size = w_at + wsize
    flags = MMAP_READY | (HAS_TOKENIZER if tokenizer is not None else 0) | (HAS_KERNELS if kernels is not None else 0)

    crcs = {}
    with open(path, "wb") as f:
        f.write(b"\0" * table_end)
        for typ in sorted(blobs):
            f.seek(place_at[typ])
            f.write(blobs[typ])
            crcs[typ] = zlib.crc32(blobs[typ])
        f.seek(w_at)
        crc, pos = 0, 0
        for a_off, buf in arrays:
            pad = b"\0" * (a_off - pos)
            f.write(pad)
            crc = zlib.crc32(pad, crc)
            for i in range(0, len(buf), 1 << 26):
                piece = buf[i:i + (1 << 26)]
                f.write(piece)
                crc = zlib.crc32(piece, crc)
            pos = a_off + len(buf)
        pad = b"\0" * (wsize - pos)
        f.write(pad)
        crcs[WEIGHT_DATA] = zlib.crc32(pad, crc)
        where = dict(place_at)
        where[WEIGHT_DATA] = w_at
        sizes = {typ: len(b) for typ, b in blobs.items()}
        sizes[WEIGHT_DATA] = wsize
        table = b"".join(struct.pack("<IIQQQ", typ, crcs[typ], where[typ], sizes[typ], 0) for typ in sorted(where))
        header = MAGIC + struct.pack("<IIIQ", VERSION, flags, n_sec, file_size) + b"\0" * 40
        f.seek(0)
        f.write(header + struct.pack("<I", zlib.crc32(header + table)) + table)
    return {"weight_offset": w_at, "weight_bytes": wsize, "tensors": layout}
