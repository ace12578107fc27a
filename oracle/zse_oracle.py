"""Oracle for the .zse container: a plain reader of the byte layout.

Test infrastructure only: tests/ and __graft_entry__.smoke() use it; the
library never does.  It shares no code with the library's native reader
(weight_only_quantized_zq_b200/csrc/zq_zse.cu) or with the package's writer.

It follows the layout stated in include/zq_zse.h, which reads the pages'
description ([wiki] "ZSE - open-source движок для запуска LLM локально на
GPU - 2026", section "Формат модели .zse": signature ZSE\\x01, version 1,
64-byte header + CRC32 + 32-byte section entries, sections CONFIG,
TOKENIZER, WEIGHT_INDEX, WEIGHT_DATA, KERNELS, weights page-aligned, tensors
256-byte aligned, flags HAS_TOKENIZER / HAS_KERNELS / MMAP_READY).  The
CRC-32 is zlib's (the IEEE 802.3 definition), a library primitive.
"""
import struct
import zlib

SECTION_NAMES = {1: "CONFIG", 2: "TOKENIZER", 3: "WEIGHT_INDEX", 4: "WEIGHT_DATA", 5: "KERNELS"}


class ZseError(ValueError):
    pass


def read(path_or_bytes):
    """Parses a whole .zse file.  Returns a dict with the header fields, the
    sections {name: (offset, size, crc_stored, crc_computed)}, the tensor
    entries and the section payloads (bytes)."""
    if isinstance(path_or_bytes, (bytes, bytearray)):
        buf = bytes(path_or_bytes)
    else:
        with open(path_or_bytes, "rb") as f:
            buf = f.read()
    if len(buf) < 68:
        raise ZseError("shorter than the header")
    magic = buf[0:4]
    version, flags, n_sec, file_size = struct.unpack_from("<IIIQ", buf, 4)
    if magic != b"ZSE\x01":
        raise ZseError("bad magic")
    if file_size != len(buf):
        raise ZseError("file size field")
    table = buf[68:68 + 32 * n_sec]
    if len(table) != 32 * n_sec:
        raise ZseError("short section table")
    header_crc = struct.unpack_from("<I", buf, 64)[0]
    if zlib.crc32(buf[0:64] + table) != header_crc:
        raise ZseError("header CRC")
    sections, payload = {}, {}
    for i in range(n_sec):
        typ, crc, off, size, reserved = struct.unpack_from("<IIQQQ", table, 32 * i)
        name = SECTION_NAMES[typ]
        data = buf[off:off + size]
        if len(data) != size:
            raise ZseError(f"section {name} outside the file")
        sections[name] = (off, size, crc, zlib.crc32(data))
        payload[name] = data
    tensors = []
    if "WEIGHT_INDEX" in payload:
        idx = payload["WEIGHT_INDEX"]
        count, esize = struct.unpack_from("<II", idx, 0)
        for i in range(count):
            e = idx[8 + esize * i: 8 + esize * (i + 1)]
            name = e[:64].split(b"\0", 1)[0].decode()
            kind, bits, group, _, rows, cols, d_off, d_len, s_off, z_off = struct.unpack_from("<IIIIQQQQQQ", e, 64)
            tensors.append({"name": name, "kind": kind, "bits": bits, "group": group, "rows": rows, "cols": cols,
                            "data_offset": d_off, "data_bytes": d_len, "scales_offset": s_off,
                            "zeros_offset": z_off})
    return {"version": version, "flags": flags, "n_sections": n_sec, "file_size": file_size,
            "header_crc": header_crc, "sections": sections, "tensors": tensors, "payload": payload}


def tensor_arrays(parsed, name):
    """(data, scales, zeros) bytes of a tensor (scales/zeros None for fp16)."""
    t = next(t for t in parsed["tensors"] if t["name"] == name)
    w = parsed["payload"]["WEIGHT_DATA"]
    data = w[t["data_offset"]:t["data_offset"] + t["data_bytes"]]
    if t["kind"] == 0:
        return data, None, None
    sz = t["rows"] * (t["cols"] // t["group"]) * 2
    return data, w[t["scales_offset"]:t["scales_offset"] + sz], w[t["zeros_offset"]:t["zeros_offset"] + sz]
