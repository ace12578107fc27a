"""The .zse container on the CPU: the oracle reader pinned to the pages'
layout and the CRC-32 definition, the package's writer checked against the
oracle, and the library's native reader checked against both (opening and
validating a file needs no GPU)."""
import struct
import zlib

import numpy as np
import pytest

from oracle import zse_oracle as zo


@pytest.fixture(scope="module")
def zq():
    import importlib.util
    import os
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    spec = importlib.util.spec_from_file_location("zq_build", os.path.join(root, "weight_only_quantized_zq_b200",
                                                                           "build.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    mod.build()
    import weight_only_quantized_zq_b200 as m
    return m


def _tensors(seed=0):
    rng = np.random.default_rng(seed)
    out = []
    for i, (bits, rows, cols) in enumerate([(4, 64, 256), (3, 40, 384), (2, 17, 128), (8, 9, 512)]):
        out.append({"name": f"layers.{i}.w", "bits": bits, "rows": rows, "cols": cols,
                    "packed": rng.integers(0, 2**32, rows * cols * bits // 32, dtype=np.uint32),
                    "scales": rng.integers(0, 2**16, (rows, cols // 128), dtype=np.uint16),
                    "zeros": rng.integers(0, 2**16, (rows, cols // 128), dtype=np.uint16)})
    out.append({"name": "embed", "rows": 33, "cols": 24,
                "data": rng.standard_normal((33, 24)).astype(np.float16)})
    return out


# ------------------------------------------------------------ oracle pins --

def test_crc32_is_the_ieee_definition():
    # the standard check value of CRC-32 (IEEE 802.3, reflected, xor-out)
    assert zlib.crc32(b"123456789") == 0xCBF43926


def _hand_built():
    """A file assembled field by field from the documented layout: one fp16
    tensor 1 x 8 and a config, no tokenizer or kernels."""
    cfg = b'{"a": 1}'
    values = np.arange(8, dtype=np.float16)
    entry = b"t0".ljust(64, b"\0") + struct.pack("<IIIIQQQQQQ", 0, 16, 0, 0, 1, 8, 0, 16, 0, 0)
    index = struct.pack("<II", 1, 128) + entry
    cfg_off, idx_off, w_off = 192, 256, 4096
    w = values.tobytes() + b"\0" * 240  # 256 bytes of weight data
    size = w_off + len(w)
    table = b"".join([struct.pack("<IIQQQ", 1, zlib.crc32(cfg), cfg_off, len(cfg), 0),
                      struct.pack("<IIQQQ", 3, zlib.crc32(index), idx_off, len(index), 0),
                      struct.pack("<IIQQQ", 4, zlib.crc32(w), w_off, len(w), 0)])
    header = b"ZSE\x01" + struct.pack("<IIIQ", 1, 4, 3, size) + b"\0" * 40
    buf = bytearray(size)
    buf[0:64] = header
    buf[64:68] = struct.pack("<I", zlib.crc32(header + table))
    buf[68:68 + len(table)] = table
    buf[cfg_off:cfg_off + len(cfg)] = cfg
    buf[idx_off:idx_off + len(index)] = index
    buf[w_off:] = w
    return bytes(buf), values


def test_oracle_reads_hand_built_file():
    buf, values = _hand_built()
    p = zo.read(buf)
    assert (p["version"], p["flags"], p["n_sections"], p["file_size"]) == (1, 4, 3, len(buf))
    assert set(p["sections"]) == {"CONFIG", "WEIGHT_INDEX", "WEIGHT_DATA"}
    for off, size, stored, computed in p["sections"].values():
        assert stored == computed
    assert p["sections"]["WEIGHT_DATA"][0] == 4096
    assert p["payload"]["CONFIG"] == b'{"a": 1}'
    (t,) = p["tensors"]
    assert (t["name"], t["kind"], t["bits"], t["rows"], t["cols"], t["data_bytes"]) == ("t0", 0, 16, 1, 8, 16)
    data, s, z = zo.tensor_arrays(p, "t0")
    assert np.array_equal(np.frombuffer(data, np.float16), values) and s is None


def test_oracle_rejects_a_flipped_header_byte():
    buf, _ = _hand_built()
    bad = bytearray(buf)
    bad[12] ^= 1  # section count
    with pytest.raises(zo.ZseError):
        zo.read(bytes(bad))


# ------------------------------------------------------------------ writer --

def test_writer_layout_matches_the_oracle(tmp_path, zq):
    from weight_only_quantized_zq_b200.zse import write_zse
    ts = _tensors()
    path = tmp_path / "m.zse"
    lay = write_zse(path, ts, config={"hidden": 3584}, tokenizer=b"tok", kernels=b"\x00\x01")
    p = zo.read(path)
    assert p["flags"] == 1 | 2 | 4
    for name, (off, size, stored, computed) in p["sections"].items():
        assert stored == computed, name
    w_off = p["sections"]["WEIGHT_DATA"][0]
    assert w_off % 4096 == 0 and w_off == lay["weight_offset"]
    assert p["payload"]["TOKENIZER"] == b"tok" and p["payload"]["KERNELS"] == b"\x00\x01"
    assert p["payload"]["CONFIG"] == b'{"hidden": 3584}'
    for t, e in zip(ts, p["tensors"]):
        assert e["name"] == t["name"]
        for k in ("data_offset", "scales_offset", "zeros_offset"):
            assert e[k] % 256 == 0
        data, s, z = zo.tensor_arrays(p, t["name"])
        if "packed" in t:
            assert data == t["packed"].tobytes() and s == t["scales"].tobytes() and z == t["zeros"].tobytes()
        else:
            assert data == t["data"].tobytes()


# ----------------------------------------------------------- native reader --

def test_native_reader_matches_the_oracle(tmp_path, zq):
    from weight_only_quantized_zq_b200.zse import write_zse
    path = tmp_path / "m.zse"
    write_zse(path, _tensors(1), config={"k": [1, 2]}, tokenizer=b"abc")
    p = zo.read(path)
    with zq.ZseFile(path) as f:
        f.verify()
        assert f.flags == p["flags"]
        assert f.tensors() == p["tensors"]
        assert f.weight_bytes == p["sections"]["WEIGHT_DATA"][1]
        assert f.section(zq.ZSE_CONFIG) == p["payload"]["CONFIG"]
        assert f.section(zq.ZSE_TOKENIZER) == b"abc"
        assert f.section(zq.ZSE_KERNELS) is None
        assert f.find("embed") == len(p["tensors"]) - 1 and f.find("nope") == -1


def test_native_reader_opens_the_hand_built_file(tmp_path, zq):
    buf, _ = _hand_built()
    path = tmp_path / "h.zse"
    path.write_bytes(buf)
    with zq.ZseFile(path) as f:
        f.verify()
        (t,) = f.tensors()
        assert (t["name"], t["rows"], t["cols"]) == ("t0", 1, 8)


def _rewrite_header(buf):
    """Recomputes the header CRC after a deliberate edit."""
    n = struct.unpack_from("<I", buf, 12)[0]
    buf[64:68] = struct.pack("<I", zlib.crc32(bytes(buf[0:64]) + bytes(buf[68:68 + 32 * n])))


@pytest.mark.parametrize("edit,status", [
    ("magic", 1), ("crc", 1), ("version", 2), ("truncate", 1), ("size_field", 1),
    ("section_oob", 1), ("dup_section", 1), ("weights_unaligned", 1), ("bad_bits", 1),
])
def test_native_reader_rejects(tmp_path, zq, edit, status):
    buf = bytearray(_hand_built()[0])
    if edit == "magic":
        buf[0] = ord("X")
    elif edit == "crc":
        buf[64] ^= 0xFF
    elif edit == "version":
        buf[4] = 2
        _rewrite_header(buf)
    elif edit == "truncate":
        buf = buf[:-1]
    elif edit == "size_field":
        buf[16] ^= 1
        _rewrite_header(buf)
    elif edit == "section_oob":
        struct.pack_into("<Q", buf, 68 + 32 * 2 + 16, 10**9)  # WEIGHT_DATA size
        _rewrite_header(buf)
    elif edit == "dup_section":
        struct.pack_into("<I", buf, 68 + 32, 1)  # WEIGHT_INDEX entry relabelled CONFIG
        _rewrite_header(buf)
    elif edit == "weights_unaligned":
        # move WEIGHT_DATA one byte later (MMAP_READY is set)
        struct.pack_into("<Q", buf, 68 + 32 * 2 + 8, 4097)
        struct.pack_into("<Q", buf, 68 + 32 * 2 + 16, 255)
        _rewrite_header(buf)
    elif edit == "bad_bits":
        struct.pack_into("<I", buf, 256 + 8 + 68, 5)  # fp16 entry with bits 5
        _rewrite_header(buf)
    path = tmp_path / "bad.zse"
    path.write_bytes(bytes(buf))
    with pytest.raises(zq.ZQError) as e:
        zq.ZseFile(path)
    assert e.value.status == status
    assert zq.zq_last_error() != ""


def test_native_verify_finds_a_flipped_weight_byte(tmp_path, zq):
    buf = bytearray(_hand_built()[0])
    buf[4096 + 3] ^= 0x10  # inside WEIGHT_DATA: the header stays valid
    path = tmp_path / "w.zse"
    path.write_bytes(bytes(buf))
    with zq.ZseFile(path) as f:
        with pytest.raises(zq.ZQError) as e:
            f.verify()
        assert "CRC" in str(e.value)


def test_native_load_rejects_null_destination(tmp_path, zq):
    path = tmp_path / "h.zse"
    path.write_bytes(_hand_built()[0])
    with zq.ZseFile(path) as f:
        assert zq._lib.zq_zse_load_weights(f._h, None, 1 << 20, None) == zq.ZQ_ERR_INVALID_ARG
        assert zq._lib.zq_zse_load_weights(f._h, 256, 16, None) == zq.ZQ_ERR_INVALID_ARG  # too small
    assert zq._lib.zq_zse_open(b"/nonexistent/x.zse", __import__("ctypes").byref(zq._P())) == zq.ZQ_ERR_INVALID_ARG


def test_no_quantize_patterns():
    """Embeddings, layer norms and every bias stay fp16; projections are
    quantized; tensors the format cannot hold (1-D, K not a multiple of 128)
    stay fp16 too."""
    from weight_only_quantized_zq_b200.zse import keep_fp16
    stay = ["model.embed_tokens.weight", "model.layers.0.input_layernorm.weight",
            "model.layers.3.post_attention_layernorm.weight", "model.norm.weight",
            "model.layers.0.self_attn.q_proj.bias", "transformer.h.0.ln_1.weight", "transformer.ln_f.weight",
            "model.decoder.embed_positions.weight"]
    quantize = ["model.layers.0.self_attn.q_proj.weight", "model.layers.0.mlp.gate_proj.weight",
                "model.layers.27.mlp.down_proj.weight", "lm_head.weight"]
    assert all(keep_fp16(n) for n in stay)
    assert not any(keep_fp16(n, (4096, 4096)) for n in quantize)
    assert keep_fp16("model.layers.0.mlp.down_proj.weight", (4096, 1000))
    assert keep_fp16("some.vector", (4096,))


def test_views_into_the_weight_section(tmp_path, zq):
    """ZseFile.views slices a buffer holding WEIGHT_DATA into every tensor's
    arrays (here a host copy of the section; on the GPU the buffer that
    load_weights filled), equal to what was written."""
    import torch
    from weight_only_quantized_zq_b200.zse import write_zse
    path = tmp_path / "v.zse"
    tensors = _tensors(5)
    write_zse(path, tensors)
    with zq.ZseFile(path) as f:
        data = f.section(zq.ZSE_WEIGHT_DATA)
        buf = torch.frombuffer(bytearray(data), dtype=torch.uint8)
        views = f.views(buf)
        with pytest.raises(zq.ZQError):
            f.views(buf[:-1])
    for t in tensors:
        v = views[t["name"]]
        if "data" in t:
            assert np.array_equal(v["data"].numpy(), t["data"])
        else:
            assert v["packed"].shape == (t["rows"], t["cols"] * t["bits"] // 32)
            assert np.array_equal(v["packed"].numpy().view(np.uint32).reshape(-1), t["packed"])
            assert np.array_equal(v["scales"].numpy().view(np.uint16), t["scales"])
            assert np.array_equal(v["zeros"].numpy().view(np.uint16), t["zeros"])
