"""GPU: the native loader streams a .zse file's weights into one device
allocation bit-exactly (checked against the oracle reader), and the linear
layer run on the loaded tensors matches the fp64 oracle."""
import time

import numpy as np
import pytest
import torch

import zq_inputs as zi
from oracle import zse_oracle as zo
from zq_testutil import assert_linear_close, u16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def zq():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import weight_only_quantized_zq_b200 as m
    return m


def test_load_weights_bit_exact_then_linear(tmp_path, zq, orc):
    from weight_only_quantized_zq_b200.zse import write_zse
    specs = [("q", 4, 512, 1024), ("o", 3, 256, 512), ("up", 2, 384, 256), ("down", 8, 128, 384)]
    tensors = []
    for i, (name, bits, N, K) in enumerate(specs):
        w = zi.weight(N, K, seed=900 + i, device="cuda")
        p, s, z = zq.quantize(w, bits)
        tensors.append({"name": name, "bits": bits, "rows": N, "cols": K, "packed": p.cpu(), "scales": s.cpu(),
                        "zeros": z.cpu()})
    emb = torch.randn(100, 64).half()
    tensors.append({"name": "embed", "rows": 100, "cols": 64, "data": emb})
    path = tmp_path / "model.zse"
    write_zse(path, tensors, config={"layers": 1})
    parsed = zo.read(path)

    with zq.ZseFile(path) as f:
        f.verify()
        dev = torch.empty(f.weight_bytes, dtype=torch.uint8, device="cuda")
        f.load_weights(dev)
        infos = {t["name"]: t for t in f.tensors()}
    # bit-exact against the oracle's view of the file
    assert np.array_equal(dev.cpu().numpy(), np.frombuffer(parsed["payload"]["WEIGHT_DATA"], np.uint8))

    x = {K: zi.activations(3, K, seed=950 + K, device="cuda") for (_, _, _, K) in specs}
    ops, outs = [], []
    for (name, bits, N, K) in specs:
        t = infos[name]
        view = lambda off, n, dt: dev[off:off + n].view(dt)
        packed = view(t["data_offset"], t["data_bytes"], torch.int32)
        G = K // 128
        scales = view(t["scales_offset"], N * G * 2, torch.int16)
        zeros = view(t["zeros_offset"], N * G * 2, torch.int16)
        out = torch.empty(3, N, dtype=torch.float16, device="cuda")
        ops.append((x[K], packed, scales, zeros, out, bits, 128, 3, N, K))
        outs.append((name, bits, N, K, out))
    zq.linear_stack(ops)
    torch.cuda.synchronize()
    for (name, bits, N, K, out) in outs:
        data, s, z = zo.tensor_arrays(parsed, name)
        p_ref = np.frombuffer(data, np.uint32).reshape(N, -1)
        s_ref = np.frombuffer(s, np.uint16).reshape(N, -1)
        z_ref = np.frombuffer(z, np.uint16).reshape(N, -1)
        y_ref, bound = orc.linear(u16(x[K]), p_ref, s_ref, z_ref, bits, N, K)
        assert_linear_close(out, y_ref, bound, f"loaded {name}")
    e = infos["embed"]
    assert torch.equal(dev[e["data_offset"]:e["data_offset"] + e["data_bytes"]].view(torch.float16).cpu().view(100, 64),
                       emb)


def test_load_weights_in_chunks(tmp_path, zq):
    """A weight section larger than two 64 MB staging chunks (ragged tail)."""
    from weight_only_quantized_zq_b200.zse import write_zse
    rng = np.random.default_rng(3)
    N, K = 8192, 17920  # 4 bits: 73.4 MB of codes + 2.3 MB of scales and zeros
    t = {"name": "big", "bits": 4, "rows": N, "cols": K,
         "packed": rng.integers(0, 2**32, N * K // 8, dtype=np.uint32),
         "scales": rng.integers(0, 2**16, (N, K // 128), dtype=np.uint16),
         "zeros": rng.integers(0, 2**16, (N, K // 128), dtype=np.uint16)}
    t2 = dict(t, name="big2")
    path = tmp_path / "big.zse"
    write_zse(path, [t, t2])
    parsed = zo.read(path)
    with zq.ZseFile(path) as f:
        wb = f.weight_bytes
        dev = torch.empty(wb, dtype=torch.uint8, device="cuda")
        assert wb > 2 * (64 << 20)
        times = []
        for _ in range(2):  # the first call also allocates the pinned staging buffers
            dev.zero_()
            torch.cuda.synchronize()
            t0 = time.perf_counter()
            f.load_weights(dev)
            times.append(time.perf_counter() - t0)
            assert np.array_equal(dev.cpu().numpy(), np.frombuffer(parsed["payload"]["WEIGHT_DATA"], np.uint8))
    print(f"zse load: first {wb / times[0] / 1e9:.2f} GB/s, again {wb / times[1] / 1e9:.2f} GB/s "
          f"({wb / 1e6:.0f} MB)")
