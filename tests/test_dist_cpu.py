"""Multi-process host logic of the replica bench, on CPU with gloo.

The path has no exchange step ("replicas only"): ranks share nothing but the
barrier and the max-over-ranks of their device times.  These tests run that
plumbing with world_size 2 on the CPU.
"""
import io
import contextlib
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _replica(rank, world, port, out_dir):
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port), "WORLD_SIZE": str(world),
                       "RANK": str(rank), "LOCAL_RANK": str(rank)})
    sys.path.insert(0, ROOT)
    import torch
    import bench
    w, r, _ = bench.dist_init("gloo")
    assert (w, r) == (world, rank)
    bench.barrier(w)
    # each rank's "device time" differs; every rank must see the maximum
    got = bench.max_over_ranks(10.0 * rank + 1.5, w)
    bench.barrier(w)
    torch.distributed.destroy_process_group()
    with open(os.path.join(out_dir, f"rank{rank}.txt"), "w") as f:
        f.write(repr(got))


def test_max_over_ranks_gloo_world2(tmp_path):
    world = 2
    mp.start_processes(_replica, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    vals = [float(open(tmp_path / f"rank{r}.txt").read()) for r in range(world)]
    assert vals == [11.5, 11.5]


def test_single_rank_needs_no_process_group(monkeypatch):
    for k in ("WORLD_SIZE", "RANK", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    sys.path.insert(0, ROOT)
    import bench
    assert bench.dist_env() == (1, 0, 0)
    assert bench.max_over_ranks(3.25, 1) == 3.25
    bench.barrier(1)  # no-op without a process group


def test_reference_arm_non_zero_rank_exits_without_work(monkeypatch):
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("LOCAL_RANK", "1")
    sys.path.insert(0, ROOT)
    import bench
    called = []
    monkeypatch.setattr(bench, "oracle_layer_sample", lambda *a, **k: called.append(1))
    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        rc = bench.main(["--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "0"])
    assert rc == 0
    assert buf.getvalue() == ""
    assert called == []


def test_traffic_key_ignores_comments_only():
    """The bench keys a captured DRAM traffic figure by a hash of the kernel's
    code: comments and whitespace do not change it, code does, and string
    literals that look like comments are code."""
    import bench
    src = 'int a = 1; // note\n/* block\n comment */ const char *s = "x//y /* z */";\nchar q = \'\\\'\';\n'
    assert bench.strip_comments(src).split() == ["int", "a", "=", "1;", "const", "char", "*s", "=",
                                                 '"x//y', "/*", 'z', '*/";', "char", "q", "=", "'\\'';"]
    assert bench.strip_comments("a /* unterminated") == "a  "
    assert bench.strip_comments("b // to the end") == "b  "
    h = bench.kernel_sha256("decode")
    assert len(h) == 64 and h == bench.kernel_sha256("decode")


def test_algorithmic_bytes_and_flops_of_the_workloads():
    """The bench's accounting (codes + fp16 scales/zeros + x + out per op;
    2*M*N*K flops) against the per-config totals worked out from that formula
    for the 7B- and 32B-shaped layers."""
    import bench
    one = bench.workload_config(1, 1, 1)
    assert one["bytes_per_step"] == 123_964_416                    # one 7B layer, M = 1
    for M, gb in ((1, 3.471), (4, 3.484), (16, 3.538), (64, 3.751)):  # 28 layers
        assert round(bench.workload_config(M, 28, 1)["bytes_per_step"] / 1e9, 3) == gb
    assert bench.workload_config(1, 1, 1, "32b-mixed")["bytes_per_step"] == 206_833_664
    pre = bench.workload_config(2048, 28, 1)
    assert round(pre["bytes_per_step"] / 1e9, 2) == 12.57
    assert round(pre["flops_per_step"] / 1e12, 2) == 26.73
    assert round(bench.workload_config(1, 1, 1)["flops_per_step"] / 1e6) == 466  # MFLOP per 7B layer


def test_clock_sampler_decodes_reasons_with_a_fake_nvml():
    """The clocks key of the bench line: median SM clock under load and the
    throttle reasons seen, from NVML's clock-event mask (a fake NVML here;
    nothing is set on any device)."""
    import threading
    import bench

    class FakeNvml:
        NVML_CLOCK_SM = 1

        def __init__(self):
            self.clocks = iter([1965, 1950, 1582, 1965, 1300])
            self.masks = iter([0x0, 0x4, 0x4, 0x0, 0x4 | 0x40])

        def nvmlDeviceGetClockInfo(self, handle, kind):
            assert handle == "h0" and kind == self.NVML_CLOCK_SM
            return next(self.clocks)

        def nvmlDeviceGetCurrentClocksEventReasons(self, handle):
            return next(self.masks)

    s = bench.ClockSampler.__new__(bench.ClockSampler)
    s.samples, s.reasons, s.max_mhz, s.period = [], set(), 1965, 0.0
    s._stop, s._thread, s._nvml, s._h = threading.Event(), None, FakeNvml(), "h0"
    for _ in range(5):
        s.sample()
    out = s.summary()
    assert out["sm_mhz"] == 1950 and out["sm_max_mhz"] == 1965
    assert out["reasons"] == ["hw_thermal_slowdown", "sw_power_cap"]
    s.sample()  # an NVML error (exhausted fake) is ignored, not raised
    assert len(s.samples) == 5


def test_oracle_small_layer_on_one_core():
    """The bench's one-core oracle figure for the M=1, N=K=512 INT4 layer runs
    on the CPU and leaves the oracle's thread count as it found it."""
    import bench
    import oracle as orc
    before = orc.get_threads()
    r = bench.oracle_config1_one_core(budget_s=0.05)
    assert r["cores"] == 1 and r["us_per_call"] > 0 and r["value"] > 0
    assert orc.get_threads() == before
