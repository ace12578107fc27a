#!/usr/bin/env python
"""Benchmark of the weight-only quantized linear on B200.

Default workload (one step): the 28-layer, Qwen2.5-7B-shaped decode stack at
M = 1 token, INT4 g128: per layer qkv 4608x3584, o 3584x3584, gate_up
37888x3584, down 3584x18944 (112 projections, 3.47 GB of packed weights,
larger than L2, so no flush is needed), run through one zq_linear_stack call.
Weights are synthetic (N(0, 0.02), seeded per tensor) and quantized on the GPU
by zq_quantize_pack; activations N(0, 1) rounded to fp16.

Metric: algorithmic HBM bytes per step (packed codes + fp16 scales/zeros + x +
out) / device time, in GB/s; also % of 8 TB/s and tokens/s-equivalent
(linear layers only: attention, norms, embeddings and lm_head excluded).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl zq|reference]
                    [--m M] [--layers L]

M <= 64 is decode (bandwidth-bound, reported against HBM; the library runs
M <= 32 on its mma.sync decode kernel and larger M on its tcgen05 tile
kernel); M > 64 is prefill (reported against the tensor peak).

--impl reference times the fp64 CPU oracle on a bounded sample of the same
workload on the host cores (rank 0 only).  With N > 1 (torchrun), each rank
runs an independent replica on its own GPU (the path has no exchange step);
value is the total over ranks / the max over ranks of the device time.
"""
import argparse
import json
import os
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import zq_inputs as zi  # noqa: E402

METRIC = "quantized-linear HBM GB/s (% of 8 TB/s) at M=1; tokens/s-equiv per layer stack"

# DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum) of the dominant
# kernel, per layer of the stack, from one ncu capture of a 4-layer stack
# (traffic grows in proportion to the layers).  Keyed by the SHA-256 of the
# kernel's code (sources without comments) at capture time: once the code
# changes the figure is stale and the roofline reports null.
CSRC = os.path.join(ROOT, "weight_only_quantized_zq_b200", "csrc")
KERNEL_SOURCES = {
    "decode": ("zq_decode.cu", "zq_device.cuh", "zq_internal.h"),
    "prefill": ("zq_prefill.cu", "zq_device.cuh", "zq_internal.h"),
}
MEASURED_TRAFFIC = {
    # (family, model, M): DRAM bytes per layer of the stack
    ("decode", "7b", 1): {  # an 8-layer launch
        "sha256": "f9572bb584c305814c8dd153e79fca8d3eed0579afc9566ea8ef798bd67b14d9",
        "bytes_per_layer": 125239776,
    },
    ("decode", "7b", 32): {  # a 4-layer launch, four token tiles
        "sha256": "f9572bb584c305814c8dd153e79fca8d3eed0579afc9566ea8ef798bd67b14d9",
        "bytes_per_layer": 128267904,
    },
    # tile kernel, one-token-half plan: a one-layer launch at M = 64
    ("prefill", "7b", 64): {
        "sha256": "731fe9bb6c01b2a07244b2d29eaddf0d9e5d87b9272e0f4f7365a2578ca25d5b",
        "bytes_per_layer": 130703104,
    },
    # tile kernel, CTA-pair plan: a one-layer launch at M = 2048
    ("prefill", "7b", 2048): {
        "sha256": "731fe9bb6c01b2a07244b2d29eaddf0d9e5d87b9272e0f4f7365a2578ca25d5b",
        "bytes_per_layer": 381221120,
    },
}
NOMINAL_HBM_GBS = 8000.0
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}


# --------------------------------------------------------------- plumbing --

def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def dist_init(backend):
    world, rank, local = dist_env()
    if world > 1:
        import datetime
        torch.distributed.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))
    return world, rank, local


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def max_over_ranks(value, world, device="cpu"):
    if world == 1:
        return value
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    return dict(FALLBACK_PEAKS, bf16_tflops_sustained=1400.0, source="fallback")


class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while running."""

    REASONS = {"hw_slowdown": 0x8, "hw_thermal_slowdown": 0x40, "sw_thermal_slowdown": 0x20,
               "sw_power_cap": 0x4, "hw_power_brake_slowdown": 0x80}

    def __init__(self, device_index, period_s=0.001):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self.period = period_s
        self._stop = threading.Event()
        self._thread = None
        try:
            import pynvml
            pynvml.nvmlInit()
            uuid = torch.cuda.get_device_properties(device_index).uuid
            handle = None
            for i in range(pynvml.nvmlDeviceGetCount()):
                h = pynvml.nvmlDeviceGetHandleByIndex(i)
                u = pynvml.nvmlDeviceGetUUID(h)
                u = u.decode() if isinstance(u, bytes) else u
                if u.replace("GPU-", "") == str(uuid).replace("GPU-", ""):
                    handle = h
            self._nvml, self._h = pynvml, handle
            if handle is not None:
                self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(handle, pynvml.NVML_CLOCK_SM)
        except Exception:
            self._nvml, self._h = None, None

    def _run(self):
        while not self._stop.is_set():
            self.sample()
            time.sleep(self.period)

    def sample(self):
        if self._h is None:
            return
        p = self._nvml
        try:
            self.samples.append(p.nvmlDeviceGetClockInfo(self._h, p.NVML_CLOCK_SM))
            mask = p.nvmlDeviceGetCurrentClocksEventReasons(self._h)
            for name, bit in self.REASONS.items():
                if mask & bit:
                    self.reasons.add(name)
        except Exception:
            pass

    def __enter__(self):
        if self._h is not None:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._thread is not None:
            self._thread.join()
        self.sample()  # one more right at the end of the region

    def summary(self):
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                "samples": len(self.samples), "source": "nvml"}


def strip_comments(src):
    """C/C++/CUDA source without its comments, each comment replaced by one
    space, string and character literals kept as they are."""
    out, i, n = [], 0, len(src)
    while i < n:
        c = src[i]
        if c in "\"'":
            j = i + 1
            while j < n and src[j] != c:
                j += 2 if src[j] == "\\" else 1
            out.append(src[i:j + 1])
            i = j + 1
        elif src.startswith("//", i):
            j = src.find("\n", i)
            i = n if j < 0 else j
            out.append(" ")
        elif src.startswith("/*", i):
            j = src.find("*/", i + 2)
            i = n if j < 0 else j + 2
            out.append(" ")
        else:
            out.append(c)
            i += 1
    return "".join(out)


def kernel_sha256(family):
    """SHA-256 of the kernel family's code: its sources with comments removed
    and whitespace runs collapsed, so that a comment edit keeps a capture's
    traffic valid and any change to the code does not."""
    import hashlib
    import re
    h = hashlib.sha256()
    for name in KERNEL_SOURCES[family]:
        with open(os.path.join(CSRC, name), encoding="utf-8") as f:
            code = re.sub(r"\s+", " ", strip_comments(f.read())).strip()
        h.update(code.encode("utf-8"))
        h.update(b"\0")
    return h.hexdigest()


def measured_traffic(family, model, M, layers):
    """DRAM bytes per launch for this workload, or None when no capture of the
    current kernel sources exists."""
    rec = MEASURED_TRAFFIC.get((family, model, M))
    if rec is None or rec["sha256"] != kernel_sha256(family):
        return None
    return rec["bytes_per_layer"] * layers


# --------------------------------------------------------------- workload --

def op_bytes(M, N, K, bits):
    return N * K * bits // 8 + 4 * N * K // 128 + 2 * M * K + 2 * M * N


# Layer shapes per model: (name, N, K, bits); and the default layer count.
MODELS = {
    "7b": ([(name, N, K, 4) for (name, N, K) in zi.QWEN7B], zi.QWEN7B_LAYERS,
           "qwen2.5-7b-shaped", "INT4 g128", "int4 weights"),
    "32b-mixed": (list(zi.QWEN32B_MIXED), zi.QWEN32B_LAYERS, "qwen2.5-32b-shaped",
                  "INT8 qkv / INT4 o / INT3 gate_up / INT2 down, g128, 0.1% outliers x20",
                  "int8/int4/int3/int2 weights"),
}


def decode_stack_shapes(layers=zi.QWEN7B_LAYERS, model="7b"):
    return [(layer, t, name, N, K, bits) for layer in range(layers)
            for t, (name, N, K, bits) in enumerate(MODELS[model][0])]


class StackWorkload:
    """All tensors of the decode stack resident on the GPU: one contiguous x
    buffer, one contiguous out buffer (views per op), packed weights per op.
    `weights` (another workload's .weights of the same model and layers) are
    reused instead of drawing and quantizing new ones."""

    def __init__(self, zq, M, device, layers=zi.QWEN7B_LAYERS, model="7b", weights=None):
        self.M = M
        shapes = decode_stack_shapes(layers, model)
        outliers = model == "32b-mixed"
        ks = sorted({K for (_, _, _, _, K, _) in shapes})
        x_elems = sum(M * K for K in ks)
        self.x_all = torch.empty(x_elems, dtype=torch.float16, device=device)
        xoff, self.x = 0, {}
        for K in ks:
            v = self.x_all[xoff:xoff + M * K].view(M, K)
            v.copy_(zi.activations(M, K, zi.seed_for(0, zi.X_SEED), device=device))
            self.x[K] = v
            xoff += M * K
        out_elems = sum(M * N for (_, _, _, N, _, _) in shapes)
        self.out_all = torch.empty(out_elems, dtype=torch.float16, device=device)
        self.ops, self.weights, self.bytes, self.flops = [], [], 0, 0
        ooff = 0
        for i, (layer, t, name, N, K, bits) in enumerate(shapes):
            if weights is None:
                w = zi.weight(N, K, zi.seed_for(layer, t), device=device, outliers=outliers)
                q = zq.quantize(w, bits)
                del w
            else:
                q = weights[i][5]
            out = self.out_all[ooff:ooff + M * N].view(M, N)
            ooff += M * N
            self.weights.append((layer, name, N, K, bits, q))
            self.ops.append((self.x[K], *q, out, bits, 128, M, N, K))
            self.bytes += op_bytes(M, N, K, bits)
            self.flops += 2 * M * N * K
        self.descs, self.n_ops = zq.make_descs(self.ops)
        self.zq = zq
        torch.cuda.synchronize()

    def second_outputs(self):
        """A second set of outputs (same weights and x) and its descriptors,
        for the end-to-end run, whose device-to-host copy of step i overlaps
        step i + 1."""
        out2 = torch.empty_like(self.out_all)
        ops2, ooff = [], 0
        for op in self.ops:
            M_, N_ = op[7], op[8]
            ops2.append(op[:4] + (out2[ooff:ooff + M_ * N_].view(M_, N_),) + op[5:])
            ooff += M_ * N_
        descs2, _ = self.zq.make_descs(ops2)
        return out2, descs2


def workload_config(M, layers, world, model="7b"):
    """The `config` object of the JSON line, shared by both arms."""
    shapes = decode_stack_shapes(layers, model)
    nbytes = sum(op_bytes(M, N, K, b) for (_, _, _, N, K, b) in shapes)
    _, _, shaped, fmt, _ = MODELS[model]
    return {"workload": f"{shaped} {'decode' if M <= 64 else 'prefill'} stack: "
                        f"{layers} layers x (qkv, o, gate_up, down), M={M}, {fmt}, "
                        f"one zq_linear_stack call",
            "layer_shapes": ", ".join(f"{name} {N}x{K} INT{b}" for (name, N, K, b) in MODELS[model][0]),
            "layers": layers, "M": M,
            "bits": sorted({b for (*_, b) in shapes}), "group": 128,
            "bytes_per_step": nbytes,
            "flops_per_step": sum(2 * M * N * K for (_, _, _, N, K, _) in shapes),
            "l2": f"inputs larger than L2 ({nbytes / 1e9:.2f} GB per step)",
            "parallelism": f"replicas x{world}"}


# ------------------------------------------------------------ oracle legs --

def oracle_layer_sample(M, seed_layer=0, frac=1.0, device_weights=None, model="7b"):
    """Host inputs for the oracle: the 4 projections of one layer (rows sample).
    device_weights: list of (name, N, K, bits, (packed, scales, zeros)) on GPU
    to copy; else the layer is drawn on the CPU and quantized by the oracle."""
    import oracle as orc
    items = []
    for t, (name, N, K, bits) in enumerate(MODELS[model][0]):
        if device_weights is not None:
            q = device_weights[t][4]
            p = q[0].view(torch.int32).cpu().numpy().view(np.uint32).reshape(N, -1)
            s = q[1].cpu().numpy().view(np.uint16)
            z = q[2].cpu().numpy().view(np.uint16)
        else:
            w = zi.weight(N, K, zi.seed_for(seed_layer, t), outliers=model == "32b-mixed").numpy()
            p, s, z = orc.quantize_pack(w, bits)
        x = zi.activations(M, K, zi.seed_for(0, zi.X_SEED)).numpy().view(np.uint16)
        rows = np.arange(0, N, max(1, int(round(1 / frac))), dtype=np.int64)
        items.append((x, p, s, z, N, K, bits, rows))
    return items


def time_oracle(items, M, budget_s=None):
    """Runs the oracle over the sample (repeating until budget_s if given);
    returns (GB/s, seconds, bytes, threads)."""
    import oracle as orc
    done_bytes, t0 = 0, time.perf_counter()
    while True:
        for (x, p, s, z, N, K, bits, rows) in items:
            orc.linear(x, p, s, z, bits, N, K, rows=rows)
            done_bytes += op_bytes(M, len(rows), K, bits)
        el = time.perf_counter() - t0
        if budget_s is None or el >= budget_s:
            break
    return done_bytes / el / 1e9, el, done_bytes, orc.get_threads()


CONFIG1_SEED = 0  # the single-layer workload draws W and x from seed 0


def oracle_config1_one_core(budget_s=0.5):
    """The small single-layer workload (M=1, N=K=512, INT4; W and x seed 0)
    through the oracle on one host core, repeated for budget_s: time per call
    and GB/s of algorithmic bytes."""
    import oracle as orc
    w = zi.weight(512, 512, CONFIG1_SEED).numpy()
    p, s, z = orc.quantize_pack(w, 4)
    x = zi.activations(1, 512, CONFIG1_SEED).numpy().view(np.uint16)
    prev = orc.get_threads()
    orc.set_threads(1)
    try:
        calls, t0 = 0, time.perf_counter()
        while True:
            orc.linear(x, p, s, z, 4, 512, 512)
            calls += 1
            el = time.perf_counter() - t0
            if el >= budget_s:
                break
    finally:
        orc.set_threads(prev)
    us = el / calls * 1e6
    return {"us_per_call": us, "value": op_bytes(1, 512, 512, 4) / (us * 1e-6) / 1e9, "unit": "GB/s",
            "cores": 1, "sample": f"M=1, N=K=512, INT4 g128, W and x seed 0: {calls} oracle calls in {el:.2f} s"}


# ------------------------------------------------------- all five configs --

def _timed(fn, stream, steps, warmup, device_index):
    """Mean device time per call of fn (CUDA events on `stream`, after
    warm-up, synchronised on both sides) and the clocks seen meanwhile."""
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(device_index) as clk:
        e0.record(stream)
        for _ in range(steps):
            fn()
        e1.record(stream)
        torch.cuda.synchronize()
    return e0.elapsed_time(e1) / steps, clk.summary()


def _hbm_entry(workload, nbytes, ms, peaks, clocks, **extra):
    gbs = nbytes / (ms / 1e3) / 1e9
    d = {"workload": workload, "value": gbs, "unit": "GB/s", "ms": ms,
         "bound": "hbm", "frac": gbs / peaks["hbm_gbs"], "peak": peaks["hbm_gbs"],
         "pct_of_8tbs": 100 * gbs / NOMINAL_HBM_GBS, "algorithmic_bytes": nbytes, "clocks": clocks}
    d.update(extra)
    return d


def run_all_configs(zq, wl, dev, stream, peaks, args, device_index):
    """Every workload the method is specified on, each timed on its own after
    the headline (which they do not touch): the single 512 x 512 layer, the
    four 7B-shaped projections one call at a time, the 7B stack at M = 4, 16
    and 64 and at M = 2048 (prefill), and the 32B-shaped mixed-precision stack.
    The 7B workloads reuse the headline's 28 layers of weights."""
    import oracle as orc
    sp = stream.cuda_stream
    out = {}

    # Config 1: M = 1, N = K = 512, INT4; W quantized by the oracle; 8 copies
    # in rotation (all of them fit in L2: the call is latency-bound).
    N = K = 512
    p, sc, z = orc.quantize_pack(zi.weight(N, K, CONFIG1_SEED).numpy(), 4)
    copies = [tuple(torch.from_numpy(a.view(np.int32 if a.dtype == np.uint32 else np.int16).copy()).to(dev)
                    for a in (p, sc, z)) for _ in range(8)]
    x1 = zi.activations(1, K, CONFIG1_SEED, device=dev)
    y1 = torch.empty(1, N, dtype=torch.float16, device=dev)
    zq.ensure_workspace(zq.zq_linear_workspace_bytes(4, 1, N, K), stream)
    state = {"i": 0}

    def call1():
        q = copies[state["i"] % 8]
        state["i"] += 1
        zq.zq_linear(x1, q[0], q[1], q[2], 4, 128, 1, N, K, y1, sp)

    ms, clk = _timed(call1, stream, 400, 20, device_index)
    out["config1_single_layer"] = _hbm_entry(
        "M=1, N=K=512, INT4 g128, one zq_linear call (W and x seed 0; 8 weight copies in rotation, "
        "141 KB each, L2-resident: latency-bound, not gated on the roofline)",
        op_bytes(1, N, K, 4), ms, peaks, clk, us_per_call=ms * 1e3)

    # Config 2: the four 7B-shaped projections at M = 1, one zq_linear call each,
    # rotating over the 28 layers' distinct weights (3.47 GB, no L2 reuse).
    per = {}
    x_by_k = {K: wl.x[K][:1] for K in wl.x}
    for t, (name, N, K, bits) in enumerate(MODELS["7b"][0]):
        layers = [w for w in wl.weights if w[1] == name]
        yb = torch.empty(1, N, dtype=torch.float16, device=dev)
        zq.ensure_workspace(zq.zq_linear_workspace_bytes(bits, 1, N, K), stream)

        def calls(layers=layers, N=N, K=K, bits=bits, yb=yb):
            for (_, _, _, _, _, q) in layers:
                zq.zq_linear(x_by_k[K], q[0], q[1], q[2], bits, 128, 1, N, K, yb, sp)

        ms, clk = _timed(calls, stream, 10, 3, device_index)
        ms_call = ms / len(layers)
        per[name] = _hbm_entry(f"{name} {N}x{K} INT4, M=1, one zq_linear call", op_bytes(1, N, K, bits),
                               ms_call, peaks, clk, us_per_call=ms_call * 1e3)
    out["config2_7b_projections_m1"] = per

    # Config 3 at M = 4, 16, 64 and config 5 (M = 2048): the 28-layer 7B stack.
    for M, steps, key in ((4, 20, "config3_7b_stack_m4"), (16, 20, "config3_7b_stack_m16"),
                          (64, 20, "config3_7b_stack_m64"), (2048, 5, "config5_7b_prefill_m2048")):
        w2 = StackWorkload(zq, M, dev, zi.QWEN7B_LAYERS, "7b", weights=wl.weights)
        zq.ensure_workspace(zq.zq_linear_stack_workspace_bytes(w2.descs, w2.n_ops), stream)
        ms, clk = _timed(lambda w2=w2: zq.zq_linear_stack(w2.descs, w2.n_ops, sp), stream, steps, 3,
                         device_index)
        name = f"28-layer 7B-shaped INT4 stack, M={M}, one zq_linear_stack call"
        if M <= 64:
            out[key] = _hbm_entry(name, w2.bytes, ms, peaks, clk, tokens_per_s_equiv=M / (ms / 1e3))
        else:
            tf = w2.flops / (ms / 1e3) / 1e12
            out[key] = {"workload": name, "value": tf, "unit": "TFLOP/s", "ms": ms, "bound": "tensor",
                        "frac": tf / peaks["bf16_tflops"], "peak": peaks["bf16_tflops"],
                        "peak_note": "measured dense bf16 burst rate (a step of tens of ms timed alone); "
                                     "fp16 has the same dense rate",
                        "frac_of_nominal_2250": tf / 2250.0, "algorithmic_flops": w2.flops,
                        "tokens_per_s_equiv": M / (ms / 1e3), "clocks": clk}
        del w2
        torch.cuda.empty_cache()

    # Config 4: the 32B-shaped mixed-precision stack (INT8 qkv, INT4 o, INT3
    # gate_up, INT2 down, 0.1% outliers x20) at M = 1.
    L32 = args.extra_32b_layers
    w4 = StackWorkload(zq, 1, dev, L32, "32b-mixed")
    zq.ensure_workspace(zq.zq_linear_stack_workspace_bytes(w4.descs, w4.n_ops), stream)
    ms, clk = _timed(lambda: zq.zq_linear_stack(w4.descs, w4.n_ops, sp), stream, 20, 3, device_index)
    out["config4_32b_mixed_m1"] = _hbm_entry(
        f"{L32}-layer 32B-shaped mixed-precision stack (qkv 7168x5120 INT8, o 5120x5120 INT4, "
        f"gate_up 55296x5120 INT3, down 5120x27648 INT2), M=1, one zq_linear_stack call "
        f"({w4.bytes / 1e9:.2f} GB of weights, larger than L2)", w4.bytes, ms, peaks, clk,
        tokens_per_s_equiv=1 / (ms / 1e3), layers=L32)
    del w4
    torch.cuda.empty_cache()
    return out


# ------------------------------------------------------------------- arms --

def run_reference(args):
    world, rank, _ = dist_env()
    if rank != 0:
        return 0
    M = args.m
    items = oracle_layer_sample(M, frac=args.ref_frac, model=args.model)
    for _ in range(args.warmup):
        time_oracle(items, M)
    vals, secs, nbytes = [], 0.0, 0
    t0 = time.perf_counter()
    for _ in range(args.steps):
        v, el, b, threads = time_oracle(items, M)
        secs += el
        nbytes += b
    total = time.perf_counter() - t0
    value = nbytes / total / 1e9
    sample = (f"each step: oracle linear on every {int(round(1 / args.ref_frac))}th row of the 4 "
              f"projections of one 7B-shaped INT4 layer at M={M} (fp64, OpenMP over rows); "
              f"throughput in the same algorithmic-byte units as the GPU arm")
    line = {"metric": METRIC, "impl": "reference", "value": value, "unit": "GB/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": total / args.steps * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(M, args.layers, args.gpus, args.model),
            "cpu_baseline": {"value": value, "unit": "GB/s", "cores": threads, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def run_zq(args):
    world, rank, local = dist_init("nccl")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    import weight_only_quantized_zq_b200 as zq
    peaks = load_peaks()
    M = args.m
    wl = StackWorkload(zq, M, dev, args.layers, args.model)
    stream = torch.cuda.current_stream(dev)
    sp = stream.cuda_stream

    # the stack's workspace is reserved once, outside every timed region
    zq.ensure_workspace(zq.zq_linear_stack_workspace_bytes(wl.descs, wl.n_ops), stream)

    def step():
        zq.zq_linear_stack(wl.descs, wl.n_ops, sp)

    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()

    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    launches0 = zq.zq_kernel_launches()
    with ClockSampler(local) as clk:
        ev0.record(stream)
        for _ in range(args.steps):
            step()
        ev1.record(stream)
        torch.cuda.synchronize()
    launches = zq.zq_kernel_launches() - launches0
    barrier(world)
    ms = ev0.elapsed_time(ev1)
    ms_max = max_over_ranks(ms, world, dev)
    ms_step = ms_max / args.steps
    value = world * wl.bytes * args.steps / (ms_max / 1e3) / 1e9

    # End to end through the public API with host buffers, per step: pinned
    # H2D of the step's activations, the stack, D2H of every output.  As a
    # serving loop would, the outputs alternate between two device buffers and
    # their D2H copy runs on a second stream, overlapping the next step; the
    # timed region ends after the last step's copy has landed.
    x_host = torch.empty(wl.x_all.numel(), dtype=torch.float16, pin_memory=True)
    x_host.copy_(wl.x_all)
    out_all2, descs2 = wl.second_outputs()
    outs = (wl.out_all, out_all2)
    descs = (wl.descs, descs2)
    out_host = [torch.empty(wl.out_all.numel(), dtype=torch.float16, pin_memory=True) for _ in range(2)]
    copy_stream = torch.cuda.Stream(dev)
    done = [torch.cuda.Event() for _ in range(2)]     # step into buffer b finished
    copied = [torch.cuda.Event() for _ in range(2)]   # D2H of buffer b finished
    torch.cuda.synchronize()
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(args.steps):
        b = i % 2
        wl.x_all.copy_(x_host, non_blocking=True)
        if i >= 2:
            stream.wait_event(copied[b])  # buffer b's previous outputs have left the GPU
        zq.zq_linear_stack(descs[b], wl.n_ops, sp)
        done[b].record(stream)
        copy_stream.wait_event(done[b])
        with torch.cuda.stream(copy_stream):
            out_host[b].copy_(outs[b], non_blocking=True)
        copied[b].record(copy_stream)
    for b in range(2):
        stream.wait_event(copied[b])
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
    e2e_value = world * wl.bytes * args.steps / (e2e_ms / 1e3) / 1e9

    # Roofline of the dominant kernel.  Decode (M <= 64): the grouped launch;
    # with M <= 32 the step is one prep launch + one decode launch, timed
    # together by the events above, so the figure is a lower bound for the
    # kernel.  Prefill (M > 64): the grouped tcgen05 launches.
    achieved = wl.bytes / (ms_step / 1e3) / 1e9
    bits_used = sorted({b for (*_, b) in decode_stack_shapes(args.layers, args.model)}, reverse=True)
    # The tile kernel's shared-memory plan: one token half when every M <= 128.
    bits_s = "|".join(str(b) for b in bits_used)
    if M <= 128:
        tile_kernel = f"prefill_kernel<{bits_s},true> (one-token-half plan)"
    elif M >= PAIR_MIN_M and 16 not in bits_used:
        tile_kernel = f"prefill_pair_kernel<{bits_s}> (CTA pairs, tcgen05.mma.cta_group::2)"
    else:
        tile_kernel = f"prefill_kernel<{bits_s},false> (two-token-half plan)"
    if M <= 64:
        roofline = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                    "frac": achieved / peaks["hbm_gbs"],
                    "traffic": measured_traffic("decode" if M <= DECODE_MAX_M else "prefill", args.model, M, args.layers),
                    "traffic_note": ("per step (one decode launch)" if M <= DECODE_MAX_M else
                                     "per step (the stack's grouped tile-kernel launches)"),
                    "algorithmic_bytes": wl.bytes,
                    "peak_source": peaks["source"],
                    "kernel": (f"decode_kernel<{'|'.join(str(b) for b in bits_used)},{zq_mt(M)}> + prep_kernel"
                               + (" (one launch pair per bit width)" if len(bits_used) > 1 else "")
                               if M <= DECODE_MAX_M else tile_kernel)}
    else:
        tflops = wl.flops / (ms_step / 1e3) / 1e12
        peak = peaks["bf16_tflops"]  # burst: a step of tens of ms, timed alone
        traffic = measured_traffic("prefill", args.model, M, args.layers)
        roofline = {"bound": "tensor", "achieved": tflops, "peak": peak, "unit": "TFLOP/s",
                    "frac": tflops / peak,
                    "traffic": None if traffic is None else traffic / (4 * args.layers),
                    "traffic_note": "per launch, averaged over the 4 projections of a layer",
                    "algorithmic_flops": wl.flops,
                    "peak_source": peaks["source"] + " (dense bf16 burst; fp16 has the same dense rate)",
                    "kernel": tile_kernel,
                    "tflops_vs_nominal_2250": tflops / 2250.0}

    configs = None
    if world == 1 and not args.no_extra:
        configs = run_all_configs(zq, wl, dev, stream, peaks, args, local)

    line = None
    if rank == 0:
        cpu = None
        if world == 1 and not args.no_cpu_baseline:
            items = oracle_layer_sample(M, device_weights=[w[1:] for w in wl.weights[:4]], frac=1.0,
                                        model=args.model)
            v, el, b, threads = time_oracle(items, M, budget_s=args.cpu_seconds)
            cpu = {"value": v, "unit": "GB/s", "cores": threads, "kind": "oracle",
                   "sample": f"oracle linear (fp64, OpenMP over rows) on all 4 projections of layer 0 "
                             f"at M={M}, repeated for {el:.1f} s ({b / 1e9:.2f} GB of algorithmic bytes)",
                   "one_core_small_layer": oracle_config1_one_core()}
        line = {"metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": f"f16 in, f32 accumulate, {MODELS[args.model][4]}", "data": "synthetic",
                "config": workload_config(M, args.layers, world, args.model),
                "pct_of_8tbs": 100 * achieved / NOMINAL_HBM_GBS,
                "tokens_per_s_equiv": world * M / (ms_step / 1e3),
                "roofline": roofline,
                "cpu_baseline": cpu,
                "e2e": {"value": e2e_value, "unit": "GB/s",
                        "h2d_bytes_per_step": wl.x_all.numel() * 2,
                        "d2h_bytes_per_step": wl.out_all.numel() * 2,
                        "ms_per_step": e2e_ms / args.steps},
                "gpu_launches": launches,
                "clocks": clk.summary(),
                "configs": configs}
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()
    return 0


DECODE_MAX_M = 32  # the library runs M <= 32 on the decode kernel
PAIR_MIN_M = 512   # and launches of b-bit codes with some M >= 512 on the CTA-pair tile kernel


def zq_mt(M):
    return 1 if M <= 8 else 2 if M <= 16 else 4


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("zq", "reference"), default="zq")
    ap.add_argument("--m", type=int, default=1, help="tokens per step (decode batch)")
    ap.add_argument("--model", choices=sorted(MODELS), default="7b",
                    help="layer shapes: the 7B INT4 stack (default) or the 32B mixed-precision stack")
    ap.add_argument("--layers", type=int, default=None, help="layers in the stack (default: the model's)")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--ref-frac", type=float, default=0.25, help="row fraction per reference step")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra", action="store_true",
                    help="skip the other workloads (single layer, projections, M = 4/16/64/2048, 32B mixed)")
    ap.add_argument("--extra-32b-layers", type=int, default=16,
                    help="layers of the 32B mixed-precision stack among the other workloads")
    args = ap.parse_args(argv)
    if args.layers is None:
        args.layers = MODELS[args.model][1]
    if args.impl == "reference":
        return run_reference(args)
    return run_zq(args)


if __name__ == "__main__":
    sys.exit(main())
