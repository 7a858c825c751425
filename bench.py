"""Benchmark: MXFP4 quantize+pack throughput on one or more B200s.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl mx|reference]
    python -m torch.distributed.run --nproc-per-node N --master-addr 127.0.0.1 \
        --master-port P bench.py --gpus N --steps K --warmup W

One step = one MXFP4 (E2M1 elements, E8M0 scales) FLOOR quantize+pack of the
MoE w13 expert stack [128, 1536, 2048] bf16 (N(0, 0.02^2) times a per-expert
U(0.5, 2) factor, seeded, generated on the device): 805,306,368 input bytes,
201,326,592 code bytes and 12,582,912 scale bytes. GB/s counts those
algorithmic bytes (bf16 in + packed out). The input is far larger than L2
(126 MB), so no flush is needed between steps. With N ranks every rank
quantizes its own stack (weak scaling: rows are independent, there is no
data exchange); the step time is the maximum over ranks.

The JSON line also carries: the roofline of the kernel (CUDA-event duration of
each launch inside the timed region against the measured HBM copy bandwidth),
the end-to-end figure through the public API with host buffers (pinned input
copied in, outputs copied out, inside the timed region), the oracle timed on
the host cores on a bounded sample (`cpu_baseline`), SM clocks sampled with
nvidia-smi during the timed region, and per-op figures for the other
workloads (`ops`).

--impl reference times the CPU oracle (the only other implementation of this
path) on the same workload, a bounded sample per step, and prints the same
line with "impl": "reference".
"""

from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import re
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MXFP4 quantize+pack GB/s (bf16 in + packed out) and % of B200 HBM peak"
WORKLOAD = "moe_w13 [128,1536,2048] bf16 -> MXFP4 (E2M1 codes [128,1536,1024] + E8M0 scales [128,1536,64]), FLOOR scaling"
EXPERTS, INTER2, HIDDEN = 128, 1536, 2048
N_ELEM = EXPERTS * INTER2 * HIDDEN
BYTES_IN = 2 * N_ELEM
BYTES_CODES = N_ELEM // 2
BYTES_SCALES = N_ELEM // 32
BYTES_STEP = BYTES_IN + BYTES_CODES + BYTES_SCALES            # 1,019,215,872
FALLBACK_HBM_GBS = 6650.0
KERNEL_SOURCES = ["fp8_quantization_mx_b200/csrc/mx_kernels.cu",
                  "fp8_quantization_mx_b200/csrc/mx_stream.cuh",
                  "fp8_quantization_mx_b200/csrc/mx_device.cuh"]
PROFILE = os.path.join(ROOT, "profiles", "quantize_fp4_floor_moe_w13.md")


# ------------------------------------------------------------------ helpers --

def kernel_source_hash() -> str:
    h = hashlib.sha256()
    for p in KERNEL_SOURCES:
        with open(os.path.join(ROOT, p), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def measured_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured (MEASURED_PEAKS.json hbm_gbs, copy burst)"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def profiled_traffic():
    """DRAM bytes per launch recorded by ncu for the timed kernel, if current."""
    try:
        text = open(PROFILE).read()
    except OSError:
        return None, "no profile"
    t = re.search(r"traffic_bytes_per_launch:\s*([0-9]+)", text)
    h = re.search(r"kernel_source_sha256_16:\s*([0-9a-f]+)", text)
    if not t or not h:
        return None, "profile lacks figures"
    if h.group(1) != kernel_source_hash():
        return None, "kernel changed since the capture"
    return int(t.group(1)), "ncu dram__bytes_read.sum + dram__bytes_write.sum"


class ClockSampler:
    """nvidia-smi clocks/throttle reasons sampled while the timed region runs."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int, period_ms: int = 50):
        self.index = index
        self.period_ms = period_ms
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", str(self.period_ms)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
            time.sleep(0.3)
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.2)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.lines:
            f = [p.strip() for p in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": [], "samples": 0}
        sm.sort()
        return {"sm_mhz": sm[len(sm) // 2], "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def _timed(fn):
    t0 = time.perf_counter()
    fn()
    return time.perf_counter() - t0


def _rows_for(fn_rows, total_rows, budget_s, probe_rows):
    """Rows of a sample that takes about budget_s, from a timed probe."""
    probe_rows = min(probe_rows, total_rows)
    dt = _timed(lambda: fn_rows(probe_rows))
    rate = probe_rows / max(dt, 1e-6)
    return int(min(total_rows, max(probe_rows, rate * budget_s)))


def oracle_baseline(x_host_rows, inputs_mod, budget_s: float = 8.0):
    """The CPU oracle on the host cores: the headline workload (MoE w13 stack,
    MXFP4 FLOOR quantize) on a bounded sample with every core and with one
    thread, then each other workload's op(s) on a bounded sample with every
    core. Input SHA-256 over each whole tensor's bf16 bytes."""
    import hashlib as _hl
    import numpy as np
    import oracle
    threads = len(os.sched_getaffinity(0))
    oracle.set_threads(threads)
    q = lambda rows: oracle.quantize(x_host_rows[:rows], 0, 0)
    nrows = _rows_for(q, x_host_rows.shape[0], budget_s, 256)
    dt = _timed(lambda: q(nrows))
    n = nrows * HIDDEN
    per_elem_bytes = 2 + 0.5 + 1 / 32
    out = {"value": n * per_elem_bytes / dt / 1e9, "unit": "GB/s", "cores": threads, "kind": "oracle",
           "cpu_model": cpu_model(),
           "sample": f"first {nrows} of {x_host_rows.shape[0]} rows of 2048 ({n} elements) of the "
                     f"headline stack, {dt:.2f} s on {threads} threads, scalar C++ oracle",
           "input_sha256": {"moe_w13_128x1536x2048": _hl.sha256(x_host_rows.tobytes()).hexdigest()},
           "input_sha256_of": "the tensors the oracle timed: the headline stack is the bench's own "
                              "input copied from the device; the other workloads are generated on "
                              "the host from the same seeds (a different stream than on the device)"}
    oracle.set_threads(1)
    r1 = _rows_for(q, x_host_rows.shape[0], 2.0, 16)
    d1 = _timed(lambda: q(r1))
    out["single_thread"] = {"value": r1 * HIDDEN * per_elem_bytes / d1 / 1e9, "unit": "GB/s",
                            "sample": f"first {r1} rows, {d1:.2f} s, 1 thread"}
    oracle.set_threads(threads)
    per_cfg = {}

    def rec(name, arr, bytes_per_elem, fn, budget=1.5, probe=64):
        rows = _rows_for(lambda r: fn(arr[:r]), arr.shape[0], budget, probe)
        dtc = _timed(lambda: fn(np.ascontiguousarray(arr[:rows])))
        ne = rows * arr.shape[1]
        per_cfg[name] = {"GB/s": round(ne * bytes_per_elem / dtc / 1e9, 4),
                         "elements_per_s": round(ne / dtc), "rows": rows, "of_rows": arr.shape[0],
                         "s": round(dtc, 3)}

    bits = inputs_mod.bf16_bits_numpy
    x1 = bits(inputs_mod.outlier_act())
    out["input_sha256"]["outlier_act_256x4096"] = _hl.sha256(x1.tobytes()).hexdigest()
    rec("outlier_act_256x4096/fp4_floor_quantize", x1, 2.53125, lambda a: oracle.quantize(a, 0, 0))
    c1, s1, _ = oracle.quantize(x1, 0, 0)
    t_deq = _timed(lambda: oracle.dequantize(c1, s1, None, 256, 4096, 0))
    per_cfg["outlier_act_256x4096/fp4_dequantize_bf16"] = {
        "GB/s": round(256 * 4096 * 2.53125 / t_deq / 1e9, 4), "rows": 256, "of_rows": 256,
        "s": round(t_deq, 3)}
    x2 = bits(inputs_mod.mlp_weight())
    out["input_sha256"]["mlp_weight_8192x3072"] = _hl.sha256(x2.tobytes()).hexdigest()
    rec("mlp_weight_8192x3072/fp8_floor_quantize", x2, 3.03125, lambda a: oracle.quantize(a, 1, 0))
    x3 = bits(inputs_mod.qat_act())
    g3 = bits(inputs_mod.qat_grad(16384, 3072))
    out["input_sha256"]["qat_act_16384x3072"] = _hl.sha256(x3.tobytes()).hexdigest()
    rec("qat_act_16384x3072/fp4_fake_quant_fwd", x3, 4, lambda a: oracle.fake_quant_fwd(a))
    rec("qat_act_16384x3072/fp4_fake_quant_bwd", x3, 6,
        lambda a: oracle.fake_quant_bwd(a, np.ascontiguousarray(g3[:a.shape[0]])))
    x4 = bits(inputs_mod.heavy_tail())
    out["input_sha256"]["heavy_tail_8192x4096"] = _hl.sha256(x4.tobytes()).hexdigest()
    for mname, m in (("FLOOR", 0), ("OAS", 3), ("MBS_STATIC", 16), ("MBS_DYNAMIC", 32)):
        rec(f"heavy_tail_8192x4096/fp4_{mname}_quantize", x4, 2.53125 + (1 / 128 if m >> 4 else 0),
            lambda a, m=m: oracle.quantize(a, 0, m), budget=1.0, probe=2 if m >> 4 == 2 else 32)
    rec("heavy_tail_8192x4096/fp4_FLOOR_block_error", x4, 2,
        lambda a: oracle.block_error(a, 0, 0, want_blocks=False))
    out["per_config"] = per_cfg
    return out


# --------------------------------------------------------------- arms --

def run_reference(args):
    """The oracle on the host cores, one bounded sample of the workload per step."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import numpy as np
    import torch
    import oracle
    from fp8_quantization_mx_b200 import inputs
    threads = len(os.sched_getaffinity(0))
    oracle.set_threads(threads)
    # a few experts of the same seeded stack, generated on the host
    x = inputs.moe_w13(experts=16, device="cpu")
    xb = inputs.bf16_bits_numpy(x).reshape(-1, HIDDEN)
    t0 = time.perf_counter()
    oracle.quantize(xb[:512], 0, 0)
    rate = 512 / max(time.perf_counter() - t0, 1e-6)
    budget = max(0.5, min(5.0, 120.0 / max(1, args.steps + args.warmup)))
    nrows = int(min(xb.shape[0], max(64, rate * budget)))
    sample = np.ascontiguousarray(xb[:nrows])
    for _ in range(args.warmup):
        oracle.quantize(sample, 0, 0)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.quantize(sample, 0, 0)
    dt = (time.perf_counter() - t0) / args.steps
    nbytes = sample.size * 2 + sample.size // 2 + sample.size // 32
    value = nbytes / dt / 1e9
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": dt * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD, "sample_rows": nrows, "rows_total": EXPERTS * INTER2},
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": threads, "kind": "oracle",
                         "sample": f"{nrows} rows of 2048 ({sample.size} elements) per step"},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def time_op(fn, reps, flush=None, stream=None):
    """Mean kernel time (ms) of fn() over reps, CUDA events on the launching stream."""
    import torch
    stream = stream or torch.cuda.current_stream()
    times = []
    for _ in range(reps):
        if flush is not None:
            flush.zero_()
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record(stream)
        fn()
        e.record(stream)
        e.synchronize()
        times.append(s.elapsed_time(e))
    times.sort()
    return times[len(times) // 2]


def stack_ops(mx, x, reps=50, only=None):
    """GB/s of every op on the 403 M-element MoE stack x [rows, 2048]: mean
    over `reps` back-to-back launches (x is far larger than L2). `only` names
    one op to run alone (for profiling)."""
    import torch
    rows, cols = x.shape
    n = x.numel()
    dev = x.device
    c4 = torch.empty(rows, cols // 2, dtype=torch.uint8, device=dev)
    c8 = torch.empty(rows, cols, dtype=torch.uint8, device=dev)
    sc = torch.empty(rows, cols // 32, dtype=torch.uint8, device=dev)
    sc16 = torch.empty(rows, cols // 16, dtype=torch.uint8, device=dev)
    mac = torch.empty(rows, cols // 128, dtype=torch.uint8, device=dev)
    sc_mma = torch.empty(mx.mx_scale_bytes(rows, cols, mx.E2M1, mx.MMA_SCALES), dtype=torch.uint8,
                         device=dev)
    y = torch.empty_like(x)
    g = torch.empty_like(x).normal_()
    fp4, fp8, fp4m = n * 2.53125, n * 3.03125, n * (2.53125 + 1 / 128)
    from fp8_quantization_mx_b200 import inputs as _inputs
    bat = {a: _inputs.bat_params(a, cols // 32, device=dev) for a in (1, 2, 4, 8)}
    ops = {
        "fp4_floor_quantize": (lambda: mx.quantize(x, mx.E2M1, mx.FLOOR, out=(c4, sc, None)), fp4),
        "fp8_floor_quantize": (lambda: mx.quantize(x, mx.E4M3, mx.FLOOR, out=(c8, sc, None)), fp8),
        "fp4_oas_quantize": (lambda: mx.quantize(x, mx.E2M1, mx.OAS, out=(c4, sc, None)), fp4),
        "fp4_mbs_static_quantize": (lambda: mx.quantize(x, mx.E2M1, mx.MBS_STATIC, out=(c4, sc, mac)), fp4m),
        "fp4_oas_mbs_static_quantize": (lambda: mx.quantize(x, mx.E2M1, mx.OAS | mx.MBS_STATIC,
                                                            out=(c4, sc, mac)), fp4m),
        "fp4_fake_quant_fwd": (lambda: mx.fake_quant(x, out=y), n * 4),
        "fp4_fake_quant_bwd": (lambda: mx.fake_quant_bwd(x, g, out=y), n * 6),
        "fp4_oas_fake_quant_fwd": (lambda: mx.fake_quant(x, mx.E2M1, mx.OAS, out=y), n * 4),
        "fp4_dequantize_bf16": (lambda: mx.dequantize(c4, sc, None, mx.E2M1, out=y), fp4),
        "fp8_dequantize_bf16": (lambda: mx.dequantize(c8, sc, None, mx.E4M3, out=y), fp8),
        "fp4_block_error": (lambda: mx.block_error(x, per_block=False), n * 2),
        "fp4_floor_quantize_mma_scales": (lambda: mx.quantize(x, mx.E2M1, mx.FLOOR | mx.MMA_SCALES,
                                                              out=(c4, sc_mma, None)), fp4),
        "nvfp4_quantize": (lambda: mx.quantize(x, mx.NVFP4, mx.FLOOR, out=(c4, sc16, None)),
                           n * (2.5 + 1 / 16)),
        "fp4b16_floor_quantize": (lambda: mx.quantize(x, mx.E2M1_B16, mx.FLOOR, out=(c4, sc16, None)),
                                  n * (2.5 + 1 / 16)),
        "e5m2_floor_quantize": (lambda: mx.quantize(x, mx.E5M2, mx.FLOOR, out=(c8, sc, None)), fp8),
        "e3m2_floor_quantize": (lambda: mx.quantize(x, mx.E3M2, mx.FLOOR, out=(c8, sc, None)), fp8),
        "e2m3_floor_quantize": (lambda: mx.quantize(x, mx.E2M3, mx.FLOOR, out=(c8, sc, None)), fp8),
        "int8_floor_quantize": (lambda: mx.quantize(x, mx.INT8, mx.FLOOR, out=(c8, sc, None)), fp8),
        "e4m3_oas_quantize": (lambda: mx.quantize(x, mx.E4M3, mx.OAS, out=(c8, sc, None)), fp8),
        "e5m2_oas_quantize": (lambda: mx.quantize(x, mx.E5M2, mx.OAS, out=(c8, sc, None)), fp8),
        "e2m3_oas_quantize": (lambda: mx.quantize(x, mx.E2M3, mx.OAS, out=(c8, sc, None)), fp8),
        "int8_dequantize_bf16": (lambda: mx.dequantize(c8, sc, None, mx.INT8, out=y), fp8),
        # BATQuant: block transform B_j (x) A (a x a, b x b), clip, MXFP4 FLOOR
        "fp4_bat_a8_quantize": (lambda: mx.bat_quantize(x, *bat[8], out=(c4, sc, None)), fp4),
        "fp4_bat_a4_quantize": (lambda: mx.bat_quantize(x, *bat[4], out=(c4, sc, None)), fp4),
        "fp4_bat_a2_quantize": (lambda: mx.bat_quantize(x, *bat[2], out=(c4, sc, None)), fp4),
        "fp4_bat_a1_quantize": (lambda: mx.bat_quantize(x, *bat[1], out=(c4, sc, None)), fp4),
        "bat_a8_apply": (lambda: mx.bat_apply(x, *bat[8], out=y), n * 4),
        "fp4_mbs_dynamic_quantize": (lambda: mx.quantize(x, mx.E2M1, mx.MBS_DYNAMIC, out=(c4, sc, mac)),
                                     fp4m),
        "fp4_oas_mbs_dynamic_quantize": (lambda: mx.quantize(x, mx.E2M1, mx.OAS | mx.MBS_DYNAMIC,
                                                             out=(c4, sc, mac)), fp4m),
    }
    # the OAS + MBS-Dynamic search is ~100x slower than a stream: fewer launches
    op_reps = {"fp4_oas_mbs_dynamic_quantize": 3}
    if only is not None:
        if only not in ops:
            raise SystemExit(f"unknown op {only!r}; one of {sorted(ops)}")
        ops = {only: ops[only]}
    res = {}
    for name, (fn, nbytes) in ops.items():
        if name == "fp4_dequantize_bf16":
            mx.quantize(x, mx.E2M1, mx.FLOOR, out=(c4, sc, None))
        if name == "fp8_dequantize_bf16":
            mx.quantize(x, mx.E4M3, mx.FLOOR, out=(c8, sc, None))
        if name == "int8_dequantize_bf16":
            mx.quantize(x, mx.INT8, mx.FLOOR, out=(c8, sc, None))
        fn()
        torch.cuda.synchronize()
        n_reps = min(reps, op_reps.get(name, reps))
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record()
        for _ in range(n_reps):
            fn()
        e.record()
        e.synchronize()
        ms = s.elapsed_time(e) / n_reps
        res[name] = {"ms": round(ms, 4), "GB/s": round(nbytes / ms / 1e6, 1)}
    del c4, c8, sc, sc16, mac, sc_mma, y, g, bat
    return res


def other_ops(mx, inputs, dev, reps=10):
    """GB/s of the other ops on their workloads (median of reps; L2 flushed before each)."""
    import torch
    flush = torch.empty(512 << 20, dtype=torch.uint8, device=dev)
    res = {}

    def rec(name, nbytes, fn):
        fn()
        torch.cuda.synchronize()
        ms = time_op(fn, reps, flush)
        res[name] = {"ms": round(ms, 4), "GB/s": round(nbytes / ms / 1e6, 1)}

    x1 = inputs.outlier_act(device=dev)
    n1 = x1.numel()
    c, s, _ = mx.quantize(x1)
    rec("outlier_act_256x4096/fp4_floor_quantize", 2 * n1 + n1 // 2 + n1 // 32, lambda: mx.quantize(x1, out=(c, s, None)))
    y1 = torch.empty_like(x1)
    rec("outlier_act_256x4096/fp4_dequantize_bf16", 2 * n1 + n1 // 2 + n1 // 32,
        lambda: mx.dequantize(c, s, None, out=y1))
    del x1, y1
    x2 = inputs.mlp_weight(device=dev)
    n2 = x2.numel()
    c2, s2, _ = mx.quantize(x2, mx.E4M3)
    rec("mlp_weight_8192x3072/fp8_floor_quantize", 2 * n2 + n2 + n2 // 32,
        lambda: mx.quantize(x2, mx.E4M3, out=(c2, s2, None)))
    y2 = torch.empty_like(x2)
    rec("mlp_weight_8192x3072/fp8_dequantize_bf16", 2 * n2 + n2 + n2 // 32,
        lambda: mx.dequantize(c2, s2, None, mx.E4M3, out=y2))
    del x2, y2, c2, s2
    for name, gen in (("qat_act_16384x3072", inputs.qat_act), ("qat_weight_8192x3072", inputs.qat_weight)):
        x3 = gen(device=dev)
        n3 = x3.numel()
        g3 = inputs.qat_grad(*x3.shape, device=dev)
        y3 = torch.empty_like(x3)
        rec(f"{name}/fp4_fake_quant_fwd", 4 * n3, lambda: mx.fake_quant(x3, out=y3))
        rec(f"{name}/fp4_fake_quant_bwd", 6 * n3, lambda: mx.fake_quant_bwd(x3, g3, out=y3))
        del x3, g3, y3
    x4 = inputs.heavy_tail(device=dev)
    n4 = x4.numel()
    # the eight MXFP4 modes, then the block-16 comparison formats of the
    # MXFP4 / NVFP4 gap analysis (MSE and SQNR on the same tensor)
    modes = [("fp4", mx.E2M1, "FLOOR", 0), ("fp4", mx.E2M1, "CEIL", 1),
             ("fp4", mx.E2M1, "OAS_RULE", 2), ("fp4", mx.E2M1, "OAS", 3),
             ("fp4", mx.E2M1, "MBS_STATIC", 16), ("fp4", mx.E2M1, "MBS_DYNAMIC", 32),
             ("fp4", mx.E2M1, "OAS+MBS_STATIC", 19), ("fp4", mx.E2M1, "OAS+MBS_DYNAMIC", 35),
             ("fp4b16", mx.E2M1_B16, "FLOOR", 0), ("fp4b16", mx.E2M1_B16, "OAS", 3),
             ("fp4b16", mx.E2M1_B16, "MBS_STATIC", 16), ("fp4b16", mx.E2M1_B16, "MBS_DYNAMIC", 32),
             ("fp4b16", mx.E2M1_B16, "OAS+MBS_DYNAMIC", 35),
             ("nvfp4", mx.NVFP4, "FLOOR", 0)]
    for fname, fmt, mname, m in modes:
        bufs = mx.quantize(x4, fmt, m)
        extra = n4 // 128 if m >> 4 else 0
        rec(f"heavy_tail_8192x4096/{fname}_{mname}_quantize",
            2 * n4 + n4 // 2 + n4 // mx.block_size(fmt) + extra,
            lambda: mx.quantize(x4, fmt, m, out=bufs))
        _, tot = mx.block_error(x4, fmt, m, per_block=False)
        rec(f"heavy_tail_8192x4096/{fname}_{mname}_block_error", 2 * n4,
            lambda: mx.block_error(x4, fmt, m, per_block=False))
        t = tot.cpu().tolist()
        res[f"heavy_tail_8192x4096/{fname}_{mname}_block_error"].update(
            {"mse": t[0] / n4, "sqnr_db": (10 * __import__("math").log10(t[1] / t[0])) if t[0] > 0 else None})
    del x4
    return res


GEMM_SHAPES = [
    # (name, M tokens, N, K): the Llama-3.2-3B MLP weight [8192, 3072] as B
    ("llama3.2-3b_mlp_prefill_4096tok", 4096, 8192, 3072),
    ("llama3.2-3b_mlp_decode_128tok", 128, 8192, 3072),
    ("square_8192", 8192, 8192, 8192),
]


def measured_fp4_peak():
    """Dense FP4 tensor peak: the measured bf16 GEMM burst x 4 (the nominal
    FP4 / bf16 ratio, 9 / 2.25 PFLOP/s)."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return 4.0 * float(json.load(f)["bf16_tflops"]), "measured bf16 burst x 4 (nominal ratio)"
    except Exception:
        return 4.0 * 1590.0, "fallback bf16 x 4"


def gemm_ops(mx, inputs, dev, reps=20):
    """The block-scaled MXFP4 GEMM D = A B^T (bf16 out) on the tensor cores:
    A pre-quantized; A quantized within the GEMM's launch, staged through
    scratch the library allocates (the default call: quant_gemm), through the
    caller's buffers (staged), or on chip in the GEMM's prologue (on_chip);
    quantize then GEMM, two launches (unfused). Median CUDA-event time of
    `reps`, L2 flushed before each. The library's block-scaled GEMM (cuBLAS
    through torch) on the same operands is timed beside it as context."""
    import torch
    F = torch.nn.functional
    flush = torch.empty(512 << 20, dtype=torch.uint8, device=dev)
    peak, peak_src = measured_fp4_peak()
    res = {"_peak_tflops": peak, "_peak_source": peak_src}
    for name, M, N, K in GEMM_SHAPES:
        a = inputs.normal_weight(M, K, seed=11, device=dev, std=1.0)
        w = inputs.normal_weight(N, K, seed=12, device=dev)
        bc, bs, _ = mx.quantize(w, mx.E2M1, mx.FLOOR | mx.MMA_SCALES)
        ac, as_, _ = mx.quantize(a, mx.E2M1, mx.FLOOR | mx.MMA_SCALES)
        d = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
        st = torch.zeros(1, dtype=torch.int32, device=dev)
        ac2, as2 = torch.empty_like(ac), torch.empty_like(as_)
        fns = {
            "quantize_a": lambda: mx.quantize(a, mx.E2M1, mx.FLOOR | mx.MMA_SCALES, out=(ac, as_, None)),
            "gemm": lambda: mx.gemm(ac, as_, bc, bs, out=d, status=st),
            "quant_gemm": lambda: mx.quant_gemm(a, bc, bs, mx.FLOOR, out=d, status=st),
            "staged_quant_gemm": lambda: mx.quant_gemm(a, bc, bs, mx.FLOOR, out=d, status=st,
                                                       a_out=(ac2, as2)),
            "on_chip_quant_gemm": lambda: mx.quant_gemm(a, bc, bs, mx.FLOOR, out=d, status=st,
                                                        on_chip=True),
            "unfused_quantize_then_gemm": lambda: (
                mx.quantize(a, mx.E2M1, mx.FLOOR | mx.MMA_SCALES, out=(ac, as_, None)),
                mx.gemm(ac, as_, bc, bs, out=d, status=st)),
        }
        r = {"M": M, "N": N, "K": K, "flop": 2.0 * M * N * K}
        for k, fn in fns.items():
            fn()
            torch.cuda.synchronize()
            ms = time_op(fn, reps, flush)
            r[k + "_us"] = round(ms * 1e3, 2)
            if k != "quantize_a":
                r[k + "_tflops"] = round(r["flop"] / (ms * 1e-3) / 1e12, 1)
        r["gemm_frac_of_peak"] = round(r["gemm_tflops"] / peak, 3)
        for k in ("quant_gemm", "staged_quant_gemm", "on_chip_quant_gemm"):
            r[k + "_vs_unfused"] = round(r["unfused_quantize_then_gemm_us"] / r[k + "_us"], 3)
        # the quantization's cost inside the fused call, as a share of the GEMM
        r["quant_gemm_overhead_of_gemm"] = round(r["quant_gemm_us"] / r["gemm_us"] - 1.0, 3)
        try:
            lib = lambda: F.scaled_mm(ac.view(torch.float4_e2m1fn_x2), bc.view(torch.float4_e2m1fn_x2).t(),
                                      as_.view(torch.float8_e8m0fnu), F.ScalingType.BlockWise1x32,
                                      bs.view(torch.float8_e8m0fnu), F.ScalingType.BlockWise1x32,
                                      swizzle_a=F.SwizzleType.SWIZZLE_32_4_4,
                                      swizzle_b=F.SwizzleType.SWIZZLE_32_4_4, output_dtype=torch.bfloat16)
            ref = lib()
            mx.gemm(ac, as_, bc, bs, out=d, status=st)
            torch.cuda.synchronize()
            r["context_library_gemm_us"] = round(time_op(lib, reps, flush) * 1e3, 2)
            r["context_library_gemm_bit_identical"] = bool(torch.equal(ref.view(torch.int16),
                                                                       d.view(torch.int16)))
        except Exception as e:   # the library path is context only
            r["context_library_gemm"] = f"unavailable: {str(e).splitlines()[0][:120]}"
        r["status"] = int(st.item())
        res[name] = r
        del a, w, bc, bs, ac, as_, ac2, as2, d
    del flush
    return res


def run_mx(args):
    import torch
    import torch.distributed as dist

    import fp8_quantization_mx_b200 as mx
    from fp8_quantization_mx_b200 import build as mxbuild
    from fp8_quantization_mx_b200 import inputs
    from fp8_quantization_mx_b200.sharding import max_over_ranks

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    if rank == 0:
        mxbuild.build()
    if world > 1:
        dist.barrier()
    mx.load_library()

    # each rank quantizes its own stack (weak scaling, no exchange)
    x = inputs.moe_w13(seed=4 + 1000 * rank, device=dev).view(-1, HIDDEN)
    codes = torch.empty(x.shape[0], HIDDEN // 2, dtype=torch.uint8, device=dev)
    scales = torch.empty(x.shape[0], HIDDEN // 32, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    rows, cols = x.shape
    sh = stream.cuda_stream
    xp, cp, sp = x.data_ptr(), codes.data_ptr(), scales.data_ptr()

    def step():
        st = mx.mx_quantize(xp, rows, cols, mx.E2M1, mx.FLOOR, cp, sp, None, sh)
        if st != 0:
            raise mx.MXError(st, "mx_quantize")

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clocks:
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        t_start.record(stream)
        for s, e in ev:
            s.record(stream)
            step()
            e.record(stream)
        t_end.record(stream)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
    total_ms = t_start.elapsed_time(t_end)
    launch_ms = sum(s.elapsed_time(e) for s, e in ev) / len(ev)
    if world > 1:
        total_ms, launch_ms = max_over_ranks([total_ms, launch_ms], dev)
    ms_per_step = total_ms / args.steps
    value = world * BYTES_STEP / (ms_per_step * 1e-3) / 1e9

    # end to end through the public API with host buffers (pinned in, pinned out)
    xh = x.cpu().pin_memory()
    hc = torch.empty(codes.shape, dtype=torch.uint8, pin_memory=True)
    hs = torch.empty(scales.shape, dtype=torch.uint8, pin_memory=True)
    e2e_steps = max(3, min(args.steps, 10))
    mx.quantize(xh, out=(hc, hs, None))
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        mx.quantize(xh, out=(hc, hs, None))
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1) / e2e_steps
    if world > 1:
        (e2e_ms,) = max_over_ranks([e2e_ms], dev)
    e2e = {"value": world * BYTES_STEP / (e2e_ms * 1e-3) / 1e9, "unit": "GB/s",
           "h2d_bytes_per_step": BYTES_IN, "d2h_bytes_per_step": BYTES_CODES + BYTES_SCALES,
           "ms_per_step": e2e_ms}
    del hc, hs

    ops = None
    if not args.no_ops and world == 1:
        ops = {"moe_w13_128x1536x2048": stack_ops(mx, x)}
        ops.update(other_ops(mx, inputs, dev))
        ops["gemm_mxfp4"] = gemm_ops(mx, inputs, dev)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = oracle_baseline(xh.view(torch.int16).numpy().view("uint16").reshape(-1, HIDDEN), inputs)
    del xh

    peak, peak_src = measured_peak()
    achieved = BYTES_STEP / (launch_ms * 1e-3) / 1e9
    traffic, traffic_src = profiled_traffic()
    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": max(3, args.warmup), "ms_per_step": ms_per_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f32", "data": "synthetic",
            "config": {"workload": WORKLOAD, "elements_per_gpu": N_ELEM,
                       "bytes_per_step_per_gpu": BYTES_STEP,
                       "l2": "input (805 MB) larger than L2 (126 MB); no flush between steps",
                       "parallelism": f"weak: {world} independent stacks, no data exchange"},
            "elements_per_s": world * N_ELEM / (ms_per_step * 1e-3),
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "peak_source": peak_src,
                         "frac_of_8000": achieved / 8000.0, "traffic": traffic,
                         "traffic_source": traffic_src, "kernel": "stream_kernel<quantize, E2M1, FLOOR>",
                         "launch_ms": launch_ms},
            "e2e": e2e,
            "gpu_launches": args.steps,
            "clocks": clocks.summary(),
        }
        if cpu is not None:
            line["cpu_baseline"] = cpu
        if ops is not None:
            line["ops"] = ops
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["mx", "reference"], default="mx")
    ap.add_argument("--no-ops", action="store_true", help="skip the per-op figures")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--profile-op", default=None,
                    help="run one op of the MoE-stack table, or gemm_{pre,fused,onchip}_MxNxK, "
                         "`--steps` times and print its figure (for profilers); no headline line")
    ap.add_argument("--profile-experts", type=int, default=32,
                    help="experts of the stack used by --profile-op (32: 201 MB of input, above L2)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args)
    if args.profile_op:
        return run_profile_op(args)
    return run_mx(args)


def run_profile_gemm(args, mx, inputs):
    """--profile-op gemm_{pre,fused,onchip}_MxNxK: `--steps` launches of the
    pre-quantized MXFP4 GEMM, the fused one (default form: staged through
    scratch) or the fused one with A quantized on chip, on the operands
    gemm_ops uses."""
    import torch
    kind, shape = args.profile_op.split("_")[1], args.profile_op.split("_")[2]
    M, N, K = (int(t) for t in shape.split("x"))
    dev = torch.device("cuda", 0)
    a = inputs.normal_weight(M, K, seed=11, device=dev, std=1.0)
    w = inputs.normal_weight(N, K, seed=12, device=dev)
    bc, bs, _ = mx.quantize(w, mx.E2M1, mx.FLOOR | mx.MMA_SCALES)
    ac, as_, _ = mx.quantize(a, mx.E2M1, mx.FLOOR | mx.MMA_SCALES)
    d = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
    fns = {"pre": lambda: mx.gemm(ac, as_, bc, bs, out=d),
           "fused": lambda: mx.quant_gemm(a, bc, bs, mx.FLOOR, out=d),
           "onchip": lambda: mx.quant_gemm(a, bc, bs, mx.FLOOR, out=d, on_chip=True)}
    fn = fns[kind]
    fn()
    torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record()
    for _ in range(args.steps):
        fn()
    e.record()
    e.synchronize()
    us = s.elapsed_time(e) / args.steps * 1e3
    print(json.dumps({"profile_op": args.profile_op, "us": round(us, 2),
                      "TFLOP/s": round(2.0 * M * N * K / us / 1e6, 1)}), flush=True)
    return 0


def run_profile_op(args):
    """One op of the MoE-stack table, alone (after the stack is generated), or
    one of the GEMMs (gemm_pre_MxNxK, gemm_fused_MxNxK, gemm_onchip_MxNxK)."""
    import torch
    import fp8_quantization_mx_b200 as mx
    from fp8_quantization_mx_b200 import build as mxbuild
    from fp8_quantization_mx_b200 import inputs
    mxbuild.build()
    mx.load_library()
    if args.profile_op.startswith("gemm_"):
        return run_profile_gemm(args, mx, inputs)
    x = inputs.moe_w13(experts=args.profile_experts, device="cuda").view(-1, HIDDEN)
    res = stack_ops(mx, x, reps=args.steps, only=args.profile_op)
    torch.cuda.synchronize()
    print(json.dumps({"profile_op": args.profile_op, **res[args.profile_op]}), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
