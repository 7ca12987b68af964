#!/usr/bin/env python
"""Benchmark of the LiteLinear forward ``ll_forward`` on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--impl ours|reference]

One step = one ``ll_forward`` (every kernel of the path) over one batch of
synthetic tokens for the named layer shape (default: the attention
projection of a 480x704x81 video latent, M=3630 tokens, K=N=2048, r=32).
Metric: algorithmic TFLOP/s, F = 2*M*(K*N + r*K + r*N) per step.

Timing: W untimed warm-up steps, then exactly K steps between a barrier +
device synchronise on both sides; each step is bracketed by CUDA events on
the launching stream and L2 is flushed between steps, outside the events,
by reading a 256 MiB buffer (a read leaves clean lines behind, so no
write-back of the flush lands inside the next timed step).  Multi-GPU (torchrun): each rank runs its own batch of
M tokens against its own copy of the factors (token-sharded replicas, no
data-path collective); the reported time is the max over ranks and the
value counts the tokens of all ranks (weak scaling).

Also reported on the same JSON line: ``e2e`` (same metric through
``ll_forward_host`` with pinned host buffers, the H2D copy of x and the
D2H copy of y inside each timed step), ``roofline`` for the dominant kernel
(per-kernel device times from the library's profiling mode), ``clocks``
(NVML samples taken during the timed region), ``gpu_launches``, and, on
rank 0 at N=1, ``cpu_baseline`` (the fp64 CPU oracle on a row sample) and
``configs``: every layer configuration (tiny, attention, the FFN pair as
the sum of up and down, the small batches M = 1, 16, 64, the 24 sweep
points), each device-timed in the same run with its dominant kernel's
roofline fraction, and the FP8-activation variant beside the bf16 path on
the large-M configurations.

``--impl reference`` times the CPU oracle instead (the reference arm of
this build) on the same workload, metric and unit.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from synth_inputs import SCALE_PER_ROW, WORKLOADS  # noqa: E402

DEFAULT_WORKLOAD = "attn_m3630_k2048_n2048_r32"
FLUSH_BYTES = 256 << 20


class L2Flush:
    """Evicts L2 between timed steps by reading a buffer twice the size of
    L2 (126 MB on B200).  A read leaves clean lines behind, so evicting them
    later costs no write-back inside the next timed step."""

    def __init__(self, device):
        import torch
        self._buf = torch.ones(FLUSH_BYTES // 4, dtype=torch.float32, device=device)
        self._out = torch.empty((), dtype=torch.float32, device=device)

    def __call__(self):
        import torch
        torch.sum(self._buf, dim=0, out=self._out)
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def work_of(w, M=None):
    M = w.M if M is None else M
    K, N, r = w.K, w.N, w.r
    flops = 2.0 * M * (K * N + r * K + r * N)
    scale_bytes = 4.0 * N if w.scale_mode == SCALE_PER_ROW else 4.0  # per-row [N] or per-tensor [1] fp32
    bytes_ = 2.0 * M * K + N * K + 2.0 * N * r + 2.0 * r * K + scale_bytes + 2.0 * N + 2.0 * M * N
    # the fused kernel (x Q^T and the up-projection; B is read by the
    # down-projection kernel only)
    main_flops = 2.0 * M * N * (K + r)
    main_bytes = bytes_ - 2.0 * r * K
    return flops, bytes_, main_flops, main_bytes


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


# Sources each kernel is compiled from: a recorded ncu capture stays valid
# while these files are unchanged.
KERNEL_SOURCES = {
    "ll_tc_kernel": ["ll_tc.cuh", "ll_kernels.cuh", "ptx.cuh"],
    "ll_tc2_kernel": ["ll_tc2.cuh", "ll_kernels.cuh", "ptx.cuh"],
    "ll_main_kernel": ["ll_kernels.cuh", "ptx.cuh"],
    "ll_lrdown_kernel": ["ll_kernels.cuh", "ptx.cuh"],
    "ll_stream_kernel": ["ll_stream.cuh", "ll_kernels.cuh", "ptx.cuh"],
    "ll_f8_kernel": ["ll_f8.cuh", "ll_kernels.cuh", "ptx.cuh"],
    "ll_xsplit_kernel": ["ll_f8.cuh", "ll_kernels.cuh", "ptx.cuh"],
    "ll_f8_stream_kernel": ["ll_f8_stream.cuh", "ll_kernels.cuh", "ptx.cuh"],
    "ll_gemv_kernel": ["ll_gemv.cuh", "ll_kernels.cuh", "ptx.cuh"],
    "ll_gemv_t_kernel": ["ll_gemv.cuh", "ll_kernels.cuh", "ptx.cuh"],
}


def kernel_source_hash(kernel):
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "rank_fp8_residual_b200", "csrc")
    names = KERNEL_SOURCES.get(kernel) or sorted(n for n in os.listdir(csrc) if n.endswith((".cu", ".cuh")))
    for n in names:
        with open(os.path.join(csrc, n), "rb") as f:
            h.update(n.encode() + f.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel, workload):
    """DRAM bytes per launch from a committed ncu capture, or None when the
    kernel's sources changed since the capture."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(p) as f:
            d = json.load(f)
    except (OSError, ValueError):
        return None
    e = d.get(workload, {}).get(kernel)
    if not e or e.get("source_hash") != kernel_source_hash(kernel):
        return None
    return e.get("dram_bytes_per_launch")


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML in a thread."""

    REASONS = {
        "gpu_idle": 0x1, "applications_clocks_setting": 0x2, "sw_power_cap": 0x4,
        "hw_slowdown": 0x8, "sync_boost": 0x10, "sw_thermal_slowdown": 0x20,
        "hw_thermal_slowdown": 0x40, "hw_power_brake_slowdown": 0x80,
        "display_clock_setting": 0x100,
    }

    def __init__(self, device_index, period_s=0.0):
        self.samples = []
        self.reasons = 0
        self.ok = False
        self.max_mhz = None
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            return
        self._t = threading.Thread(target=self._run, args=(period_s,), daemon=True)

    def _run(self, period):
        nv = self._nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                fn = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                    nv.nvmlDeviceGetCurrentClocksThrottleReasons
                self.reasons |= fn(self._h)
            except Exception:
                pass
            if period > 0:
                time.sleep(period)

    def start(self):
        if self.ok:
            self._t.start()

    def stop(self):
        if self.ok:
            self._stop.set()
            self._t.join()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0,
                    "source": "nvml unavailable" if not self.ok else "nvml"}
        names = [k for k, v in self.REASONS.items() if self.reasons & v and k != "gpu_idle"]
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": names, "samples": len(self.samples), "source": "nvml"}


def cpu_baseline(w, budget_s=8.0):
    """The fp64 oracle, as it stands, on a bounded row sample of the
    workload, in the bench's unit (algorithmic TFLOP/s)."""
    import oracle
    inp = w.inputs()
    probe = max(1, min(w.M, 16))
    rows = list(range(probe))
    t0 = time.perf_counter()
    oracle.forward_inputs(inp, rows=rows)
    dt = max(time.perf_counter() - t0, 1e-6)
    n = int(min(w.M, max(probe, probe * budget_s / dt)))
    step = max(1, w.M // n)
    rows = list(range(0, w.M, step))[:n]
    t0 = time.perf_counter()
    oracle.forward_inputs(inp, rows=rows)
    dt = time.perf_counter() - t0
    flops = work_of(w, M=len(rows))[0]
    return {"value": flops / dt / 1e12, "unit": "TFLOP/s", "cores": oracle.num_threads(),
            "kind": "oracle",
            "sample": f"{len(rows)} of {w.M} token rows (every {step}th), full N={w.N}, "
                      f"{dt:.2f} s wall"}


def config_of(w, world, variant):
    """The configuration both arms report (the same dict, so the two lines
    compare like with like)."""
    return {"workload": w.name, "M": w.M, "K": w.K, "N": w.N, "r": w.r,
            "scale_mode": "per_row" if w.scale_mode == SCALE_PER_ROW else "per_tensor",
            "global_tokens": world * w.M, "parallelism": f"token-sharded replicas x{world}",
            "variant": variant, "l2": "flushed between steps (256 MiB read, outside the step events)"}


def run_reference(args, w):
    """Reference arm: the CPU oracle timed step by step on a row sample."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import oracle
    inp = w.inputs()
    probe = list(range(min(w.M, 8)))
    t0 = time.perf_counter()
    oracle.forward_inputs(inp, rows=probe)
    per_row = max((time.perf_counter() - t0) / len(probe), 1e-7)
    # each step ~0.5 s so that warm-up + steps stay within a few minutes
    nrows = int(max(1, min(w.M, 0.5 / per_row)))
    stride = max(1, w.M // nrows)
    for i in range(args.warmup):
        oracle.forward_inputs(inp, rows=list(range(i % stride, w.M, stride))[:nrows])
    times = []
    for i in range(args.steps):
        rows = list(range(i % stride, w.M, stride))[:nrows]
        t0 = time.perf_counter()
        oracle.forward_inputs(inp, rows=rows)
        times.append(time.perf_counter() - t0)
    total = sum(times)
    flops = work_of(w, M=nrows)[0]
    value = args.steps * flops / total / 1e12
    sample = f"{nrows} of {w.M} token rows per step (stride {stride}), full N={w.N}"
    line = {
        "impl": "reference", "metric": "ll_forward TFLOP/s (algorithmic)", "value": value,
        "unit": "TFLOP/s", "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * total / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_of(w, args.gpus, args.variant),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": oracle.num_threads(),
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))
    return 0


VARIANT_NAMES = ("auto", "tc", "tc_pair", "small", "stream", "fp8_split", "fp8_act", "gemv")


def variant_id(ll, name):
    return getattr(ll, "LL_VARIANT_" + name.upper())


def roofline_of(w, kernel_ms, peaks, peak_src, fp8_act=False):
    """Roofline of the dominant kernel: algorithmic flops (tensor-bound) or
    bytes (HBM-bound) of that kernel / its event-timed duration.  The fused
    kernel's work is x Q^T and the up-projection, 2MN(K + r) flops and every
    compulsory byte but B's (read by the down-projection only).  The peak is
    the measured bf16 tensor rate, doubled for the one-term FP8 variant (e4m3
    operands: the nominal fp8 / bf16 ratio), or the measured copy bandwidth."""
    _, _, main_flops, main_bytes = work_of(w)
    dom = max(kernel_ms, key=kernel_ms.get)
    ms = kernel_ms[dom]
    t_peak = peaks["bf16_tflops"] * (2.0 if fp8_act else 1.0)
    if main_flops / (t_peak * 1e12) >= main_bytes / (peaks["hbm_gbs"] * 1e9):
        ach = main_flops / (ms * 1e-3) / 1e12
        src = ("e4m3 (2 x bf16 burst, nominal ratio)" if fp8_act else "bf16 burst") + f", of {peak_src}"
        roof = {"bound": "tensor", "achieved": ach, "peak": t_peak, "unit": "TFLOP/s", "frac": ach / t_peak,
                "peak_source": src}
    else:
        ach = main_bytes / (ms * 1e-3) / 1e9
        roof = {"bound": "hbm", "achieved": ach, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": ach / peaks["hbm_gbs"], "peak_source": f"copy bandwidth, of {peak_src}"}
    roof["kernel"] = dom
    roof["kernel_ms"] = ms
    return roof


def time_forward(ll, h, x, y, M, flush, stream, steps, warmup):
    """Median device time (ms) of one forward between CUDA events, L2
    flushed before each, and the per-kernel times of profiled forwards."""
    import torch
    ev = []
    with torch.cuda.stream(stream):
        for i in range(warmup + steps):
            flush()
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(stream)
            ll.ll_forward(h, x, y, M, stream)
            b.record(stream)
            if i >= warmup:
                ev.append((a, b))
    torch.cuda.synchronize()
    st = ll.ll_status(h)
    if st != ll.LL_OK:
        raise SystemExit(f"device status: {ll.status_string(st)}")
    ms = sorted(a.elapsed_time(b) for a, b in ev)
    ll.ll_set_profiling(h, True)
    per = {}
    with torch.cuda.stream(stream):
        for i in range(3):
            flush()
            ll.ll_forward(h, x, y, M, stream)
            for name, t in ll.ll_kernel_times(h):
                per.setdefault(name, []).append(t)
    ll.ll_set_profiling(h, False)
    torch.cuda.synchronize()
    return ms[len(ms) // 2], {k: statistics.median(v) for k, v in per.items()}


def run_configs(ll, dev, flush, stream, peaks, peak_src, steps=10, warmup=3):
    """Every layer configuration, device-timed in this run (AUTO dispatch),
    with the dominant kernel's roofline fraction; the FFN pair also as the
    sum of up and down; the FP8-activation variant beside the bf16 path on
    the large-M configurations.  Activations are drawn on the device from a
    seeded generator; L2 is flushed before every forward."""
    import torch
    from synth_inputs import FFN_PAIR, SMALL_BATCH
    names = (["tiny_m64_k256_n256_r16", "attn_m3630_k2048_n2048_r32"] + list(FFN_PAIR) + list(SMALL_BATCH) +
             sorted((n for n in WORKLOADS if n.startswith("sweep_")),
                    key=lambda n: (WORKLOADS[n].K, WORKLOADS[n].N, WORKLOADS[n].r, WORKLOADS[n].M)))
    fp8_act_on = {"attn_m3630_k2048_n2048_r32"} | set(FFN_PAIR)
    out, layers = {}, {}
    for n in names:
        w = WORKLOADS[n]
        key = (w.K, w.N, w.r, w.scale_mode, w.scale_value, w.scale_range)
        if key not in layers:
            for old in layers.values():
                old.close()
            layers.clear()
            B, A, Q, scale, bias = w.weights(seed=0)
            layer = ll.LiteLinearLayer(w.N, w.K, w.r, w.scale_mode)
            layer.set_weights(A.to(dev) if A is not None else None, B.to(dev) if B is not None else None,
                              Q.to(dev), scale.to(dev), bias.to(dev) if bias is not None else None)
            layers[key] = layer
        h = layers[key].handle
        ll.ll_reserve(h, w.M)
        g = torch.Generator(device=dev)
        g.manual_seed(7)
        x = torch.randn(w.M, w.K, generator=g, device=dev).to(torch.bfloat16)
        y = torch.empty(w.M, w.N, dtype=torch.bfloat16, device=dev)
        flops, bytes_, _, _ = work_of(w)
        for vname in ("auto", "fp8_act") if n in fp8_act_on else ("auto",):
            ll.ll_set_variant(h, variant_id(ll, vname))
            ms, kms = time_forward(ll, h, x, y, w.M, flush, stream, steps, warmup)
            roof = roofline_of(w, kms, peaks, peak_src, fp8_act=vname == "fp8_act")
            key_out = n if vname == "auto" else n + "@fp8_act"
            out[key_out] = {"us": round(ms * 1e3, 2), "tflops": round(flops / (ms * 1e-3) / 1e12, 1),
                            "gbs": round(bytes_ / (ms * 1e-3) / 1e9, 1), "kernel": roof["kernel"],
                            "kernel_us": round(roof["kernel_ms"] * 1e3, 2), "bound": roof["bound"],
                            "frac": round(roof["frac"], 3),
                            "kernels_us": {k: round(v * 1e3, 2) for k, v in kms.items()}}
        ll.ll_set_variant(h, ll.LL_VARIANT_AUTO)
        del x, y
    for old in layers.values():
        old.close()
    for suffix in ("", "@fp8_act"):
        up, down = out.get(FFN_PAIR[0] + suffix), out.get(FFN_PAIR[1] + suffix)
        if up and down:
            wu, wd = WORKLOADS[FFN_PAIR[0]], WORKLOADS[FFN_PAIR[1]]
            us = up["us"] + down["us"]
            fl = work_of(wu)[0] + work_of(wd)[0]
            mf = work_of(wu)[2] + work_of(wd)[2]
            kus = up["kernel_us"] + down["kernel_us"]
            peak = peaks["bf16_tflops"] * (2.0 if suffix else 1.0)
            out["ffn_pair_sum" + suffix] = {"us": round(us, 2), "tflops": round(fl / (us * 1e-6) / 1e12, 1),
                                            "kernel_us": round(kus, 2), "bound": "tensor",
                                            "frac": round(mf / (kus * 1e-6) / 1e12 / peak, 3)}
    return out


def run_page_suite(args):
    """The FFN shapes of the LiteLinear README's LTX-Video benchmark table
    (its "Performance Benchmark on shapes captured from LTX-Video" section):
    every (projection, M) row timed on its own, and the count-weighted total
    of the rows, which is the table's TOTAL row (in ms)."""
    import torch
    import rank_fp8_residual_b200 as ll
    from synth_inputs import PAGE_MICROBENCH, page_workload

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    flush = L2Flush(dev)
    stream = torch.cuda.Stream(device=dev)
    steps = max(1, min(args.steps, 30))
    rows, total_ms, total_flops_calls = [], 0.0, 0.0
    layers = {}
    for cfg, m, count in PAGE_MICROBENCH:
        w = WORKLOADS[page_workload(cfg, m, args.rank)]
        key = (w.K, w.N)
        if key not in layers:  # one layer per projection: the factors do not depend on M
            B, A, Q, scale, bias = w.weights(seed=0)
            layer = ll.LiteLinearLayer(w.N, w.K, w.r, w.scale_mode)
            layer.set_weights(A.to(dev), B.to(dev), Q.to(dev), scale.to(dev), bias.to(dev))
            layers[key] = layer
        h = layers[key].handle
        ll.ll_reserve(h, w.M)
        # Activations drawn on the device (the largest row block is 1.4 GB).
        g = torch.Generator(device=dev)
        g.manual_seed(1000 + m)
        x = torch.randn(w.M, w.K, generator=g, device=dev).to(torch.bfloat16)
        y = torch.empty(w.M, w.N, dtype=torch.bfloat16, device=dev)
        ev = []
        with torch.cuda.stream(stream):
            for i in range(args.warmup + steps):
                flush()
                a = torch.cuda.Event(enable_timing=True)
                b = torch.cuda.Event(enable_timing=True)
                a.record(stream)
                ll.ll_forward(h, x, y, w.M, stream)
                b.record(stream)
                if i >= args.warmup:
                    ev.append((a, b))
        torch.cuda.synchronize()
        st = ll.ll_status(h)
        if st != ll.LL_OK:
            raise SystemExit(f"device status: {ll.status_string(st)}")
        us = sorted(a.elapsed_time(b) * 1e3 for a, b in ev)
        med = us[len(us) // 2]
        flops = work_of(w)[0]
        rows.append({"cfg": cfg, "M": m, "K": w.K, "N": w.N, "count": count, "us": round(med, 2),
                     "tflops": round(flops / (med * 1e-6) / 1e12, 1)})
        total_ms += count * med * 1e-3
        total_flops_calls += count * flops
        del x, y
    for layer in layers.values():
        layer.close()
    line = {
        "metric": "LTX-Video FFN shapes, count-weighted total time", "value": total_ms, "unit": "ms",
        "higher_is_better": False, "n_gpus": 1, "steps": steps, "warmup": args.warmup,
        "dtype": "bf16", "data": "synthetic",
        "config": {"workload": f"page_microbench_r{args.rank}", "rank": args.rank,
                   "reading": "w1 = 4096 -> 16384, w2 = 16384 -> 4096 (K, N not on the page)",
                   "l2": "flushed between calls (256 MiB read, outside the events)", "rows": rows},
        "tflops_weighted": total_flops_calls / (total_ms * 1e-3) / 1e12,
        "vs_baseline": None,
    }
    print(json.dumps(line))
    return 0


def run_crossover_suite(args):
    """Every kernel variant against the token count M at K = 4096,
    N = 16384 and the given rank (the sweep's shape family): where the
    streaming, small-tile and fused large-M kernels cross over, and what the
    AUTO dispatch picks."""
    import torch
    import rank_fp8_residual_b200 as ll
    from synth_inputs import make_weights

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    flush = L2Flush(dev)
    stream = torch.cuda.Stream(device=dev)
    K, N, r = 4096, 16384, args.rank
    B, A, Q, scale, bias = make_weights(K, N, r, seed=0)
    layer = ll.LiteLinearLayer(N, K, r, SCALE_PER_ROW)
    layer.set_weights(A.to(dev), B.to(dev), Q.to(dev), scale.to(dev), bias.to(dev))
    h = layer.handle
    steps = max(1, min(args.steps, 30))
    variants = {"stream": ll.LL_VARIANT_STREAM, "small": ll.LL_VARIANT_SMALL, "tc": ll.LL_VARIANT_TC,
                "tc_pair": ll.LL_VARIANT_TC_PAIR, "auto": ll.LL_VARIANT_AUTO}
    points = []
    for M in (1, 16, 32, 64, 96, 128, 192, 256, 384, 512, 1024, 2048, 4096, 8192, 16384):
        ll.ll_reserve(h, M)
        g = torch.Generator(device=dev)
        g.manual_seed(2000 + M)
        x = torch.randn(M, K, generator=g, device=dev).to(torch.bfloat16)
        y = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
        row = {"M": M}
        for name, v in variants.items():
            if name == "stream" and M > 64:
                continue  # the streaming kernel serves M <= 64 only
            if name == "tc_pair" and M <= 64:
                continue
            ll.ll_set_variant(h, v)
            ev = []
            with torch.cuda.stream(stream):
                for i in range(args.warmup + steps):
                    flush()
                    a = torch.cuda.Event(enable_timing=True)
                    b = torch.cuda.Event(enable_timing=True)
                    a.record(stream)
                    ll.ll_forward(h, x, y, M, stream)
                    b.record(stream)
                    if i >= args.warmup:
                        ev.append((a, b))
            torch.cuda.synchronize()
            st = ll.ll_status(h)
            if st != ll.LL_OK:
                raise SystemExit(f"device status: {ll.status_string(st)}")
            us = sorted(a.elapsed_time(b) * 1e3 for a, b in ev)
            row[name] = round(us[len(us) // 2], 2)
        timed = {k: v for k, v in row.items() if k not in ("M", "auto")}
        row["fastest"] = min(timed, key=timed.get)
        points.append(row)
        del x, y
    layer.close()
    line = {"metric": "ll_forward time per variant against M", "value": None, "unit": "us",
            "higher_is_better": False, "n_gpus": 1, "steps": steps, "warmup": args.warmup,
            "dtype": "bf16", "data": "synthetic",
            "config": {"workload": f"crossover_k{K}_n{N}_r{r}", "l2": "flushed between calls",
                       "points": points}}
    print(json.dumps(line))
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-configs", action="store_true", help="skip the per-configuration timings")
    ap.add_argument("--variant", default="auto", choices=list(VARIANT_NAMES),
                    help="kernel variant (auto picks by token count)")
    ap.add_argument("--suite", default=None, choices=["page", "crossover"],
                    help="page: the README's LTX-Video FFN shapes, count-weighted total; "
                         "crossover: every kernel variant against M (one GPU)")
    ap.add_argument("--rank", type=int, default=64, choices=[32, 64], help="rank of the --suite shapes")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.suite == "page":
        return run_page_suite(args)
    if args.suite == "crossover":
        return run_crossover_suite(args)
    w = WORKLOADS[args.workload]
    if args.impl == "reference":
        return run_reference(args, w)

    import torch
    import rank_fp8_residual_b200 as ll

    from rank_fp8_residual_b200 import replicas
    rank, world, local_rank = replicas.rank_env()
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        replicas.init("nccl", device=dev)

    # Factors are shared (seed 0); each rank draws its own tokens.
    inp = w.inputs(seed=0)
    if rank != 0:
        from synth_inputs import make_x
        inp.x = make_x(w.M, w.K, seed=replicas.token_seed(rank))
    layer = ll.LiteLinearLayer(w.N, w.K, w.r, w.scale_mode)
    layer.set_weights(inp.A.to(dev) if inp.A is not None else None,
                      inp.B.to(dev) if inp.B is not None else None,
                      inp.Q.to(dev), inp.scale.to(dev),
                      inp.bias.to(dev) if inp.bias is not None else None)
    h = layer.handle
    ll.ll_set_variant(h, variant_id(ll, args.variant))
    ll.ll_reserve(h, w.M)
    x = inp.x.to(dev)
    y = torch.empty(w.M, w.N, dtype=torch.bfloat16, device=dev)
    flush = L2Flush(dev)
    stream = torch.cuda.Stream(device=dev)
    flops, bytes_, main_flops, main_bytes = work_of(w)

    barrier = replicas.barrier

    def max_over_ranks(v):
        return replicas.max_over_ranks(v, device=dev)

    # --------------------------------------------------- device-timed steps
    # The K steps are timed R times back to back (R from the warm-up's pace,
    # so that the timed region spans >= 50 ms and the NVML sampler sees it
    # many times); value and ms_per_step are the means over all R * K steps.
    with torch.cuda.stream(stream):
        w0 = torch.cuda.Event(enable_timing=True)
        w1 = torch.cuda.Event(enable_timing=True)
        for i in range(args.warmup):
            if i == 1:
                w0.record(stream)
            flush()
            ll.ll_forward(h, x, y, w.M, stream)
        w1.record(stream)
        torch.cuda.synchronize()
        est_ms = max(w0.elapsed_time(w1) / max(args.warmup - 1, 1), 1e-3)
        repeats = max(1, math.ceil(50.0 / (args.steps * est_ms)))
        repeats = int(max_over_ranks(float(repeats)))  # every rank times the same number of steps
        n_timed = repeats * args.steps
        ev0 = [torch.cuda.Event(enable_timing=True) for _ in range(n_timed)]
        ev1 = [torch.cuda.Event(enable_timing=True) for _ in range(n_timed)]
        launches = 0
        sampler = ClockSampler(local_rank)
        barrier()
        torch.cuda.synchronize()
        sampler.start()
        for i in range(n_timed):
            flush()
            ev0[i].record(stream)
            ll.ll_forward(h, x, y, w.M, stream)
            ev1[i].record(stream)
            launches += ll.ll_last_launch_count(h)
        torch.cuda.synchronize()
        barrier()
        sampler.stop()
    step_ms = [a.elapsed_time(b) for a, b in zip(ev0, ev1)]
    total_ms = max_over_ranks(sum(step_ms))
    st = ll.ll_status(h)
    if st != ll.LL_OK:
        raise SystemExit(f"device status after timing: {ll.status_string(st)}")
    value = replicas.aggregate_rate(flops, n_timed, total_ms * 1e-3, world) / 1e12

    # ------------------------------------------- end to end (host buffers)
    xh = inp.x.contiguous().pin_memory()
    yh = torch.empty(w.M, w.N, dtype=torch.bfloat16).pin_memory()
    e2e_steps = max(3, min(args.steps, 50))
    with torch.cuda.stream(stream):
        for _ in range(3):
            ll.ll_forward_host(h, xh.data_ptr(), yh.data_ptr(), w.M, stream)
        e0 = [torch.cuda.Event(enable_timing=True) for _ in range(e2e_steps)]
        e1 = [torch.cuda.Event(enable_timing=True) for _ in range(e2e_steps)]
        barrier()
        torch.cuda.synchronize()
        for i in range(e2e_steps):
            flush()
            e0[i].record(stream)
            ll.ll_forward_host(h, xh.data_ptr(), yh.data_ptr(), w.M, stream)
            e1[i].record(stream)
        torch.cuda.synchronize()
        barrier()
    e2e_ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in zip(e0, e1)))
    e2e_value = world * e2e_steps * flops / (e2e_ms * 1e-3) / 1e12

    # ------------------------------------ per-kernel times (profiling mode)
    ll.ll_set_profiling(h, True)
    prof_steps = max(3, min(args.steps, 50))
    per_kernel = {}
    with torch.cuda.stream(stream):
        for i in range(prof_steps + 2):
            flush()
            ll.ll_forward(h, x, y, w.M, stream)
            if i >= 2:
                for name, ms in ll.ll_kernel_times(h):
                    per_kernel.setdefault(name, []).append(ms)
    ll.ll_set_profiling(h, False)
    torch.cuda.synchronize()
    kernel_ms = {k: statistics.mean(v) for k, v in per_kernel.items()}
    dom = max(kernel_ms, key=kernel_ms.get)
    dom_ms = max_over_ranks(kernel_ms[dom])

    peaks, peak_src = load_peaks()
    roof = roofline_of(w, dict(kernel_ms, **{dom: dom_ms}), peaks, peak_src, fp8_act=args.variant == "fp8_act")
    roof["traffic"] = recorded_traffic(dom, w.name)
    roof["kernel_ms_all"] = kernel_ms

    line = {
        "metric": "ll_forward TFLOP/s (algorithmic)",
        "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": total_ms / n_timed, "higher_is_better": True,
        "timed_repeats": repeats, "timed_steps_total": n_timed,
        "scaling": "weak", "vs_baseline": None,
        # the arithmetic of the dominant kernel: bf16 x bf16 MMAs, or e4m3 x e4m3 (FP8-operand kernel)
        "dtype": "e4m3" if roof["kernel"] == "ll_f8_kernel" else "bf16", "data": "synthetic",
        "config": config_of(w, world, args.variant),
        "hbm_gbs_algorithmic": world * n_timed * bytes_ / (total_ms * 1e-3) / 1e9,
        "e2e": {"value": e2e_value, "unit": "TFLOP/s", "h2d_bytes_per_step": 2 * w.M * w.K,
                "d2h_bytes_per_step": 2 * w.M * w.N, "steps": e2e_steps,
                "api": "ll_forward_host (pinned host buffers)"},
        "gpu_launches": launches, "gpu_launches_per_step": launches // n_timed,
        "roofline": roof,
        "clocks": sampler.summary(),
    }
    layer.close()
    if rank == 0 and world == 1 and not args.no_configs:
        line["configs"] = run_configs(ll, dev, flush, stream, peaks, peak_src)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w)
    if world > 1:
        replicas.barrier()
        replicas.finalize()
    if rank == 0:
        print(json.dumps(line))
    return 0


if __name__ == "__main__":
    sys.exit(main())
