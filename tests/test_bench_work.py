"""The bench's algorithmic work per forward, against the configurations'
figures worked out from their shapes (flops 2M(KN + rK + rN); bytes: x, Q,
A, B, the scale ([N] per row or [1] per tensor), the bias and y, each once),
and which roofline bounds each configuration."""
import importlib.util
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    argv = sys.argv
    sys.argv = ["bench"]
    try:
        spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
        mod = importlib.util.module_from_spec(spec)
        spec.loader.exec_module(mod)
    finally:
        sys.argv = argv
    return mod


BENCH = _bench()


@pytest.mark.parametrize("name,gflop,mb", [
    ("tiny_m64_k256_n256_r16", 0.00944, 0.149),
    ("attn_m3630_k2048_n2048_r32", 31.40, 34.21),
    ("ffn_up_m3630_k2048_n8192_r64", 126.6, 92.48),
    ("ffn_down_m3630_k8192_n2048_r64", 126.6, 92.44),
    ("small_m1_k4096_n16384_r512", 0.155, 88.15),
    ("small_m16_k4096_n16384_r512", 2.48, 88.77),
    ("small_m64_k4096_n16384_r512", 9.93, 90.73),
])
def test_work_matches_config_table(name, gflop, mb):
    flops, bytes_, main_flops, main_bytes = BENCH.work_of(BENCH.WORKLOADS[name])
    assert flops / 1e9 == pytest.approx(gflop, rel=2e-3)
    assert bytes_ / 1e6 == pytest.approx(mb, rel=1e-3)
    w = BENCH.WORKLOADS[name]
    # The fused kernel's share drops the down-projection: its flops 2MrK and
    # the read of B (2rK bytes).
    assert flops - main_flops == pytest.approx(2.0 * w.M * w.r * w.K)
    assert bytes_ - main_bytes == pytest.approx(2.0 * w.r * w.K)


@pytest.mark.parametrize("name,bound", [
    ("attn_m3630_k2048_n2048_r32", "tensor"),
    ("ffn_up_m3630_k2048_n8192_r64", "tensor"),
    ("ffn_down_m3630_k8192_n2048_r64", "tensor"),
    ("sweep_m1024_k4096_n4096_r32", "tensor"),
    ("small_m1_k4096_n16384_r512", "hbm"),
    ("small_m64_k4096_n16384_r512", "hbm"),
])
def test_roofline_bound(name, bound):
    peaks = BENCH.FALLBACK_PEAKS
    ridge = peaks["bf16_tflops"] * 1e12 / (peaks["hbm_gbs"] * 1e9)
    _, _, main_flops, main_bytes = BENCH.work_of(BENCH.WORKLOADS[name])
    assert ("tensor" if main_flops / main_bytes >= ridge else "hbm") == bound


def test_recorded_traffic_follows_source_hash(tmp_path, monkeypatch):
    """A recorded capture counts only while the kernel's sources are the
    ones it was taken from."""
    name, kern = "attn_m3630_k2048_n2048_r32", "ll_tc_kernel"
    got = BENCH.recorded_traffic(kern, name)
    import json
    rec = json.load(open(os.path.join(ROOT, "profiles", "traffic.json")))
    entry = rec.get(name, {}).get(kern)
    if entry is None or entry["source_hash"] != BENCH.kernel_source_hash(kern):
        assert got is None
    else:
        assert got == entry["dram_bytes_per_launch"]
    monkeypatch.setattr(BENCH, "kernel_source_hash", lambda k: "0000000000000000")
    assert BENCH.recorded_traffic(kern, name) is None
