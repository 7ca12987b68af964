"""Parity of the FP8-operand streaming kernel (M <= 64, through the C ABI)
with the CPU oracle.

Up to 64 tokens the FP8-operand variants run ll_f8_stream_kernel: the
residual codes go from HBM straight into kind::f8f6f4 MMAs against the
per-token e4m3fn split of x, and the weight bytes are dealt out to the CTAs
in equal contiguous ranges, so most 128-feature tiles are finished from
fp32 partials of several CTAs.  LL_VARIANT_FP8_SPLIT is graded against the
exact oracle, LL_VARIANT_FP8_ACT against its FP8ACT mode; the bound is the
bf16 path's, per element: |y_gpu - y_ref| <= 8e-3*|y_ref| + 2e-3*RMS(y_ref).
"""
import pytest
import torch

import oracle
import rank_fp8_residual_b200 as ll
from synth_inputs import SCALE_PER_TENSOR, WORKLOADS, make_inputs

from llgpu import DeviceLayer, check, run

pytestmark = pytest.mark.gpu

FP8 = [ll.LL_VARIANT_FP8_SPLIT, ll.LL_VARIANT_FP8_ACT]
NAME = {ll.LL_VARIANT_FP8_SPLIT: "fp8-split", ll.LL_VARIANT_FP8_ACT: "fp8-act"}


def _mode(variant):
    return oracle.EXACT if variant == ll.LL_VARIANT_FP8_SPLIT else oracle.FP8ACT


def _full(inp, what, variant, epilogue=ll.LL_EPILOGUE_NONE):
    y = run(inp, variant, epilogue)
    ref = oracle.forward_inputs(inp, mode=_mode(variant), epilogue=epilogue)
    return check(y, ref, what=f"{what} [{NAME[variant]}]")


def _launched(inp, variant):
    d = DeviceLayer(inp, variant)
    try:
        ll.ll_set_profiling(d.h, True)
        d.forward(inp.x)
        torch.cuda.synchronize()
        return [n for n, _ in ll.ll_kernel_times(d.h)]
    finally:
        d.close()


@pytest.mark.parametrize("variant", FP8)
def test_runs_the_streaming_kernel(variant):
    names = _launched(make_inputs(40, 512, 1000, 40, seed=1), variant)
    assert names == ["ll_xsplit_kernel", "ll_lrdown_kernel", "ll_f8_stream_kernel"]
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    kernel, bt, _ = ll.ll_plan(1000, 512, 40, 40, sms, variant)
    assert kernel == variant and bt == 48


@pytest.mark.parametrize("variant", FP8)
@pytest.mark.parametrize("M", [1, 2, 15, 16, 17, 31, 33, 48, 63, 64])
def test_token_counts(M, variant):
    # 8 feature tiles of 11 weight units each over ~130 CTAs: nearly every
    # tile is finished from partials of several CTAs.
    _full(make_inputs(M, 1040, 1000, 40, scale_range=(1e-3, 3e-3), seed=100 + M), f"M={M}", variant)


@pytest.mark.parametrize("variant", FP8)
@pytest.mark.parametrize("M,K,N,r", [(64, 256, 256, 16), (7, 272, 264, 1), (50, 4096, 2048, 512),
                                     (33, 16, 8, 0), (20, 128, 136, 200), (64, 8192, 512, 64)])
def test_shapes(M, K, N, r, variant):
    _full(make_inputs(M, K, N, r, seed=M + K + N + r), f"{M}x{K}x{N} r{r}", variant)


@pytest.mark.parametrize("variant", FP8)
def test_tiny_config(variant):
    _full(WORKLOADS["tiny_m64_k256_n256_r16"].inputs(), "tiny", variant)


@pytest.mark.parametrize("variant", FP8)
@pytest.mark.parametrize("name", ["small_m1_k4096_n16384_r512", "small_m16_k4096_n16384_r512",
                                  "small_m64_k4096_n16384_r512"])
def test_small_batch_full(name, variant):
    _full(WORKLOADS[name].inputs(), name, variant)


@pytest.mark.parametrize("variant", FP8)
def test_rank_zero_and_residual_zero(variant):
    _full(make_inputs(64, 512, 520, 0, seed=2), "r=0", variant)
    _full(make_inputs(64, 512, 520, 64, seed=3, q_zero=True), "Q=0", variant)


@pytest.mark.parametrize("variant", FP8)
def test_per_tensor_scale_zero_and_negative_rows(variant):
    _full(make_inputs(30, 640, 392, 24, scale_mode=SCALE_PER_TENSOR, bias=False, seed=4), "per-tensor", variant)
    inp = make_inputs(30, 640, 392, 40, scale_range=(1e-3, 3e-3), seed=5)
    inp.scale[::7] = 0.0
    inp.scale[5] = -2e-3
    _full(inp, "zero-scale rows", variant)


@pytest.mark.parametrize("variant", FP8)
def test_gelu_epilogue(variant):
    _full(make_inputs(24, 1024, 1000, 32, seed=6), "GELU", variant, ll.LL_EPILOGUE_GELU_TANH)


@pytest.mark.parametrize("variant", FP8)
def test_repeated_calls_are_bitwise_identical(variant):
    """Split tiles are summed in CTA order whichever CTA arrives last."""
    inp = make_inputs(48, 2048, 2056, 64, seed=7)
    d = DeviceLayer(inp, variant)
    try:
        a = d.forward(inp.x)
        for _ in range(3):
            assert torch.equal(d.forward(inp.x), a)
    finally:
        d.close()


def test_split_matches_exact_streaming_kernel_within_bound():
    """The two-term split and the exact-widening streaming kernel agree with
    each other within the bound, on the small-batch shape at M = 16."""
    inp = WORKLOADS["small_m16_k4096_n16384_r512"].inputs()
    a = run(inp, ll.LL_VARIANT_FP8_SPLIT)
    b = run(inp, ll.LL_VARIANT_STREAM)
    check(a, b.to(torch.float64).numpy(), what="fp8-split vs stream")
