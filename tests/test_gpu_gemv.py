"""Parity of the CUDA-core GEMV variant (M <= 4, through the C ABI) with
the exact CPU oracle of y = (x B^T) A^T + scale * (x Q^T) + bias (LiteLinear
README, introduction), per element |err| <= 8e-3*|y_ref| + 2e-3*RMS(y_ref)
with RMS over the whole output of the call.
"""
import pytest
import torch

import oracle
import rank_fp8_residual_b200 as ll
from synth_inputs import SCALE_PER_TENSOR, WORKLOADS, make_inputs

from llgpu import DeviceLayer, check, run

pytestmark = pytest.mark.gpu

G = ll.LL_VARIANT_GEMV


def _full(inp, what, epilogue=ll.LL_EPILOGUE_NONE):
    y = run(inp, G, epilogue)
    return check(y, oracle.forward_inputs(inp, epilogue=epilogue), what=f"{what} [gemv]")


def _launched(inp):
    d = DeviceLayer(inp, G)
    try:
        ll.ll_set_profiling(d.h, True)
        d.forward(inp.x)
        torch.cuda.synchronize()
        return [n for n, _ in ll.ll_kernel_times(d.h)]
    finally:
        d.close()


def test_runs_the_gemv_kernels():
    assert _launched(make_inputs(3, 512, 264, 40, seed=1)) == ["ll_gemv_t_kernel", "ll_gemv_kernel"]
    assert _launched(make_inputs(2, 512, 264, 0, seed=1)) == ["ll_gemv_kernel"]
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    assert ll.ll_plan(16384, 4096, 512, 4, sms, G)[:2] == (G, 4)
    # x no longer fits beside the load ring, or more than 4 tokens: SMALL
    assert ll.ll_plan(1024, 12800, 64, 4, sms, G)[0] == ll.LL_VARIANT_SMALL
    assert ll.ll_plan(1024, 1024, 64, 5, sms, G)[0] == ll.LL_VARIANT_SMALL


@pytest.mark.parametrize("M", [1, 2, 3, 4])
@pytest.mark.parametrize("K,N,r", [(272, 264, 40), (1040, 1000, 64), (4096, 2056, 512), (16, 8, 1)])
def test_shapes(M, K, N, r):
    _full(make_inputs(M, K, N, r, scale_range=(1e-3, 3e-3), seed=M * 7 + K + r), f"M={M} {K}x{N} r{r}")


@pytest.mark.parametrize("name", ["small_m1_k4096_n16384_r512"])
def test_small_batch_full(name):
    _full(WORKLOADS[name].inputs(), name)


@pytest.mark.parametrize("M", [1, 4])
def test_small_batch_shape_at_m(M):
    w = WORKLOADS["small_m1_k4096_n16384_r512"]
    _full(make_inputs(M, w.K, w.N, w.r, scale_mode=SCALE_PER_TENSOR, seed=50 + M), f"small batch M={M}")


def test_widest_x_that_fits():
    _full(make_inputs(4, 12288, 520, 32, seed=3), "M=4 K=12288")


def test_rank_zero_residual_zero_and_scales():
    _full(make_inputs(4, 512, 520, 0, seed=4), "r=0")
    _full(make_inputs(4, 512, 520, 64, seed=5, q_zero=True), "Q=0")
    inp = make_inputs(3, 640, 392, 40, scale_range=(1e-3, 3e-3), seed=6)
    inp.scale[::7] = 0.0
    inp.scale[5] = -2e-3
    _full(inp, "zero-scale rows")
    _full(make_inputs(2, 640, 392, 24, scale_mode=SCALE_PER_TENSOR, bias=False, seed=7), "per-tensor, no bias")


def test_gelu_epilogue():
    _full(make_inputs(4, 1024, 1000, 32, seed=8), "GELU", ll.LL_EPILOGUE_GELU_TANH)


def test_repeated_calls_are_bitwise_identical():
    inp = make_inputs(4, 2048, 2056, 64, seed=9)
    d = DeviceLayer(inp, G)
    try:
        a = d.forward(inp.x)
        for _ in range(2):
            assert torch.equal(d.forward(inp.x), a)
    finally:
        d.close()
