"""The host-side plan query (ll_plan) names the kernel a forward runs."""
import pytest
import torch

import rank_fp8_residual_b200 as ll
from synth_inputs import make_weights

pytestmark = pytest.mark.gpu

NAMES = {ll.LL_VARIANT_TC: "ll_tc_kernel", ll.LL_VARIANT_TC_PAIR: "ll_tc2_kernel",
         ll.LL_VARIANT_SMALL: "ll_main_kernel", ll.LL_VARIANT_STREAM: "ll_stream_kernel",
         ll.LL_VARIANT_FP8_SPLIT: "ll_f8_kernel", ll.LL_VARIANT_GEMV: "ll_gemv_kernel"}


@pytest.mark.parametrize("M,N", [(1, 2048), (16, 2048), (64, 2048), (100, 2048), (256, 2048), (300, 2048), (1024, 2048),
                                 (300, 4096), (1024, 4096)])
def test_plan_matches_launched_kernel(M, N):
    K, r = 1024, 64
    dev = torch.device("cuda")
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    B, A, Q, scale, bias = make_weights(K, N, r, seed=3)
    h = ll.ll_create(N, K, r, ll.LL_SCALE_PER_ROW)
    try:
        ll.ll_set_weights(h, A.to(dev), B.to(dev), Q.to(dev), scale.to(dev), bias.to(dev))
        x = torch.randn(M, K, device=dev).to(torch.bfloat16)
        y = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
        ll.ll_set_profiling(h, True)
        ll.ll_forward(h, x, y, M)
        torch.cuda.synchronize()
        names = [n for n, _ in ll.ll_kernel_times(h)]
        kernel, _, _ = ll.ll_plan(N, K, r, M, sms)
        assert names[-1] == NAMES[kernel]
        if kernel == ll.LL_VARIANT_FP8_SPLIT:
            assert names[:2] == ["ll_xsplit_kernel", "ll_lrdown_kernel"]
        elif kernel == ll.LL_VARIANT_GEMV:
            assert names[0] == "ll_gemv_t_kernel"
        else:
            assert names[0] == "ll_lrdown_kernel"
    finally:
        ll.ll_destroy(h)
