"""Failure detection without a GPU fault: every device-side wait of the
kernels is bounded.  With the debug switch that makes the TMA producers
issue nothing, the consumers' waits run out after the (short) limit, the
kernels record LL_ERR_DEVICE_TIMEOUT in the handle's status word and
return, and the same handle then computes a correct forward: the CUDA
context stays usable and no state (status word, tile counters, split-K
counters) is left behind."""
import pytest
import torch

import oracle
import rank_fp8_residual_b200 as ll
from synth_inputs import make_inputs

from llgpu import DeviceLayer, check

pytestmark = pytest.mark.gpu

CASES = [(ll.LL_VARIANT_TC, 600), (ll.LL_VARIANT_SMALL, 100), (ll.LL_VARIANT_STREAM, 40),
         (ll.LL_VARIANT_TC_PAIR, 600), (ll.LL_VARIANT_AUTO, 3000), (ll.LL_VARIANT_FP8_SPLIT, 600),
         (ll.LL_VARIANT_FP8_ACT, 300)]


@pytest.mark.parametrize("variant,M", CASES)
def test_withheld_loads_time_out_and_the_handle_recovers(variant, M):
    inp = make_inputs(M, 512, 520, 64, seed=90 + M)
    d = DeviceLayer(inp, variant)
    try:
        x = inp.x.cuda()
        y = torch.empty(M, inp.N, dtype=torch.bfloat16, device="cuda")
        ll.ll_set_debug(d.h, True, 1_000_000)  # waits give up after about 1 ms
        ll.ll_forward(d.h, x, y, M)
        torch.cuda.synchronize()
        assert ll.ll_status(d.h) == ll.LL_ERR_DEVICE_TIMEOUT
        assert ll.ll_status(d.h) == ll.LL_OK  # reading the status clears it
        ll.ll_set_debug(d.h, False, 2_000_000_000)
        for _ in range(2):  # the counters the timed-out launch used are back at zero
            y2 = d.forward(inp.x)
            mode = oracle.FP8ACT if variant == ll.LL_VARIANT_FP8_ACT else oracle.EXACT
            check(y2.cpu(), oracle.forward_inputs(inp, mode=mode), what=f"after timeout, variant {variant}")
    finally:
        d.close()
