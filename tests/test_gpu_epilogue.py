"""Fused epilogue activations through the C ABI against the oracle: GELU
(tanh form) on every kernel variant, and GEGLU (h * gelu(g) over the two
halves of the output, LiteLinear README "Usage": the GEGLU projection of the
LTX feed-forward) on the FP8-operand kernel, with the bound of the parity
tests on the activated output:
|err| <= 8e-3*|y_ref| + 2e-3*RMS(y_ref)."""
import pytest
import torch

import oracle
import rank_fp8_residual_b200 as ll
from synth_inputs import SCALE_PER_TENSOR, make_inputs

from llgpu import DeviceLayer, check, run

pytestmark = pytest.mark.gpu

GELU, GEGLU = ll.LL_EPILOGUE_GELU_TANH, ll.LL_EPILOGUE_GEGLU_TANH


def _mode(v):
    return oracle.FP8ACT if v == ll.LL_VARIANT_FP8_ACT else oracle.EXACT


@pytest.mark.parametrize("variant,M", [(ll.LL_VARIANT_TC, 600), (ll.LL_VARIANT_SMALL, 300), (ll.LL_VARIANT_TC_PAIR, 200),
                                       (ll.LL_VARIANT_STREAM, 40), (ll.LL_VARIANT_FP8_SPLIT, 600),
                                       (ll.LL_VARIANT_FP8_ACT, 600), (ll.LL_VARIANT_AUTO, 3000)])
def test_gelu_on_every_variant(variant, M):
    # outputs of order one so that GELU's curved part is exercised
    inp = make_inputs(M, 512, 520, 48, scale_range=(1e-2, 3e-2), seed=200 + M)
    y = run(inp, variant, GELU)
    check(y, oracle.forward_inputs(inp, mode=_mode(variant), epilogue=oracle.EPILOGUE_GELU_TANH),
          what=f"GELU, variant {variant}")


@pytest.mark.parametrize("variant", [ll.LL_VARIANT_AUTO, ll.LL_VARIANT_FP8_SPLIT, ll.LL_VARIANT_FP8_ACT])
@pytest.mark.parametrize("M,K,N,r", [(1, 256, 512, 16), (300, 1024, 1024, 40), (3630, 2048, 2048, 64)])
def test_geglu(M, K, N, r, variant):
    inp = make_inputs(M, K, N, r, scale_range=(1e-2, 3e-2), seed=300 + M)
    y = run(inp, variant, GEGLU)
    assert y.shape == (M, N // 2)
    check(y, oracle.forward_inputs(inp, mode=_mode(variant), epilogue=oracle.EPILOGUE_GEGLU_TANH),
          what=f"GEGLU {M}x{K}x{N} r{r}, variant {variant}")


def test_geglu_per_tensor_scale_without_bias():
    inp = make_inputs(257, 512, 768, 24, scale_mode=SCALE_PER_TENSOR, scale_value=2e-2, bias=False, seed=310)
    check(run(inp, ll.LL_VARIANT_AUTO, GEGLU),
          oracle.forward_inputs(inp, epilogue=oracle.EPILOGUE_GEGLU_TANH), what="GEGLU per-tensor")


def test_geglu_rules():
    inp = make_inputs(64, 256, 512, 16, seed=320)
    h = ll.ll_create(520, 256, 16, ll.LL_SCALE_PER_ROW)
    try:
        with pytest.raises(ll.LLError) as e:  # N % 256 != 0
            ll.ll_set_epilogue(h, GEGLU)
        assert e.value.code == ll.LL_ERR_UNSUPPORTED
        with pytest.raises(ll.LLError) as e:
            ll.ll_set_epilogue(h, 7)
        assert e.value.code == ll.LL_ERR_INVALID_ARG
    finally:
        ll.ll_destroy(h)
    d = DeviceLayer(inp)
    try:
        ll.ll_set_epilogue(d.h, GEGLU)  # the weights were stored in the plain order
        x = inp.x.cuda()
        y = torch.empty(64, 256, dtype=torch.bfloat16, device="cuda")
        with pytest.raises(ll.LLError) as e:
            ll.ll_forward(d.h, x, y, 64)
        assert e.value.code == ll.LL_ERR_NOT_READY
        ll.ll_set_weights(d.h, d.A, d.B, d.Q, d.scale, d.bias)
        ll.ll_set_variant(d.h, ll.LL_VARIANT_TC)
        with pytest.raises(ll.LLError) as e:  # GEGLU runs on the FP8-operand kernel only
            ll.ll_forward(d.h, x, y, 64)
        assert e.value.code == ll.LL_ERR_UNSUPPORTED
        ll.ll_set_variant(d.h, ll.LL_VARIANT_AUTO)
        ll.ll_forward(d.h, x, y, 64)
        torch.cuda.synchronize()
        check(y.cpu(), oracle.forward_inputs(inp, epilogue=oracle.EPILOGUE_GEGLU_TANH), what="GEGLU after re-set")
    finally:
        d.close()
