"""Pins for the oracle's epilogue activations (GELU in its tanh form, and
GEGLU over the two halves of the output; LiteLinear README, "Usage": the
GEGLU projection of the LTX feed-forward routed through LiteLinear) against
torch's own GELU and closed forms."""
import numpy as np
import torch

import oracle


def test_gelu_matches_torch_tanh_gelu():
    v = np.concatenate([np.linspace(-12, 12, 4001), np.random.default_rng(0).standard_normal(2000) * 3])
    ref = torch.nn.functional.gelu(torch.from_numpy(v), approximate="tanh").numpy()
    # equal up to the rounding order of the two binary64 evaluations
    np.testing.assert_allclose(oracle.gelu_tanh(v), ref, rtol=1e-13, atol=1e-15)


def test_gelu_closed_forms():
    g = oracle.gelu_tanh
    assert g(np.array([0.0]))[0] == 0.0
    v = np.linspace(-30, 30, 601)
    # gelu(v) - gelu(-v) = v exactly in the reals (the tanh terms cancel)
    np.testing.assert_allclose(g(v) - g(-v), v, rtol=0, atol=1e-12)
    assert abs(g(np.array([30.0]))[0] - 30.0) < 1e-12 and abs(g(np.array([-30.0]))[0]) < 1e-12


def test_geglu_halves():
    rng = np.random.default_rng(1)
    y = rng.standard_normal((5, 8))
    ref = y[:, :4] * torch.nn.functional.gelu(torch.from_numpy(y[:, 4:]), approximate="tanh").numpy()
    np.testing.assert_allclose(oracle.apply_epilogue(y, oracle.EPILOGUE_GEGLU_TANH), ref, rtol=1e-14)
    assert oracle.apply_epilogue(y, oracle.EPILOGUE_NONE) is y
