"""The decomposition step on the GPU (LiteLinear README, "Usage":
LiteLinear.from_dense): the residual's e4m3fn codes and scales from
ll_quantize_residual, bit for bit against the oracle on the same W, A, B
(both take every rounding decision in the same precision), and a layer
built by from_dense checked against the oracle and against its weight.
"""
import numpy as np
import pytest
import torch

import oracle
import rank_fp8_residual_b200 as ll
from synth_inputs import make_x, to_numpy_bits

from llgpu import check

pytestmark = pytest.mark.gpu


def _factors(N, K, r, seed):
    g = torch.Generator().manual_seed(seed)
    W = torch.randn(N, K, generator=g).to(torch.bfloat16)
    A = (0.5 * torch.randn(N, r, generator=g)).to(torch.bfloat16) if r else None
    B = torch.randn(r, K, generator=g).to(torch.bfloat16) if r else None
    return W, A, B


@pytest.mark.parametrize("mode", [ll.LL_SCALE_PER_ROW, ll.LL_SCALE_PER_TENSOR])
@pytest.mark.parametrize("N,K,r", [(8, 16, 1), (64, 272, 0), (300, 1024, 40), (129, 4096, 512)])
def test_residual_codes_match_oracle(N, K, r, mode):
    W, A, B = _factors(N, K, r, seed=N + K + r)
    if N >= 64:
        W[5] = 0.0          # a row whose residual is A B alone
        W[7] *= 1000.0      # a row far above the others
    dev = torch.device("cuda")
    Q = torch.empty(N, K, dtype=torch.uint8, device=dev)
    s = torch.empty(N if mode == ll.LL_SCALE_PER_ROW else 1, dtype=torch.float32, device=dev)
    ll.ll_quantize_residual(W.to(dev), A.to(dev) if A is not None else None, B.to(dev) if B is not None else None,
                            N, K, r, mode, Q, s)
    torch.cuda.synchronize()
    Q_ref, s_ref = oracle.residual_quant(to_numpy_bits(W), to_numpy_bits(A), to_numpy_bits(B), mode)
    assert np.array_equal(s.cpu().numpy(), s_ref)
    assert np.array_equal(Q.cpu().numpy(), Q_ref)


def test_from_dense_layer_matches_oracle_and_weight():
    """W = (rank-32 part) + noise: the layer from from_dense computes the
    oracle's forward of its own factors, and A B + scale * Q reproduces W
    within half an e4m3fn step of the residual."""
    N, K, r, M = 512, 1024, 32, 300
    g = torch.Generator().manual_seed(9)
    L = torch.randn(N, r, generator=g) @ torch.randn(r, K, generator=g) / r ** 0.5
    W = (L + 0.05 * torch.randn(N, K, generator=g)).to(torch.bfloat16)
    dev = torch.device("cuda")
    A, B, Q, s = ll.from_dense(W.to(dev), r)
    layer = ll.LiteLinearLayer(N, K, r, ll.LL_SCALE_PER_ROW)
    try:
        layer.set_weights(A, B, Q, s, None)
        x = make_x(M, K, seed=9)
        y = layer.forward(x.to(dev)).cpu()
    finally:
        layer.close()
    Ab, Bb, Qb, sb = (to_numpy_bits(t.cpu()) for t in (A, B, Q, s))
    check(y, oracle.forward(to_numpy_bits(x), Bb, Ab, Qb, sb, ll.LL_SCALE_PER_ROW), what="from_dense layer")
    a = A.cpu().to(torch.float64).numpy()
    b = B.cpu().to(torch.float64).numpy()
    w = W.to(torch.float64).numpy()
    R = w - a @ b
    dq = torch.from_numpy(Qb).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    sv = sb.astype(np.float64)[:, None]
    bound = sv * np.maximum(2.0 ** -4 * np.abs(R / sv), 2.0 ** -10) * (1 + 1e-6) + 1e-12
    assert np.all(np.abs(a @ b + sv * dq - w) <= bound)
    # the SVD took the low-rank part: the residual is the noise, far below W
    assert np.sqrt(np.mean(R ** 2)) < 0.1 * np.sqrt(np.mean(w ** 2))
