"""ll_forward_noalloc: the forward for callers that may not allocate device
memory (a host framework whose allocator owns the GPU's memory, a plug-in
that may only use the buffers it is handed, a loop that cannot stall on
cudaMalloc / cudaFree).  It takes every buffer from the caller and keeps
its intermediates in a static device array that all calls on a GPU share.

The checks run calls in a row through the C ABI, with different shapes, so
each call after the first starts on the previous call's left-over scratch
contents; each output must match the CPU oracle of
y = (x B^T) A^T + scale * (x Q^T) + bias (LiteLinear README, introduction)
within the bound the parity tests use:
|y - y_ref| <= 8e-3*|y_ref| + 2e-3*RMS(y_ref).  This file is named to be
collected last.
"""
import numpy as np
import pytest
import torch

import oracle
import rank_fp8_residual_b200 as ll
from synth_inputs import SCALE_PER_TENSOR, make_inputs

from llgpu import check

pytestmark = pytest.mark.gpu


def _noalloc(inp, M=None):
    dev = torch.device("cuda")
    M = inp.M if M is None else M
    x = inp.x.to(dev)
    A = inp.A.to(dev) if inp.A is not None else None
    B = inp.B.to(dev) if inp.B is not None else None
    Q = inp.Q.to(dev)
    scale = inp.scale.to(dev)
    bias = inp.bias.to(dev) if inp.bias is not None else None
    y = torch.full((M, inp.N), float("nan"), dtype=torch.bfloat16, device=dev)
    ll.ll_forward_noalloc(x, A, B, Q, scale, inp.scale_mode, bias, y, M, inp.N, inp.K, inp.r)
    torch.cuda.synchronize()
    return y.cpu()


def test_noalloc_matches_the_oracle_on_calls_in_a_row():
    cases = [
        (make_inputs(1100, 2048, 1032, 96, scale_range=(1e-3, 3e-3), seed=71), "split-K partials in use"),
        (make_inputs(77, 4096, 520, 48, scale_mode=SCALE_PER_TENSOR, bias=False, seed=72), "per-tensor scale"),
        (make_inputs(33, 256, 264, 0, scale_range=(1e-3, 3e-3), seed=74), "r = 0"),
        (make_inputs(300, 512, 392, 40, scale_range=(1e-3, 3e-3), seed=75), "after r = 0"),
    ]
    for inp, what in cases:
        check(_noalloc(inp), oracle.forward_inputs(inp), what=f"ll_forward_noalloc ({what})")


def test_noalloc_rejects_requests_beyond_its_scratch():
    r, K, N = 512, 64, 64
    M = (ll.LL_NOALLOC_SCRATCH_BYTES - 256) // (4 * r) + 1  # one row more than the scratch holds
    inp = make_inputs(M, K, N, r, seed=73)
    dev = torch.device("cuda")
    x = inp.x.to(dev)
    y = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
    A, B, Q, scale = inp.A.to(dev), inp.B.to(dev), inp.Q.to(dev), inp.scale.to(dev)
    with pytest.raises(ll.LLError) as e:
        ll.ll_forward_noalloc(x, A, B, Q, scale, inp.scale_mode, None, y, M, N, K, r)
    assert e.value.code == ll.LL_ERR_SCRATCH_LIMIT
    # One row fewer fits: its values, on a sample of rows that includes the
    # last ones, against the oracle.
    y.fill_(float("nan"))
    ll.ll_forward_noalloc(x, A, B, Q, scale, inp.scale_mode, None, y, M - 1, N, K, r)
    torch.cuda.synchronize()
    rows = sorted(set(np.random.default_rng(73).choice(M - 1, 200, replace=False).tolist()) | {0, M - 3, M - 2})
    inp.bias = None
    check(y[rows].cpu(), oracle.forward_inputs(inp, rows=rows), what="one row under the scratch limit")
    assert torch.isnan(y[M - 1].float()).all()  # the last row was not asked for


def test_noalloc_rejects_overlap_with_an_input():
    inp = make_inputs(64, 256, 256, 32, seed=76)
    dev = torch.device("cuda")
    x, A, B, Q = inp.x.to(dev), inp.A.to(dev), inp.B.to(dev), inp.Q.to(dev)
    scale, bias = inp.scale.to(dev), inp.bias.to(dev)
    big = torch.empty(48 * 1024, dtype=torch.bfloat16, device=dev)  # 96 KB
    y = big[: 64 * 256].view(64, 256)                                  # bytes 0 .. 32 KB
    Qalias = big.view(torch.uint8)[16384:16384 + 256 * 256].view(256, 256)  # starts inside y
    Qalias.copy_(Q)
    with pytest.raises(ll.LLError) as e:
        ll.ll_forward_noalloc(x, A, B, Qalias, scale, inp.scale_mode, bias, y, 64, 256, 256, 32)
    assert e.value.code == ll.LL_ERR_INVALID_ARG
