"""ll_forward_noalloc: the forward for callers that may not allocate device
memory (a host framework whose allocator owns the GPU's memory, a plug-in
that may only use the buffers it is handed, a loop that cannot stall on
cudaMalloc / cudaFree).  It takes every buffer from the caller and keeps
its intermediates in a static device array that all calls on a GPU share.

The check runs two calls in a row, through the C ABI, with different
shapes, so the second call starts on the first call's left-over scratch
contents; each must match the handle-based ll_forward within the bound the
parity tests use: |y - y_ref| <= 8e-3*|y_ref| + 2e-3*RMS(y_ref), with
y_ref = ll_forward's output.  This file is named to be collected last.
"""
import pytest
import torch

import rank_fp8_residual_b200 as ll
from synth_inputs import SCALE_PER_TENSOR, make_inputs

from llgpu import DeviceLayer, check

pytestmark = pytest.mark.gpu


def _noalloc(inp):
    dev = torch.device("cuda")
    x = inp.x.to(dev)
    A = inp.A.to(dev) if inp.A is not None else None
    B = inp.B.to(dev) if inp.B is not None else None
    Q = inp.Q.to(dev)
    scale = inp.scale.to(dev)
    bias = inp.bias.to(dev) if inp.bias is not None else None
    y = torch.full((inp.M, inp.N), float("nan"), dtype=torch.bfloat16, device=dev)
    ll.ll_forward_noalloc(x, A, B, Q, scale, inp.scale_mode, bias, y, inp.M, inp.N, inp.K, inp.r)
    torch.cuda.synchronize()
    return y.cpu()


def _existing(inp):
    d = DeviceLayer(inp)
    try:
        return d.forward(inp.x).cpu()
    finally:
        d.close()


def test_noalloc_matches_ll_forward_on_two_calls_in_a_row():
    first = make_inputs(1100, 2048, 1032, 96, scale_range=(1e-3, 3e-3), seed=71)  # split-K partials in use
    second = make_inputs(77, 4096, 520, 40 + 8, scale_mode=SCALE_PER_TENSOR, bias=False, seed=72)
    for inp, what in [(first, "first call"), (second, "second call")]:
        y_na = _noalloc(inp)
        y_ref = _existing(inp).to(torch.float64).numpy()
        check(y_na, y_ref, what=f"ll_forward_noalloc {what} vs ll_forward")


def test_noalloc_rejects_requests_beyond_its_scratch():
    r = 512
    M = (ll.LL_NOALLOC_SCRATCH_BYTES - 256) // (4 * r) + 1  # one row more than the scratch holds
    inp = make_inputs(8, 64, 64, r, seed=73)
    dev = torch.device("cuda")
    x = torch.zeros(M, 64, dtype=torch.bfloat16, device=dev)
    y = torch.empty(M, 64, dtype=torch.bfloat16, device=dev)
    with pytest.raises(ll.LLError) as e:
        ll.ll_forward_noalloc(x, inp.A.to(dev), inp.B.to(dev), inp.Q.to(dev), inp.scale.to(dev), inp.scale_mode,
                              None, y, M, 64, 64, r)
    assert e.value.code == ll.LL_ERR_SCRATCH_LIMIT
    # one row fewer fits
    ll.ll_forward_noalloc(x, inp.A.to(dev), inp.B.to(dev), inp.Q.to(dev), inp.scale.to(dev), inp.scale_mode,
                          None, y, M - 1, 64, 64, r)
    torch.cuda.synchronize()
    assert torch.all(torch.isfinite(y[:M - 1].float()))
