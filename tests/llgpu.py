"""Helpers for the GPU tests: run the CUDA library through its C ABI on a
synth_inputs.LayerInputs and compare with the oracle."""
from __future__ import annotations

import numpy as np
import torch

import oracle
import rank_fp8_residual_b200 as ll


class DeviceLayer:
    """Library handle with the layer's factors uploaded."""

    def __init__(self, inp, variant=ll.LL_VARIANT_AUTO):
        self.inp = inp
        self.h = ll.ll_create(inp.N, inp.K, inp.r, inp.scale_mode)
        ll.ll_set_variant(self.h, variant)
        dev = torch.device("cuda")
        self.A = inp.A.to(dev) if inp.A is not None else None
        self.B = inp.B.to(dev) if inp.B is not None else None
        self.Q = inp.Q.to(dev)
        self.scale = inp.scale.to(dev)
        self.bias = inp.bias.to(dev) if inp.bias is not None else None
        ll.ll_set_weights(self.h, self.A, self.B, self.Q, self.scale, self.bias)

    def forward(self, x_cpu, stream=None):
        x = x_cpu.to("cuda")
        y = torch.empty(x.shape[0], self.inp.N, dtype=torch.bfloat16, device="cuda")
        ll.ll_forward(self.h, x, y, x.shape[0], stream)
        torch.cuda.synchronize()
        st = ll.ll_status(self.h)
        assert st == ll.LL_OK, ll.status_string(st)
        return y

    def close(self):
        ll.ll_destroy(self.h)


def run(inp, variant=ll.LL_VARIANT_AUTO):
    d = DeviceLayer(inp, variant)
    try:
        return d.forward(inp.x).cpu()
    finally:
        d.close()


def check(y_gpu: torch.Tensor, y_ref: np.ndarray, rms: float | None = None, what: str = ""):
    """Per-element bound |err| <= 8e-3*|y_ref| + 2e-3*RMS(y_ref)."""
    y = y_gpu.to(torch.float64).numpy()
    assert y.shape == y_ref.shape, (y.shape, y_ref.shape)
    assert np.all(np.isfinite(y)), f"{what}: non-finite output"
    bound = oracle.tolerance_bound(y_ref, rms)
    err = np.abs(y - y_ref)
    ratio = err / np.maximum(bound, 1e-300)
    nfail = int(np.count_nonzero(err > bound))
    worst = np.unravel_index(int(np.argmax(ratio)), ratio.shape) if ratio.size else None
    msg = (f"{what}: {nfail} of {err.size} elements out of bound; max err/bound "
           f"{float(ratio.max()) if ratio.size else 0:.3g} at {worst}: gpu {y[worst] if worst else None} "
           f"ref {y_ref[worst] if worst else None}")
    assert nfail == 0, msg
    return float(ratio.max()) if ratio.size else 0.0
