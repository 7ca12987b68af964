"""Helpers for the GPU tests: run the CUDA library through its C ABI on a
synth_inputs.LayerInputs and compare with the oracle."""
from __future__ import annotations

import math

import numpy as np
import torch

import oracle
import rank_fp8_residual_b200 as ll


class DeviceLayer:
    """Library handle with the layer's factors uploaded."""

    def __init__(self, inp, variant=ll.LL_VARIANT_AUTO, epilogue=ll.LL_EPILOGUE_NONE):
        self.inp = inp
        self.h = ll.ll_create(inp.N, inp.K, inp.r, inp.scale_mode)
        ll.ll_set_variant(self.h, variant)
        ll.ll_set_epilogue(self.h, epilogue)
        self.n_out = inp.N // 2 if epilogue == ll.LL_EPILOGUE_GEGLU_TANH else inp.N
        dev = torch.device("cuda")
        self.A = inp.A.to(dev) if inp.A is not None else None
        self.B = inp.B.to(dev) if inp.B is not None else None
        self.Q = inp.Q.to(dev)
        self.scale = inp.scale.to(dev)
        self.bias = inp.bias.to(dev) if inp.bias is not None else None
        ll.ll_set_weights(self.h, self.A, self.B, self.Q, self.scale, self.bias)

    def forward(self, x_cpu, stream=None):
        x = x_cpu.to("cuda")
        y = torch.empty(x.shape[0], self.n_out, dtype=torch.bfloat16, device="cuda")
        ll.ll_forward(self.h, x, y, x.shape[0], stream)
        torch.cuda.synchronize()
        st = ll.ll_status(self.h)
        assert st == ll.LL_OK, ll.status_string(st)
        return y

    def close(self):
        ll.ll_destroy(self.h)


def run(inp, variant=ll.LL_VARIANT_AUTO, epilogue=ll.LL_EPILOGUE_NONE):
    d = DeviceLayer(inp, variant, epilogue)
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


# Throughput of the oracle on the GPU machine's host (16 cores), measured by
# bench.py's CPU-baseline leg: 0.06 TFLOP/s.  Shapes whose full oracle run
# would take longer than FULL_ORACLE_S are checked on a strided row subset.
ORACLE_TFLOPS = 0.06
FULL_ORACLE_S = 30.0


def oracle_seconds(M, K, N, r):
    return (2.0 * M * N * (K + r) + 2.0 * M * K * r) / (ORACLE_TFLOPS * 1e12)


def checked_rows(M, K, N, r, tile=256, stride=8):
    """All rows when the full oracle fits FULL_ORACLE_S, else every
    `stride`-th row plus every row of the last (partial) token tile.
    Returns (rows or None for all, label)."""
    if oracle_seconds(M, K, N, r) <= FULL_ORACLE_S:
        return None, "full"
    last = (M - 1) // tile * tile
    rows = sorted(set(range(0, M, stride)) | set(range(last, M)))
    return rows, f"rows every {stride}th + last tile ({len(rows)} of {M})"


def check_streamed(outputs, inp, rows=None, block=512, what=""):
    """Check GPU outputs (name -> CPU bf16 tensor [M, N]) against the exact
    oracle, computed block by block over `rows` (None: all rows), with the
    per-element bound |err| <= 8e-3*|y_ref| + 2e-3*RMS(y_ref), RMS over all
    checked rows.  Memory stays bounded by the block; pass / fail is exact:
    an element fails iff err - 8e-3*|y_ref| > 2e-3*RMS."""
    M = inp.M
    idx = list(range(M)) if rows is None else list(rows)
    sumsq, count = 0.0, 0
    worst = {k: (-np.inf, None) for k in outputs}  # excess, (row, col, gpu, ref)
    for b0 in range(0, len(idx), block):
        rb = idx[b0:b0 + block]
        ref = oracle.forward_inputs(inp, rows=rb)
        sumsq += float(np.sum(np.square(ref)))
        count += ref.size
        for k, y in outputs.items():
            yb = y[rb].to(torch.float64).numpy()
            assert np.all(np.isfinite(yb)), f"{what} [{k}]: non-finite output"
            ex = np.abs(yb - ref) - 8e-3 * np.abs(ref)
            i = np.unravel_index(int(np.argmax(ex)), ex.shape)
            if ex[i] > worst[k][0]:
                worst[k] = (float(ex[i]), (rb[i[0]], int(i[1]), float(yb[i]), float(ref[i])))
    rms = math.sqrt(sumsq / max(count, 1))
    for k, (ex, where) in worst.items():
        assert ex <= 2e-3 * rms, (f"{what} [{k}]: element out of bound at {where}, "
                                  f"excess {ex:.3g} > 2e-3*RMS {2e-3 * rms:.3g}")
    return rms
