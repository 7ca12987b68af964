"""Parity at the full sizes of the layer configurations: the FFN pair, all
24 points of the (M, K, N, r) sweep, and the 28 LTX-Video FFN shapes of the
LiteLinear README's kernel benchmark ("Performance Benchmark on shapes
captured from LTX-Video"; K and N read as 4096 <-> 16384, ranks 32 and 64).

Each shape runs through the C ABI on the variant AUTO dispatches and on the
FP8-operand two-term variant, and both outputs are checked against the exact
oracle of y = (x B^T) A^T + scale * (x Q^T) + bias (LiteLinear README,
introduction) with the per-element bound
|err| <= 8e-3*|y_ref| + 2e-3*RMS(y_ref), RMS over the checked output.  The
whole output is checked wherever the oracle needs at most ~30 s on the GPU
box's 16 host cores (at its measured 0.06 TFLOP/s); larger shapes are
checked on every 8th row plus every row of the last, partial token tile,
as the test id says.
"""
import pytest

import rank_fp8_residual_b200 as ll
from synth_inputs import WORKLOADS

from llgpu import check_streamed, checked_rows, run

pytestmark = pytest.mark.gpu

FFN = ["ffn_up_m3630_k2048_n8192_r64", "ffn_down_m3630_k8192_n2048_r64"]
SWEEP = sorted((n for n in WORKLOADS if n.startswith("sweep_")),
               key=lambda n: (WORKLOADS[n].N, WORKLOADS[n].M, WORKLOADS[n].r))
PAGE = sorted((n for n in WORKLOADS if n.startswith("page_")),
              key=lambda n: (WORKLOADS[n].r, WORKLOADS[n].K, WORKLOADS[n].M))


def _params(names):
    out = []
    for n in names:
        w = WORKLOADS[n]
        _, label = checked_rows(w.M, w.K, w.N, w.r)
        out.append(pytest.param(n, id=f"{n}-{'full' if label == 'full' else 'rows-every-8th'}"))
    return out


def _check(name):
    w = WORKLOADS[name]
    inp = w.inputs()
    rows, label = checked_rows(w.M, w.K, w.N, w.r)
    outs = {"auto": run(inp, ll.LL_VARIANT_AUTO), "fp8-split": run(inp, ll.LL_VARIANT_FP8_SPLIT)}
    check_streamed(outs, inp, rows, what=f"{name} ({label})")


@pytest.mark.parametrize("name", _params(FFN))
def test_ffn_pair_full_output(name):
    _check(name)


@pytest.mark.parametrize("name", _params(SWEEP))
def test_sweep_point(name):
    _check(name)


@pytest.mark.parametrize("name", _params(PAGE))
def test_page_microbench_shape(name):
    _check(name)
