"""Parity of the CUDA path (through the C ABI) with the CPU oracle.

Bar (per element): |y_gpu - y_ref| <= 8e-3*|y_ref| + 2e-3*RMS(y_ref), with
y_ref the binary64 oracle of y = (x B^T) A^T + scale * (x Q^T) + bias
(LiteLinear README, introduction) and RMS over the output of the call (over
the sampled rows where only rows are sampled).  The widening check is exact.
"""
import numpy as np
import pytest
import torch

import oracle
import rank_fp8_residual_b200 as ll
from synth_inputs import (SCALE_PER_ROW, SCALE_PER_TENSOR, WORKLOADS, LayerInputs, make_inputs)

from llgpu import DeviceLayer, check, run

pytestmark = pytest.mark.gpu


VARIANTS = [ll.LL_VARIANT_TC, ll.LL_VARIANT_SMALL, ll.LL_VARIANT_TC_PAIR]
# The streaming variant serves M <= 64 only (larger M runs the SMALL kernel).
SMALL_M_VARIANTS = VARIANTS + [ll.LL_VARIANT_STREAM]
VNAME = {ll.LL_VARIANT_TC: "tc", ll.LL_VARIANT_SMALL: "small", ll.LL_VARIANT_AUTO: "auto",
         ll.LL_VARIANT_TC_PAIR: "tc-pair", ll.LL_VARIANT_STREAM: "stream"}


def _full(inp, what, variant=ll.LL_VARIANT_AUTO):
    y = run(inp, variant)
    return check(y, oracle.forward_inputs(inp), what=f"{what} [{VNAME[variant]}]")


@pytest.mark.parametrize("variant", VARIANTS)
def test_widening_is_exact_for_every_code(variant):
    """One-hot tokens pick single residual codes: y[m, n] = Q[n, m] exactly.
    Every non-NaN code appears in every K position, so the swizzled shared
    memory reads and the TMEM lane mapping are covered too."""
    K = N = M = 256
    n = torch.arange(N).view(N, 1)
    k = torch.arange(K).view(1, K)
    codes = ((n + k) % 256).to(torch.uint8)
    codes[(codes == 0x7F) | (codes == 0xFF)] = 0
    x = torch.eye(M, K, dtype=torch.bfloat16)
    inp = LayerInputs(M, K, N, 0, SCALE_PER_TENSOR, x, None, None, codes,
                      torch.ones(1, dtype=torch.float32), None)
    y = run(inp, variant).to(torch.float64)
    expect = codes.view(torch.float8_e4m3fn).to(torch.float64).t()  # [M=K, N]
    assert torch.equal(y, expect)


@pytest.mark.parametrize("K", [256, 272])
def test_widening_is_exact_for_every_code_streaming(K):
    """The same check for the streaming kernel, which takes at most 64
    tokens: four calls of 64 one-hot tokens cover all K positions (K = 272
    exercises the 2-D loads of a K that is not a multiple of 64)."""
    N = 256
    n = torch.arange(N).view(N, 1)
    k = torch.arange(K).view(1, K)
    codes = ((n + k) % 256).to(torch.uint8)
    codes[(codes == 0x7F) | (codes == 0xFF)] = 0
    expect_all = codes.view(torch.float8_e4m3fn).to(torch.float64).t()  # [K, N]
    for k0 in range(0, K, 64):
        M = min(64, K - k0)
        x = torch.zeros(M, K, dtype=torch.bfloat16)
        x[torch.arange(M), k0 + torch.arange(M)] = 1.0
        inp = LayerInputs(M, K, N, 0, SCALE_PER_TENSOR, x, None, None, codes,
                          torch.ones(1, dtype=torch.float32), None)
        y = run(inp, ll.LL_VARIANT_STREAM).to(torch.float64)
        assert torch.equal(y, expect_all[k0:k0 + M])


def test_tiny_config():
    _full(WORKLOADS["tiny_m64_k256_n256_r16"].inputs(), "tiny")


@pytest.mark.parametrize("variant", VARIANTS)
@pytest.mark.parametrize("M,K,N,r", [(300, 272, 392, 40), (129, 1024, 136, 64), (517, 384, 1000, 200),
                                     (1100, 320, 264, 96)])
def test_ragged_multi_tile(M, K, N, r, variant):
    inp = make_inputs(M, K, N, r, scale_range=(1e-3, 3e-3), seed=M)
    _full(inp, f"ragged {M}x{K}x{N} r{r}", variant)


@pytest.mark.parametrize("variant", VARIANTS)
def test_rank_zero(variant):
    _full(make_inputs(600, 256, 256, 0, seed=1), "r=0", variant)


@pytest.mark.parametrize("variant", VARIANTS)
def test_residual_zero_is_low_rank_only(variant):
    _full(make_inputs(600, 256, 256, 32, seed=2, q_zero=True), "Q=0", variant)


@pytest.mark.parametrize("variant", VARIANTS)
def test_per_tensor_scale_and_no_bias(variant):
    _full(make_inputs(450, 320, 264, 24, scale_mode=SCALE_PER_TENSOR, bias=False, seed=3),
          "per-tensor, no bias", variant)


@pytest.mark.parametrize("variant", VARIANTS)
def test_zero_scale_rows(variant):
    """Rows with scale 0 keep only their low-rank term and bias."""
    inp = make_inputs(520, 256, 392, 40, scale_range=(1e-3, 3e-3), seed=4)
    inp.scale[::7] = 0.0
    inp.scale[5] = -2e-3  # a negative scale is a valid multiplier
    _full(inp, "zero-scale rows", variant)


def test_scale_far_outside_fold_range_is_rejected():
    """The fused large-M kernel carries A / scale as a bf16 pair; a scale
    that would push it past 2^100 is reported instead of losing accuracy."""
    inp = make_inputs(8, 64, 64, 8, seed=5)
    inp.scale[3] = 1e-35
    h = ll.ll_create(64, 64, 8, SCALE_PER_ROW)
    try:
        with pytest.raises(ll.LLError) as e:
            ll.ll_set_weights(h, inp.A.cuda(), inp.B.cuda(), inp.Q.cuda(), inp.scale.cuda(),
                              inp.bias.cuda())
        assert e.value.code == ll.LL_ERR_UNSUPPORTED
    finally:
        ll.ll_destroy(h)


@pytest.mark.parametrize("variant", SMALL_M_VARIANTS)
@pytest.mark.parametrize("M", [1, 2, 15, 16, 17, 31, 33, 48, 63, 64])
def test_small_token_counts(M, variant):
    _full(make_inputs(M, 512, 1024, 96, seed=10 + M), f"M={M}", variant)


@pytest.mark.parametrize("M,K,N,r", [(5, 272, 392, 40), (40, 1024, 136, 64), (64, 384, 1000, 200),
                                     (17, 4096, 2056, 512), (64, 2048, 20480, 32)])
def test_streaming_ragged(M, K, N, r):
    """Ragged feature tails, K not a multiple of 64, every rank chunking,
    and more feature tiles than SMs (persistent CTAs)."""
    inp = make_inputs(M, K, N, r, scale_range=(1e-3, 3e-3), seed=M + N)
    inp.scale[::11] = 0.0
    _full(inp, f"stream {M}x{K}x{N} r{r}", ll.LL_VARIANT_STREAM)


@pytest.mark.parametrize("variant", [ll.LL_VARIANT_STREAM])
@pytest.mark.parametrize("case", ["r0", "q0", "per_tensor_no_bias"])
def test_streaming_special_cases(case, variant):
    if case == "r0":
        inp = make_inputs(50, 256, 256, 0, seed=51)
    elif case == "q0":
        inp = make_inputs(50, 256, 256, 32, seed=52, q_zero=True)
    else:
        inp = make_inputs(45, 320, 264, 24, scale_mode=SCALE_PER_TENSOR, bias=False, seed=53)
    _full(inp, f"stream {case}", variant)


@pytest.mark.parametrize("variant", VARIANTS)
@pytest.mark.parametrize("M", [127, 128, 129, 255, 256, 257, 511, 513])
def test_token_tile_edges(M, variant):
    _full(make_inputs(M, 128, 256, 16, seed=20 + M), f"M={M}", variant)


@pytest.mark.parametrize("variant", VARIANTS)
@pytest.mark.parametrize("r", [1, 31, 32, 33, 63, 64, 65, 96, 128, 160, 256, 320, 512])
def test_rank_edges(r, variant):
    _full(make_inputs(300, 256, 256, r, seed=30 + r), f"r={r}", variant)


@pytest.mark.parametrize("r", [1, 33, 64, 65, 160, 512])
def test_rank_edges_streaming(r):
    _full(make_inputs(37, 256, 256, r, seed=60 + r), f"stream r={r}", ll.LL_VARIANT_STREAM)


def test_attention_projection_full():
    _full(WORKLOADS["attn_m3630_k2048_n2048_r32"].inputs(), "attn_m3630_k2048_n2048_r32")


@pytest.mark.parametrize("name", ["small_m1_k4096_n16384_r512", "small_m16_k4096_n16384_r512",
                                  "small_m64_k4096_n16384_r512"])
def test_small_batch_full(name):
    _full(WORKLOADS[name].inputs(), name)


def test_repeated_calls_are_bitwise_identical():
    inp = make_inputs(700, 512, 640, 64, seed=40)
    d = DeviceLayer(inp)
    try:
        a = d.forward(inp.x)
        b = d.forward(inp.x)
        assert torch.equal(a, b)
    finally:
        d.close()


@pytest.mark.parametrize("M", [333, 1000, 3000])
def test_forward_host_matches_device(M):
    """The host-buffer forward (in chunks of 256-token tiles, copies
    overlapped with the forwards) meets the bound against the oracle, also
    on a second call that reuses its staging buffers; in one chunk it gives
    the device forward's bits."""
    inp = make_inputs(M, 256, 264, 32, seed=41)
    d = DeviceLayer(inp)
    try:
        y_dev = d.forward(inp.x).cpu()
        ref = oracle.forward_inputs(inp)
        xh = inp.x.contiguous().pin_memory()
        for _ in range(2):
            yh = torch.full((inp.M, inp.N), float("nan"), dtype=torch.bfloat16).pin_memory()
            ll.ll_forward_host(d.h, xh.data_ptr(), yh.data_ptr(), inp.M, None)
            torch.cuda.synchronize()
            check(yh.clone(), ref, what=f"ll_forward_host M={M}")
            if M < 512:
                assert torch.equal(yh, y_dev)
    finally:
        d.close()


def test_set_weights_rejects_nan_codes():
    inp = make_inputs(8, 64, 64, 8, seed=42)
    inp.Q[3, 5] = 0xFF
    h = ll.ll_create(64, 64, 8, SCALE_PER_ROW)
    try:
        with pytest.raises(ll.LLError) as e:
            ll.ll_set_weights(h, inp.A.cuda(), inp.B.cuda(), inp.Q.cuda(), inp.scale.cuda(),
                              inp.bias.cuda())
        assert e.value.code == ll.LL_ERR_NAN_CODE
        x = torch.zeros(8, 64, dtype=torch.bfloat16, device="cuda")
        y = torch.empty(8, 64, dtype=torch.bfloat16, device="cuda")
        with pytest.raises(ll.LLError) as e:
            ll.ll_forward(h, x, y, 8)
        assert e.value.code == ll.LL_ERR_NOT_READY
    finally:
        ll.ll_destroy(h)


def test_argument_errors_on_device():
    inp = make_inputs(8, 64, 64, 8, seed=43)
    d = DeviceLayer(inp)
    try:
        x = torch.zeros(9, 64, dtype=torch.bfloat16, device="cuda")
        y = torch.empty(9, 64, dtype=torch.bfloat16, device="cuda")
        for args, code in [((x, y, -1), ll.LL_ERR_INVALID_ARG),
                           ((x.view(-1)[1:].data_ptr(), y, 4), ll.LL_ERR_INVALID_ARG),  # misaligned
                           ((x, x, 4), ll.LL_ERR_INVALID_ARG)]:                          # overlap
            with pytest.raises(ll.LLError) as e:
                ll.ll_forward(d.h, *args)
            assert e.value.code == code
        ll.ll_forward(d.h, x, y, 0)  # M == 0 is a no-op
        bad = inp.scale.clone()
        bad[0] = float("inf")
        with pytest.raises(ll.LLError) as e:
            ll.ll_set_weights(d.h, d.A, d.B, d.Q, bad.cuda(), d.bias)
        assert e.value.code == ll.LL_ERR_INVALID_ARG
        with pytest.raises(ll.LLError) as e:  # host pointer where a device pointer is required
            ll.ll_set_weights(d.h, d.A, d.B, inp.Q.data_ptr(), d.scale, d.bias)
        assert e.value.code == ll.LL_ERR_INVALID_ARG
    finally:
        d.close()


def test_set_weights_and_forward_reject_misaligned_pointers():
    """A, B and Q must be 16-byte aligned for ll_set_weights, x and y for
    ll_forward (scale 4-byte, bias 2-byte), as the header states."""
    inp = make_inputs(8, 64, 64, 8, seed=44)
    d = DeviceLayer(inp)
    try:
        def shifted(t):  # the same bytes, 2 bytes past a 16-byte boundary
            buf = torch.empty(t.numel() * t.element_size() + 16, dtype=torch.uint8, device="cuda")
            return buf[2:2 + t.numel() * t.element_size()].data_ptr()
        for which in ("A", "B", "Q"):
            args = {"A": d.A, "B": d.B, "Q": d.Q}
            args[which] = shifted(args[which])
            with pytest.raises(ll.LLError) as e:
                ll.ll_set_weights(d.h, args["A"], args["B"], args["Q"], d.scale, d.bias)
            assert e.value.code == ll.LL_ERR_INVALID_ARG, which
        y = torch.empty(8, 64, dtype=torch.bfloat16, device="cuda")
        x = inp.x.cuda()
        with pytest.raises(ll.LLError) as e:
            ll.ll_forward(d.h, shifted(x), y, 8)
        assert e.value.code == ll.LL_ERR_INVALID_ARG
        with pytest.raises(ll.LLError) as e:
            ll.ll_forward(d.h, x, shifted(y), 8)
        assert e.value.code == ll.LL_ERR_INVALID_ARG
    finally:
        d.close()
