"""Pins for the oracle's FP8-activation readings (modes FP8ACT / FP8SPLIT and
the per-token quantiser behind them), against facts fixed outside the
oracle: torch's own float8_e4m3fn rounding, hand-derived closed forms, and
properties that follow from the e4m3fn format (every finite e4m3fn value
is a dyadic number with at most 4 significant bits and an exponent of at
least -9).

The readings (LiteLinear README, "Features": e4m3fn is the layer's FP8
format; its LTX-Video kernel benchmark's fused "Accel" column): a token row
x_m is scaled by the power of two 2^e_m, the smallest with
max_k |x_mk| <= 448 * 2^e_m, and rounded to e4m3fn (nearest, ties to even):
hi = e4m3(x / 2^e_m).  The two-term expansion adds lo = e4m3(x / 2^e_m - hi).
"""
import math

import numpy as np
import pytest
import torch

import oracle
from synth_inputs import SCALE_PER_ROW, make_inputs, to_numpy_bits


def _all_finite_bf16():
    codes = np.arange(65536, dtype=np.uint32)
    f = (codes << 16).view(np.float32)
    return f[np.isfinite(f)].astype(np.float64)


def _torch_e4m3_code(v: float) -> int:
    return int(torch.tensor([v], dtype=torch.float32).to(torch.float8_e4m3fn).view(torch.uint8)[0])


# ---------------------------------------------------------------- encoder

def test_e4m3_encoder_matches_torch_on_every_bf16_value_in_range():
    """Every bf16 value with |v| <= 464 rounds to the same code as torch's
    float32 -> float8_e4m3fn conversion (round to nearest even).  Above 464
    torch gives NaN; the oracle saturates (checked separately)."""
    vals = _all_finite_bf16()
    vals = vals[np.abs(vals) <= 448.0]
    ref = torch.from_numpy(vals.astype(np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([oracle.enc_e4m3_rne(float(v)) for v in vals], dtype=np.uint8)
    bad = np.nonzero(got != ref)[0]
    assert bad.size == 0, [(vals[i], hex(got[i]), hex(ref[i])) for i in bad[:5]]


@pytest.mark.parametrize("v,code", [
    (1.0, 0x38), (448.0, 0x7E), (-448.0, 0xFE), (500.0, 0x7E), (1e30, 0x7E), (-1e30, 0xFE),
    (2.0 ** -9, 0x01), (2.0 ** -10, 0x00),           # a tie between 0 and the smallest subnormal: even (0)
    (3 * 2.0 ** -10, 0x02),                           # tie between 0x01 and 0x02: even
    (7.5 * 2.0 ** -9, 0x08),                          # tie across the subnormal / normal boundary
    (1.0625, 0x38), (1.1875, 0x3A),                   # ties 1 | 1.125 and 1.125 | 1.25
    (-0.0, 0x80), (0.0, 0x00),
])
def test_e4m3_encoder_closed_forms(v, code):
    assert oracle.enc_e4m3_rne(v) == code


def test_e4m3_encoder_roundtrip_and_nan():
    for c in range(256):
        if c in (0x7F, 0xFF):
            continue
        assert oracle.enc_e4m3_rne(oracle.dec_e4m3(c)) == c, hex(c)
    assert oracle.enc_e4m3_rne(float("nan")) == 0x7F


def test_e4m3_encoder_matches_torch_on_random_midpoints():
    """Exact midpoints between neighbouring codes and points just beside
    them (all representable in float32, so torch rounds them once)."""
    rng = np.random.default_rng(5)
    for _ in range(2000):
        c = int(rng.integers(0, 0x7E))
        a, b = oracle.dec_e4m3(c), oracle.dec_e4m3(c + 1)
        mid = (a + b) / 2
        for v in (mid, np.nextafter(np.float32(mid), np.float32(0)), np.nextafter(np.float32(mid), np.float32(1e9))):
            v = float(v)
            for s in (1.0, -1.0):
                assert oracle.enc_e4m3_rne(s * v) == _torch_e4m3_code(s * v), (s * v, c)


# ------------------------------------------------------- token exponent

@pytest.mark.parametrize("amax,e", [
    (448.0, 0), (449.0, 1), (450.0, 1), (224.0, -1), (224.5, 0), (896.0, 1), (896.5, 2),
    (1.0, -8), (1.75, -8), (1.7500001, -7), (0.0, 0),
    (1e-300, -126), (1e300, 126),
])
def test_token_exponent_closed_forms(amax, e):
    """The smallest e with amax <= 448 * 2^e (clamped to [-126, 126])."""
    assert oracle.token_exp(amax) == e


def test_token_exponent_is_minimal_over_bf16():
    rng = np.random.default_rng(3)
    for v in rng.choice(_all_finite_bf16(), 3000):
        a = abs(float(v))
        if a == 0:
            continue
        e = oracle.token_exp(a)
        if -126 < e < 126:
            assert a <= 448.0 * 2.0 ** e and a > 448.0 * 2.0 ** (e - 1), (a, e)


# ------------------------------------------------------------- quantiser

def test_quantiser_two_term_error_bound_and_exact_range():
    """For every bf16 value u with |u| <= 448 (a row scaled so that its
    maximum is 448, e = 0): hi + lo reproduces u exactly when |u| >= 1/4
    (u - hi is then a multiple of 2^(E-7) of magnitude at most 2^(E-4),
    which e4m3fn holds exactly), and within 2^-10 (half the smallest
    subnormal step) otherwise."""
    vals = _all_finite_bf16()
    vals = vals[np.abs(vals) <= 448.0]
    bits = (vals.astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    row = np.concatenate([bits, np.array([0x43E0], dtype=np.uint16)])  # 448 keeps e = 0
    e, hi, lo = oracle.quant_x(row[None, :], 2)
    assert e[0] == 0
    dec = np.array([oracle.dec_e4m3(c) for c in range(256)])
    dec[[0x7F, 0xFF]] = np.nan
    u = np.concatenate([vals, [448.0]])
    err = np.abs(u - dec[hi[0]] - dec[lo[0]])
    assert np.all(err[np.abs(u) >= 0.25] == 0.0)
    assert np.all(err <= 2.0 ** -10)
    # hi alone is the nearest e4m3fn value: within half a step of u
    step = np.where(np.abs(u) < 2.0 ** -6, 2.0 ** -9, 2.0 ** (np.floor(np.log2(np.maximum(np.abs(u), 1e-300))) - 3))
    assert np.all(np.abs(u - dec[hi[0]]) <= step / 2)


def test_quantiser_scales_rows_by_their_own_power_of_two():
    """Scaling a row by 2^j moves its exponent by j and leaves its codes."""
    x = make_inputs(4, 96, 16, 0, seed=9).x
    xb = to_numpy_bits(x)
    e0, h0, l0 = oracle.quant_x(xb, 2)
    for j in (-20, -3, 5, 40):
        xs = to_numpy_bits((x.to(torch.float64) * 2.0 ** j).to(torch.bfloat16))
        e1, h1, l1 = oracle.quant_x(xs, 2)
        assert np.array_equal(e1, e0 + j)
        assert np.array_equal(h1, h0) and np.array_equal(l1, l0)


def test_quantiser_is_identity_on_e4m3_rows_with_max_448():
    """A row whose values are e4m3fn values and whose maximum is 448 has
    e = 0, hi = its own codes and lo = 0."""
    rng = np.random.default_rng(11)
    codes = rng.integers(0, 0x7E, size=(3, 64)).astype(np.uint8)
    codes |= (rng.integers(0, 2, size=codes.shape) * 0x80).astype(np.uint8)
    codes[:, 7] = 0x7E
    vals = codes.view(np.uint8)
    f = torch.from_numpy(vals).view(torch.float8_e4m3fn).to(torch.bfloat16)
    e, hi, lo = oracle.quant_x(to_numpy_bits(f), 2)
    assert np.all(e == 0)
    # -0 and +0 both encode as a zero code of the same sign
    assert np.array_equal(hi, codes)
    assert np.all((lo == 0) | (lo == 0x80))


# --------------------------------------------------- FP8 forward readings

def _one_by_one(mode):
    # x = bf16(0.3) = 0.30078125; B = 1, A = 1; Q = 0x38 (1.0); scale 0.5; bias 0.25
    x = np.array([[0x3E9A]], dtype=np.uint16)
    assert oracle.dec_bf16(0x3E9A) == 0.30078125
    one = np.array([[0x3F80]], dtype=np.uint16)
    Q = np.array([[0x38]], dtype=np.uint8)
    s = np.array([0.5], dtype=np.float32)
    b = np.array([0x3E80], dtype=np.uint16)  # 0.25
    return oracle.forward(x, one, one, Q, s, SCALE_PER_ROW, b, mode=mode)[0, 0]


def test_fp8act_closed_form():
    """max |x| = 0.30078125 gives e = -10 (448 * 2^-11 < 0.3008 <= 448 * 2^-10);
    x / 2^-10 = 308 rounds to the e4m3fn value 320 (step 32 between 256
    and 448), so the residual term sees 320 * 2^-10 = 0.3125, while the
    low-rank term keeps x:  y = 0.5 * 0.3125 * 1 + 0.30078125 * 1 * 1 + 0.25."""
    assert _one_by_one(oracle.FP8ACT) == 0.5 * 0.3125 + 0.30078125 + 0.25


def test_fp8split_closed_form():
    """The two-term expansion: 308 = 320 + (-12), and -12 = -1.5 * 2^3 is an
    e4m3fn value, so the residual term sees x exactly."""
    assert _one_by_one(oracle.FP8SPLIT) == 0.5 * 0.30078125 + 0.30078125 + 0.25
    assert _one_by_one(oracle.FP8SPLIT) == _one_by_one(oracle.EXACT)


def test_fp8act_equals_exact_on_e4m3_valued_rows():
    """Rows that are e4m3fn values with a maximum of 448 are not changed by
    the quantisation, so every FP8 reading equals the exact one."""
    inp = make_inputs(6, 64, 40, 8, seed=12)
    rng = np.random.default_rng(12)
    codes = rng.integers(0, 0x7E, size=(6, 64)).astype(np.uint8)
    codes[:, 3] = 0x7E
    inp.x = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.bfloat16)
    ref = oracle.forward_inputs(inp)
    for mode in (oracle.FP8ACT, oracle.FP8SPLIT):
        assert np.array_equal(oracle.forward_inputs(inp, mode=mode), ref)


def test_fp8act_residual_term_uses_dequantised_rows():
    """FP8ACT with zero low-rank factors and zero bias is the scaled FP8
    linear on the dequantised rows 2^e * hi, computed here with numpy from
    the quantiser's codes and torch's e4m3fn decoding."""
    inp = make_inputs(9, 128, 24, 4, seed=13)
    inp.A = torch.zeros_like(inp.A)
    inp.bias = None
    e, hi, _ = oracle.quant_x(to_numpy_bits(inp.x), 1)
    xq = torch.from_numpy(hi).view(torch.float8_e4m3fn).to(torch.float64).numpy() * np.ldexp(1.0, e)[:, None]
    W = torch.from_numpy(to_numpy_bits(inp.Q)).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    ref = (xq @ W.T) * inp.scale.numpy().astype(np.float64)[None, :]
    got = oracle.forward_inputs(inp, mode=oracle.FP8ACT)
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-300)


def test_fp8_modes_are_row_local():
    """A row's result does not depend on the other rows (the scale is per
    token): a subset of rows gives the matching rows."""
    inp = make_inputs(20, 96, 32, 8, seed=14)
    for mode in (oracle.FP8ACT, oracle.FP8SPLIT):
        full = oracle.forward_inputs(inp, mode=mode)
        rows = [19, 3, 7]
        assert np.array_equal(oracle.forward_inputs(inp, mode=mode, rows=rows), full[rows])


def test_fp8split_is_within_the_bound_of_exact():
    """The two-term expansion differs from x only below 2^-2 * 2^e_m, by at
    most 2^-10 * 2^e_m, so on the workload distributions its forward lies
    far inside the accuracy bound around the exact forward."""
    inp = make_inputs(64, 512, 96, 16, scale_range=(1e-3, 3e-3), seed=15)
    ex = oracle.forward_inputs(inp)
    sp = oracle.forward_inputs(inp, mode=oracle.FP8SPLIT)
    bound = oracle.tolerance_bound(ex)
    assert np.max(np.abs(sp - ex) / bound) < 0.05
