"""Pins for the CPU oracle against facts fixed outside the oracle itself.

The oracle (oracle/ll_oracle.c) is the binary64 definition of the LiteLinear
forward (LiteLinear README, introduction, display formula
y = (x B^T) A^T + scale * (x Q_fp8^T) + bias).  None of these tests re-types
that formula around the oracle's own helpers: they compare it against
torch's independent float8_e4m3fn / bfloat16 conversions, exact rational
arithmetic, numpy matrix products on independently decoded operands,
hand-computed closed forms, and structural invariants.
"""
import math
import random
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from synth_inputs import (SCALE_PER_ROW, SCALE_PER_TENSOR, make_inputs, to_numpy_bits)


# ---------------------------------------------------------------- decoders

def _torch_e4m3(codes):
    return torch.tensor(codes, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64)


def test_e4m3_decoder_exhaustive_vs_torch():
    """All 256 e4m3fn codes decode to torch's float8_e4m3fn values (NaN for
    the two NaN codes).  The README names e4m3fn as the residual format."""
    ref = _torch_e4m3(list(range(256))).numpy()
    for c in range(256):
        v = oracle.dec_e4m3(c)
        if math.isnan(ref[c]):
            assert math.isnan(v), hex(c)
        else:
            assert v == ref[c], (hex(c), v, ref[c])
            assert math.copysign(1.0, v) == math.copysign(1.0, ref[c]), hex(c)


@pytest.mark.parametrize("code,value", [
    (0x7E, 448.0),          # largest finite e4m3fn
    (0x01, 2.0 ** -9),      # smallest subnormal
    (0x07, 7 * 2.0 ** -9),  # largest subnormal
    (0x08, 2.0 ** -6),      # smallest normal
    (0x38, 1.0),
    (0x40, 2.0),
    (0xB8, -1.0),
    (0x00, 0.0),
])
def test_e4m3_decoder_special_values(code, value):
    assert oracle.dec_e4m3(code) == value


def test_e4m3_decoder_signed_zero_and_nan():
    v = oracle.dec_e4m3(0x80)
    assert v == 0.0 and math.copysign(1.0, v) == -1.0
    assert math.isnan(oracle.dec_e4m3(0x7F))
    assert math.isnan(oracle.dec_e4m3(0xFF))


def test_e4m3_decoder_monotone_and_odd():
    vals = [oracle.dec_e4m3(c) for c in range(0x7F)]
    assert all(a < b for a, b in zip(vals, vals[1:]))
    for c in range(0x7F):
        assert oracle.dec_e4m3(c | 0x80) == -oracle.dec_e4m3(c)


def test_e4m3_roundtrip_through_torch_encoder():
    """torch's round-to-nearest e4m3fn encoder maps every decoded value
    back to its own code."""
    for c in range(256):
        if c in (0x7F, 0xFF):
            continue
        v = oracle.dec_e4m3(c)
        back = torch.tensor([v], dtype=torch.float64).to(torch.float8_e4m3fn).view(torch.uint8)
        assert int(back[0]) == c or (v == 0.0 and int(back[0]) in (0x00, 0x80))


def test_bf16_decoder_exhaustive_vs_torch():
    bits = np.arange(65536, dtype=np.uint16)
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    got = np.array([oracle.dec_bf16(int(b)) for b in bits])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])
    assert np.array_equal(np.signbit(got[~nan]), np.signbit(ref[~nan]))


def test_bf16_encoder_vs_torch_on_float32_values():
    """For values exactly representable in float32, torch's float32->bf16
    conversion is a single round-to-nearest-even; the oracle must agree,
    including exact midpoints (ties to even) and subnormals."""
    rng = np.random.default_rng(7)
    f = rng.standard_normal(20000).astype(np.float32) * np.float32(10.0) ** rng.integers(-30, 30, 20000).astype(np.float32)
    # Exact midpoints between adjacent bf16 values: low 16 bits = 0x8000.
    mid = (rng.integers(0, 2 ** 31, 5000, dtype=np.uint32) & 0xFFFF0000) | 0x8000
    # Subnormal float32 values and values near the bf16 overflow threshold.
    sub = (rng.integers(1, 0x007FFFFF, 2000, dtype=np.uint32)).view(np.float32)
    big = np.array([3.3895314e38, 3.3961776e38, 3.4e38, -3.39e38], dtype=np.float32)
    vals = np.concatenate([f, mid.view(np.float32), sub, big]).astype(np.float32)
    vals = vals[np.isfinite(vals)]
    ref = torch.from_numpy(vals).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = np.array([oracle.enc_bf16_rne(float(v)) for v in vals], dtype=np.uint16)
    bad = np.nonzero(got != ref)[0]
    assert bad.size == 0, [(float(vals[i]), hex(got[i]), hex(ref[i])) for i in bad[:5]]


def test_bf16_encoder_ties_to_even_in_binary64():
    one = 1.0
    ulp = 2.0 ** -7
    assert oracle.enc_bf16_rne(one + ulp / 2) == 0x3F80          # tie -> even (1.0)
    assert oracle.enc_bf16_rne(one + 3 * ulp / 2) == 0x3F82      # tie -> even (1+2ulp)
    assert oracle.enc_bf16_rne(one + ulp / 2 + 2.0 ** -40) == 0x3F81  # just above tie
    assert oracle.enc_bf16_rne(-0.0) == 0x8000
    assert oracle.enc_bf16_rne(float("inf")) == 0x7F80


# ------------------------------------------------------------ closed forms

def _bf16_bits(v):
    return int(torch.tensor([v], dtype=torch.float64).to(torch.bfloat16).view(torch.int16)[0]) & 0xFFFF


def _run(x, B, A, Q, s, mode_s, bias, **kw):
    def u16(a):
        return None if a is None else np.array([[_bf16_bits(v) for v in row] for row in a], dtype=np.uint16)
    return oracle.forward(u16(x), u16(B), u16(A), np.array(Q, dtype=np.uint8),
                          np.array(s, dtype=np.float32), mode_s,
                          None if bias is None else np.array([_bf16_bits(v) for v in bias], dtype=np.uint16), **kw)


def test_hand_computed_1x1():
    """M=K=N=r=1: x=1, B=1, A=1, Q=0x38 (1.0), s=0.5, bias=0.25 gives
    y = (1*1)*1 + 0.5*(1*1) + 0.25 = 1.75 exactly."""
    y = _run([[1.0]], [[1.0]], [[1.0]], [[0x38]], [0.5], SCALE_PER_ROW, [0.25])
    assert y.shape == (1, 1) and y[0, 0] == 1.75


def test_hand_computed_signs_and_subnormal():
    """x=-2, B=0.5, A=3, Q=0x81 (-2^-9), s=4, bias=-1:
    t = -1, y = -1*3 + 4*(-2 * -2^-9) - 1 = -4 + 2^-6."""
    y = _run([[-2.0]], [[0.5]], [[3.0]], [[0x81]], [4.0], SCALE_PER_TENSOR, [-1.0])
    assert y[0, 0] == -4.0 + 2.0 ** -6


def test_hand_computed_2x2():
    """M=1, K=2, N=2, r=1.  x=[1,2]; B=[[1,-1]] so t=-1; A=[[2],[0.5]];
    Q=[[1.0, 0.5],[448, -2^-6]] (codes 0x38,0x30,0x7E,0x88); s=[0.25, 1];
    bias=[0, 8].
    y0 = -1*2   + 0.25*(1 + 1)          + 0 = -1.5
    y1 = -1*0.5 + 1*(448 - 2*2^-6)      + 8 = 455.5 - 2^-5
    """
    y = _run([[1.0, 2.0]], [[1.0, -1.0]], [[2.0], [0.5]], [[0x38, 0x30], [0x7E, 0x88]],
             [0.25, 1.0], SCALE_PER_ROW, [0.0, 8.0])
    assert y[0, 0] == -1.5
    assert y[0, 1] == 455.5 - 2.0 ** -5


def test_golden_fixture_cases():
    """tests/golden/closed_form_cases.txt: hand-derived small cases."""
    import os
    path = os.path.join(os.path.dirname(__file__), "golden", "closed_form_cases.txt")
    cases = []
    with open(path) as f:
        cur = {}
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, _, val = line.partition("=")
            key = key.strip()
            val = val.strip()
            if key == "case":
                if cur:
                    cases.append(cur)
                cur = {"name": val}
            else:
                cur[key] = eval(val, {"__builtins__": {}}, {})  # literal lists/numbers only
        if cur:
            cases.append(cur)
    assert len(cases) >= 3
    for c in cases:
        y = _run(c["x"], c.get("B"), c.get("A"), c["Q"], c["scale"], c["scale_mode"], c.get("bias"))
        assert np.array_equal(y, np.array(c["y"], dtype=np.float64)), c["name"]


# ---------------------------------------------------------- exact rationals

def _frac_bf16(bits):
    return Fraction(float(torch.tensor([bits], dtype=torch.int16).view(torch.bfloat16).to(torch.float64)[0]))


def _exact_forward(inp):
    """Exact rational evaluation with Python Fractions; operands decoded by
    torch (independent of the oracle's decoders)."""
    M, K, N, r = inp.M, inp.K, inp.N, inp.r
    xf = [[Fraction(float(v)) for v in row] for row in inp.x.to(torch.float64).tolist()]
    Qf = [[Fraction(float(v)) for v in row] for row in inp.Q.view(torch.float8_e4m3fn).to(torch.float64).tolist()]
    Bf = [[Fraction(float(v)) for v in row] for row in inp.B.to(torch.float64).tolist()] if r else []
    Af = [[Fraction(float(v)) for v in row] for row in inp.A.to(torch.float64).tolist()] if r else []
    sf = [Fraction(float(v)) for v in inp.scale.tolist()]
    bf = [Fraction(float(v)) for v in inp.bias.to(torch.float64).tolist()] if inp.bias is not None else [Fraction(0)] * N
    y = []
    for m in range(M):
        t = [sum(xf[m][k] * Bf[j][k] for k in range(K)) for j in range(r)]
        row = []
        for n in range(N):
            yq = sum(xf[m][k] * Qf[n][k] for k in range(K))
            ylr = sum(t[j] * Af[n][j] for j in range(r))
            s = sf[n] if inp.scale_mode == SCALE_PER_ROW else sf[0]
            row.append(s * yq + ylr + bf[n])
        y.append(row)
    return y


@pytest.mark.parametrize("seed", range(12))
def test_bruteforce_exact_rationals(seed):
    rnd = random.Random(seed)
    M, K, N = rnd.randint(1, 6), rnd.randint(1, 8), rnd.randint(1, 6)
    r = rnd.randint(0, 5)
    mode = rnd.choice([SCALE_PER_ROW, SCALE_PER_TENSOR])
    inp = make_inputs(M, K, N, r, scale_mode=mode, scale_range=(1e-3, 3.0), seed=100 + seed,
                      bias=bool(seed % 3))
    y = oracle.forward_inputs(inp)
    ex = _exact_forward(inp)
    for m in range(M):
        for n in range(N):
            e = float(ex[m][n])
            assert abs(y[m, n] - e) <= 1e-14 * max(1.0, abs(e)), (m, n, y[m, n], e)


# --------------------------------------------------------------- invariants

def _np_dec(inp):
    x = inp.x.to(torch.float64).numpy()
    Q = inp.Q.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    B = inp.B.to(torch.float64).numpy() if inp.r else None
    A = inp.A.to(torch.float64).numpy() if inp.r else None
    s = inp.scale.to(torch.float64).numpy()
    if inp.scale_mode == SCALE_PER_TENSOR:
        s = np.full(inp.N, s[0])
    b = inp.bias.to(torch.float64).numpy() if inp.bias is not None else np.zeros(inp.N)
    return x, Q, B, A, s, b


def _close(a, b, rel=1e-12):
    scale = np.maximum(1.0, np.abs(b))
    assert np.all(np.abs(a - b) <= rel * scale * 10), float(np.max(np.abs(a - b) / scale))


def test_r0_is_scaled_fp8_linear():
    """With r = 0 the layer is the scaled FP8 linear scale*(x Q^T) + bias."""
    inp = make_inputs(37, 96, 48, 0, scale_range=(1e-3, 3e-3), seed=3)
    x, Q, _, _, s, b = _np_dec(inp)
    _close(oracle.forward_inputs(inp), (x @ Q.T) * s[None, :] + b[None, :])


def test_q0_is_svd_linear_layer():
    """With every residual code 0 the layer is SVDLinearLayer.forward
    (tt_compressor page): F.linear(F.linear(x, B), A) + bias."""
    inp = make_inputs(29, 80, 40, 7, seed=4, q_zero=True)
    x, _, B, A, _, b = _np_dec(inp)
    _close(oracle.forward_inputs(inp), (x @ B.T) @ A.T + b[None, :])


def test_dense_weight_equivalence():
    """y = x W^T + bias with the reconstructed W = A B + diag(scale) Q
    (README introduction: W ~= A*B + Q_fp8)."""
    for mode in (SCALE_PER_ROW, SCALE_PER_TENSOR):
        inp = make_inputs(33, 128, 72, 12, scale_mode=mode, scale_range=(1e-3, 3e-3), seed=5)
        x, Q, B, A, s, b = _np_dec(inp)
        W = A @ B + s[:, None] * Q
        _close(oracle.forward_inputs(inp), x @ W.T + b[None, :])


def test_linearity_in_x():
    inp = make_inputs(16, 64, 32, 8, seed=6)
    inp2 = make_inputs(16, 64, 32, 8, seed=6)
    inp2.x = (inp.x.to(torch.float32) * -2.0).to(torch.bfloat16)  # exact in bf16
    y1 = oracle.forward_inputs(inp)
    y2 = oracle.forward_inputs(inp2)
    b = inp.bias.to(torch.float64).numpy()
    _close(y2 - b, -2.0 * (y1 - b))


def test_row_permutation_and_row_subset():
    inp = make_inputs(21, 64, 24, 5, seed=8)
    full = oracle.forward_inputs(inp)
    perm = np.random.default_rng(0).permutation(21)
    inp.x = inp.x[torch.from_numpy(perm)]
    assert np.array_equal(oracle.forward_inputs(inp), full[perm])
    rows = [20, 0, 7, 7]
    sub = oracle.forward_inputs(inp, rows=rows)
    assert np.array_equal(sub, full[perm][rows])


def test_per_tensor_equals_uniform_per_row():
    a = make_inputs(9, 32, 16, 4, scale_mode=SCALE_PER_TENSOR, seed=9)
    y_t = oracle.forward_inputs(a)
    a.scale = torch.full((16,), float(a.scale[0]), dtype=torch.float32)
    a.scale_mode = SCALE_PER_ROW
    assert np.array_equal(oracle.forward_inputs(a), y_t)


def test_bias_none_equals_zero_bias():
    a = make_inputs(5, 32, 16, 4, seed=10, bias=False)
    y0 = oracle.forward_inputs(a)
    a.bias = torch.zeros(16, dtype=torch.bfloat16)
    assert np.array_equal(oracle.forward_inputs(a), y0)


def test_mirror_mode_rounds_t_to_bf16():
    """MIRROR = EXACT with t replaced by its bf16 rounding (torch's rounding
    of the numpy-computed t, which is float32-exact here because x, B are
    small integers)."""
    rng = np.random.default_rng(11)
    M, K, N, r = 6, 16, 8, 4
    inp = make_inputs(M, K, N, r, seed=11)
    inp.x = torch.from_numpy(rng.integers(-8, 8, (M, K)).astype(np.float32)).to(torch.bfloat16)
    inp.B = torch.from_numpy(rng.integers(-8, 8, (r, K)).astype(np.float32) / 3.0).to(torch.bfloat16)
    x, Q, B, A, s, b = _np_dec(inp)
    t = x @ B.T
    assert np.all(t.astype(np.float32).astype(np.float64) == t)
    tb = torch.from_numpy(t.astype(np.float32)).to(torch.bfloat16).to(torch.float64).numpy()
    ref = (x @ Q.T) * s[None, :] + tb @ A.T + b[None, :]
    _close(oracle.forward_inputs(inp, mode=oracle.MIRROR), ref)


def test_degenerate_shapes():
    # M = 0: empty output; K = 0: y = bias.
    inp = make_inputs(0, 16, 8, 4, seed=12)
    assert oracle.forward_inputs(inp).shape == (0, 8)
    inp = make_inputs(3, 0, 8, 4, seed=12)
    y = oracle.forward_inputs(inp)
    assert np.array_equal(y, np.tile(inp.bias.to(torch.float64).numpy(), (3, 1)))


def test_rejects_bad_arguments():
    x = np.zeros((2, 4), np.uint16)
    Q = np.zeros((3, 4), np.uint8)
    with pytest.raises(ValueError):
        oracle.forward(x, None, None, Q, np.ones(3, np.float32), 7)
    with pytest.raises(ValueError):
        oracle.forward(x, None, None, Q, np.ones(3, np.float32), 1, rows=[2])


def test_tolerance_bound_definition():
    y = np.array([[1.0, -3.0], [0.0, 2.0]])
    rms = math.sqrt((1 + 9 + 0 + 4) / 4)
    assert np.allclose(oracle.tolerance_bound(y), 8e-3 * np.abs(y) + 2e-3 * rms)
