"""Pins for the oracle's residual quantisation (the step of the layer's
decomposition after the SVD; LiteLinear README, "Usage": from_dense), against
facts fixed outside the oracle: torch's float8_e4m3fn rounding, hand-derived
closed forms, and properties of the e4m3fn format.

Reading: R = W - A B, scale = max|R| / 448 (per row, or over the tensor)
rounded to binary32, Q = e4m3fn(R / scale) (nearest, ties to even), the
division taken in binary64 and rounded to binary32 before the e4m3fn
rounding.
"""
import numpy as np
import pytest
import torch

import oracle
from synth_inputs import to_numpy_bits

ROW, TENSOR = 1, 0


def _bits(t):
    return to_numpy_bits(t.to(torch.bfloat16).contiguous())


def _dec_e4m3(codes):
    return torch.from_numpy(np.ascontiguousarray(codes)).view(torch.float8_e4m3fn).to(torch.float64).numpy()


def test_closed_form_single_row():
    """W = [448, -224, 1, 0], r = 0: max |R| = 448 gives scale 1 and the codes
    of the values themselves (-224 = -1.75 * 2^7: sign, exponent field 14,
    mantissa 6)."""
    W = _bits(torch.tensor([[448.0, -224.0, 1.0, 0.0]]))
    Q, s = oracle.residual_quant(W, None, None, ROW)
    assert s.tolist() == [1.0]
    assert Q.tolist() == [[0x7E, 0xF6, 0x38, 0x00]]


def test_exact_low_rank_weight_has_zero_residual():
    """W = A B exactly (small integers, exact in bf16): R = 0, scale 0 and
    every code 0, in both modes."""
    rng = np.random.default_rng(1)
    A = torch.from_numpy(rng.integers(-3, 4, size=(6, 2)).astype(np.float32))
    B = torch.from_numpy(rng.integers(-3, 4, size=(2, 32)).astype(np.float32))
    W = A @ B
    for mode in (ROW, TENSOR):
        Q, s = oracle.residual_quant(_bits(W), _bits(A), _bits(B), mode)
        assert np.all(s == 0) and np.all(Q == 0)


def test_residual_is_weight_minus_low_rank():
    """With A = 0 the residual is W itself: the per-row scale is max|W_n| / 448
    in binary32 and the codes equal torch's float8_e4m3fn rounding of
    (binary32)(W / scale)."""
    rng = np.random.default_rng(2)
    W = torch.from_numpy(rng.standard_normal((5, 40)).astype(np.float32)).to(torch.bfloat16)
    A = torch.zeros(5, 3)
    B = torch.from_numpy(rng.standard_normal((3, 40)).astype(np.float32))
    Q, s = oracle.residual_quant(_bits(W), _bits(A), _bits(B), ROW)
    w = W.to(torch.float64).numpy()
    amax = np.abs(w).max(axis=1)
    assert np.array_equal(s, (amax / 448.0).astype(np.float32))
    u = (w / s.astype(np.float64)[:, None]).astype(np.float32)
    ref = torch.from_numpy(u).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(Q, ref)


def test_largest_residual_maps_to_448_and_error_bound():
    """Every nonzero row's largest |R| becomes the code of 448 (binary32
    rounding of the scale can only move R / scale within 448 * (1 +- 2^-24),
    which rounds or saturates to 448), and every element of s * dec(Q) lies
    within half an e4m3fn step of R: |R/s - dec(Q)| <= max(2^-4 |R/s|, 2^-10)
    (plus the binary32 rounding of R / s)."""
    rng = np.random.default_rng(3)
    N, K, r = 9, 96, 4
    W = torch.from_numpy(rng.standard_normal((N, K)).astype(np.float32))
    A = torch.from_numpy(0.3 * rng.standard_normal((N, r)).astype(np.float32))
    B = torch.from_numpy(rng.standard_normal((r, K)).astype(np.float32))
    Wb, Ab, Bb = _bits(W), _bits(A), _bits(B)
    Q, s = oracle.residual_quant(Wb, Ab, Bb, ROW)
    w = Wb.view(np.int16).astype(np.int32) << 16
    w = w.astype(np.uint32).view(np.float32).astype(np.float64)
    a = (Ab.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    b = (Bb.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    R = w - a @ b
    dq = _dec_e4m3(Q)
    for n in range(N):
        i = int(np.argmax(np.abs(R[n])))
        assert abs(dq[n, i]) == 448.0
        u = R[n] / float(s[n])
        bound = np.maximum(2.0 ** -4 * np.abs(u), 2.0 ** -10) * (1 + 1e-6) + 1e-6
        assert np.all(np.abs(u - dq[n]) <= bound)


def test_per_tensor_scale_is_the_largest_row_scale():
    """binary32 rounding is monotone, so the per-tensor scale is the largest
    per-row scale, and rows holding the tensor's maximum get the same codes."""
    rng = np.random.default_rng(4)
    W = torch.from_numpy(rng.standard_normal((7, 64)).astype(np.float32))
    W[3] *= 10.0
    A = torch.from_numpy(rng.standard_normal((7, 2)).astype(np.float32))
    B = torch.from_numpy(0.1 * rng.standard_normal((2, 64)).astype(np.float32))
    Qr, sr = oracle.residual_quant(_bits(W), _bits(A), _bits(B), ROW)
    Qt, st = oracle.residual_quant(_bits(W), _bits(A), _bits(B), TENSOR)
    assert st.shape == (1,) and st[0] == sr.max()
    n = int(np.argmax(sr))
    assert np.array_equal(Qt[n], Qr[n])


def test_zero_rank_and_zero_weight():
    Q, s = oracle.residual_quant(_bits(torch.zeros(3, 16)), None, None, ROW)
    assert np.all(Q == 0) and np.all(s == 0)
