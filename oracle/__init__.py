"""Python access to the C oracle (oracle/ll_oracle.c).

TEST INFRASTRUCTURE ONLY: the test suite, ``__graft_entry__.smoke()`` and
the benchmark's CPU-baseline leg are the only callers.  The product path
never imports this package.

The oracle is the plain binary64 definition of the LiteLinear forward
(LiteLinear README, introduction, the display formula
``y = (x B^T) A^T + scale * (x Q_fp8^T) + bias``).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

EXACT = 0
MIRROR = 1
FP8ACT = 2     # x in x Q^T quantised per token to one e4m3fn term
FP8SPLIT = 3   # x in x Q^T as the two-term e4m3fn expansion (diagnostic)

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ll_oracle.c")
_LIB = os.path.join(_HERE, "libll_oracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (OpenMP) into oracle/libll_oracle.so."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
                               "-fno-fast-math", "-ffp-contract=off",
                               _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def lib():
    global _lib
    if _lib is None:
        L = ctypes.CDLL(build())
        L.llo_dec_e4m3.restype = ctypes.c_double
        L.llo_dec_e4m3.argtypes = [ctypes.c_uint8]
        L.llo_dec_bf16.restype = ctypes.c_double
        L.llo_dec_bf16.argtypes = [ctypes.c_uint16]
        L.llo_enc_bf16_rne.restype = ctypes.c_uint16
        L.llo_enc_bf16_rne.argtypes = [ctypes.c_double]
        L.llo_num_threads.restype = ctypes.c_int
        L.llo_enc_e4m3_rne.restype = ctypes.c_uint8
        L.llo_enc_e4m3_rne.argtypes = [ctypes.c_double]
        L.llo_token_exp.restype = ctypes.c_int
        L.llo_token_exp.argtypes = [ctypes.c_double]
        L.llo_residual_quant.restype = ctypes.c_int
        L.llo_residual_quant.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p,
                                         ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p]
        L.llo_quant_x.restype = ctypes.c_int
        L.llo_quant_x.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_void_p, ctypes.c_int,
                                  ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
        p = ctypes.c_void_p
        L.llo_forward.restype = ctypes.c_int
        L.llo_forward.argtypes = [ctypes.c_int] * 4 + [p, p, p, p, p, ctypes.c_int, p,
                                                       ctypes.c_int, p, ctypes.c_int, p]
        _lib = L
    return _lib


def dec_e4m3(c: int) -> float:
    return lib().llo_dec_e4m3(int(c))


def dec_bf16(b: int) -> float:
    return lib().llo_dec_bf16(int(b))


def enc_bf16_rne(v: float) -> int:
    return lib().llo_enc_bf16_rne(float(v))


def enc_e4m3_rne(v: float) -> int:
    return lib().llo_enc_e4m3_rne(float(v))


def token_exp(amax: float) -> int:
    return lib().llo_token_exp(float(amax))


def quant_x(x, terms: int):
    """Per-token e4m3fn quantisation of x (uint16 bf16 bits [M, K]):
    returns (e [M] int32, hi [M, K] uint8, lo [M, K] uint8 or None), with
    x[m, k] ~= 2^e[m] * (hi + lo) (lo only for terms == 2)."""
    x = np.ascontiguousarray(x, dtype=np.uint16)
    M, K = x.shape
    e = np.zeros(M, dtype=np.int32)
    hi = np.zeros((M, K), dtype=np.uint8)
    lo = np.zeros((M, K), dtype=np.uint8) if terms == 2 else None
    rc = lib().llo_quant_x(M, K, _ptr(x), int(terms), _ptr(e), _ptr(hi), _ptr(lo))
    if rc != 0:
        raise ValueError("oracle rejected its arguments")
    return e, hi, lo


def residual_quant(W, A, B, scale_mode):
    """The residual quantisation of the decomposition step: W, A, B as bf16
    bits (uint16 [N, K], [N, r] or None, [r, K] or None).  Returns
    (Q uint8 [N, K], scale float32 [N] or [1])."""
    W = np.ascontiguousarray(W, dtype=np.uint16)
    N, K = W.shape
    if A is None or B is None:
        r = 0
    else:
        A = np.ascontiguousarray(A, dtype=np.uint16)
        B = np.ascontiguousarray(B, dtype=np.uint16)
        r = A.shape[1]
        assert A.shape == (N, r) and B.shape == (r, K)
    Q = np.zeros((N, K), dtype=np.uint8)
    scale = np.zeros(N if scale_mode == 1 else 1, dtype=np.float32)
    rc = lib().llo_residual_quant(N, K, r, _ptr(W), _ptr(A) if r else None, _ptr(B) if r else None,
                                  int(scale_mode), _ptr(Q), _ptr(scale))
    if rc != 0:
        raise ValueError("oracle rejected its arguments")
    return Q, scale


def num_threads() -> int:
    return lib().llo_num_threads()


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def forward(x, B, A, Q, scale, scale_mode, bias=None, mode=EXACT, rows=None):
    """Reference forward in binary64.

    x: uint16 [M,K] (bf16 bits); B: uint16 [r,K] or None; A: uint16 [N,r]
    or None; Q: uint8 [N,K] (e4m3fn codes); scale: float32 [N] or [1];
    bias: uint16 [N] or None.  rows: optional int sequence of row indices
    of x to evaluate.  Returns float64 [len(rows) or M, N].
    """
    x = np.ascontiguousarray(x, dtype=np.uint16)
    Q = np.ascontiguousarray(Q, dtype=np.uint8)
    M, K = x.shape
    N = Q.shape[0]
    assert Q.shape == (N, K)
    if B is None or A is None:
        r = 0
        B = A = None
    else:
        B = np.ascontiguousarray(B, dtype=np.uint16)
        A = np.ascontiguousarray(A, dtype=np.uint16)
        r = B.shape[0]
        assert B.shape == (r, K) and A.shape == (N, r)
    scale = np.ascontiguousarray(scale, dtype=np.float32)
    if bias is not None:
        bias = np.ascontiguousarray(bias, dtype=np.uint16)
        assert bias.shape == (N,)
    if rows is not None:
        rows = np.ascontiguousarray(rows, dtype=np.int32)
        nrows = rows.shape[0]
    else:
        nrows = M
    y = np.empty((nrows, N), dtype=np.float64)
    rc = lib().llo_forward(M, K, N, r, _ptr(x), _ptr(B), _ptr(A), _ptr(Q), _ptr(scale),
                           int(scale_mode), _ptr(bias), int(mode), _ptr(rows), nrows,
                           _ptr(y))
    if rc != 0:
        raise ValueError("oracle rejected its arguments")
    return y


EPILOGUE_NONE = 0
EPILOGUE_GELU_TANH = 1
EPILOGUE_GEGLU_TANH = 2


def gelu_tanh(v: np.ndarray) -> np.ndarray:
    """GELU in its tanh form, v / 2 * (1 + tanh(sqrt(2/pi) (v + 0.044715 v^3)))
    (the approximation the LTX feed-forward's GELU uses), in binary64."""
    return 0.5 * v * (1.0 + np.tanh(np.sqrt(2.0 / np.pi) * (v + 0.044715 * v ** 3)))


def apply_epilogue(y: np.ndarray, epilogue: int) -> np.ndarray:
    """The fused activation on the layer's output y [rows, N]: none, GELU of
    every element, or GEGLU: h * gelu(g) with h = y[:, :N/2], g = y[:, N/2:]
    (the LiteLinear README's GEGLU projection, "Usage": replace_activation_proj_)."""
    if epilogue == EPILOGUE_NONE:
        return y
    if epilogue == EPILOGUE_GELU_TANH:
        return gelu_tanh(y)
    if epilogue == EPILOGUE_GEGLU_TANH:
        n = y.shape[1] // 2
        return y[:, :n] * gelu_tanh(y[:, n:])
    raise ValueError("unknown epilogue")


def forward_inputs(inp, mode=EXACT, rows=None, epilogue=EPILOGUE_NONE):
    """forward() on a synth_inputs.LayerInputs, then the epilogue activation."""
    from synth_inputs import to_numpy_bits
    y = forward(to_numpy_bits(inp.x), to_numpy_bits(inp.B), to_numpy_bits(inp.A),
                to_numpy_bits(inp.Q), to_numpy_bits(inp.scale), inp.scale_mode,
                to_numpy_bits(inp.bias), mode=mode, rows=rows)
    return apply_epilogue(y, epilogue)


def tolerance_bound(y_ref: np.ndarray, rms: float | None = None) -> np.ndarray:
    """Per-element acceptance bound |err| <= 8e-3*|y_ref| + 2e-3*RMS(y_ref),
    RMS over the whole output tensor of the call (or the given value)."""
    if rms is None:
        rms = float(np.sqrt(np.mean(np.square(y_ref)))) if y_ref.size else 0.0
    return 8e-3 * np.abs(y_ref) + 2e-3 * rms
