"""Python binding of the B200 LiteLinear forward library.

Thin ctypes marshalling over the C ABI in include/rank_fp8_residual.h; every
step of the forward runs in the library's CUDA kernels.  Functions keep the
C names and accept either raw integers (device addresses, stream handles)
or torch tensors / streams, from which they take ``data_ptr()`` and
``cuda_stream``.  There is no CPU fallback: importing raises if the shared
library has not been built (``python rank_fp8_residual_b200/build.py``).
"""
from __future__ import annotations

import ctypes
import os

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "librank_fp8_residual_b200.so")

LL_SCALE_PER_TENSOR = 0
LL_SCALE_PER_ROW = 1

LL_OK = 0
LL_ERR_INVALID_ARG = 1
LL_ERR_UNSUPPORTED = 2
LL_ERR_NOT_READY = 3
LL_ERR_NAN_CODE = 4
LL_ERR_OOM = 5
LL_ERR_CUDA = 6
LL_ERR_DEVICE_TIMEOUT = 7
LL_ERR_SCRATCH_LIMIT = 8

# Size of the static device scratch used by ll_forward_noalloc.
LL_NOALLOC_SCRATCH_BYTES = 16 * 1024 * 1024

LL_VARIANT_AUTO = 0
LL_VARIANT_TC = 1
LL_VARIANT_SMALL = 2
LL_VARIANT_TC_PAIR = 3
LL_VARIANT_STREAM = 4
LL_VARIANT_FP8_SPLIT = 5
LL_VARIANT_FP8_ACT = 6
LL_VARIANT_GEMV = 7

LL_EPILOGUE_NONE = 0
LL_EPILOGUE_GELU_TANH = 1
LL_EPILOGUE_GEGLU_TANH = 2

# Every symbol the header declares, with (restype, argtypes).
_P = ctypes.c_void_p
_SIGNATURES = {
    "ll_create": (_P, [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int]),
    "ll_set_weights": (ctypes.c_int, [_P, _P, _P, _P, _P, _P]),
    "ll_forward": (ctypes.c_int, [_P, _P, _P, ctypes.c_int, _P]),
    "ll_forward_host": (ctypes.c_int, [_P, _P, _P, ctypes.c_int, _P]),
    "ll_reserve": (ctypes.c_int, [_P, ctypes.c_int]),
    "ll_set_variant": (ctypes.c_int, [_P, ctypes.c_int]),
    "ll_set_epilogue": (ctypes.c_int, [_P, ctypes.c_int]),
    "ll_status": (ctypes.c_int, [_P]),
    "ll_set_debug": (ctypes.c_int, [_P, ctypes.c_int, ctypes.c_uint64]),
    "ll_destroy": (None, [_P]),
    "ll_last_error": (ctypes.c_int, []),
    "ll_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "ll_last_launch_count": (ctypes.c_int, [_P]),
    "ll_set_profiling": (ctypes.c_int, [_P, ctypes.c_int]),
    "ll_kernel_times": (ctypes.c_int, [_P, _P, ctypes.c_int]),
    "ll_kernel_name": (ctypes.c_char_p, [_P, ctypes.c_int]),
    "ll_forward_noalloc": (ctypes.c_int, [_P, _P, _P, _P, _P, ctypes.c_int, _P, _P, ctypes.c_int, ctypes.c_int,
                                          ctypes.c_int, ctypes.c_int, _P]),
    "ll_quantize_residual": (ctypes.c_int, [_P, _P, _P, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                            _P, _P, _P]),
    "ll_quantize_x": (ctypes.c_int, [_P, ctypes.c_int, ctypes.c_int, ctypes.c_int, _P, _P, _P, _P]),
    "ll_plan": (ctypes.c_int, [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                               _P, _P, _P]),
}


class LLError(RuntimeError):
    def __init__(self, code: int, what: str = ""):
        self.code = code
        super().__init__(f"{what}: {status_string(code)} (code {code})" if what else status_string(code))


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python rank_fp8_residual_b200/build.py`")
    lib = ctypes.CDLL(LIB_PATH)
    for name, (res, args) in _SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


_lib = _load()


def _addr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(s):
    if s is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(s, int):
        return s
    return s.cuda_stream


def status_string(code: int) -> str:
    return _lib.ll_status_string(int(code)).decode()


def ll_last_error() -> int:
    return _lib.ll_last_error()


def ll_create(N: int, K: int, r: int, scale_mode: int) -> int:
    h = _lib.ll_create(int(N), int(K), int(r), int(scale_mode))
    if not h:
        raise LLError(_lib.ll_last_error(), "ll_create")
    return h


def ll_set_weights(h: int, A, B, Q, scale, bias=None) -> None:
    rc = _lib.ll_set_weights(h, _addr(A), _addr(B), _addr(Q), _addr(scale), _addr(bias))
    if rc != LL_OK:
        raise LLError(rc, "ll_set_weights")


def ll_forward(h: int, x, y, M: int, stream=None) -> None:
    rc = _lib.ll_forward(h, _addr(x), _addr(y), int(M), _stream(stream))
    if rc != LL_OK:
        raise LLError(rc, "ll_forward")


def ll_forward_host(h: int, x_host, y_host, M: int, stream=None) -> None:
    rc = _lib.ll_forward_host(h, _addr(x_host), _addr(y_host), int(M), _stream(stream))
    if rc != LL_OK:
        raise LLError(rc, "ll_forward_host")


def ll_reserve(h: int, max_M: int) -> None:
    rc = _lib.ll_reserve(h, int(max_M))
    if rc != LL_OK:
        raise LLError(rc, "ll_reserve")


def ll_set_variant(h: int, variant: int) -> None:
    rc = _lib.ll_set_variant(h, int(variant))
    if rc != LL_OK:
        raise LLError(rc, "ll_set_variant")


def ll_set_epilogue(h: int, epilogue: int) -> None:
    rc = _lib.ll_set_epilogue(h, int(epilogue))
    if rc != LL_OK:
        raise LLError(rc, "ll_set_epilogue")


def ll_status(h: int) -> int:
    return _lib.ll_status(h)


def ll_set_debug(h: int, withhold_producer: bool, timeout_ns: int) -> None:
    rc = _lib.ll_set_debug(h, int(bool(withhold_producer)), int(timeout_ns))
    if rc != LL_OK:
        raise LLError(rc, "ll_set_debug")


def ll_destroy(h: int) -> None:
    _lib.ll_destroy(h)


def ll_last_launch_count(h: int) -> int:
    return _lib.ll_last_launch_count(h)


def ll_set_profiling(h: int, enable: bool) -> None:
    rc = _lib.ll_set_profiling(h, int(bool(enable)))
    if rc != LL_OK:
        raise LLError(rc, "ll_set_profiling")


def ll_kernel_times(h: int):
    """[(kernel name, device ms)] of the last profiled forward."""
    buf = (ctypes.c_float * 8)()
    n = _lib.ll_kernel_times(h, ctypes.cast(buf, ctypes.c_void_p), 8)
    if n < 0:
        raise LLError(LL_ERR_CUDA, "ll_kernel_times")
    return [(_lib.ll_kernel_name(h, i).decode(), float(buf[i])) for i in range(min(n, 8))]


def ll_forward_noalloc(x, A, B, Q, scale, scale_mode: int, bias, y, M: int, N: int, K: int, r: int,
                       stream=None) -> None:
    """Forward for callers that may not allocate device memory: no handle,
    every buffer the caller's, scratch in the library's static device array
    (LL_NOALLOC_SCRATCH_BYTES per GPU).  Calls on one device must not
    overlap on the GPU; the first call on a device should precede any
    stream capture."""
    rc = _lib.ll_forward_noalloc(_addr(x), _addr(A), _addr(B), _addr(Q), _addr(scale), int(scale_mode), _addr(bias),
                                 _addr(y), int(M), int(N), int(K), int(r), _stream(stream))
    if rc != LL_OK:
        raise LLError(rc, "ll_forward_noalloc")


def ll_quantize_x(x, M: int, K: int, terms: int, e_out, hi, lo=None, stream=None) -> None:
    """Per-token e4m3fn codes of x (bf16 [M, K]): e_out int32 [M], hi uint8
    [M, K] and, for terms == 2, lo uint8 [M, K] (device buffers)."""
    rc = _lib.ll_quantize_x(_addr(x), int(M), int(K), int(terms), _addr(e_out), _addr(hi), _addr(lo),
                            _stream(stream))
    if rc != LL_OK:
        raise LLError(rc, "ll_quantize_x")


def ll_quantize_residual(W, A, B, N: int, K: int, r: int, scale_mode: int, Q, scale, stream=None) -> None:
    """Residual codes and scale of the decomposition step (device buffers):
    W bf16 [N, K], A bf16 [N, r], B bf16 [r, K] -> Q uint8 [N, K], scale
    float32 [N] or [1]."""
    rc = _lib.ll_quantize_residual(_addr(W), _addr(A), _addr(B), int(N), int(K), int(r), int(scale_mode), _addr(Q),
                                   _addr(scale), _stream(stream))
    if rc != LL_OK:
        raise LLError(rc, "ll_quantize_residual")


def from_dense(W, r: int, scale_mode: int = LL_SCALE_PER_ROW):
    """Decompose a dense weight W (CUDA bf16 [N, K], nn.Linear layout) into
    the layer's factors (LiteLinear README, "Usage": from_dense):
    A = U_r S_r and B = V_r^T from torch's SVD (a library routine, run once
    when a layer is built), rounded to bf16, and the residual's e4m3fn codes
    and scale from ll_quantize_residual.  Returns (A, B, Q, scale)."""
    import torch
    N, K = W.shape
    r = int(r)
    if r > 0:
        U, S, Vh = torch.linalg.svd(W.to(torch.float32), full_matrices=False)
        A = (U[:, :r] * S[:r]).to(torch.bfloat16).contiguous()
        B = Vh[:r].to(torch.bfloat16).contiguous()
    else:
        A = B = None
    Q = torch.empty(N, K, dtype=torch.uint8, device=W.device)
    scale = torch.empty(N if scale_mode == LL_SCALE_PER_ROW else 1, dtype=torch.float32, device=W.device)
    ll_quantize_residual(W.contiguous(), A, B, N, K, r, scale_mode, Q, scale)
    return A, B, Q, scale


def ll_plan(N: int, K: int, r: int, M: int, num_sms: int, variant: int = 0):
    """(kernel variant, tokens per tile, down-projection K splits) that a
    forward of M tokens would use on an (N, K, r) layer with num_sms SMs.
    Host arithmetic only; works without a GPU."""
    k, bt, ks = ctypes.c_int(0), ctypes.c_int(0), ctypes.c_int(0)
    rc = _lib.ll_plan(int(N), int(K), int(r), int(M), int(num_sms), int(variant), ctypes.byref(k), ctypes.byref(bt),
                      ctypes.byref(ks))
    if rc != LL_OK:
        raise LLError(rc, "ll_plan")
    return k.value, bt.value, ks.value


class LiteLinearLayer:
    """Owns one library handle; ``forward(x)`` returns a new bf16 tensor.

    Tensors must be CUDA tensors on the current device: A bf16 [N,r],
    B bf16 [r,K], Q uint8 (e4m3fn codes) [N,K], scale float32 [N] or [1],
    bias bf16 [N] or None.
    """

    def __init__(self, N: int, K: int, r: int, scale_mode: int = LL_SCALE_PER_ROW,
                 epilogue: int = LL_EPILOGUE_NONE):
        self.N, self.K, self.r, self.scale_mode = N, K, r, scale_mode
        self.handle = ll_create(N, K, r, scale_mode)
        self.epilogue = epilogue
        if epilogue != LL_EPILOGUE_NONE:
            ll_set_epilogue(self.handle, epilogue)

    @property
    def out_features(self) -> int:
        return self.N // 2 if self.epilogue == LL_EPILOGUE_GEGLU_TANH else self.N

    def set_weights(self, A, B, Q, scale, bias=None):
        ll_set_weights(self.handle, A, B, Q, scale, bias)

    @classmethod
    def from_dense(cls, W, r: int, bias=None, scale_mode: int = LL_SCALE_PER_ROW):
        """A layer from a dense CUDA bf16 weight [out, in] (see from_dense)."""
        N, K = W.shape
        A, B, Q, scale = from_dense(W, r, scale_mode)
        layer = cls(N, K, r, scale_mode)
        layer.set_weights(A, B, Q, scale, bias)
        return layer

    def forward(self, x, out=None, stream=None):
        import torch
        M = x.shape[0]
        if out is None:
            out = torch.empty(M, self.out_features, dtype=torch.bfloat16, device=x.device)
        ll_forward(self.handle, x, out, M, stream)
        return out

    def close(self):
        if self.handle:
            ll_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
