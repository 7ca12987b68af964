"""The C-ABI library loads and exports every function include/*.h declares;
host-side argument checks reject bad calls before touching a GPU."""
import ctypes
import glob
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    names = []
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        src = open(h).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        names += re.findall(r"\b(ll_[a-z_0-9]+)\s*\(", src)
    return sorted(set(names))


def test_header_declares_the_boundary():
    names = _declared_functions()
    for n in ("ll_create", "ll_set_weights", "ll_forward", "ll_destroy", "ll_last_error",
              "ll_status_string", "ll_status", "ll_forward_host", "ll_reserve"):
        assert n in names


def test_library_exports_every_declared_symbol():
    import rank_fp8_residual_b200 as ll
    lib = ctypes.CDLL(ll.LIB_PATH)
    missing = [n for n in _declared_functions() if not hasattr(lib, n)]
    assert not missing, missing
    # the binding wraps every declared function under the same name
    for n in _declared_functions():
        assert n in ll._SIGNATURES, n


def test_status_strings():
    import rank_fp8_residual_b200 as ll
    assert ll.status_string(ll.LL_OK) == "ok"
    assert "NaN" in ll.status_string(ll.LL_ERR_NAN_CODE)
    assert ll.status_string(12345) == "unknown status"


@pytest.mark.parametrize("N,K,r,mode", [(7, 64, 4, 1), (8, 15, 4, 1), (8, 64, -1, 1),
                                          (8, 64, 4, 2), (0, 64, 4, 1), (8, 0, 0, 0)])
def test_create_rejects_bad_shapes_without_a_gpu(N, K, r, mode):
    import rank_fp8_residual_b200 as ll
    with pytest.raises(ll.LLError) as e:
        ll.ll_create(N, K, r, mode)
    assert e.value.code == ll.LL_ERR_INVALID_ARG


def test_create_rank_above_limit_is_unsupported():
    import rank_fp8_residual_b200 as ll
    with pytest.raises(ll.LLError) as e:
        ll.ll_create(64, 64, 513, 1)
    assert e.value.code == ll.LL_ERR_UNSUPPORTED


def test_null_handle_calls_fail_cleanly():
    import rank_fp8_residual_b200 as ll
    lib = ll._lib
    assert lib.ll_forward(None, None, None, 4, None) == ll.LL_ERR_INVALID_ARG
    assert lib.ll_last_error() == ll.LL_ERR_INVALID_ARG
    assert lib.ll_set_weights(None, None, None, None, None, None) == ll.LL_ERR_INVALID_ARG
    assert lib.ll_forward_host(None, None, None, 1, None) == ll.LL_ERR_INVALID_ARG
    assert lib.ll_reserve(None, 4) == ll.LL_ERR_INVALID_ARG
    assert lib.ll_set_variant(None, 0) == ll.LL_ERR_INVALID_ARG
    assert lib.ll_set_debug(None, 0, 1) == ll.LL_ERR_INVALID_ARG
    assert lib.ll_last_launch_count(None) == 0
    lib.ll_destroy(None)


def test_binding_has_no_cpu_fallback(monkeypatch, tmp_path):
    """Importing the binding without the built library raises."""
    import importlib.util
    import sys
    src = os.path.join(ROOT, "rank_fp8_residual_b200", "__init__.py")
    pkg = tmp_path / "rank_fp8_residual_b200"
    pkg.mkdir()
    (pkg / "__init__.py").write_text(open(src).read())
    spec = importlib.util.spec_from_file_location("llcopy", str(pkg / "__init__.py"))
    mod = importlib.util.module_from_spec(spec)
    with pytest.raises(ImportError):
        spec.loader.exec_module(mod)


def test_noalloc_argument_checks_need_no_gpu():
    """ll_forward_noalloc rejects bad shapes and modes before any CUDA call."""
    import rank_fp8_residual_b200 as ll
    f = ll._lib.ll_forward_noalloc
    P = None
    assert f(P, P, P, P, P, 1, P, P, 0, 64, 64, 8, P) == ll.LL_OK          # M == 0 is a no-op
    assert f(P, P, P, P, P, 1, P, P, 4, 60, 64, 8, P) == ll.LL_ERR_INVALID_ARG   # N % 8
    assert f(P, P, P, P, P, 1, P, P, 4, 64, 40, 8, P) == ll.LL_ERR_INVALID_ARG   # K % 16
    assert f(P, P, P, P, P, 1, P, P, 4, 64, 64, 513, P) == ll.LL_ERR_INVALID_ARG  # r > 512
    assert f(P, P, P, P, P, 5, P, P, 4, 64, 64, 8, P) == ll.LL_ERR_INVALID_ARG   # scale mode
    assert f(P, P, P, P, P, 1, P, P, 4, 64, 64, 12, P) == ll.LL_ERR_UNSUPPORTED  # r % 8
    assert f(P, P, P, P, P, 1, P, P, 4, 64, 64, 8, P) == ll.LL_ERR_INVALID_ARG   # null pointers
    assert ll.ll_last_error() == ll.LL_ERR_INVALID_ARG


def test_misaligned_pointers_are_rejected_before_any_gpu_work():
    """The header's alignment rule (16 bytes for x, y, A, B, Q and the e4m3
    code buffers; 4 for scale and token exponents; 2 for bias) is checked
    before any CUDA call: fake addresses suffice, no GPU is touched."""
    import rank_fp8_residual_b200 as ll
    good = 0x100000
    bad16 = good + 2
    base = dict(x=good, A=good, B=good, Q=good, scale=good, bias=good, y=good + 0x800000)
    for name in ("x", "A", "B", "Q", "y"):
        a = dict(base, **{name: bad16})
        with pytest.raises(ll.LLError) as e:
            ll.ll_forward_noalloc(a["x"], a["A"], a["B"], a["Q"], a["scale"], 1, a["bias"], a["y"],
                                  64, 256, 256, 32, stream=0)
        assert e.value.code == ll.LL_ERR_INVALID_ARG, name
    with pytest.raises(ll.LLError) as e:
        ll.ll_forward_noalloc(good, good, good, good, good + 2, 1, good, good + 0x800000, 64, 256, 256, 32, stream=0)
    assert e.value.code == ll.LL_ERR_INVALID_ARG
    with pytest.raises(ll.LLError) as e:
        ll.ll_forward_noalloc(good, good, good, good, good, 1, good + 1, good + 0x800000, 64, 256, 256, 32, stream=0)
    assert e.value.code == ll.LL_ERR_INVALID_ARG
    for x, e_out, hi, lo in ((bad16, good, good, good), (good, good + 2, good, good), (good, good, bad16, good),
                             (good, good, good, bad16)):
        with pytest.raises(ll.LLError) as e:
            ll.ll_quantize_x(x, 8, 64, 2, e_out, hi, lo, stream=0)
        assert e.value.code == ll.LL_ERR_INVALID_ARG


def test_binding_constants_match_the_header():
    """Every `LL_NAME = value` enumerator of include/*.h has the same value in
    the Python binding."""
    import rank_fp8_residual_b200 as ll
    found = {}
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        src = re.sub(r"/\*.*?\*/", "", open(h).read(), flags=re.S)
        for name, val in re.findall(r"\b(LL_[A-Z_0-9]+)\s*=\s*(\d+)", src):
            found[name] = int(val)
    assert "LL_VARIANT_GEMV" in found and "LL_EPILOGUE_GEGLU_TANH" in found
    for name, val in found.items():
        assert getattr(ll, name) == val, name
