"""The C ABI on the CPU: the library loads, exports every declared entry point,
and rejects bad arguments on the host before touching a device."""
import ctypes
import os
import re

import numpy as np
import pytest

import target_attention_jagged_b200 as S
from target_attention_jagged_b200 import stca as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names |= set(re.findall(r"\b(stca_\w+)\s*\(", src))
    return sorted(names)


def test_header_declares_the_boundary():
    names = declared_functions()
    for must in ("stca_init", "stca_encode", "stca_forward", "stca_destroy"):
        assert must in names


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(S.LIB_PATH)
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing
    assert set(declared_functions()) == set(B.EXPORTS)


@pytest.mark.parametrize("off,total,nonempty,ok", [
    ([0, 3, 5], 5, True, True),
    ([0, 5], 5, True, True),
    ([0, 3, 3], 3, True, False),      # empty history
    ([0, 3, 3], 3, False, True),      # empty target list is fine
    ([1, 3], 3, True, False),         # must start at 0
    ([0, 4, 3], 3, True, False),      # decreasing
    ([0, 3, 5], 6, True, False),      # wrong total
    ([0], 0, True, False),            # R = 0
])
def test_validate_offsets(off, total, nonempty, ok):
    rc = S.stca_validate_offsets(off, total, nonempty)
    assert (rc == 0) == ok
    if not ok:
        assert rc == B.STCA_EINVAL and S.stca_last_error()


def _weights(d, r, M, dtype=np.float32):
    rng = np.random.default_rng(0)
    z = lambda *s: rng.standard_normal(s).astype(dtype)  # noqa: E731
    return {"Wu": [z(d, r * d) for _ in range(M)], "Wg": [z(d, r * d) for _ in range(M)],
            "Wd": [z(r * d, d) for _ in range(M)], "Wq": [z(d, d) for _ in range(M)],
            "Wk": [z(d, d) for _ in range(M)], "Wv": [z(d, d) for _ in range(M)],
            "Wo": [z(d, d) for _ in range(M)],
            "Wc": [None] + [z((i + 1) * d, d) for i in range(1, M)]}


@pytest.mark.parametrize("d,h,r,M,dtype,word", [
    (12, 2, 1, 1, S.STCA_F32, "d must"),      # d % 8
    (16, 3, 1, 1, S.STCA_F32, "h must"),      # h does not divide d
    (16, 16, 1, 1, S.STCA_F32, "even"),       # odd d / h
    (16, 2, 0, 1, S.STCA_F32, "r"),           # r < 1
    (16, 2, 1, 0, S.STCA_F32, "M must"),      # M < 1
    (16, 2, 1, 17, S.STCA_F32, "M must"),     # M too large
    (16, 2, 1, 1, 7, "dtype"),                # dtype
    (2048, 2, 1, 1, S.STCA_F32, "d must"),    # d too large
    (1024, 2, 8, 1, S.STCA_F32, "r*d"),       # r*d too large
])
def test_init_rejects_bad_sizes_on_host(d, h, r, M, dtype, word):
    out = ctypes.c_void_p()
    rc = B._lib.stca_init(ctypes.byref(B._Weights()), d, h, r, M, dtype, 0, ctypes.byref(out))
    assert rc == B.STCA_EINVAL and out.value is None
    assert word in S.stca_last_error()


def test_init_rejects_null_weight_fields_on_host():
    out = ctypes.c_void_p()
    rc = B._lib.stca_init(ctypes.byref(B._Weights()), 16, 2, 1, 1, S.STCA_F32, 0,
                          ctypes.byref(out))
    assert rc == B.STCA_EINVAL and "NULL" in S.stca_last_error()
    assert B._lib.stca_init(None, 16, 2, 1, 1, 0, 0, ctypes.byref(out)) == B.STCA_EINVAL


def test_init_rejects_missing_fusion_weights():
    w = _weights(8, 1, 2)
    w["Wc"] = None
    with pytest.raises((S.StcaError, ValueError)):
        B.stca_init(w, 8, 2, 1, 2, S.STCA_F32)


def test_null_handle_calls_fail_cleanly():
    lib = B._lib
    off = (ctypes.c_int64 * 2)(0, 4)
    assert lib.stca_encode(None, None, off, 1, 4, None) == B.STCA_EINVAL
    assert lib.stca_forward(None, None, off, 4, None, None) == B.STCA_EINVAL
    assert lib.stca_encode_forward(None, None, off, 1, 4, None, off, 4, None, None) == B.STCA_EINVAL
    assert lib.stca_set_option(None, 1, 0) == B.STCA_EINVAL
    v = ctypes.c_int64()
    assert lib.stca_get_option(None, 1, ctypes.byref(v)) == B.STCA_EINVAL
    assert lib.stca_device_status(None, None) == B.STCA_EINVAL
    assert lib.stca_head(None, None, 4, None, None, None) == B.STCA_EINVAL
    assert lib.stca_forward_head(None, None, off, 4, None, None, None) == B.STCA_EINVAL
    assert lib.stca_forward_static(None, None, off, 4, None, None) == B.STCA_EINVAL
    assert lib.stca_get_encoded(None, 0, None, None) == B.STCA_EINVAL
    ms = (ctypes.c_double * 4)()
    n = (ctypes.c_int64 * 4)()
    assert lib.stca_kernel_times(None, ms, n, 4) == B.STCA_EINVAL
    # the backward pieces
    assert lib.stca_encode_backward(None, 0, None, 4, None, None, None, None, None, None, None,
                                    None) == B.STCA_EINVAL
    assert lib.stca_attention_backward(None, 0, None, off, 4, None, None, None, None) == B.STCA_EINVAL
    assert lib.stca_output_backward(None, 0, None, 4, None, None, None, None, None) == B.STCA_EINVAL
    assert lib.stca_query_backward(None, 0, None, 4, None, None, None, None, None) == B.STCA_EINVAL
    assert lib.stca_query_init_backward(None, None, 4, None, None, None, None, None, None, None,
                                        None) == B.STCA_EINVAL
    assert lib.stca_fusion_backward(None, 1, None, None, 4, None, 0, None, None, None, None, None, None,
                                    None) == B.STCA_EINVAL
    assert "NULL" in S.stca_last_error()
    lib.stca_destroy(None)   # accepted


@pytest.mark.parametrize("given", [("Wz",), ("Wz", "zWu", "zWg"), ("zWd",)])
def test_init_rejects_partial_head_weights_on_host(given):
    # the four prediction-head matrices of Eq. (9) come together or not at all
    d, r, M = 8, 1, 1
    w = _weights(d, r, M)
    shapes = {"Wz": ((M + 1) * d, d), "zWu": (d, r * d), "zWg": (d, r * d), "zWd": (r * d, d)}
    for k in given:
        w[k] = np.ones(shapes[k], dtype=np.float32)
    with pytest.raises(S.StcaError) as e:
        B.stca_init(w, d, 2, r, M, S.STCA_F32)
    assert e.value.code == B.STCA_EINVAL and "together" in str(e.value)


def test_weight_dtype_checked_by_binding():
    w = _weights(8, 1, 1, dtype=np.float64)
    with pytest.raises(TypeError):
        B.stca_init(w, 8, 2, 1, 1, S.STCA_F32)
