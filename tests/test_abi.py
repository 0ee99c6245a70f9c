"""The C ABI on the host: the library loads, exports every function include/kvq.h
declares, and rejects bad arguments before touching a device (no GPU needed)."""
import ctypes
import ctypes.util
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "kvq.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(kvq_[a-z_]+)\s*\(", src)))


def test_header_declares_the_boundary():
    names = _declared()
    for n in ("kvq_plan_create", "kvq_plan_destroy", "kvq_encode", "kvq_encode_batch", "kvq_decode",
              "kvq_workspace_size", "kvq_attend_decode", "kvq_attend_decode_ref", "kvq_status_string",
              "kvq_last_error", "kvq_poll_device_errors", "kvq_attend_decode_batch",
              "kvq_attend_decode_noalloc", "kvq_attend_decode_append", "kvq_plan_create_transform",
              "kvq_plan_transform", "kvq_plan_create_ex", "kvq_plan_bits", "kvq_attend_split_info",
              "kvq_debug_wait_timeout", "kvq_set_decode_path", "kvq_get_decode_path"):
        assert n in names


def test_library_exports_every_declared_symbol():
    from rotated_int4_kv_b200 import LIB_PATH

    lib = ctypes.CDLL(LIB_PATH)
    missing = [n for n in _declared() if not hasattr(lib, n)]
    assert not missing, missing


def test_status_strings_and_host_checks():
    from rotated_int4_kv_b200 import _lib as kvq_lib
    from rotated_int4_kv_b200 import lib

    assert lib.kvq_status_string(0) == b"ok"
    assert lib.kvq_status_string(-4) == b"cache capacity exceeded"
    P = ctypes.c_void_p
    # null plan / bad sizes are refused on the host, before any CUDA call
    assert lib.kvq_encode(None, None, 1, 1, 1, None, None, 4, 0, None) == -1
    assert lib.kvq_decode(None, None, None, 1, 1, 4, 0, 1, None, None) == -1
    assert lib.kvq_attend_decode(None, None, None, None, None, None, None, 1, 4, 1, 64, None, 64,
                                 ctypes.c_float(0), None, None, 0, None) == -1
    assert lib.kvq_attend_decode_ref(None, None, None, 1, 4, 1, 100, 64, None, 64, ctypes.c_float(0), None, None,
                                     0, None) == -2
    assert lib.kvq_attend_decode_append(None, None, None, None, None, None, None, None, None, 1, 4, 1, 64, 10,
                                        ctypes.c_float(0), None, None, 0, None) == -1
    assert b"null plan" in lib.kvq_last_error()
    assert lib.kvq_attend_decode_partial(None, None, None, None, None, None, None, 1, 4, 1, 64, 0, 32,
                                         ctypes.c_float(0), None, None, 0, None) == -1
    assert lib.kvq_attend_combine(None, None, 2, 1, 4, None, None) == -1
    assert lib.kvq_encode_batch(None, -1, None) == -1
    assert lib.kvq_encode_batch(None, 0, None) == 0
    assert lib.kvq_attend_decode_batch(None, -1, 1, 4, 1, 64, None, 64, ctypes.c_float(0), None, 0, None) == -1
    assert lib.kvq_attend_decode_batch(None, 0, 1, 4, 1, 64, None, 64, ctypes.c_float(0), None, 0, None) == 0
    # planning query and the wait self-test: argument checks before any device call
    assert lib.kvq_attend_split_info(0, 8, 1, 128, 32, 4, 1024, None, None, None) == -1
    assert lib.kvq_attend_split_info(1, 6, 4, 128, 32, 4, 1024, None, None, None) == -2
    assert lib.kvq_attend_split_info(1, 8, 1, 96, 32, 4, 1024, None, None, None) == -2
    assert lib.kvq_attend_split_info(1, 8, 1, 128, 32, 5, 1024, None, None, None) == -2
    # decode kernel selection: 0 (tensor cores, the default) or 1 (register FFT)
    assert lib.kvq_get_decode_path() == 0
    assert lib.kvq_set_decode_path(2) == -1 and lib.kvq_set_decode_path(-1) == -1
    assert lib.kvq_get_decode_path() == 0
    assert lib.kvq_set_decode_path(1) == 0 and lib.kvq_get_decode_path() == 1
    assert lib.kvq_set_decode_path(0) == 0
    assert lib.kvq_debug_wait_timeout(0, None) == -1
    assert lib.kvq_debug_wait_timeout(2000000, None) == -1
    jobs = (kvq_lib.AttendJob * 2)()  # null plans: refused before any CUDA call
    assert lib.kvq_attend_decode_batch(jobs, 2, 1, 4, 1, 64, None, 64, ctypes.c_float(0), None, 0, None) == -1
    assert b"job 0" in lib.kvq_last_error()
    h = P()
    signs = (ctypes.c_int8 * 128)(*([1] * 128))
    lam = (ctypes.c_float * 128)(*([1.0] * 128))
    assert lib.kvq_plan_create(ctypes.byref(h), 96, 32, signs, lam) == -2      # head_dim
    assert lib.kvq_plan_create(ctypes.byref(h), 128, 24, signs, lam) == -2     # group
    assert lib.kvq_plan_create_transform(ctypes.byref(h), 128, 32, signs, lam, 2) == -2  # transform
    assert lib.kvq_plan_transform(None) == -1
    assert lib.kvq_plan_create_ex(ctypes.byref(h), 128, 32, signs, lam, 0, 5) == -2  # code width
    assert b"bits" in lib.kvq_last_error()
    assert lib.kvq_plan_bits(None) == -1
    bad = (ctypes.c_int8 * 128)(*([1] * 127 + [0]))
    assert lib.kvq_plan_create(ctypes.byref(h), 128, 32, bad, lam) == -1       # sign value
    neg = (ctypes.c_float * 128)(*([1.0] * 127 + [-1.0]))
    assert lib.kvq_plan_create(ctypes.byref(h), 128, 32, signs, neg) == -1     # lambda value
    assert b"lambda" in lib.kvq_last_error()


def test_workspace_size_is_monotone_in_capacity():
    from rotated_int4_kv_b200 import lib

    prev = 0
    for T in (0, 64, 1000, 4096, 32768, 131072):
        n = lib.kvq_workspace_size(4, 64, 8, 128, T)
        assert n >= prev and n % 4 == 0
        prev = n
    assert lib.kvq_workspace_size(1, 12, 5, 128, 64) == 0   # Hq % Hkv != 0
    assert lib.kvq_workspace_size(1, 4, 1, 64, 64) == 0     # head_dim


def _has_gpu():
    try:
        import torch
        return torch.cuda.is_available()
    except Exception:
        return False


@pytest.mark.skipif(_has_gpu(), reason="a CUDA device is present")
def test_plan_create_without_gpu_fails_cleanly():
    from rotated_int4_kv_b200 import lib

    h = ctypes.c_void_p()
    signs = (ctypes.c_int8 * 128)(*([1] * 128))
    lam = (ctypes.c_float * 128)(*([1.0] * 128))
    assert lib.kvq_plan_create(ctypes.byref(h), 128, 32, signs, lam) == -7
