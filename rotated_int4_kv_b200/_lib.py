"""ctypes loader for the in-tree ``libkvq.so``; fails loudly when it is missing."""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libkvq.so")

KVQ_OK = 0
STATUS_NAMES = {0: "KVQ_OK", -1: "KVQ_ERR_INVALID_ARG", -2: "KVQ_ERR_UNSUPPORTED", -3: "KVQ_ERR_ALIGNMENT",
                -4: "KVQ_ERR_CAPACITY", -5: "KVQ_ERR_CUDA", -6: "KVQ_ERR_WORKSPACE", -7: "KVQ_ERR_DEVICE"}


class KvqError(RuntimeError):
    def __init__(self, status: int, where: str, detail: str):
        self.status = status
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)} ({detail})")


class EncodeJob(ctypes.Structure):
    """Mirror of ``kvq_encode_job`` in include/kvq.h."""
    _fields_ = [("plan", ctypes.c_void_p), ("x", ctypes.c_void_p), ("codes", ctypes.c_void_p),
                ("scales", ctypes.c_void_p), ("B", ctypes.c_int), ("H", ctypes.c_int), ("n", ctypes.c_int),
                ("T_cap", ctypes.c_int), ("pos", ctypes.c_int)]


class AttendJob(ctypes.Structure):
    """Mirror of ``kvq_attend_job`` in include/kvq.h."""
    _fields_ = [("pk", ctypes.c_void_p), ("pv", ctypes.c_void_p), ("q", ctypes.c_void_p),
                ("k_codes", ctypes.c_void_p), ("k_scales", ctypes.c_void_p), ("v_codes", ctypes.c_void_p),
                ("v_scales", ctypes.c_void_p), ("out", ctypes.c_void_p)]


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with `python rotated_int4_kv_b200/build.py` "
                          "(nvcc, sm_100a). There is no fallback implementation.")
    lib = ctypes.CDLL(LIB_PATH)
    P, I, F, S, U32P = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t, ctypes.POINTER(ctypes.c_uint32)
    sig = {
        "kvq_plan_create": (I, [ctypes.POINTER(P), I, I, P, P]),
        "kvq_plan_create_transform": (I, [ctypes.POINTER(P), I, I, P, P, I]),
        "kvq_plan_transform": (I, [P]),
        "kvq_plan_create_ex": (I, [ctypes.POINTER(P), I, I, P, P, I, I]),
        "kvq_plan_bits": (I, [P]),
        "kvq_plan_destroy": (I, [P]),
        "kvq_plan_head_dim": (I, [P]),
        "kvq_plan_group": (I, [P]),
        "kvq_encode": (I, [P, P, I, I, I, P, P, I, I, P]),
        "kvq_encode_batch": (I, [ctypes.POINTER(EncodeJob), I, P]),
        "kvq_decode": (I, [P, P, P, I, I, I, I, I, P, P]),
        "kvq_workspace_size": (S, [I, I, I, I, I]),
        "kvq_attend_decode": (I, [P, P, P, P, P, P, P, I, I, I, I, P, I, F, P, P, S, P]),
        "kvq_attend_decode_append": (I, [P, P, P, P, P, P, P, P, P, I, I, I, I, I, F, P, P, S, P]),
        "kvq_attend_decode_partial": (I, [P, P, P, P, P, P, P, I, I, I, I, I, I, F, P, P, S, P]),
        "kvq_attend_combine": (I, [P, P, I, I, I, P, P]),
        "kvq_attend_decode_ref": (I, [P, P, P, I, I, I, I, I, P, I, F, P, P, S, P]),
        "kvq_attend_decode_noalloc": (I, [P, P, P, P, P, P, P, I, I, I, I, P, I, F, P, P]),
        "kvq_attend_decode_batch": (I, [ctypes.POINTER(AttendJob), I, I, I, I, I, P, I, F, P, S, P]),
        "kvq_poll_device_errors": (I, [U32P]),
        "kvq_attend_split_info": (I, [I, I, I, I, I, I, I, ctypes.POINTER(I), ctypes.POINTER(I), ctypes.POINTER(I)]),
        "kvq_debug_wait_timeout": (I, [ctypes.c_uint32, P]),
        "kvq_set_encode_path": (I, [I]),
        "kvq_get_encode_path": (I, []),
        "kvq_set_decode_path": (I, [I]),
        "kvq_get_decode_path": (I, []),
        "kvq_status_string": (ctypes.c_char_p, [I]),
        "kvq_last_error": (ctypes.c_char_p, []),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


lib = _load()


def check(status: int, where: str) -> None:
    if status != KVQ_OK:
        raise KvqError(status, where, lib.kvq_last_error().decode(errors="replace"))
