"""B200-native SRFT-int4 KV-cache compression and decode attention.

The compute path lives in ``libkvq.so`` (hand-written CUDA for sm_100a, C ABI in
``include/kvq.h``); this package only marshals torch tensors into it.
"""
from ._lib import LIB_PATH, KvqError, lib  # noqa: F401
from .cache import Int4KVCache  # noqa: F401
from .api import (Plan, attend_combine, attend_decode, attend_decode_append, attend_decode_batch,  # noqa: F401
                  attend_decode_context_parallel, attend_decode_noalloc, attend_decode_partial, attend_decode_ref,
                  attend_split_info, debug_wait_timeout, gather_partials,
                  decode, encode, encode_batch, get_decode_path, get_encode_path, make_workspace, poll_device_errors,
                  set_decode_path, set_encode_path, workspace_size)

__all__ = ["Plan", "Int4KVCache", "attend_decode_partial", "attend_combine", "gather_partials",
           "attend_decode_context_parallel", "encode", "encode_batch", "decode", "attend_decode", "attend_decode_append", "attend_decode_batch",
           "attend_decode_noalloc", "attend_decode_ref", "attend_split_info", "debug_wait_timeout", "workspace_size", "make_workspace", "poll_device_errors",
           "set_encode_path", "get_encode_path", "set_decode_path", "get_decode_path",
           "KvqError", "LIB_PATH", "lib"]
