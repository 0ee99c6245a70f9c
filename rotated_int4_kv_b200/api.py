"""torch-facing wrappers over the C ABI (argument marshalling only).

Every call passes raw device pointers and the current CUDA stream to
``libkvq.so``; all arithmetic runs in the library's CUDA kernels.
"""
from __future__ import annotations

import ctypes

import numpy as np
import torch

from ._lib import AttendJob, EncodeJob, check, lib


def _stream(stream) -> ctypes.c_void_p:
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _ptr(t) -> ctypes.c_void_p:
    return ctypes.c_void_p(0 if t is None else t.data_ptr())


def _need(t: torch.Tensor, name: str, dtype, shape=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.device.type != "cuda":
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


TRANSFORMS = {"srft": 0, "srht": 1}


class Plan:
    """A (sign vector s, lambda) transform plan on the current CUDA device; transform
    "srft" (the pages' method, default) or "srht" (the Hadamard variant); bits 4 (int4
    codes, two per byte, default) or 8 (int8 codes, one byte each). Code buffers hold
    head_dim * bits / 8 bytes per cached vector."""

    def __init__(self, signs, lam, group: int = 32, transform: str = "srft", bits: int = 4):
        s = np.ascontiguousarray(np.asarray(signs, dtype=np.int8))
        l = np.ascontiguousarray(np.asarray(lam, dtype=np.float32))
        if s.ndim != 1 or l.shape != s.shape:
            raise ValueError("signs and lambda must be 1-D arrays of the same length")
        if transform not in TRANSFORMS:
            raise ValueError(f"transform must be one of {sorted(TRANSFORMS)}")
        self.head_dim = int(s.shape[0])
        self.group = int(group)
        self.transform = transform
        self.bits = int(bits)
        self._h = ctypes.c_void_p()
        check(lib.kvq_plan_create_ex(ctypes.byref(self._h), self.head_dim, self.group,
                                     s.ctypes.data_as(ctypes.c_void_p), l.ctypes.data_as(ctypes.c_void_p),
                                     TRANSFORMS[transform], self.bits),
              "kvq_plan_create_ex")
        self._lib = lib

    @property
    def code_row_bytes(self) -> int:
        return self.head_dim * self.bits // 8

    @property
    def handle(self) -> ctypes.c_void_p:
        return self._h

    def close(self) -> None:
        if getattr(self, "_h", None) and self._h.value:
            self._lib.kvq_plan_destroy(self._h)
            self._h = ctypes.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def encode(plan: Plan, x: torch.Tensor, codes: torch.Tensor, scales: torch.Tensor, pos: int = 0,
           stream=None) -> None:
    """Encode x [B, H, n, D] fp16 into cache rows pos..pos+n-1 of codes / scales."""
    B, H, n, D = x.shape
    _same_dim(D, plan)
    T_cap = codes.shape[2]
    _need(x, "x", torch.float16)
    _need(codes, "codes", torch.uint8, (B, H, T_cap, D * plan.bits // 8))
    _need(scales, "scales", torch.float16, (B, H, T_cap, D // plan.group))
    check(lib.kvq_encode(plan.handle, _ptr(x), B, H, n, _ptr(codes), _ptr(scales), T_cap, int(pos),
                         _stream(stream)), "kvq_encode")


def encode_batch(jobs, stream=None) -> None:
    """Grouped encode: ``jobs`` is a sequence of (plan, x, codes, scales, pos) tuples,
    each exactly what :func:`encode` takes; all run in one launch (up to 64 per launch)."""
    arr = (EncodeJob * max(1, len(jobs)))()
    for i, (plan, x, codes, scales, pos) in enumerate(jobs):
        B, H, n, D = x.shape
        _same_dim(D, plan)
        T_cap = codes.shape[2]
        _need(x, f"jobs[{i}].x", torch.float16)
        _need(codes, f"jobs[{i}].codes", torch.uint8, (B, H, T_cap, D * plan.bits // 8))
        _need(scales, f"jobs[{i}].scales", torch.float16, (B, H, T_cap, D // plan.group))
        arr[i] = EncodeJob(plan.handle.value, x.data_ptr(), codes.data_ptr(), scales.data_ptr(), B, H, n, T_cap,
                           int(pos))
    check(lib.kvq_encode_batch(arr, len(jobs), _stream(stream)), "kvq_encode_batch")


ENCODE_PATHS = {"auto": 0, "fft": 1, "tensor": 2, "split": 3}


def set_encode_path(path: str) -> None:
    """Select the encode kernel: "auto" (tensor cores where supported), "fft"
    (register FFT), "tensor" (tensor cores, dense product) or "split" (tensor cores,
    radix-2 split; head_dim 256 SRFT plans only)."""
    check(lib.kvq_set_encode_path(ENCODE_PATHS[path]), "kvq_set_encode_path")


def get_encode_path() -> str:
    v = int(lib.kvq_get_encode_path())
    return {n: k for k, n in ENCODE_PATHS.items()}[v]


DECODE_PATHS = {"tensor": 0, "fft": 1}


def set_decode_path(path: str) -> None:
    """Select the decode kernel: "tensor" (default: fp16 dequantised codes times the
    plan's fp16 decode matrix on the tensor cores) or "fft" (register inverse transform
    in fp32)."""
    check(lib.kvq_set_decode_path(DECODE_PATHS[path]), "kvq_set_decode_path")


def get_decode_path() -> str:
    v = int(lib.kvq_get_decode_path())
    return {n: k for k, n in DECODE_PATHS.items()}[v]


def decode(plan: Plan, codes: torch.Tensor, scales: torch.Tensor, t0: int, n: int, out: torch.Tensor = None,
           stream=None) -> torch.Tensor:
    """Decode cache rows t0..t0+n-1 into fp16 [B, H, n, D]."""
    B, H, T_cap, _ = codes.shape
    D = plan.head_dim
    _need(codes, "codes", torch.uint8, (B, H, T_cap, plan.code_row_bytes))
    _need(scales, "scales", torch.float16, (B, H, T_cap, D // plan.group))
    if out is None:
        out = torch.empty((B, H, n, D), dtype=torch.float16, device=codes.device)
    _need(out, "out", torch.float16, (B, H, n, D))
    check(lib.kvq_decode(plan.handle, _ptr(codes), _ptr(scales), B, H, T_cap, int(t0), int(n), _ptr(out),
                         _stream(stream)), "kvq_decode")
    return out


def _same_dim(D: int, *plans) -> None:
    """The C ABI sizes every row by the plan's head_dim; a tensor of another head_dim
    would be read or written past its end, so it is refused here."""
    for pl in plans:
        if pl.head_dim != D:
            raise ValueError(f"tensor head_dim {D} does not match the plan's head_dim {pl.head_dim}")


def workspace_size(B: int, Hq: int, Hkv: int, head_dim: int, T_cap: int) -> int:
    return int(lib.kvq_workspace_size(B, Hq, Hkv, head_dim, T_cap))


def make_workspace(B: int, Hq: int, Hkv: int, head_dim: int, T_cap: int, device=None) -> torch.Tensor:
    """A zero-initialised workspace (its counters must start at zero)."""
    n = max(16, workspace_size(B, Hq, Hkv, head_dim, T_cap))
    return torch.zeros(n, dtype=torch.uint8, device=device or torch.device("cuda"))


def attend_decode(pk: Plan, pv: Plan, q, k_codes, k_scales, v_codes, v_scales, seq_lens=None, T_len=None,
                  softmax_scale: float = 0.0, out=None, workspace=None, stream=None) -> torch.Tensor:
    """One-query decode attention on the packed int4 cache (rotated domain)."""
    B, Hq, D = q.shape
    _same_dim(D, pk, pv)
    _, Hkv, T_cap, half = k_codes.shape
    _need(q, "q", torch.float16)
    for name, t in (("k_codes", k_codes), ("v_codes", v_codes)):
        _need(t, name, torch.uint8, (B, Hkv, T_cap, D * pk.bits // 8))
    for name, t in (("k_scales", k_scales), ("v_scales", v_scales)):
        _need(t, name, torch.float16, (B, Hkv, T_cap, D // pk.group))
    if seq_lens is not None:
        _need(seq_lens, "seq_lens", torch.int32, (B,))
    if T_len is None:
        T_len = T_cap if seq_lens is None else 0
    if out is None:
        out = torch.empty((B, Hq, D), dtype=torch.float16, device=q.device)
    _need(out, "out", torch.float16, (B, Hq, D))
    if workspace is None:
        workspace = make_workspace(B, Hq, Hkv, D, T_cap, q.device)
    check(lib.kvq_attend_decode(pk.handle, pv.handle, _ptr(q), _ptr(k_codes), _ptr(k_scales), _ptr(v_codes),
                                _ptr(v_scales), B, Hq, Hkv, T_cap, _ptr(seq_lens), int(T_len),
                                float(softmax_scale), _ptr(out), _ptr(workspace), workspace.numel(),
                                _stream(stream)), "kvq_attend_decode")
    return out


def attend_decode_append(pk: Plan, pv: Plan, q, k_new, v_new, k_codes, k_scales, v_codes, v_scales, pos: int,
                         softmax_scale: float = 0.0, out=None, workspace=None, stream=None) -> torch.Tensor:
    """One decode step in one launch: encode the new token's K and V rows (fp16
    [B, Hkv, D] or [B, Hkv, 1, D]) into the caches at token ``pos`` and attend over
    tokens 0 .. pos (see kvq_attend_decode_append)."""
    B, Hq, D = q.shape
    _same_dim(D, pk, pv)
    _, Hkv, T_cap, _ = k_codes.shape
    _need(q, "q", torch.float16)
    for name, t in (("k_new", k_new), ("v_new", v_new)):
        if tuple(t.shape) not in ((B, Hkv, D), (B, Hkv, 1, D)):
            raise ValueError(f"{name}: expected shape {(B, Hkv, D)}, got {tuple(t.shape)}")
        _need(t, name, torch.float16)
    for name, t in (("k_codes", k_codes), ("v_codes", v_codes)):
        _need(t, name, torch.uint8, (B, Hkv, T_cap, D * pk.bits // 8))
    for name, t in (("k_scales", k_scales), ("v_scales", v_scales)):
        _need(t, name, torch.float16, (B, Hkv, T_cap, D // pk.group))
    if out is None:
        out = torch.empty((B, Hq, D), dtype=torch.float16, device=q.device)
    _need(out, "out", torch.float16, (B, Hq, D))
    if workspace is None:
        workspace = make_workspace(B, Hq, Hkv, D, T_cap, q.device)
    check(lib.kvq_attend_decode_append(pk.handle, pv.handle, _ptr(q), _ptr(k_new), _ptr(v_new), _ptr(k_codes),
                                       _ptr(k_scales), _ptr(v_codes), _ptr(v_scales), B, Hq, Hkv, T_cap, int(pos),
                                       float(softmax_scale), _ptr(out), _ptr(workspace), workspace.numel(),
                                       _stream(stream)), "kvq_attend_decode_append")
    return out


def attend_decode_partial(pk: Plan, pv: Plan, q, k_codes, k_scales, v_codes, v_scales, t_begin: int, t_end: int,
                          softmax_scale: float = 0.0, partial=None, workspace=None, stream=None) -> torch.Tensor:
    """Sequence-sharded decode, step 1: the softmax partial of every query head over
    cached tokens [t_begin, t_end) (fp32 [B, Hq, D + 4]; see kvq_attend_decode_partial)."""
    B, Hq, D = q.shape
    _same_dim(D, pk, pv)
    _, Hkv, T_cap, _ = k_codes.shape
    _need(q, "q", torch.float16)
    for name, t in (("k_codes", k_codes), ("v_codes", v_codes)):
        _need(t, name, torch.uint8, (B, Hkv, T_cap, D * pk.bits // 8))
    for name, t in (("k_scales", k_scales), ("v_scales", v_scales)):
        _need(t, name, torch.float16, (B, Hkv, T_cap, D // pk.group))
    if partial is None:
        partial = torch.empty((B, Hq, D + 4), dtype=torch.float32, device=q.device)
    _need(partial, "partial", torch.float32, (B, Hq, D + 4))
    if workspace is None:
        workspace = make_workspace(B, Hq, Hkv, D, T_cap, q.device)
    check(lib.kvq_attend_decode_partial(pk.handle, pv.handle, _ptr(q), _ptr(k_codes), _ptr(k_scales), _ptr(v_codes),
                                        _ptr(v_scales), B, Hq, Hkv, T_cap, int(t_begin), int(t_end),
                                        float(softmax_scale), _ptr(partial), _ptr(workspace), workspace.numel(),
                                        _stream(stream)), "kvq_attend_decode_partial")
    return partial


def attend_combine(pv: Plan, partials, out=None, stream=None) -> torch.Tensor:
    """Sequence-sharded decode, step 2: merge partials fp32 [N, B, Hq, D + 4] and un-rotate
    (see kvq_attend_combine); returns fp16 [B, Hq, D]."""
    N, B, Hq, D4 = partials.shape
    D = D4 - 4
    _same_dim(D, pv)
    _need(partials, "partials", torch.float32)
    if out is None:
        out = torch.empty((B, Hq, D), dtype=torch.float16, device=partials.device)
    _need(out, "out", torch.float16, (B, Hq, D))
    check(lib.kvq_attend_combine(pv.handle, _ptr(partials), N, B, Hq, _ptr(out), _stream(stream)),
          "kvq_attend_combine")
    return out


def gather_partials(partial: torch.Tensor, group=None) -> torch.Tensor:
    """All-gather of one softmax partial per rank of a context-parallel group (NCCL on
    GPUs; any torch.distributed backend): returns [world, *partial.shape], rank order."""
    import torch.distributed as dist

    world = dist.get_world_size(group)
    bufs = [torch.empty_like(partial) for _ in range(world)]
    dist.all_gather(bufs, partial.contiguous(), group=group)
    return torch.stack(bufs)


def attend_decode_context_parallel(pk: Plan, pv: Plan, q, k_codes, k_scales, v_codes, v_scales, t_begin: int,
                                   t_end: int, group=None, softmax_scale: float = 0.0, out=None,
                                   workspace=None) -> torch.Tensor:
    """Decode attention over a sequence sharded across the ranks of ``group``: each rank
    holds its slice [t_begin, t_end) of every (b, kv head) in its caches and passes the
    same q; the partials are all-gathered ((D + 4) * 4 bytes per query head per rank) and
    every rank merges them into the same output."""
    part = attend_decode_partial(pk, pv, q, k_codes, k_scales, v_codes, v_scales, t_begin, t_end,
                                 softmax_scale=softmax_scale, workspace=workspace)
    return attend_combine(pv, gather_partials(part, group), out=out)


def attend_decode_batch(jobs, seq_lens=None, T_len=None, softmax_scale: float = 0.0, workspace=None,
                        stream=None) -> list:
    """Grouped int4 decode attention: ``jobs`` is a sequence of
    (pk, pv, q, k_codes, k_scales, v_codes, v_scales[, out]) tuples of one shape,
    each exactly what :func:`attend_decode` takes; up to 32 run per launch.
    Returns the list of outputs."""
    if not jobs:
        return []
    q0, kc0 = jobs[0][2], jobs[0][3]
    B, Hq, D = q0.shape
    _, Hkv, T_cap, _ = kc0.shape
    arr = (AttendJob * len(jobs))()
    outs = []
    for i, job in enumerate(jobs):
        pk, pv, q, k_codes, k_scales, v_codes, v_scales = job[:7]
        _same_dim(D, pk, pv)
        out = job[7] if len(job) > 7 and job[7] is not None else torch.empty((B, Hq, D), dtype=torch.float16,
                                                                             device=q.device)
        _need(q, f"jobs[{i}].q", torch.float16, (B, Hq, D))
        for name, t in (("k_codes", k_codes), ("v_codes", v_codes)):
            _need(t, f"jobs[{i}].{name}", torch.uint8, (B, Hkv, T_cap, D * pk.bits // 8))
        for name, t in (("k_scales", k_scales), ("v_scales", v_scales)):
            _need(t, f"jobs[{i}].{name}", torch.float16, (B, Hkv, T_cap, D // pk.group))
        _need(out, f"jobs[{i}].out", torch.float16, (B, Hq, D))
        arr[i] = AttendJob(pk.handle.value, pv.handle.value, q.data_ptr(), k_codes.data_ptr(), k_scales.data_ptr(),
                           v_codes.data_ptr(), v_scales.data_ptr(), out.data_ptr())
        outs.append(out)
    if seq_lens is not None:
        _need(seq_lens, "seq_lens", torch.int32, (B,))
    if T_len is None:
        T_len = T_cap if seq_lens is None else 0
    if workspace is None:
        workspace = make_workspace(min(len(jobs), 32) * B, Hq, Hkv, D, T_cap, q0.device)
    check(lib.kvq_attend_decode_batch(arr, len(jobs), B, Hq, Hkv, T_cap, _ptr(seq_lens), int(T_len),
                                      float(softmax_scale), _ptr(workspace), workspace.numel(), _stream(stream)),
          "kvq_attend_decode_batch")
    return outs


def attend_decode_noalloc(pk: Plan, pv: Plan, q, k_codes, k_scales, v_codes, v_scales, seq_lens=None, T_len=None,
                          softmax_scale: float = 0.0, out=None, stream=None) -> torch.Tensor:
    """kvq_attend_decode_noalloc: the int4 decode attention for callers that cannot
    allocate device memory; its scratch is a static array inside the library
    (8 MiB, shared by all calls: calls that overlap on the GPU race)."""
    B, Hq, D = q.shape
    _same_dim(D, pk, pv)
    _, Hkv, T_cap, half = k_codes.shape
    _need(q, "q", torch.float16)
    for name, t in (("k_codes", k_codes), ("v_codes", v_codes)):
        _need(t, name, torch.uint8, (B, Hkv, T_cap, D * pk.bits // 8))
    for name, t in (("k_scales", k_scales), ("v_scales", v_scales)):
        _need(t, name, torch.float16, (B, Hkv, T_cap, D // pk.group))
    if seq_lens is not None:
        _need(seq_lens, "seq_lens", torch.int32, (B,))
    if T_len is None:
        T_len = T_cap if seq_lens is None else 0
    if out is None:
        out = torch.empty((B, Hq, D), dtype=torch.float16, device=q.device)
    _need(out, "out", torch.float16, (B, Hq, D))
    check(lib.kvq_attend_decode_noalloc(pk.handle, pv.handle, _ptr(q), _ptr(k_codes), _ptr(k_scales),
                                        _ptr(v_codes), _ptr(v_scales), B, Hq, Hkv, T_cap, _ptr(seq_lens),
                                        int(T_len), float(softmax_scale), _ptr(out), _stream(stream)),
          "kvq_attend_decode_noalloc")
    return out


def attend_decode_ref(q, k, v, seq_lens=None, T_len=None, softmax_scale: float = 0.0, out=None, workspace=None,
                      stream=None) -> torch.Tensor:
    """The fp16-cache comparator kernel on the same shapes."""
    B, Hq, D = q.shape
    _, Hkv, T_cap, _ = k.shape
    _need(q, "q", torch.float16)
    _need(k, "k", torch.float16, (B, Hkv, T_cap, D))
    _need(v, "v", torch.float16, (B, Hkv, T_cap, D))
    if seq_lens is not None:
        _need(seq_lens, "seq_lens", torch.int32, (B,))
    if T_len is None:
        T_len = T_cap if seq_lens is None else 0
    if out is None:
        out = torch.empty((B, Hq, D), dtype=torch.float16, device=q.device)
    _need(out, "out", torch.float16, (B, Hq, D))
    if workspace is None:
        workspace = make_workspace(B, Hq, Hkv, D, T_cap, q.device)
    check(lib.kvq_attend_decode_ref(_ptr(q), _ptr(k), _ptr(v), B, Hq, Hkv, D, T_cap, _ptr(seq_lens), int(T_len),
                                    float(softmax_scale), _ptr(out), _ptr(workspace), workspace.numel(),
                                    _stream(stream)), "kvq_attend_decode_ref")
    return out


def poll_device_errors() -> int:
    flags = ctypes.c_uint32(0)
    check(lib.kvq_poll_device_errors(ctypes.byref(flags)), "kvq_poll_device_errors")
    return int(flags.value)


def attend_split_info(B: int, Hq: int, Hkv: int, head_dim: int, T: int, group: int = 32, bits: int = 4):
    """(splits, cluster, head_tiles) that the attention entry points choose for these
    shapes on the current device (bits 16 = the fp16 comparator). A unit whose
    splits / cluster > 1 merges its cluster partials through the workspace."""
    s, c, h = ctypes.c_int(0), ctypes.c_int(0), ctypes.c_int(0)
    check(lib.kvq_attend_split_info(B, Hq, Hkv, head_dim, group, bits, T, ctypes.byref(s), ctypes.byref(c),
                                    ctypes.byref(h)), "kvq_attend_split_info")
    return int(s.value), int(c.value), int(h.value)


def debug_wait_timeout(limit_us: int, stream=None) -> None:
    """Launch the library's bounded-wait self-test: one CTA waits on a barrier that never
    completes with a budget of limit_us, then raises the load-timeout flag (1) that
    :func:`poll_device_errors` reports."""
    check(lib.kvq_debug_wait_timeout(int(limit_us), _stream(stream)), "kvq_debug_wait_timeout")
