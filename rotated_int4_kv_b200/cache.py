"""A preallocated int4 KV cache over the library's entry points.

The pages put their fused encode kernel behind a cache object of the model runtime
("When Quantization Is Free", gist.science/de/paper/2605.05699, "Methodik" 2): every
new K/V row is compressed on arrival and attention reads the compressed cache. This
class is the torch-level counterpart: it owns the per-layer code and scale buffers,
the (s, lambda) plans and the write position, and every operation is one or two
calls into libkvq (no arithmetic here).
"""
from __future__ import annotations

import numpy as np
import torch

from .api import (Plan, attend_decode, attend_decode_append, decode, encode_batch, make_workspace)


class Int4KVCache:
    """Per-layer int4 K and V caches of ``capacity`` tokens for ``batch`` sequences.

    ``k_params`` / ``v_params``: one (signs, lambda) pair for every layer, or a list of
    ``layers`` pairs (K and V get separate transforms); ``transform`` "srft" or "srht";
    ``bits`` 4 (int4 codes) or 8 (int8 codes). All sequences of the batch share the
    write position of a layer.
    """

    def __init__(self, layers: int, batch: int, kv_heads: int, head_dim: int, capacity: int, k_params, v_params,
                 device=None, group: int = 32, transform: str = "srft", bits: int = 4):
        if layers <= 0 or batch <= 0 or kv_heads <= 0 or capacity <= 0:
            raise ValueError("layers, batch, kv_heads and capacity must be positive")
        self.device = torch.device(device) if device is not None else torch.device("cuda")
        self.layers, self.batch, self.kv_heads, self.head_dim, self.group = layers, batch, kv_heads, head_dim, group
        self.bits = bits
        self.capacity = capacity + (capacity & 1)  # the attention kernels fetch scale rows in 16-byte units

        def per_layer(params):
            # one (signs, lambda) pair, or a list of one pair per layer
            first = np.asarray(params[0])
            if first.ndim == 1:
                return [params] * layers
            if len(params) != layers:
                raise ValueError(f"expected one (signs, lambda) pair or {layers} of them")
            return list(params)

        with torch.cuda.device(self.device):
            self.k_plans = [Plan(s, lam, group, transform, bits) for s, lam in per_layer(k_params)]
            self.v_plans = [Plan(s, lam, group, transform, bits) for s, lam in per_layer(v_params)]
        shape_c = (batch, kv_heads, self.capacity, head_dim * bits // 8)
        shape_s = (batch, kv_heads, self.capacity, head_dim // group)
        self.k_codes = [torch.zeros(shape_c, dtype=torch.uint8, device=self.device) for _ in range(layers)]
        self.v_codes = [torch.zeros(shape_c, dtype=torch.uint8, device=self.device) for _ in range(layers)]
        self.k_scales = [torch.zeros(shape_s, dtype=torch.float16, device=self.device) for _ in range(layers)]
        self.v_scales = [torch.zeros(shape_s, dtype=torch.float16, device=self.device) for _ in range(layers)]
        self.pos = [0] * layers
        self._ws = {}

    # -------------------------------------------------------------- bookkeeping
    def seq_length(self, layer: int = 0) -> int:
        return self.pos[layer]

    def reset(self) -> None:
        self.pos = [0] * self.layers

    def memory_bytes(self) -> int:
        """Device bytes of all code and scale buffers."""
        per = sum(t.numel() * t.element_size() for t in (self.k_codes[0], self.v_codes[0], self.k_scales[0],
                                                          self.v_scales[0]))
        return per * self.layers

    @staticmethod
    def compression_ratio(head_dim: int, group: int = 32, bits: int = 4) -> float:
        """fp16 K/V bytes over code + fp16 scale bytes for the same tokens (int4: 3.56 at G = 32)."""
        return (2 * head_dim) / (head_dim * bits // 8 + 2 * (head_dim // group))

    def compression_vs_fp16(self) -> float:
        return self.compression_ratio(self.head_dim, self.group, self.bits)

    def _workspace(self, q_heads: int) -> torch.Tensor:
        ws = self._ws.get(q_heads)
        if ws is None:
            ws = make_workspace(self.batch, q_heads, self.kv_heads, self.head_dim, self.capacity, self.device)
            self._ws[q_heads] = ws
        return ws

    def _room(self, layer: int, n: int) -> None:
        if self.pos[layer] + n > self.capacity:
            raise ValueError(f"layer {layer}: {self.pos[layer]} + {n} tokens exceed the capacity {self.capacity}")

    # -------------------------------------------------------------- operations
    def update(self, layer: int, k: torch.Tensor, v: torch.Tensor, stream=None) -> None:
        """Append n tokens: k, v fp16 [batch, kv_heads, n, head_dim] (one grouped encode launch)."""
        n = k.shape[2]
        if tuple(v.shape) != tuple(k.shape):
            raise ValueError("k and v must have the same shape")
        self._room(layer, n)
        p = self.pos[layer]
        encode_batch([(self.k_plans[layer], k, self.k_codes[layer], self.k_scales[layer], p),
                      (self.v_plans[layer], v, self.v_codes[layer], self.v_scales[layer], p)], stream=stream)
        self.pos[layer] = p + n

    def attend(self, layer: int, q: torch.Tensor, out=None, softmax_scale: float = 0.0, stream=None) -> torch.Tensor:
        """One-query attention of q fp16 [batch, q_heads, head_dim] over the cached tokens."""
        return attend_decode(self.k_plans[layer], self.v_plans[layer], q, self.k_codes[layer], self.k_scales[layer],
                             self.v_codes[layer], self.v_scales[layer], T_len=self.pos[layer],
                             softmax_scale=softmax_scale, out=out, workspace=self._workspace(q.shape[1]),
                             stream=stream)

    def step(self, layer: int, q: torch.Tensor, k_new: torch.Tensor, v_new: torch.Tensor, out=None,
             softmax_scale: float = 0.0, stream=None) -> torch.Tensor:
        """One decode step in one launch: append the token k_new, v_new (fp16 [batch, kv_heads, head_dim]
        or [batch, kv_heads, 1, head_dim]) and attend over the cache including it."""
        self._room(layer, 1)
        p = self.pos[layer]
        o = attend_decode_append(self.k_plans[layer], self.v_plans[layer], q, k_new, v_new, self.k_codes[layer],
                                 self.k_scales[layer], self.v_codes[layer], self.v_scales[layer], p,
                                 softmax_scale=softmax_scale, out=out, workspace=self._workspace(q.shape[1]),
                                 stream=stream)
        self.pos[layer] = p + 1
        return o

    def dequantize(self, layer: int, t0: int = 0, n: int = None, stream=None):
        """(K, V) fp16 [batch, kv_heads, n, head_dim] of cached tokens t0 .. t0 + n - 1 (decode kernel)."""
        if n is None:
            n = self.pos[layer] - t0
        k = decode(self.k_plans[layer], self.k_codes[layer], self.k_scales[layer], t0, n, stream=stream)
        v = decode(self.v_plans[layer], self.v_codes[layer], self.v_scales[layer], t0, n, stream=stream)
        return k, v
