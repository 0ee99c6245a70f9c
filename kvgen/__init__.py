"""Seeded synthetic inputs for the SRFT-int4 KV-cache path.

This module is the only code shared by the CPU oracle tests and the CUDA path's
tests and benchmark. It draws random numbers and nothing else: it holds none of
the method's arithmetic (no transform, no scaling rule, no quantiser, no
packing). What the method itself draws at random -- the fixed +/-1 sign vector
of the sign-randomised FFT and the per-channel lambda factors -- is drawn here
and handed to both sides as plain inputs.

Streams are keyed by ``numpy.random.SeedSequence(seed).spawn``-style keys
(layer, kind), so that each (layer, K-or-V) pair has its own independent draw
regardless of how many layers a workload has.

Workload recipes (shapes, value distributions), one per benchmark workload:

* ``toy``       1 layer, 1 KV head, D=128, 256 tokens, K and V ~ N(0,1) with 4
                 seed-chosen channels x20.
* ``gemma``     Gemma-3-1B-shaped prefill: 26 layers, 1 KV head, 4 query heads,
                 D=256, batch 1, prefix 4096, K/V ~ N(0,1) x per-channel
                 lognormal(sigma=1) scale.
* ``qwen``      Qwen2.5-1.5B-shaped decode: 28 layers, 2 KV heads, 12 query
                 heads, D=128, batch 1, context 256..4096; K ~ N(0,1) with 8
                 outlier channels x50, V ~ N(0,1).
* ``mistral``   Mistral-7B-shaped batched decode: 32 layers, 8 KV heads, 32
                 query heads, D=128, batch 16, context 32768; K/V ~
                 Student-t(3) x per-channel lognormal(sigma=1), clamped to the
                 fp16 range.
* ``longctx``   D=128, 8 KV heads, 64 query heads, batch 4, context 8K..128K;
                 K/V ~ Student-t(3).
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

DEFAULT_SEED = 0xC0FFEE
FP16_MAX = 65504.0

_KIND_ID = {"k": 0, "v": 1, "q": 2, "x": 3}


@dataclass(frozen=True)
class Workload:
    name: str
    layers: int
    h_kv: int
    h_q: int
    head_dim: int
    batch: int
    contexts: tuple
    k_dist: str
    v_dist: str
    k_outliers: int = 0
    k_outlier_gain: float = 1.0
    v_outliers: int = 0
    v_outlier_gain: float = 1.0
    group: int = 32
    extra: dict = field(default_factory=dict)


WORKLOADS = {
    "toy": Workload("toy", 1, 1, 1, 128, 1, (256,), "normal", "normal",
                    k_outliers=4, k_outlier_gain=20.0, v_outliers=4, v_outlier_gain=20.0),
    "gemma": Workload("gemma", 26, 1, 4, 256, 1, (4096,), "normal_lognormal", "normal_lognormal"),
    "qwen": Workload("qwen", 28, 2, 12, 128, 1, (256, 512, 1024, 4096), "normal", "normal",
                     k_outliers=8, k_outlier_gain=50.0),
    "mistral": Workload("mistral", 32, 8, 32, 128, 16, (32768,), "t3_lognormal", "t3_lognormal"),
    "longctx": Workload("longctx", 1, 8, 64, 128, 4, (8192, 16384, 32768, 65536, 131072),
                        "t3", "t3", extra={"stream_batch": 256}),
}


def _rng(seed: int, layer: int, kind: str, salt: int = 0) -> np.random.Generator:
    ss = np.random.SeedSequence(entropy=int(seed), spawn_key=(int(layer), _KIND_ID[kind], int(salt)))
    return np.random.default_rng(ss)


def plan_params(head_dim: int, seed: int = DEFAULT_SEED, layer: int = 0, kind: str = "k"):
    """Draw the fixed random sign vector s (int8, +/-1) and lambda (float32).

    s = 1 - 2*integers(0, 2, D); then lambda = 2**uniform(-1, 1, D), i.e.
    log-uniform on [0.5, 2]. Drawn in that order from the (layer, kind) stream.
    """
    g = _rng(seed, layer, kind, salt=1)
    signs = (1 - 2 * g.integers(0, 2, size=head_dim)).astype(np.int8)
    lam = np.exp2(g.uniform(-1.0, 1.0, size=head_dim)).astype(np.float32)
    return signs, lam


def channel_gains(wl: Workload, which: str, seed: int, layer: int) -> np.ndarray:
    """Per-channel multiplicative gains (original, un-rotated channel domain)."""
    D = wl.head_dim
    g = _rng(seed, layer, which, salt=2)
    dist = wl.k_dist if which == "k" else wl.v_dist
    gains = np.ones(D, dtype=np.float64)
    if dist.endswith("lognormal"):
        gains *= np.exp(g.standard_normal(D))
    n_out = wl.k_outliers if which == "k" else wl.v_outliers
    gain = wl.k_outlier_gain if which == "k" else wl.v_outlier_gain
    if n_out:
        idx = g.choice(D, size=n_out, replace=False)
        gains[idx] *= gain
    return gains


def _base_samples(dist: str, g: np.random.Generator, shape) -> np.ndarray:
    if dist.startswith("normal"):
        return g.standard_normal(shape)
    if dist.startswith("t3"):
        z = g.standard_normal(shape)
        chi2 = g.standard_normal(shape) ** 2 + g.standard_normal(shape) ** 2 + g.standard_normal(shape) ** 2
        return z / np.sqrt(chi2 / 3.0)
    raise ValueError(dist)


def kv_numpy(wl: Workload, which: str, shape, seed: int = DEFAULT_SEED, layer: int = 0,
             salt: int = 0) -> np.ndarray:
    """fp16 K or V values of the given shape [..., D] (numpy; small sizes)."""
    g = _rng(seed, layer, which, salt=10 + salt)
    dist = wl.k_dist if which == "k" else wl.v_dist
    vals = _base_samples(dist, g, tuple(shape)) * channel_gains(wl, which, seed, layer)
    return np.clip(vals, -FP16_MAX, FP16_MAX).astype(np.float16)


def q_numpy(shape, seed: int = DEFAULT_SEED, layer: int = 0, salt: int = 0) -> np.ndarray:
    g = _rng(seed, layer, "q", salt=20 + salt)
    return g.standard_normal(tuple(shape)).astype(np.float16)


def uniform_numpy(shape, lo: float, hi: float, seed: int = DEFAULT_SEED, salt: int = 0) -> np.ndarray:
    g = _rng(seed, 0, "x", salt=30 + salt)
    return g.uniform(lo, hi, size=tuple(shape))


# ---------------------------------------------------------------------------
# torch generators for full-size workloads (device-side draws; same recipes)
# ---------------------------------------------------------------------------

def _torch_gen(torch, device, seed: int, layer: int, kind: str, salt: int):
    ss = np.random.SeedSequence(entropy=int(seed), spawn_key=(int(layer), _KIND_ID[kind], 100 + int(salt)))
    s64 = int(ss.generate_state(1, dtype=np.uint64)[0] & ((1 << 63) - 1))
    gen = torch.Generator(device=device)
    gen.manual_seed(s64)
    return gen


def kv_torch(wl: Workload, which: str, shape, device, seed: int = DEFAULT_SEED, layer: int = 0,
             salt: int = 0, out=None):
    """fp16 K or V of the given shape, drawn on ``device`` with torch's generator.

    Same distribution recipe as :func:`kv_numpy` (different stream). If ``out``
    is given (an fp16 tensor of ``shape``) it is filled in place.
    """
    import torch

    gen = _torch_gen(torch, device, seed, layer, which, salt)
    dist = wl.k_dist if which == "k" else wl.v_dist
    gains = torch.tensor(channel_gains(wl, which, seed, layer), dtype=torch.float32, device=device)
    shape = tuple(shape)
    if out is not None and not out.is_contiguous():
        tmp = kv_torch(wl, which, shape, device, seed=seed, layer=layer, salt=salt)
        out.copy_(tmp)
        return out
    if out is None:
        out = torch.empty(shape, dtype=torch.float16, device=device)
    # draw in slabs along the leading dims to bound the fp32 temporaries
    flat = out.view(-1, shape[-1])
    rows = flat.shape[0]
    slab = max(1, (1 << 26) // shape[-1])
    for r0 in range(0, rows, slab):
        r1 = min(rows, r0 + slab)
        z = torch.randn((r1 - r0, shape[-1]), generator=gen, device=device, dtype=torch.float32)
        if dist.startswith("t3"):
            c = torch.randn((3, r1 - r0, shape[-1]), generator=gen, device=device, dtype=torch.float32)
            z = z / torch.sqrt((c * c).sum(0) / 3.0)
        z = z * gains
        flat[r0:r1] = z.clamp_(-FP16_MAX, FP16_MAX).to(torch.float16)
    return out


def q_torch(shape, device, seed: int = DEFAULT_SEED, layer: int = 0, salt: int = 0):
    import torch

    gen = _torch_gen(torch, device, seed, layer, "q", salt)
    return torch.randn(tuple(shape), generator=gen, device=device, dtype=torch.float32).to(torch.float16)
