"""Plain fp64 CPU oracle for SRFT-int4 KV-cache compression and decode attention.

TEST INFRASTRUCTURE ONLY. Only the test suite, the package smoke check and the
benchmark's CPU-baseline / reference arm may import, call or execute anything
in this package. The library (``rotated_int4_kv_b200``) never imports it, and
this module imports nothing from the library: the two share no code. Inputs
come from ``kvgen`` (random draws only).

Sources, cited by page and section (the pages are web renderings of the paper
"When Quantization Is Free: An int4 KV Cache That Outruns fp16 on Apple
Silicon", arXiv 2605.05699):

  [ABS]  paperdance.org/p/2605.05699 -- the English abstract: one fused kernel
         applies a random-sign FFT, a factor per channel and an absolute-maximum
         scale per channel group, and packs two 4-bit codes per byte; the cache
         stays about 3x smaller than fp16.
  [M1]   gist.science/de/paper/2605.05699, "Methodik" 1 (SRFT): the unitary DFT F
         applied after a fixed random +-1 sign vector s, its complex output packed
         to real values.
  [M2]   same page, "Methodik" 2 (fused kernel), its five steps: load and sign
         multiply; FFT passes; Hermitian unpack into a real representation;
         per-channel lambda, per-group abs-max reduction and rounding to signed
         int4; two int4 values packed into one byte.
  [M3]   same page, "Methodik" 3 (scaling strategies): per-channel factor (one
         per coordinate) combined with per-group scaling.
  [RES]  same page, "Wichtige Ergebnisse" / Speichereffizienz: 3.0-3.56x
         persistent compression.

Readings taken where the pages leave a step open:

  * Real basis ("pack"): rows in the order DC, (cos_k, sin_k) for
    k = 1..D/2-1, Nyquist; row 2k-1 = sqrt(2/D) cos(2 pi k n / D), row 2k =
    sqrt(2/D) sin(2 pi k n / D), row 0 = 1/sqrt(D), row D-1 = (-1)^n/sqrt(D).
  * lambda multiplies the rotated channels (after the transform) [M2].
  * Group = G contiguous rotated channels (G = 32 in the product; any G | D
    here). scale = fp16 round-to-nearest-even of absmax/7, clamped to 65504;
    the quantiser divides by that stored fp16 scale.
  * Codes: round half to even, clamped to [-7, 7]; a zero scale gives zero
    codes. Two's-complement nibbles, even element in the low nibble.
  * int8 codes ([M2] names "signed int4/int8" as the rounding target and
    defines int8 no further): the same steps with 127 in place of 7 (scale =
    fp16 round-to-nearest-even of min(absmax/127, 65504), codes clamped to [-127, 127], -128 never
    produced), one two's-complement byte per code, channel i at byte i. Every
    function taking ``bits`` accepts 4 (default) or 8.
  * Decode: x_hat = diag(s) F_r^T (c * scale / lambda).
  * Attention (not on the pages): softmax(sigma <q, x_hat_K>) weighted sum of
    x_hat_V, sigma = 1/sqrt(D) by default; query head h reads KV head
    h // (Hq / Hkv).
  * SRHT variant ([M1] "Begruendung"/"Ergebnis": the Hadamard transform is the
    common alternative, statistically indistinguishable in quality; the pages
    define it no further): R = H_D diag(s) / sqrt(D) with H_D the Sylvester
    Hadamard matrix in natural order, H[i][j] = (-1)^popcount(i & j); the same
    sign vector, lambda after the rotation, and the same group, scale, code and
    pack steps. Every function taking ``transform`` accepts "srft" (default)
    or "srht".

Parity pins: every function here is checked against closed forms, brute force and
invariants in ``tests/test_oracle_pins.py`` (the SRFT path), ``tests/test_oracle_srht_pins.py``
(the Hadamard variant) and ``tests/test_oracle_int8_pins.py`` (int8 codes), each with
planted mistakes that the pins must reject.
"""
from __future__ import annotations

import math

import numpy as np

FP16_MAX = 65504.0
QMAX = 7


def qmax(bits: int = 4) -> int:
    """Largest code magnitude of a signed b-bit code with symmetric range: 7 or 127."""
    if bits not in (4, 8):
        raise ValueError("bits must be 4 or 8")
    return (1 << (bits - 1)) - 1


# ---------------------------------------------------------------------------
# The transform [M1], [M2]
# ---------------------------------------------------------------------------

def real_dft_basis(D: int) -> np.ndarray:
    """F_r: the D x D orthonormal real DFT basis (rows = output channels).

    F is the unitary DFT [M1]; "pack" turns its Hermitian-symmetric output into
    D real numbers [M2]: DC, then (cos_k, sin_k) pairs, then Nyquist. Angles
    are taken from the exact integer k*n mod D so each entry is accurate to
    about 1e-16.
    """
    if D < 2 or D % 2:
        raise ValueError("D must be even and >= 2")
    n = np.arange(D)
    F = np.zeros((D, D), dtype=np.float64)
    F[0, :] = 1.0 / math.sqrt(D)
    amp = math.sqrt(2.0 / D)
    for k in range(1, D // 2):
        ang = 2.0 * math.pi * ((k * n) % D) / D
        F[2 * k - 1, :] = amp * np.cos(ang)
        F[2 * k, :] = amp * np.sin(ang)
    F[D - 1, :] = np.where(n % 2 == 0, 1.0, -1.0) / math.sqrt(D)
    return F


def srft_matrix(signs: np.ndarray) -> np.ndarray:
    """R = F_r . diag(s) [M1]."""
    s = np.asarray(signs, dtype=np.float64)
    return real_dft_basis(s.shape[0]) * s[None, :]


def hadamard_matrix(D: int) -> np.ndarray:
    """The Sylvester Hadamard matrix of order D (a power of two), natural order:
    H_1 = [1], H_2n = [[H_n, H_n], [H_n, -H_n]] (entries +-1, fp64)."""
    if D < 1 or D & (D - 1):
        raise ValueError("the Hadamard transform needs a power-of-two length")
    H = np.ones((1, 1))
    while H.shape[0] < D:
        H = np.block([[H, H], [H, -H]])
    return H


def srht_matrix(signs: np.ndarray) -> np.ndarray:
    """R = H_D . diag(s) / sqrt(D) (the SRHT reading above)."""
    s = np.asarray(signs, dtype=np.float64)
    D = s.shape[0]
    return hadamard_matrix(D) * s[None, :] / math.sqrt(D)


def rotation_matrix(signs: np.ndarray, transform: str = "srft") -> np.ndarray:
    if transform == "srft":
        return srft_matrix(signs)
    if transform == "srht":
        return srht_matrix(signs)
    raise ValueError(f"unknown transform {transform!r}")


def srft_forward(x: np.ndarray, signs: np.ndarray, lam: np.ndarray, transform: str = "srft") -> np.ndarray:
    """y = lambda * (R . x) over the last axis in fp64, R = F_r diag(s) [M1], [M2]
    (or the SRHT's H diag(s) / sqrt(D))."""
    x = np.asarray(x, dtype=np.float64)
    R = rotation_matrix(signs, transform)
    lam64 = np.asarray(lam, dtype=np.float64)
    return (x @ R.T) * lam64


def srft_inverse(y: np.ndarray, signs: np.ndarray, lam: np.ndarray, transform: str = "srft") -> np.ndarray:
    """x = R^T . (y / lambda): the exact inverse of srft_forward."""
    y = np.asarray(y, dtype=np.float64) / np.asarray(lam, dtype=np.float64)
    R = rotation_matrix(signs, transform)
    return y @ R


# ---------------------------------------------------------------------------
# The quantiser [M2], [M3]
# ---------------------------------------------------------------------------

def group_scales(y: np.ndarray, G: int, bits: int = 4) -> np.ndarray:
    """Per-group abs-max scale: min(absmax/qmax, 65504) rounded to fp16 (ties to even); fp16 array [..., D/G]."""
    y = np.asarray(y, dtype=np.float64)
    D = y.shape[-1]
    if D % G:
        raise ValueError("G must divide D")
    a = np.abs(y).reshape(y.shape[:-1] + (D // G, G)).max(axis=-1)
    return np.minimum(a / qmax(bits), FP16_MAX).astype(np.float16)


def quantize(y: np.ndarray, scales16: np.ndarray, G: int, bits: int = 4):
    """Signed codes c = clamp(rint(y / scale), -qmax, qmax); 0 where scale == 0.

    Returns (codes int8 [..., D], pre-rounding values y/scale fp64 [..., D]).
    """
    y = np.asarray(y, dtype=np.float64)
    D = y.shape[-1]
    sc = np.repeat(np.asarray(scales16, dtype=np.float64), G, axis=-1)
    with np.errstate(divide="ignore", invalid="ignore"):
        u = np.where(sc > 0, y / np.where(sc > 0, sc, 1.0), 0.0)
    codes = np.clip(np.rint(u), -qmax(bits), qmax(bits)).astype(np.int8)
    assert codes.shape[-1] == D
    return codes, u


def pack_nibbles(codes: np.ndarray) -> np.ndarray:
    """Two int4 codes per byte [M2]: byte j = (c[2j] & 0xF) | (c[2j+1] & 0xF) << 4."""
    c = np.asarray(codes, dtype=np.int64)
    lo = c[..., 0::2] & 0xF
    hi = c[..., 1::2] & 0xF
    return (lo | (hi << 4)).astype(np.uint8)


def unpack_nibbles(packed: np.ndarray) -> np.ndarray:
    """Inverse of pack_nibbles: signed codes in [-8, 7] (int8 [..., 2*nbytes])."""
    b = np.asarray(packed, dtype=np.int64)
    lo = b & 0xF
    hi = (b >> 4) & 0xF
    lo = np.where(lo >= 8, lo - 16, lo)
    hi = np.where(hi >= 8, hi - 16, hi)
    out = np.empty(b.shape[:-1] + (2 * b.shape[-1],), dtype=np.int8)
    out[..., 0::2] = lo
    out[..., 1::2] = hi
    return out


def pack_codes(codes: np.ndarray, bits: int = 4) -> np.ndarray:
    """Stored code bytes: nibble pairs (bits = 4) or one two's-complement byte per code (bits = 8)."""
    if qmax(bits) == 7:
        return pack_nibbles(codes)
    return (np.asarray(codes, dtype=np.int64) & 0xFF).astype(np.uint8)


def unpack_codes(packed: np.ndarray, bits: int = 4) -> np.ndarray:
    """Inverse of pack_codes: signed codes, int8 [..., D]."""
    if qmax(bits) == 7:
        return unpack_nibbles(packed)
    b = np.asarray(packed, dtype=np.int64)
    return np.where(b >= 128, b - 256, b).astype(np.int8)


def encode(x: np.ndarray, signs: np.ndarray, lam: np.ndarray, G: int = 32, transform: str = "srft",
           bits: int = 4):
    """The encode path of [ABS]/[M2] over the last axis.

    Returns dict(packed=uint8 [..., D*bits/8], scales=float16 [..., D/G],
    codes=int8 [..., D], y=fp64 [..., D], u=fp64 pre-rounding y/scale).
    """
    y = srft_forward(x, signs, lam, transform)
    scales = group_scales(y, G, bits)
    codes, u = quantize(y, scales, G, bits)
    return {"packed": pack_codes(codes, bits), "scales": scales, "codes": codes, "y": y, "u": u}


def dequantize(codes: np.ndarray, scales16: np.ndarray, G: int) -> np.ndarray:
    """c_hat = c * scale (fp64), scale taken from the stored fp16 value."""
    sc = np.repeat(np.asarray(scales16, dtype=np.float64), G, axis=-1)
    return np.asarray(codes, dtype=np.float64) * sc


def decode(packed: np.ndarray, scales16: np.ndarray, signs: np.ndarray, lam: np.ndarray,
           G: int = 32, transform: str = "srft", bits: int = 4) -> np.ndarray:
    """x_hat = R^T (c*scale / lambda), fp64 [..., D]."""
    return srft_inverse(dequantize(unpack_codes(packed, bits), scales16, G), signs, lam, transform)


def compressed_bytes_per_vector(D: int, G: int, bits: int = 4) -> int:
    """D*bits/8 bytes of codes plus one fp16 scale per group [RES]."""
    qmax(bits)
    return D * bits // 8 + 2 * (D // G)


# ---------------------------------------------------------------------------
# Decode attention (read path; not described on the pages)
# ---------------------------------------------------------------------------

def _softmax_weighted(scores: np.ndarray, values: np.ndarray) -> np.ndarray:
    m = scores.max()
    p = np.exp(scores - m)
    return (p[:, None] * values).sum(axis=0) / p.sum()


def attend_decode(q: np.ndarray, k_hat: np.ndarray, v_hat: np.ndarray, seq_lens,
                  sigma: float | None = None) -> np.ndarray:
    """One-query decode attention in the original domain, fp64.

    q [B, Hq, D]; k_hat, v_hat [B, Hkv, T, D] (already decoded, fp64 or fp16);
    seq_lens [B]. Query head h reads KV head h // (Hq // Hkv).
    """
    q = np.asarray(q, dtype=np.float64)
    B, Hq, D = q.shape
    Hkv = k_hat.shape[1]
    grp = Hq // Hkv
    if sigma is None:
        sigma = 1.0 / math.sqrt(D)
    out = np.zeros((B, Hq, D), dtype=np.float64)
    for b in range(B):
        T = int(seq_lens[b])
        for h in range(Hq):
            kh = h // grp
            K = np.asarray(k_hat[b, kh, :T], dtype=np.float64)
            V = np.asarray(v_hat[b, kh, :T], dtype=np.float64)
            out[b, h] = _softmax_weighted(sigma * (K @ q[b, h]), V)
    return out


def attend_decode_int4(q, k_packed, k_scales, v_packed, v_scales, k_params, v_params, seq_lens,
                       G: int = 32, sigma: float | None = None, transform: str = "srft",
                       bits: int = 4) -> np.ndarray:
    """Attention over a packed int4 (or int8) cache: decode K and V, then attend_decode.

    k_params / v_params = (signs, lambda) of the K and V transforms.
    """
    T = int(np.max(seq_lens))
    kh = decode(k_packed[:, :, :T], k_scales[:, :, :T], k_params[0], k_params[1], G, transform, bits)
    vh = decode(v_packed[:, :, :T], v_scales[:, :, :T], v_params[0], v_params[1], G, transform, bits)
    return attend_decode(q, kh, vh, seq_lens, sigma)


def attend_decode_int4_rotated(q, k_packed, k_scales, v_packed, v_scales, k_params, v_params,
                               seq_lens, G: int = 32, sigma: float | None = None,
                               transform: str = "srft", bits: int = 4) -> np.ndarray:
    """The same attention computed in the rotated domain.

    q_t = Lambda_K^-1 R_K q; score_t = sigma * sum_g scale_{t,g} sum_{i in g} q_t[i] c_t[i];
    o_t = sum_t p_t c_hat^V_t; o = R_V^T Lambda_V^-1 o_t. Equal to
    attend_decode_int4 because R is orthogonal: <q, R^T L^-1 c_hat> =
    <L^-1 R q, c_hat>.
    """
    q = np.asarray(q, dtype=np.float64)
    B, Hq, D = q.shape
    Hkv = k_packed.shape[1]
    grp = Hq // Hkv
    if sigma is None:
        sigma = 1.0 / math.sqrt(D)
    Rk = rotation_matrix(k_params[0], transform)
    Rv = rotation_matrix(v_params[0], transform)
    lk = np.asarray(k_params[1], dtype=np.float64)
    lv = np.asarray(v_params[1], dtype=np.float64)
    out = np.zeros((B, Hq, D), dtype=np.float64)
    for b in range(B):
        T = int(seq_lens[b])
        for h in range(Hq):
            kv = h // grp
            qt = (Rk @ q[b, h]) / lk
            ck = dequantize(unpack_codes(k_packed[b, kv, :T], bits), k_scales[b, kv, :T], G)
            cv = dequantize(unpack_codes(v_packed[b, kv, :T], bits), v_scales[b, kv, :T], G)
            ot = _softmax_weighted(sigma * (ck @ qt), cv)
            out[b, h] = Rv.T @ (ot / lv)
    return out


def attend_decode_fp16(q, k16, v16, seq_lens, sigma: float | None = None) -> np.ndarray:
    """The fp16-cache comparator: the same attention on fp16 K/V, computed in fp64."""
    return attend_decode(q, np.asarray(k16, dtype=np.float64), np.asarray(v16, dtype=np.float64),
                         seq_lens, sigma)
