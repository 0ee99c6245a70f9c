"""Pins of the CPU oracle to things other than itself.

Each pin checks the oracle against what the pages and the mathematics fix:
closed forms of a hand-worked D=8 example (tests/golden/srft_d8_hand.txt),
brute-force complex DFTs built from complex exponentials, numpy's real FFT as
an independent library witness, orthonormality / round-trip invariants,
quantiser invariants (code range, abs-max -> +/-7, |y - c*scale| <= scale/2,
ties to even), nibble-order byte examples, and attention special cases.

The mutation tests at the bottom plant plausible mistakes in copies of oracle
steps (on the CPU) and assert that at least one pin rejects each of them.
"""
import cmath
import dataclasses
import math

import numpy as np
import pytest

import kvgen
import oracle
from tests.golden_io import read_cases

POW2 = [2, 4, 8, 16, 32, 64, 128, 256]


# ---------------------------------------------------------------------------
# reusable pin checks (take the implementation under test as arguments)
# ---------------------------------------------------------------------------

def brute_real_basis(D):
    """Real basis rows built from the complex DFT W[k,n] = exp(-2 pi i k n / D)/sqrt(D)
    by pure-Python loops: DC = Re W0, cos_k = sqrt2 Re Wk, sin_k = -sqrt2 Im Wk,
    Nyquist = Re W_{D/2}."""
    rows = []
    W = [[cmath.exp(-2j * math.pi * k * n / D) / math.sqrt(D) for n in range(D)] for k in range(D // 2 + 1)]
    rows.append([w.real for w in W[0]])
    for k in range(1, D // 2):
        rows.append([math.sqrt(2) * w.real for w in W[k]])
        rows.append([-math.sqrt(2) * w.imag for w in W[k]])
    rows.append([w.real for w in W[D // 2]])
    return np.array(rows)


def rfft_witness(x, s, lam):
    """y from numpy.fft.rfft of s*x, mapped to the (DC, cos, sin, ..., Nyquist) basis."""
    D = x.shape[-1]
    X = np.fft.rfft(np.asarray(x, np.float64) * s, axis=-1)
    y = np.empty(x.shape, np.float64)
    y[..., 0] = X[..., 0].real / math.sqrt(D)
    y[..., 1:D - 1:2] = math.sqrt(2.0 / D) * X[..., 1:D // 2].real
    y[..., 2:D - 1:2] = -math.sqrt(2.0 / D) * X[..., 1:D // 2].imag
    y[..., D - 1] = X[..., D // 2].real / math.sqrt(D)
    return y * lam


def check_brute_basis(basis_fn):
    for D in (4, 8, 16):
        if not np.allclose(basis_fn(D), brute_real_basis(D), rtol=0, atol=1e-12):
            return False
    return True


def check_rfft_witness(forward_fn):
    for D in POW2[2:]:
        x = kvgen.uniform_numpy((17, D), -3, 3, salt=D)
        s, lam = kvgen.plan_params(D, seed=D)
        y = forward_fn(x, s, lam)
        ref = rfft_witness(x, s, lam.astype(np.float64))
        if not np.allclose(y, ref, rtol=0, atol=1e-12 * np.abs(ref).max()):
            return False
    return True


def check_golden(encode_fn):
    for c in read_cases("srft_d8_hand.txt"):
        x = np.array(c["x"], np.float64)
        G = c["G"][0]
        enc = encode_fn(x, np.array(c["s"]), np.array(c["lam"]), G)
        if not np.allclose(enc["y"], c["y"], rtol=0, atol=1e-12):
            return False
        if not np.array_equal(enc["scales"].astype(np.float64), np.array(c["scale"])):
            return False
        if not np.array_equal(enc["codes"], np.array(c["codes"])):
            return False
        if not np.array_equal(enc["packed"], np.array(c["bytes"], np.uint8)):
            return False
    return True


def check_ties(quantize_fn):
    sc = 0.25  # exact in fp16; absmax 1.75 -> scale fp16(1.75/7) = 0.25
    u = np.array([7, 2.5, 3.5, -2.5, -3.5, 0.5, -0.5, 1.5])
    codes, _ = quantize_fn(u * sc, np.array([sc], np.float16), 8)
    return np.array_equal(codes, np.array([7, 2, 4, -2, -4, 0, 0, 2]))


# ---------------------------------------------------------------------------
# the pins
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("D", POW2 + [6, 12])
def test_basis_orthonormal(D):
    F = oracle.real_dft_basis(D)
    assert np.abs(F @ F.T - np.eye(D)).max() < 1e-12
    assert np.abs(F.T @ F - np.eye(D)).max() < 1e-12


def test_basis_matches_brute_complex_dft():
    assert check_brute_basis(oracle.real_dft_basis)


def test_forward_matches_numpy_rfft():
    assert check_rfft_witness(oracle.srft_forward)


@pytest.mark.parametrize("D", [8, 128, 256])
def test_roundtrip_and_parseval(D):
    x = kvgen.uniform_numpy((9, D), -5, 5, salt=7)
    s, lam = kvgen.plan_params(D, seed=3)
    y = oracle.srft_forward(x, s, lam)
    assert np.abs(oracle.srft_inverse(y, s, lam) - x).max() < 1e-12 * np.abs(x).max()
    y1 = oracle.srft_forward(x, s, np.ones(D))
    assert np.allclose((y1 ** 2).sum(-1), (x ** 2).sum(-1), rtol=1e-12)


def test_golden_hand_worked_d8():
    assert check_golden(oracle.encode)


def test_golden_decode_hand_d8():
    # codes (7,0,...,0) with scale 1655/4096, s=+1, lambda=1: x_hat = 7*scale/sqrt(8) * ones
    packed = oracle.pack_nibbles(np.array([7, 0, 0, 0, 0, 0, 0, 0]))
    xh = oracle.decode(packed, np.array([1655 / 4096], np.float16), np.ones(8), np.ones(8), 8)
    assert np.allclose(xh, 7 * (1655 / 4096) / math.sqrt(8), rtol=0, atol=1e-14)


def test_ties_to_even():
    assert check_ties(oracle.quantize)


def test_fp16_scale_rounding_ties():
    # a/7 exactly halfway between fp16 neighbours rounds to the even mantissa
    y = np.zeros((2, 8))
    y[0, 0] = 7 * (1 + 2 ** -11)        # between 1 and 1+2^-10 -> 1
    y[1, 0] = 7 * (1 + 3 * 2 ** -11)    # between 1+2^-10 and 1+2^-9 -> 1+2^-9
    sc = oracle.group_scales(y, 8).astype(np.float64)[:, 0]
    assert sc[0] == 1.0 and sc[1] == 1 + 2 ** -9


def test_scale_overflow_zero_and_clamp():
    y = np.zeros((3, 8))
    y[0, :] = [1e6, -2e5, 0, 0, 0, 0, 0, 1]
    y[2, :] = [9.8 * 2.0 ** -24, 0, 0, 0, 0, 0, 0, 0]  # a/7 = 1.4 fp16 subnormal ulps -> 1 ulp; u = 9.8
    sc = oracle.group_scales(y, 8)
    assert float(sc[0, 0]) == 65504.0
    codes, _ = oracle.quantize(y, sc, 8)
    assert list(codes[0, :2]) == [7, -3]            # 1e6/65504 clamps to 7; -2e5/65504 = -3.05 -> -3
    assert float(sc[1, 0]) == 0.0 and not codes[1].any()
    assert float(sc[2, 0]) == 2.0 ** -24 and codes[2, 0] == 7 and np.abs(codes).max() <= 7


@pytest.mark.parametrize("wl", ["toy", "gemma", "mistral"])
def test_quantizer_invariants(wl):
    w = kvgen.WORKLOADS[wl]
    D = w.head_dim
    x = kvgen.kv_numpy(w, "k", (64, D), salt=1)
    s, lam = kvgen.plan_params(D)
    enc = oracle.encode(x, s, lam, 32)
    codes, y, sc = enc["codes"], enc["y"], enc["scales"].astype(np.float64)
    assert codes.min() >= -7 and codes.max() <= 7
    yg = y.reshape(64, D // 32, 32)
    cg = codes.reshape(64, D // 32, 32)
    am = np.abs(yg).argmax(-1)
    assert np.all(np.abs(np.take_along_axis(cg, am[..., None], -1)) == 7)
    err = np.abs(yg - cg * sc[..., None])
    assert np.all(err <= sc[..., None] / 2 * (1 + 1e-12))
    # decode error bound: ||x - x_hat||^2 <= sum_i (scale_g(i) / (2 lambda_i))^2
    xh = oracle.decode(enc["packed"], enc["scales"], s, lam, 32)
    bound = ((np.repeat(sc, 32, -1) / (2 * lam.astype(np.float64))) ** 2).sum(-1)
    assert np.all(((x.astype(np.float64) - xh) ** 2).sum(-1) <= bound * (1 + 1e-9))


def test_nibble_bytes():
    c = np.array([1, -1, 7, -7, 0, 3, -8, 7])
    assert list(oracle.pack_nibbles(c)) == [0xF1, 0x97, 0x30, 0x78]
    allb = np.arange(256, dtype=np.uint8)
    assert np.array_equal(oracle.pack_nibbles(oracle.unpack_nibbles(allb)), allb)


def test_compression_ratio():
    # 16 bits -> 4-bit codes plus one fp16 scale per 32: 3.56x
    assert oracle.compressed_bytes_per_vector(128, 32) == 72
    assert oracle.compressed_bytes_per_vector(256, 32) == 144
    assert abs(2 * 128 / 72 - 3.56) < 0.005


# ---------------------------------------------------------------------------
# attention pins
# ---------------------------------------------------------------------------

def _packed_cache(B, Hkv, T, D, seed=5):
    w = kvgen.WORKLOADS["qwen"]
    ks, kl = kvgen.plan_params(D, seed=seed, kind="k")
    vs, vl = kvgen.plan_params(D, seed=seed, kind="v")
    k = kvgen.kv_numpy(w, "k", (B, Hkv, T, D), seed=seed)
    v = kvgen.kv_numpy(w, "v", (B, Hkv, T, D), seed=seed)
    ek, ev = oracle.encode(k, ks, kl), oracle.encode(v, vs, vl)
    return ek, ev, (ks, kl), (vs, vl)


def test_attention_rotated_equals_unrotated():
    B, Hkv, Hq, T, D = 2, 2, 6, 37, 128
    ek, ev, kp, vp = _packed_cache(B, Hkv, T, D)
    q = kvgen.q_numpy((B, Hq, D))
    lens = np.array([37, 20])
    o1 = oracle.attend_decode_int4(q, ek["packed"], ek["scales"], ev["packed"], ev["scales"], kp, vp, lens)
    o2 = oracle.attend_decode_int4_rotated(q, ek["packed"], ek["scales"], ev["packed"], ev["scales"],
                                           kp, vp, lens)
    assert np.abs(o1 - o2).max() < 1e-12 * np.abs(o1).max()


def test_attention_special_cases():
    B, Hkv, Hq, T, D = 1, 1, 2, 9, 128
    ek, ev, kp, vp = _packed_cache(B, Hkv, T, D, seed=9)
    q = kvgen.q_numpy((B, Hq, D), salt=3)
    vh = oracle.decode(ev["packed"], ev["scales"], *vp)
    # T = 1 -> o = x_hat_V[0]
    o = oracle.attend_decode_int4(q, ek["packed"], ek["scales"], ev["packed"], ev["scales"], kp, vp, [1])
    assert np.allclose(o[0, 0], vh[0, 0, 0], rtol=0, atol=1e-12)
    # sigma -> 0 gives the mean of the values
    o = oracle.attend_decode_int4(q, ek["packed"], ek["scales"], ev["packed"], ev["scales"], kp, vp, [T],
                                  sigma=0.0)
    assert np.allclose(o[0, 1], vh[0, 0].mean(0), rtol=0, atol=1e-12)
    # identical keys -> mean of the values
    kp_same = np.repeat(ek["packed"][:, :, :1], T, axis=2)
    ks_same = np.repeat(ek["scales"][:, :, :1], T, axis=2)
    o = oracle.attend_decode_int4(q, kp_same, ks_same, ev["packed"], ev["scales"], kp, vp, [T])
    assert np.allclose(o[0, 0], vh[0, 0].mean(0), rtol=0, atol=1e-12)


def test_attention_brute_force_tiny():
    # softmax written out with Python floats on a 3-token, D=4 case
    q = np.array([[[0.5, -1.0, 2.0, 0.25]]])
    K = np.array([[[[1, 0, 0, 1], [0, 1, -1, 0], [2, 2, 0, -1]]]], np.float64)
    V = np.array([[[[1, 2, 3, 4], [-1, 0, 1, 0], [0.5, 0.5, -2, 1]]]], np.float64)
    o = oracle.attend_decode(q, K, V, [3], sigma=0.5)
    sc = [0.5 * sum(q[0, 0, i] * K[0, 0, t, i] for i in range(4)) for t in range(3)]
    e = [math.exp(v) for v in sc]
    ref = [sum(e[t] * V[0, 0, t, i] for t in range(3)) / sum(e) for i in range(4)]
    assert np.allclose(o[0, 0], ref, rtol=1e-14)


def test_attention_fp16_comparator_and_gqa_mapping():
    B, Hkv, Hq, T, D = 1, 2, 4, 5, 8
    wl = dataclasses.replace(kvgen.WORKLOADS["toy"], head_dim=D, k_outliers=0, v_outliers=0)
    k = kvgen.kv_numpy(wl, "k", (B, Hkv, T, D))
    v = kvgen.kv_numpy(wl, "v", (B, Hkv, T, D))
    q = kvgen.q_numpy((B, Hq, D))
    o = oracle.attend_decode_fp16(q, k, v, [T])
    # heads 2, 3 read KV head 1: swapping KV head 0's data must not change them
    k2 = k.copy()
    k2[:, 0] = k2[:, 0, ::-1]
    o2 = oracle.attend_decode_fp16(q, k2, v, [T])
    assert np.array_equal(o[:, 2:], o2[:, 2:])
    assert not np.allclose(o[:, :2], o2[:, :2])


# ---------------------------------------------------------------------------
# planted mistakes: each must be rejected by at least one pin
# ---------------------------------------------------------------------------

def _mut_basis_sin_sign(D):
    F = oracle.real_dft_basis(D)
    F[2:D - 1:2] *= -1
    return F


def _mut_basis_swap_cos_sin(D):
    F = oracle.real_dft_basis(D).copy()
    F[1:D - 1:2], F[2:D - 1:2] = F[2:D - 1:2].copy(), F[1:D - 1:2].copy()
    return F


def _mut_forward_transposed(x, s, lam):
    R = oracle.srft_matrix(s)
    return (np.asarray(x, np.float64) @ R) * lam


def _mut_forward_lambda_before(x, s, lam):
    return oracle.srft_forward(np.asarray(x, np.float64) * lam, s, np.ones_like(lam))


def _mut_forward_sign_after(x, s, lam):
    return oracle.srft_forward(x, np.ones_like(s), lam) * s


def _encode_with(forward=None, scales=None, quant=None, pack=None):
    def enc(x, s, lam, G):
        y = (forward or oracle.srft_forward)(x, s, lam)
        sc = (scales or oracle.group_scales)(y, G)
        codes, u = (quant or oracle.quantize)(y, sc, G)
        return {"y": y, "scales": sc, "codes": codes, "packed": (pack or oracle.pack_nibbles)(codes)}
    return enc


def _mut_scales_div8(y, G):
    a = np.abs(y).reshape(y.shape[:-1] + (-1, G)).max(-1)
    return (a / 8).astype(np.float16)


def _mut_scales_fp32_truncate(y, G):
    a = np.abs(y).reshape(y.shape[:-1] + (-1, G)).max(-1) / 7
    # round toward zero instead of to nearest
    return np.float16(np.trunc(a * 2 ** 14) / 2 ** 14)


def _mut_quant_half_up(y, sc, G):
    s = np.repeat(sc.astype(np.float64), G, -1)
    u = y / s
    return np.clip(np.floor(u + 0.5), -7, 7).astype(np.int8), u


def _mut_pack_swapped(codes):
    c = np.asarray(codes, np.int64)
    return ((c[..., 1::2] & 0xF) | ((c[..., 0::2] & 0xF) << 4)).astype(np.uint8)


def _mut_pack_sign_magnitude(codes):
    c = np.asarray(codes, np.int64)
    sm = np.where(c < 0, 8 | (-c), c) & 0xF
    return (sm[..., 0::2] | (sm[..., 1::2] << 4)).astype(np.uint8)


def _all_pins_pass(basis=None, forward=None, enc=None, quant=None):
    return (check_brute_basis(basis or oracle.real_dft_basis)
            and check_rfft_witness(forward or oracle.srft_forward)
            and check_golden(enc or oracle.encode)
            and check_ties(quant or oracle.quantize))


def test_unmutated_oracle_passes_all_pins():
    assert _all_pins_pass()


@pytest.mark.parametrize("mutant", [
    dict(basis=_mut_basis_sin_sign),
    dict(basis=_mut_basis_swap_cos_sin),
    dict(forward=_mut_forward_transposed, enc=_encode_with(forward=_mut_forward_transposed)),
    dict(forward=_mut_forward_lambda_before, enc=_encode_with(forward=_mut_forward_lambda_before)),
    dict(forward=_mut_forward_sign_after, enc=_encode_with(forward=_mut_forward_sign_after)),
    dict(enc=_encode_with(scales=_mut_scales_div8)),
    dict(enc=_encode_with(scales=_mut_scales_fp32_truncate)),
    dict(quant=_mut_quant_half_up),
    dict(enc=_encode_with(pack=_mut_pack_swapped)),
    dict(enc=_encode_with(pack=_mut_pack_sign_magnitude)),
], ids=["sin-sign", "cos-sin-swap", "transposed", "lambda-before", "sign-after", "absmax/8",
        "scale-truncate", "round-half-up", "nibble-swap", "sign-magnitude"])
def test_planted_mistake_is_rejected(mutant):
    assert not _all_pins_pass(**mutant)
