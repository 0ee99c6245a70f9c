"""Pins of the oracle's int8-code variant ("When Quantization Is Free",
gist.science/de/paper/2605.05699, "Methodik" 2: rounding to signed int4/int8; the pages
do not define int8 further, the reading is the int4 quantiser with 127 in place of 7 and
one two's-complement byte per code, see the oracle's header).

Pinned to: closed forms of the D = 8 hand example, an exhaustive nearest-integer search
(an independent route to round-half-even + clamp), the two's-complement byte encoding
of every code, the per-group error bound |y - c scale| <= scale / 2, the byte count,
the int4 path left unchanged, and the rotation invariance of attention over an int8
cache. Planted mistakes must be rejected."""
import math

import numpy as np

import oracle


def _nearest_code(u, qm):
    """argmin_k |u - k| over k in [-qm, qm], ties to the even k (exhaustive)."""
    ks = np.arange(-qm, qm + 1)
    d = np.abs(u - ks)
    best = d.min()
    cand = ks[np.isclose(d, best, rtol=0, atol=1e-12)]
    if len(cand) > 1:
        cand = cand[cand % 2 == 0]
    return int(cand[0])


# ---------------------------------------------------------------- checks (take the function under test)
def check_closed_forms(encode):
    D = 8
    s = np.ones(D)
    lam = np.ones(D)
    # all ones: only the DC channel, value sqrt(8); its code is +127
    e = encode(np.ones((1, D)), s, lam, 8, "srft", 8)
    sc = np.float16(math.sqrt(8) / 127)
    if e["scales"][0, 0] != sc or list(e["codes"][0]) != [127] + [0] * 7:
        return False
    # (-1)^n: only the Nyquist channel (row D-1)
    e = encode(np.array([[(-1.0) ** n for n in range(D)]]), s, lam, 8, "srft", 8)
    if list(e["codes"][0]) != [0] * 7 + [127]:
        return False
    # negative all ones: -127 in the DC channel, stored as the byte 0x81
    e = encode(-np.ones((1, D)), s, lam, 8, "srft", 8)
    return list(e["codes"][0]) == [-127] + [0] * 7 and e["packed"][0, 0] == 0x81


def check_exhaustive_rounding(quantize):
    rng = np.random.default_rng(11)
    G = 16
    y = rng.standard_normal((6, 32)) * np.exp(rng.standard_normal((6, 1)))
    y[0, :3] = [0.5, -1.5, 2.5]  # exact ties once the scale is 1
    scales = oracle.group_scales(y, G, 8)
    scales[0, 0] = np.float16(1.0)
    codes, u = quantize(y, scales, G, 8)
    for idx in np.ndindex(u.shape):
        if codes[idx] != _nearest_code(u[idx], 127):
            return False
    return list(codes[0, :3]) == [0, -2, 2]


def check_byte_encoding(pack, unpack):
    codes = np.arange(-127, 128, dtype=np.int8)[None, :]
    packed = pack(codes, 8)
    want = np.array([c & 0xFF for c in range(-127, 128)], dtype=np.uint8)
    if packed.dtype != np.uint8 or not np.array_equal(packed[0], want):
        return False
    return np.array_equal(unpack(packed, 8), codes)


def check_error_bound(encode):
    rng = np.random.default_rng(3)
    for D, G in ((128, 32), (256, 16)):
        s = 1 - 2 * rng.integers(0, 2, D)
        lam = np.exp2(rng.uniform(-1, 1, D))
        x = (rng.standard_normal((50, D)) * np.exp(rng.standard_normal(D))).astype(np.float16)
        e = encode(x, s, lam, G, "srft", 8)
        sc = np.repeat(e["scales"].astype(np.float64), G, axis=-1)
        err = np.abs(e["y"] - e["codes"] * sc)
        if np.any(err > sc / 2 * (1 + 1e-12)):
            return False
        # every group's extreme channel reaches +-127 (the scale is rounded, so +-126 or +-127)
        mx = np.abs(e["codes"].astype(np.int64)).reshape(50, D // G, G).max(axis=-1)
        if np.any(mx < 126):
            return False
    return True


# ---------------------------------------------------------------- pins
def test_int8_closed_forms():
    assert check_closed_forms(oracle.encode)


def test_int8_rounding_is_nearest_integer_ties_even():
    assert check_exhaustive_rounding(oracle.quantize)


def test_int8_byte_encoding():
    assert check_byte_encoding(oracle.pack_codes, oracle.unpack_codes)


def test_int8_error_bound():
    assert check_error_bound(oracle.encode)


def test_int8_bytes_per_vector_and_qmax():
    assert oracle.qmax(4) == 7 and oracle.qmax(8) == 127
    assert oracle.compressed_bytes_per_vector(128, 32, 8) == 128 + 8
    assert oracle.compressed_bytes_per_vector(256, 16, 8) == 256 + 32
    assert oracle.compressed_bytes_per_vector(128, 32) == 72


def test_int4_path_unchanged_by_bits_default():
    rng = np.random.default_rng(9)
    D = 128
    s = 1 - 2 * rng.integers(0, 2, D)
    lam = np.exp2(rng.uniform(-1, 1, D))
    x = rng.standard_normal((4, D)).astype(np.float16)
    a = oracle.encode(x, s, lam, 32)
    b = oracle.encode(x, s, lam, 32, "srft", 4)
    assert np.array_equal(a["packed"], b["packed"]) and np.array_equal(a["scales"], b["scales"])
    assert np.abs(a["codes"]).max() <= 7


def test_int8_decode_error_below_int4():
    rng = np.random.default_rng(4)
    D = 128
    s = 1 - 2 * rng.integers(0, 2, D)
    lam = np.exp2(rng.uniform(-1, 1, D))
    x = rng.standard_normal((64, D)).astype(np.float16)
    err = {}
    for bits in (4, 8):
        e = oracle.encode(x, s, lam, 32, "srft", bits)
        xh = oracle.decode(e["packed"], e["scales"], s, lam, 32, "srft", bits)
        err[bits] = np.linalg.norm(xh - x.astype(np.float64)) / np.linalg.norm(x.astype(np.float64))
    # step size 127/7 = 18x smaller: the relative error falls by about that factor
    assert err[8] < err[4] / 10 and err[8] < 1e-2


def test_int8_attention_rotation_invariance():
    rng = np.random.default_rng(8)
    B, Hq, Hkv, T, D, G = 1, 4, 2, 40, 128, 32
    kp = (1 - 2 * rng.integers(0, 2, D), np.exp2(rng.uniform(-1, 1, D)))
    vp = (1 - 2 * rng.integers(0, 2, D), np.exp2(rng.uniform(-1, 1, D)))
    k = rng.standard_normal((B, Hkv, T, D)).astype(np.float16)
    v = rng.standard_normal((B, Hkv, T, D)).astype(np.float16)
    q = rng.standard_normal((B, Hq, D)).astype(np.float16)
    ek = oracle.encode(k, *kp, G, "srft", 8)
    ev = oracle.encode(v, *vp, G, "srft", 8)
    lens = [T]
    a = oracle.attend_decode_int4(q, ek["packed"], ek["scales"], ev["packed"], ev["scales"], kp, vp, lens, G,
                                  bits=8)
    b = oracle.attend_decode_int4_rotated(q, ek["packed"], ek["scales"], ev["packed"], ev["scales"], kp, vp,
                                          lens, G, bits=8)
    assert np.allclose(a, b, rtol=0, atol=1e-12 * np.abs(a).max())
    # and it is close to attention on the fp16 inputs (int8 error is small)
    f = oracle.attend_decode_fp16(q, k, v, lens)
    assert np.linalg.norm(a - f) / np.linalg.norm(f) < 1e-2


# ---------------------------------------------------------------- planted mistakes (on the CPU oracle)
def _encode_clamped_at_7(x, s, lam, G=32, transform="srft", bits=4):
    e = oracle.encode(x, s, lam, G, transform, bits)
    e["codes"] = np.clip(e["codes"], -7, 7)
    e["packed"] = oracle.pack_codes(e["codes"], bits)
    return e


def _encode_scale_over_128(x, s, lam, G=32, transform="srft", bits=4):
    y = oracle.srft_forward(x, s, lam, transform)
    D = y.shape[-1]
    a = np.abs(y).reshape(y.shape[:-1] + (D // G, G)).max(axis=-1)
    scales = np.minimum(a / 128, 65504).astype(np.float16)
    codes, u = oracle.quantize(y, scales, G, bits)
    return {"packed": oracle.pack_codes(codes, bits), "scales": scales, "codes": codes, "y": y, "u": u}


def _quantize_half_away(y, scales16, G, bits=4):
    codes, u = oracle.quantize(y, scales16, G, bits)
    c = np.clip(np.sign(u) * np.floor(np.abs(u) + 0.5), -127, 127).astype(np.int8)
    return c, u


def _pack_offset_binary(codes, bits=4):
    return (np.asarray(codes, dtype=np.int64) + 128).astype(np.uint8)


def test_planted_mistakes_are_rejected():
    assert not check_closed_forms(_encode_clamped_at_7)
    assert not check_closed_forms(_encode_scale_over_128)
    assert not check_error_bound(_encode_clamped_at_7)
    assert not check_exhaustive_rounding(_quantize_half_away)
    assert not check_byte_encoding(_pack_offset_binary, oracle.unpack_codes)
