"""Pins of the oracle's SRHT variant (the Hadamard rotation the pages compare with the
SRFT: "When Quantization Is Free", gist.science/de/paper/2605.05699, "Methodik" 1,
"Begruendung" / "Ergebnis"; the pages do not define it further, the reading is the
Sylvester matrix in natural order scaled by 1/sqrt(D), see the oracle's header).

Pinned to: the entry formula (-1)^popcount(i & j) (brute force, D <= 256), scipy's
Hadamard matrix (a library witness), an in-place fast Walsh-Hadamard butterfly (an
independent O(D log D) route), orthonormality and round trips, closed forms, and the
rotation invariance of attention. Planted mistakes must be rejected."""
import math

import numpy as np
import pytest

import kvgen
import oracle

POW2 = [1, 2, 4, 8, 16, 32, 64, 128, 256]


def _popcount_matrix(D):
    i = np.arange(D)[:, None]
    j = np.arange(D)[None, :]
    bits = np.vectorize(lambda v: bin(int(v)).count("1"))(i & j)
    return np.where(bits % 2 == 0, 1.0, -1.0)


def _fwht(x):
    """In-place fast Walsh-Hadamard butterflies over the last axis (unnormalised)."""
    y = np.array(x, dtype=np.float64, copy=True)
    D = y.shape[-1]
    h = 1
    while h < D:
        for i in range(0, D, 2 * h):
            a = y[..., i:i + h].copy()
            b = y[..., i + h:i + 2 * h].copy()
            y[..., i:i + h] = a + b
            y[..., i + h:i + 2 * h] = a - b
        h *= 2
    return y


def check_entries(hadamard):
    return all(np.array_equal(hadamard(D), _popcount_matrix(D)) for D in POW2)


def check_fwht_witness(forward):
    rng = np.random.default_rng(5)
    for D in (8, 128, 256):
        s = 1 - 2 * rng.integers(0, 2, D)
        lam = np.exp2(rng.uniform(-1, 1, D))
        x = rng.standard_normal((3, D))
        ref = _fwht(x * s) / math.sqrt(D) * lam
        if not np.allclose(forward(x, s, lam), ref, rtol=0, atol=1e-12 * np.abs(ref).max()):
            return False
    return True


def check_closed_forms(forward):
    for D in (8, 128):
        one, lam = np.ones(D, np.int8), np.ones(D)
        e0 = np.zeros(D)
        e0[0] = 1
        if not np.allclose(forward(e0, one, lam), np.full(D, 1 / math.sqrt(D)), atol=1e-15):
            return False
        y = forward(np.ones(D), one, lam)
        if abs(y[0] - math.sqrt(D)) > 1e-12 or np.abs(y[1:]).max() > 1e-12:
            return False
        # x = (+1 x D/2, -1 x D/2) is row D/2 of H: only channel D/2, value sqrt(D)
        x = np.concatenate([np.ones(D // 2), -np.ones(D // 2)])
        y = forward(x, one, lam)
        if abs(y[D // 2] - math.sqrt(D)) > 1e-12 or np.abs(np.delete(y, D // 2)).max() > 1e-12:
            return False
    return True


def _srht_forward(x, s, lam):
    return oracle.srft_forward(x, s, lam, "srht")


def test_hadamard_entries_and_library_witness():
    scipy_linalg = pytest.importorskip("scipy.linalg")
    assert check_entries(oracle.hadamard_matrix)
    for D in POW2:
        assert np.array_equal(oracle.hadamard_matrix(D), scipy_linalg.hadamard(D).astype(np.float64))
    with pytest.raises(ValueError):
        oracle.hadamard_matrix(96)


@pytest.mark.parametrize("D", [8, 128, 256])
def test_srht_orthonormal_symmetric_roundtrip(D):
    H = oracle.hadamard_matrix(D)
    assert np.array_equal(H, H.T)
    assert np.array_equal(H @ H, D * np.eye(D))
    s, lam = kvgen.plan_params(D)
    R = oracle.srht_matrix(s)
    assert np.abs(R @ R.T - np.eye(D)).max() < 1e-13
    x = np.random.default_rng(2).standard_normal((4, D))
    y = _srht_forward(x, s, lam)
    assert np.abs(oracle.srft_inverse(y, s, lam, "srht") - x).max() < 1e-12
    # Parseval after removing lambda
    assert np.allclose((y / lam) ** 2 @ np.ones(D), (x ** 2).sum(-1), rtol=1e-12)


def test_srht_matches_fast_butterflies_and_closed_forms():
    assert check_fwht_witness(_srht_forward)
    assert check_closed_forms(_srht_forward)


def test_srht_encode_closed_form_codes():
    # D = 8, s = +1, lambda = 1, G = 8: x = ones -> y = (sqrt 8, 0, ...) -> codes (7, 0, ..., 0)
    D = 8
    enc = oracle.encode(np.ones(D), np.ones(D, np.int8), np.ones(D), 8, "srht")
    assert enc["codes"].tolist() == [7, 0, 0, 0, 0, 0, 0, 0]
    assert float(enc["scales"][0]) == float(np.float16(math.sqrt(8) / 7))
    dec = oracle.decode(enc["packed"], enc["scales"], np.ones(D, np.int8), np.ones(D), 8, "srht")
    assert np.abs(dec - 1.0).max() <= float(enc["scales"][0]) / 2 / math.sqrt(8) + 1e-12


def test_srht_attention_rotated_equals_unrotated():
    B, Hkv, Hq, T, D = 2, 2, 6, 29, 128
    w = kvgen.WORKLOADS["qwen"]
    kp, vp = kvgen.plan_params(D, kind="k"), kvgen.plan_params(D, kind="v")
    k = kvgen.kv_numpy(w, "k", (B, Hkv, T, D))
    v = kvgen.kv_numpy(w, "v", (B, Hkv, T, D))
    ek = oracle.encode(k, kp[0], kp[1], 32, "srht")
    ev = oracle.encode(v, vp[0], vp[1], 32, "srht")
    q = kvgen.q_numpy((B, Hq, D))
    lens = np.array([29, 11])
    o1 = oracle.attend_decode_int4(q, ek["packed"], ek["scales"], ev["packed"], ev["scales"], kp, vp, lens,
                                   transform="srht")
    o2 = oracle.attend_decode_int4_rotated(q, ek["packed"], ek["scales"], ev["packed"], ev["scales"], kp, vp,
                                           lens, transform="srht")
    assert np.abs(o1 - o2).max() < 1e-12 * np.abs(o1).max()
    # and the SRHT cache decodes to something else than the SRFT reading of it
    o3 = oracle.attend_decode_int4(q, ek["packed"], ek["scales"], ev["packed"], ev["scales"], kp, vp, lens)
    assert not np.allclose(o1, o3)


# planted mistakes in copies of the SRHT steps: each must fail a pin
def _mut_walsh_order(D):
    # sequency (Walsh) order instead of natural order: rows sorted by sign changes
    H = oracle.hadamard_matrix(D)
    changes = (np.diff(H, axis=1) != 0).sum(1)
    return H[np.argsort(changes, kind="stable")]


def _mut_unnormalised(x, s, lam):
    return oracle.srft_forward(x, s, lam, "srht") * math.sqrt(np.asarray(s).shape[0])


def _mut_sign_after(x, s, lam):
    return oracle.srft_forward(x, np.ones_like(s), lam, "srht") * s


@pytest.mark.parametrize("mutant,check", [
    (_mut_walsh_order, check_entries),
    (_mut_unnormalised, check_fwht_witness),
    (_mut_unnormalised, check_closed_forms),
    (_mut_sign_after, check_fwht_witness),
], ids=["walsh-order", "unnormalised-fwht", "unnormalised-closed", "sign-after"])
def test_planted_srht_mistake_is_rejected(mutant, check):
    assert not check(mutant)
