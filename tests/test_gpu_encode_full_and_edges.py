"""Encode parity at the benchmark's exact launch, and on the quantiser's edge inputs.

* The benchmark's timed encode is one grouped kvq_encode_batch launch of 52 jobs
  (26 layers x K and V, each 4096 vectors of D = 256, int4 codes, SRFT plans with
  their own s and lambda). The same launch runs here on both encode paths, and every
  row of every job -- so the first and last tile of each job and the rows on both
  sides of every 128-row tile boundary -- is checked against the oracle, on every
  encode path (auto, register FFT, dense tensor-core product, radix-2 split).
* The quantiser's edge cases ("Methodik" 2 of gist.science/de/paper/2605.05699:
  per-group abs-max scale and rounding to signed int4), whose oracle behaviour the
  pins in tests/test_oracle_pins.py fix: groups whose absmax / 7 exceeds the fp16
  range (scale clamped to 65504, codes clamped to +-7), groups small enough for an
  fp16-subnormal scale (codes clamped where the coarse scale would round to 8), and
  all-zero vectors (zero scale, zero codes). They run through every encode path at
  both head dims and through the fused append of kvq_attend_decode_append.
"""
import numpy as np
import pytest

import kvgen
import oracle
from tests.parity import MAX_BOUNDARY_FRAC, check_encode, check_rel_l2

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

# boundary mismatches and elements over every encode of this file (the acceptance rule
# bounds the fraction over all elements encoded, not per small case)
_TALLY = {"bad": 0, "all": 0}


@pytest.fixture(scope="module")
def kvq():
    import rotated_int4_kv_b200 as k
    return k


@pytest.fixture
def encode_path(kvq, request):
    kvq.set_encode_path(request.param)
    yield request.param
    kvq.set_encode_path("auto")


@pytest.mark.parametrize("encode_path", ["auto", "fft", "tensor", "split"], indirect=True)
def test_gemma_step_grouped_encode_every_row(kvq, encode_path):
    """The benchmark's encode launch (bench.py, default workload, rank 0, first input set)."""
    wl = kvgen.WORKLOADS["gemma"]
    L, Hkv, D, T, G = wl.layers, wl.h_kv, wl.head_dim, wl.contexts[0], wl.group
    seed = kvgen.DEFAULT_SEED
    dev = torch.device("cuda")
    NJ = 2 * L
    params = [kvgen.plan_params(D, seed=seed, layer=j // 2, kind="kv"[j % 2]) for j in range(NJ)]
    plans = [kvq.Plan(s, lam, group=G) for s, lam in params]
    x = torch.empty((NJ, Hkv, T, D), dtype=torch.float16, device=dev)
    for j in range(NJ):
        kvgen.kv_torch(wl, "kv"[j % 2], (1, Hkv, T, D), dev, seed=seed, layer=j // 2, salt=0, out=x[j:j + 1])
    codes = torch.full((NJ, Hkv, T, D // 2), 0xA5, dtype=torch.uint8, device=dev)
    scales = torch.full((NJ, Hkv, T, D // G), 7.0, dtype=torch.float16, device=dev)
    kvq.encode_batch([(plans[j], x[j:j + 1], codes[j:j + 1], scales[j:j + 1], 0) for j in range(NJ)])
    torch.cuda.synchronize()
    assert kvq.poll_device_errors() == 0
    xs, cs, ss = x.cpu().numpy(), codes.cpu().numpy(), scales.cpu().numpy()
    n_bad = n_all = 0
    for j in range(NJ):
        s, lam = params[j]
        nb, na = check_encode(xs[j, 0], s, lam, G, cs[j, 0], ss[j, 0], label=f"{encode_path} job {j}",
                              count_only=True)
        n_bad += nb
        n_all += na
    assert n_all == NJ * T * D
    _TALLY["bad"] += n_bad
    _TALLY["all"] += n_all
    assert n_bad <= MAX_BOUNDARY_FRAC * n_all, f"{n_bad} boundary mismatches of {n_all}"


def edge_vectors(D, lam, signs, n_each=4, seed=0):
    """fp16 rows [4 * n_each, D]: clamp rows, subnormal-scale rows, zero rows, ordinary rows.

    Clamp rows: s * (45000 cos(2 pi k n / D)) plus uniform noise of +-20000 (|x| <= 65000),
    with k chosen so that lambda of channel 2k-1 is >= 1.5: that channel reaches
    lambda * 45000 * sqrt(D / 2) / 7 > 65504 (scale clamped, code clamped to 7), the other
    channels carry the noise. Subnormal rows: N(0, 1) * 1e-5 (fp16-subnormal inputs and
    scales). Zero rows: all zeros."""
    rng = np.random.default_rng(seed)
    n = np.arange(D)
    cand = [k for k in range(1, D // 2) if lam[2 * k - 1] >= 1.5]
    assert cand, "no channel with lambda >= 1.5"
    rows = []
    for i in range(n_each):
        k = cand[i % len(cand)]
        wave = 45000.0 * np.cos(2 * np.pi * ((k * n) % D) / D) * signs
        rows.append(wave + rng.uniform(-20000, 20000, D))
    for _ in range(n_each):
        rows.append(rng.standard_normal(D) * 1e-5)
    for _ in range(n_each):
        rows.append(np.zeros(D))
    for _ in range(n_each):
        rows.append(rng.standard_normal(D))
    x = np.asarray(rows, dtype=np.float64).astype(np.float16)
    assert np.isfinite(x.astype(np.float64)).all() and np.abs(x.astype(np.float64)).max() <= 65504
    return x


def _expect_edge_effects(x16, s, lam, G, scales):
    """The edge cases are really exercised: some scale at 65504, some fp16-subnormal
    nonzero scale, zero scales on the zero rows."""
    sc = scales.astype(np.float64)
    assert (sc == 65504.0).any(), "no clamped scale"
    assert ((sc > 0) & (sc < 2.0 ** -14)).any(), "no fp16-subnormal scale"
    zero_rows = ~np.any(x16.astype(np.float64) != 0, axis=-1)
    assert zero_rows.any() and (sc[zero_rows] == 0).all()


@pytest.mark.parametrize("encode_path", ["tensor", "fft", "split"], indirect=True)
@pytest.mark.parametrize("D", [128, 256])
def test_quantiser_edges_on_both_encode_paths(kvq, encode_path, D):
    if encode_path == "split" and D != 256:
        pytest.skip("the radix-2 split kernel serves head_dim 256")
    s, lam = kvgen.plan_params(D, seed=31, kind="k")
    plan = kvq.Plan(s, lam)
    x16 = edge_vectors(D, lam, s, n_each=40, seed=D)
    rng = np.random.default_rng(1)
    x16 = x16[rng.permutation(len(x16))]  # edge rows spread over the tile, next to ordinary rows
    n = len(x16)
    dev = torch.device("cuda")
    codes = torch.full((1, 1, n + 3, D // 2), 0xA5, dtype=torch.uint8, device=dev)
    scales = torch.full((1, 1, n + 3, D // 32), 7.0, dtype=torch.float16, device=dev)
    kvq.encode(plan, torch.from_numpy(x16[None, None]).to(dev), codes, scales, 2)
    torch.cuda.synchronize()
    assert kvq.poll_device_errors() == 0
    c = codes.cpu().numpy()[0, 0, 2:2 + n]
    sc = scales.cpu().numpy()[0, 0, 2:2 + n]
    _expect_edge_effects(x16, s, lam, 32, sc)
    # zero rows: every code byte 0
    zero_rows = ~np.any(x16.astype(np.float64) != 0, axis=-1)
    assert not c[zero_rows].any()
    nb, na = check_encode(x16, s, lam, 32, c, sc, label=f"edges {encode_path} D{D}", count_only=True)
    _TALLY["bad"] += nb
    _TALLY["all"] += na
    # the clamped channel carries code +-7 with the 65504 scale
    codes_g = oracle.unpack_nibbles(c)
    clamped = np.repeat(sc.astype(np.float64) == 65504.0, 32, axis=-1)
    assert (np.abs(codes_g[clamped]) == 7).any()
    # rows outside the written range untouched
    cc = codes.cpu().numpy()[0, 0]
    assert (cc[:2] == 0xA5).all() and (cc[2 + n:] == 0xA5).all()


@pytest.mark.parametrize("D", [128, 256])
@pytest.mark.parametrize("which", ["k", "v"])
def test_quantiser_edges_in_fused_append(kvq, D, which):
    """The new token's K (or V) row of a fused-append step takes each edge value in turn
    (clamp, subnormal, zero); the other of K / V is ordinary. The appended row passes the
    encode rule against the oracle and the attention output matches the oracle on the
    GPU's own cache."""
    wl = kvgen.WORKLOADS["gemma" if D == 256 else "qwen"]
    B, Hkv, Hq, T_cap, pos = 1, 2, 8, 260, 257
    dev = torch.device("cuda")
    params = {kind: kvgen.plan_params(D, seed=37, kind=kind) for kind in ("k", "v")}
    plans = {kind: kvq.Plan(*params[kind]) for kind in ("k", "v")}
    caches, xs = {}, {}
    for kind in ("k", "v"):
        x = kvgen.kv_numpy(wl, kind, (B, Hkv, pos, D), seed=37)
        codes = torch.zeros((B, Hkv, T_cap, D // 2), dtype=torch.uint8, device=dev)
        scales = torch.zeros((B, Hkv, T_cap, D // 32), dtype=torch.float16, device=dev)
        kvq.encode(plans[kind], torch.from_numpy(x).to(dev), codes, scales, 0)
        caches[kind] = (codes, scales)
    s, lam = params[which]
    edge = edge_vectors(D, lam, s, n_each=2, seed=5)
    other = "v" if which == "k" else "k"
    q16 = kvgen.q_numpy((B, Hq, D), salt=4)
    q = torch.from_numpy(q16).to(dev)
    seen = []
    for kind_rows in (edge[0:2], edge[2:4], edge[4:6]):  # clamp, subnormal, zero (one row per kv head)
        new = {which: kind_rows.reshape(B, Hkv, D),
               other: kvgen.kv_numpy(wl, other, (B, Hkv, D), seed=38 + len(seen))}
        out = kvq.attend_decode_append(plans["k"], plans["v"], q, torch.from_numpy(new["k"]).to(dev),
                                       torch.from_numpy(new["v"]).to(dev), *caches["k"], *caches["v"], pos)
        torch.cuda.synchronize()
        assert kvq.poll_device_errors() == 0
        for kind in ("k", "v"):
            ps, pl = params[kind]
            nb, na = check_encode(new[kind][:, :, None], ps, pl, 32,
                                  caches[kind][0][:, :, pos:pos + 1].cpu().numpy(),
                                  caches[kind][1][:, :, pos:pos + 1].cpu().numpy(),
                                  label=f"append {which} {D} row {len(seen)} {kind}", count_only=True)
            _TALLY["bad"] += nb
            _TALLY["all"] += na
        seen.append(caches[which][1][:, :, pos].cpu().numpy())
        ref = oracle.attend_decode_int4(q16, caches["k"][0].cpu().numpy(), caches["k"][1].cpu().numpy(),
                                        caches["v"][0].cpu().numpy(), caches["v"][1].cpu().numpy(), params["k"],
                                        params["v"], [pos + 1] * B)
        check_rel_l2(out.cpu().numpy().astype(np.float64).reshape(-1, D), ref.reshape(-1, D),
                     label=f"append {which} D{D} row {len(seen)}")
    clamp_sc, sub_sc, zero_sc = (x.astype(np.float64) for x in seen)
    assert (clamp_sc == 65504.0).any()
    assert ((sub_sc > 0) & (sub_sc < 2.0 ** -14)).any()
    assert (zero_sc == 0).all()


def test_boundary_fraction_over_this_file():
    if _TALLY["all"] == 0:
        pytest.skip("runs after the encode cases of this file")
    assert _TALLY["bad"] <= MAX_BOUNDARY_FRAC * _TALLY["all"], f"{_TALLY['bad']} boundary mismatches of {_TALLY['all']}"
