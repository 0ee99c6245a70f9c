"""Seeded random shapes through the whole path against the oracle: head_dim, code width,
group size, transform, batch, KV heads, GQA ratio, cache capacity and ragged lengths
(empty sequences included) are drawn per case; each cache is encoded in two calls split
at a random position, every code row is checked against the oracle's encode, and decode
attention over ragged lengths against the oracle on the same packed cache, with the
acceptance rules of the fixed cases. Small sizes, so the oracle stays quick."""
import numpy as np
import pytest

import kvgen
import oracle
from tests.parity import BOUNDARY_TALLY, MAX_BOUNDARY_FRAC_INT8, check_encode, check_rel_l2

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

N_CASES = 24


def _case(i):
    rng = np.random.default_rng(1000 + i)
    D = int(rng.choice([128, 256]))
    bits = int(rng.choice([4, 8]))
    G = int(rng.choice([32, 16]))
    xf = str(rng.choice(["srft", "srht"]))
    B = int(rng.integers(1, 4))
    Hkv = int(rng.integers(1, 4))
    ratio = int(rng.choice([1, 2, 4, 6, 8, 12]))
    T_cap = 2 * int(rng.integers(1, 700))
    lens = [int(rng.integers(0, T_cap + 1)) for _ in range(B)]
    if i % 5 == 0:
        lens[0] = 0
    return dict(D=D, bits=bits, G=G, xf=xf, B=B, Hkv=Hkv, Hq=Hkv * ratio, T_cap=T_cap, lens=lens, seed=2000 + i)


CASES = [_case(i) for i in range(N_CASES)]


@pytest.mark.parametrize("c", CASES, ids=[f"D{c['D']}-i{c['bits']}-G{c['G']}-{c['xf']}-B{c['B']}-kv{c['Hkv']}-q{c['Hq']}"
                                           f"-T{c['T_cap']}" for c in CASES])
def test_random_shape(c):
    import rotated_int4_kv_b200 as kvq

    D, bits, G, xf, B, Hkv, Hq, T_cap, lens = (c[k] for k in ("D", "bits", "G", "xf", "B", "Hkv", "Hq", "T_cap", "lens"))
    wl = kvgen.WORKLOADS["qwen" if D == 128 else "gemma"]
    dev = torch.device("cuda")
    cache = {}
    for kind in ("k", "v"):
        s, lam = kvgen.plan_params(D, seed=c["seed"], kind=kind)
        plan = kvq.Plan(s, lam, G, xf, bits)
        x16 = kvgen.kv_numpy(wl, kind, (B, Hkv, T_cap, D), seed=c["seed"])
        codes = torch.zeros((B, Hkv, T_cap, D * bits // 8), dtype=torch.uint8, device=dev)
        scales = torch.zeros((B, Hkv, T_cap, D // G), dtype=torch.float16, device=dev)
        # the cache in two encodes: rows [0, pos) then [pos, T_cap)
        pos = int(np.random.default_rng(c["seed"]).integers(0, T_cap + 1))
        if pos:
            kvq.encode(plan, torch.from_numpy(np.ascontiguousarray(x16[:, :, :pos])).to(dev), codes, scales, 0)
        if T_cap - pos:
            kvq.encode(plan, torch.from_numpy(np.ascontiguousarray(x16[:, :, pos:])).to(dev), codes, scales, pos)
        cache[kind] = (plan, (s, lam), codes, scales, x16)
    q16 = kvgen.q_numpy((B, Hq, D), seed=c["seed"])
    k, v = cache["k"], cache["v"]
    out = kvq.attend_decode(k[0], v[0], torch.from_numpy(q16).to(dev), k[2], k[3], v[2], v[3],
                            seq_lens=torch.tensor(lens, dtype=torch.int32, device=dev))
    torch.cuda.synchronize()
    assert kvq.poll_device_errors() == 0
    got = out.cpu().numpy().astype(np.float64)
    kc, ks, vc, vs = (t.cpu().numpy() for t in (k[2], k[3], v[2], v[3]))
    # the codes of every row against the oracle's encode (with the GPU's stored scales)
    for kind, (cc, ss) in (("k", (kc, ks)), ("v", (vc, vs))):
        plan_params = cache[kind][1]
        nb, na = check_encode(cache[kind][4], plan_params[0], plan_params[1], G, cc, ss, label=f"{kind} codes",
                              count_only=True, transform=xf, bits=bits)
        if bits == 4:
            BOUNDARY_TALLY["bad"] += nb
            BOUNDARY_TALLY["all"] += na
        else:
            assert nb <= max(1, MAX_BOUNDARY_FRAC_INT8 * na), (nb, na)
    for b in range(B):
        if lens[b] == 0:
            assert np.all(got[b] == 0), "an empty sequence must give zeros"
            continue
        ref = oracle.attend_decode_int4(q16[b:b + 1], kc[b:b + 1], ks[b:b + 1], vc[b:b + 1], vs[b:b + 1], k[1], v[1],
                                        [lens[b]], G, transform=xf, bits=bits)
        check_rel_l2(got[b:b + 1].reshape(-1, D), ref.reshape(-1, D), label=f"b{b} T{lens[b]}")


APPEND_CASES = [c for i, c in enumerate(CASES) if i % 2 == 0]


@pytest.mark.parametrize("c", APPEND_CASES, ids=[f"D{c['D']}-i{c['bits']}-G{c['G']}-{c['xf']}-B{c['B']}-kv{c['Hkv']}"
                                                  f"-q{c['Hq']}-T{c['T_cap']}" for c in APPEND_CASES])
def test_random_append_and_partials(c):
    """The fused append at a random position, then the sequence split into random slices
    (partials + combine), both against the oracle on the GPU's own cache."""
    import rotated_int4_kv_b200 as kvq

    D, bits, G, xf, B, Hkv, Hq, T_cap = (c[k] for k in ("D", "bits", "G", "xf", "B", "Hkv", "Hq", "T_cap"))
    wl = kvgen.WORKLOADS["qwen" if D == 128 else "gemma"]
    dev = torch.device("cuda")
    rng = np.random.default_rng(c["seed"] + 7)
    pos = int(rng.integers(0, T_cap))  # the new token's row; rows [0, pos) are cached
    cache = {}
    for kind in ("k", "v"):
        s, lam = kvgen.plan_params(D, seed=c["seed"], kind=kind)
        plan = kvq.Plan(s, lam, G, xf, bits)
        codes = torch.zeros((B, Hkv, T_cap, D * bits // 8), dtype=torch.uint8, device=dev)
        scales = torch.zeros((B, Hkv, T_cap, D // G), dtype=torch.float16, device=dev)
        if pos:
            x16 = kvgen.kv_numpy(wl, kind, (B, Hkv, pos, D), seed=c["seed"])
            kvq.encode(plan, torch.from_numpy(x16).to(dev), codes, scales, 0)
        new = kvgen.kv_numpy(wl, kind, (B, Hkv, D), seed=c["seed"], salt=5)
        cache[kind] = (plan, (s, lam), codes, scales, new)
    q16 = kvgen.q_numpy((B, Hq, D), seed=c["seed"], salt=3)
    q = torch.from_numpy(q16).to(dev)
    k, v = cache["k"], cache["v"]
    out = kvq.attend_decode_append(k[0], v[0], q, torch.from_numpy(k[4]).to(dev), torch.from_numpy(v[4]).to(dev),
                                   k[2], k[3], v[2], v[3], pos)
    torch.cuda.synchronize()
    assert kvq.poll_device_errors() == 0
    kc, ks, vc, vs = (t.cpu().numpy() for t in (k[2], k[3], v[2], v[3]))
    T = pos + 1
    ref = oracle.attend_decode_int4(q16, kc, ks, vc, vs, k[1], v[1], [T] * B, G, transform=xf, bits=bits)
    check_rel_l2(out.cpu().numpy().astype(np.float64).reshape(-1, D), ref.reshape(-1, D), label=f"append pos {pos}")
    # the same T tokens in random slices (even starts), merged by the combine kernel
    cuts = sorted({0, T} | {2 * int(x) for x in rng.integers(0, T // 2 + 1, size=int(rng.integers(1, 4)))})
    cuts = [x for x in cuts if x <= T]
    if cuts[-1] != T:
        cuts.append(T)
    parts = [kvq.attend_decode_partial(k[0], v[0], q, k[2], k[3], v[2], v[3], cuts[j], cuts[j + 1])
             for j in range(len(cuts) - 1)]
    merged = kvq.attend_combine(v[0], torch.stack(parts))
    torch.cuda.synchronize()
    assert kvq.poll_device_errors() == 0
    check_rel_l2(merged.cpu().numpy().astype(np.float64).reshape(-1, D), ref.reshape(-1, D), label=f"slices {cuts}")


def test_head_dim_mismatch_is_refused():
    """The C ABI sizes rows by the plan's head_dim: the binding refuses tensors of another
    head_dim before anything is launched."""
    import rotated_int4_kv_b200 as kvq

    pk = kvq.Plan(*kvgen.plan_params(128, kind="k"))
    pv = kvq.Plan(*kvgen.plan_params(128, kind="v"))
    dev = torch.device("cuda")
    x = torch.zeros((1, 1, 4, 64), dtype=torch.float16, device=dev)
    codes = torch.zeros((1, 1, 4, 32), dtype=torch.uint8, device=dev)
    scales = torch.zeros((1, 1, 4, 2), dtype=torch.float16, device=dev)
    with pytest.raises(ValueError, match="head_dim"):
        kvq.encode(pk, x, codes, scales)
    q = torch.zeros((1, 4, 64), dtype=torch.float16, device=dev)
    with pytest.raises(ValueError, match="head_dim"):
        kvq.attend_decode(pk, pv, q, codes, scales, codes, scales, T_len=4)
    with pytest.raises(ValueError, match="head_dim"):
        kvq.attend_decode_batch([(pk, pv, q, codes, scales, codes, scales)], T_len=4)
    with pytest.raises(ValueError, match="head_dim"):
        kvq.attend_combine(pv, torch.zeros((2, 1, 4, 68), dtype=torch.float32, device=dev))
