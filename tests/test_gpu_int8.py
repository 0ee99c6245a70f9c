"""GPU parity of int8-code plans (the pages' "Methodik" 2 rounds to signed int4/int8;
int8 here is the int4 quantiser with 127 in place of 7 and one byte per code) on every
entry point that serves them, against the oracle with bits = 8: the tensor-core encode
(D = 128 / 256, G = 32 / 16, SRFT / SRHT), decode, decode attention (GQA, ragged
lengths, several tiles and a ragged tail, batched jobs, the allocation-free variant),
the fused append, sequence-sharded partials and the cache wrapper; both encode paths
(tensor cores, register FFT)."""
import numpy as np
import pytest

import kvgen
import oracle
from tests.parity import MAX_BOUNDARY_FRAC_INT8, check_encode, check_rel_l2

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu
BITS = 8
TALLY = {"bad": 0, "all": 0}


@pytest.fixture(scope="module")
def kvq():
    import rotated_int4_kv_b200 as k
    return k


def _plan(kvq, D, kind, G=32, xf="srft", layer=0, seed=81):
    s, lam = kvgen.plan_params(D, seed=seed, layer=layer, kind=kind)
    return kvq.Plan(s, lam, G, xf, BITS), (s, lam)


@pytest.mark.parametrize("path", ["tensor", "fft", "split"])
@pytest.mark.parametrize("xf", ["srft", "srht"])
@pytest.mark.parametrize("wl_name,B,H,n,G", [("qwen", 2, 2, 130, 32), ("gemma", 1, 1, 300, 32), ("toy", 1, 1, 77, 16),
                                             ("gemma", 2, 1, 65, 16), ("mistral", 1, 3, 513, 32)])
def test_int8_encode_decode(kvq, path, xf, wl_name, B, H, n, G):
    wl = kvgen.WORKLOADS[wl_name]
    D = wl.head_dim
    if path == "split" and (D != 256 or xf != "srft"):
        pytest.skip("the radix-2 split kernel serves head_dim 256 SRFT plans")
    plan, (s, lam) = _plan(kvq, D, "k", G, xf)
    assert plan.bits == 8 and plan.code_row_bytes == D
    x16 = kvgen.kv_numpy(wl, "k", (B, H, n, D), seed=81)
    T_cap, pos = n + 6, 3
    codes = torch.full((B, H, T_cap, D), 0xA5, dtype=torch.uint8, device="cuda")
    scales = torch.full((B, H, T_cap, D // G), 7.0, dtype=torch.float16, device="cuda")
    kvq.set_encode_path(path)
    try:
        kvq.encode(plan, torch.from_numpy(x16).cuda(), codes, scales, pos)
    finally:
        kvq.set_encode_path("auto")
    torch.cuda.synchronize()
    assert kvq.poll_device_errors() == 0
    c, sc = codes.cpu().numpy(), scales.cpu().numpy()
    nb, na = check_encode(x16, s, lam, G, c[:, :, pos:pos + n], sc[:, :, pos:pos + n], label=f"{wl_name} {xf} {path}",
                          count_only=True, transform=xf, bits=BITS)
    TALLY["bad"] += nb
    TALLY["all"] += na
    # rows outside [pos, pos + n) untouched; no code is -128
    assert np.all(c[:, :, :pos] == 0xA5) and np.all(c[:, :, pos + n:] == 0xA5)
    assert not np.any(c[:, :, pos:pos + n] == 0x80)
    out = kvq.decode(plan, codes, scales, pos, n)
    torch.cuda.synchronize()
    ref = oracle.decode(c[:, :, pos:pos + n], sc[:, :, pos:pos + n], s, lam, G, xf, BITS)
    check_rel_l2(out.cpu().numpy().astype(np.float64).reshape(-1, D), ref.reshape(-1, D), label="decode")
    # int8 codes reconstruct the input about 18x more closely than int4 (sanity on the real data)
    x = x16.astype(np.float64).reshape(-1, D)
    assert np.linalg.norm(ref.reshape(-1, D) - x) / np.linalg.norm(x) < 2e-2


def test_int8_grouped_encode_batch(kvq):
    wl = kvgen.WORKLOADS["gemma"]
    D, G, n = wl.head_dim, 32, 200
    jobs, refs = [], []
    for layer in range(3):
        for kind in ("k", "v"):
            plan, (s, lam) = _plan(kvq, D, kind, G, layer=layer)
            x16 = kvgen.kv_numpy(wl, kind, (1, 1, n, D), seed=82, layer=layer)
            codes = torch.zeros((1, 1, n, D), dtype=torch.uint8, device="cuda")
            scales = torch.zeros((1, 1, n, D // G), dtype=torch.float16, device="cuda")
            jobs.append((plan, torch.from_numpy(x16).cuda(), codes, scales, 0))
            refs.append((x16, s, lam))
    kvq.encode_batch(jobs)
    torch.cuda.synchronize()
    for (plan, _, codes, scales, _), (x16, s, lam) in zip(jobs, refs):
        nb, na = check_encode(x16, s, lam, G, codes.cpu().numpy(), scales.cpu().numpy(), label="batch",
                              count_only=True, bits=BITS)
        TALLY["bad"] += nb
        TALLY["all"] += na


def test_int8_and_int4_plans_do_not_mix(kvq):
    D = 128
    plan, _ = _plan(kvq, D, "k")
    codes = torch.zeros((1, 1, 4, D), dtype=torch.uint8, device="cuda")
    scales = torch.zeros((1, 1, 4, D // 32), dtype=torch.float16, device="cuda")
    s, lam = kvgen.plan_params(D, kind="v")
    pv4 = kvq.Plan(s, lam)  # int4
    q = torch.zeros((1, 4, D), dtype=torch.float16, device="cuda")
    with pytest.raises(kvq.KvqError, match="INVALID_ARG"):
        kvq.attend_decode(plan, pv4, q, codes, scales, codes, scales, T_len=4)


def _cache(kvq, wl, B, Hkv, T_cap, T_fill, G=32, xf="srft", layer=0, seed=83):
    D = wl.head_dim
    out = {}
    for kind in ("k", "v"):
        plan, params = _plan(kvq, D, kind, G, xf, layer=layer, seed=seed)
        codes = torch.zeros((B, Hkv, T_cap, D), dtype=torch.uint8, device="cuda")
        scales = torch.zeros((B, Hkv, T_cap, D // G), dtype=torch.float16, device="cuda")
        if T_fill:
            x = torch.from_numpy(kvgen.kv_numpy(wl, kind, (B, Hkv, T_fill, D), seed=seed, layer=layer)).cuda()
            kvq.encode(plan, x, codes, scales, 0)
        out[kind] = dict(plan=plan, params=params, codes=codes, scales=scales)
    return out


def _oracle(q16, cache, lens, G=32, xf="srft"):
    k, v = cache["k"], cache["v"]
    return oracle.attend_decode_int4(q16, k["codes"].cpu().numpy(), k["scales"].cpu().numpy(), v["codes"].cpu().numpy(),
                                     v["scales"].cpu().numpy(), k["params"], v["params"], lens, G, transform=xf,
                                     bits=BITS)


ATT_CASES = [
    # (workload, B, Hkv, Hq, T_cap, lens, G, transform)
    ("qwen", 1, 2, 12, 1024, None, 32, "srft"),
    ("qwen", 2, 2, 12, 300, [300, 41], 32, "srft"),
    ("longctx", 1, 1, 16, 200, None, 32, "srft"),        # two head tiles
    ("gemma", 1, 1, 4, 2048, None, 32, "srft"),          # D = 256
    ("gemma", 2, 2, 6, 334, [333, 17], 32, "srft"),      # ragged tail
    ("mistral", 2, 2, 8, 3000, [3000, 2077], 32, "srft"),
    ("qwen", 1, 2, 12, 700, None, 16, "srft"),
    ("gemma", 1, 1, 4, 500, None, 16, "srft"),
    ("qwen", 1, 2, 12, 900, None, 32, "srht"),
    ("gemma", 1, 1, 4, 600, [555], 32, "srht"),
    ("qwen", 1, 2, 12, 64, [0], 32, "srft"),             # empty sequence
]


@pytest.mark.parametrize("case", ATT_CASES, ids=[f"{c[0]}-B{c[1]}-T{c[4]}-G{c[6]}-{c[7]}" for c in ATT_CASES])
def test_int8_attention(kvq, case):
    wl_name, B, Hkv, Hq, T_cap, lens, G, xf = case
    wl = kvgen.WORKLOADS[wl_name]
    D = wl.head_dim
    cache = _cache(kvq, wl, B, Hkv, T_cap, T_cap, G, xf)
    q16 = kvgen.q_numpy((B, Hq, D), salt=21)
    q = torch.from_numpy(q16).cuda()
    k, v = cache["k"], cache["v"]
    if lens is None:
        out = kvq.attend_decode(k["plan"], v["plan"], q, k["codes"], k["scales"], v["codes"], v["scales"], T_len=T_cap)
        lens = [T_cap] * B
    else:
        out = kvq.attend_decode(k["plan"], v["plan"], q, k["codes"], k["scales"], v["codes"], v["scales"],
                                seq_lens=torch.tensor(lens, dtype=torch.int32, device="cuda"))
    torch.cuda.synchronize()
    assert kvq.poll_device_errors() == 0
    got = out.cpu().numpy().astype(np.float64)
    for b in range(B):
        if lens[b] == 0:
            assert np.all(got[b] == 0)
    live = [b for b in range(B) if lens[b] > 0]
    if live:
        ref = _oracle(q16[live], {kk: dict(vv, codes=vv["codes"][live], scales=vv["scales"][live])
                                  for kk, vv in cache.items()}, [lens[b] for b in live], G, xf)
        check_rel_l2(got[live].reshape(-1, D), ref.reshape(-1, D), label=f"int8 {case}")


def test_int8_attention_batch_and_noalloc_match_single(kvq):
    wl = kvgen.WORKLOADS["qwen"]
    D, B, Hkv, Hq, T = wl.head_dim, 1, 2, 12, 777
    caches = [_cache(kvq, wl, B, Hkv, T + 1, T, layer=l) for l in range(3)]
    qs = [torch.from_numpy(kvgen.q_numpy((B, Hq, D), salt=30 + l)).cuda() for l in range(3)]
    single = [kvq.attend_decode(c["k"]["plan"], c["v"]["plan"], q, c["k"]["codes"], c["k"]["scales"], c["v"]["codes"],
                                c["v"]["scales"], T_len=T) for c, q in zip(caches, qs)]
    jobs = [(c["k"]["plan"], c["v"]["plan"], q, c["k"]["codes"], c["k"]["scales"], c["v"]["codes"], c["v"]["scales"])
            for c, q in zip(caches, qs)]
    batched = kvq.attend_decode_batch(jobs, T_len=T)
    c0 = caches[0]
    na = kvq.attend_decode_noalloc(c0["k"]["plan"], c0["v"]["plan"], qs[0], c0["k"]["codes"], c0["k"]["scales"],
                                   c0["v"]["codes"], c0["v"]["scales"], T_len=T)
    torch.cuda.synchronize()
    assert kvq.poll_device_errors() == 0
    for a, b in zip(single, batched):
        check_rel_l2(b.cpu().numpy().astype(np.float64).reshape(-1, D), a.cpu().numpy().astype(np.float64).reshape(-1, D),
                     tol=1e-3, label="batch vs single")
    check_rel_l2(na.cpu().numpy().astype(np.float64).reshape(-1, D),
                 single[0].cpu().numpy().astype(np.float64).reshape(-1, D), tol=1e-3, label="noalloc vs single")
    ref = _oracle(kvgen.q_numpy((B, Hq, D), salt=30), c0, [T])
    check_rel_l2(single[0].cpu().numpy().astype(np.float64).reshape(-1, D), ref.reshape(-1, D), label="vs oracle")


@pytest.mark.parametrize("wl_name,B,Hkv,Hq,T_cap,pos,G", [("qwen", 1, 2, 12, 516, 514, 32), ("gemma", 1, 1, 4, 258, 257, 32),
                                                           ("qwen", 1, 2, 12, 64, 0, 32), ("qwen", 2, 2, 12, 300, 131, 16),
                                                           ("gemma", 1, 1, 4, 130, 77, 16)])
def test_int8_fused_append(kvq, wl_name, B, Hkv, Hq, T_cap, pos, G):
    wl = kvgen.WORKLOADS[wl_name]
    D = wl.head_dim
    cache = _cache(kvq, wl, B, Hkv, T_cap, pos, G)
    before = {kind: cache[kind]["codes"].clone() for kind in ("k", "v")}
    new = {kind: kvgen.kv_numpy(wl, kind, (B, Hkv, D), seed=84) for kind in ("k", "v")}
    q16 = kvgen.q_numpy((B, Hq, D), salt=22)
    k, v = cache["k"], cache["v"]
    out = kvq.attend_decode_append(k["plan"], v["plan"], torch.from_numpy(q16).cuda(),
                                   torch.from_numpy(new["k"]).cuda(), torch.from_numpy(new["v"]).cuda(),
                                   k["codes"], k["scales"], v["codes"], v["scales"], pos)
    torch.cuda.synchronize()
    assert kvq.poll_device_errors() == 0
    for kind in ("k", "v"):
        c = cache[kind]
        nb, na = check_encode(new[kind][:, :, None], c["params"][0], c["params"][1], G,
                              c["codes"][:, :, pos:pos + 1].cpu().numpy(), c["scales"][:, :, pos:pos + 1].cpu().numpy(),
                              label=f"append {kind}", count_only=True, bits=BITS)
        TALLY["bad"] += nb
        TALLY["all"] += na
        # every other row untouched
        diff = (c["codes"] != before[kind]).any(dim=-1).cpu().numpy()
        assert not diff[:, :, :pos].any() and not diff[:, :, pos + 1:].any()
    ref = _oracle(q16, cache, [pos + 1] * B, G)
    check_rel_l2(out.cpu().numpy().astype(np.float64).reshape(-1, D), ref.reshape(-1, D), label=f"append {wl_name}")


def test_int8_partials_combine(kvq):
    wl = kvgen.WORKLOADS["qwen"]
    D, B, Hkv, Hq, T = wl.head_dim, 1, 2, 12, 1200
    cache = _cache(kvq, wl, B, Hkv, T, T)
    k, v = cache["k"], cache["v"]
    q16 = kvgen.q_numpy((B, Hq, D), salt=23)
    q = torch.from_numpy(q16).cuda()
    cuts = [0, 400, 1000, 1200]
    parts = [kvq.attend_decode_partial(k["plan"], v["plan"], q, k["codes"], k["scales"], v["codes"], v["scales"],
                                       cuts[i], cuts[i + 1]) for i in range(len(cuts) - 1)]
    out = kvq.attend_combine(v["plan"], torch.stack(parts))
    torch.cuda.synchronize()
    assert kvq.poll_device_errors() == 0
    ref = _oracle(q16, cache, [T])
    check_rel_l2(out.cpu().numpy().astype(np.float64).reshape(-1, D), ref.reshape(-1, D), label="partials")


def test_int8_cache_wrapper(kvq):
    wl = kvgen.WORKLOADS["qwen"]
    D, B, Hkv, Hq = wl.head_dim, 1, 2, 12
    kp = kvgen.plan_params(D, seed=85, kind="k")
    vp = kvgen.plan_params(D, seed=85, kind="v")
    cache = kvq.Int4KVCache(1, B, Hkv, D, 300, kp, vp, bits=8)
    assert cache.k_codes[0].shape[-1] == D
    assert cache.compression_vs_fp16() == pytest.approx(2 * D / (D + 2 * D // 32))
    xk = torch.from_numpy(kvgen.kv_numpy(wl, "k", (B, Hkv, 200, D), seed=85)).cuda()
    xv = torch.from_numpy(kvgen.kv_numpy(wl, "v", (B, Hkv, 200, D), seed=85)).cuda()
    cache.update(0, xk, xv)
    q16 = kvgen.q_numpy((B, Hq, D), salt=24)
    kn = torch.from_numpy(kvgen.kv_numpy(wl, "k", (B, Hkv, D), seed=86)).cuda()
    vn = torch.from_numpy(kvgen.kv_numpy(wl, "v", (B, Hkv, D), seed=86)).cuda()
    out = cache.step(0, torch.from_numpy(q16).cuda(), kn, vn)
    torch.cuda.synchronize()
    assert kvq.poll_device_errors() == 0 and cache.seq_length(0) == 201
    ref = oracle.attend_decode_int4(q16, cache.k_codes[0].cpu().numpy(), cache.k_scales[0].cpu().numpy(),
                                    cache.v_codes[0].cpu().numpy(), cache.v_scales[0].cpu().numpy(), kp, vp, [201], 32,
                                    bits=BITS)
    check_rel_l2(out.cpu().numpy().astype(np.float64).reshape(-1, D), ref.reshape(-1, D), label="cache step")


def test_int8_boundary_fraction_over_all_cases():
    if TALLY["all"] == 0:
        pytest.skip("no int8 encode ran")
    assert TALLY["bad"] <= MAX_BOUNDARY_FRAC_INT8 * TALLY["all"], TALLY
