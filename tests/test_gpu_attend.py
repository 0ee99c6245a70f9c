"""GPU parity of kvq_attend_decode (int4, rotated domain) and kvq_attend_decode_ref
(fp16) against the oracle, through the C ABI. The int4 oracle runs on the GPU's
own packed cache (codes and scales copied back), per the acceptance rule."""
import numpy as np
import pytest

import kvgen
import oracle
from tests.parity import check_rel_l2

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def kvq():
    import rotated_int4_kv_b200 as k
    return k


def _build_cache(kvq, wl, B, Hkv, T_cap, T_fill, seed=21, layer=0):
    D = wl.head_dim
    dev = torch.device("cuda")
    out = {}
    for kind in ("k", "v"):
        s, lam = kvgen.plan_params(D, seed=seed, layer=layer, kind=kind)
        plan = kvq.Plan(s, lam)
        x = torch.from_numpy(kvgen.kv_numpy(wl, kind, (B, Hkv, T_fill, D), seed=seed, layer=layer)).to(dev)
        codes = torch.zeros((B, Hkv, T_cap, D // 2), dtype=torch.uint8, device=dev)
        scales = torch.zeros((B, Hkv, T_cap, D // 32), dtype=torch.float16, device=dev)
        kvq.encode(plan, x, codes, scales, 0)
        out[kind] = dict(plan=plan, params=(s, lam), x=x, codes=codes, scales=scales)
    return out


def _oracle_int4(q16, cache, lens, sigma=None):
    k, v = cache["k"], cache["v"]
    return oracle.attend_decode_int4(q16, k["codes"].cpu().numpy(), k["scales"].cpu().numpy(),
                                     v["codes"].cpu().numpy(), v["scales"].cpu().numpy(), k["params"],
                                     v["params"], lens, 32, sigma)


CASES = [
    # (workload, B, Hkv, Hq, T_cap, lens)  lens: None -> T_len = T_cap
    ("toy", 1, 1, 1, 256, None),
    ("qwen", 1, 2, 12, 1024, None),
    ("qwen", 2, 2, 12, 1000, [1000, 531]),
    ("qwen", 3, 2, 4, 130, [1, 0, 129]),
    ("mistral", 2, 8, 32, 700, [700, 65]),
    ("longctx", 1, 2, 16, 300, None),          # GQA 8
    ("longctx", 1, 1, 16, 200, [77]),           # GQA 16: two head tiles
    ("gemma", 1, 1, 4, 4096, None),             # D = 256
    ("gemma", 2, 2, 6, 334, [333, 17]),         # D = 256, GQA 3, ragged (odd lengths)
]


def _ids(cases):
    return [f"{c[0]}-B{c[1]}kv{c[2]}q{c[3]}T{c[4]}" + ("" if c[5] is None else "ragged") for c in cases]


@pytest.mark.parametrize("case", CASES, ids=_ids(CASES))
def test_attend_int4_matches_oracle(kvq, case):
    wl_name, B, Hkv, Hq, T_cap, lens = case
    wl = kvgen.WORKLOADS[wl_name]
    D = wl.head_dim
    cache = _build_cache(kvq, wl, B, Hkv, T_cap, T_cap)
    q16 = kvgen.q_numpy((B, Hq, D), salt=5)
    q = torch.from_numpy(q16).cuda()
    if lens is None:
        out = kvq.attend_decode(cache["k"]["plan"], cache["v"]["plan"], q, cache["k"]["codes"],
                                cache["k"]["scales"], cache["v"]["codes"], cache["v"]["scales"], T_len=T_cap)
        lens_np = [T_cap] * B
    else:
        sl = torch.tensor(lens, dtype=torch.int32, device="cuda")
        out = kvq.attend_decode(cache["k"]["plan"], cache["v"]["plan"], q, cache["k"]["codes"],
                                cache["k"]["scales"], cache["v"]["codes"], cache["v"]["scales"], seq_lens=sl)
        lens_np = lens
    torch.cuda.synchronize()
    assert kvq.poll_device_errors() == 0
    got = out.cpu().numpy().astype(np.float64)
    ref = np.zeros((B, Hq, D))
    live = [i for i in range(B) if lens_np[i] > 0]
    if live:
        sub = _oracle_int4(q16[live], {k: dict(v, codes=v["codes"][live], scales=v["scales"][live])
                                       for k, v in cache.items()}, [lens_np[i] for i in live])
        ref[live] = sub
    for i in range(B):
        if lens_np[i] == 0:
            assert not got[i].any(), "empty sequence must give zeros"
    if live:
        check_rel_l2(got[live].reshape(-1, D), ref[live].reshape(-1, D), label=str(case))


@pytest.mark.parametrize("case", CASES, ids=_ids(CASES))
def test_attend_fp16_ref_matches_oracle(kvq, case):
    wl_name, B, Hkv, Hq, T_cap, lens = case
    wl = kvgen.WORKLOADS[wl_name]
    D = wl.head_dim
    k16 = kvgen.kv_numpy(wl, "k", (B, Hkv, T_cap, D), seed=31)
    v16 = kvgen.kv_numpy(wl, "v", (B, Hkv, T_cap, D), seed=31)
    q16 = kvgen.q_numpy((B, Hq, D), salt=6)
    k, v, q = (torch.from_numpy(a).cuda() for a in (k16, v16, q16))
    if lens is None:
        out = kvq.attend_decode_ref(q, k, v, T_len=T_cap)
        lens_np = [T_cap] * B
    else:
        out = kvq.attend_decode_ref(q, k, v, seq_lens=torch.tensor(lens, dtype=torch.int32, device="cuda"))
        lens_np = lens
    torch.cuda.synchronize()
    assert kvq.poll_device_errors() == 0
    got = out.cpu().numpy().astype(np.float64)
    live = [i for i in range(B) if lens_np[i] > 0]
    for i in range(B):
        if lens_np[i] == 0:
            assert not got[i].any()
    if live:
        ref = oracle.attend_decode_fp16(q16[live], k16[live], v16[live], [lens_np[i] for i in live])
        check_rel_l2(got[live].reshape(-1, D), ref.reshape(-1, D), label=str(case))


def test_attend_split_independence_and_workspace_reuse(kvq):
    """The same inputs through T_len (split chosen from T_len) and through seq_lens
    (split chosen from T_cap), twice on one workspace, agree to fp32 noise."""
    wl = kvgen.WORKLOADS["qwen"]
    B, Hkv, Hq, T_cap, T = 1, 2, 12, 8192, 600
    cache = _build_cache(kvq, wl, B, Hkv, T_cap, T_cap, seed=5)
    q = torch.from_numpy(kvgen.q_numpy((B, Hq, 128), salt=9)).cuda()
    ws = kvq.make_workspace(B, Hq, Hkv, 128, T_cap)
    args = (cache["k"]["plan"], cache["v"]["plan"], q, cache["k"]["codes"], cache["k"]["scales"],
            cache["v"]["codes"], cache["v"]["scales"])
    a = kvq.attend_decode(*args, T_len=T, workspace=ws).float()
    b = kvq.attend_decode(*args, seq_lens=torch.tensor([T], dtype=torch.int32, device="cuda"), workspace=ws).float()
    c2 = kvq.attend_decode(*args, T_len=T, workspace=ws).float()
    torch.cuda.synchronize()
    assert torch.equal(a, c2)
    assert float((a - b).norm() / a.norm()) < 1e-3
    assert not torch.count_nonzero(ws[:64])  # counters left at zero


def test_attend_errors(kvq):
    wl = kvgen.WORKLOADS["toy"]
    cache = _build_cache(kvq, wl, 1, 1, 64, 64)
    q = torch.zeros((1, 1, 128), dtype=torch.float16, device="cuda")
    args = (cache["k"]["plan"], cache["v"]["plan"], q, cache["k"]["codes"], cache["k"]["scales"],
            cache["v"]["codes"], cache["v"]["scales"])
    with pytest.raises(kvq.KvqError) as e:
        kvq.attend_decode(*args, T_len=65)
    assert e.value.status == -4
    with pytest.raises(kvq.KvqError) as e:
        kvq.attend_decode(*args, T_len=10, workspace=torch.zeros(8, dtype=torch.uint8, device="cuda"))
    assert e.value.status == -6


def test_mistral_full_size_sampled(kvq):
    """Mistral-7B-shaped batched decode at full size (B=16, 8 KV heads, 32 query heads,
    T=32768, D=128), one layer, in the bench's launch configuration; sampled
    (b, q head) rows checked against the oracle on the same packed cache."""
    wl = kvgen.WORKLOADS["mistral"]
    B, Hkv, Hq, T, D = wl.batch, wl.h_kv, wl.h_q, wl.contexts[0], wl.head_dim
    dev = torch.device("cuda")
    plans, caches = {}, {}
    for kind in ("k", "v"):
        s, lam = kvgen.plan_params(D, layer=0, kind=kind)
        plans[kind] = (kvq.Plan(s, lam), (s, lam))
        codes = torch.empty((B, Hkv, T, D // 2), dtype=torch.uint8, device=dev)
        scales = torch.empty((B, Hkv, T, D // 32), dtype=torch.float16, device=dev)
        for b in range(B):
            x = kvgen.kv_torch(wl, kind, (1, Hkv, T, D), dev, layer=0, salt=b)
            kvq.encode(plans[kind][0], x, codes[b:b + 1], scales[b:b + 1], 0)
            if kind == "k" and b == 3:
                k16_b3 = x.clone()
            if kind == "v" and b == 3:
                v16_b3 = x.clone()
        caches[kind] = (codes, scales)
    q = kvgen.q_torch((B, Hq, D), dev)
    out = kvq.attend_decode(plans["k"][0], plans["v"][0], q, caches["k"][0], caches["k"][1], caches["v"][0],
                            caches["v"][1], T_len=T)
    torch.cuda.synchronize()
    assert kvq.poll_device_errors() == 0
    q16 = q.cpu().numpy()
    for b, kvh in ((0, 0), (3, 5), (15, 7)):
        sl = slice(kvh, kvh + 1)
        hq = slice(kvh * 4, kvh * 4 + 4)
        kc = caches["k"][0][b:b + 1, sl].cpu().numpy()
        ks = caches["k"][1][b:b + 1, sl].cpu().numpy()
        vc = caches["v"][0][b:b + 1, sl].cpu().numpy()
        vs = caches["v"][1][b:b + 1, sl].cpu().numpy()
        ref = oracle.attend_decode_int4(q16[b:b + 1, hq], kc, ks, vc, vs, plans["k"][1], plans["v"][1], [T])
        check_rel_l2(out[b:b + 1, hq].cpu().numpy().reshape(-1, D), ref.reshape(-1, D), label=f"b{b} kv{kvh}")
    # the fp16 comparator on the same shapes (batch entry 3's real K/V; others random)
    k16 = torch.empty((B, Hkv, T, D), dtype=torch.float16, device=dev)
    v16 = torch.empty_like(k16)
    kvgen.kv_torch(wl, "k", (B, Hkv, T, D), dev, layer=1, out=k16)
    kvgen.kv_torch(wl, "v", (B, Hkv, T, D), dev, layer=1, out=v16)
    k16[3], v16[3] = k16_b3[0], v16_b3[0]
    o16 = kvq.attend_decode_ref(q, k16, v16, T_len=T)
    torch.cuda.synchronize()
    for kvh in (0, 6):
        hq = slice(kvh * 4, kvh * 4 + 4)
        ref = oracle.attend_decode_fp16(q16[3:4, hq], k16[3:4, kvh:kvh + 1].cpu().numpy(),
                                        v16[3:4, kvh:kvh + 1].cpu().numpy(), [T])
        check_rel_l2(o16[3:4, hq].cpu().numpy().reshape(-1, D), ref.reshape(-1, D), label=f"fp16 kv{kvh}")


BATCH_CASES = [
    # (workload, njobs, B, Hkv, Hq, T_cap, lens): each job its own layer (plans, cache, query)
    ("gemma", 5, 1, 1, 4, 1024, None),          # D = 256, one launch
    ("qwen", 35, 1, 2, 12, 256, [200]),         # D = 128, two launches (32 + 3 jobs)
    ("mistral", 3, 2, 8, 32, 514, [514, 3]),    # ragged batch entries
]


@pytest.mark.parametrize("case", BATCH_CASES, ids=[f"{c[0]}-x{c[1]}" for c in BATCH_CASES])
def test_attend_batch_matches_oracle_per_job(kvq, case):
    wl_name, nj, B, Hkv, Hq, T_cap, lens = case
    wl = kvgen.WORKLOADS[wl_name]
    D = wl.head_dim
    caches = [_build_cache(kvq, wl, B, Hkv, T_cap, T_cap, seed=31, layer=j) for j in range(nj)]
    qs16 = [kvgen.q_numpy((B, Hq, D), salt=100 + j) for j in range(nj)]
    jobs = [(c["k"]["plan"], c["v"]["plan"], torch.from_numpy(q).cuda(), c["k"]["codes"], c["k"]["scales"],
             c["v"]["codes"], c["v"]["scales"]) for c, q in zip(caches, qs16)]
    sl = None if lens is None else torch.tensor(lens * (B // len(lens)) if len(lens) < B else lens,
                                                dtype=torch.int32, device="cuda")
    lens_np = [T_cap] * B if sl is None else sl.cpu().tolist()
    outs = kvq.attend_decode_batch(jobs, seq_lens=sl, T_len=T_cap if sl is None else None)
    singles = [kvq.attend_decode(*j, seq_lens=sl, T_len=T_cap if sl is None else None) for j in jobs]
    torch.cuda.synchronize()
    assert kvq.poll_device_errors() == 0
    for j in range(nj):
        got = outs[j].cpu().numpy().astype(np.float64)
        one = singles[j].cpu().numpy().astype(np.float64)
        # another split of the same sums: equal to fp32 noise
        check_rel_l2(got.reshape(-1, D), one.reshape(-1, D), tol=1e-3, label=f"job {j} vs single call")
        if j in (0, nj - 1):
            ref = _oracle_int4(qs16[j], caches[j], lens_np)
            check_rel_l2(got.reshape(-1, D), ref.reshape(-1, D), tol=2e-3, label=f"job {j} vs oracle")


def test_attend_batch_rejects_mixed_head_dims(kvq):
    g, q = kvgen.WORKLOADS["gemma"], kvgen.WORKLOADS["qwen"]
    cg_ = _build_cache(kvq, g, 1, 1, 64, 64)
    cq = _build_cache(kvq, q, 1, 1, 64, 64)
    jobs = [(c["k"]["plan"], c["v"]["plan"], torch.zeros((1, 4, w.head_dim), dtype=torch.float16, device="cuda"),
             c["k"]["codes"], c["k"]["scales"], c["v"]["codes"], c["v"]["scales"])
            for c, w in ((cg_, g), (cq, q))]
    with pytest.raises(Exception):
        kvq.attend_decode_batch(jobs, T_len=64)


APPEND_CASES = [
    # (workload, B, Hkv, Hq, T_cap, pos): the new token goes to row pos, tokens 0 .. pos attended
    ("toy", 1, 1, 1, 256, 255),
    ("qwen", 1, 2, 12, 1026, 1024),
    ("qwen", 1, 2, 12, 64, 0),                  # empty cache: only the new token
    ("qwen", 3, 2, 12, 200, 130),               # ragged last stage
    ("mistral", 2, 8, 32, 700, 513),
    ("longctx", 1, 1, 16, 200, 77),             # GQA 16: two head tiles append the same token
    ("gemma", 1, 1, 4, 4098, 4096),             # D = 256
    ("gemma", 2, 2, 6, 334, 333),               # D = 256, GQA 3
]


@pytest.mark.parametrize("case", APPEND_CASES, ids=[f"{c[0]}-B{c[1]}kv{c[2]}q{c[3]}pos{c[5]}" for c in APPEND_CASES])
def test_attend_append_matches_encode_then_attend(kvq, case):
    """kvq_attend_decode_append = kvq_encode of the new token at pos + kvq_attend_decode
    over pos + 1 tokens: the row it writes passes the encode acceptance rule against the
    oracle, no other row changes, and its output matches the oracle on the GPU's own
    cache and the two-call path."""
    from tests.parity import BOUNDARY_TALLY, check_encode

    wl_name, B, Hkv, Hq, T_cap, pos = case
    wl = kvgen.WORKLOADS[wl_name]
    D = wl.head_dim
    dev = torch.device("cuda")
    cache = {}
    for kind in ("k", "v"):
        s, lam = kvgen.plan_params(D, seed=23, layer=1, kind=kind)
        plan = kvq.Plan(s, lam)
        x = kvgen.kv_numpy(wl, kind, (B, Hkv, pos + 1, D), seed=23, layer=1)
        codes = torch.full((B, Hkv, T_cap, D // 2), 0x5A, dtype=torch.uint8, device=dev)
        scales = torch.full((B, Hkv, T_cap, D // 32), 3.0, dtype=torch.float16, device=dev)
        if pos > 0:
            kvq.encode(plan, torch.from_numpy(np.ascontiguousarray(x[:, :, :pos])).to(dev), codes, scales, 0)
        cache[kind] = dict(plan=plan, params=(s, lam), x=x, codes=codes, scales=scales,
                           new=torch.from_numpy(np.ascontiguousarray(x[:, :, pos])).to(dev))
    q16 = kvgen.q_numpy((B, Hq, D), salt=9)
    q = torch.from_numpy(q16).to(dev)
    k, v = cache["k"], cache["v"]
    # the two-call path on copies of the caches
    kc2, ks2, vc2, vs2 = (t.clone() for t in (k["codes"], k["scales"], v["codes"], v["scales"]))
    kvq.encode(k["plan"], k["new"].unsqueeze(2), kc2, ks2, pos)
    kvq.encode(v["plan"], v["new"].unsqueeze(2), vc2, vs2, pos)
    out2 = kvq.attend_decode(k["plan"], v["plan"], q, kc2, ks2, vc2, vs2, T_len=pos + 1)
    before = [t.clone() for t in (k["codes"], k["scales"], v["codes"], v["scales"])]
    out = kvq.attend_decode_append(k["plan"], v["plan"], q, k["new"], v["new"], k["codes"], k["scales"],
                                   v["codes"], v["scales"], pos)
    torch.cuda.synchronize()
    assert kvq.poll_device_errors() == 0
    # the appended rows: encode acceptance against the oracle
    for kind in ("k", "v"):
        c = cache[kind]
        s, lam = c["params"]
        nb, na = check_encode(c["x"][:, :, pos:pos + 1], s, lam, 32, c["codes"][:, :, pos:pos + 1].cpu().numpy(),
                              c["scales"][:, :, pos:pos + 1].cpu().numpy(), label=f"{case} {kind}", count_only=True)
        BOUNDARY_TALLY["bad"] += nb
        BOUNDARY_TALLY["all"] += na
    # every other row untouched
    for t_after, t_before in zip((k["codes"], k["scales"], v["codes"], v["scales"]), before):
        keep = torch.ones(T_cap, dtype=torch.bool, device=dev)
        keep[pos] = False
        assert torch.equal(t_after[:, :, keep], t_before[:, :, keep])
    got = out.cpu().numpy().astype(np.float64)
    ref = _oracle_int4(q16, cache, [pos + 1] * B)
    check_rel_l2(got.reshape(-1, D), ref.reshape(-1, D), label=str(case))
    check_rel_l2(got.reshape(-1, D), out2.cpu().numpy().astype(np.float64).reshape(-1, D), label=f"{case} vs two calls")


def test_attend_append_rejects_bad_positions(kvq):
    wl = kvgen.WORKLOADS["qwen"]
    D, B, Hkv, Hq, T_cap = wl.head_dim, 1, 2, 12, 64
    s, lam = kvgen.plan_params(D, kind="k")
    pk = kvq.Plan(s, lam)
    pv = kvq.Plan(*kvgen.plan_params(D, kind="v"))
    dev = torch.device("cuda")
    q = torch.zeros((B, Hq, D), dtype=torch.float16, device=dev)
    kn = torch.zeros((B, Hkv, D), dtype=torch.float16, device=dev)
    codes = torch.zeros((B, Hkv, T_cap, D // 2), dtype=torch.uint8, device=dev)
    scales = torch.zeros((B, Hkv, T_cap, D // 32), dtype=torch.float16, device=dev)
    with pytest.raises(kvq.KvqError, match="CAPACITY"):
        kvq.attend_decode_append(pk, pv, q, kn, kn, codes, scales, codes.clone(), scales.clone(), T_cap)
    with pytest.raises(kvq.KvqError, match="INVALID_ARG"):
        kvq.attend_decode_append(pk, pv, q, kn, kn, codes, scales, codes.clone(), scales.clone(), -1)


G16_CASES = [
    # (workload, B, Hkv, Hq, T_cap, lens)
    ("qwen", 1, 2, 12, 1024, None),
    ("qwen", 2, 2, 12, 300, [300, 41]),
    ("longctx", 1, 1, 16, 200, None),           # two head tiles
    ("gemma", 1, 1, 4, 2048, None),             # D = 256
    ("gemma", 2, 2, 6, 334, [333, 17]),
]


@pytest.mark.parametrize("case", G16_CASES, ids=_ids(G16_CASES))
def test_attend_group16_matches_oracle(kvq, case):
    """Scale groups of 16 channels (the pages' "Methodik" 3 figure): attention and the fused
    append on G = 16 caches, against the oracle with G = 16."""
    from tests.parity import BOUNDARY_TALLY, check_encode

    wl_name, B, Hkv, Hq, T_cap, lens = case
    wl = kvgen.WORKLOADS[wl_name]
    D, G = wl.head_dim, 16
    dev = torch.device("cuda")
    cache = {}
    for kind in ("k", "v"):
        s, lam = kvgen.plan_params(D, seed=27, kind=kind)
        plan = kvq.Plan(s, lam, G)
        x = torch.from_numpy(kvgen.kv_numpy(wl, kind, (B, Hkv, T_cap - 1, D), seed=27)).to(dev)
        codes = torch.zeros((B, Hkv, T_cap, D // 2), dtype=torch.uint8, device=dev)
        scales = torch.zeros((B, Hkv, T_cap, D // G), dtype=torch.float16, device=dev)
        kvq.encode(plan, x, codes, scales, 0)
        cache[kind] = dict(plan=plan, params=(s, lam), codes=codes, scales=scales)
    k, v = cache["k"], cache["v"]
    q16 = kvgen.q_numpy((B, Hq, D), salt=14)
    q = torch.from_numpy(q16).to(dev)
    lens_np = [T_cap - 1] * B if lens is None else [min(L, T_cap - 1) for L in lens]
    sl = torch.tensor(lens_np, dtype=torch.int32, device=dev)
    out = kvq.attend_decode(k["plan"], v["plan"], q, k["codes"], k["scales"], v["codes"], v["scales"], seq_lens=sl)
    torch.cuda.synchronize()
    assert kvq.poll_device_errors() == 0

    def oracle_out(lens_):
        return oracle.attend_decode_int4(q16, k["codes"].cpu().numpy(), k["scales"].cpu().numpy(),
                                         v["codes"].cpu().numpy(), v["scales"].cpu().numpy(), k["params"],
                                         v["params"], lens_, G)

    check_rel_l2(out.cpu().numpy().astype(np.float64).reshape(-1, D), oracle_out(lens_np).reshape(-1, D),
                 label=f"G16 {case}")
    if lens is None:
        # the fused append at pos = T_cap - 1 with G = 16
        new = {kind: kvgen.kv_numpy(wl, kind, (B, Hkv, D), seed=28) for kind in ("k", "v")}
        pos = T_cap - 1
        out2 = kvq.attend_decode_append(k["plan"], v["plan"], q, torch.from_numpy(new["k"]).to(dev),
                                        torch.from_numpy(new["v"]).to(dev), k["codes"], k["scales"], v["codes"],
                                        v["scales"], pos)
        torch.cuda.synchronize()
        assert kvq.poll_device_errors() == 0
        for kind in ("k", "v"):
            c = cache[kind]
            nb, na = check_encode(new[kind][:, :, None], c["params"][0], c["params"][1], G,
                                  c["codes"][:, :, pos:pos + 1].cpu().numpy(),
                                  c["scales"][:, :, pos:pos + 1].cpu().numpy(), label=f"G16 append {kind}",
                                  count_only=True)
            BOUNDARY_TALLY["bad"] += nb
            BOUNDARY_TALLY["all"] += na
        check_rel_l2(out2.cpu().numpy().astype(np.float64).reshape(-1, D), oracle_out([pos + 1] * B).reshape(-1, D),
                     label=f"G16 append {case}")
