"""Sequence-sharded (context-parallel) decode on one GPU: the cache's token range is cut
into slices, each slice's softmax partial comes from kvq_attend_decode_partial (what each
GPU of a context-parallel group computes over its own slice), the stacked partials (what
the all-gather delivers) go to kvq_attend_combine, and the result must equal
kvq_attend_decode over the whole range and the oracle on the same packed cache."""
import numpy as np
import pytest

import kvgen
import oracle
from tests.parity import check_rel_l2

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

CASES = [
    # (workload, B, Hkv, Hq, T, cuts, transform, G)
    ("qwen", 1, 2, 12, 1500, [0, 500, 1000, 1500], "srft", 32),
    ("qwen", 2, 2, 12, 900, [0, 300, 300, 900], "srft", 32),     # an empty slice
    ("longctx", 1, 1, 16, 640, [0, 128, 640], "srft", 32),       # two head tiles
    ("gemma", 1, 1, 4, 2048, [0, 1024, 2048], "srft", 32),       # D = 256
    ("gemma", 1, 2, 6, 700, [0, 350, 700], "srht", 32),
    ("qwen", 1, 2, 12, 600, [0, 200, 600], "srft", 16),
]


@pytest.mark.parametrize("case", CASES, ids=[f"{c[0]}-T{c[4]}-{len(c[5]) - 1}parts-{c[6]}-G{c[7]}" for c in CASES])
def test_partials_combine_to_the_full_attention(case):
    import rotated_int4_kv_b200 as kvq

    wl_name, B, Hkv, Hq, T, cuts, xf, G = case
    wl = kvgen.WORKLOADS[wl_name]
    D = wl.head_dim
    dev = torch.device("cuda")
    cache = {}
    for kind in ("k", "v"):
        s, lam = kvgen.plan_params(D, seed=71, kind=kind)
        plan = kvq.Plan(s, lam, G, xf)
        x = torch.from_numpy(kvgen.kv_numpy(wl, kind, (B, Hkv, T, D), seed=71)).to(dev)
        codes = torch.zeros((B, Hkv, T, D // 2), dtype=torch.uint8, device=dev)
        scales = torch.zeros((B, Hkv, T, D // G), dtype=torch.float16, device=dev)
        kvq.encode(plan, x, codes, scales, 0)
        cache[kind] = dict(plan=plan, params=(s, lam), codes=codes, scales=scales)
    k, v = cache["k"], cache["v"]
    q16 = kvgen.q_numpy((B, Hq, D), salt=15)
    q = torch.from_numpy(q16).to(dev)
    parts = [kvq.attend_decode_partial(k["plan"], v["plan"], q, k["codes"], k["scales"], v["codes"], v["scales"],
                                       a, b) for a, b in zip(cuts[:-1], cuts[1:])]
    out = kvq.attend_combine(v["plan"], torch.stack(parts))
    full = kvq.attend_decode(k["plan"], v["plan"], q, k["codes"], k["scales"], v["codes"], v["scales"], T_len=T)
    torch.cuda.synchronize()
    assert kvq.poll_device_errors() == 0
    for a, b, prt in zip(cuts[:-1], cuts[1:], parts):
        if a == b:  # an empty slice: m = -inf, l = 0, o = 0
            pc = prt.cpu().numpy()
            assert np.all(np.isneginf(pc[..., 0])) and not pc[..., 1].any() and not pc[..., 4:].any()
    got = out.cpu().numpy().astype(np.float64).reshape(-1, D)
    check_rel_l2(got, full.cpu().numpy().astype(np.float64).reshape(-1, D), tol=1e-3, label=f"{case} vs one call")
    ref = oracle.attend_decode_int4(q16, k["codes"].cpu().numpy(), k["scales"].cpu().numpy(), v["codes"].cpu().numpy(),
                                    v["scales"].cpu().numpy(), k["params"], v["params"], [T] * B, G, transform=xf)
    check_rel_l2(got, ref.reshape(-1, D), label=f"{case} vs oracle")


def test_partial_rejects_bad_ranges():
    import rotated_int4_kv_b200 as kvq

    D = 128
    pk = kvq.Plan(*kvgen.plan_params(D, kind="k"))
    pv = kvq.Plan(*kvgen.plan_params(D, kind="v"))
    q = torch.zeros((1, 4, D), dtype=torch.float16, device="cuda")
    codes = torch.zeros((1, 1, 64, D // 2), dtype=torch.uint8, device="cuda")
    scales = torch.zeros((1, 1, 64, D // 32), dtype=torch.float16, device="cuda")
    with pytest.raises(kvq.KvqError, match="ALIGNMENT"):
        kvq.attend_decode_partial(pk, pv, q, codes, scales, codes, scales, 3, 40)
    with pytest.raises(kvq.KvqError, match="CAPACITY"):
        kvq.attend_decode_partial(pk, pv, q, codes, scales, codes, scales, 0, 66)
    with pytest.raises(kvq.KvqError, match="INVALID_ARG"):
        kvq.attend_decode_partial(pk, pv, q, codes, scales, codes, scales, 40, 20)
