"""GPU parity of the SRHT plans (R = H diag(s) / sqrt(D)) on every entry point, against
the oracle's SRHT: encode on both paths (tensor cores, Walsh-Hadamard butterflies),
decode, decode attention (D = 128 and 256, GQA, ragged lengths), the fused append and
the cache wrapper. The acceptance rules are those of the SRFT tests."""
import numpy as np
import pytest

import kvgen
import oracle
from tests.parity import BOUNDARY_TALLY, check_encode, check_rel_l2

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu
XF = "srht"


@pytest.fixture(scope="module")
def kvq():
    import rotated_int4_kv_b200 as k
    return k


def _plan(kvq, D, kind, layer=0, G=32, seed=61):
    s, lam = kvgen.plan_params(D, seed=seed, layer=layer, kind=kind)
    return kvq.Plan(s, lam, G, XF), (s, lam)


@pytest.mark.parametrize("path", ["tensor", "fft"])
@pytest.mark.parametrize("wl_name,B,H,n,G", [("qwen", 2, 2, 130, 32), ("gemma", 1, 1, 300, 32), ("toy", 1, 1, 77, 16),
                                             ("gemma", 2, 1, 65, 16)])
def test_srht_encode_decode(kvq, path, wl_name, B, H, n, G):
    wl = kvgen.WORKLOADS[wl_name]
    D = wl.head_dim
    plan, (s, lam) = _plan(kvq, D, "k", G=G)
    x16 = kvgen.kv_numpy(wl, "k", (B, H, n, D), seed=61)
    T_cap, pos = n + 6, 3
    codes = torch.full((B, H, T_cap, D // 2), 0xA5, dtype=torch.uint8, device="cuda")
    scales = torch.full((B, H, T_cap, D // G), 7.0, dtype=torch.float16, device="cuda")
    kvq.set_encode_path(path)
    try:
        kvq.encode(plan, torch.from_numpy(x16).cuda(), codes, scales, pos)
    finally:
        kvq.set_encode_path("auto")
    torch.cuda.synchronize()
    assert kvq.poll_device_errors() == 0
    c, sc = codes.cpu().numpy(), scales.cpu().numpy()
    nb, na = check_encode(x16, s, lam, G, c[:, :, pos:pos + n], sc[:, :, pos:pos + n], label=f"{wl_name} {path}",
                          count_only=True, transform=XF)
    BOUNDARY_TALLY["bad"] += nb
    BOUNDARY_TALLY["all"] += na
    assert np.all(c[:, :, :pos] == 0xA5) and np.all(c[:, :, pos + n:] == 0xA5)
    # decode of the GPU's own codes against the oracle's decode of them
    out = kvq.decode(plan, codes, scales, pos, n)
    torch.cuda.synchronize()
    ref = oracle.decode(c[:, :, pos:pos + n], sc[:, :, pos:pos + n], s, lam, G, XF)
    check_rel_l2(out.cpu().numpy().astype(np.float64).reshape(-1, D), ref.reshape(-1, D), label="decode")


def _srht_cache(kvq, wl, B, Hkv, T_cap, T_fill, layer=0):
    D = wl.head_dim
    out = {}
    for kind in ("k", "v"):
        plan, params = _plan(kvq, D, kind, layer=layer)
        x = torch.from_numpy(kvgen.kv_numpy(wl, kind, (B, Hkv, T_fill, D), seed=62, layer=layer)).cuda()
        codes = torch.zeros((B, Hkv, T_cap, D // 2), dtype=torch.uint8, device="cuda")
        scales = torch.zeros((B, Hkv, T_cap, D // 32), dtype=torch.float16, device="cuda")
        if T_fill:
            kvq.encode(plan, x, codes, scales, 0)
        out[kind] = dict(plan=plan, params=params, codes=codes, scales=scales)
    return out


def _oracle(q16, cache, lens):
    k, v = cache["k"], cache["v"]
    return oracle.attend_decode_int4(q16, k["codes"].cpu().numpy(), k["scales"].cpu().numpy(), v["codes"].cpu().numpy(),
                                     v["scales"].cpu().numpy(), k["params"], v["params"], lens, 32, transform=XF)


@pytest.mark.parametrize("wl_name,B,Hkv,Hq,T_cap,lens", [("qwen", 1, 2, 12, 1024, None), ("qwen", 2, 2, 12, 300, [300, 41]),
                                                          ("longctx", 1, 1, 16, 200, None),
                                                          ("gemma", 1, 1, 4, 2048, None),
                                                          ("gemma", 2, 2, 6, 334, [333, 17])])
def test_srht_attention(kvq, wl_name, B, Hkv, Hq, T_cap, lens):
    wl = kvgen.WORKLOADS[wl_name]
    D = wl.head_dim
    cache = _srht_cache(kvq, wl, B, Hkv, T_cap, T_cap)
    q16 = kvgen.q_numpy((B, Hq, D), salt=12)
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
    ref = _oracle(q16, cache, lens)
    check_rel_l2(out.cpu().numpy().astype(np.float64).reshape(-1, D), ref.reshape(-1, D), label=f"srht {wl_name}")


@pytest.mark.parametrize("wl_name,B,Hkv,Hq,T_cap,pos", [("qwen", 1, 2, 12, 516, 514), ("gemma", 1, 1, 4, 258, 257),
                                                         ("qwen", 1, 2, 12, 64, 0)])
def test_srht_fused_append(kvq, wl_name, B, Hkv, Hq, T_cap, pos):
    wl = kvgen.WORKLOADS[wl_name]
    D = wl.head_dim
    cache = _srht_cache(kvq, wl, B, Hkv, T_cap, pos)
    new = {kind: kvgen.kv_numpy(wl, kind, (B, Hkv, D), seed=63) for kind in ("k", "v")}
    q16 = kvgen.q_numpy((B, Hq, D), salt=13)
    k, v = cache["k"], cache["v"]
    out = kvq.attend_decode_append(k["plan"], v["plan"], torch.from_numpy(q16).cuda(),
                                   torch.from_numpy(new["k"]).cuda(), torch.from_numpy(new["v"]).cuda(),
                                   k["codes"], k["scales"], v["codes"], v["scales"], pos)
    torch.cuda.synchronize()
    assert kvq.poll_device_errors() == 0
    for kind in ("k", "v"):
        c = cache[kind]
        nb, na = check_encode(new[kind][:, :, None], c["params"][0], c["params"][1], 32,
                              c["codes"][:, :, pos:pos + 1].cpu().numpy(), c["scales"][:, :, pos:pos + 1].cpu().numpy(),
                              label=f"append {kind}", count_only=True, transform=XF)
        BOUNDARY_TALLY["bad"] += nb
        BOUNDARY_TALLY["all"] += na
    ref = _oracle(q16, cache, [pos + 1] * B)
    check_rel_l2(out.cpu().numpy().astype(np.float64).reshape(-1, D), ref.reshape(-1, D), label=f"append {wl_name}")


def test_srht_and_srft_plans_do_not_mix(kvq):
    D = 128
    pk, _ = _plan(kvq, D, "k")
    s, lam = kvgen.plan_params(D, kind="v")
    pv = kvq.Plan(s, lam)  # SRFT
    assert pk.transform == "srht" and pv.transform == "srft"
    q = torch.zeros((1, 4, D), dtype=torch.float16, device="cuda")
    codes = torch.zeros((1, 1, 64, D // 2), dtype=torch.uint8, device="cuda")
    scales = torch.zeros((1, 1, 64, D // 32), dtype=torch.float16, device="cuda")
    with pytest.raises(kvq.KvqError, match="INVALID_ARG"):
        kvq.attend_decode(pk, pv, q, codes, scales, codes, scales, T_len=64)


def test_srht_boundary_fraction_over_all_cases():
    """The 1e-5 bound on boundary mismatches, over every element encoded in the session."""
    from tests.parity import MAX_BOUNDARY_FRAC

    if BOUNDARY_TALLY["all"] == 0:
        pytest.skip("runs after the encode cases")
    assert BOUNDARY_TALLY["bad"] <= MAX_BOUNDARY_FRAC * BOUNDARY_TALLY["all"], BOUNDARY_TALLY
