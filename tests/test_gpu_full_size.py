"""Parity at the benchmark's full sizes, in the launch configurations bench.py times,
on sampled outputs the oracle computes one by one:

* the Gemma-3-1B-shaped prefill step's grouped decode attention: 26 jobs (layers) x 1 KV
  head x 4 query heads x 4096 tokens, D = 256, one kvq_attend_decode_batch launch (five
  splits per layer in one cluster, warp pairs over the channel halves); sampled layers
  against the oracle on the GPU's own caches, every layer against its single-job call;
* the long-context sweep's largest case: B = 4, 8 KV heads, 64 query heads, 131072
  tokens, D = 128, int4 and int8 codes; sampled (b, KV head) units against the oracle.
"""
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


def test_gemma_grouped_attention_full_size(kvq):
    wl = kvgen.WORKLOADS["gemma"]
    L, Hkv, Hq, T, D = wl.layers, wl.h_kv, wl.h_q, wl.contexts[0], wl.head_dim
    dev = torch.device("cuda")
    layers = []
    for l in range(L):
        entry = {}
        for kind in ("k", "v"):
            s, lam = kvgen.plan_params(D, layer=l, kind=kind)
            plan = kvq.Plan(s, lam)
            x = kvgen.kv_torch(wl, kind, (1, Hkv, T, D), dev, layer=l)
            codes = torch.empty((1, Hkv, T, D // 2), dtype=torch.uint8, device=dev)
            scales = torch.empty((1, Hkv, T, D // 32), dtype=torch.float16, device=dev)
            kvq.encode(plan, x, codes, scales, 0)
            entry[kind] = (plan, (s, lam), codes, scales)
        entry["q"] = kvgen.q_torch((1, Hq, D), dev, layer=l)
        layers.append(entry)
    jobs = [(e["k"][0], e["v"][0], e["q"], e["k"][2], e["k"][3], e["v"][2], e["v"][3]) for e in layers]
    outs = kvq.attend_decode_batch(jobs, T_len=T)
    singles = [kvq.attend_decode(*j, T_len=T) for j in jobs]
    torch.cuda.synchronize()
    assert kvq.poll_device_errors() == 0
    for l in range(L):
        check_rel_l2(outs[l].cpu().numpy().astype(np.float64).reshape(-1, D),
                     singles[l].cpu().numpy().astype(np.float64).reshape(-1, D), tol=1e-3, label=f"layer {l}")
    for l in (0, 11, 25):
        e = layers[l]
        ref = oracle.attend_decode_int4(e["q"].cpu().numpy(), e["k"][2].cpu().numpy(), e["k"][3].cpu().numpy(),
                                        e["v"][2].cpu().numpy(), e["v"][3].cpu().numpy(), e["k"][1], e["v"][1], [T])
        check_rel_l2(outs[l].cpu().numpy().astype(np.float64).reshape(-1, D), ref.reshape(-1, D),
                     label=f"layer {l} vs oracle")


@pytest.mark.parametrize("bits", [4, 8])
def test_long_context_128k_sampled(kvq, bits):
    wl = kvgen.WORKLOADS["longctx"]
    B, Hkv, Hq, D, G = wl.batch, wl.h_kv, wl.h_q, wl.head_dim, wl.group
    T = max(wl.contexts)
    assert T == 131072
    dev = torch.device("cuda")
    cache = {}
    for kind in ("k", "v"):
        s, lam = kvgen.plan_params(D, kind=kind)
        plan = kvq.Plan(s, lam, G, "srft", bits)
        codes = torch.empty((B, Hkv, T, D * bits // 8), dtype=torch.uint8, device=dev)
        scales = torch.empty((B, Hkv, T, D // G), dtype=torch.float16, device=dev)
        for b in range(B):
            x = kvgen.kv_torch(wl, kind, (1, Hkv, T, D), dev, salt=b)
            kvq.encode(plan, x, codes[b:b + 1], scales[b:b + 1], 0)
            del x
        cache[kind] = (plan, (s, lam), codes, scales)
    q = kvgen.q_torch((B, Hq, D), dev)
    k, v = cache["k"], cache["v"]
    out = kvq.attend_decode(k[0], v[0], q, k[2], k[3], v[2], v[3], T_len=T)
    torch.cuda.synchronize()
    assert kvq.poll_device_errors() == 0
    q16 = q.cpu().numpy()
    grp = Hq // Hkv
    for b, kvh in ((0, 0), (3, 7)):
        sl = slice(kvh, kvh + 1)
        hq = slice(kvh * grp, (kvh + 1) * grp)
        ref = oracle.attend_decode_int4(q16[b:b + 1, hq], k[2][b:b + 1, sl].cpu().numpy(),
                                        k[3][b:b + 1, sl].cpu().numpy(), v[2][b:b + 1, sl].cpu().numpy(),
                                        v[3][b:b + 1, sl].cpu().numpy(), k[1], v[1], [T], G, bits=bits)
        check_rel_l2(out[b:b + 1, hq].cpu().numpy().astype(np.float64).reshape(-1, D), ref.reshape(-1, D),
                     label=f"int{bits} b{b} kv{kvh}")
