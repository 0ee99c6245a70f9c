"""kvq_attend_decode_noalloc: the int4 decode attention for callers that cannot
allocate device memory (memory planned up front, code running under stream
capture, hosts whose allocator belongs to someone else). Its scratch is a static
array inside the library, so this checks, through the C ABI, that two calls in a
row give what the workspace-taking kvq_attend_decode gives. Every call passes
real, correctly sized device buffers.

Kept in a file that pytest collects last; it must pass on its own in a fresh
process and after every other test."""
import numpy as np
import pytest

import kvgen
from tests.parity import REL_L2, check_rel_l2

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


def _cache(kvq, wl, B, Hkv, T, seed):
    D = wl.head_dim
    dev = torch.device("cuda")
    out = {}
    for kind in ("k", "v"):
        plan = kvq.Plan(*kvgen.plan_params(D, seed=seed, kind=kind))
        x = kvgen.kv_torch(wl, kind, (B, Hkv, T, D), dev, seed=seed)
        codes = torch.zeros((B, Hkv, T, D // 2), dtype=torch.uint8, device=dev)
        scales = torch.zeros((B, Hkv, T, D // 32), dtype=torch.float16, device=dev)
        kvq.encode(plan, x, codes, scales, 0)
        out[kind] = (plan, codes, scales)
    return out


@pytest.mark.parametrize("name,B,Hkv,Hq,T,lens,multi", [
    ("qwen", 2, 2, 12, 1000, [1000, 377], False),
    ("gemma", 1, 1, 4, 4096, None, False),
    # one unit over 128K tokens: its splits span several clusters, so the cluster
    # partials are written to and merged from the static scratch, not only the counters
    ("longctx", 1, 1, 8, 131072, None, True),
])
def test_noalloc_matches_workspace_entry_point_twice(name, B, Hkv, Hq, T, lens, multi):
    import rotated_int4_kv_b200 as kvq

    wl = kvgen.WORKLOADS[name]
    D = wl.head_dim
    if multi:
        S, C, _ = kvq.attend_split_info(B, Hq, Hkv, D, T)
        assert S // C > 1, f"split {S} in clusters of {C}: the scratch's partial region would not be used"
    c = _cache(kvq, wl, B, Hkv, T, seed=41)
    q = torch.from_numpy(kvgen.q_numpy((B, Hq, D), salt=13)).cuda()
    sl = None if lens is None else torch.tensor(lens, dtype=torch.int32, device="cuda")
    args = (c["k"][0], c["v"][0], q, c["k"][1], c["k"][2], c["v"][1], c["v"][2])
    ref = kvq.attend_decode(*args, seq_lens=sl, T_len=T if sl is None else None).float().cpu().numpy()
    for _ in range(2):  # the static scratch keeps the previous call's contents
        got = kvq.attend_decode_noalloc(*args, seq_lens=sl, T_len=T if sl is None else None)
        torch.cuda.synchronize()
        check_rel_l2(got.float().cpu().numpy().reshape(-1, D), ref.reshape(-1, D), tol=REL_L2, label=name)
    assert kvq.poll_device_errors() == 0
