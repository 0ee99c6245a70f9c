"""The attention kernels' less-travelled paths, through the C ABI:

* units whose splits span several thread-block clusters: the cluster partials go
  through the workspace and the last cluster (atomic counter) merges them. The
  split is read back with kvq_attend_split_info and asserted before the launch,
  so each case is known to take that path; outputs are compared with the oracle
  run on the GPU's own packed cache (int4 and int8 codes, D = 128 and 256, ragged
  lengths) or on the fp16 cache (the comparator kernel);
* the bounded-wait failure path: a wait that runs out raises the device error
  flag, the flag is reported once by kvq_poll_device_errors, and the context
  stays usable for the next launch.
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


def _packed_cache(kvq, wl, B, Hkv, T_cap, D, G, bits, seed):
    dev = torch.device("cuda")
    out = {}
    for kind in ("k", "v"):
        s, lam = kvgen.plan_params(D, seed=seed, kind=kind)
        plan = kvq.Plan(s, lam, G, "srft", bits)
        codes = torch.empty((B, Hkv, T_cap, D * bits // 8), dtype=torch.uint8, device=dev)
        scales = torch.empty((B, Hkv, T_cap, D // G), dtype=torch.float16, device=dev)
        x = kvgen.kv_torch(wl, kind, (B, Hkv, T_cap, D), dev, seed=seed)
        kvq.encode(plan, x, codes, scales, 0)
        del x
        out[kind] = (plan, (s, lam), codes, scales)
    return out


MULTI_CLUSTER = [
    # (workload, B, Hkv, Hq, T_cap, seq_lens, G, bits)
    ("longctx", 1, 1, 8, 131072, [130001], 32, 4),
    ("gemma", 1, 1, 4, 65536, None, 32, 4),
    ("longctx", 2, 1, 8, 65536, [65536, 40003], 32, 8),
    ("qwen", 1, 1, 6, 65536, None, 16, 4),
]


@pytest.mark.parametrize("case", MULTI_CLUSTER, ids=[f"{c[0]}-B{c[1]}Hq{c[3]}T{c[4]}G{c[6]}b{c[7]}" for c in MULTI_CLUSTER])
def test_workspace_merge_of_several_clusters(kvq, case):
    name, B, Hkv, Hq, T_cap, lens, G, bits = case
    wl = kvgen.WORKLOADS[name]
    D = wl.head_dim
    S, C, HT = kvq.attend_split_info(B, Hq, Hkv, D, T_cap, G, bits)
    assert S // C > 1, f"split {S} in clusters of {C}: one cluster per unit, the workspace merge would not run"
    cache = _packed_cache(kvq, wl, B, Hkv, T_cap, D, G, bits, seed=77)
    k, v = cache["k"], cache["v"]
    q = kvgen.q_torch((B, Hq, D), torch.device("cuda"), seed=77)
    sl = None if lens is None else torch.tensor(lens, dtype=torch.int32, device="cuda")
    out = kvq.attend_decode(k[0], v[0], q, k[2], k[3], v[2], v[3], seq_lens=sl,
                            T_len=T_cap if sl is None else None)
    torch.cuda.synchronize()
    assert kvq.poll_device_errors() == 0
    lens_np = [T_cap] * B if lens is None else lens
    ref = oracle.attend_decode_int4(q.cpu().numpy(), k[2].cpu().numpy(), k[3].cpu().numpy(), v[2].cpu().numpy(),
                                    v[3].cpu().numpy(), k[1], v[1], lens_np, G, bits=bits)
    check_rel_l2(out.cpu().numpy().astype(np.float64).reshape(-1, D), ref.reshape(-1, D), label=str(case))


def test_workspace_merge_fp16_comparator(kvq):
    wl = kvgen.WORKLOADS["longctx"]
    B, Hkv, Hq, T, D = 1, 1, 8, 65536, 128
    S, C, _ = kvq.attend_split_info(B, Hq, Hkv, D, T, 32, 16)
    assert S // C > 1, f"split {S} in clusters of {C}"
    dev = torch.device("cuda")
    k = kvgen.kv_torch(wl, "k", (B, Hkv, T, D), dev, seed=5)
    v = kvgen.kv_torch(wl, "v", (B, Hkv, T, D), dev, seed=5)
    q = kvgen.q_torch((B, Hq, D), dev, seed=5)
    out = kvq.attend_decode_ref(q, k, v, T_len=T - 3)
    torch.cuda.synchronize()
    assert kvq.poll_device_errors() == 0
    ref = oracle.attend_decode_fp16(q.cpu().numpy(), k.cpu().numpy(), v.cpu().numpy(), [T - 3])
    check_rel_l2(out.cpu().numpy().astype(np.float64).reshape(-1, D), ref.reshape(-1, D), label="fp16")


def test_split_info_matches_single_cluster_latency_shape(kvq):
    # the Qwen-shaped decode at 1K tokens runs one cluster per unit (no workspace merge)
    S, C, HT = kvq.attend_split_info(1, 12, 2, 128, 1024)
    assert HT == 1 and S >= 1 and S % C == 0 and S // C == 1


def test_bounded_wait_runs_out_and_reports(kvq):
    assert kvq.poll_device_errors() == 0
    kvq.debug_wait_timeout(2000)  # 2 ms budget on a barrier that never completes
    assert kvq.poll_device_errors() == 1  # the load-timeout flag, raised once
    assert kvq.poll_device_errors() == 0  # and cleared by the poll
    # the context is still usable: an ordinary attention call afterwards is correct
    wl = kvgen.WORKLOADS["toy"]
    D, T = 128, 256
    cache = _packed_cache(kvq, wl, 1, 1, T, D, 32, 4, seed=3)
    k, v = cache["k"], cache["v"]
    q = kvgen.q_torch((1, 2, D), torch.device("cuda"), seed=3)
    out = kvq.attend_decode(k[0], v[0], q, k[2], k[3], v[2], v[3], T_len=T)
    torch.cuda.synchronize()
    assert kvq.poll_device_errors() == 0
    ref = oracle.attend_decode_int4(q.cpu().numpy(), k[2].cpu().numpy(), k[3].cpu().numpy(), v[2].cpu().numpy(),
                                    v[3].cpu().numpy(), k[1], v[1], [T])
    check_rel_l2(out.cpu().numpy().astype(np.float64).reshape(-1, D), ref.reshape(-1, D), label="after timeout")
