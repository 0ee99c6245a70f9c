"""Multi-rank host logic of bench.py on CPU with the gloo backend (world size 2):
the max-over-ranks reduction of timings and the weak-scaling throughput, and
the reference arm's rank-0-only behaviour."""
import json
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


WORKER = r"""
import os, sys, json, datetime
sys.path.insert(0, sys.argv[1])
import torch.distributed as dist
import bench
dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
r = dist.get_rank(); w = dist.get_world_size()
local = [10.0 + r, 3.0 * (2 - r), 1.5]
mx = bench.max_over_ranks(local, dist, "cpu")
val = bench.job_throughput(w, 1000, mx[0], 10)
print(json.dumps({"rank": r, "max": mx, "value": val}))
dist.barrier()
dist.destroy_process_group()
"""


def _launch(n, code_or_args, extra_env=None, timeout=120):
    port = _free_port()
    procs = []
    for r in range(n):
        env = dict(os.environ, RANK=str(r), LOCAL_RANK=str(r), WORLD_SIZE=str(n), MASTER_ADDR="127.0.0.1",
                   MASTER_PORT=str(port))
        env.update(extra_env or {})
        procs.append(subprocess.Popen([sys.executable] + code_or_args, env=env, stdout=subprocess.PIPE,
                                      stderr=subprocess.PIPE, text=True, cwd=ROOT))
    outs = []
    for p in procs:
        o, e = p.communicate(timeout=timeout)
        assert p.returncode == 0, e[-2000:]
        outs.append(o)
    return outs


def test_max_over_ranks_and_weak_scaling_gloo():
    outs = _launch(2, ["-c", WORKER, ROOT])
    res = [json.loads(o.strip().splitlines()[-1]) for o in outs]
    for r in res:
        assert r["max"] == [11.0, 6.0, 1.5]
        # 2 ranks x 1000 units per step, 11 ms for 10 steps -> 2000 / 1.1 ms
        assert abs(r["value"] - 2 * 1000 / 1.1e-3 / 1e6) < 1e-9


@pytest.mark.slow
def test_reference_arm_prints_on_rank0_only():
    outs = _launch(2, ["bench.py", "--impl", "reference", "--steps", "1", "--warmup", "3", "--gpus", "2"],
                   timeout=600)
    lines0 = [l for l in outs[0].splitlines() if l.startswith("{")]
    assert len(lines0) == 1 and json.loads(lines0[0])["impl"] == "reference"
    assert not [l for l in outs[1].splitlines() if l.startswith("{")]


CP_WORKER = r"""
import os, sys, json, datetime
sys.path.insert(0, sys.argv[1])
import numpy as np
import torch
import torch.distributed as dist
from rotated_int4_kv_b200 import gather_partials
dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
r = dist.get_rank(); w = dist.get_world_size()
# one query head, D = 8 values per token; rank r holds tokens [16 r, 16 r + 16) (rank 1's slice is
# empty when EMPTY is set) and forms its partial (m, l, pad, pad, o[D]) in base 2 like the kernels
rng = np.random.default_rng(3)
T, D = 32, 8
s2 = rng.standard_normal(T) * 3.0          # base-2 scaled scores of all tokens
V = rng.standard_normal((T, D))
lo, hi = 16 * r, 16 * r + 16
if os.environ.get("EMPTY") and r == 1:
    hi = lo
part = np.zeros(D + 4)
if hi > lo:
    m = s2[lo:hi].max()
    p = np.exp2(s2[lo:hi] - m)
    part[0], part[1], part[4:] = m, p.sum(), p @ V[lo:hi]
else:
    part[0] = -np.inf
g = gather_partials(torch.from_numpy(part)[None, None], None).numpy()   # [w, 1, 1, D + 4]
parts = g[:, 0, 0]
M = parts[:, 0].max()
wts = np.where(np.isneginf(parts[:, 0]), 0.0, np.exp2(parts[:, 0] - M))
out = (wts @ parts[:, 4:]) / (wts @ parts[:, 1])
keep = slice(0, 16) if os.environ.get("EMPTY") else slice(0, T)
pf = np.exp2(s2[keep] - s2[keep].max())
ref = (pf @ V[keep]) / pf.sum()
print(json.dumps({"rank": r, "order": parts[:, 0].tolist(), "err": float(np.abs(out - ref).max())}))
dist.barrier()
dist.destroy_process_group()
"""


@pytest.mark.parametrize("empty", [False, True])
def test_context_parallel_gather_and_merge_gloo(empty):
    """gather_partials over two gloo ranks returns the partials in rank order, and their
    log-sum-exp merge equals the softmax over the union of the slices (an empty slice,
    m = -inf, drops out)."""
    outs = _launch(2, ["-c", CP_WORKER, ROOT], extra_env={"EMPTY": "1"} if empty else None)
    res = [json.loads(o.strip().splitlines()[-1]) for o in outs]
    for r in res:
        assert r["err"] < 1e-12
        assert r["order"] == res[0]["order"]
