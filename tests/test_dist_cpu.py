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
