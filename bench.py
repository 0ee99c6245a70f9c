#!/usr/bin/env python
"""Benchmark of the SRFT-int4 KV-cache hot path on B200.

Workload (default): Gemma-3-1B-shaped prefill -- 26 layers, 1 KV head, 4 query
heads, D=256, batch 1, 4096-token prefix, group 32. One step = encode the full
K and V cache of every layer (52 jobs x 4096 vectors, one grouped kvq_encode_batch
launch) and then one 1-token int4 decode attention per layer (26 jobs in one
grouped kvq_attend_decode_batch launch). Both phases are replayed as CUDA graphs; inputs
rotate over three distinct input sets so that every step reads its 109 MB of
fp16 K/V from HBM, not from the 126 MB L2.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl kvq|reference]

Prints one JSON line (rank 0). Under torchrun each rank runs its own copy of the
workload (weak scaling, no collective on the data path); the timed region is
bracketed by a barrier and device synchronisation and the max over ranks is used.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import kvgen  # noqa: E402

METRIC = "encode Mvec/s (ns/vec) and int4 decode-attn GB/s, % of B200 HBM roofline"
WORKLOAD = "gemma"
N_INPUT_SETS = 3
TRANSFORM = "srft"
BITS = 4


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


# DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum, bytes per launch) of
# the step's kernels from one ncu capture, valid only for the kernel sources it was
# taken on (a digest of the files below); after any change the figure is null
# until a new capture. Summaries and commands: profiles/.
KERNEL_SOURCES = {
    "encode": ["kvq_codec.cu", "kvq_ptx.cuh", "srft_fft.cuh", "kvq_internal.h"],
    "encode_tc": ["kvq_encode_tc.cu", "kvq_ptx.cuh", "kvq_quant.cuh", "kvq_internal.h"],
    "encode_split": ["kvq_encode_tc.cu", "kvq_ptx.cuh", "kvq_quant.cuh", "kvq_internal.h", "srft_fft.cuh"],
    "attend": ["kvq_attend.cu", "kvq_ptx.cuh", "kvq_quant.cuh", "kvq_internal.h"],
    "decode_tc": ["kvq_decode_tc.cu", "kvq_ptx.cuh", "kvq_internal.h"],
}
NCU_TRAFFIC = {
    # kernel -> (source digest at capture time, bytes per launch)
    "encode": ("e66cb71d3607", 112104533),       # register-FFT encode, Gemma step (52 jobs)
    "encode_tc": ("4a3236741c4b", 124388608),    # tensor-core encode, Gemma step (52 jobs)
    "attend": ("a61a78c8ce3e", 32586240),        # grouped int4 attention, Gemma step (26 jobs)
    # tensor-core decode of the step's 52 caches: 30.85 MB read + 51.41 MB written during the launch
    # (the rest of its 109 MB output is written back from L2 after it ends)
    "decode_tc": ("171497c41872", 83871360),
}


def _tensor_peak() -> float:
    """Measured sustained dense bf16 TFLOP/s (the encode runs inside a long step), else 1400."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        if "bf16_tflops_sustained" in d:
            return float(d["bf16_tflops_sustained"])
    return 1400.0


def _source_digest(kind: str) -> str:
    import hashlib

    h = hashlib.sha256()
    for f in KERNEL_SOURCES[kind]:
        with open(os.path.join(ROOT, "rotated_int4_kv_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:12]


def _ncu_traffic(kind: str):
    # captured on the default step (SRFT plans, int4 codes); other variants have no figure
    if TRANSFORM != "srft" or BITS != 4:
        return None
    rec = NCU_TRAFFIC.get(kind)
    return rec[1] if rec is not None and rec[0] == _source_digest(kind) else None


# DRAM traffic per launch of the int4 attention kernel at the attention arms' shapes
# (one ncu capture each, keyed like NCU_TRAFFIC by the kernel sources' digest)
NCU_TRAFFIC_ATTN = {
    # arm -> (source digest at capture time, bytes per launch): int4 attention, one layer
    "mistral_32k": ("a61a78c8ce3e", 606666368),   # B=16, 8/32 heads, 32769 tokens: median read + write of 6 launches
    "longctx_128k": ("a61a78c8ce3e", 605429376),  # B=4, 8/64 heads, 131073 tokens: median read + write of 6 launches
}


def _ncu_traffic_attn(arm: str):
    if TRANSFORM != "srft" or BITS != 4:
        return None
    rec = NCU_TRAFFIC_ATTN.get(arm)
    return rec[1] if rec is not None and rec[0] == _source_digest("attend") else None


def _encode_kernel(path: str, D: int, G: int):
    """(traffic key, kernel name, tensor flops per vector or None) of the encode `path` runs.
    Mirrors the library's dispatch: "auto" is the dense tensor-core product. Tensor work
    per vector: the dense
    product X [W_hi; W_lo]^T is 2 x D x 2D flops (SRHT: the exact W, 2 x D x D); the split
    is two 128-point products (E, O), each hi + lo: 2 x 2 x 2 x 128 x 128 = 2 D^2 at D = 256."""
    xf = int(TRANSFORM == "srht")
    if path == "fft":
        return "encode", f"encode_kernel<{D},{G},{xf},{BITS},64>", None
    if path == "split":
        return "encode_split", f"encode_split_kernel<{G},{BITS},64>", 2 * D * D
    return "encode_tc", f"encode_tc_kernel<{D},{xf},{G},{BITS},64>", (2 if xf else 4) * D * D


def _algo_bytes(D: int, G: int = 32, bits: int = 4):
    vec = 2 * D + D * bits // 8 + 2 * (D // G)   # encode: fp16 in + codes + scales out
    tok = 2 * (D * bits // 8 + 2 * (D // G))     # quantised attention: K and V codes + scales per token x kv head
    return vec, tok


# ---------------------------------------------------------------- multi-rank helpers
def max_over_ranks(values, dist=None, device=None):
    """Element-wise max of per-rank timings (all ranks call it, in the same order)."""
    if dist is None:
        return [float(v) for v in values]
    import torch
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def job_throughput(world: int, units_per_rank: int, ms_total: float, steps: int) -> float:
    """Whole-job units/s (in millions) for weak scaling: every rank processes units_per_rank per step."""
    return world * units_per_rank / (ms_total / steps * 1e-3) / 1e6


# ---------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi clock/throttle sampling in the background (100 ms period)."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None
        self.lines = []
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.idx}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
        if self.thread is not None:
            self.thread.join(timeout=2)

    def summary(self, t0: float, t1: float):
        rows = []
        for ts, line in self.lines:
            if t0 <= ts <= t1:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


# ---------------------------------------------------------------- CPU oracle sample
def oracle_sample(wl, seed: int, layer: int = 0):
    """One layer of the step on the host: K and V encode (2 x T vectors) and the
    1-token int4 decode attention over them, with the fp64 oracle as it stands."""
    import oracle
    D, T, G = wl.head_dim, wl.contexts[0], wl.group
    ks, kl = kvgen.plan_params(D, seed=seed, layer=layer, kind="k")
    vs, vl = kvgen.plan_params(D, seed=seed, layer=layer, kind="v")
    k = kvgen.kv_numpy(wl, "k", (1, wl.h_kv, T, D), seed=seed, layer=layer)
    v = kvgen.kv_numpy(wl, "v", (1, wl.h_kv, T, D), seed=seed, layer=layer)
    q = kvgen.q_numpy((1, wl.h_q, D), seed=seed, layer=layer)
    t0 = time.perf_counter()
    ek = oracle.encode(k, ks, kl, G, TRANSFORM, BITS)
    ev = oracle.encode(v, vs, vl, G, TRANSFORM, BITS)
    oracle.attend_decode_int4(q, ek["packed"], ek["scales"], ev["packed"], ev["scales"], (ks, kl), (vs, vl), [T], G,
                              transform=TRANSFORM, bits=BITS)
    dt = time.perf_counter() - t0
    return 2 * wl.h_kv * T, dt


def _blas_threads():
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        return max([i.get("num_threads", 1) for i in info] or [1])
    except Exception:
        return os.cpu_count() or 1


def cpu_baseline(wl, budget_s: float = 10.0, single_budget_s: float = 5.0):
    """The oracle on the host's cores (BLAS threads = all cores), plus the same sample with
    one BLAS thread."""
    def run(budget):
        vecs, secs, n = 0, 0.0, 0
        while secs < budget or n < 1:
            v, dt = oracle_sample(wl, seed=kvgen.DEFAULT_SEED, layer=n % wl.layers)
            vecs += v
            secs += dt
            n += 1
        return vecs / secs / 1e6, n, secs

    value, n, secs = run(budget_s)
    single = None
    try:
        from threadpoolctl import threadpool_limits
        with threadpool_limits(limits=1):
            v1, n1, s1 = run(single_budget_s)
        single = {"value": v1, "cores": 1, "sample": f"{n1} layers, {s1:.1f} s"}
    except ImportError:
        pass
    return {"value": value, "unit": "Mvec/s", "cores": _blas_threads(), "os_cpu_count": os.cpu_count(),
            "kind": "oracle",
            "sample": f"{n} x one layer of the step (K+V encode of {2 * wl.h_kv * wl.contexts[0]} vectors, D="
                      f"{wl.head_dim}, plus the 1-token int{BITS} attention over {wl.contexts[0]} tokens), "
                      f"{secs:.1f} s of host time",
            "single_thread": single}


# ---------------------------------------------------------------- reference arm
def run_reference(args, rank: int, world: int):
    if rank != 0:
        return 0
    wl = kvgen.WORKLOADS[WORKLOAD]
    for _ in range(args.warmup):
        oracle_sample(wl, seed=kvgen.DEFAULT_SEED)
    vecs, secs = 0, 0.0
    for s in range(args.steps):
        v, dt = oracle_sample(wl, seed=kvgen.DEFAULT_SEED, layer=s % wl.layers)
        vecs += v
        secs += dt
    val = vecs / secs / 1e6
    sample = (f"each step = one layer of the workload on the host (K+V encode of {2 * wl.h_kv * wl.contexts[0]} "
              f"vectors + 1-token int4 attention over {wl.contexts[0]} tokens)")
    line = {"impl": "reference", "metric": METRIC, "value": val, "unit": "Mvec/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * secs / max(1, args.steps),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": dict(_config(wl), encode_path=args.encode_path),
            "step_sample": {"layers_per_timed_step": 1, "layers_per_gpu_step": wl.layers,
                            "note": "each timed step of this arm is one layer of the workload on the host; "
                                    "value (Mvec/s) is per vector and so comparable, ms_per_step is not"},
            "cpu_baseline": {"value": val, "unit": "Mvec/s", "cores": _blas_threads(),
                             "os_cpu_count": os.cpu_count(), "kind": "oracle", "sample": sample},
            "e2e": {"value": val, "unit": "Mvec/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# the plans' rotation: "srft" (the pages' method, the default) or "srht" (--transform)
TRANSFORM = "srft"


def _config(wl):
    return {"workload": "gemma3-1b-prefill: encode K+V of 26 layers x 4096 tokens, then 1-token int4 decode "
                        "attention per layer", "transform": TRANSFORM, "bits": BITS,
            "layers": wl.layers, "kv_heads": wl.h_kv, "q_heads": wl.h_q, "head_dim": wl.head_dim,
            "batch": wl.batch, "prefix": wl.contexts[0], "group": wl.group,
            "l2": f"inputs rotate over {N_INPUT_SETS} distinct input sets (3 x 109 MB) so each step reads HBM"}


# ---------------------------------------------------------------- kvq arm
def run_kvq(args, rank: int, world: int):
    import torch

    import rotated_int4_kv_b200 as kvq

    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=180))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    kvq.set_encode_path(args.encode_path)
    wl = kvgen.WORKLOADS[WORKLOAD]
    L, Hkv, Hq, D, T, G = wl.layers, wl.h_kv, wl.h_q, wl.head_dim, wl.contexts[0], wl.group
    seed = kvgen.DEFAULT_SEED + 1000 * rank
    NJ = 2 * L
    vec_b, tok_b = _algo_bytes(D, G, BITS)

    # plans (per layer and K/V), inputs, caches
    plans = []
    for l in range(L):
        for kind in ("k", "v"):
            s, lam = kvgen.plan_params(D, seed=seed, layer=l, kind=kind)
            plans.append(kvq.Plan(s, lam, group=G, transform=TRANSFORM, bits=BITS))
    X = []
    for i in range(N_INPUT_SETS):
        x = torch.empty((NJ, Hkv, T, D), dtype=torch.float16, device=dev)
        for j in range(NJ):
            kvgen.kv_torch(wl, "kv"[j % 2], (1, Hkv, T, D), dev, seed=seed, layer=j // 2, salt=i, out=x[j:j + 1])
        X.append(x)
    codes = torch.empty((NJ, Hkv, T, D * BITS // 8), dtype=torch.uint8, device=dev)
    scales = torch.empty((NJ, Hkv, T, D // G), dtype=torch.float16, device=dev)
    q = torch.stack([kvgen.q_torch((1, Hq, D), dev, seed=seed, layer=l) for l in range(L)])  # [L, 1, Hq, D]
    out = torch.empty((L, 1, Hq, D), dtype=torch.float16, device=dev)
    ws = kvq.make_workspace(min(L, 32), Hq, Hkv, D, T, dev)

    def jobs_for(i):
        return [(plans[j], X[i][j:j + 1], codes[j:j + 1], scales[j:j + 1], 0) for j in range(NJ)]

    att_jobs = [(plans[2 * l], plans[2 * l + 1], q[l], codes[2 * l:2 * l + 1], scales[2 * l:2 * l + 1],
                 codes[2 * l + 1:2 * l + 2], scales[2 * l + 1:2 * l + 2], out[l]) for l in range(L)]

    def attn_phase():
        # the layers' attentions are independent in this step: one grouped launch
        kvq.attend_decode_batch(att_jobs, T_len=T, workspace=ws)

    # eager run first (one-time kernel attribute setup happens outside capture)
    kvq.encode_batch(jobs_for(0))
    attn_phase()
    torch.cuda.synchronize()
    assert kvq.poll_device_errors() == 0
    if args.ncu:
        # profiling mode: a few eager steps, nothing timed (the launches an ncu capture selects from)
        for s in range(args.steps):
            kvq.encode_batch(jobs_for(s % N_INPUT_SETS))
            attn_phase()
        # then the decode launch of the measurement below (not part of the step), once per
        # step, over the step's 52 packed caches with one plan (same shape and traffic)
        kvq.set_decode_path(args.decode_path)
        dec_out = torch.empty((NJ, Hkv, T, D), dtype=torch.float16, device=dev)
        for s in range(args.steps):
            kvq.decode(plans[0], codes, scales, 0, T, out=dec_out)
        torch.cuda.synchronize()
        assert kvq.poll_device_errors() == 0
        print(json.dumps({"ncu_mode": True, "steps": args.steps, "launches_per_step": 2,
                          "decode_launches": args.steps}), flush=True)
        return 0

    g_enc, g_att = [], []
    cap_stream = torch.cuda.Stream(device=dev)
    for i in range(N_INPUT_SETS):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=cap_stream):
            kvq.encode_batch(jobs_for(i))
        g_enc.append(g)
    ga = torch.cuda.CUDAGraph()
    with torch.cuda.graph(ga, stream=cap_stream):
        attn_phase()
    g_att.append(ga)
    torch.cuda.synchronize()

    def step(i, ev_a=None, ev_b=None):
        if ev_a is not None:
            ev_a.record()
        g_enc[i % N_INPUT_SETS].replay()
        if ev_b is not None:
            ev_b.record()
        g_att[0].replay()

    clk = ClockSampler(local)
    clk.start()
    # soak so the clocks reach their loaded steady state before warm-up and timing
    t_soak = time.time()
    i = 0
    while time.time() - t_soak < 1.5:
        step(i)
        i += 1
        if i % 64 == 0:
            torch.cuda.synchronize()
    for w in range(args.warmup):
        step(w)
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    ev_a = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ev_b = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    wall0 = time.time()
    t_start.record()
    for s in range(args.steps):
        step(s, ev_a[s], ev_b[s])
    t_end.record()
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    wall1 = time.time()
    ms = t_start.elapsed_time(t_end)
    enc_ms = [a.elapsed_time(b) for a, b in zip(ev_a, ev_b)]
    att_ms = [ev_b[s].elapsed_time(ev_a[s + 1]) for s in range(args.steps - 1)] + [ev_b[-1].elapsed_time(t_end)]
    ms, enc_avg, att_avg = max_over_ranks([ms, float(np.mean(enc_ms)), float(np.mean(att_ms))], dist, dev)
    assert kvq.poll_device_errors() == 0

    # ---- end to end through the C ABI with host buffers (pinned), copies in the timed region
    e2e_steps = max(3, min(args.steps, 10))
    x_host = [torch.empty(X[0].shape, dtype=torch.float16, pin_memory=True) for _ in range(2)]
    for hbuf in x_host:
        hbuf.copy_(X[0])
    q_host = q.cpu().pin_memory()
    out_host = torch.empty(out.shape, dtype=torch.float16, pin_memory=True)
    x_dev = X[0]
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record()
    for s in range(e2e_steps):
        x_dev.copy_(x_host[s % 2], non_blocking=True)
        q.copy_(q_host, non_blocking=True)
        kvq.encode_batch(jobs_for(0))
        attn_phase()
        out_host.copy_(out, non_blocking=True)
    e1.record()
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1) / e2e_steps
    h2d = x_dev.numel() * 2 + q.numel() * 2
    d2h = out.numel() * 2

    # ---- decode (the inverse, not part of the step): one launch over 52 packed caches of
    # the step's shape as a batch of 52, one plan for all (the same launch is checked row by
    # row against the oracle). The caches of the three input sets (3 x 30.7 MB) are decoded
    # in turn, so each launch reads codes that 218 MB of other traffic has pushed out of L2;
    # the 109 MB fp16 output streams to HBM.
    kvq.set_decode_path(args.decode_path)
    dec_sets = []
    for i in range(N_INPUT_SETS):
        dc, dsc = torch.empty_like(codes), torch.empty_like(scales)
        kvq.encode(plans[0], X[i], dc, dsc, 0)
        dec_sets.append((dc, dsc))
    dec_out = torch.empty((NJ, Hkv, T, D), dtype=torch.float16, device=dev)

    def dec_all():
        for dc, dsc in dec_sets:
            kvq.decode(plans[0], dc, dsc, 0, T, out=dec_out)

    ms_dec = _graph_time(torch, dec_all, 20, 3) / N_INPUT_SETS
    ms_dec = max_over_ranks([ms_dec], dist, dev)[0]
    del dec_out, dec_sets
    assert kvq.poll_device_errors() == 0

    # ---- the attention half of the metric at bandwidth-bound and latency-bound shapes:
    # int4 against the fp16 comparator on identical shapes (decode_case), each a CUDA
    # graph of back-to-back calls; the big caches (604 MB int4 / 2.15 GB fp16) exceed L2
    attn_arms = None
    arms0 = time.time()
    if not args.skip_attention_arms:
        attn_arms = {}
        for key, wname, T, layers, distinct, variants in (
                ("mistral_32k", "mistral", 32768, 4, 1, False),
                ("longctx_128k", "longctx", 131072, 4, 1, False),
                ("qwen_1k_step", "qwen", 1024, 28, 4, True),
                ("qwen_4k_step", "qwen", 4096, 28, 4, True)):
            case = decode_case(kvq, torch, kvgen.WORKLOADS[wname], T, layers, distinct, args.steps, args.warmup,
                               seed, dev, step_variants=variants)
            for f in ("int4_attn_ms", "fp16_attn_ms"):
                case[f] = max_over_ranks([case[f]], dist, dev)[0]
            case["attn_speedup"] = case["fp16_attn_ms"] / case["int4_attn_ms"]
            case["int4_traffic_bytes_per_launch"] = _ncu_traffic_attn(key)
            attn_arms[key] = case
    arms1 = time.time()
    clk.stop()
    if attn_arms is not None:
        arm_clocks = clk.summary(arms0, arms1)
        attn_arms["clocks"] = {"sm_mhz": arm_clocks["sm_mhz"], "sm_max_mhz": arm_clocks["sm_max_mhz"],
                               "reasons": arm_clocks["reasons"], "samples": arm_clocks["samples"]}

    vec_step = NJ * Hkv * T
    value = job_throughput(world, vec_step, ms, args.steps)
    hbm, peak_kind = _peaks()
    enc_gbs = vec_step * vec_b / (enc_avg * 1e-3) / 1e9
    att_bytes = L * Hkv * T * tok_b
    att_gbs = att_bytes / (att_avg * 1e-3) / 1e9
    clocks = clk.summary(wall0 - 1.0, wall1 + 0.2)
    # roofline of the kernel with the larger share of the step (each phase is one launch)
    src = "measured (MEASURED_PEAKS.json hbm_gbs, burst copy)" if peak_kind == "measured" else "fallback 6.65 TB/s"
    enc_key, enc_kernel, fpv = _encode_kernel(kvq.get_encode_path(), D, G)
    # the tensor-core encode's own work (context for the HBM roofline)
    tensor = None
    if fpv is not None:
        tflops = vec_step * fpv / (enc_avg * 1e-3) / 1e12
        tensor = {"flops_per_vec": fpv, "achieved_TFLOP_s": tflops,
                  "peak_TFLOP_s": _tensor_peak(), "frac": tflops / _tensor_peak(),
                  "peak_source": "measured (MEASURED_PEAKS.json bf16_tflops_sustained; fp16 runs at the bf16 rate)"}
    if enc_avg >= att_avg:
        roof = {"bound": "hbm", "achieved": enc_gbs, "peak": hbm, "unit": "GB/s", "frac": enc_gbs / hbm,
                "traffic": _ncu_traffic(enc_key), "kernel": enc_kernel,
                "share": enc_avg / (enc_avg + att_avg), "peak_source": src}
    else:
        roof = {"bound": "hbm", "achieved": att_gbs, "peak": hbm, "unit": "GB/s", "frac": att_gbs / hbm,
                "traffic": _ncu_traffic("attend"), "kernel": f"attend_kernel<{D},{'int4' if BITS == 4 else 'int8'},{G}>",
                "share": att_avg / (enc_avg + att_avg), "peak_source": src}
    res = None
    if rank == 0:
        cpu = cpu_baseline(wl) if world == 1 else None
        res = {
            "metric": METRIC, "value": value, "unit": "Mvec/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f32", "data": "synthetic", "config": dict(_config(wl), encode_path=args.encode_path),
            "encode": {"kernel_us": 1e3 * enc_avg, "ns_per_vec": 1e6 * enc_avg / vec_step,
                       "Mvec_s": vec_step / (enc_avg * 1e-3) / 1e6, "GB_s": enc_gbs,
                       "frac_hbm": enc_gbs / hbm, "frac_hbm_8TBs_nominal": enc_gbs / 8000.0,
                       "bytes_per_vec": vec_b},
            "attention": {"phase_us": 1e3 * att_avg, "us_per_layer": 1e3 * att_avg / L,
                          "tokens_heads_per_s": L * Hkv * T / (att_avg * 1e-3), "GB_s": att_gbs,
                          "frac_hbm": att_gbs / hbm, "bytes_per_token_head": tok_b},
            "roofline": roof,
            "kernels": {  # both launches of the step, each timed with CUDA events on its stream
                "encode": {"kernel": enc_kernel, "us": 1e3 * enc_avg, "traffic": _ncu_traffic(enc_key),
                           "achieved_GB_s": enc_gbs, "frac": enc_gbs / hbm, "share": enc_avg / (enc_avg + att_avg),
                           "tensor": tensor},
                "attention": {"kernel": f"attend_kernel<{D},{'int4' if BITS == 4 else 'int8'},{G}>", "us": 1e3 * att_avg, "achieved_GB_s": att_gbs,
                              "frac": att_gbs / hbm, "share": att_avg / (enc_avg + att_avg),
                              "traffic": _ncu_traffic("attend")},
            },
            "decode": {"kernel_us": 1e3 * ms_dec, "ns_per_vec": 1e6 * ms_dec / vec_step,
                       "GB_s": vec_step * vec_b / (ms_dec * 1e-3) / 1e9,
                       "frac_hbm": vec_step * vec_b / (ms_dec * 1e-3) / 1e9 / hbm, "bytes_per_vec": vec_b,
                       "kernel": (f"decode_tc_kernel<{D},{BITS},{G}>" if args.decode_path == "tensor"
                                  else f"decode_kernel<{D},{G},{BITS}>"),
                       "path": args.decode_path,
                       "traffic": _ncu_traffic("decode_tc") if args.decode_path == "tensor" else None,
                       "l2": "one launch over 52 caches of the step's shape; three cache sets decoded in turn "
                             "(codes read from HBM)"},
            "attention_arms": attn_arms,
            "cpu_baseline": cpu,
            "e2e": {"value": world * vec_step / (e2e_ms * 1e-3) / 1e6, "unit": "Mvec/s",
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
            "gpu_launches": args.steps * 2,
            "clocks": {"sm_mhz": clocks["sm_mhz"], "sm_max_mhz": clocks["sm_max_mhz"], "reasons": clocks["reasons"],
                       "samples": clocks["samples"]},
        }
    for g in g_enc + g_att:
        g.reset()
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    if res is not None:
        print(json.dumps(res), flush=True)
    return 0


# ---------------------------------------------------------------- other workloads (decode-attention table)
def _graph_time(torch, fn, steps, warmup):
    """Capture fn() (one step) in a CUDA graph and time `steps` replays (ms per step)."""
    fn()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    with torch.cuda.graph(g, stream=s):
        fn()
    for _ in range(warmup):
        g.replay()
    torch.cuda.synchronize()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(steps):
        g.replay()
    b.record()
    torch.cuda.synchronize()
    g.reset()
    return a.elapsed_time(b) / steps


def decode_case(kvq, torch, wl, T, layers, distinct, steps, warmup, seed, dev, batch=None, step_variants=True):
    """One context length of a decode-step workload: int4 against the fp16 comparator.

    Per layer (a CUDA graph of `layers` layers cycling over `distinct` caches): the int4
    step is one fused launch (kvq_attend_decode_append: the new token's K/V encoded at T,
    attention over T + 1); the two-launch int4 step (encode, then attention) beside it;
    the fp16 step is two one-token append copies + the fp16 attention kernel. Attention
    alone is timed for both caches. With step_variants=False only the two attention-alone
    graphs run (bandwidth-bound shapes, where the append is noise)."""
    D, Hkv, Hq, G = wl.head_dim, wl.h_kv, wl.h_q, wl.group
    B = wl.batch if batch is None else batch
    vec_b, tok_b = _algo_bytes(D, G, BITS)
    hbm, _ = _peaks()
    T_cap = T + 2
    plans, caches, k16s, v16s = [], [], [], []
    for l in range(distinct):
        pk = kvq.Plan(*kvgen.plan_params(D, seed=seed, layer=l, kind="k"), transform=TRANSFORM, bits=BITS)
        pv = kvq.Plan(*kvgen.plan_params(D, seed=seed, layer=l, kind="v"), transform=TRANSFORM, bits=BITS)
        plans.append((pk, pv))
        c = {}
        for kind, pl in (("k", pk), ("v", pv)):
            codes = torch.zeros((B, Hkv, T_cap, D * BITS // 8), dtype=torch.uint8, device=dev)
            scales = torch.zeros((B, Hkv, T_cap, D // G), dtype=torch.float16, device=dev)
            x16 = torch.zeros((B, Hkv, T_cap, D), dtype=torch.float16, device=dev)
            for b in range(B):
                kvgen.kv_torch(wl, kind, (1, Hkv, T, D), dev, seed=seed, layer=l, salt=b, out=x16[b:b + 1, :, :T])
                kvq.encode(pl, x16[b:b + 1, :, :T].contiguous(), codes[b:b + 1], scales[b:b + 1], 0)
            c[kind] = (codes, scales)
            (k16s if kind == "k" else v16s).append(x16)
        caches.append(c)
    q = [kvgen.q_torch((B, Hq, D), dev, seed=seed, layer=l) for l in range(distinct)]
    newk = [kvgen.kv_torch(wl, "k", (B, Hkv, 1, D), dev, seed=seed, layer=l, salt=99) for l in range(distinct)]
    newv = [kvgen.kv_torch(wl, "v", (B, Hkv, 1, D), dev, seed=seed, layer=l, salt=98) for l in range(distinct)]
    out = torch.empty((B, Hq, D), dtype=torch.float16, device=dev)
    ws = [kvq.make_workspace(B, Hq, Hkv, D, T_cap, dev) for _ in range(distinct)]

    def step_int4():
        # one launch per layer: the new token's K/V encoded at T and attention over T + 1
        for l in range(layers):
            d = l % distinct
            pk, pv = plans[d]
            kc, ks = caches[d]["k"]
            vc, vs = caches[d]["v"]
            kvq.attend_decode_append(pk, pv, q[d], newk[d], newv[d], kc, ks, vc, vs, T, out=out, workspace=ws[d])

    def step_int4_two_launches():
        for l in range(layers):
            d = l % distinct
            pk, pv = plans[d]
            kc, ks = caches[d]["k"]
            vc, vs = caches[d]["v"]
            kvq.encode_batch([(pk, newk[d], kc, ks, T), (pv, newv[d], vc, vs, T)])
            kvq.attend_decode(pk, pv, q[d], kc, ks, vc, vs, T_len=T + 1, out=out, workspace=ws[d])

    def step_fp16():
        for l in range(layers):
            d = l % distinct
            k16s[d][:, :, T:T + 1].copy_(newk[d])
            v16s[d][:, :, T:T + 1].copy_(newv[d])
            kvq.attend_decode_ref(q[d], k16s[d], v16s[d], T_len=T + 1, out=out, workspace=ws[d])

    def attn_only_int4():
        for l in range(layers):
            d = l % distinct
            pk, pv = plans[d]
            kvq.attend_decode(pk, pv, q[d], *caches[d]["k"], *caches[d]["v"], T_len=T + 1, out=out,
                              workspace=ws[d])

    def attn_only_fp16():
        for l in range(layers):
            d = l % distinct
            kvq.attend_decode_ref(q[d], k16s[d], v16s[d], T_len=T + 1, out=out, workspace=ws[d])

    a4 = _graph_time(torch, attn_only_int4, steps, warmup)
    a16 = _graph_time(torch, attn_only_fp16, steps, warmup)
    tokheads = layers * B * Hkv * (T + 1)
    S, C, _ = kvq.attend_split_info(B, Hq, Hkv, D, T + 1, G, BITS)
    case = {
        "T": T, "batch": B, "kv_heads": Hkv, "q_heads": Hq, "head_dim": D, "layers": layers,
        "distinct_layer_caches": distinct,
        "int4_attn_ms": a4, "fp16_attn_ms": a16, "attn_speedup": a16 / a4,
        "int4_us_per_layer": 1e3 * a4 / layers, "fp16_us_per_layer": 1e3 * a16 / layers,
        "int4_tokens_heads_per_s": tokheads / (a4 * 1e-3),
        "int4_attn_GB_s": tokheads * tok_b / (a4 * 1e-3) / 1e9,
        "int4_frac_hbm": tokheads * tok_b / (a4 * 1e-3) / 1e9 / hbm,
        "fp16_attn_GB_s": tokheads * 4 * D / (a16 * 1e-3) / 1e9,
        "fp16_frac_hbm": tokheads * 4 * D / (a16 * 1e-3) / 1e9 / hbm,
        "bytes_per_token_head": tok_b, "int4_split": {"splits": S, "cluster": C},
        "l2": ("working set > L2 (HBM-bound)" if distinct * B * Hkv * T * tok_b > 126e6
               else "working set fits in L2: latency of an L2-warm decode loop"),
    }
    if step_variants:
        ms4 = _graph_time(torch, step_int4, steps, warmup)
        ms4_2 = _graph_time(torch, step_int4_two_launches, steps, warmup)
        ms16 = _graph_time(torch, step_fp16, steps, warmup)
        case.update({"int4_step_ms": ms4, "int4_step_two_launch_ms": ms4_2, "fp16_step_ms": ms16,
                     "step_speedup": ms16 / ms4, "int4_step_us_per_layer": 1e3 * ms4 / layers,
                     "fp16_step_us_per_layer": 1e3 * ms16 / layers})
    assert kvq.poll_device_errors() == 0
    del caches, k16s, v16s, plans, ws
    torch.cuda.empty_cache()
    return case


def run_decode_workload(args, rank: int, world: int):
    """Decode-step workloads: per layer, append one token of K and V to the cache and run
    one-query decode attention over it, int4 against the fp16 comparator (decode_case).
    Steps are CUDA graphs."""
    import torch

    import rotated_int4_kv_b200 as kvq

    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    wl = kvgen.WORKLOADS[args.workload]
    D, Hkv, Hq, B, G = wl.head_dim, wl.h_kv, wl.h_q, wl.batch, wl.group
    seed = kvgen.DEFAULT_SEED + 1000 * rank
    vec_b, tok_b = _algo_bytes(D, G, BITS)
    contexts = wl.contexts if args.contexts is None else tuple(int(c) for c in args.contexts.split(","))
    layers = wl.layers if args.layers is None else args.layers
    distinct = min(layers, max(1, args.distinct_layers))
    cases = [decode_case(kvq, torch, wl, T, layers, distinct, args.steps, args.warmup, seed, dev) for T in contexts]
    stream_enc = None
    sb = wl.extra.get("stream_batch") if wl.extra else None
    if sb:
        # streaming encode: one token per step for each of sb sequences x Hkv heads x {K, V}
        # (one grouped launch per step; a few MB, so this measures latency, not HBM)
        pk, pv = (kvq.Plan(*kvgen.plan_params(D, seed=seed, layer=0, kind=k), transform=TRANSFORM, bits=BITS)
                  for k in ("k", "v"))
        xk = kvgen.kv_torch(wl, "k", (sb, Hkv, 1, D), dev, seed=seed, layer=0, salt=77)
        xv = kvgen.kv_torch(wl, "v", (sb, Hkv, 1, D), dev, seed=seed, layer=0, salt=78)
        kc = torch.zeros((sb, Hkv, 2, D * BITS // 8), dtype=torch.uint8, device=dev)
        ks = torch.zeros((sb, Hkv, 2, D // G), dtype=torch.float16, device=dev)
        vc, vs = torch.zeros_like(kc), torch.zeros_like(ks)
        nvec = 2 * sb * Hkv
        stream_enc = {"sequences": sb, "vectors_per_step": nvec, "l2": "inputs fit in L2: launch latency"}
        for path in ("tensor", "fft"):
            kvq.set_encode_path(path)
            try:
                ms_e = _graph_time(torch, lambda: kvq.encode_batch([(pk, xk, kc, ks, 0), (pv, xv, vc, vs, 0)]),
                                   args.steps, args.warmup)
            finally:
                kvq.set_encode_path("auto")
            stream_enc[path] = {"us_per_step": ms_e * 1e3, "ns_per_vec": ms_e * 1e6 / nvec,
                                "GB_s": nvec * vec_b / (ms_e * 1e-3) / 1e9}
        assert kvq.poll_device_errors() == 0
    big = cases[-1]
    line = {"metric": METRIC, "value": big["int4_attn_GB_s"], "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": big["int4_step_ms"],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": args.workload, "transform": TRANSFORM, "bits": BITS, "layers": layers, "kv_heads": Hkv,
                       "q_heads": Hq, "head_dim": D,
                       "batch": B, "contexts": list(contexts), "group": G},
            "cases": cases}
    if stream_enc is not None:
        line["streaming_encode"] = stream_enc
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="kvq", choices=["kvq", "reference"])
    ap.add_argument("--workload", default=WORKLOAD, choices=["gemma", "mistral", "qwen", "longctx"],
                    help="gemma (default) = the headline prefill-encode step; the others time decode steps")
    ap.add_argument("--contexts", default=None, help="comma-separated context lengths (decode workloads)")
    ap.add_argument("--layers", type=int, default=None, help="layers per decode step (default: the model's)")
    ap.add_argument("--distinct-layers", type=int, default=4,
                    help="distinct per-layer caches cycled through a decode step (each > L2 for the big shapes)")
    ap.add_argument("--ncu", action="store_true",
                    help="profiling mode: run --steps eager steps without timing, for ncu captures")
    ap.add_argument("--transform", default="srft", choices=["srft", "srht"],
                    help="the plans' rotation: srft (the pages' method) or srht (the Hadamard variant)")
    ap.add_argument("--bits", type=int, default=4, choices=[4, 8],
                    help="code width of the plans: 4 (the pages' int4, default) or 8 (int8 codes)")
    ap.add_argument("--skip-attention-arms", action="store_true",
                    help="default workload: leave out the int4-vs-fp16 attention arms (Mistral 32K, 128K, Qwen step)")
    ap.add_argument("--decode-path", default="tensor", choices=["tensor", "fft"],
                    help="kvq_decode kernel for the decode measurement (not part of the timed step)")
    ap.add_argument("--encode-path", default="auto", choices=["auto", "fft", "tensor", "split"],
                    help="encode kernel of the prefill step: tensor cores where supported (auto), "
                         "the register FFT, the dense tensor-core product, or the radix-2 split "
                         "(head_dim 256 SRFT)")
    args = ap.parse_args(argv)
    global TRANSFORM, BITS
    TRANSFORM = args.transform
    BITS = args.bits
    if args.warmup < 3:
        args.warmup = 3
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if args.impl == "reference":
        return run_reference(args, rank, world)
    if args.workload != WORKLOAD:
        return run_decode_workload(args, rank, world)
    return run_kvq(args, rank, world)


if __name__ == "__main__":
    sys.exit(main())
