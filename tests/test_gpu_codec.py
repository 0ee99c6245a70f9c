"""GPU parity of kvq_encode / kvq_decode against the oracle (through the C ABI)."""
import math

import numpy as np
import pytest

import kvgen
import oracle
from tests.parity import BOUNDARY_TALLY, MAX_BOUNDARY_FRAC, check_encode, check_rel_l2

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def kvq():
    import rotated_int4_kv_b200 as k
    return k


def _run_encode(kvq, plan, x16, T_cap, pos, G, fill=0xA5):
    B, H, n, D = x16.shape
    dev = torch.device("cuda")
    x = torch.from_numpy(x16).to(dev)
    codes = torch.full((B, H, T_cap, D // 2), fill, dtype=torch.uint8, device=dev)
    scales = torch.full((B, H, T_cap, D // G), 7.0, dtype=torch.float16, device=dev)
    kvq.encode(plan, x, codes, scales, pos)
    torch.cuda.synchronize()
    assert kvq.poll_device_errors() == 0
    return codes.cpu().numpy(), scales.cpu().numpy()


CASES = [
    # (workload, B, H, n, T_cap, pos, G)
    ("toy", 1, 1, 256, 256, 0, 32),
    ("toy", 1, 1, 256, 300, 37, 32),       # offset into a larger cache
    ("qwen", 1, 2, 1, 64, 17, 32),          # one appended token per head
    ("qwen", 3, 2, 129, 200, 5, 32),        # ragged tail (129 = 128 + 1), several (b, h)
    ("mistral", 2, 8, 77, 80, 3, 32),       # heavy tails, lognormal channel gains
    ("gemma", 1, 1, 300, 512, 100, 32),     # D = 256
    ("gemma", 2, 3, 5, 16, 11, 32),         # D = 256, tiny n, several heads per tile
    ("toy", 2, 2, 100, 128, 0, 16),         # G = 16
    ("gemma", 1, 2, 70, 70, 0, 16),         # D = 256, G = 16
]


_TALLY = BOUNDARY_TALLY  # shared with the fused-append tests
PATHS = ["fft", "tensor", "split"]  # split: the radix-2 split kernel (head_dim 256 SRFT plans)


@pytest.fixture
def encode_path(kvq, request):
    kvq.set_encode_path(request.param)
    yield request.param
    kvq.set_encode_path("auto")


@pytest.mark.parametrize("encode_path", PATHS, indirect=True)
@pytest.mark.parametrize("case", CASES, ids=[f"{c[0]}-B{c[1]}H{c[2]}n{c[3]}cap{c[4]}pos{c[5]}G{c[6]}" for c in CASES])
def test_encode_matches_oracle(kvq, case, encode_path):
    wl_name, B, H, n, T_cap, pos, G = case
    wl = kvgen.WORKLOADS[wl_name]
    D = wl.head_dim
    if encode_path == "split" and D != 256:
        pytest.skip("the radix-2 split kernel serves head_dim 256")
    s, lam = kvgen.plan_params(D, seed=11)
    plan = kvq.Plan(s, lam, group=G)
    x16 = kvgen.kv_numpy(wl, "k", (B, H, n, D), seed=12)
    codes, scales = _run_encode(kvq, plan, x16, T_cap, pos, G)
    nb, na = check_encode(x16, s, lam, G, codes[:, :, pos:pos + n], scales[:, :, pos:pos + n], label=str(case),
                          count_only=True)
    _TALLY["bad"] += nb
    _TALLY["all"] += na
    # rows outside [pos, pos+n) are untouched
    assert np.all(codes[:, :, :pos] == 0xA5) and np.all(codes[:, :, pos + n:] == 0xA5)
    assert np.all(scales[:, :, :pos] == 7.0) and np.all(scales[:, :, pos + n:] == 7.0)



def test_encode_boundary_fraction_over_all_cases():
    if _TALLY["all"] == 0:
        pytest.skip("runs after the encode cases")
    assert _TALLY["bad"] <= MAX_BOUNDARY_FRAC * _TALLY["all"], f"{_TALLY['bad']} boundary mismatches of {_TALLY['all']}"


@pytest.mark.parametrize("D", [128, 256])
def test_encode_closed_forms(kvq, D):
    """s = +1, lambda = 1: x = ones -> only DC; x = (-1)^n -> only Nyquist;
    x = e0 -> codes follow the closed form 1/sqrt(D) vs sqrt(2/D)."""
    s = np.ones(D, np.int8)
    lam = np.ones(D, np.float32)
    plan = kvq.Plan(s, lam)
    n = np.arange(D)
    xs = np.stack([np.ones(D), np.where(n % 2 == 0, 1.0, -1.0), (n == 0).astype(float)]).astype(np.float16)
    codes, scales = _run_encode(kvq, plan, xs[None, None], 3, 0, 32)
    c = oracle.unpack_nibbles(codes[0, 0])
    sc = scales[0, 0].astype(np.float64)
    assert c[0, 0] == 7 and not c[0, 1:].any()
    assert float(sc[0, 0]) == float(np.float16(math.sqrt(D) / 7)) and not sc[0, 1:].any()
    assert c[1, D - 1] == 7 and not c[1, :D - 1].any()
    # e0: every cos row and DC/Nyquist carry the same sign; sin rows are 0
    amax = math.sqrt(2.0 / D)
    scale = float(np.float16(amax / 7))
    exp = np.zeros(D, int)
    exp[1:D - 1:2] = 7 if round(amax / scale) >= 7 else round(amax / scale)
    exp[0] = exp[D - 1] = int(np.rint((1 / math.sqrt(D)) / scale))
    assert np.array_equal(c[2], exp)


@pytest.mark.parametrize("case", CASES[:7], ids=[f"{c[0]}-n{c[3]}" for c in CASES[:7]])
def test_decode_matches_oracle(kvq, case):
    wl_name, B, H, n, T_cap, pos, G = case
    wl = kvgen.WORKLOADS[wl_name]
    D = wl.head_dim
    s, lam = kvgen.plan_params(D, seed=13, kind="v")
    plan = kvq.Plan(s, lam, group=G)
    x16 = kvgen.kv_numpy(wl, "v", (B, H, n, D), seed=14)
    dev = torch.device("cuda")
    codes = torch.zeros((B, H, T_cap, D // 2), dtype=torch.uint8, device=dev)
    scales = torch.zeros((B, H, T_cap, D // G), dtype=torch.float16, device=dev)
    kvq.encode(plan, torch.from_numpy(x16).to(dev), codes, scales, pos)
    out = kvq.decode(plan, codes, scales, pos, n)
    torch.cuda.synchronize()
    assert kvq.poll_device_errors() == 0
    cn, sn = codes.cpu().numpy()[:, :, pos:pos + n], scales.cpu().numpy()[:, :, pos:pos + n]
    ref = oracle.decode(cn, sn, s, lam, G)
    check_rel_l2(out.cpu().numpy().reshape(-1, D), ref.reshape(-1, D), label=str(case))


def test_encode_empty_and_errors(kvq):
    D = 128
    s, lam = kvgen.plan_params(D)
    plan = kvq.Plan(s, lam)
    dev = torch.device("cuda")
    codes = torch.zeros((1, 1, 4, D // 2), dtype=torch.uint8, device=dev)
    scales = torch.zeros((1, 1, 4, D // 32), dtype=torch.float16, device=dev)
    kvq.encode(plan, torch.zeros((1, 1, 0, D), dtype=torch.float16, device=dev), codes, scales, 4)
    with pytest.raises(kvq.KvqError) as e:
        kvq.encode(plan, torch.zeros((1, 1, 2, D), dtype=torch.float16, device=dev), codes, scales, 3)
    assert e.value.status == -4
    torch.cuda.synchronize()
    assert not codes.any()


def test_gemma_full_size_sampled(kvq):
    """Gemma-3-1B-shaped prefill at full size (26 layers x {K,V} x 4096 tokens, D=256)
    in the bench's launch configuration; sampled rows checked against the oracle."""
    wl = kvgen.WORKLOADS["gemma"]
    D, T = wl.head_dim, wl.contexts[0]
    dev = torch.device("cuda")
    rng = np.random.default_rng(0)
    n_bad = n_all = 0
    for layer in (0, 13, 25):
        for kind in ("k", "v"):
            s, lam = kvgen.plan_params(D, layer=layer, kind=kind)
            plan = kvq.Plan(s, lam)
            x = kvgen.kv_torch(wl, kind, (1, 1, T, D), dev, layer=layer)
            codes = torch.empty((1, 1, T, D // 2), dtype=torch.uint8, device=dev)
            scales = torch.empty((1, 1, T, D // 32), dtype=torch.float16, device=dev)
            kvq.encode(plan, x, codes, scales, 0)
            torch.cuda.synchronize()
            idx = np.sort(rng.choice(T, 512, replace=False))
            x16 = x[0, 0].cpu().numpy()[idx]
            nb, na = check_encode(x16, s, lam, 32, codes[0, 0].cpu().numpy()[idx], scales[0, 0].cpu().numpy()[idx],
                                  label=f"gemma L{layer}{kind}", count_only=True)
            n_bad += nb
            n_all += na
    assert n_bad <= MAX_BOUNDARY_FRAC * n_all, f"{n_bad} boundary mismatches of {n_all}"
    assert kvq.poll_device_errors() == 0


def test_encode_batch_matches_single_calls(kvq):
    """Grouped encode of many (plan, x, cache) jobs with different shapes equals the
    single-call encode of each job, bit for bit, and matches the oracle."""
    dev = torch.device("cuda")
    jobs, singles, inputs = [], [], []
    shapes = [("qwen", 1, 2, 1, 8, 3), ("qwen", 2, 2, 200, 256, 40), ("toy", 1, 1, 256, 256, 0),
              ("mistral", 3, 8, 17, 20, 2), ("qwen", 1, 2, 130, 130, 0)] * 14  # 70 jobs: two launches
    for i, (wl_name, B, H, n, T_cap, pos) in enumerate(shapes):
        wl = kvgen.WORKLOADS[wl_name]
        s, lam = kvgen.plan_params(128, layer=i, kind="k")
        plan = kvq.Plan(s, lam)
        x16 = kvgen.kv_numpy(wl, "k", (B, H, n, 128), layer=i)
        x = torch.from_numpy(x16).to(dev)
        mk = lambda: (torch.full((B, H, T_cap, 64), 0x5A, dtype=torch.uint8, device=dev),
                      torch.full((B, H, T_cap, 4), 3.0, dtype=torch.float16, device=dev))
        c1, s1 = mk()
        c2, s2 = mk()
        jobs.append((plan, x, c1, s1, pos))
        singles.append((plan, x, c2, s2, pos))
        inputs.append((x16, s, lam, pos, n))
    kvq.encode_batch(jobs)
    for j in singles:
        kvq.encode(*j)
    torch.cuda.synchronize()
    assert kvq.poll_device_errors() == 0
    n_bad = n_all = 0
    for (_, _, c1, s1, _), (_, _, c2, s2, _), (x16, s, lam, pos, n) in zip(jobs, singles, inputs):
        assert torch.equal(c1, c2) and torch.equal(s1, s2)
        nb, na = check_encode(x16, s, lam, 32, c1.cpu().numpy()[:, :, pos:pos + n], s1.cpu().numpy()[:, :, pos:pos + n],
                              count_only=True)
        n_bad += nb
        n_all += na
    assert n_bad <= MAX_BOUNDARY_FRAC * n_all, f"{n_bad} boundary mismatches of {n_all}"


def test_encode_batch_rejects_mixed_head_dims(kvq):
    dev = torch.device("cuda")
    p1 = kvq.Plan(*kvgen.plan_params(128))
    p2 = kvq.Plan(*kvgen.plan_params(256))
    j1 = (p1, torch.zeros((1, 1, 4, 128), dtype=torch.float16, device=dev),
          torch.zeros((1, 1, 4, 64), dtype=torch.uint8, device=dev),
          torch.zeros((1, 1, 4, 4), dtype=torch.float16, device=dev), 0)
    j2 = (p2, torch.zeros((1, 1, 4, 256), dtype=torch.float16, device=dev),
          torch.zeros((1, 1, 4, 128), dtype=torch.uint8, device=dev),
          torch.zeros((1, 1, 4, 8), dtype=torch.float16, device=dev), 0)
    with pytest.raises(kvq.KvqError) as e:
        kvq.encode_batch([j1, j2])
    assert e.value.status == -1


def test_split_path_refuses_other_plans(kvq):
    dev = torch.device("cuda")
    plan = kvq.Plan(*kvgen.plan_params(128))
    codes = torch.zeros((1, 1, 4, 64), dtype=torch.uint8, device=dev)
    scales = torch.zeros((1, 1, 4, 4), dtype=torch.float16, device=dev)
    kvq.set_encode_path("split")
    try:
        with pytest.raises(kvq.KvqError) as e:
            kvq.encode(plan, torch.zeros((1, 1, 4, 128), dtype=torch.float16, device=dev), codes, scales, 0)
    finally:
        kvq.set_encode_path("auto")
    assert e.value.status == -2
