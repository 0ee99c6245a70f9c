"""kvq_decode on both of its kernels against the oracle (through the C ABI).

The decode is the inverse of the encode of "When Quantization Is Free"
(gist.science/de/paper/2605.05699, "Methodik" 1-2) applied to the dequantised codes:
x_hat = diag(s) Q^T Lambda^-1 (c * scale). Each case encodes with the GPU, then
compares the GPU's decode of the GPU's own cache with the oracle's fp64 decode of the
same codes and scales (relative L2 within 2e-3 per vector and overall).

* every shape of the encode parity cases (ragged tails, offsets into a larger cache,
  several (b, h) per tile, n = 1) on the tensor-core and the register-FFT kernel;
* every plan variant (head_dim 128 / 256, group 32 / 16, int4 / int8, SRFT / SRHT);
* the quantiser's edge rows (scale clamped to 65504, fp16-subnormal scales, zeros);
* the benchmark's decode launch: 52 caches x 4096 vectors of D = 256 in one call,
  every row against the oracle.
"""
import numpy as np
import pytest

import kvgen
import oracle
from tests.parity import check_rel_l2
from tests.test_gpu_codec import CASES
from tests.test_gpu_encode_full_and_edges import edge_vectors

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

PATHS = ["tensor", "fft"]


@pytest.fixture(scope="module")
def kvq():
    import rotated_int4_kv_b200 as k
    return k


@pytest.fixture
def decode_path(kvq, request):
    kvq.set_decode_path(request.param)
    yield request.param
    kvq.set_decode_path("tensor")


def _encode(kvq, plan, x16, T_cap, pos):
    B, H, n, D = x16.shape
    dev = torch.device("cuda")
    codes = torch.zeros((B, H, T_cap, D * plan.bits // 8), dtype=torch.uint8, device=dev)
    scales = torch.zeros((B, H, T_cap, D // plan.group), dtype=torch.float16, device=dev)
    kvq.encode(plan, torch.from_numpy(x16).to(dev), codes, scales, pos)
    return codes, scales


def _decode_and_check(kvq, plan, codes, scales, pos, n, s, lam, G, transform="srft", bits=4, label=""):
    B, H, T_cap, _ = codes.shape
    D = plan.head_dim
    # rows of the output that a wrong row mapping or tail handling would leave untouched
    out = torch.full((B, H, n, D), float("nan"), dtype=torch.float16, device=codes.device)
    kvq.decode(plan, codes, scales, pos, n, out=out)
    torch.cuda.synchronize()
    assert kvq.poll_device_errors() == 0
    got = out.cpu().numpy().astype(np.float64)
    assert np.isfinite(got).all(), f"{label}: non-finite output"
    cn = codes.cpu().numpy()[:, :, pos:pos + n]
    sn = scales.cpu().numpy()[:, :, pos:pos + n]
    ref = oracle.decode(cn, sn, s, lam, G, transform, bits)
    check_rel_l2(got.reshape(-1, D), ref.reshape(-1, D), label=label)
    return got, ref


@pytest.mark.parametrize("decode_path", PATHS, indirect=True)
@pytest.mark.parametrize("case", CASES, ids=[f"{c[0]}-B{c[1]}H{c[2]}n{c[3]}cap{c[4]}pos{c[5]}G{c[6]}" for c in CASES])
def test_decode_shapes(kvq, case, decode_path):
    wl_name, B, H, n, T_cap, pos, G = case
    wl = kvgen.WORKLOADS[wl_name]
    D = wl.head_dim
    s, lam = kvgen.plan_params(D, seed=13, kind="v")
    plan = kvq.Plan(s, lam, group=G)
    x16 = kvgen.kv_numpy(wl, "v", (B, H, n, D), seed=14)
    codes, scales = _encode(kvq, plan, x16, T_cap, pos)
    _decode_and_check(kvq, plan, codes, scales, pos, n, s, lam, G, label=f"{decode_path} {case}")


VARIANTS = [(D, G, bits, xf) for D in (128, 256) for G in (32, 16) for bits in (4, 8) for xf in ("srft", "srht")]


@pytest.mark.parametrize("decode_path", PATHS, indirect=True)
@pytest.mark.parametrize("variant", VARIANTS, ids=[f"D{v[0]}G{v[1]}b{v[2]}{v[3]}" for v in VARIANTS])
def test_decode_plan_variants(kvq, variant, decode_path):
    """Three tiles plus a ragged tail over two (b, h), read at an offset of a larger cache."""
    D, G, bits, xf = variant
    wl = kvgen.WORKLOADS["gemma" if D == 256 else "mistral"]
    s, lam = kvgen.plan_params(D, seed=17, kind="v")
    plan = kvq.Plan(s, lam, group=G, transform=xf, bits=bits)
    B, H, n, T_cap, pos = 1, 2, 200, 230, 19
    x16 = kvgen.kv_numpy(wl, "v", (B, H, n, D), seed=18)
    codes, scales = _encode(kvq, plan, x16, T_cap, pos)
    _decode_and_check(kvq, plan, codes, scales, pos, n, s, lam, G, xf, bits, label=f"{decode_path} {variant}")


@pytest.mark.parametrize("decode_path", PATHS, indirect=True)
@pytest.mark.parametrize("D", [128, 256])
def test_decode_edge_rows(kvq, D, decode_path):
    """Clamped (65504) and fp16-subnormal scales and all-zero rows decode like the oracle;
    zero rows decode to exact zeros."""
    s, lam = kvgen.plan_params(D, seed=31, kind="k")
    plan = kvq.Plan(s, lam)
    x16 = edge_vectors(D, lam, s, n_each=40, seed=D)
    rng = np.random.default_rng(2)
    x16 = x16[rng.permutation(len(x16))]
    n = len(x16)
    codes, scales = _encode(kvq, plan, x16[None, None], n, 0)
    sc = scales.cpu().numpy().astype(np.float64)
    assert (sc == 65504.0).any() and ((sc > 0) & (sc < 2.0 ** -14)).any()
    got, _ = _decode_and_check(kvq, plan, codes, scales, 0, n, s, lam, 32, label=f"{decode_path} edges D{D}")
    zero_rows = ~np.any(x16.astype(np.float64) != 0, axis=-1)
    assert zero_rows.any() and not got[0, 0][zero_rows].any()


@pytest.mark.parametrize("decode_path", PATHS, indirect=True)
def test_decode_benchmark_launch_every_row(kvq, decode_path):
    """The benchmark's decode: the step's 52 packed caches (26 layers x K and V, 4096
    vectors of D = 256 each) decoded in one call with one plan, every row checked."""
    wl = kvgen.WORKLOADS["gemma"]
    L, Hkv, D, T, G = wl.layers, wl.h_kv, wl.head_dim, wl.contexts[0], wl.group
    NJ = 2 * L
    dev = torch.device("cuda")
    s, lam = kvgen.plan_params(D, seed=kvgen.DEFAULT_SEED, layer=0, kind="k")
    plan = kvq.Plan(s, lam, group=G)
    x = torch.empty((NJ, Hkv, T, D), dtype=torch.float16, device=dev)
    for j in range(NJ):
        kvgen.kv_torch(wl, "kv"[j % 2], (1, Hkv, T, D), dev, seed=kvgen.DEFAULT_SEED, layer=j // 2, salt=0,
                       out=x[j:j + 1])
    codes = torch.zeros((NJ, Hkv, T, D // 2), dtype=torch.uint8, device=dev)
    scales = torch.zeros((NJ, Hkv, T, D // G), dtype=torch.float16, device=dev)
    kvq.encode(plan, x, codes, scales, 0)
    _decode_and_check(kvq, plan, codes, scales, 0, T, s, lam, G, label=f"{decode_path} benchmark launch")


def test_decode_paths_agree_closely(kvq):
    """The two kernels on the same cache: within the tensor-core path's own error budget
    (2^-11 relative roundings of the operands and the output)."""
    D, G = 256, 32
    s, lam = kvgen.plan_params(D, seed=41, kind="v")
    plan = kvq.Plan(s, lam, group=G)
    x16 = kvgen.kv_numpy(kvgen.WORKLOADS["gemma"], "v", (2, 2, 333, D), seed=42)
    codes, scales = _encode(kvq, plan, x16, 333, 0)
    outs = {}
    for path in PATHS:
        kvq.set_decode_path(path)
        outs[path] = kvq.decode(plan, codes, scales, 0, 333).cpu().numpy().astype(np.float64)
    kvq.set_decode_path("tensor")
    assert kvq.poll_device_errors() == 0
    check_rel_l2(outs["tensor"].reshape(-1, D), outs["fft"].reshape(-1, D), tol=1e-3, label="tensor vs fft")
