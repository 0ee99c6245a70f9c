"""Int4KVCache (the torch-level cache over the C ABI) on the GPU: a prefill by update(),
decode steps by step() (the fused append), attend() and dequantize(), each against the
oracle on the cache's own packed codes and against the plain entry points."""
import numpy as np
import pytest

import kvgen
import oracle
from tests.parity import check_rel_l2

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("wl_name,B,Hkv,Hq,prefill,steps", [("qwen", 2, 2, 12, 200, 3), ("gemma", 1, 1, 4, 130, 2)])
def test_cache_prefill_steps_attend(wl_name, B, Hkv, Hq, prefill, steps):
    import rotated_int4_kv_b200 as kvq

    wl = kvgen.WORKLOADS[wl_name]
    D, L = wl.head_dim, 2
    kp = [kvgen.plan_params(D, seed=41, layer=l, kind="k") for l in range(L)]
    vp = [kvgen.plan_params(D, seed=41, layer=l, kind="v") for l in range(L)]
    cache = kvq.Int4KVCache(L, B, Hkv, D, prefill + steps + 1, kp, vp)
    assert cache.capacity % 2 == 0 and cache.capacity >= prefill + steps + 1
    dev = torch.device("cuda")
    T = prefill + steps
    for layer in range(L):
        xk = kvgen.kv_numpy(wl, "k", (B, Hkv, T, D), seed=41, layer=layer)
        xv = kvgen.kv_numpy(wl, "v", (B, Hkv, T, D), seed=41, layer=layer)
        cache.update(layer, torch.from_numpy(np.ascontiguousarray(xk[:, :, :prefill])).to(dev),
                     torch.from_numpy(np.ascontiguousarray(xv[:, :, :prefill])).to(dev))
        assert cache.seq_length(layer) == prefill
        for t in range(steps):
            q16 = kvgen.q_numpy((B, Hq, D), salt=100 + t, layer=layer)
            q = torch.from_numpy(q16).to(dev)
            pos = prefill + t
            o = cache.step(layer, q, torch.from_numpy(np.ascontiguousarray(xk[:, :, pos])).to(dev),
                           torch.from_numpy(np.ascontiguousarray(xv[:, :, pos])).to(dev))
            assert cache.seq_length(layer) == pos + 1
            # attend() over the same cache gives the same output (no further append)
            o2 = cache.attend(layer, q)
            torch.cuda.synchronize()
            assert kvq.poll_device_errors() == 0
            check_rel_l2(o.cpu().numpy().astype(np.float64).reshape(-1, D),
                         o2.cpu().numpy().astype(np.float64).reshape(-1, D), tol=1e-3, label="step vs attend")
            kc, ks = cache.k_codes[layer].cpu().numpy(), cache.k_scales[layer].cpu().numpy()
            vc, vs = cache.v_codes[layer].cpu().numpy(), cache.v_scales[layer].cpu().numpy()
            ref = oracle.attend_decode_int4(q16, kc, ks, vc, vs, kp[layer], vp[layer], [pos + 1] * B, 32)
            check_rel_l2(o.cpu().numpy().astype(np.float64).reshape(-1, D), ref.reshape(-1, D),
                         label=f"{wl_name} layer {layer} step {t}")
        # dequantize() = the oracle's decode of the cache's own codes
        k_hat, v_hat = cache.dequantize(layer)
        torch.cuda.synchronize()
        assert tuple(k_hat.shape) == (B, Hkv, T, D)
        ok = oracle.decode(cache.k_codes[layer].cpu().numpy()[:, :, :T], cache.k_scales[layer].cpu().numpy()[:, :, :T],
                           kp[layer][0], kp[layer][1], 32)
        check_rel_l2(k_hat.cpu().numpy().astype(np.float64).reshape(-1, D), ok.reshape(-1, D), label="dequantize K")
    with pytest.raises(ValueError, match="capacity"):
        for _ in range(cache.capacity):
            cache.update(0, torch.zeros((B, Hkv, 1, D), dtype=torch.float16, device=dev),
                         torch.zeros((B, Hkv, 1, D), dtype=torch.float16, device=dev))
    cache.reset()
    assert cache.seq_length(0) == 0
