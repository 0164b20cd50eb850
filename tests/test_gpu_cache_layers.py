"""One GPU expert cache shared by several layers (the global LRU over
(layer, expert) keys) and its elastic resize, on the GPU: every layer step's
fills equal the oracle LRU's, every output equals the oracle layer's, and
after shrinking and growing the cache the device slot tables and every
slot's bytes match the oracle's residency and the host blobs."""
import numpy as np
import pytest
import torch

import synth
from oracle import lru as L
from oracle import moe as M
from tests.gpu_util import check_tol, load_moe, require_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def moe():
    require_gpu()
    return load_moe()


def test_shared_cache_layers_with_resize(moe):
    from expert_offload_serving_b200.layer import ExpertCache, MoeLayer, pack_pool
    n_layers, T, steps = 3, 2, 30
    cfg = synth.LayerConfig("layers", E=32, k=4, d=512, I=256, fmt="mxfp4", bias_std=0.5, rho=0.9)
    s = moe.shape(cfg.E, cfg.d, cfg.I, cfg.fmt)
    w_cpu, pools = [], []
    for l in range(n_layers):
        w = synth.make_experts(cfg, range(cfg.E), seed=100 + l, device="cuda")
        w_cpu.append({k: v.cpu() for k, v in w.items()})
        pools.append(pack_pool(cfg.E, cfg.d, cfg.I, cfg.fmt, w_cpu[l], range(cfg.E), pin=True))
    cache = ExpertCache(s, 20, pools)
    layers = [MoeLayer(cfg.E, cfg.d, cfg.I, cfg.fmt, cfg.k, T, cache=cache, layer_id=l) for l in range(n_layers)]
    traces = [synth.make_trace(cfg, T, steps=steps, seed=200 + l) for l in range(n_layers)]
    ref = L.LRUCache(20, n_layers * cfg.E)
    deq = {}

    def weights(l):
        def w(e):
            if (l, e) not in deq:
                deq[(l, e)] = M.dequant_expert(cfg.fmt, w_cpu[l], e)
            return deq[(l, e)]
        return w
    resizes = {10: 12, 20: 28}
    outs = []
    for t in range(steps):
        if t in resizes:
            # the grow moves into a pool the caller allocated
            pool = torch.empty((resizes[t], cache.B),
                               dtype=torch.uint8, device="cuda") if t == 20 else None
            assert cache.resize(resizes[t], new_pool=pool) == ref.resize(resizes[t])
            for l in range(n_layers):        # the tables were rewritten on the stream
                assert layers[l].slot.cpu().tolist() == ref.slot_of_expert[l * cfg.E:(l + 1) * cfg.E]
        for l in range(n_layers):
            logits, x = traces[l][t]
            idx, _ = M.route_topk(logits.numpy(), cfg.k)
            U = sorted(set(idx.ravel().tolist()))
            clock = t * n_layers + l
            fills = layers[l].prepare(clock, U, protect=U)
            _, ref_fills = ref.step(clock, [l * cfg.E + e for e in U])
            assert fills == [(key - l * cfg.E, slot, old) for key, slot, old in ref_fills], (t, l)
            outs.append((l, t, layers[l].forward(logits.cuda(), x.cuda()).clone()))
    torch.cuda.synchronize()
    for l in range(n_layers):
        moe.moe_check_status(layers[l].status)
        assert layers[l].slot.cpu().tolist() == ref.slot_of_expert[l * cfg.E:(l + 1) * cfg.E]
    for slot, key in enumerate(ref.expert_of_slot):
        if key >= 0:
            l, e = divmod(key, cfg.E)
            assert torch.equal(cache.pool[slot].cpu(), pools[l][e]), (slot, key)
    for l, t, out in outs:
        logits, x = traces[l][t]
        r = M.moe_layer(x.double().numpy(), logits.numpy(), cfg.k, weights(l))["out"]
        check_tol(out.cpu().numpy(), r, 1e-4, 1e-5)
