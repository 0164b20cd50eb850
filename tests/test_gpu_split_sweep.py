"""The q sweep of the split/merge configuration: at each step of a drifting
routing trace, a fraction q of the step's cache misses is filled into GPU
slots (the misses with the most routed tokens first) and the rest is computed
on the host (by the oracle here), whose gate-weighted partial sum is merged
by moe_combine_merge.  For every q the merged output must equal the plain
layer.  The per-q GPU-side time (fills + permute + FFN + merge) and host-side
time are written to $MOE_REPORT_DIR/split_sweep.json when that is set.

Dims are reduced (d=1024, I=512; E=256, k=6, T=8, 64 slots as configured) so
that the float64 host share stays tractable; the full-shape split/merge
parity is covered by test_gpu_parity.test_host_partial_merge_and_q_sweep."""
import json
import os
import time

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


def test_q_sweep(moe):
    from expert_offload_serving_b200.layer import MoeLayer, pack_pool
    cfg = synth.LayerConfig("split_sweep", E=256, k=6, d=1024, I=512, fmt="mxfp4", bias_std=0.5,
                            n_slots=64, steps=16, rho=0.9, host_frac=0.3)
    T = 8
    w = synth.make_experts(cfg, range(cfg.E), 0, device="cuda")
    w_cpu = {k: v.cpu() for k, v in w.items()}
    host_pool = pack_pool(cfg.E, cfg.d, cfg.I, cfg.fmt, w_cpu, range(cfg.E), pin=True)
    trace = synth.make_trace(cfg, T, steps=cfg.steps, seed=5)
    deq = {}

    def weights(e):
        if e not in deq:
            deq[e] = tuple(m.astype(np.float32) for m in M.dequant_expert(cfg.fmt, w_cpu, e))
        return deq[e]

    report = []
    for q in [i / 10 for i in range(11)]:
        layer = MoeLayer(cfg.E, cfg.d, cfg.I, cfg.fmt, cfg.k, T, host_pool=host_pool, n_slots=cfg.n_slots)
        lru = L.LRUCache(cfg.n_slots, cfg.E)
        gpu_ms = host_ms = 0.0
        n_fill = n_host = 0
        for t, (logits, x) in enumerate(trace):
            layer.route(logits.cuda())
            idx = layer.idx[:T].cpu().numpy()
            U = sorted(set(idx.ravel().tolist()))
            tok = np.bincount(idx.ravel(), minlength=cfg.E)
            misses = [e for e in U if not lru.resident(e)]
            filled, host = L.split_misses(misses, tok, q)
            gpu_set = [e for e in U if e not in host]
            ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
            ev[0].record()
            fills = layer.prepare(t, gpu_set, protect=U)
            assert fills == lru.step(t, gpu_set, protect=U)[1]
            layer.permute(T)
            layer.ffn(x.cuda())
            ev[1].record()                      # GPU share up to the merge point
            h0 = time.perf_counter()
            hp = M.moe_layer(x.double().numpy(), logits.numpy(), cfg.k, weights, experts=host)["out"]
            host_ms += (time.perf_counter() - h0) * 1e3
            hp_dev = torch.from_numpy(hp.astype(np.float32)).cuda()
            ev[2].record()
            layer.combine(T, host_partial=hp_dev)
            ev[3].record()
            out = layer.out[:T].cpu().numpy()
            gpu_ms += ev[0].elapsed_time(ev[1]) + ev[2].elapsed_time(ev[3])
            ref = M.moe_layer(x.double().numpy(), logits.numpy(), cfg.k, weights)["out"]
            check_tol(out, ref)
            check_tol(out, ref, 1e-4, 1e-5)
            n_fill += len(fills)
            n_host += len(host)
        moe.moe_check_status(layer.status)
        steps = len(trace)
        report.append({"q": q, "gpu_ms_per_step": round(gpu_ms / steps, 4),
                       "host_ms_per_step": round(host_ms / steps, 3),
                       "fills_per_step": round(n_fill / steps, 2), "host_experts_per_step": round(n_host / steps, 2)})
        layer.cache.close()
    # more filling means fewer host experts
    assert report[0]["host_experts_per_step"] >= report[-1]["host_experts_per_step"]
    assert report[-1]["host_experts_per_step"] == 0
    out_dir = os.environ.get("MOE_REPORT_DIR")
    if out_dir:
        os.makedirs(out_dir, exist_ok=True)
        with open(os.path.join(out_dir, "split_sweep.json"), "w") as f:
            json.dump({"config": "E=256 k=6 d=1024 I=512 MXFP4 T=8, 64 slots, 16-step AR(1) trace; "
                                 "host share computed by the float64 oracle", "sweep": report}, f, indent=1)


@pytest.mark.parametrize("q", [0.0, 0.5, 1.0, None])
def test_split_step_host_kernel_concurrent(moe, q):
    """MoeLayer.split_step: the step's misses split by q (None: q* from given
    bandwidths), the GPU share filled on the side stream while the host share
    runs in moe_host_expert_ffn on CPU threads, merged by the combine.  Every
    step's split and fills equal the oracle's, and its output the oracle
    layer's."""
    from expert_offload_serving_b200.layer import MoeLayer, pack_pool
    # 32 slots: a step of T = 4 tokens can need 24 (q = 1 fills every miss)
    cfg = synth.LayerConfig("split_step", E=64, k=6, d=512, I=256, fmt="mxfp4", bias_std=0.5, n_slots=32,
                            rho=0.9)
    T = 4
    bw = (50.0, 120.0)
    w = synth.make_experts(cfg, range(cfg.E), 0, device="cuda")
    w_cpu = {k: v.cpu() for k, v in w.items()}
    host_pool = pack_pool(cfg.E, cfg.d, cfg.I, cfg.fmt, w_cpu, range(cfg.E), pin=True)
    layer = MoeLayer(cfg.E, cfg.d, cfg.I, cfg.fmt, cfg.k, T, host_pool=host_pool, n_slots=cfg.n_slots)
    lru = L.LRUCache(cfg.n_slots, cfg.E)
    deq = {}

    def weights(e):
        if e not in deq:
            deq[e] = M.dequant_expert(cfg.fmt, w_cpu, e)
        return deq[e]
    n_host = 0
    for t, (logits, x) in enumerate(synth.make_trace(cfg, T, steps=20, seed=9)):
        res = layer.split_step(t, logits.cuda(), x.cuda(), q=q, bw=bw, threads=4)
        idx, _ = M.route_topk(logits.numpy(), cfg.k)
        U = sorted(set(idx.ravel().tolist()))
        tok = np.bincount(idx.ravel(), minlength=cfg.E)
        misses = [e for e in U if not lru.resident(e)]
        qq = q if q is not None else (L.q_star(len(misses), *bw) / len(misses) if misses else 0.0)
        filled, host = L.split_misses(misses, tok, qq)
        assert (res["filled"], res["host"]) == (filled, host), f"step {t}"
        gpu_set = sorted(set(U) - set(host))
        assert res["fills"] == lru.step(t, gpu_set, protect=U)[1], f"step {t}"
        out = layer.out[:T].cpu().numpy()
        ref = M.moe_layer(x.double().numpy(), logits.numpy(), cfg.k, weights)["out"]
        check_tol(out, ref, 1e-4, 1e-5)
        n_host += len(host)
    moe.moe_check_status(layer.status)
    assert layer.slot.cpu().tolist() == lru.slot_of_expert
    if q != 1.0:
        assert n_host > 0
