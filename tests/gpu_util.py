"""Shared helpers of the GPU parity tests: building layers from the seeded
generators, running the oracle on the same inputs, and the tolerance check."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import synth
from oracle import moe as M

# Layer-output tolerance: max |err| <= 2e-2 * max |ref| and
# mean |err| / mean |ref| <= 5e-3 against the float64 oracle.
MAX_REL = 2e-2
MEAN_REL = 5e-3


def require_gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def load_moe():
    import expert_offload_serving_b200 as moe
    import os
    if not os.path.exists(moe.LIB_PATH):
        from expert_offload_serving_b200 import build
        build.build()
    moe.lib()
    return moe


def check_tol(out, ref, max_rel=MAX_REL, mean_rel=MEAN_REL):
    out = np.asarray(out, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    err = np.abs(out - ref)
    m = float(err.max() / max(np.abs(ref).max(), 1e-30))
    r = float(err.mean() / max(np.abs(ref).mean(), 1e-30))
    assert np.isfinite(out).all(), "non-finite output"
    assert m <= max_rel, f"max err {m:.3e} x max|ref| above {max_rel}"
    assert r <= mean_rel, f"mean rel err {r:.3e} above {mean_rel}"
    return m, r


class Built:
    """A resident layer holding only the experts the routing selects (in
    shuffled slots, so the slot table is exercised), plus its oracle."""

    def __init__(self, cfg, T, seed=0, act="none", logits=None, x=None, experts=None, slot_seed=None,
                 gen_device="cuda"):
        from expert_offload_serving_b200.layer import MoeLayer, pack_pool
        self.cfg, self.T = cfg, T
        if logits is None:
            logits, x = synth.make_routing(cfg, T, seed)
        self.logits, self.x = logits, x
        idx, _ = M.route_topk(logits.numpy(), cfg.k)
        used = sorted(set(idx.ravel().tolist())) if experts is None else list(experts)
        rng = np.random.default_rng(1000 + seed if slot_seed is None else slot_seed)
        order = list(rng.permutation(used))                 # expert stored at slot n = order[n]
        self.used, self.order = used, order
        w = synth.make_experts(cfg, order, seed, device=gen_device)
        self.w_cpu = {k: v.cpu() for k, v in w.items()}
        pool = pack_pool(cfg.E, cfg.d, cfg.I, cfg.fmt, self.w_cpu, order, pin=False).cuda()
        self.layer = MoeLayer(cfg.E, cfg.d, cfg.I, cfg.fmt, cfg.k, T, device_pool=pool, act=act)
        self.layer.slot.fill_(-1)
        for n, e in enumerate(order):
            self.layer.slot[e] = n
        self.pos = {e: n for n, e in enumerate(order)}
        self._deq = {}
        self.act = act

    def weights(self, e):
        if e not in self._deq:
            self._deq[e] = M.dequant_expert(self.cfg.fmt, self.w_cpu, self.pos[e])
        return self._deq[e]

    def oracle(self, experts=None, tokens=None):
        return M.moe_layer(self.x.double().numpy(), self.logits.numpy(), self.cfg.k, self.weights,
                           experts=experts, tokens=tokens, act=self.act)

    def run(self, host_partial=None):
        out = self.layer.forward(self.logits.cuda(), self.x.cuda(), host_partial=host_partial)
        torch.cuda.synchronize()
        return out


# ---------------------------------------------------------------- pooled oracle
# The float64 oracle costs ~1.3 s per full-size expert (dequantisation), so
# full-size checks split the experts into subsets, run moe_layer on each
# subset in a spawned worker, and add the subset outputs: the layer is the sum
# of its expert subsets (the split invariance the oracle is pinned to).  The
# canonical weights reach the workers as .npy files mapped read-only.

def _np_of(t):
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.bfloat16:
        t = t.view(torch.int16)
    return t.numpy()


def _oracle_subset(args):
    wdir, keys, fmt, pos, x, logits, k, experts, act = args
    from threadpoolctl import threadpool_limits
    w = {key: np.load(f"{wdir}/{key}.npy", mmap_mode="r") for key in keys}
    with threadpool_limits(1):
        return M.moe_layer(x, logits, k, lambda e: M.dequant_expert(fmt, w, pos[e]), experts=experts,
                           act=act)["out"]


def pooled_oracle(x, logits, k, fmt, w_cpu, pos, experts, act="none", workers=None):
    """moe_layer(x, logits, k, ...)["out"] over `experts`, whose canonical
    weights sit at w_cpu[key][pos[e]], computed by a spawn pool."""
    import multiprocessing as mp
    import os
    import tempfile
    experts = sorted(int(e) for e in experts)
    n = workers or max(1, min(16, len(os.sched_getaffinity(0))))
    chunks = [experts[i::n] for i in range(n) if experts[i::n]]
    x = np.asarray(x, dtype=np.float64)
    logits = np.asarray(logits, dtype=np.float32)
    with tempfile.TemporaryDirectory() as wdir:
        keys = list(w_cpu.keys())
        for key in keys:
            np.save(f"{wdir}/{key}.npy", _np_of(w_cpu[key]))
        args = [(wdir, keys, fmt, dict(pos), x, logits, k, c, act) for c in chunks]
        with mp.get_context("spawn").Pool(len(chunks)) as pool:
            outs = pool.map(_oracle_subset, args)
    return np.sum(outs, axis=0)
