"""Pins of oracle.moe: routing, permutation and the layer against brute force,
library routines and invariants (no GPU)."""
import math

import numpy as np
import pytest
import torch

import synth
from oracle import formats as F
from oracle import moe as M


# ---------------------------------------------------------------- routing
def brute_topk(row, k):
    order = sorted(range(len(row)), key=lambda e: (-float(row[e]), e))
    return order[:k]


def check_route(logits, k):
    idx, gate = M.route_topk(logits, k)
    for t in range(logits.shape[0]):
        assert idx[t].tolist() == brute_topk(logits[t], k)
        sel = [float(logits[t, e]) for e in idx[t]]
        z = [math.exp(v - sel[0]) for v in sel]
        for j in range(k):
            assert abs(gate[t, j] - z[j] / sum(z)) <= 1e-15
    return idx, gate


def test_route_brute_force_random():
    rng = np.random.default_rng(0)
    for E, k in ((8, 2), (16, 5), (33, 7), (256, 6)):
        logits = rng.standard_normal((6, E)).astype(np.float32)
        check_route(logits, k)


def test_route_ties_to_lowest_index():
    rng = np.random.default_rng(1)
    logits = rng.integers(-2, 3, size=(20, 12)).astype(np.float32)   # many ties
    idx, _ = check_route(logits, 5)
    l = np.zeros((1, 6), dtype=np.float32)
    l[0, 1] = -0.0
    l[0, 4] = -0.0
    idx, gate = M.route_topk(l, 6)
    assert idx[0].tolist() == [0, 1, 2, 3, 4, 5]         # -0.0 ties +0.0
    assert np.allclose(gate, 1 / 6)


def test_route_matches_torch_topk_on_distinct_values():
    rng = np.random.default_rng(2)
    logits = rng.standard_normal((50, 128)).astype(np.float32)
    idx, gate = M.route_topk(logits, 8)
    v, i = torch.topk(torch.from_numpy(logits).double(), 8, dim=1)
    assert np.array_equal(idx, i.numpy())
    full = torch.softmax(torch.from_numpy(logits).double(), dim=1)
    sel = torch.gather(full, 1, i)
    assert np.allclose(gate, (sel / sel.sum(1, keepdim=True)).numpy(), rtol=1e-13, atol=0)


def test_route_gates_simplex_and_sorted():
    rng = np.random.default_rng(3)
    logits = (rng.standard_normal((100, 256)) * 3).astype(np.float32)
    _, gate = M.route_topk(logits, 6)
    assert np.allclose(gate.sum(1), 1.0, atol=1e-14)
    assert np.all(np.diff(gate, axis=1) <= 0)


def test_route_k_equals_E():
    rng = np.random.default_rng(4)
    logits = rng.standard_normal((3, 5)).astype(np.float32)
    idx, gate = check_route(logits, 5)
    ref = torch.softmax(torch.from_numpy(logits).double(), 1).numpy()
    assert np.allclose(np.take_along_axis(ref, idx.astype(np.int64), 1), gate, rtol=1e-13)


# ---------------------------------------------------------------- permutation
def check_permute(idx, E):
    offsets, perm, inv_perm = M.permute(idx, E)
    flat = idx.ravel().tolist()
    n = len(flat)
    ref = sorted(range(n), key=lambda p: flat[p])      # Python's sort is stable
    assert perm.tolist() == ref
    assert offsets[0] == 0 and offsets[-1] == n
    for e in range(E):
        grp = perm[offsets[e]:offsets[e + 1]]
        assert all(flat[p] == e for p in grp)
        assert np.all(np.diff(grp) > 0)
    assert np.array_equal(inv_perm[perm], np.arange(n))
    return offsets, perm, inv_perm


def test_permute_brute_force():
    rng = np.random.default_rng(5)
    for T, k, E in ((1, 1, 1), (4, 2, 8), (64, 8, 128), (37, 6, 256), (5, 3, 1000)):
        idx = np.stack([rng.choice(E, k, replace=False) for _ in range(T)]).astype(np.int32)
        check_permute(idx, E)


def test_permute_empty_experts_and_skew():
    idx = np.array([[3, 1], [3, 0], [3, 1]], dtype=np.int32)
    offsets, perm, inv = check_permute(idx, 6)
    assert offsets.tolist() == [0, 1, 3, 3, 6, 6, 6]
    assert perm.tolist() == [3, 1, 5, 0, 2, 4]


# ---------------------------------------------------------------- layer
def test_single_expert_k1_is_dense_swiglu():
    """E=1, k=1: gate 1, so the layer is a dense SwiGLU FFN (torch silu + matmul)."""
    rng = np.random.default_rng(6)
    T, d, I = 5, 64, 48
    x = rng.standard_normal((T, d))
    wg, wu, wd = (rng.standard_normal(s) * 0.1 for s in ((I, d), (I, d), (d, I)))
    logits = rng.standard_normal((T, 1)).astype(np.float32)
    res = M.moe_layer(x, logits, 1, lambda e: (wg, wu, wd))
    xt, g, u, dd = (torch.from_numpy(a) for a in (x, wg, wu, wd))
    ref = (torch.nn.functional.silu(xt @ g.T) * (xt @ u.T)) @ dd.T
    assert np.allclose(res["out"], ref.numpy(), rtol=1e-13, atol=1e-15)


def _tiny_layer(seed=0):
    cfg = synth.CONFIGS["tiny"]
    logits, x = synth.make_routing(cfg, 4, seed)
    w = synth.make_experts(cfg, range(cfg.E), seed)
    deq = {e: M.dequant_expert("bf16", w, e) for e in range(cfg.E)}
    xs = x.double().numpy()
    return cfg, logits.numpy(), xs, deq


def test_layer_brute_force_loops_tiny():
    """Pure-Python loops over tokens, selected experts, rows and columns."""
    cfg, logits, x, deq = _tiny_layer()
    res = M.moe_layer(x, logits, cfg.k, lambda e: deq[e])
    T, d, I = x.shape[0], cfg.d, cfg.I
    for t in range(T):
        row = logits[t].tolist()
        sel = sorted(range(cfg.E), key=lambda e: (-row[e], e))[:cfg.k]
        ex = [math.exp(row[e] - row[sel[0]]) for e in sel]
        out = [0.0] * d
        for j, e in enumerate(sel):
            wg, wu, wd = (m.tolist() for m in deq[e])
            xt = x[t].tolist()
            a = []
            for i in range(I):
                h = sum(wg[i][c] * xt[c] for c in range(d))
                u = sum(wu[i][c] * xt[c] for c in range(d))
                a.append(h / (1.0 + math.exp(-h)) * u)
            g = ex[j] / sum(ex)
            for c in range(d):
                out[c] += g * sum(wd[c][i] * a[i] for i in range(I))
        assert np.allclose(res["out"][t], out, rtol=1e-11, atol=1e-13)


def test_token_order_invariance():
    cfg, logits, x, deq = _tiny_layer(1)
    res = M.moe_layer(x, logits, cfg.k, lambda e: deq[e])
    p = np.array([2, 0, 3, 1])
    res2 = M.moe_layer(x[p], logits[p], cfg.k, lambda e: deq[e])
    assert np.array_equal(res2["out"], res["out"][p])


@pytest.mark.parametrize("dtype,tol", [(np.float64, 1e-12), (np.float32, 1e-6)])
def test_split_invariance(dtype, tol):
    """Any expert subset A plus its complement B sums to the whole layer (the
    exact merge of host-computed and GPU-computed partial sums)."""
    cfg, logits, x, deq = _tiny_layer(2)
    full = M.moe_layer(x, logits, cfg.k, lambda e: deq[e], dtype=dtype)["out"]
    rng = np.random.default_rng(7)
    for _ in range(3):
        A = set(rng.choice(cfg.E, 3, replace=False).tolist())
        B = set(range(cfg.E)) - A
        oa = M.moe_layer(x, logits, cfg.k, lambda e: deq[e], experts=A, dtype=dtype)["out"]
        ob = M.moe_layer(x, logits, cfg.k, lambda e: deq[e], experts=B, dtype=dtype)["out"]
        err = np.abs(oa + ob - full).max() / np.abs(full).max()
        assert err <= tol


def test_token_subset_matches_full():
    cfg, logits, x, deq = _tiny_layer(3)
    full = M.moe_layer(x, logits, cfg.k, lambda e: deq[e])["out"]
    part = M.moe_layer(x, logits, cfg.k, lambda e: deq[e], tokens=[1, 3])["out"]
    # BLAS may block a smaller row count differently: equal to the last bits
    assert np.allclose(part[[1, 3]], full[[1, 3]], rtol=1e-14, atol=1e-16)
    assert not part[[0, 2]].any()


def test_per_pair_outputs_recombine():
    cfg, logits, x, deq = _tiny_layer(4)
    res = M.moe_layer(x, logits, cfg.k, lambda e: deq[e])
    y = M.per_pair_outputs(x, logits, cfg.k, lambda e: deq[e])
    out = np.zeros_like(res["out"])
    for p in range(y.shape[0]):
        t, j = divmod(p, cfg.k)
        out[t] += res["gate"][t, j] * y[p]
    assert np.allclose(out, res["out"], rtol=1e-14, atol=1e-16)


def test_quantised_formats_dequant_into_layer():
    """A layer on MXFP4 / NVFP4 weights equals the same layer on the dense
    fp64 matrices its codes decode to (dequantisation is the only new step)."""
    for name in ("decode_mxfp4", "prefill_nvfp4"):
        base = synth.CONFIGS[name]
        cfg = synth.LayerConfig(name, E=4, k=2, d=128, I=64, fmt=base.fmt)
        w = synth.make_experts(cfg, range(cfg.E), 0)
        logits, x = synth.make_routing(cfg, 3, 0)
        deq = {e: M.dequant_expert(cfg.fmt, w, e) for e in range(cfg.E)}
        # the generator's encoding is close to the N(0, 0.02^2) draws it came from
        for e in range(cfg.E):
            for m in deq[e]:
                assert 0.012 < m.std() < 0.03
        res = M.moe_layer(x.double().numpy(), logits.numpy(), cfg.k, lambda e: deq[e])
        assert np.isfinite(res["out"]).all() and np.abs(res["out"]).max() > 0


def test_act_quant_mode_close_to_unquantised():
    """NVFP4 activation quantisation perturbs the layer by a few percent, not more."""
    cfg, logits, x, deq = _tiny_layer(5)
    a = M.moe_layer(x, logits, cfg.k, lambda e: deq[e])["out"]
    b = M.moe_layer(x, logits, cfg.k, lambda e: deq[e], act="nvfp4")["out"]
    rel = np.abs(a - b).mean() / np.abs(a).mean()
    assert 0.005 < rel < 0.2
