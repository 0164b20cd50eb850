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


# ---------------------------------------------------------------- act = "nvfp4"
# A layer worked by hand for the FP4 x FP4 reading: x and the SwiGLU output a
# are each quantised to NVFP4 (blocks of 16 along K, unit tensor scale, scale
# = E4M3(amax/6), codes = E2M1 nearest with ties to the even mantissa) before
# the product that consumes them.  T = 1, d = 32 (two x blocks), I = 16 (one a
# block), one expert, k = 1 (gate 1).
_X_B0 = [3.0, -1.25, 0.3, 0.75, -0.1, 2.2, 1.0, -3.0, 0.5, 0.26, -2.6, 1.74, 0.0, -0.74, 1.5, 2.5]
# block 0: amax 3 -> s = 0.5 (exact E4M3).  x/s = 6, -2.5 (tie -> -2), 0.6 -> 0.5,
# 1.5, -0.2 -> -0, 4.4 -> 4, 2, -6, 1, 0.52 -> 0.5, -5.2 -> -6, 3.48 -> 3, 0,
# -1.48 -> -1.5, 3, 5 (tie -> 4); times s:
_XQ_B0 = [3.0, -1.0, 0.25, 0.75, -0.0, 2.0, 1.0, -3.0, 0.5, 0.25, -3.0, 1.5, 0.0, -0.75, 1.5, 2.0]
# block 1 = 4 x block 0: amax 12 -> s = 2, the same codes, values x 4.
_C = [0.375, -0.15625, 0.0625, 0.21875, 0.34375, 0.046875, 0.015625, -0.09375]


def _hand_layer():
    d, I = 32, 16
    x = np.array(_X_B0 + [4.0 * v for v in _X_B0])[None, :]
    wg = np.zeros((I, d))
    wu = np.zeros((I, d))
    wd = np.zeros((d, I))
    for i in range(I):
        sgn = 1.0 if i % 2 == 0 else -1.0
        # h = +-(64 xq0 + 64 xq1 + 256 xq2) = +-(192 - 64 + 64) = +-192: silu(192) = 192
        # exactly in float64 and silu(-192) ~ -1e-81, which is -0 in fp32
        wg[i, 0], wg[i, 1], wg[i, 2] = 64 * sgn, 64 * sgn, 256 * sgn
        # u = xq5 * w = 2 * w: c_m on even rows, 1 on odd rows
        wu[i, 5] = _C[i // 2] / 2 if i % 2 == 0 else 0.5
        wd[i, i] = 1 / 8              # out[c] = a_q[c] / 8 for c < 16
        wd[16, i] = 1 / 16            # out[16] = sum(a_q) / 16
    return x, wg, wu, wd


def _hand_expected():
    # a (even rows) = 192 c = 72, -30, 12, 42, 66, 9, 3, -18; odd rows -0.
    # amax 72 -> s = 12 (exact E4M3); a/s = 16 c = 6, -2.5 (tie -> -2), 1,
    # 3.5 (tie -> 4), 5.5 -> 6, 0.75 (tie -> 1), 0.25 (tie -> 0), -1.5;
    # a_q = 72, -24, 12, 48, 72, 12, 0, -18.
    aq = [72.0, -24.0, 12.0, 48.0, 72.0, 12.0, 0.0, -18.0]
    out = np.zeros(32)
    for m, v in enumerate(aq):
        out[2 * m] = v / 8
    out[16] = sum(aq) / 16            # 174 / 16 = 10.875
    return out


def test_act_nvfp4_quantises_x_by_hand():
    x, *_ = _hand_layer()
    deq, s, _ = F.nvfp4_quantize_rows(x.astype(np.float32))
    assert s.tolist() == [[0.5, 2.0]]
    assert deq[0].tolist() == _XQ_B0 + [4.0 * v for v in _XQ_B0]
    assert np.signbit(deq[0, 4]) and np.signbit(deq[0, 20])      # -0.1 keeps its sign bit


def test_act_nvfp4_layer_hand_worked():
    x, wg, wu, wd = _hand_layer()
    y = M.swiglu_ffn(x, wg, wu, wd, act="nvfp4")
    assert y[0].tolist() == _hand_expected().tolist()
    res = M.moe_layer(x, np.zeros((1, 1), np.float32), 1, lambda e: (wg, wu, wd), act="nvfp4")
    assert res["out"][0].tolist() == _hand_expected().tolist()


def test_act_none_layer_differs_from_hand_worked():
    """Without activation quantisation the same layer is not the hand-worked
    result (h = 188.8, u = 1.1 c): the quantisation is what that pin checks."""
    x, wg, wu, wd = _hand_layer()
    y = M.swiglu_ffn(x, wg, wu, wd, act="none")
    assert abs(y[0, 0] - 188.8 * 1.1 * _C[0] / 8) < 1e-9
    assert y[0].tolist() != _hand_expected().tolist()


# ---------------------------------------------------------------- NVFP4 weights
_E2M1_MAG = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def test_nvfp4_dequant_expert_tensor_scale_order():
    """dequant_expert applies the fp32 tensor scales to gate, up and down in
    that order, and each E4M3 block scale to its own 16 elements of a row.
    Codes: element (r, c) of every matrix holds magnitude (r + c) % 8 with the
    sign bit set on odd rows; block b of every row has scale 2^b; tensor
    scales gate 2, up 1/2, down 1/4."""
    I, d = 16, 32
    def mat(R, K):
        codes = np.array([[((r + c) % 8) | (8 if r % 2 else 0) for c in range(K)] for r in range(R)], np.uint8)
        packed = (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)
        sc = np.array([[0x38 + 8 * b for b in range(K // 16)] for _ in range(R)], np.uint8)   # 2^b
        want = np.array([[(-1.0 if r % 2 else 1.0) * _E2M1_MAG[(r + c) % 8] * 2.0 ** (c // 16)
                          for c in range(K)] for r in range(R)])
        return packed[None], sc[None], want
    (cg, sg, g), (cu, su, u), (cd, sd, dn) = mat(I, d), mat(I, d), mat(d, I)
    w = dict(wg=cg, sg=sg, wu=cu, su=su, wd=cd, sd=sd, ts=np.array([[2.0, 0.5, 0.25]], np.float32))
    G, U, D = M.dequant_expert("nvfp4", w, 0)
    assert np.array_equal(G, 2.0 * g)
    assert np.array_equal(U, 0.5 * u)
    assert np.array_equal(D, 0.25 * dn)
