"""Plant plausible mistakes in the oracle (CPU only) and check that a pin fails
for each: a dropped term, a wrong sign or index, a transposed operand, a wrong
rounding rule, a wrong tie-break."""
import numpy as np
import pytest

from oracle import formats as F
from oracle import lru as L
from oracle import moe as M

from tests import test_oracle_formats as PF
from tests import test_oracle_layer as PL
from tests import test_oracle_lru as PR


def _fails(fn, *a):
    try:
        fn(*a)
    except (AssertionError, L.CapacityError, ValueError):
        return True
    return False


def test_silu_without_h_factor_is_caught(monkeypatch):
    monkeypatch.setattr(M, "silu", lambda h: 1.0 / (1.0 + np.exp(-h)))
    assert _fails(PL.test_single_expert_k1_is_dense_swiglu)


def test_swapped_up_and_down_roles_is_caught(monkeypatch):
    orig = M.swiglu_ffn

    def bad(xr, wg, wu, wd, act="none", dtype=np.float64):
        return orig(xr, wu, wg, wd, act=act, dtype=dtype)        # gate/up exchanged
    monkeypatch.setattr(M, "swiglu_ffn", bad)
    assert _fails(PL.test_single_expert_k1_is_dense_swiglu)


def test_gates_not_renormalised_is_caught(monkeypatch):
    orig = M.route_topk

    def bad(logits, k):
        idx, _ = orig(logits, k)
        l = np.asarray(logits, dtype=np.float64)
        full = np.exp(l - l.max(1, keepdims=True))
        full /= full.sum(1, keepdims=True)
        return idx, np.take_along_axis(full, idx.astype(np.int64), 1)
    monkeypatch.setattr(M, "route_topk", bad)
    assert _fails(PL.test_route_brute_force_random)
    assert _fails(PL.test_route_gates_simplex_and_sorted)


def test_ties_to_highest_index_is_caught(monkeypatch):
    def bad(logits, k):
        l = np.asarray(logits, dtype=np.float32)
        E = l.shape[1]
        order = E - 1 - np.argsort(-l[:, ::-1].astype(np.float64), axis=1, kind="stable")
        idx = order[:, :k].astype(np.int32)
        sel = np.take_along_axis(l, idx, 1).astype(np.float64)
        z = np.exp(sel - sel[:, :1])
        return idx, z / z.sum(1, keepdims=True)
    monkeypatch.setattr(M, "route_topk", bad)
    assert _fails(PL.test_route_ties_to_lowest_index)


def test_unstable_permutation_is_caught(monkeypatch):
    orig = M.permute

    def bad(idx, E):
        off, perm, inv = orig(idx, E)
        perm = perm.copy()
        for e in range(E):
            perm[off[e]:off[e + 1]] = perm[off[e]:off[e + 1]][::-1]
        inv = np.empty_like(perm)
        inv[perm] = np.arange(perm.size)
        return off, perm, inv
    monkeypatch.setattr(M, "permute", bad)
    assert _fails(PL.test_permute_brute_force)


def test_off_by_one_combine_index_is_caught(monkeypatch):
    orig = M.moe_layer

    def bad(*a, **kw):
        r = orig(*a, **kw)
        r["out"] = np.roll(r["out"], 1, axis=1)
        return r
    monkeypatch.setattr(M, "moe_layer", bad)
    assert _fails(PL.test_layer_brute_force_loops_tiny)


def test_wrong_e2m1_magnitude_is_caught(monkeypatch):
    orig = F.e2m1_decode
    monkeypatch.setattr(F, "e2m1_decode", lambda c: np.where(np.abs(orig(c)) == 6, np.sign(orig(c)) * 5, orig(c)))
    assert _fails(PF.test_e2m1_table_facts)


def test_wrong_e4m3_bias_is_caught(monkeypatch):
    monkeypatch.setattr(F, "e4m3_decode", lambda c: F.__dict__["e8m0_decode"](c) * 0 + 1.0)
    assert _fails(PF.test_e4m3_decode_matches_torch_all_codes)


def test_round_half_away_from_zero_is_caught(monkeypatch):
    monkeypatch.setattr(F, "_rne_grid", lambda a, step: np.floor(a / step + 0.5) * step)
    assert _fails(PF.test_nvfp4_block_hand_worked)
    assert _fails(PF.test_e4m3_round_vs_torch_and_brute_force)


def test_most_recent_victim_is_caught(monkeypatch):
    # the module's victim choice calls min(); planting max() picks the newest slot
    monkeypatch.setattr(L, "min", max, raising=False)
    assert _fails(PR.test_hand_worked_trace)


# ---- act = "nvfp4": the FP4 prefill reading quantises x before GEMM1 and a
# before GEMM2; each plausible misplacement must fail the hand-worked layer.
def _q(v, block=16):
    return F.nvfp4_quantize_rows(np.asarray(v, np.float32), block)[0]


def _plant_ffn(monkeypatch, body):
    def bad(xr, wg, wu, wd, act="none", dtype=np.float64):
        if act != "nvfp4":
            return M.__dict__["_orig_swiglu"](xr, wg, wu, wd, act=act, dtype=dtype)
        return body(np.asarray(xr, np.float64), np.asarray(wg), np.asarray(wu), np.asarray(wd))
    monkeypatch.setitem(M.__dict__, "_orig_swiglu", M.swiglu_ffn)
    monkeypatch.setattr(M, "swiglu_ffn", bad)


def test_nvfp4_x_quantised_but_not_a_is_caught(monkeypatch):
    _plant_ffn(monkeypatch, lambda x, g, u, d: (M.silu(_q(x) @ g.T) * (_q(x) @ u.T)) @ d.T)
    assert _fails(PL.test_act_nvfp4_layer_hand_worked)


def test_nvfp4_a_quantised_but_not_x_is_caught(monkeypatch):
    _plant_ffn(monkeypatch, lambda x, g, u, d: _q(M.silu(x @ g.T) * (x @ u.T)) @ d.T)
    assert _fails(PL.test_act_nvfp4_layer_hand_worked)


def test_nvfp4_a_quantised_before_the_product_is_caught(monkeypatch):
    _plant_ffn(monkeypatch, lambda x, g, u, d: (_q(M.silu(_q(x) @ g.T)) * _q(_q(x) @ u.T)) @ d.T)
    assert _fails(PL.test_act_nvfp4_layer_hand_worked)


def test_nvfp4_x_blocks_of_32_is_caught(monkeypatch):
    _plant_ffn(monkeypatch, lambda x, g, u, d: _q(M.silu(_q(x, 32) @ g.T) * (_q(x, 32) @ u.T)) @ d.T)
    assert _fails(PL.test_act_nvfp4_layer_hand_worked)


def test_nvfp4_scale_from_amax_over_4_is_caught(monkeypatch):
    orig = F.e4m3_round
    # the quantiser's only e4m3_round call takes amax/6; planting amax/4 there
    monkeypatch.setattr(F, "e4m3_round", lambda v: orig(np.asarray(v, np.float32) * np.float32(1.5)))
    assert _fails(PL.test_act_nvfp4_quantises_x_by_hand)
    assert _fails(PL.test_act_nvfp4_layer_hand_worked)


def test_nvfp4_tensor_scales_reversed_is_caught(monkeypatch):
    orig = F.dequant_nvfp4
    calls = []

    def bad(codes, scales, ts):
        calls.append(ts)
        return orig(codes, scales, {2.0: 0.25, 0.25: 2.0}.get(float(ts), ts))   # gate <-> down
    monkeypatch.setattr(F, "dequant_nvfp4", bad)
    assert _fails(PL.test_nvfp4_dequant_expert_tensor_scale_order)
    assert len(calls) == 3


def test_resize_keeping_the_oldest_is_caught(monkeypatch):
    orig = L.LRUCache.resize

    def bad(self, n):
        self.last_used = [-v for v in self.last_used]      # ranks the oldest first
        r = orig(self, n)
        self.last_used = [-v for v in self.last_used]
        return r
    monkeypatch.setattr(L.LRUCache, "resize", bad)
    assert _fails(PR.test_resize_hand_worked)
