"""The host share of a split step (moe_host_expert_ffn) against the oracle, on
the CPU: for every weight format and blob layout, the partial sum over a
host-computed expert subset equals oracle.moe_layer restricted to that subset.
Also the bandwidth profile's host leg (no GPU needed)."""
import numpy as np
import pytest
import torch

import synth
from oracle import moe as M


@pytest.fixture(scope="module")
def moe():
    import expert_offload_serving_b200 as m
    from tests.gpu_util import load_moe
    load_moe()
    return m


def _layer(fmt, d, I, E=12, k=3, T=9, seed=0):
    from expert_offload_serving_b200.layer import pack_pool
    import expert_offload_serving_b200 as m
    cfg = synth.LayerConfig("host", E=E, k=k, d=d, I=I, fmt=fmt)
    logits, x = synth.make_routing(cfg, T, seed)
    w = synth.make_experts(cfg, range(E), seed)
    pool = pack_pool(E, d, I, fmt, w, range(E), pin=False)
    idx, gate = M.route_topk(logits.numpy(), k)
    return cfg, m.shape(E, d, I, fmt), pool, w, logits, x, idx, gate


def _run(moe, s, pool, x, idx, gate, experts, threads=0):
    T = x.shape[0]
    out = torch.full((T, s.d), float("nan"), dtype=torch.float32)
    moe.moe_host_expert_ffn(s, pool, experts, x.contiguous(), torch.from_numpy(idx.astype(np.int32)),
                            torch.from_numpy(gate.astype(np.float32)), out, threads)
    return out.numpy()


@pytest.mark.parametrize("fmt,d,I", [("bf16", 256, 256), ("bf16", 264, 136), ("mxfp4", 512, 256),
                                     ("mxfp4", 288, 96), ("nvfp4", 256, 128)])
def test_host_expert_ffn_matches_oracle(moe, fmt, d, I):
    cfg, s, pool, w, logits, x, idx, gate = _layer(fmt, d, I)
    used = sorted(set(idx.ravel().tolist()))
    host = used[::2]
    out = _run(moe, s, pool, x, idx, gate, host)
    ref = M.moe_layer(x.double().numpy(), logits.numpy(), cfg.k, lambda e: M.dequant_expert(fmt, w, e),
                      experts=host)["out"]
    err = np.abs(out - ref)
    assert err.max() <= 1e-5 * np.abs(ref).max()
    assert err.mean() <= 1e-6 * np.abs(ref).mean()
    # tokens with no host pair get exact zeros
    none = [t for t in range(x.shape[0]) if not set(idx[t].tolist()) & set(host)]
    assert not out[none].any()


def test_host_expert_ffn_thread_count_does_not_change_result(moe):
    cfg, s, pool, w, logits, x, idx, gate = _layer("mxfp4", 512, 256, T=16, seed=3)
    used = sorted(set(idx.ravel().tolist()))
    a = _run(moe, s, pool, x, idx, gate, used, threads=1)
    b = _run(moe, s, pool, x, idx, gate, used, threads=4)
    c = _run(moe, s, pool, x, idx, gate, list(reversed(used)) + used[:2], threads=3)   # order, duplicates
    assert np.array_equal(a, b) and np.array_equal(a, c)


def test_host_expert_ffn_empty_and_bad_ids(moe):
    cfg, s, pool, w, logits, x, idx, gate = _layer("bf16", 256, 256)
    unused = sorted(set(range(cfg.E)) - set(idx.ravel().tolist()))
    assert not _run(moe, s, pool, x, idx, gate, []).any()
    if unused:
        assert not _run(moe, s, pool, x, idx, gate, unused[:1]).any()
    with pytest.raises(moe.MoeError) as ei:
        _run(moe, s, pool, x, idx, gate, [cfg.E])
    assert ei.value.status == moe.MOE_ERR_INVALID_ARG


def test_host_expert_ffn_full_size_expert(moe):
    """One expert of the cached-decode workload (E=256, d=4096, I=2048,
    MXFP4, stage-tiled blob) for two tokens."""
    from expert_offload_serving_b200.layer import pack_pool
    cfg = synth.CONFIGS["decode_mxfp4"]
    e = 7
    w = synth.make_experts(cfg, [e], 0)
    s = moe.shape(cfg.E, cfg.d, cfg.I, cfg.fmt)
    B = moe.moe_expert_blob_bytes(s)
    pool = torch.zeros((cfg.E, B), dtype=torch.uint8)
    pool[e] = pack_pool(cfg.E, cfg.d, cfg.I, cfg.fmt, w, [e], pin=False)[0]
    x = synth.make_routing(cfg, 2, 1)[1]
    idx = np.array([[e, 1, 2, 3, 4, 5], [0, 1, 2, e, 4, 5]], dtype=np.int32)
    gate = np.full((2, 6), 1 / 6)
    out = _run(moe, s, pool, x, idx, gate, [e])
    deq = M.dequant_expert(cfg.fmt, w, 0)
    ref = M.swiglu_ffn(x.double().numpy(), *deq) / 6
    err = np.abs(out - ref)
    assert err.max() <= 1e-5 * np.abs(ref).max() and err.mean() <= 1e-6 * np.abs(ref).mean()


def test_profile_bandwidth_host_leg(moe):
    cfg, s, pool, w, logits, x, idx, gate = _layer("mxfp4", 512, 256)
    h2d, host = moe.moe_profile_bandwidth(s, pool, 4)
    assert h2d == 0.0 and host > 0.0
