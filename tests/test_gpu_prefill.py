"""GPU parity of the FP4 tensor-core path (MOE_FFN_ACT_NVFP4): NVFP4 weights,
activations quantised to NVFP4 before each product, tcgen05 block-scaled MMA.
The oracle runs the same layer definition (act="nvfp4")."""
import numpy as np
import pytest
import torch

import synth
from tests.gpu_util import Built, check_tol, load_moe, require_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def moe():
    require_gpu()
    return load_moe()


def _cfg(name, E, k, d, I):
    return synth.LayerConfig(name, E=E, k=k, d=d, I=I, fmt="nvfp4", act="nvfp4")


@pytest.mark.parametrize("tiles", ["auto", "cta", "pair"])
@pytest.mark.parametrize("E,k,d,I,T", [
    (8, 2, 512, 256, 64),       # one chunk per expert, partial N
    (4, 2, 256, 256, 400),      # ~200 rows per expert: one pair chunk each, two 128-row tiles
    (4, 2, 256, 256, 700),      # ~350 rows per expert: two pair chunks (224 + ~126), three tiles
    (2, 1, 512, 256, 500),      # ~250 rows per expert: a full pair chunk and a ragged ~26-row tail
    (16, 4, 1024, 512, 37),     # ragged small groups
    (8, 1, 256, 512, 1),        # a single token
])
def test_prefill_small(moe, monkeypatch, E, k, d, I, T, tiles):
    """Both tile families (CTA pairs over 224-row chunks, single CTAs over
    128-row groups; "auto" takes the library's choice by rows per expert)."""
    if tiles != "auto":
        monkeypatch.setenv("MOE_PREFILL_TILES", tiles)
    b = Built(_cfg("pf", E, k, d, I), T, seed=E + T, act="nvfp4")
    out = b.run().cpu().numpy()
    moe.moe_check_status(b.layer.status)
    ref = b.oracle()
    m, r = check_tol(out, ref["out"])
    print(f"prefill E={E} d={d} I={I} T={T} tiles={tiles}: max {m:.2e} mean-rel {r:.2e}")


def test_prefill_host_partial_merge(moe):
    cfg = _cfg("pf_merge", 8, 2, 512, 256)
    b = Built(cfg, 48, seed=3, act="nvfp4")
    full = b.run().cpu().numpy()
    host = b.used[:3]
    hp = b.oracle(experts=host)["out"].astype(np.float32)
    for e in host:
        b.layer.slot[e] = -1
    out = b.run(host_partial=torch.from_numpy(hp).cuda()).cpu().numpy()
    check_tol(out, b.oracle()["out"])
    check_tol(out, full, 1e-3, 1e-4)


def test_activation_codes_bit_exact(moe):
    """The NVFP4 quantisation of x (first stage of the tensor-core path) takes
    its decisions in fp32 exactly as the oracle does: every per-token scale
    and dequantised code must match bit for bit.  Reads the workspace's
    per-token region (codes [T][d/2], then scales [T][d/16] at the next
    1024-byte boundary)."""
    from oracle import formats as F
    cfg = _cfg("pf_codes", 8, 2, 512, 256)
    T = 96
    b = Built(cfg, T, seed=21, act="nvfp4")
    b.run()
    ws = b.layer.workspace.cpu().numpy()
    d = cfg.d
    codes = ws[: T * d // 2].reshape(T, d // 2)
    off = (T * d // 2 + 1023) // 1024 * 1024
    scales = ws[off: off + T * d // 16].reshape(T, d // 16)
    deq_ref, s_ref, _ = F.nvfp4_quantize_rows(b.x.float().numpy())
    got_s = F.e4m3_decode(scales)
    assert np.array_equal(got_s, s_ref)
    got = F.e2m1_decode(F.unpack_nibbles(codes)) * np.repeat(got_s, 16, axis=1)
    assert np.array_equal(got, deq_ref)


@pytest.mark.parametrize("double_buffer", [True, False])
def test_streamed_prefill_matches_resident_layers(moe, double_buffer):
    """Three NVFP4 layers whose pools stay in pinned host memory, streamed
    into two full-layer buffers (one copying while the other computes): each
    layer's output equals the same layer run from a resident pool up to the
    order of the fused combine's atomic adds, and the oracle within the bar."""
    from expert_offload_serving_b200.layer import MoeLayer, StreamedPrefill, pack_pool
    from oracle import moe as M
    cfg = _cfg("stream", 16, 4, 512, 256)
    T, n_layers = 128, 3
    pools, inputs, w_cpu = [], [], []
    for l in range(n_layers):
        w = synth.make_experts(cfg, range(cfg.E), seed=50 + l, device="cuda")
        w_cpu.append({k: v.cpu() for k, v in w.items()})
        pools.append(pack_pool(cfg.E, cfg.d, cfg.I, cfg.fmt, w_cpu[l], range(cfg.E), pin=True))
        logits, x = synth.make_routing(cfg, T, 60 + l)
        inputs.append((logits, x))
    sp = StreamedPrefill(cfg.E, cfg.d, cfg.I, cfg.k, T, pools)
    outs = sp.run([(lg.cuda(), x.cuda()) for lg, x in inputs], double_buffer=double_buffer, keep_outputs=True)
    torch.cuda.synchronize()
    for l in range(n_layers):
        res = MoeLayer(cfg.E, cfg.d, cfg.I, cfg.fmt, cfg.k, T, device_pool=pools[l].cuda(), act="nvfp4")
        ref_gpu = res.forward(inputs[l][0].cuda(), inputs[l][1].cuda())
        check_tol(outs[l].cpu().numpy(), ref_gpu.cpu().numpy(), 1e-5, 1e-6)
        ref = M.moe_layer(inputs[l][1].double().numpy(), inputs[l][0].numpy(), cfg.k,
                          lambda e: M.dequant_expert(cfg.fmt, w_cpu[l], e), act="nvfp4")["out"]
        check_tol(outs[l].cpu().numpy(), ref)
    for L_ in sp.layers:
        moe.moe_check_status(L_.status)
