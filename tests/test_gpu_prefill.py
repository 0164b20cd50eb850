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


@pytest.mark.parametrize("E,k,d,I,T", [
    (8, 2, 512, 256, 64),       # one chunk per expert, partial N
    (4, 2, 256, 256, 400),      # 200 rows per expert: two chunks (128 + 72)
    (16, 4, 1024, 512, 37),     # ragged small groups
    (8, 1, 256, 512, 1),        # a single token
])
def test_prefill_small(moe, E, k, d, I, T):
    b = Built(_cfg("pf", E, k, d, I), T, seed=E + T, act="nvfp4")
    out = b.run().cpu().numpy()
    moe.moe_check_status(b.layer.status)
    ref = b.oracle()
    m, r = check_tol(out, ref["out"])
    print(f"prefill E={E} d={d} I={I} T={T}: max {m:.2e} mean-rel {r:.2e}")


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


def test_prefill_full_size_sampled(moe):
    """The prefill workload itself (E=256, k=6, d=4096, I=2048, T=4096):
    indices and permutation bit-exact; sampled tokens' outputs vs the oracle."""
    from oracle import moe as M
    cfg = synth.CONFIGS["prefill_nvfp4"]
    T = 4096
    b = Built(cfg, T, seed=0, act="nvfp4")
    out = b.run().cpu().numpy()
    moe.moe_check_status(b.layer.status)
    idx, _ = M.route_topk(b.logits.numpy(), cfg.k)
    off, perm, _ = M.permute(idx, cfg.E)
    assert np.array_equal(b.layer.idx.cpu().numpy(), idx)
    assert np.array_equal(b.layer.offsets.cpu().numpy(), off)
    assert np.array_equal(b.layer.perm[: T * cfg.k].cpu().numpy(), perm)
    assert np.isfinite(out).all()
    toks = [0, 1, 2047, 4095]
    ref = b.oracle(tokens=toks)["out"]
    check_tol(out[toks], ref[toks])


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
