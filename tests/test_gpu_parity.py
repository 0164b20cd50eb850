"""GPU parity of every step of the layer against the CPU oracle, through the
C ABI: indices and permutations bit-exact, outputs within the stated
tolerance, on the seeded workloads and their edge cases."""
import numpy as np
import pytest
import torch

import synth
from oracle import lru as L
from oracle import moe as M
from tests.gpu_util import Built, check_tol, load_moe, require_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def moe():
    require_gpu()
    return load_moe()


# ---------------------------------------------------------------- step 1
@pytest.mark.parametrize("T,E,k", [(1, 8, 2), (5, 33, 7), (64, 128, 8), (4096, 256, 6), (3, 1000, 32),
                                   (7, 1024, 1), (2, 5, 5), (300, 64, 4)])
def test_route_topk_parity(moe, T, E, k):
    rng = np.random.default_rng(T * 7 + E)
    logits = rng.standard_normal((T, E)).astype(np.float32)
    if E >= 16:   # constructed ties and signed zeros
        logits[:, 3] = logits[:, 1]
        logits[0, :6] = 0.0
        logits[0, 2] = -0.0
        logits[-1, :] = np.round(logits[-1, :])
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    gate = torch.empty((T, k), dtype=torch.float32, device="cuda")
    moe.moe_route_topk(torch.from_numpy(logits).cuda(), k, idx, gate)
    ref_idx, ref_gate = M.route_topk(logits, k)
    assert np.array_equal(idx.cpu().numpy(), ref_idx)
    assert np.abs(gate.cpu().numpy() - ref_gate).max() <= 2e-6


def test_route_topk_empty(moe):
    idx = torch.empty((0, 2), dtype=torch.int32, device="cuda")
    moe.moe_route_topk(torch.empty((0, 8), device="cuda"), 2, idx, idx.float())


# ---------------------------------------------------------------- step 2
@pytest.mark.parametrize("T,k,E", [(1, 2, 8), (64, 8, 128), (128, 8, 128), (129, 8, 128), (4096, 6, 256),
                                   (1000, 7, 1000), (333, 3, 1024), (2, 1, 1)])
def test_permute_parity(moe, T, k, E):
    rng = np.random.default_rng(T + 31 * k + E)
    if k <= E:
        idx = np.stack([rng.choice(E, k, replace=False) for _ in range(T)]).astype(np.int32)
    else:
        idx = rng.integers(0, E, (T, k)).astype(np.int32)
    if E > 4:
        idx[: T // 2, 0] = 2                       # skew: one hot expert
    d_idx = torch.from_numpy(idx).cuda()
    off = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    perm = torch.empty(T * k, dtype=torch.int32, device="cuda")
    inv = torch.empty(T * k, dtype=torch.int32, device="cuda")
    sb = moe.moe_permute_scratch_bytes(T, k, E)
    scratch = torch.empty(max(sb, 16), dtype=torch.uint8, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    moe.moe_permute(d_idx, E, off, perm, inv, scratch=scratch, dev_status=st)
    moe.moe_check_status(st)
    r_off, r_perm, r_inv = M.permute(idx, E)
    assert np.array_equal(off.cpu().numpy(), r_off)
    assert np.array_equal(perm.cpu().numpy(), r_perm)
    assert np.array_equal(inv.cpu().numpy(), r_inv)


@pytest.mark.parametrize("T", [4, 2000])
def test_permute_reports_bad_expert(moe, T):
    E, k = 16, 2
    idx = np.tile(np.array([[1, 2]], dtype=np.int32), (T, 1))
    idx[1, 1] = 16                                 # out of range
    off = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    perm = torch.empty(T * k, dtype=torch.int32, device="cuda")
    inv = torch.empty(T * k, dtype=torch.int32, device="cuda")
    scratch = torch.empty(max(moe.moe_permute_scratch_bytes(T, k, E), 16), dtype=torch.uint8, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    moe.moe_permute(torch.from_numpy(idx).cuda(), E, off, perm, inv, scratch=scratch, dev_status=st)
    with pytest.raises(moe.MoeError) as ei:
        moe.moe_check_status(st)
    assert ei.value.status == moe.MOE_ERR_DEVICE
    o = off.cpu().numpy()
    assert o[-1] == T * k - 1 and inv.cpu().numpy()[3] == -1


def test_permute_scratch_too_small(moe):
    T, k, E = 2000, 2, 16
    idx = torch.zeros((T, k), dtype=torch.int32, device="cuda")
    off = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    perm = torch.empty(T * k, dtype=torch.int32, device="cuda")
    with pytest.raises(moe.MoeError) as ei:
        moe.moe_permute(idx, E, off, perm, perm.clone(), scratch=torch.empty(8, dtype=torch.uint8, device="cuda"))
    assert ei.value.status == moe.MOE_ERR_CAPACITY


# ---------------------------------------------------------------- steps 3-4, full layer
def test_layer_tiny(moe):
    b = Built(synth.CONFIGS["tiny"], 4)
    out = b.run().cpu().numpy()
    ref = b.oracle()
    check_tol(out, ref["out"])
    assert np.array_equal(b.layer.idx.cpu().numpy(), ref["idx"])
    assert np.array_equal(b.layer.perm.cpu().numpy()[:8], ref["perm"])
    m, r = check_tol(out, ref["out"], 1e-4, 1e-5)    # fp32 path: far inside the bar


@pytest.mark.parametrize("T", [1, 16, 64])
def test_layer_decode_bf16(moe, T):
    b = Built(synth.CONFIGS["decode_bf16"], T, seed=T)
    out = b.run().cpu().numpy()
    ref = b.oracle()
    check_tol(out, ref["out"])
    check_tol(out, ref["out"], 1e-4, 1e-5)
    assert np.array_equal(b.layer.idx[:T].cpu().numpy(), ref["idx"])
    assert np.array_equal(b.layer.offsets.cpu().numpy(), ref["offsets"])


@pytest.mark.parametrize("T", [1, 8])
def test_layer_decode_mxfp4(moe, T):
    b = Built(synth.CONFIGS["decode_mxfp4"], T, seed=3 + T)
    out = b.run().cpu().numpy()
    ref = b.oracle()
    check_tol(out, ref["out"])
    check_tol(out, ref["out"], 1e-4, 1e-5)


@pytest.mark.parametrize("T", [1, 5])
def test_layer_decode_nvfp4_weights(moe, T):
    """NVFP4 weights on the CUDA-core path (activations unquantised)."""
    b = Built(synth.CONFIGS["prefill_nvfp4"], T, seed=11 + T)
    out = b.run().cpu().numpy()
    ref = b.oracle()
    check_tol(out, ref["out"])
    check_tol(out, ref["out"], 1e-4, 1e-5)


@pytest.mark.parametrize("fmt,d,I", [("bf16", 264, 136), ("bf16", 8, 8), ("mxfp4", 288, 96),
                                     ("nvfp4", 384, 128)])
def test_layer_ragged_shapes(moe, fmt, d, I):
    """K not a multiple of the 32-lane stride, tiny and odd sizes."""
    cfg = synth.LayerConfig("ragged", E=12, k=3, d=d, I=I, fmt=fmt)
    b = Built(cfg, 9, seed=5)
    check_tol(b.run().cpu().numpy(), b.oracle()["out"], 1e-4, 1e-5)


@pytest.mark.parametrize("fmt", ["bf16", "mxfp4"])
def test_many_tokens_per_expert(moe, fmt):
    """Groups of more than one 32-pair chunk on the tensor-core path (skewed
    routing, T=64, E=8; d, I multiples of 256)."""
    cfg = synth.LayerConfig("skew", E=8, k=2, d=512, I=256, fmt=fmt, bias_std=2.0)
    b = Built(cfg, 64, seed=2)
    check_tol(b.run().cpu().numpy(), b.oracle()["out"], 1e-4, 1e-5)
    assert (np.diff(b.layer.offsets.cpu().numpy()) > 32).any()


@pytest.mark.parametrize("fmt", ["bf16", "mxfp4"])
@pytest.mark.parametrize("T", [8, 9, 16, 17])
def test_chunk_width_boundary(moe, fmt, T):
    """The MXFP4 path runs 8-pair chunks up to T = 8, 16-pair chunks up to
    T = 16 and 32-pair chunks above; bf16 16-pair chunks up to T = 16.  E = 4,
    k = 4 puts every token on every expert, so the groups fill a chunk
    exactly (8, 16) or spill one pair past it (9, 17)."""
    cfg = synth.LayerConfig("full", E=4, k=4, d=512, I=256, fmt=fmt)
    b = Built(cfg, T, seed=7)
    check_tol(b.run().cpu().numpy(), b.oracle()["out"], 1e-4, 1e-5)
    assert (np.diff(b.layer.offsets.cpu().numpy()) == T).all()


def test_y_perm_rows_match_pairs(moe):
    cfg = synth.CONFIGS["decode_bf16"]
    b = Built(cfg, 16, seed=4)
    b.run()
    y = b.layer.y_perm[:16 * cfg.k].cpu().numpy()
    ref = M.per_pair_outputs(b.x.double().numpy(), b.logits.numpy(), cfg.k, b.weights)
    inv = b.layer.inv_perm[:16 * cfg.k].cpu().numpy()
    check_tol(y[inv], ref, 1e-4, 1e-5)


@pytest.mark.parametrize("T", [1, 16])
def test_fused_out_matches_combine(moe, T):
    """out += gate * y in the FFN epilogue equals y_perm + combine."""
    cfg = synth.CONFIGS["decode_bf16"]
    b = Built(cfg, T, seed=6)
    ref = b.run().clone()
    L_ = b.layer
    out = torch.zeros_like(ref)
    moe.moe_expert_ffn(L_.s, b.x.cuda(), cfg.k, L_.offsets, L_.perm, L_.slot, L_.pool, L_.n_slots,
                       gate=L_.gate, out=out, workspace=L_.workspace, dev_status=L_.status)
    torch.cuda.synchronize()
    assert torch.allclose(out, ref, rtol=1e-5, atol=1e-6 * ref.abs().max().item())


def test_slot_assignment_invariance(moe):
    """The same experts in different slots give bit-identical output."""
    cfg = synth.CONFIGS["decode_mxfp4"]
    a = Built(cfg, 8, seed=9, slot_seed=1).run().cpu()
    b = Built(cfg, 8, seed=9, slot_seed=2).run().cpu()
    assert torch.equal(a, b)


def test_host_partial_merge_and_q_sweep(moe):
    """Split/merge: a random 30% of the step's experts are host-computed (their
    gate-weighted sum comes from the oracle), the rest run on the GPU with the
    host experts' slots set to -1; the merged output equals the all-GPU one."""
    cfg = synth.CONFIGS["split_merge"]
    trace = synth.make_trace(cfg, 8, steps=3, seed=7)
    for t, (logits, x) in enumerate(trace):
        b = Built(cfg, 8, seed=t, logits=logits, x=x)
        full = b.run().cpu().numpy()
        U = b.used
        n_host = int(np.floor(0.3 * len(U) + 0.5))
        host = np.random.default_rng(7 * 1000003 + t).choice(sorted(U), n_host, replace=False).tolist()
        hp = b.oracle(experts=host)["out"].astype(np.float32)
        ref = b.oracle()["out"]
        slot_save = b.layer.slot.clone()
        for q in (0.0, 0.5, 1.0):
            gpu_extra = host[: int(np.floor(q * len(host) + 0.5))]   # the host share shrinks as q grows
            host_now = [e for e in host if e not in gpu_extra]
            b.layer.slot.copy_(slot_save)
            for e in host_now:
                b.layer.slot[e] = -1
            hp = b.oracle(experts=host_now)["out"].astype(np.float32)
            out = b.run(host_partial=torch.from_numpy(hp).cuda()).cpu().numpy()
            check_tol(out, ref)
            # the merge itself adds the host partial exactly; merged and all-GPU
            # outputs differ by the GPU path's own rounding on the host share
            check_tol(out, full, 1e-4, 1e-5)
        b.layer.slot.copy_(slot_save)


def test_cached_layer_trace(moe):
    """Cached mode on a drifting trace: LRU fills from a pinned host pool on a
    side stream.  The device slot table and slot contents follow the oracle
    LRU, and the output matches the oracle at every step."""
    from expert_offload_serving_b200.layer import MoeLayer, pack_pool
    base = synth.CONFIGS["decode_mxfp4"]
    cfg = synth.LayerConfig("cached", E=64, k=6, d=512, I=256, fmt="mxfp4", bias_std=0.5, n_slots=16,
                            rho=0.9)
    w = synth.make_experts(cfg, range(cfg.E), 0, device="cuda")
    w_cpu = {k: v.cpu() for k, v in w.items()}
    host_pool = pack_pool(cfg.E, cfg.d, cfg.I, cfg.fmt, w_cpu, range(cfg.E), pin=True)
    T = 2
    layer = MoeLayer(cfg.E, cfg.d, cfg.I, cfg.fmt, cfg.k, T, host_pool=host_pool, n_slots=cfg.n_slots)
    ref_lru = L.LRUCache(cfg.n_slots, cfg.E)
    deq = {}

    def weights(e):
        if e not in deq:
            deq[e] = M.dequant_expert(cfg.fmt, w_cpu, e)
        return deq[e]
    for t, (logits, x) in enumerate(synth.make_trace(cfg, T, steps=25, seed=3)):
        dl = logits.cuda()
        layer.route(dl)
        U = sorted(set(layer.idx[:T].cpu().numpy().ravel().tolist()))
        fills = layer.prepare(t, U)
        assert fills == ref_lru.step(t, U)[1]
        layer.permute(T)
        layer.ffn(x.cuda())
        layer.combine(T)
        # the main stream waited for this step's fills: once it drains, the side stream is idle
        torch.cuda.current_stream().synchronize()
        assert layer.side.query()
        out = layer.out[:T].cpu().numpy()
        ref = M.moe_layer(x.double().numpy(), logits.numpy(), cfg.k, weights)["out"]
        check_tol(out, ref, 1e-4, 1e-5)
        assert layer.slot.cpu().tolist() == ref_lru.slot_of_expert
    pool = layer.pool.cpu()
    for s, e in enumerate(ref_lru.expert_of_slot):
        if e >= 0:
            assert torch.equal(pool[s], host_pool[e])
    moe.moe_check_status(layer.status)


def test_ffn_reports_bad_slot(moe):
    cfg = synth.CONFIGS["tiny"]
    b = Built(cfg, 4)
    b.layer.slot[b.used[0]] = 10_000                 # beyond n_slots
    b.run()
    with pytest.raises(moe.MoeError) as ei:
        moe.moe_check_status(b.layer.status)
    assert ei.value.status == moe.MOE_ERR_DEVICE


def test_ffn_reports_bad_slot_tensor_core_path(moe):
    """The same error from the tcgen05 decode GEMV (bf16 tile layout)."""
    cfg = synth.LayerConfig("tc_bad_slot", E=8, k=2, d=512, I=256, fmt="bf16")
    b = Built(cfg, 4)
    b.layer.slot[b.used[0]] = 10_000
    b.run()
    with pytest.raises(moe.MoeError) as ei:
        moe.moe_check_status(b.layer.status)
    assert ei.value.status == moe.MOE_ERR_DEVICE


def test_layer_max_experts_and_k(moe):
    """E = 1024 and k = 32, the ABI's upper bounds, on the tensor-core path
    (a 1025-entry unit table in shared memory)."""
    cfg = synth.LayerConfig("maxek", E=1024, k=32, d=256, I=256, fmt="bf16", bias_std=0.5)
    b = Built(cfg, 3, seed=8)
    check_tol(b.run().cpu().numpy(), b.oracle()["out"], 1e-4, 1e-5)


def _mx_layer_with(scale_byte=None, x_scale=None, which="sg"):
    cfg = synth.LayerConfig("mx_range", E=8, k=2, d=512, I=256, fmt="mxfp4")
    logits, x = synth.make_routing(cfg, 2, 4)
    if x_scale is not None:
        x = (x.float() * x_scale).to(torch.bfloat16)
    b = Built(cfg, 2, seed=4, logits=logits, x=x)
    if scale_byte is not None:
        from expert_offload_serving_b200.layer import pack_pool
        b.w_cpu[which][0].fill_(scale_byte)
        b.layer.pool.copy_(pack_pool(cfg.E, cfg.d, cfg.I, cfg.fmt, b.w_cpu, b.order, pin=False))
    return b


@pytest.mark.parametrize("scale_byte,x_scale,which", [(127 + 14, None, "sg"), (127 - 24, None, "sg"),
                                                     (127 + 40, None, "sd"), (127 - 60, None, "sd"),
                                                     (None, 1e5, "sg"), (None, 1e-6, "sg")])
def test_mxfp4_wide_scale_and_activation_range_is_exact(moe, scale_byte, x_scale, which):
    """The tensor core applies the E8M0 block scales itself and the
    activations enter as E4M3 terms under E8M0 scales of their own, so block
    scales far outside f16 (2^14, 2^-24 on the gate rows, 2^40, 2^-60 on the
    down projection) and activations of 1e5 or 1e-6 still match the oracle,
    with no status reported."""
    b = _mx_layer_with(scale_byte, x_scale, which)
    out = b.run().cpu().numpy()
    moe.moe_check_status(b.layer.status)
    check_tol(out, b.oracle()["out"], 1e-4, 1e-5)


def test_mxfp4_edge_scales_are_exact(moe):
    """Scales 2^-23 (gate) and 2^13 (down projection) match the oracle."""
    for byte, which in ((127 - 23, "sg"), (127 + 13, "sd")):
        b = _mx_layer_with(byte, None, which)
        out = b.run().cpu().numpy()
        moe.moe_check_status(b.layer.status)
        check_tol(out, b.oracle()["out"], 1e-4, 1e-5)


def test_mxfp4_mixed_block_scales_are_exact(moe):
    """Every block of every routed expert gets its own E8M0 scale, gate rows in
    2^[-23, 2] and the down projection in 2^[-23, 13], so one MMA meets block
    scales 2^36 apart; the output still matches the oracle."""
    cfg = synth.LayerConfig("mx_mixed", E=8, k=2, d=512, I=256, fmt="mxfp4")
    logits, x = synth.make_routing(cfg, 4, 4)
    b = Built(cfg, 4, seed=4, logits=logits, x=x)
    from expert_offload_serving_b200.layer import pack_pool
    g = torch.Generator().manual_seed(9)
    for key, hi in (("sg", 127 + 2), ("sd", 127 + 13)):
        for t in b.w_cpu[key]:
            t.copy_(torch.randint(127 - 23, hi + 1, t.shape, generator=g, dtype=torch.int64).to(t.dtype))
    b._deq.clear()
    b.layer.pool.copy_(pack_pool(cfg.E, cfg.d, cfg.I, cfg.fmt, b.w_cpu, b.order, pin=False))
    out = b.run().cpu().numpy()
    moe.moe_check_status(b.layer.status)
    check_tol(out, b.oracle()["out"], 1e-4, 1e-5)


def test_mxfp4_zero_block_with_smallest_scale_is_exact(moe):
    """A block of zero codes encoded with E8M0 byte 0 (2^-127, as MXFP4
    writers emit for all-zero blocks) is exact on the tensor-core path: no
    error is reported and the output matches the oracle."""
    cfg = synth.LayerConfig("mx_zero", E=8, k=2, d=512, I=256, fmt="mxfp4")
    logits, x = synth.make_routing(cfg, 2, 4)
    b = Built(cfg, 2, seed=4, logits=logits, x=x)
    from expert_offload_serving_b200.layer import pack_pool
    for key, sk in (("wg", "sg"), ("wd", "sd")):
        b.w_cpu[key][0][:8, :16] = 0           # 8 rows: their first 32-element block is all zeros
        b.w_cpu[sk][0][:8, 0] = 0              # with the smallest scale
    b._deq.clear()
    b.layer.pool.copy_(pack_pool(cfg.E, cfg.d, cfg.I, cfg.fmt, b.w_cpu, b.order, pin=False))
    out = b.run().cpu().numpy()
    moe.moe_check_status(b.layer.status)
    check_tol(out, b.oracle()["out"], 1e-4, 1e-5)
