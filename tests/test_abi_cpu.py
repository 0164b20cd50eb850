"""The C ABI on the CPU: the library loads and exports every declared symbol,
host-only calls work, arguments are rejected before any CUDA call, and the
cache's host bookkeeping makes the oracle's LRU decisions (no GPU needed)."""
import ctypes
import json
import os
import re

import numpy as np
import pytest
import torch

import synth
from oracle import formats as F
from oracle import lru as L

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def moe():
    from expert_offload_serving_b200 import build
    build.build()
    import expert_offload_serving_b200 as m
    m.lib()
    return m


def header_functions():
    text = open(os.path.join(ROOT, "include", "moe.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z_0-9]+)\s*\(", text)))


def test_every_declared_symbol_is_exported_and_bound(moe):
    names = header_functions()
    assert len(names) >= 15
    L_ = moe.lib()
    for n in names:
        assert hasattr(L_, n), n
    assert sorted(moe.declared_symbols()) == names


def test_abi_version(moe):
    assert moe.moe_abi_version() == 1


@pytest.mark.parametrize("name,expect", [
    ("decode_bf16", 3 * 2048 * 768 * 2),
    ("decode_mxfp4", 3 * 4096 * 2048 // 2 + 3 * 4096 * 2048 // 32),
    ("prefill_nvfp4", 3 * 4096 * 2048 // 2 + 3 * 4096 * 2048 // 16 + 256),
])
def test_blob_bytes(moe, name, expect):
    c = synth.CONFIGS[name]
    assert moe.moe_expert_blob_bytes(moe.shape(c.E, c.d, c.I, c.fmt)) == expect


@pytest.mark.parametrize("E,d,I,fmt", [(0, 64, 64, "bf16"), (2000, 64, 64, "bf16"), (4, 60, 64, "bf16"),
                                       (4, 48, 64, "mxfp4"), (4, 64, 64, "nvfp4"), (4, 64, 64, 7)])
def test_invalid_shapes_have_no_blob(moe, E, d, I, fmt):
    assert moe.moe_expert_blob_bytes(moe.shape(E, d, I, fmt)) == 0


def _host_ptr(a):
    return a.ctypes.data


def test_argument_errors_before_any_cuda_call(moe):
    """Every check runs before the first CUDA call: on a machine without a GPU
    each bad call returns MOE_ERR_INVALID_ARG (never MOE_ERR_CUDA).  The buffer
    is 256-byte aligned so that only the intended argument is wrong."""
    L_ = moe.lib()
    raw = np.zeros(2048, dtype=np.float32)
    shift = (-_host_ptr(raw)) % 256 // 4
    buf = raw[shift: shift + 1024]
    p = _host_ptr(buf)
    assert p % 256 == 0
    assert L_.moe_route_topk(p, 4, 8, 9, p, p, None) == moe.MOE_ERR_INVALID_ARG      # k > E
    assert L_.moe_route_topk(p, 4, 2000, 2, p, p, None) == moe.MOE_ERR_INVALID_ARG   # E > 1024
    assert L_.moe_route_topk(p, 4, 64, 33, p, p, None) == moe.MOE_ERR_INVALID_ARG    # k > 32
    assert L_.moe_route_topk(None, 4, 8, 2, p, p, None) == moe.MOE_ERR_INVALID_ARG   # null
    assert b"k=" in L_.moe_last_error() or b"null" in L_.moe_last_error()
    assert L_.moe_permute(p, 4, 2, 0, p, p, p, None, 0, None, None) == moe.MOE_ERR_INVALID_ARG
    s_bad = moe.shape(8, 60, 64, "bf16")
    assert L_.moe_expert_ffn(s_bad, p, 4, 2, p, p, p, p, 8, p, p, None, 0, p, 1 << 20, None,
                             None) == moe.MOE_ERR_INVALID_ARG
    s = moe.shape(8, 64, 64, "bf16")
    assert L_.moe_expert_ffn(s, p, 4, 2, p, p, p, p, 8, p, None, None, 0, p, 1 << 20, None,
                             None) == moe.MOE_ERR_INVALID_ARG                          # no output
    assert L_.moe_expert_ffn(s, p + 4, 4, 2, p, p, p, p, 8, p, p, None, 0, p, 1 << 20, None,
                             None) == moe.MOE_ERR_INVALID_ARG                          # misaligned x
    assert L_.moe_expert_ffn(s, p, 4, 2, p, p, p, p, 8, p, p, None, 1, p, 1 << 20, None,
                             None) == moe.MOE_ERR_INVALID_ARG                          # act flag, bf16
    assert b"NVFP4" in L_.moe_last_error()
    s_nv = moe.shape(8, 384, 256, "nvfp4")
    assert L_.moe_expert_ffn(s_nv, p, 4, 2, p, p, p, p, 8, p, None, p, 1, p, 1 << 30, None,
                             None) == moe.MOE_ERR_INVALID_ARG                          # d % 256 != 0
    assert L_.moe_expert_ffn(s, p, 4, 2, p, p, p, p, 8, p, p, None, 0, p, 16, None,
                             None) == moe.MOE_ERR_CAPACITY                             # workspace too small
    assert L_.moe_combine_merge(p, p, p, p, None, None, 4, 2, 6, 8, p, None) == moe.MOE_ERR_INVALID_ARG
    assert L_.moe_cache_fill(None, None, 0, 0, None, 0, None, None, None, None, None) == \
        moe.MOE_ERR_INVALID_ARG


def _aligned_host_buffer(n_floats=1 << 16):
    raw = np.zeros(n_floats + 64, dtype=np.float32)
    shift = (-_host_ptr(raw)) % 256 // 4
    buf = raw[shift: shift + n_floats]
    assert _host_ptr(buf) % 256 == 0
    return buf


def _forward(moe, s, p, T, k, flags=0, scratch_bytes=1 << 20, out=None, y_perm=None):
    out = p if out is None else out
    y_perm = p if y_perm is None else y_perm
    return moe.lib().moe_layer_forward(s, p, p, T, k, p, p, p, p, p, p, scratch_bytes, p, p, 8,
                                       None if flags else y_perm, flags, p, 1 << 30, None, out, None, None)


def test_layer_forward_checks_every_step_before_enqueueing(moe):
    """moe_layer_forward rejects a bad argument of any of its four steps before
    the first step is enqueued: no CUDA call happens, so on any machine the
    status is the argument error itself, never MOE_ERR_CUDA."""
    buf = _aligned_host_buffer()
    p = _host_ptr(buf)
    bf16 = moe.shape(8, 256, 256, "bf16")
    assert _forward(moe, moe.shape(8, 60, 64, "bf16"), p, 4, 2) == moe.MOE_ERR_INVALID_ARG     # FFN shape
    assert _forward(moe, bf16, p, 4, 9) == moe.MOE_ERR_INVALID_ARG                             # route: k > E
    assert _forward(moe, bf16, p, 4, 2, out=p + 4) == moe.MOE_ERR_INVALID_ARG                  # combine: out
    assert b"16-byte" in moe.lib().moe_last_error()
    assert _forward(moe, bf16, p, 4, 2, y_perm=p + 4) == moe.MOE_ERR_INVALID_ARG               # FFN: y_perm
    assert _forward(moe, bf16, p, 4, 2, flags=1) == moe.MOE_ERR_INVALID_ARG                    # act flag, bf16
    assert b"NVFP4" in moe.lib().moe_last_error()
    big = moe.shape(256, 256, 256, "bf16")
    assert _forward(moe, big, p, 4096, 6, scratch_bytes=16) == moe.MOE_ERR_CAPACITY            # permute scratch


@pytest.mark.skipif(torch.cuda.is_available(), reason="valid calls would launch on host pointers")
def test_valid_arguments_pass_every_check(moe):
    """The converse: arguments that are valid pass every check and reach the
    device query, which is what fails on a host without a GPU (MOE_ERR_CUDA)."""
    L_ = moe.lib()
    buf = _aligned_host_buffer()
    p = _host_ptr(buf)
    s = moe.shape(8, 256, 256, "bf16")

    def reached_device(st):
        return st == moe.MOE_ERR_CUDA and b"cudaGetDevice" in L_.moe_last_error()

    assert reached_device(L_.moe_route_topk(p, 4, 8, 2, p, p, None))
    assert reached_device(L_.moe_permute(p, 4, 2, 8, p, p, p, None, 0, None, None))
    need = moe.moe_permute_scratch_bytes(4096, 6, 256)
    assert need > 0
    assert reached_device(L_.moe_permute(p, 4096, 6, 256, p, p, p, p, need, None, None))
    assert reached_device(L_.moe_expert_ffn(s, p, 4, 2, p, p, p, p, 8, p, p, None, 0, p, 1 << 20, None, None))
    assert reached_device(L_.moe_combine_merge(p, p, p, p, p, None, 4, 2, 256, 8, p, None))
    assert reached_device(_forward(moe, s, p, 4, 2))
    assert reached_device(_forward(moe, moe.shape(8, 256, 256, "nvfp4"), p, 4, 2, flags=1))


def test_workspace_and_scratch_sizes(moe):
    s = moe.shape(128, 2048, 768, "bf16")
    assert moe.moe_expert_ffn_workspace_bytes(s, 64, 8) >= 64 * 8 * 768 * 4
    assert moe.moe_permute_scratch_bytes(64, 8, 128) == 0           # one tile
    assert moe.moe_permute_scratch_bytes(4096, 6, 256) == 24 * 256 * 4


def test_workspace_never_shrinks_with_T(moe):
    """A layer sizes its FFN workspace once, for its largest step, and runs
    smaller steps on it; so the size must not decrease with T for any path,
    including across the FP4 prefill's switch from single-CTA tiles to CTA
    pairs at T*k = 128*E (where the tile family, and its layout, changes)."""
    cases = [(moe.shape(128, 2048, 768, "bf16"), 8, 0), (moe.shape(256, 4096, 2048, "mxfp4"), 6, 0),
             (moe.shape(256, 4096, 2048, "nvfp4"), 6, 0), (moe.shape(256, 4096, 2048, "nvfp4"), 6, 1),
             (moe.shape(16, 1024, 512, "nvfp4"), 4, 1)]
    for s, k, flags in cases:
        switch = 128 * s.E // k
        Ts = sorted(set(list(range(1, 70)) + list(range(switch - 40, switch + 40)) + list(range(1, 40000, 331))))
        sizes = [moe.moe_expert_ffn_workspace_bytes(s, T, k, flags) for T in Ts]
        assert all(a <= b for a, b in zip(sizes, sizes[1:])), (s.fmt, flags)
        assert sizes[0] > 0


def test_ffn_launch_count(moe):
    """moe_expert_ffn_launches reports the kernels an FFN call launches: the
    decode schedule (one cooperative GEMV launch only for single-token MXFP4
    steps, unless MOE_DECODE_SCHEDULE fixes it), the MXFP4 split of x, the
    CUDA-core pair, the four prefill kernels; 0 for invalid arguments."""
    import os
    if os.environ.get("MOE_DECODE_SCHEDULE"):
        pytest.skip("the schedule is fixed by the environment")
    bf16 = moe.shape(128, 2048, 768, "bf16")
    mx = moe.shape(256, 4096, 2048, "mxfp4")
    assert moe.moe_expert_ffn_launches(bf16, 64, 8) == 2           # gate/up + down
    assert moe.moe_expert_ffn_launches(bf16, 1, 8) == 2
    assert moe.moe_expert_ffn_launches(mx, 8, 6) == 3              # split of x + gate/up + down
    assert moe.moe_expert_ffn_launches(mx, 1, 6) == 2              # split of x + one cooperative launch
    assert moe.moe_expert_ffn_launches(moe.shape(12, 264, 136, "bf16"), 9, 3) == 2   # CUDA cores
    assert moe.moe_expert_ffn_launches(moe.shape(256, 4096, 2048, "nvfp4"), 4096, 6, moe.MOE_FFN_ACT_NVFP4) == 4
    assert moe.moe_expert_ffn_launches(bf16, 0, 8) == 0
    assert moe.moe_expert_ffn_launches(bf16, 4, 0) == 0


def _canonical(name, E=3):
    base = synth.CONFIGS[name]
    cfg = synth.LayerConfig(name, E=E, k=2, d=256, I=128, fmt=base.fmt)
    return cfg, synth.make_experts(cfg, range(E), seed=3)


def test_pack_bf16_tile_layout(moe):
    """bf16 blobs with d, I multiples of 256 hold W_gu (gate and up rows
    interleaved in blocks of 64: row 128b + j = gate row 64b + j, row
    128b + 64 + j = up row 64b + j) in the wg + wu regions and W_d in the wd
    region, each as tiles of 128 rows x 64 elements (16 KB) ordered
    [row / 128][k / 64]; in a tile, row r is a 128-byte line whose 16-byte
    chunk c sits at chunk position c ^ (r % 8)."""
    from expert_offload_serving_b200.layer import pack_pool
    cfg = synth.LayerConfig("blk", E=2, k=1, d=512, I=256, fmt="bf16")
    w = synth.make_experts(cfg, range(2), seed=4)
    pool = pack_pool(cfg.E, cfg.d, cfg.I, cfg.fmt, w, range(2), pin=False).numpy()
    m = cfg.I * cfg.d

    def unpack(region, R, K):
        words = region.view(np.uint16)
        out = np.empty((R, K), dtype=np.uint16)
        k = np.arange(K)
        for r in range(R):
            tile = (r // 128) * (K // 64) + k // 64
            rr = r % 128
            pos = tile * 16384 + rr * 128 + (((k // 8) % 8) ^ (rr % 8)) * 16 + (k % 8) * 2
            out[r] = words[pos // 2]
        return out

    for e in range(2):
        b = pool[e]
        src = {key: w[key][e].contiguous().view(torch.int16).numpy().view(np.uint16) for key in ("wg", "wu", "wd")}
        gu = unpack(b[:2 * 2 * m], 2 * cfg.I, cfg.d)
        for i in range(cfg.I):
            assert np.array_equal(gu[(i // 64) * 128 + i % 64], src["wg"][i])
            assert np.array_equal(gu[(i // 64) * 128 + 64 + i % 64], src["wu"][i])
        assert np.array_equal(unpack(b[2 * 2 * m:3 * 2 * m], cfg.d, cfg.I), src["wd"])


def test_pack_mxfp4_tiled_layout(moe):
    """MXFP4 blobs with d, I multiples of 256 hold W_gu (gate and up rows
    interleaved in blocks of 64) and then W_d as tiles of 128 rows x 256
    elements ordered [row / 128][k / 256], 17408 bytes each: the codes (row r
    = the 128 bytes at 128 r, unswizzled), then the E8M0 scales as two
    tensor-core scale-factor atoms (32-element block j of the tile in atom
    j // 4; row r at (r % 32) * 16 + (r // 32) * 4 + j % 4)."""
    from expert_offload_serving_b200.layer import pack_pool
    cfg = synth.LayerConfig("mxt", E=1, k=1, d=512, I=256, fmt="mxfp4")
    w = synth.make_experts(cfg, range(1), seed=6)
    blob = pack_pool(cfg.E, cfg.d, cfg.I, cfg.fmt, w, range(1), pin=False).numpy()[0]
    tile_bytes = 128 * 128 + 128 * 8

    def unpack(region, R, K):
        codes = np.empty((R, K // 2), dtype=np.uint8)
        scales = np.empty((R, K // 32), dtype=np.uint8)
        b = np.arange(K // 2)
        jj = np.arange(K // 32)
        for r in range(R):
            rr = r % 128
            tile = (r // 128) * (K // 256) + b // 128
            codes[r] = region[tile * tile_bytes + rr * 128 + b % 128]
            stile = (r // 128) * (K // 256) + jj // 8
            j8 = jj % 8
            scales[r] = region[stile * tile_bytes + 16384 + (j8 // 4) * 512 + (rr % 32) * 16 + (rr // 32) * 4 + j8 % 4]
        return codes, scales

    gu_bytes = 2 * cfg.I * (cfg.d // 2 + cfg.d // 32)
    gc, gs = unpack(blob[:gu_bytes], 2 * cfg.I, cfg.d)
    for i in range(cfg.I):
        rg, ru = (i // 64) * 128 + i % 64, (i // 64) * 128 + 64 + i % 64
        assert np.array_equal(gc[rg], w["wg"][0][i].numpy()) and np.array_equal(gs[rg], w["sg"][0][i].numpy())
        assert np.array_equal(gc[ru], w["wu"][0][i].numpy()) and np.array_equal(gs[ru], w["su"][0][i].numpy())
    dc, ds = unpack(blob[gu_bytes:], cfg.d, cfg.I)
    assert np.array_equal(dc, w["wd"][0].numpy()) and np.array_equal(ds, w["sd"][0].numpy())


@pytest.mark.parametrize("name", ["tiny", "decode_mxfp4", "prefill_nvfp4"])
def test_pack_expert_layout(moe, name):
    """Blob regions hold the canonical tensors (NVFP4: gate/up rows interleaved
    in blocks of 64, scales in the MMA atom layout: row r, block b at
    ((r/128)*(K/64) + b/4)*512 + (r%32)*16 + ((r/32)%4)*4 + b%4)."""
    from expert_offload_serving_b200.layer import pack_pool
    cfg, w = _canonical(name)
    pool = pack_pool(cfg.E, cfg.d, cfg.I, cfg.fmt, w, range(cfg.E), pin=False).numpy()
    m = cfg.I * cfg.d
    for e in range(cfg.E):
        b = pool[e]
        if cfg.fmt == "bf16":
            for n, key in enumerate(("wg", "wu", "wd")):
                ref = w[key][e].contiguous().view(torch.uint8).numpy().ravel()
                assert np.array_equal(b[n * 2 * m:(n + 1) * 2 * m], ref)
            continue
        if cfg.fmt == "mxfp4":
            for n, key in enumerate(("wg", "wu", "wd")):
                assert np.array_equal(b[n * m // 2:(n + 1) * m // 2], w[key][e].numpy().ravel())
            base = 3 * m // 2
            for n, key in enumerate(("sg", "su", "sd")):
                assert np.array_equal(b[base + n * m // 32: base + (n + 1) * m // 32], w[key][e].numpy().ravel())
            continue
        # NVFP4: W_gu interleaves gate and up rows in blocks of 64
        rb = cfg.d // 2
        gu = b[:m].reshape(2 * cfg.I, rb)
        i = np.arange(cfg.I)
        rg = (i // 64) * 128 + i % 64
        assert np.array_equal(gu[rg], w["wg"][e].numpy())
        assert np.array_equal(gu[rg + 64], w["wu"][e].numpy())
        assert np.array_equal(b[m:m + m // 2], w["wd"][e].numpy().ravel())

        def atoms(reg, R, K):
            rr, bb = np.meshgrid(np.arange(R), np.arange(K // 16), indexing="ij")
            off = ((rr // 128) * (K // 64) + bb // 4) * 512 + (rr % 32) * 16 + ((rr // 32) % 4) * 4 + bb % 4
            return reg[off]
        sgu = atoms(b[3 * m // 2: 3 * m // 2 + m // 8], 2 * cfg.I, cfg.d)
        assert np.array_equal(sgu[rg], w["sg"][e].numpy())
        assert np.array_equal(sgu[rg + 64], w["su"][e].numpy())
        base = 3 * m // 2 + m // 8
        assert np.array_equal(atoms(b[base: base + m // 16], cfg.d, cfg.I), w["sd"][e].numpy())
        ts = b[base + m // 16: base + m // 16 + 12].view(np.float32)
        assert np.array_equal(ts, w["ts"][e].numpy())


def test_cache_planner_matches_oracle_lru(moe):
    """A plan-only cache handle makes exactly the oracle's LRU decisions on a
    drifting-bias routing trace, including protected host-computed experts."""
    cfg = synth.CONFIGS["decode_mxfp4"]
    trace = synth.make_trace(cfg, 8, steps=60, seed=1)
    s = moe.shape(cfg.E, cfg.d, cfg.I, cfg.fmt)
    c = moe.MoeCache(s, cfg.n_slots)
    ref = L.LRUCache(cfg.n_slots, cfg.E)
    from oracle import moe as M
    rng = np.random.default_rng(0)
    total_fills = 0
    for t, (logits, _) in enumerate(trace):
        idx, _ = M.route_topk(logits.numpy(), cfg.k)
        U = sorted(set(idx.ravel().tolist()))
        host = set(rng.choice(U, len(U) // 4, replace=False).tolist())
        gpu = [e for e in U if e not in host or ref.resident(e)]
        got = c.fill(gpu, t, protect=U)
        hits, fills = ref.step(t, gpu, protect=U)
        assert got == fills
        total_fills += len(fills)
        soe, eos, lu = c.query()
        assert soe == ref.slot_of_expert and eos == ref.expert_of_slot and lu == ref.last_used
    assert total_fills > cfg.n_slots            # the trace evicts


def test_layered_cache_planner_and_resize_match_oracle(moe):
    """A plan-only cache shared by 4 layers makes the oracle's decisions over
    keys l*E + e (clock = step * L + layer), and resizes (shrink, grow,
    shrink) keep the same residents in the same slots as the oracle's."""
    from oracle import moe as M
    cfg = synth.CONFIGS["decode_mxfp4"]
    Lyr, S = 4, 48
    s = moe.shape(cfg.E, cfg.d, cfg.I, cfg.fmt)
    c = moe.MoeCache(s, S, n_layers=Lyr)
    ref = L.LRUCache(S, Lyr * cfg.E)
    traces = [synth.make_trace(cfg, 4, steps=40, seed=10 + l) for l in range(Lyr)]
    sizes = {12: 24, 22: 60, 31: 30}
    for t in range(40):
        if t in sizes:
            assert c.resize(sizes[t]) == ref.resize(sizes[t])
        for l in range(Lyr):
            idx, _ = M.route_topk(traces[l][t][0].numpy(), cfg.k)
            U = sorted(set(idx.ravel().tolist()))
            clock = t * Lyr + l
            got = c.fill(U, clock, protect=U, layer=l)
            hits, fills = ref.step(clock, [l * cfg.E + e for e in U])
            assert got == [(key - l * cfg.E, slot, old) for key, slot, old in fills]
        soe, eos, lu = c.query()
        assert soe == ref.slot_of_expert and eos == ref.expert_of_slot and lu == ref.last_used


def test_cache_capacity_error_leaves_state(moe):
    s = moe.shape(16, 64, 64, "bf16")
    c = moe.MoeCache(s, 2)
    c.fill([1, 2], 0)
    before = c.query()
    with pytest.raises(moe.MoeError) as ei:
        c.fill([3, 4, 5], 1)
    assert ei.value.status == moe.MOE_ERR_CAPACITY
    assert c.query() == before


@pytest.mark.skipif(torch.cuda.is_available(), reason="the copies would run")
def test_cache_failed_fill_makes_the_cache_unusable(moe):
    """A fill whose copies cannot be enqueued (here: no GPU) fails with
    MOE_ERR_CUDA and leaves the host bookkeeping as it was; every later fill
    fails the same way until the cache is recreated, since a copy may already
    have reached a victim slot whose table entry was never rewritten."""
    buf = _aligned_host_buffer()             # stands in for the pools; never touched
    p = _host_ptr(buf)
    s = moe.shape(16, 64, 64, "bf16")
    c = moe.MoeCache(s, 2, slot_pool=p, host_pool=p, slot_of_expert_dev=p)
    before = c.query()
    with pytest.raises(moe.MoeError) as ei:
        c.fill([1, 2], 0)
    assert ei.value.status == moe.MOE_ERR_CUDA
    assert c.query() == before
    with pytest.raises(moe.MoeError) as ei:
        c.fill([3], 1)
    assert ei.value.status == moe.MOE_ERR_CUDA
    assert b"recreate" in moe.lib().moe_last_error()
    planner = moe.MoeCache(s, 2)             # a plan-only handle enqueues nothing and is unaffected
    assert planner.fill([1, 2], 0) == [(1, 0, -1), (2, 1, -1)]


def test_layer_rejects_inputs_its_buffers_cannot_hold(moe):
    """The C calls see plain pointers, so MoeLayer checks the sizes of its own
    buffers (T_max tokens) and the input tensors before any call: a batch
    larger than T_max, or logits / x / host_partial of the wrong shape or type,
    raise ValueError instead of letting a kernel write past a buffer."""
    from expert_offload_serving_b200.layer import MoeLayer
    E, d, I, k, T_max = 8, 256, 256, 2, 4
    B = moe.moe_expert_blob_bytes(moe.shape(E, d, I, "bf16"))
    layer = MoeLayer(E, d, I, "bf16", k, T_max, device="cpu", device_pool=torch.zeros((E, B), dtype=torch.uint8))
    logits = torch.zeros((T_max + 1, E), dtype=torch.float32)
    x = torch.zeros((T_max + 1, d), dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="T_max"):
        layer.forward(logits, x)
    with pytest.raises(ValueError, match="T_max"):
        layer.route(logits)
    with pytest.raises(ValueError, match="T_max"):
        layer.permute(T_max + 1)
    with pytest.raises(ValueError, match="logits"):
        layer.forward(logits[:2].double(), x[:2])
    with pytest.raises(ValueError, match="x:"):
        layer.forward(logits[:2], x[:2].float())
    with pytest.raises(ValueError, match="x:"):
        layer.forward(logits[:2], torch.zeros((2, 2 * d), dtype=torch.bfloat16)[:, ::2])
    with pytest.raises(ValueError, match="host_partial"):
        layer.forward(logits[:2], x[:2], host_partial=torch.zeros((2, d), dtype=torch.float64))


def test_bindings_check_buffers_before_the_call(moe):
    """The bindings marshal tensors into plain pointers, so they first check
    that each device buffer is a contiguous CUDA tensor of the documented
    dtype large enough for the call: a host tensor or a short buffer raises
    ValueError instead of reaching a kernel."""
    idx = torch.zeros((4, 2), dtype=torch.int32)
    with pytest.raises(ValueError, match="logits: expected a contiguous CUDA"):
        moe.moe_route_topk(torch.zeros((4, 8)), 2, idx, torch.zeros((4, 2)))
    with pytest.raises(ValueError, match="idx: expected a contiguous CUDA"):
        moe.moe_permute(idx, 8, torch.zeros(9, dtype=torch.int32), idx.view(-1), idx.view(-1))
    s = moe.shape(8, 256, 256, "bf16")
    with pytest.raises(ValueError, match="x: expected"):
        moe.moe_expert_ffn(s, torch.zeros((4, 256)), 2, None, None, None, None, 8)
    if torch.cuda.is_available():
        short = torch.zeros(7, dtype=torch.int32, device="cuda")
        with pytest.raises(ValueError, match="holds 7 elements"):
            moe.moe_route_topk(torch.zeros((4, 8), device="cuda"), 2, short,
                               torch.zeros((4, 2), device="cuda"))


def test_split_misses_matches_oracle(moe, golden_dir):
    """moe_split_misses (host only) makes the oracle's choices: for q in
    [0, 1] the floor(q*m + 0.5) misses with the most routed tokens, ties to
    the lower id; for q* the oracle's count at the bandwidths the pages print
    for their workstation (pinned host memory and PCIe)."""
    fig = json.load(open(os.path.join(golden_dir, "pages_figures.json")))["glm_workstation_bandwidth"]
    bw_pcie, bw_host = fig["pcie_gbs"], fig["host_gbs"]
    rng = np.random.default_rng(5)
    for trial in range(300):
        E = int(rng.integers(1, 300))
        m = int(rng.integers(0, min(E, 40) + 1))
        misses = rng.choice(E, m, replace=False).tolist()
        tok = rng.integers(0, 4, E).tolist()           # small counts: many ties
        for q in (0.0, 0.3, 0.5, 1.0, float(rng.uniform())):
            assert moe.moe_split_misses(misses, tok, q) == L.split_misses(misses, tok, q)
        n = L.q_star(m, bw_pcie, bw_host)
        filled, host = moe.moe_split_misses(misses, tok, None, bw_pcie, bw_host)
        assert len(filled) == n and len(filled) + len(host) == m
        if m:
            assert (filled, host) == L.split_misses(misses, tok, n / m)
    for bad in (dict(misses=[1, 1], q=0.5), dict(misses=[300], q=0.5), dict(misses=[1], q=1.5),
                dict(misses=[1], q=None)):
        with pytest.raises(moe.MoeError) as ei:
            moe.moe_split_misses(bad["misses"], [1] * 16, bad["q"])
        assert ei.value.status == moe.MOE_ERR_INVALID_ARG
