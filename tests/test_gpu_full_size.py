"""GPU parity at the full configured sizes, every output row compared.

* Prefill, NVFP4 (E=256, k=6, d=4096, I=2048, T=4096): indices and
  permutation bit-exact, and all 4096 output rows against the oracle, which
  covers every expert's padded groups, every 128-row chunk and every tile of
  both GEMMs.
* Decode with the expert cache, MXFP4 (E=256, k=6, d=4096, I=2048, 64 slots,
  the 256-step AR(1) trace, T=1 and T=8): every step's fills equal the oracle
  LRU's, every step's output matches the oracle, and at the end the device
  slot table and all 64 slots' bytes equal the oracle's residency and the host
  blobs.  The routing is known in advance, so step t+1's fills are enqueued
  with no host synchronisation after step t: the fills' wait on the previous
  step's last reader of the pool and slot table is what keeps them apart.

The float64 oracle runs on a spawn pool over expert subsets
(tests.gpu_util.pooled_oracle)."""
import numpy as np
import pytest
import torch

import synth
from oracle import lru as L
from oracle import moe as M
from tests.gpu_util import Built, check_tol, load_moe, pooled_oracle, require_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def moe():
    require_gpu()
    return load_moe()


def test_prefill_full_size_every_row(moe, monkeypatch):
    """Every row at T = 4096, from the tiles the library picks there (single
    CTAs: 96 rows per expert on average) and from CTA pairs forced."""
    cfg = synth.CONFIGS["prefill_nvfp4"]
    T = 4096
    b = Built(cfg, T, seed=0, act="nvfp4")
    out = b.run().cpu().numpy()
    moe.moe_check_status(b.layer.status)
    monkeypatch.setenv("MOE_PREFILL_TILES", "pair")
    out_pair = b.run().cpu().numpy()
    moe.moe_check_status(b.layer.status)
    monkeypatch.delenv("MOE_PREFILL_TILES")
    idx, _ = M.route_topk(b.logits.numpy(), cfg.k)
    off, perm, _ = M.permute(idx, cfg.E)
    assert np.array_equal(b.layer.idx.cpu().numpy(), idx)
    assert np.array_equal(b.layer.offsets.cpu().numpy(), off)
    assert np.array_equal(b.layer.perm[: T * cfg.k].cpu().numpy(), perm)
    assert len(b.used) == cfg.E                      # every expert's groups are exercised
    ref = pooled_oracle(b.x.double().numpy(), b.logits.numpy(), cfg.k, cfg.fmt, b.w_cpu, b.pos, b.used,
                        act="nvfp4")
    for name, o in (("picked", out), ("pair", out_pair)):
        m, r = check_tol(o, ref)
        # no row is far off even if the layer as a whole is within tolerance
        row_err = np.abs(o - ref).max(axis=1) / np.abs(ref).max()
        assert row_err.max() <= 2e-2
        print(f"prefill full size, all rows ({name} tiles): max {m:.2e} mean-rel {r:.2e}")


@pytest.mark.parametrize("T", [1, 8])
def test_cached_trace_full_config(moe, T):
    from expert_offload_serving_b200.layer import MoeLayer, pack_pool
    cfg = synth.CONFIGS["decode_mxfp4"]
    w = synth.make_experts(cfg, range(cfg.E), 0, device="cuda")
    w_cpu = {k: v.cpu() for k, v in w.items()}
    del w
    host_pool = pack_pool(cfg.E, cfg.d, cfg.I, cfg.fmt, w_cpu, range(cfg.E), pin=True)
    layer = MoeLayer(cfg.E, cfg.d, cfg.I, cfg.fmt, cfg.k, T, host_pool=host_pool, n_slots=cfg.n_slots)
    trace = synth.make_trace(cfg, T, steps=cfg.steps, seed=11)
    logits_all = torch.cat([l for l, _ in trace])
    x_all = torch.cat([x for _, x in trace])
    dlog = logits_all.cuda()
    dx = x_all.cuda()
    torch.cuda.synchronize()
    lru = L.LRUCache(cfg.n_slots, cfg.E)
    outs = []
    n_fills = 0
    for t in range(cfg.steps):
        idx, _ = M.route_topk(logits_all[t * T:(t + 1) * T].numpy(), cfg.k)
        U = sorted(set(idx.ravel().tolist()))
        fills = layer.prepare(t, U)
        assert fills == lru.step(t, U)[1], f"step {t}"
        n_fills += len(fills)
        out = layer.forward(dlog[t * T:(t + 1) * T], dx[t * T:(t + 1) * T])
        outs.append(out.clone())                     # on the stream: no host synchronisation
    torch.cuda.synchronize()
    moe.moe_check_status(layer.status)
    assert layer.slot.cpu().tolist() == lru.slot_of_expert
    for s, e in enumerate(lru.expert_of_slot):
        assert e >= 0
        assert torch.equal(layer.pool[s], host_pool[e].cuda()), f"slot {s} (expert {e})"
    assert n_fills > cfg.n_slots                     # the trace evicts
    got = torch.cat(outs).cpu().numpy()
    # the oracle of all steps at once: tokens are independent, so one batch of
    # steps*T tokens gives every step's output
    used = sorted(set(M.route_topk(logits_all.numpy(), cfg.k)[0].ravel().tolist()))
    ref = pooled_oracle(x_all.double().numpy(), logits_all.numpy(), cfg.k, cfg.fmt, w_cpu,
                        {e: e for e in range(cfg.E)}, used)
    check_tol(got, ref, 1e-4, 1e-5)
    for t in range(cfg.steps):                       # and every step on its own
        check_tol(got[t * T:(t + 1) * T], ref[t * T:(t + 1) * T])
