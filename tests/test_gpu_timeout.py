"""The bounded-wait error path of the tensor-core kernels, made to run on
purpose without faulting anything: with moe_set_test_stall on, CTA 0 of each
tensor-core kernel waits on a barrier that nothing arrives on; with the wait
limit at 5 ms that wait runs out, the CTA records MOE_ERR_TIMEOUT, stops
issuing, drains the copies and MMAs it issued and frees its tensor memory.
The call must return promptly with MOE_ERR_TIMEOUT in the status word, and
the next normal call on the same context must match the oracle."""
import time

import pytest

import synth
from tests.gpu_util import Built, check_tol, load_moe, require_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def moe():
    require_gpu()
    return load_moe()


@pytest.mark.parametrize("fmt", ["bf16", "mxfp4", "nvfp4", "nvfp4_pair"])
def test_wait_expiry_is_reported_and_the_context_recovers(moe, monkeypatch, fmt):
    if fmt == "nvfp4_pair":                  # the CTA-pair FP4 GEMMs (the default here is single CTAs)
        monkeypatch.setenv("MOE_PREFILL_TILES", "pair")
        fmt = "nvfp4"
    act = "nvfp4" if fmt == "nvfp4" else "none"
    cfg = synth.LayerConfig("stall", E=8, k=2, d=512, I=256, fmt=fmt, act=act)
    b = Built(cfg, 16, seed=1, act=act)
    ref = b.oracle()["out"]
    check_tol(b.run().cpu().numpy(), ref)
    prev_limit = moe.moe_set_wait_limit_ns(5_000_000)
    moe.moe_set_test_stall(True)
    try:
        t0 = time.perf_counter()
        b.run()
        with pytest.raises(moe.MoeError) as ei:
            moe.moe_check_status(b.layer.status)
        assert ei.value.status == moe.MOE_ERR_TIMEOUT
        assert time.perf_counter() - t0 < 30.0
    finally:
        moe.moe_set_test_stall(False)
        moe.moe_set_wait_limit_ns(prev_limit)
    for _ in range(2):
        out = b.run().cpu().numpy()
        moe.moe_check_status(b.layer.status)
        check_tol(out, ref)
        if act == "none":
            check_tol(out, ref, 1e-4, 1e-5)
