"""moe_permute_noalloc: the permutation for callers that cannot allocate
device memory (for example inside a host engine that already reserved the
device's memory for its own pool).  It must give the same offsets, perm and
inv_perm as the oracle's stable counting sort and as moe_permute with
caller-provided scratch -- bit for bit, since they are integers -- on
consecutive calls that reuse its fixed scratch array.

This file is collected last on purpose: it must pass in a fresh process
(first call sets the array's device address up) and after every other test."""
import numpy as np
import pytest
import torch

from oracle import moe as M
from tests.gpu_util import load_moe, require_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def moe():
    require_gpu()
    return load_moe()


def _both(moe, idx_np, E):
    T, k = idx_np.shape
    idx = torch.from_numpy(idx_np).cuda()
    outs = []
    for noalloc in (False, True):
        off = torch.full((E + 1,), -7, dtype=torch.int32, device="cuda")
        perm = torch.full((T * k,), -7, dtype=torch.int32, device="cuda")
        inv = torch.full((T * k,), -7, dtype=torch.int32, device="cuda")
        st = torch.zeros(1, dtype=torch.int32, device="cuda")
        if noalloc:
            moe.moe_permute_noalloc(idx, E, off, perm, inv, dev_status=st)
        else:
            sb = moe.moe_permute_scratch_bytes(T, k, E)
            scratch = torch.empty(max(sb, 16), dtype=torch.uint8, device="cuda")
            moe.moe_permute(idx, E, off, perm, inv, scratch=scratch, dev_status=st)
        moe.moe_check_status(st)
        outs.append((off.cpu().numpy(), perm.cpu().numpy(), inv.cpu().numpy()))
    return outs


@pytest.mark.parametrize("T,k,E", [(4096, 6, 256), (3000, 8, 128)])
def test_noalloc_matches_scratch_path_twice(moe, T, k, E):
    """Two calls in a row with different routings (the second reuses the
    scratch the first left behind) equal the oracle's and moe_permute's results."""
    assert moe.moe_permute_scratch_bytes(T, k, E) > 0          # the scratch path is exercised
    for seed in (1, 2):
        rng = np.random.default_rng(seed)
        idx = np.stack([rng.choice(E, k, replace=False) for _ in range(T)]).astype(np.int32)
        if seed == 2:
            idx[: T // 3, 0] = 5                                  # a different, skewed histogram
        (a_off, a_perm, a_inv), (b_off, b_perm, b_inv) = _both(moe, idx, E)
        r_off, r_perm, r_inv = M.permute(idx, E)
        assert np.array_equal(b_off, r_off)
        assert np.array_equal(b_perm, r_perm)
        assert np.array_equal(b_inv, r_inv)
        assert np.array_equal(a_off, b_off)
        assert np.array_equal(a_perm, b_perm)
        assert np.array_equal(a_inv, b_inv)


def test_noalloc_single_tile(moe):
    rng = np.random.default_rng(3)
    idx = np.stack([rng.choice(128, 8, replace=False) for _ in range(64)]).astype(np.int32)
    (a, b) = _both(moe, idx, 128)
    for x, y, r in zip(a, b, M.permute(idx, 128)):
        assert np.array_equal(y, r)
        assert np.array_equal(x, y)


def test_noalloc_rejects_oversize(moe):
    E, k = 1024, 8
    T = moe.MOE_PERMUTE_NOALLOC_MAX_SCRATCH // (4 * E) * 1024 // k + 1024
    assert moe.moe_permute_scratch_bytes(T, k, E) > moe.MOE_PERMUTE_NOALLOC_MAX_SCRATCH
    idx = torch.zeros((T, k), dtype=torch.int32, device="cuda")
    off = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    perm = torch.empty(T * k, dtype=torch.int32, device="cuda")
    with pytest.raises(moe.MoeError) as ei:
        moe.moe_permute_noalloc(idx, E, off, perm, perm.clone())
    assert ei.value.status == moe.MOE_ERR_CAPACITY
    assert "scratch" in str(ei.value)
