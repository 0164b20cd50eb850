"""Pins of oracle.formats against library decoders/encoders, brute force and
hand-worked closed forms (no GPU)."""
import numpy as np
import pytest
import torch

from oracle import formats as F


def _brute_nearest(values, grid):
    """Nearest grid value, ties to the candidate with even mantissa (given as
    a parallel array of parities), by exhaustive search."""
    grid = np.asarray(grid, dtype=np.float64)
    out = np.empty_like(values)
    for n, v in enumerate(values):
        dist = np.abs(grid[:, 0] - v)
        best = dist.min()
        cands = grid[dist == best]
        if len(cands) > 1:
            cands = cands[cands[:, 1] == 0]
        out[n] = cands[0, 0]
    return out


def test_e4m3_decode_matches_torch_all_codes():
    codes = np.arange(256, dtype=np.uint8)
    ours = F.e4m3_decode(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(np.isnan(ours), np.isnan(ref))
    ok = ~np.isnan(ref)
    assert np.array_equal(ours[ok], ref[ok])
    assert np.array_equal(np.signbit(ours[ok]), np.signbit(ref[ok]))


def test_e8m0_decode_matches_torch_all_codes():
    codes = np.arange(256, dtype=np.uint8)
    ours = F.e8m0_decode(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e8m0fnu).to(torch.float64).numpy()
    assert np.array_equal(np.isnan(ours), np.isnan(ref))
    ok = ~np.isnan(ref)
    assert np.array_equal(ours[ok], ref[ok])


def test_e2m1_table_facts():
    v = F.e2m1_decode(np.arange(16))
    # OCP MX v1.0 FP4 E2M1: 8 magnitudes, max normal 6, min normal 1, min subnormal 0.5
    assert list(v[:8]) == [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    assert np.array_equal(v[8:], -v[:8])
    assert np.signbit(v[8])
    # every E2M1 value is an E4M3 value: re-encode the fields and decode with torch
    for c in range(16):
        s, e, m = c >> 3, (c >> 1) & 3, c & 1
        if e == 0 and m == 0:
            b = s << 7
        elif e == 0:
            b = (s << 7) | ((-1 + 7) << 3)            # 0.5 = 2^-1
        else:
            b = (s << 7) | ((e - 1 + 7) << 3) | (m << 2)
        ref = torch.tensor([b], dtype=torch.uint8).view(torch.float8_e4m3fn).double().item()
        assert ref == v[c]


def _e2m1_grid():
    mags = F.e2m1_decode(np.arange(8))
    par = np.arange(8) & 1
    return np.stack([np.concatenate([mags, -mags]), np.concatenate([par, par])], axis=1)


def test_e2m1_round_vs_brute_force():
    mags = F.e2m1_decode(np.arange(8))
    mids = (mags[1:] + mags[:-1]) / 2
    rng = np.random.default_rng(1)
    vals = np.concatenate([mags, mids, mids + 1e-6, mids - 1e-6, [6.5, 7.0, 100.0, 1e30],
                           rng.uniform(-8, 8, 2000).astype(np.float32)])
    vals = np.concatenate([vals, -vals]).astype(np.float32).astype(np.float64)
    ours = F.e2m1_round(vals)
    clipped = np.clip(vals, -6, 6)
    ref = _brute_nearest(clipped, _e2m1_grid())
    assert np.array_equal(ours, ref)


def test_e2m1_encode_roundtrip():
    v = F.e2m1_decode(np.arange(16))
    codes = F.e2m1_encode(v)
    assert np.array_equal(codes, np.arange(16, dtype=np.uint8))


def test_e4m3_round_vs_torch_and_brute_force():
    rng = np.random.default_rng(2)
    finite = np.arange(256, dtype=np.uint8)
    dec = F.e4m3_decode(finite)
    ok = ~np.isnan(dec)
    grid_vals = dec[ok]
    pos = np.unique(grid_vals[grid_vals >= 0])
    mids = (pos[1:] + pos[:-1]) / 2
    vals = np.concatenate([pos, mids, rng.uniform(-448, 448, 5000),
                           rng.standard_normal(3000) * 0.01, rng.standard_normal(2000) * 1e-3])
    vals = np.concatenate([vals, -vals]).astype(np.float32)
    ours = F.e4m3_round(vals)
    ref = torch.from_numpy(vals).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(ours, ref)
    # brute force on the midpoints and a sample
    mant_par = (finite[ok] & 1).astype(np.float64)
    grid = np.stack([grid_vals, mant_par], axis=1)
    sub = np.concatenate([mids[:40], mids[-40:], vals[:200]]).astype(np.float32).astype(np.float64)
    assert np.array_equal(F.e4m3_round(sub), _brute_nearest(sub, grid))


def test_e4m3_saturates():
    v = np.array([448.0, 449.0, 464.0, 480.0, 1e9, -1e9], dtype=np.float32)
    assert list(F.e4m3_round(v)) == [448.0, 448.0, 448.0, 448.0, 448.0, -448.0]


def test_e4m3_encode_roundtrip_all_finite():
    codes = np.arange(256, dtype=np.uint8)
    dec = F.e4m3_decode(codes)
    ok = ~np.isnan(dec)
    assert np.array_equal(F.e4m3_encode(dec[ok]), codes[ok])


def test_nvfp4_block_hand_worked():
    # amax = 12 -> s = e4m3(12/6) = 2 exactly; ratios v/s chosen to hit ties
    v = np.array([12, -6, 3, 1, 5, 7, 0.5, -0.4, 9, 10, 11, 2, 4, -8, 0, 1.5], dtype=np.float32)
    deq, s, codes = F.nvfp4_quantize_rows(v[None, :])
    assert s.tolist() == [[2.0]]
    # ratios: 6,-3,1.5,.5,2.5,3.5,.25,-.2,4.5,5,5.5,1,2,-4,0,.75 -> RNE on the E2M1 grid
    expect_q = [6, -3, 1.5, 0.5, 2, 4, 0, -0.0, 4, 4, 6, 1, 2, -4, 0, 1]
    assert deq[0].tolist() == [2.0 * q for q in expect_q]


def test_nvfp4_scale_rounding_hand_worked():
    # amax = 7 -> 7/6 = 1.1666.. in fp32 -> E4M3 spacing 1/8 on [1,2): 1.125
    v = np.zeros((1, 16), dtype=np.float32)
    v[0, 0] = 7.0
    v[0, 1] = -3.0
    deq, s, _ = F.nvfp4_quantize_rows(v)
    assert s[0, 0] == 1.125
    # 7/1.125 = 6.22 -> 6 ; -3/1.125 = -2.67 -> -3
    assert deq[0, 0] == 6 * 1.125 and deq[0, 1] == -3 * 1.125


def test_mxfp4_dequant_closed_form():
    # one row, 64 elements: block 0 scale 2^-3, block 1 scale 2^2
    codes = np.arange(64) % 16
    packed = (codes[0::2] | (codes[1::2] << 4)).astype(np.uint8)[None, :]
    scales = np.array([[127 - 3, 127 + 2]], dtype=np.uint8)
    w = F.dequant_mxfp4(packed, scales)
    base = F.e2m1_decode(codes)
    assert np.array_equal(w[0, :32], base[:32] / 8.0)
    assert np.array_equal(w[0, 32:], base[32:] * 4.0)


def test_nvfp4_dequant_closed_form():
    codes = np.arange(32) % 16
    packed = (codes[0::2] | (codes[1::2] << 4)).astype(np.uint8)[None, :]
    scales = F.e4m3_encode(np.array([[0.75, 3.5]]))
    w = F.dequant_nvfp4(packed, scales, np.float32(0.01))
    base = F.e2m1_decode(codes)
    g = float(np.float32(0.01))
    assert np.array_equal(w[0, :16], base[:16] * 0.75 * g)
    assert np.array_equal(w[0, 16:], base[16:] * 3.5 * g)


def test_bf16_decode():
    x = torch.tensor([1.0, -2.5, 3.140625, 0.0, -0.0, 1e-3]).to(torch.bfloat16)
    bits = x.view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(F.bf16_decode(bits), x.double().numpy())
