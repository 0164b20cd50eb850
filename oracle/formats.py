"""Number formats of the expert weights and the quantised activations.

The pages name the formats only (explainx.ai hardware guide: "433GB NVFP4
routed experts"; freetoken.wiki: "NVFP4 or MXFP4 build"; fervorai.dev, "What to
know before you commit": NVFP4, MXFP4, FP8, BF16).  Their bit layouts follow
the public definitions: OCP Microscaling Formats (MX) v1.0 for E2M1 and E8M0,
and the FP8 E4M3 "fn" encoding (bias 7, no infinities, S.1111.111 = NaN).

Decoders map codes to exact float64 values from the bit fields.  Encoders
round a given fp32 value to the nearest representable value, ties to even
mantissa, and saturate to the largest finite magnitude ("satfinite").

Pins (tests/test_oracle_formats.py): every E4M3 and E8M0 code against torch's
float8_e4m3fn / float8_e8m0fnu decoders; the E4M3 encoder against torch's
round-to-nearest-even cast; both encoders against a brute-force nearest search
over every representable value and every midpoint; E2M1 against the facts the
OCP definition fixes (8 magnitudes, max 6, min subnormal 0.5).
"""
from __future__ import annotations

import numpy as np

E2M1_MAX = 6.0
E4M3_MAX = 448.0


def e2m1_decode(codes) -> np.ndarray:
    """E2M1: 1 sign bit, 2 exponent bits (bias 1), 1 mantissa bit; exponent 0
    is subnormal with value m * 2^-1."""
    c = np.asarray(codes).astype(np.int64)
    s = (c >> 3) & 1
    e = (c >> 1) & 3
    m = c & 1
    mag = np.where(e == 0, m * 0.5, (1.0 + m * 0.5) * np.exp2(e - 1.0))
    return np.where(s == 1, -mag, mag).astype(np.float64)


def e4m3_decode(codes) -> np.ndarray:
    """E4M3 (fn): 1 sign, 4 exponent bits (bias 7), 3 mantissa bits; exponent
    0 is subnormal (m/8 * 2^-6); exponent 15 with mantissa 7 is NaN."""
    c = np.asarray(codes).astype(np.int64)
    s = (c >> 7) & 1
    e = (c >> 3) & 15
    m = c & 7
    mag = np.where(e == 0, (m / 8.0) * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2(e - 7.0))
    mag = np.where((e == 15) & (m == 7), np.nan, mag)
    return np.where(s == 1, -mag, mag).astype(np.float64)


def e8m0_decode(codes) -> np.ndarray:
    """E8M0: an unsigned biased exponent, value 2^(code-127); 255 is NaN."""
    c = np.asarray(codes).astype(np.int64)
    v = np.exp2(c.astype(np.float64) - 127.0)
    return np.where(c == 255, np.nan, v)


def _rne_grid(a: np.ndarray, step: np.ndarray) -> np.ndarray:
    # a >= 0 exactly representable in float64; a/step is exact (step a power of 2)
    return np.rint(a / step) * step            # np.rint rounds half to even


def e2m1_round(v) -> np.ndarray:
    """Nearest E2M1 value to each fp32 v (ties to even mantissa, satfinite).
    Grid spacing 0.5 on [0,2), 1 on [2,4), 2 on [4,6]."""
    v = np.asarray(v, dtype=np.float32).astype(np.float64)
    a = np.abs(v)
    step = np.where(a < 2.0, 0.5, np.where(a < 4.0, 1.0, 2.0))
    q = np.minimum(_rne_grid(a, step), E2M1_MAX)
    return np.copysign(q, v)


def e2m1_encode(v) -> np.ndarray:
    """Codes 0..15 of e2m1_round(v); a value rounding to zero keeps its sign bit."""
    q = e2m1_round(v)
    a = np.abs(q)
    e = np.where(a < 1.0, 0, np.floor(np.log2(np.maximum(a, 1.0))).astype(np.int64) + 1)
    m = np.where(e == 0, (a / 0.5).astype(np.int64), ((a / np.exp2(e - 1.0) - 1.0) * 2).astype(np.int64))
    code = (e << 1) | m
    return (code | (np.signbit(q).astype(np.int64) << 3)).astype(np.uint8)


def e4m3_round(v) -> np.ndarray:
    """Nearest E4M3 value to each fp32 v (ties to even mantissa, satfinite 448).
    Normal binade [2^e, 2^(e+1)) has spacing 2^(e-3); below 2^-6 the subnormal
    spacing is 2^-9."""
    v = np.asarray(v, dtype=np.float32).astype(np.float64)
    a = np.abs(v)
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    step = np.where(a < 2.0 ** -6, 2.0 ** -9, np.exp2(e - 3.0))
    q = np.minimum(_rne_grid(a, step), E4M3_MAX)
    return np.copysign(q, v)


def e4m3_encode(v) -> np.ndarray:
    """Bytes of e4m3_round(v)."""
    q = e4m3_round(v)
    a = np.abs(q)
    sub = a < 2.0 ** -6
    e = np.floor(np.log2(np.where(sub, 1.0, a)))
    m_sub = np.rint(a / 2.0 ** -9)
    m_nrm = np.rint((a / np.exp2(e) - 1.0) * 8.0)
    exp_field = np.where(sub, 0, e + 7).astype(np.int64)
    man = np.where(sub, m_sub, m_nrm).astype(np.int64)
    return ((np.signbit(q).astype(np.int64) << 7) | (exp_field << 3) | man).astype(np.uint8)


def unpack_nibbles(packed) -> np.ndarray:
    """[..., K/2] bytes -> [..., K] codes; element 2i is the low nibble."""
    p = np.asarray(packed, dtype=np.uint8)
    out = np.empty(p.shape[:-1] + (p.shape[-1] * 2,), dtype=np.uint8)
    out[..., 0::2] = p & 0x0F
    out[..., 1::2] = p >> 4
    return out


def bf16_decode(bits) -> np.ndarray:
    """bfloat16 bit patterns (uint16) -> float64 (the upper half of an fp32)."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


def dequant_mxfp4(codes_packed, scales) -> np.ndarray:
    """MXFP4 matrix [R, K]: value = e2m1(code) * 2^(scale-127), one E8M0 scale
    per 32 consecutive K elements."""
    v = e2m1_decode(unpack_nibbles(codes_packed))
    s = e8m0_decode(scales)
    return v * np.repeat(s, 32, axis=-1)


def dequant_nvfp4(codes_packed, scales, tensor_scale) -> np.ndarray:
    """NVFP4 matrix [R, K]: value = e2m1(code) * e4m3(scale) * tensor_scale, one
    E4M3 scale per 16 consecutive K elements and one fp32 scale per matrix.
    The triple product is exact in float64 (2 + 4 + 24 significant bits)."""
    v = e2m1_decode(unpack_nibbles(codes_packed))
    s = e4m3_decode(scales)
    return v * np.repeat(s, 16, axis=-1) * np.float64(np.float32(tensor_scale))


def nvfp4_quantize_rows(v, block: int = 16):
    """Activation quantisation to NVFP4 with unit tensor scale, per `block`
    consecutive elements of the last axis (the layer's reading for FP4 x FP4
    products; the pages give no activation format):
        amax = max|v|;  s = e4m3_round(amax / 6)   [fp32 division]
        q_i  = e2m1_round(v_i / s)                 [fp32 division], 0 where s = 0
    Returns (dequantised values float64, scales float64, codes uint8)."""
    v = np.asarray(v, dtype=np.float32)
    shp = v.shape
    blk = v.reshape(shp[:-1] + (shp[-1] // block, block))
    amax = np.max(np.abs(blk), axis=-1)
    s = e4m3_round(np.float32(amax) / np.float32(6.0))
    s32 = s.astype(np.float32)
    with np.errstate(divide="ignore", invalid="ignore"):
        ratio = np.where(s32[..., None] > 0, blk / np.where(s32[..., None] > 0, s32[..., None], 1),
                         np.float32(0)).astype(np.float32)
    q = e2m1_round(ratio)
    deq = (q * s[..., None]).reshape(shp)
    return deq, s, e2m1_encode(ratio).reshape(shp)
