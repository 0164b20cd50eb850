"""Seeded synthetic inputs for the routed-expert MoE layer.

This module only draws random numbers and writes them in the canonical
(unpacked) storage formats; it holds none of the layer's arithmetic.  Both the
CUDA path (tests, bench) and the CPU oracle consume what it returns.

Workload shapes follow the FreeToken write-ups: DeepSeek-V4-Flash routes each
token through 6 of 256 experts (freetoken.wiki "FreeToken 753b model",
"FreeToken 753b Model Explained"; ainewsfeed.tech, second paragraph), the
formats are BF16, MXFP4 and NVFP4 (explainx.ai hardware guide, GLM-5.2 setup
table; fervorai.dev, "What to know before you commit").  The per-config sizes
(d, I, T, slot count, trace length, weight and bias spreads) are the build's
configuration, listed in ``CONFIGS``.

Canonical storage:
  * BF16   -- ``wg``/``wu`` [E, I, d] and ``wd`` [E, d, I] as ``torch.bfloat16``.
  * MXFP4  -- codes [E, R, K/2] uint8 (element 2i in the low nibble, 2i+1 in the
              high nibble), E8M0 scale bytes [E, R, K/32] uint8.
  * NVFP4  -- codes as above, E4M3 scale bytes [E, R, K/16] uint8, and one
              fp32 tensor scale per matrix: ``ts`` [E, 3] (gate, up, down).

Random draws: routing inputs come from ``numpy.random.default_rng(seed)`` in the
order bias, logits, activations; weights come from a ``torch.Generator`` on the
requested device seeded per expert, so any subset of experts can be redrawn
alone.  CPU and CUDA generators give different streams: a test draws once and
shares the tensors.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np
import torch

__all__ = ["LayerConfig", "CONFIGS", "make_routing", "make_trace", "make_experts",
           "pack_nibbles", "E2M1_MAGNITUDES"]


@dataclass(frozen=True)
class LayerConfig:
    name: str
    E: int
    k: int
    d: int
    I: int
    fmt: str                      # "bf16" | "mxfp4" | "nvfp4"
    T: tuple = (4,)
    w_std: float = 0.02
    bias_std: float = 0.0         # per-expert routing bias spread
    n_slots: int = 0              # GPU expert-cache slots (0: every expert resident)
    steps: int = 1                # routing-trace length
    rho: float = 0.0              # AR(1) coefficient of the drifting bias
    host_frac: float = 0.0        # share of a step's experts computed on the host
    act: str = "none"             # "nvfp4": activations quantised before each GEMM
    extra: dict = field(default_factory=dict)


CONFIGS = {
    "tiny": LayerConfig("tiny", E=8, k=2, d=256, I=128, fmt="bf16", T=(4,)),
    "decode_bf16": LayerConfig("decode_bf16", E=128, k=8, d=2048, I=768, fmt="bf16",
                               T=(1, 16, 64), bias_std=0.5),
    "decode_mxfp4": LayerConfig("decode_mxfp4", E=256, k=6, d=4096, I=2048, fmt="mxfp4",
                                T=(1, 8), bias_std=0.5, n_slots=64, steps=256, rho=0.9),
    "prefill_nvfp4": LayerConfig("prefill_nvfp4", E=256, k=6, d=4096, I=2048, fmt="nvfp4",
                                 T=(4096,), act="nvfp4"),
    "split_merge": LayerConfig("split_merge", E=256, k=6, d=4096, I=2048, fmt="mxfp4",
                               T=(8,), bias_std=0.5, n_slots=64, steps=256, rho=0.9,
                               host_frac=0.3),
}

# E2M1 magnitudes in code order 0..7 (OCP Microscaling Formats v1.0, FP4 E2M1).
E2M1_MAGNITUDES = (0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0)


def make_routing(cfg: LayerConfig, T: int, seed: int = 0):
    """Router logits fp32 [T, E] (N(0,1) plus a per-expert bias) and activations
    x [T, d] as bf16 (N(0,1) rounded to bf16).  Draw order: bias, logits, x."""
    rng = np.random.default_rng(seed)
    bias = rng.standard_normal(cfg.E) * cfg.bias_std if cfg.bias_std > 0 else np.zeros(cfg.E)
    logits = (rng.standard_normal((T, cfg.E)) + bias[None, :]).astype(np.float32)
    x = torch.from_numpy(rng.standard_normal((T, cfg.d)).astype(np.float32)).to(torch.bfloat16)
    return torch.from_numpy(logits), x


def make_trace(cfg: LayerConfig, T: int, steps: int | None = None, seed: int = 0):
    """A routing trace whose per-expert bias drifts as an AR(1) process:
    b_0 ~ N(0, s^2), b_t = rho*b_{t-1} + sqrt(1-rho^2)*s*eps_t; logits_t = N(0,1) + b_t.
    Yields (logits fp32 [T,E], x bf16 [T,d]) per step."""
    steps = cfg.steps if steps is None else steps
    rng = np.random.default_rng(seed)
    s = cfg.bias_std
    b = rng.standard_normal(cfg.E) * s
    innov = math.sqrt(1.0 - cfg.rho * cfg.rho) * s
    out = []
    for t in range(steps):
        if t > 0:
            b = cfg.rho * b + innov * rng.standard_normal(cfg.E)
        logits = (rng.standard_normal((T, cfg.E)) + b[None, :]).astype(np.float32)
        x = rng.standard_normal((T, cfg.d)).astype(np.float32)
        out.append((torch.from_numpy(logits), torch.from_numpy(x).to(torch.bfloat16)))
    return out


# ---------------------------------------------------------------------------
# weight encoders (input recipe only: they decide which codes the layer sees)
# ---------------------------------------------------------------------------

def _nearest_e2m1(v: torch.Tensor) -> torch.Tensor:
    """Codes 0..15 of the E2M1 value nearest to v (ties to the even code), with
    magnitudes above 6 clamped to 6.  A table search, used only to draw inputs."""
    mags = torch.tensor(E2M1_MAGNITUDES, dtype=torch.float32, device=v.device)
    mids = (mags[1:] + mags[:-1]) * 0.5
    a = v.abs().clamp(max=6.0)
    i = torch.bucketize(a, mids)                     # a <= mid -> lower index
    at_mid = (i < 7) & (a == mids[i.clamp(max=6)])   # exact tie: lower index chosen
    odd_lower = at_mid & (i % 2 == 1)
    i = torch.where(odd_lower, i + 1, i)
    sign = (v < 0) & (i > 0)
    return (i + sign.to(i.dtype) * 8).to(torch.uint8)


def pack_nibbles(codes: torch.Tensor) -> torch.Tensor:
    """[..., K] codes 0..15 -> [..., K/2] bytes, element 2i in the low nibble."""
    c = codes.to(torch.uint8)
    return (c[..., 0::2] | (c[..., 1::2] << 4)).contiguous()


def _mx_encode(w: torch.Tensor):
    """MXFP4 encoding of w [R, K] by the OCP MX v1.0 rule: per 32-element block,
    X = floor(log2(amax)) - 2, scale byte X + 127, codes = nearest E2M1 of v / 2^X."""
    R, K = w.shape
    blk = w.reshape(R, K // 32, 32)
    amax = blk.abs().amax(dim=-1)
    _, ex = torch.frexp(amax)                        # amax = m * 2^ex, m in [0.5, 1)
    X = (ex - 1 - 2).to(torch.int32)
    X = torch.where(amax > 0, X, torch.full_like(X, -127)).clamp(-127, 127)
    scale = torch.ldexp(torch.ones_like(amax), X)
    codes = _nearest_e2m1(blk / scale[..., None]).reshape(R, K)
    return pack_nibbles(codes), (X + 127).to(torch.uint8)


def _nv_encode(w: torch.Tensor):
    """NVFP4 encoding of w [R, K]: tensor scale g = amax/(6*448); per 16-element
    block an E4M3 scale s = e4m3(amax_blk / 6 / g); codes = nearest E2M1 of v/(s*g)."""
    R, K = w.shape
    g = (w.abs().amax() / (6.0 * 448.0)).to(torch.float32)
    if float(g) == 0.0:
        g = torch.tensor(1.0, device=w.device)
    blk = w.reshape(R, K // 16, 16)
    amax = blk.abs().amax(dim=-1)
    s8 = (amax / 6.0 / g).clamp(max=448.0).to(torch.float8_e4m3fn)
    s = s8.to(torch.float32)
    denom = (s * g)[..., None]
    q = torch.where(denom > 0, blk / torch.where(denom > 0, denom, torch.ones_like(denom)),
                    torch.zeros_like(blk))
    codes = _nearest_e2m1(q).reshape(R, K)
    return pack_nibbles(codes), s8.view(torch.uint8), g.reshape(())


def make_experts(cfg: LayerConfig, experts, seed: int = 0, device="cpu"):
    """Canonical weights of the listed experts, stacked in list order.
    Expert e draws gate [I,d], up [I,d], down [d,I] from N(0, w_std^2) with a
    generator seeded by (seed, e), then encodes them in cfg.fmt."""
    experts = list(experts)
    out = {k: [] for k in ("wg", "wu", "wd", "sg", "su", "sd", "ts")}
    for e in experts:
        gen = torch.Generator(device=device)
        gen.manual_seed(int(seed) * 1_000_003 + int(e) + 1)
        mats = [torch.randn(shape, generator=gen, device=device, dtype=torch.float32) * cfg.w_std
                for shape in ((cfg.I, cfg.d), (cfg.I, cfg.d), (cfg.d, cfg.I))]
        if cfg.fmt == "bf16":
            for key, m in zip(("wg", "wu", "wd"), mats):
                out[key].append(m.to(torch.bfloat16))
        elif cfg.fmt == "mxfp4":
            for key, skey, m in zip(("wg", "wu", "wd"), ("sg", "su", "sd"), mats):
                c, s = _mx_encode(m)
                out[key].append(c)
                out[skey].append(s)
        elif cfg.fmt == "nvfp4":
            ts = []
            for key, skey, m in zip(("wg", "wu", "wd"), ("sg", "su", "sd"), mats):
                c, s, g = _nv_encode(m)
                out[key].append(c)
                out[skey].append(s)
                ts.append(g)
            out["ts"].append(torch.stack(ts))
        else:
            raise ValueError(f"unknown weight format {cfg.fmt!r}")
        del mats
    return {k: torch.stack(v) for k, v in out.items() if v}
