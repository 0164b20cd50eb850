"""The routed-expert MoE layer forward, written out plainly.

What the pages fix (titles and sections):
  * Each token is routed to k of E experts (freetoken.wiki "FreeToken 753b
    model", "FreeToken 753b Model Explained": 6 of 256 experts per layer) and
    expert choice is per token (explainx.ai hardware guide, "Decode: decide
    whether to move an expert or compute where it lives").
  * Misses are split between GPU cache fills and CPU execution, and the
    CPU-side and GPU-side partial sums are added exactly: the split changes
    the schedule, it skips or approximates no expert (explainx.ai, same
    section; ainewsfeed.tech third paragraph: the router is left unchanged).
    So the layer's result does not depend on where an expert runs, and this
    oracle is the plain MoE definition, independent of cache state and split.

Readings where the pages are silent:
  * gates = softmax over the k selected logits (equal to the full softmax
    renormalised over the selected experts);
  * order of selected experts: logit descending, ties to the lower index;
    -0.0 and +0.0 tie;
  * permutation: stable counting sort of pair ids p = t*k + j by expert;
  * expert FFN = SwiGLU without biases: y = W_d (silu(W_g x) * (W_u x)),
    silu(h) = h / (1 + exp(-h)), W_g, W_u [I, d], W_d [d, I];
  * combine: out[t] = sum_j gate[t,j] * y[t,j] over the pairs whose expert is
    in the evaluated set; a host partial is such a sum over the host set;
  * act="nvfp4": x and the SwiGLU output are quantised to NVFP4 (unit tensor
    scale) before the two products, the decision taken in fp32
    (formats.nvfp4_quantize_rows).

Pins (tests/test_oracle_layer.py): brute force on tiny
inputs in pure-Python loops; E=1, k=1 equals a dense SwiGLU from torch's silu
and matmul; token-order invariance; subset A plus complement B equals the
whole layer; top-k against a sorted() brute force with constructed ties;
act="nvfp4" against a layer worked by hand (its quantised x and a written out,
ties included), with planted misplacements of either quantisation failing it
(tests/test_oracle_mutations.py); dequant_expert's NVFP4 tensor scales against
hand-set, distinct gate / up / down scales.
"""
from __future__ import annotations

import numpy as np

from . import formats


def route_topk(logits, k: int):
    """Top-k experts per token and their softmax-renormalised gates.
    logits fp32 [T, E] -> idx int32 [T, k] (logit desc, index asc), gate float64 [T, k]."""
    l = np.asarray(logits, dtype=np.float32)
    T, E = l.shape
    assert 1 <= k <= E
    # stable sort of the negated logits keeps equal logits in index order
    order = np.argsort(-l.astype(np.float64), axis=1, kind="stable")
    idx = order[:, :k].astype(np.int32)
    sel = np.take_along_axis(l, idx, axis=1).astype(np.float64)
    z = np.exp(sel - sel[:, :1])
    gate = z / z.sum(axis=1, keepdims=True)
    return idx, gate


def permute(idx, E: int):
    """Stable counting sort of pairs p = t*k + j by expert idx[t, j].
    Returns offsets int32 [E+1] (exclusive scan of counts), perm int32 [T*k]
    (sorted position -> p, ascending p within an expert) and inv_perm (p -> position)."""
    flat = np.asarray(idx, dtype=np.int64).ravel()
    counts = np.bincount(flat, minlength=E)
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    perm = np.argsort(flat, kind="stable").astype(np.int32)
    inv_perm = np.empty_like(perm)
    inv_perm[perm] = np.arange(perm.size, dtype=np.int32)
    return offsets, perm, inv_perm


def silu(h):
    return h / (1.0 + np.exp(-h))


def swiglu_ffn(xr, wg, wu, wd, act: str = "none", dtype=np.float64):
    """One expert on rows xr [n, d]: y = (silu(xr wg^T) * (xr wu^T)) wd^T."""
    xr = np.asarray(xr, dtype=dtype)
    if act == "nvfp4":
        xr = formats.nvfp4_quantize_rows(xr.astype(np.float32))[0].astype(dtype)
    wg = np.asarray(wg, dtype=dtype)
    wu = np.asarray(wu, dtype=dtype)
    wd = np.asarray(wd, dtype=dtype)
    h = xr @ wg.T
    u = xr @ wu.T
    a = silu(h) * u
    if act == "nvfp4":
        a = formats.nvfp4_quantize_rows(a.astype(np.float32))[0].astype(dtype)
    return a @ wd.T


def dequant_expert(fmt: str, w: dict, e: int):
    """fp64 (W_g, W_u, W_d) of expert e from the canonical tensors of
    synth.make_experts (indexable by e, numpy or torch)."""
    def np_(t):
        t = t[e]
        if hasattr(t, "detach"):
            t = t.detach().cpu()
            if str(t.dtype) == "torch.bfloat16":
                t = t.view(__import__("torch").int16)
            t = t.numpy()
        return t
    if fmt == "bf16":
        return tuple(formats.bf16_decode(np_(w[key]).view(np.uint16)) for key in ("wg", "wu", "wd"))
    if fmt == "mxfp4":
        return tuple(formats.dequant_mxfp4(np_(w[c]), np_(w[s]))
                     for c, s in (("wg", "sg"), ("wu", "su"), ("wd", "sd")))
    if fmt == "nvfp4":
        ts = np_(w["ts"])
        return tuple(formats.dequant_nvfp4(np_(w[c]), np_(w[s]), ts[i])
                     for i, (c, s) in enumerate((("wg", "sg"), ("wu", "su"), ("wd", "sd"))))
    raise ValueError(fmt)


def moe_layer(x, logits, k: int, expert_weights, *, experts=None, tokens=None,
              act: str = "none", dtype=np.float64):
    """The layer forward.

    x [T, d] (float values, e.g. bf16 decoded), logits fp32 [T, E],
    expert_weights(e) -> (W_g, W_u, W_d) as float arrays.
    experts: iterable of expert ids whose pairs are evaluated (None: all) --
      the subset sum used for host partials and for the split invariance.
    tokens: iterable of token ids to evaluate (None: all); the others stay 0.
    Returns dict(out [T, d], idx, gate, offsets, perm, inv_perm)."""
    x = np.asarray(x, dtype=np.float64)
    T, d = x.shape
    E = np.asarray(logits).shape[1]
    idx, gate = route_topk(logits, k)
    offsets, perm, inv_perm = permute(idx, E)
    subset = None if experts is None else set(int(e) for e in experts)
    tok = np.arange(T) if tokens is None else np.asarray(sorted(set(int(t) for t in tokens)))
    tokset = set(int(t) for t in tok)
    out = np.zeros((T, d), dtype=dtype)
    # group the evaluated pairs by expert, as the permutation does
    for e in range(E):
        if subset is not None and e not in subset:
            continue
        pos = range(offsets[e], offsets[e + 1])
        pairs = [int(perm[q]) for q in pos if int(perm[q]) // k in tokset]
        if not pairs:
            continue
        rows = np.array([p // k for p in pairs])
        wg, wu, wd = expert_weights(e)
        y = swiglu_ffn(x[rows], wg, wu, wd, act=act, dtype=dtype)
        for r, p in enumerate(pairs):
            t, j = divmod(p, k)
            out[t] += gate[t, j] * y[r]
    return dict(out=out, idx=idx, gate=gate, offsets=offsets, perm=perm, inv_perm=inv_perm)


def per_pair_outputs(x, logits, k, expert_weights, *, pairs=None, act="none"):
    """Unweighted expert outputs y[p] [n_pairs, d] for the listed pair ids
    (all pairs if None), in the given order."""
    x = np.asarray(x, dtype=np.float64)
    T, d = x.shape
    idx, _ = route_topk(logits, k)
    pairs = list(range(T * k)) if pairs is None else [int(p) for p in pairs]
    out = np.zeros((len(pairs), d))
    by_e = {}
    for n, p in enumerate(pairs):
        by_e.setdefault(int(idx.ravel()[p]), []).append(n)
    for e, ns in by_e.items():
        wg, wu, wd = expert_weights(e)
        rows = np.array([pairs[n] // k for n in ns])
        out[ns] = swiglu_ffn(x[rows], wg, wu, wd, act=act)
    return out
