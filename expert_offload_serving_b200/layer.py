"""Host orchestration of one routed-expert MoE layer on top of the C ABI.

`MoeLayer` owns the device buffers (through torch) and issues the five steps
on a CUDA stream: moe_route_topk -> (moe_cache_fill) -> moe_permute ->
moe_expert_ffn -> moe_combine_merge.  All arithmetic runs in libmoe's
kernels; this module only allocates, packs expert blobs with moe_pack_expert
and sequences the calls.
"""
from __future__ import annotations

import threading
import time

import torch

from . import (MOE_FFN_ACT_NVFP4, FORMATS, MoeCache, _check, lib, moe_combine_merge, moe_expert_blob_bytes,
               moe_expert_ffn, moe_expert_ffn_workspace_bytes, moe_host_expert_ffn, moe_pack_expert, moe_permute,
               moe_permute_scratch_bytes, moe_route_topk, moe_split_misses, shape)


def _u8(t: torch.Tensor) -> torch.Tensor:
    t = t.contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.uint8)
    return t


def pack_pool(E: int, d: int, I: int, fmt: str, weights: dict, experts, pin: bool = True) -> torch.Tensor:
    """Blobs of the listed experts, in list order, as one CPU uint8 tensor
    [len(experts), blob_bytes] (pinned if requested).  `weights` holds the
    canonical tensors of synth.make_experts indexed by position in `experts`."""
    s = shape(E, d, I, fmt)
    B = moe_expert_blob_bytes(s)
    pool = torch.empty((len(experts), B), dtype=torch.uint8, pin_memory=pin)
    cpu = {k: v.cpu().contiguous() for k, v in weights.items()}
    for n in range(len(experts)):
        args = [cpu[k][n] for k in ("wg", "wu", "wd")]
        sc = [cpu[k][n] if k in cpu else None for k in ("sg", "su", "sd")]
        ts = cpu["ts"][n].to(torch.float32).contiguous() if "ts" in cpu else None
        moe_pack_expert(s, *[_u8(a) for a in args], *sc, tensor_scales=ts, blob_out=pool[n])
    return pool


class ExpertCache:
    """The GPU expert cache of one or more layers of the same shape: one device
    slot pool, one device slot table per layer, the host bookkeeping
    (moe_cache_*), the side stream the fills run on and the two events that
    order them.  With several layers it is the global LRU over (layer, expert)
    keys; resize() rebuilds it under a new slot budget at a safe point."""

    def __init__(self, s, n_slots: int, host_pools, device="cuda"):
        host_pools = list(host_pools) if isinstance(host_pools, (list, tuple)) else [host_pools]
        self.s, self.n_layers, self.n_slots = s, len(host_pools), n_slots
        self.dev = torch.device(device)
        self.B = moe_expert_blob_bytes(s)
        self.host_pools = host_pools
        self.pool = torch.empty((n_slots, self.B), dtype=torch.uint8, device=self.dev)
        self.tables = [torch.full((s.E,), -1, dtype=torch.int32, device=self.dev) for _ in host_pools]
        self.handle = MoeCache(s, n_slots, self.pool, host_pools if self.n_layers > 1 else host_pools[0],
                               self.tables if self.n_layers > 1 else self.tables[0], n_layers=self.n_layers)
        self.side = torch.cuda.Stream(device=self.dev)
        # torch creates a CUDA event lazily on first record: record both now
        # so that their handles exist when the library records and waits on them
        self.fill_done = torch.cuda.Event()
        self.reads_done = torch.cuda.Event()
        self.fill_done.record(self.side)
        self.reads_done.record()
        self.version = 0                     # bumped when the pool moves

    def fill(self, layer: int, experts, step: int, protect=()):
        return self.handle.fill(experts, step, protect, side=self.side, reads_done=self.reads_done,
                                fill_done=self.fill_done, layer=layer)

    def resize(self, new_n_slots: int, stream=None, new_pool=None):
        """Elastic resize at a safe point: a new pool of new_n_slots blobs
        (allocated here, or the caller's uint8 [new_n_slots, blob bytes]
        device tensor) receives the most recently used residents
        (device-to-device copies on `stream`, after the last recorded reader);
        the old pool's memory goes back to torch's allocator once the stream
        has passed the copies.  Returns [(key, old slot)] per kept resident."""
        s = torch.cuda.current_stream() if stream is None else stream
        if new_pool is None:
            new_pool = torch.empty((new_n_slots, self.B), dtype=torch.uint8, device=self.dev)
        elif (new_pool.dtype != torch.uint8 or tuple(new_pool.shape) != (new_n_slots, self.B)
              or new_pool.device.type != "cuda" or not new_pool.is_contiguous()
              or new_pool.device.index != (self.dev.index if self.dev.index is not None
                                           else torch.cuda.current_device())):
            raise ValueError(f"new_pool must be a contiguous uint8 [{new_n_slots}, {self.B}] tensor on {self.dev}")
        kept = self.handle.resize(new_n_slots, new_pool, stream=s, reads_done=self.reads_done)
        self.pool.record_stream(s)
        self.pool = new_pool
        self.n_slots = new_n_slots
        self.version += 1
        self.reads_done.record(s)            # the next fill waits for the moves
        return kept

    def close(self):
        self.handle.close()


class MoeLayer:
    """One MoE layer of shape (E, d, I, fmt) with top-k routing.

    Resident mode: `device_pool` holds all E blobs, expert e in slot e.
    Cached mode: `host_pool` (pinned, E blobs) plus `n_slots` device slots
    managed by the LRU cache -- or `cache` (an ExpertCache shared by several
    layers) and this layer's `layer_id` in it; call `prepare(step, experts)`
    to fill.  act="nvfp4" selects the FP4 tensor-core FFN (fused combine)."""

    def __init__(self, E, d, I, fmt, k, T_max, device="cuda", device_pool=None, host_pool=None,
                 n_slots=None, act="none", cache=None, layer_id=0):
        self.E, self.d, self.I, self.k, self.fmt, self.act = E, d, I, k, fmt, act
        self.s = shape(E, d, I, fmt)
        self.B = moe_expert_blob_bytes(self.s)
        self.dev = torch.device(device)
        self.T_max = T_max
        self.flags = MOE_FFN_ACT_NVFP4 if act == "nvfp4" else 0
        i32 = dict(dtype=torch.int32, device=self.dev)
        f32 = dict(dtype=torch.float32, device=self.dev)
        n = T_max * k
        self.idx = torch.empty((T_max, k), **i32)
        self.gate = torch.empty((T_max, k), **f32)
        self.offsets = torch.empty((E + 1,), **i32)
        self.perm = torch.empty((max(n, 1),), **i32)
        self.inv_perm = torch.empty((max(n, 1),), **i32)
        sb = moe_permute_scratch_bytes(T_max, k, E)
        self.scratch = torch.empty((max(sb, 256),), dtype=torch.uint8, device=self.dev)
        wb = moe_expert_ffn_workspace_bytes(self.s, T_max, k, self.flags)
        self.workspace = torch.empty((max(wb, 256),), dtype=torch.uint8, device=self.dev)
        self.y_perm = None if act == "nvfp4" else torch.empty((max(n, 1), d), **f32)
        self.out = torch.empty((T_max, d), **f32)
        self.status = torch.zeros((1,), **i32)
        self.cache = None
        self.xcache = None
        if device_pool is not None:
            assert device_pool.shape[1] == self.B
            self._pool = device_pool
            self._n_slots = device_pool.shape[0]
            self.slot = torch.full((E,), -1, **i32)
            self.slot[: min(E, self._n_slots)] = torch.arange(min(E, self._n_slots), **i32)
        else:
            if cache is None:
                assert host_pool is not None and n_slots is not None
                cache = ExpertCache(self.s, n_slots, host_pool, device=self.dev)
            self.xcache, self.layer_id = cache, layer_id
            self.cache = cache.handle
            self.host_pool = cache.host_pools[layer_id]
            self.slot = cache.tables[layer_id]
            self.side, self.fill_done, self.reads_done = cache.side, cache.fill_done, cache.reads_done
            self._pool_version = cache.version

    @property
    def pool(self):
        return self._pool if self.xcache is None else self.xcache.pool

    @property
    def n_slots(self):
        return self._n_slots if self.xcache is None else self.xcache.n_slots

    # -- argument checks ---------------------------------------------------------
    # The C calls see plain pointers, so the sizes of the layer's own buffers
    # (T_max tokens) are enforced here, before any call is made.
    def _check_T(self, T: int) -> int:
        if not 0 <= T <= self.T_max:
            raise ValueError(f"T={T} outside [0, {self.T_max}]: the layer's buffers hold T_max={self.T_max} tokens")
        return T

    def _check_tensor(self, name, t, shape, dtype):
        if t is None:
            return
        same_device = t.device.type == self.dev.type and (self.dev.index is None or t.device.index == self.dev.index)
        if tuple(t.shape) != tuple(shape) or t.dtype != dtype or not t.is_contiguous() or not same_device:
            raise ValueError(f"{name}: expected a contiguous {dtype} tensor of shape {tuple(shape)} on {self.dev}, "
                             f"got {t.dtype} {tuple(t.shape)} on {t.device}")

    # -- steps -----------------------------------------------------------------
    def route(self, logits, stream=None):
        T = self._check_T(logits.shape[0])
        moe_route_topk(logits, self.k, self.idx[:T], self.gate[:T], stream)

    def prepare(self, step: int, gpu_experts, protect=(), stream=None):
        """Cached mode: make `gpu_experts` resident for this step (LRU fills on
        the side stream); the main stream waits for the fills.  With a shared
        cache, `step` is the cache's clock (increasing over layers and steps)."""
        fills = self.xcache.fill(self.layer_id, gpu_experts, step, protect)
        s = stream or torch.cuda.current_stream()
        if fills:
            s.wait_event(self.fill_done)
        return fills

    def permute(self, T, stream=None):
        self._check_T(T)
        moe_permute(self.idx[:T], self.E, self.offsets, self.perm, self.inv_perm,
                    scratch=self.scratch, dev_status=self.status, stream=stream)

    def _record_reads_done(self, stream):
        # the next fill's copies into a victim slot, and its slot-table update,
        # wait on this event: it must follow the last kernel of the step that
        # reads the pool or the slot table
        if self.xcache is not None:
            if stream is None:
                rs = torch.cuda.current_stream()
            else:
                rs = torch.cuda.ExternalStream(stream) if isinstance(stream, int) else stream
            self.xcache.reads_done.record(rs)

    def ffn(self, x, stream=None, out=None, host_partial=None):
        """The expert FFN.  act="nvfp4": the FFN adds gate-weighted outputs
        into `out` itself (fused combine), so `out` is first set to
        host_partial, or to zero; combine() is then not called."""
        T = self._check_T(x.shape[0])
        if self.act == "nvfp4":
            self._check_tensor("host_partial", host_partial, (T, self.d), torch.float32)
            o = out if out is not None else self.out[:T]
            s = torch.cuda.current_stream() if stream is None else (
                torch.cuda.ExternalStream(stream) if isinstance(stream, int) else stream)
            with torch.cuda.stream(s):
                if host_partial is not None:
                    o.copy_(host_partial)
                else:
                    o.zero_()
            moe_expert_ffn(self.s, x, self.k, self.offsets, self.perm, self.slot, self.pool, self.n_slots,
                           gate=self.gate, out=o, flags=self.flags,
                           workspace=self.workspace, dev_status=self.status, stream=stream)
            self._record_reads_done(stream)          # the fused FFN is the step's last reader
        else:
            if host_partial is not None:
                raise ValueError("host_partial belongs to combine() unless act='nvfp4'")
            moe_expert_ffn(self.s, x, self.k, self.offsets, self.perm, self.slot, self.pool, self.n_slots,
                           y_perm=self.y_perm, workspace=self.workspace, dev_status=self.status,
                           stream=stream)

    def combine(self, T, host_partial=None, stream=None, out=None):
        if self.act == "nvfp4":
            raise RuntimeError("act='nvfp4' combines inside ffn() (fused into the down projection); "
                               "pass host_partial to ffn() instead")
        self._check_T(T)
        self._check_tensor("host_partial", host_partial, (T, self.d), torch.float32)
        moe_combine_merge(self.y_perm, self.idx[:T], self.gate[:T], self.inv_perm, self.slot, host_partial,
                          self.E, out if out is not None else self.out[:T], stream)
        self._record_reads_done(stream)              # combine reads the slot table

    def split_step(self, step: int, logits, x, q=None, bw=(0.0, 0.0), threads: int = 0, stream=None):
        """One cached decode step whose misses are split between GPU fills and
        host computation, the two running at once (explainx.ai hardware guide,
        "Decode": the q* policy splits misses so both paths run concurrently;
        their partial sums merge exactly).

        route -> read the routing back -> split the misses (moe_split_misses:
        q in [0, 1], or q=None for q* from bw = (pcie GB/s, host GB/s)) ->
        fill the GPU share on the side stream -> permute + FFN on `stream`
        while a CPU thread runs moe_host_expert_ffn over the host share ->
        upload the host partial -> combine.  Returns the step's split
        (hits, filled, host, fills) and the host kernel's wall time (host_ms)."""
        if self.cache is None or self.act == "nvfp4":
            raise RuntimeError("split_step needs cached mode and the unfused FFN")
        T = self._check_T(x.shape[0])
        s = torch.cuda.current_stream() if stream is None else stream
        if not hasattr(self, "_split_bufs"):
            pin = dict(pin_memory=True)
            self._split_bufs = dict(
                idx=torch.empty((self.T_max, self.k), dtype=torch.int32, **pin),
                gate=torch.empty((self.T_max, self.k), dtype=torch.float32, **pin),
                x=torch.empty((self.T_max, self.d), dtype=torch.bfloat16, **pin),
                hp=torch.empty((self.T_max, self.d), dtype=torch.float32, **pin),
                hp_dev=torch.empty((self.T_max, self.d), dtype=torch.float32, device=self.dev),
                routed=torch.cuda.Event())
        b = self._split_bufs
        with torch.cuda.stream(s):
            self.route(logits, stream=s)
            b["idx"][:T].copy_(self.idx[:T], non_blocking=True)
            b["gate"][:T].copy_(self.gate[:T], non_blocking=True)
            b["x"][:T].copy_(x, non_blocking=True)
            b["routed"].record(s)
        b["routed"].synchronize()
        idx = b["idx"][:T]
        flat = idx.reshape(-1).tolist()
        U = sorted(set(flat))
        resident = self.cache.query()[0][self.layer_id * self.E:(self.layer_id + 1) * self.E]
        hits = [e for e in U if resident[e] >= 0]
        misses = [e for e in U if resident[e] < 0]
        tpe = [0] * self.E
        for e in flat:
            tpe[e] += 1
        filled, host = moe_split_misses(misses, tpe, q, *bw)
        fills = self.prepare(step, sorted(hits + filled), protect=U, stream=s)
        err, host_ms = [], [0.0]

        def host_share():
            try:
                t0 = time.perf_counter()
                moe_host_expert_ffn(self.s, self.host_pool, host, b["x"][:T], idx, b["gate"][:T], b["hp"][:T],
                                    threads)
                host_ms[0] = (time.perf_counter() - t0) * 1e3
            except Exception as ex:         # re-raised on the calling thread
                err.append(ex)
        th = threading.Thread(target=host_share) if host else None
        if th is not None:
            th.start()
        self.permute(T, stream=s)
        self.ffn(x, stream=s)
        if th is not None:
            th.join()
            if err:
                raise err[0]
            with torch.cuda.stream(s):
                b["hp_dev"][:T].copy_(b["hp"][:T], non_blocking=True)
        self.combine(T, host_partial=b["hp_dev"][:T] if host else None, stream=s)
        return dict(hits=hits, filled=filled, host=host, fills=fills, host_ms=host_ms[0])

    def forward(self, logits, x, host_partial=None, stream=None):
        """All steps through moe_layer_forward (one C call); returns out [T, d]
        (a view of an internal buffer, overwritten by the next call).  Cached
        mode: call prepare() first; the step's reads of the pool and the slot
        table are then recorded for the next fill to wait on."""
        T = self._check_T(x.shape[0])
        self._check_tensor("logits", logits, (T, self.E), torch.float32)
        self._check_tensor("x", x, (T, self.d), torch.bfloat16)
        self._check_tensor("host_partial", host_partial, (T, self.d), torch.float32)
        if self.xcache is not None and self._pool_version != self.xcache.version:
            self.__dict__.pop("_fwd_args", None)            # the pool moved (resize)
            self._pool_version = self.xcache.version
        if not hasattr(self, "_fwd_args"):
            # device addresses of the layer's own buffers, resolved once
            nb = lambda t: t.numel() * t.element_size()
            self._fwd_args = (self.idx.data_ptr(), self.gate.data_ptr(), self.offsets.data_ptr(),
                              self.perm.data_ptr(), self.inv_perm.data_ptr(), self.scratch.data_ptr(),
                              nb(self.scratch), self.slot.data_ptr(), self.pool.data_ptr(), self.n_slots,
                              0 if self.y_perm is None else self.y_perm.data_ptr(), self.flags,
                              self.workspace.data_ptr(), nb(self.workspace))
        s = (torch.cuda.current_stream() if stream is None else stream)
        s = s if isinstance(s, int) else s.cuda_stream
        hp = 0 if host_partial is None else host_partial.data_ptr()
        _check(lib().moe_layer_forward(self.s, logits.data_ptr(), x.data_ptr(), T, self.k, *self._fwd_args, hp,
                                       self.out.data_ptr(), self.status.data_ptr(), s))
        self._record_reads_done(stream)
        return self.out[:T]


class StreamedPrefill:
    """Prefill through n layers whose expert pools stay in pinned host memory
    (explainx.ai hardware guide, "Prefill: load almost every expert without
    idling the GPU": many tokens reach nearly every expert, so each layer's
    whole pool is streamed over PCIe into one of two full-layer buffers while
    the GPU computes the previous layer from the other).

    Two device buffers of E blobs each, two MoeLayer views over them (expert e
    in slot e, the FP4 tensor-core FFN), a copy stream, and per buffer a
    `copied` and a `computed` event: the copy of layer l + 1 into buffer
    (l + 1) % 2 waits for layer l - 1's compute on that buffer; layer l's
    compute waits for its copy.  double_buffer=False issues each layer's copy
    only after the previous layer's compute (the pages' ablation)."""

    def __init__(self, E, d, I, k, T_max, host_pools, device="cuda", act="nvfp4"):
        self.host_pools = list(host_pools)
        s = shape(E, d, I, "nvfp4")
        B = moe_expert_blob_bytes(s)
        for p in self.host_pools:
            if tuple(p.shape) != (E, B) or p.dtype != torch.uint8 or not p.is_pinned():
                raise ValueError(f"host pools must be pinned uint8 [{E}, {B}]")
        self.dev = torch.device(device)
        self.bufs = [torch.empty((E, B), dtype=torch.uint8, device=self.dev) for _ in range(2)]
        self.layers = [MoeLayer(E, d, I, "nvfp4", k, T_max, device=self.dev, device_pool=b, act=act)
                       for b in self.bufs]
        self.copy = torch.cuda.Stream(device=self.dev)
        self.copied = [torch.cuda.Event() for _ in range(2)]
        self.computed = [torch.cuda.Event() for _ in range(2)]
        for ev in self.computed + self.copied:
            ev.record()                      # every event has a handle before it is waited on

    def _issue_copy(self, l):
        b = l % 2
        with torch.cuda.stream(self.copy):
            self.copy.wait_event(self.computed[b])
            self.bufs[b].copy_(self.host_pools[l], non_blocking=True)
            self.copied[b].record(self.copy)

    def run(self, inputs, double_buffer=True, stream=None, keep_outputs=False):
        """inputs: one (logits [T, E] fp32, x [T, d] bf16) device pair per layer.
        Returns the per-layer outputs (clones) if keep_outputs."""
        s = torch.cuda.current_stream() if stream is None else stream
        outs = []
        n = len(inputs)
        if n > len(self.host_pools):
            raise ValueError(f"{n} layers of input for {len(self.host_pools)} host pools")
        if double_buffer:
            self._issue_copy(0)
        for l in range(n):
            b = l % 2
            if double_buffer:
                if l + 1 < n:
                    self._issue_copy(l + 1)
            else:
                self.copy.wait_event(self.computed[(l + 1) % 2])   # the previous layer has finished
                self._issue_copy(l)
            s.wait_event(self.copied[b])
            logits, x = inputs[l]
            out = self.layers[b].forward(logits, x, stream=s)
            if keep_outputs:
                with torch.cuda.stream(s):
                    outs.append(out.clone())
            self.computed[b].record(s)
        return outs
