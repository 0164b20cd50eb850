"""Host orchestration of one routed-expert MoE layer on top of the C ABI.

`MoeLayer` owns the device buffers (through torch) and issues the five steps
on a CUDA stream: moe_route_topk -> (moe_cache_fill) -> moe_permute ->
moe_expert_ffn -> moe_combine_merge.  All arithmetic runs in libmoe's
kernels; this module only allocates, packs expert blobs with moe_pack_expert
and sequences the calls.
"""
from __future__ import annotations

import torch

from . import (MOE_FFN_ACT_NVFP4, FORMATS, MoeCache, _check, lib, moe_combine_merge, moe_expert_blob_bytes,
               moe_expert_ffn, moe_expert_ffn_workspace_bytes, moe_pack_expert, moe_permute,
               moe_permute_scratch_bytes, moe_route_topk, shape)


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


class MoeLayer:
    """One MoE layer of shape (E, d, I, fmt) with top-k routing.

    Resident mode: `device_pool` holds all E blobs, expert e in slot e.
    Cached mode: `host_pool` (pinned, E blobs) plus `n_slots` device slots
    managed by the LRU cache; call `prepare(step, idx_host)` to fill.
    act="nvfp4" selects the FP4 tensor-core FFN (fused combine)."""

    def __init__(self, E, d, I, fmt, k, T_max, device="cuda", device_pool=None, host_pool=None,
                 n_slots=None, act="none"):
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
        if device_pool is not None:
            assert device_pool.shape[1] == self.B
            self.pool = device_pool
            self.n_slots = device_pool.shape[0]
            self.slot = torch.full((E,), -1, **i32)
            self.slot[: min(E, self.n_slots)] = torch.arange(min(E, self.n_slots), **i32)
        else:
            assert host_pool is not None and n_slots is not None
            self.host_pool = host_pool
            self.n_slots = n_slots
            self.pool = torch.empty((n_slots, self.B), dtype=torch.uint8, device=self.dev)
            self.slot = torch.full((E,), -1, **i32)
            self.cache = MoeCache(self.s, n_slots, self.pool, host_pool, self.slot)
            self.side = torch.cuda.Stream(device=self.dev)
            # torch creates a CUDA event lazily on first record: record both now
            # so that their handles exist when the library records and waits on them
            self.fill_done = torch.cuda.Event()
            self.reads_done = torch.cuda.Event()
            self.fill_done.record(self.side)
            self.reads_done.record()

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
        the side stream); the main stream waits for the fills."""
        fills = self.cache.fill(gpu_experts, step, protect, side=self.side,
                                reads_done=self.reads_done, fill_done=self.fill_done)
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
        if self.cache is not None:
            if stream is None:
                rs = torch.cuda.current_stream()
            else:
                rs = torch.cuda.ExternalStream(stream) if isinstance(stream, int) else stream
            self.reads_done.record(rs)

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

    def forward(self, logits, x, host_partial=None, stream=None):
        """All steps through moe_layer_forward (one C call); returns out [T, d]
        (a view of an internal buffer, overwritten by the next call).  Cached
        mode: call prepare() first; the step's reads of the pool and the slot
        table are then recorded for the next fill to wait on."""
        T = self._check_T(x.shape[0])
        self._check_tensor("logits", logits, (T, self.E), torch.float32)
        self._check_tensor("x", x, (T, self.d), torch.bfloat16)
        self._check_tensor("host_partial", host_partial, (T, self.d), torch.float32)
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
