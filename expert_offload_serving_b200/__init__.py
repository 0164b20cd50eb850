"""B200 routed-expert MoE layer: Python binding of libmoe.so.

The functions here carry the C ABI's names (include/moe.h) and only marshal
arguments: torch tensors give device pointers, torch streams give
cudaStream_t.  Every step of the layer runs in libmoe's CUDA kernels; there is
no Python or CPU fallback, and loading fails loudly if the library is absent.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe.so")

MOE_OK, MOE_ERR_INVALID_ARG, MOE_ERR_UNSUPPORTED, MOE_ERR_CUDA, MOE_ERR_CAPACITY, \
    MOE_ERR_TIMEOUT, MOE_ERR_DEVICE = range(7)
STATUS_NAMES = ["MOE_OK", "MOE_ERR_INVALID_ARG", "MOE_ERR_UNSUPPORTED", "MOE_ERR_CUDA",
                "MOE_ERR_CAPACITY", "MOE_ERR_TIMEOUT", "MOE_ERR_DEVICE"]
MOE_W_BF16, MOE_W_MXFP4, MOE_W_NVFP4 = 0, 1, 2
FORMATS = {"bf16": MOE_W_BF16, "mxfp4": MOE_W_MXFP4, "nvfp4": MOE_W_NVFP4}
MOE_FFN_ACT_NVFP4 = 1


class MoeError(RuntimeError):
    def __init__(self, status: int, msg: str):
        name = STATUS_NAMES[status] if 0 <= status < len(STATUS_NAMES) else str(status)
        super().__init__(f"{name}: {msg}")
        self.status = status


class moe_shape(ctypes.Structure):
    _fields_ = [("E", ctypes.c_int32), ("d", ctypes.c_int32), ("I", ctypes.c_int32),
                ("fmt", ctypes.c_int32)]


_P = ctypes.c_void_p
_I = ctypes.c_int
_SZ = ctypes.c_size_t
_SIGS = {
    "moe_abi_version": (_I, []),
    "moe_last_error": (ctypes.c_char_p, []),
    "moe_set_wait_limit_ns": (ctypes.c_uint64, [ctypes.c_uint64]),
    "moe_set_test_stall": (_I, [_I]),
    "moe_expert_blob_bytes": (_SZ, [moe_shape]),
    "moe_pack_expert": (_I, [moe_shape, _P, _P, _P, _P, _P, _P, _P, _P]),
    "moe_route_topk": (_I, [_P, _I, _I, _I, _P, _P, _P]),
    "moe_permute_scratch_bytes": (_SZ, [_I, _I, _I]),
    "moe_permute": (_I, [_P, _I, _I, _I, _P, _P, _P, _P, _SZ, _P, _P]),
    "moe_permute_noalloc": (_I, [_P, _I, _I, _I, _P, _P, _P, _P, _P]),
    "moe_expert_ffn_workspace_bytes": (_SZ, [moe_shape, _I, _I, _I]),
    "moe_expert_ffn_launches": (_I, [moe_shape, _I, _I, _I]),
    "moe_expert_ffn": (_I, [moe_shape, _P, _I, _I, _P, _P, _P, _P, _I, _P, _P, _P, _I, _P, _SZ, _P, _P]),
    "moe_combine_merge": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _P, _P]),
    "moe_layer_forward": (_I, [moe_shape, _P, _P, _I, _I, _P, _P, _P, _P, _P, _P, _SZ, _P, _P, _I, _P, _I, _P,
                               _SZ, _P, _P, _P, _P]),
    "moe_split_misses": (_I, [_P, _I, _P, _I, ctypes.c_double, ctypes.c_double, ctypes.c_double, _P, _P, _P,
                              _P]),
    "moe_host_expert_ffn": (_I, [moe_shape, _P, _P, _I, _P, _P, _P, _I, _I, _P, _I]),
    "moe_profile_bandwidth": (_I, [moe_shape, _P, _I, _P, _SZ, _I, _P, ctypes.POINTER(ctypes.c_double),
                                   ctypes.POINTER(ctypes.c_double)]),
    "moe_cache_create": (_I, [moe_shape, _I, _P, _P, _P, ctypes.POINTER(_P)]),
    "moe_cache_fill": (_I, [_P, _P, _I, _I, _P, _I, _P, _P, _P, _P, _P]),
    "moe_cache_create_layers": (_I, [moe_shape, _I, _I, _P, _P, _P, ctypes.POINTER(_P)]),
    "moe_cache_fill_layer": (_I, [_P, _I, _P, _I, _I, _P, _I, _P, _P, _P, _P, _P]),
    "moe_cache_resize": (_I, [_P, _I, _P, _P, _P, _P, _P]),
    "moe_cache_query": (_I, [_P, _P, _P, _P]),
    "moe_cache_destroy": (_I, [_P]),
    "moe_check_status": (_I, [_P, _P]),
}

_lib = None


def lib():
    """The loaded libmoe.so (ctypes.CDLL); raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              "`python -m expert_offload_serving_b200.build` (nvcc, sm_100a)")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def declared_symbols():
    return list(_SIGS)


def _check(status: int):
    if status != MOE_OK:
        raise MoeError(status, lib().moe_last_error().decode(errors="replace"))


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _dev(name, t, n, dtype):
    """The C calls see plain pointers: a device buffer must be a contiguous CUDA
    tensor of the documented dtype holding the n elements the call touches
    (checked here, since the library cannot see sizes)."""
    if t is None:
        return
    if not t.is_cuda or t.dtype != dtype or not t.is_contiguous():
        raise ValueError(f"{name}: expected a contiguous CUDA {dtype} tensor, got {t.dtype} on {t.device}"
                         f"{'' if t.is_contiguous() else ' (not contiguous)'}")
    if t.numel() < n:
        raise ValueError(f"{name} holds {t.numel()} elements; the call touches {n}")


def _stream(s):
    if s is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(s, int):
        return s
    return s.cuda_stream


def _event(ev):
    """cudaEvent_t of a torch.cuda.Event.  torch creates the CUDA event only on
    its first record, so an event that was never recorded has no handle yet."""
    if ev is None:
        return None
    h = ev.cuda_event
    if not h:
        raise ValueError("torch.cuda.Event has no CUDA event yet: record it once before passing it")
    return h


def shape(E: int, d: int, I: int, fmt) -> moe_shape:
    return moe_shape(E, d, I, FORMATS[fmt] if isinstance(fmt, str) else int(fmt))


# ------------------------------------------------------------------ the ABI
def moe_abi_version() -> int:
    return lib().moe_abi_version()


def moe_set_wait_limit_ns(ns: int) -> int:
    """Limit of the tensor-core kernels' bounded waits for later launches (0:
    the default 2 s); returns the previous limit.  A testing aid."""
    return int(lib().moe_set_wait_limit_ns(int(ns)))


def moe_set_test_stall(on: bool) -> bool:
    """Testing aid: while on, CTA 0 of each tensor-core kernel waits on a
    barrier nothing arrives on, so the bounded-wait abort path runs."""
    return bool(lib().moe_set_test_stall(1 if on else 0))


def moe_expert_blob_bytes(s: moe_shape) -> int:
    return lib().moe_expert_blob_bytes(s)


def moe_pack_expert(s: moe_shape, wg, wu, wd, sg=None, su=None, sd=None, tensor_scales=None, blob_out=None):
    """Canonical CPU tensors -> blob_out (CPU uint8 tensor of moe_expert_blob_bytes)."""
    _check(lib().moe_pack_expert(s, _ptr(wg), _ptr(wu), _ptr(wd), _ptr(sg), _ptr(su), _ptr(sd),
                                 _ptr(tensor_scales), _ptr(blob_out)))


def moe_route_topk(logits, k: int, idx, gate, stream=None):
    T, E = logits.shape
    _dev("logits", logits, T * E, torch.float32)
    _dev("idx", idx, T * k, torch.int32)
    _dev("gate", gate, T * k, torch.float32)
    _check(lib().moe_route_topk(_ptr(logits), T, E, k, _ptr(idx), _ptr(gate), _stream(stream)))


def moe_permute_scratch_bytes(T: int, k: int, E: int) -> int:
    return lib().moe_permute_scratch_bytes(T, k, E)


def _permute_buffers(idx, E, offsets, perm, inv_perm):
    T, k = idx.shape
    _dev("idx", idx, T * k, torch.int32)
    _dev("offsets", offsets, E + 1, torch.int32)
    _dev("perm", perm, T * k, torch.int32)
    _dev("inv_perm", inv_perm, T * k, torch.int32)
    return T, k


def moe_permute(idx, E: int, offsets, perm, inv_perm, scratch=None, dev_status=None, stream=None):
    T, k = _permute_buffers(idx, E, offsets, perm, inv_perm)
    nbytes = 0 if scratch is None else scratch.numel() * scratch.element_size()
    _check(lib().moe_permute(_ptr(idx), T, k, E, _ptr(offsets), _ptr(perm), _ptr(inv_perm),
                             _ptr(scratch), nbytes, _ptr(dev_status), _stream(stream)))


MOE_PERMUTE_NOALLOC_MAX_SCRATCH = 262144


def moe_permute_noalloc(idx, E: int, offsets, perm, inv_perm, dev_status=None, stream=None):
    """moe_permute without a scratch argument: for callers that cannot
    allocate device memory (the library's fixed scratch array is used)."""
    T, k = _permute_buffers(idx, E, offsets, perm, inv_perm)
    _check(lib().moe_permute_noalloc(_ptr(idx), T, k, E, _ptr(offsets), _ptr(perm), _ptr(inv_perm),
                                     _ptr(dev_status), _stream(stream)))


def moe_expert_ffn_workspace_bytes(s: moe_shape, T: int, k: int, flags: int = 0) -> int:
    return lib().moe_expert_ffn_workspace_bytes(s, T, k, flags)


def moe_expert_ffn_launches(s: moe_shape, T: int, k: int, flags: int = 0) -> int:
    """Kernels one moe_expert_ffn call launches (no device work)."""
    return lib().moe_expert_ffn_launches(s, T, k, flags)


def moe_expert_ffn(s: moe_shape, x, k: int, offsets, perm, slot_of_expert, slot_pool, n_slots: int,
                   gate=None, y_perm=None, out=None, flags: int = 0, workspace=None,
                   dev_status=None, stream=None):
    T = x.shape[0]
    _dev("x", x, T * s.d, torch.bfloat16)
    _dev("offsets", offsets, s.E + 1, torch.int32)
    _dev("perm", perm, T * k, torch.int32)
    _dev("slot_of_expert", slot_of_expert, s.E, torch.int32)
    _dev("slot_pool", slot_pool, n_slots * moe_expert_blob_bytes(s), torch.uint8)
    _dev("gate", gate, T * k, torch.float32)
    _dev("y_perm", y_perm, T * k * s.d, torch.float32)
    _dev("out", out, T * s.d, torch.float32)
    nbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib().moe_expert_ffn(s, _ptr(x), T, k, _ptr(offsets), _ptr(perm), _ptr(slot_of_expert),
                                _ptr(slot_pool), n_slots, _ptr(gate), _ptr(y_perm), _ptr(out), flags,
                                _ptr(workspace), nbytes, _ptr(dev_status), _stream(stream)))


def moe_combine_merge(y_perm, idx, gate, inv_perm, slot_of_expert, host_partial, E: int, out, stream=None):
    T, k = idx.shape
    d = out.shape[1]
    _dev("y_perm", y_perm, T * k * d, torch.float32)
    _dev("idx", idx, T * k, torch.int32)
    _dev("gate", gate, T * k, torch.float32)
    _dev("inv_perm", inv_perm, T * k, torch.int32)
    _dev("slot_of_expert", slot_of_expert, E, torch.int32)
    _dev("host_partial", host_partial, T * d, torch.float32)
    _dev("out", out, T * d, torch.float32)
    _check(lib().moe_combine_merge(_ptr(y_perm), _ptr(idx), _ptr(gate), _ptr(inv_perm),
                                   _ptr(slot_of_expert), _ptr(host_partial), T, k, d, E, _ptr(out),
                                   _stream(stream)))


def moe_layer_forward(s: moe_shape, logits, x, k: int, idx, gate, offsets, perm, inv_perm, scratch,
                      slot_of_expert, slot_pool, n_slots: int, y_perm, flags, workspace, host_partial, out,
                      dev_status=None, stream=None):
    """All four steps in one call (moe_route_topk -> moe_permute ->
    moe_expert_ffn -> moe_combine_merge); x [T, d] gives T."""
    T = x.shape[0]
    n = T * k
    for name, t, need, dt in (("logits", logits, T * s.E, torch.float32), ("x", x, T * s.d, torch.bfloat16),
                              ("idx", idx, n, torch.int32), ("gate", gate, n, torch.float32),
                              ("offsets", offsets, s.E + 1, torch.int32), ("perm", perm, n, torch.int32),
                              ("inv_perm", inv_perm, n, torch.int32), ("slot_of_expert", slot_of_expert, s.E, torch.int32),
                              ("slot_pool", slot_pool, n_slots * moe_expert_blob_bytes(s), torch.uint8),
                              ("y_perm", y_perm, n * s.d, torch.float32),
                              ("host_partial", host_partial, T * s.d, torch.float32), ("out", out, T * s.d, torch.float32)):
        _dev(name, t, need, dt)
    sb = 0 if scratch is None else scratch.numel() * scratch.element_size()
    wb = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib().moe_layer_forward(s, _ptr(logits), _ptr(x), T, k, _ptr(idx), _ptr(gate), _ptr(offsets), _ptr(perm),
                                   _ptr(inv_perm), _ptr(scratch), sb, _ptr(slot_of_expert), _ptr(slot_pool),
                                   n_slots, _ptr(y_perm), flags, _ptr(workspace), wb, _ptr(host_partial),
                                   _ptr(out), _ptr(dev_status), _stream(stream)))


def moe_split_misses(misses, tokens_per_expert, q=None, bw_pcie=0.0, bw_host=0.0):
    """The q split of a step's misses (host only): returns (filled, host), two
    ascending lists of expert ids.  q=None selects the q* policy from the
    bandwidths; otherwise floor(q*m + 0.5) misses are filled."""
    m = len(misses)
    E = len(tokens_per_expert)
    ms = (ctypes.c_int32 * max(1, m))(*[int(e) for e in misses])
    tok = (ctypes.c_int32 * max(1, E))(*[int(t) for t in tokens_per_expert])
    f = (ctypes.c_int32 * max(1, m))()
    h = (ctypes.c_int32 * max(1, m))()
    nf, nh = ctypes.c_int32(0), ctypes.c_int32(0)
    _check(lib().moe_split_misses(ms, m, tok, E, -1.0 if q is None else float(q), float(bw_pcie), float(bw_host),
                                  f, ctypes.byref(nf), h, ctypes.byref(nh)))
    return [f[i] for i in range(nf.value)], [h[i] for i in range(nh.value)]


def _host(name, t, n, dtype):
    """A host buffer of the host-only calls: a contiguous CPU tensor of the
    documented dtype holding n elements."""
    if t.is_cuda or t.dtype != dtype or not t.is_contiguous() or t.numel() < n:
        raise ValueError(f"{name}: expected a contiguous CPU {dtype} tensor of >= {n} elements, "
                         f"got {t.dtype} {tuple(t.shape)} on {t.device}")


def moe_host_expert_ffn(s: moe_shape, host_pool, experts, x, idx, gate, out, n_threads: int = 0):
    """The host share of a split step (host only): out [T, d] fp32 = the
    gate-weighted SwiGLU sum over the pairs whose expert is in `experts`,
    computed on the CPU from the host pool's blobs.  x bf16 [T, d], idx int32
    [T, k], gate fp32 [T, k]: CPU tensors.  Releases the GIL while it runs."""
    T, k = idx.shape
    B = moe_expert_blob_bytes(s)
    _host("host_pool", host_pool, s.E * B, torch.uint8)
    _host("x", x, T * s.d, torch.bfloat16)
    _host("idx", idx, T * k, torch.int32)
    _host("gate", gate, T * k, torch.float32)
    _host("out", out, T * s.d, torch.float32)
    ex = (ctypes.c_int32 * max(1, len(experts)))(*[int(e) for e in experts])
    _check(lib().moe_host_expert_ffn(s, _ptr(host_pool), ex, len(experts), _ptr(x), _ptr(idx), _ptr(gate), T, k,
                                     _ptr(out), int(n_threads)))


def moe_profile_bandwidth(s: moe_shape, host_pool, n_blobs: int, dev_buf=None, n_threads: int = 0, stream=None):
    """(pinned host -> device GB/s, host expert-kernel GB/s) measured on this
    machine; dev_buf None skips the copy measurement."""
    B = moe_expert_blob_bytes(s)
    _host("host_pool", host_pool, n_blobs * B, torch.uint8)
    if dev_buf is not None:
        _dev("dev_buf", dev_buf, B, torch.uint8)
    h2d, hst = ctypes.c_double(0), ctypes.c_double(0)
    _check(lib().moe_profile_bandwidth(s, _ptr(host_pool), int(n_blobs), _ptr(dev_buf),
                                       0 if dev_buf is None else dev_buf.numel(), int(n_threads),
                                       _stream(stream) if dev_buf is not None else None,
                                       ctypes.byref(h2d), ctypes.byref(hst)))
    return h2d.value, hst.value


def moe_check_status(dev_status, stream=None):
    _check(lib().moe_check_status(_ptr(dev_status), _stream(stream)))


class MoeCache:
    """Handle of the host-side LRU bookkeeping (moe_cache_*).  n_layers > 1:
    one cache shared by several layers (host_pool and slot_of_expert_dev are
    then lists with one entry per layer)."""

    def __init__(self, s: moe_shape, n_slots: int, slot_pool=None, host_pool=None, slot_of_expert_dev=None,
                 n_layers: int = 1):
        h = ctypes.c_void_p()
        if n_layers == 1 and not isinstance(host_pool, (list, tuple)):
            _check(lib().moe_cache_create(s, n_slots, _ptr(slot_pool), _ptr(host_pool),
                                          _ptr(slot_of_expert_dev), ctypes.byref(h)))
        else:
            if slot_pool is None:
                hp = tb = None
            else:
                if len(host_pool) != n_layers or len(slot_of_expert_dev) != n_layers:
                    raise ValueError(f"{n_layers} layers need {n_layers} host pools and slot tables")
                hp = (ctypes.c_void_p * n_layers)(*[_ptr(p) for p in host_pool])
                tb = (ctypes.c_void_p * n_layers)(*[_ptr(t) for t in slot_of_expert_dev])
            _check(lib().moe_cache_create_layers(s, n_layers, n_slots, _ptr(slot_pool), hp, tb, ctypes.byref(h)))
        self.h = h
        self.E, self.n_slots, self.n_layers = s.E, n_slots, n_layers

    def fill(self, experts, step: int, protect=(), side=None, reads_done=None, fill_done=None, layer: int = 0):
        """moe_cache_fill_layer; returns the list of (expert, slot, evicted key) fills."""
        ex = (ctypes.c_int32 * max(1, len(experts)))(*[int(e) for e in experts])
        pr = (ctypes.c_int32 * max(1, len(protect)))(*[int(e) for e in protect])
        fills = (ctypes.c_int32 * (3 * max(1, len(experts))))()
        nf = ctypes.c_int32(0)
        side_h = None if side is None else _stream(side)
        _check(lib().moe_cache_fill_layer(self.h, int(layer), ex, len(experts), step, pr, len(protect), side_h,
                                          _event(reads_done), _event(fill_done), fills, ctypes.byref(nf)))
        return [(fills[3 * i], fills[3 * i + 1], fills[3 * i + 2]) for i in range(nf.value)]

    def resize(self, new_n_slots: int, new_slot_pool=None, stream=None, reads_done=None):
        """moe_cache_resize; returns [(key, old slot)] of the kept residents in
        their new slot order."""
        kept = (ctypes.c_int32 * (2 * max(1, min(self.n_slots, new_n_slots))))()
        nk = ctypes.c_int32(0)
        st = None if new_slot_pool is None else _stream(stream)
        _check(lib().moe_cache_resize(self.h, int(new_n_slots), _ptr(new_slot_pool), st, _event(reads_done), kept,
                                      ctypes.byref(nk)))
        self.n_slots = new_n_slots
        return [(kept[2 * i], kept[2 * i + 1]) for i in range(nk.value)]

    def query(self):
        soe = (ctypes.c_int32 * (self.E * self.n_layers))()
        eos = (ctypes.c_int32 * self.n_slots)()
        lu = (ctypes.c_int32 * self.n_slots)()
        _check(lib().moe_cache_query(self.h, soe, eos, lu))
        return list(soe), list(eos), list(lu)

    def close(self):
        if self.h:
            lib().moe_cache_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
