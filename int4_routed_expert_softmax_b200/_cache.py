"""ctypes binding of the expert cache and the split layer calls of libmoe
(include/moe.h).  Argument marshalling only; the cache policy, the copies and
every kernel live in libmoe.so."""
from __future__ import annotations

import ctypes
import os

import numpy as np
import torch

from ._lib import MoeDims, MoeError, _arg, _ptr, _rows, _stream, lib

MOE_CACHE_DEVICE, MOE_CACHE_HOST = 0, 1
MOE_FAULT_NONE, MOE_FAULT_COPY, MOE_FAULT_ALLOC = 0, 1, 2
MOE_ERR_IO = -10


class CacheStats(ctypes.Structure):
    _fields_ = [(n, ctypes.c_uint64) for n in (
        "hits", "misses", "prefetches", "prefetch_hits", "evictions", "bytes_h2d", "copy_errors")] + [
        (n, ctypes.c_int32) for n in ("slots", "slots_per_layer", "pinned", "resident")]

    def as_dict(self):
        return {n: getattr(self, n) for n, _ in self._fields_}


_sig_done = False


def _sigs():
    global _sig_done
    if _sig_done:
        return lib()
    L = lib()
    P, i32, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t
    D = ctypes.POINTER(MoeDims)
    I32P = ctypes.POINTER(ctypes.c_int32)
    sig = {
        "expert_cache_create": (ctypes.c_int, [D, i32, P, sz, i32, ctypes.POINTER(P)]),
        "expert_cache_destroy": (None, [P]),
        "expert_cache_pin": (ctypes.c_int, [P, i32, I32P, i32, P]),
        "expert_cache_unpin": (ctypes.c_int, [P, i32, I32P, i32]),
        "expert_cache_evict": (ctypes.c_int, [P, i32, I32P, i32]),
        "expert_cache_prefetch": (ctypes.c_int, [P, i32, I32P, i32, P]),
        "expert_cache_acquire": (ctypes.c_int, [P, i32, I32P, i32, P, P, ctypes.POINTER(P)]),
        "expert_cache_release": (ctypes.c_int, [P, i32, P]),
        "expert_cache_learn_pins": (ctypes.c_int, [P, i32, I32P, i32, P]),
        "expert_cache_resident": (ctypes.c_int, [P, i32, i32]),
        "expert_cache_pinned": (ctypes.c_int, [P, i32, i32]),
        "expert_cache_stats": (ctypes.c_int, [P, ctypes.POINTER(CacheStats)]),
        "expert_cache_inject_fault": (ctypes.c_int, [P, i32, i32]),
        "moe_layer_route": (ctypes.c_int, [D, i32, P, P, P, sz, P, P]),
        "moe_read_union": (ctypes.c_int, [D, i32, P, I32P, I32P, P]),
        "moe_layer_experts": (ctypes.c_int, [D, i32, P, P, P, sz, P]),
        "moe_tiered_layer_forward": (ctypes.c_int, [P, i32, D, i32, P, P, P, P, P, sz, P, sz, P, P, P,
                                                    I32P]),
        "moe_usage_save": (ctypes.c_int, [ctypes.c_char_p, i32, i32, ctypes.POINTER(ctypes.c_uint64)]),
        "moe_usage_load": (ctypes.c_int, [ctypes.c_char_p, i32, i32, ctypes.POINTER(ctypes.c_uint64), i32]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args
    _sig_done = True
    return L


def _ilist(xs):
    xs = [int(v) for v in xs]
    return (ctypes.c_int32 * max(1, len(xs)))(*xs), len(xs)


def _chk(fn, rc):
    if rc < 0:
        raise MoeError(fn, rc)
    return rc


def _nbytes(t: torch.Tensor | None) -> int:
    return 0 if t is None else t.numel() * t.element_size()


def inject_fault(kind: int, count: int, cache: "ExpertCache | None" = None) -> None:
    _chk("expert_cache_inject_fault",
         _sigs().expert_cache_inject_fault(cache.handle if cache else None, kind, count))


class ExpertCache:
    """HBM (or, with backend=MOE_CACHE_HOST, host-emulated) expert cache.
    host_blobs: n_layers lists of E+1 host buffers (tensors or numpy arrays,
    pinned for asynchronous copies); they must outlive the cache."""

    def __init__(self, d: MoeDims, n_layers: int, host_blobs, hbm_bytes: int,
                 backend: int = MOE_CACHE_DEVICE):
        L = _sigs()
        ptrs = []
        for layer in host_blobs:
            for b in layer:
                ptrs.append(b.data_ptr() if isinstance(b, torch.Tensor) else b.ctypes.data)
        self._keep = host_blobs
        self._arr = (ctypes.c_void_p * len(ptrs))(*ptrs)
        self.d = d
        self.n_layers = n_layers
        h = ctypes.c_void_p()
        _chk("expert_cache_create",
             L.expert_cache_create(ctypes.byref(d), n_layers, self._arr, hbm_bytes, backend, ctypes.byref(h)))
        self.handle = h

    def close(self):
        if self.handle:
            _sigs().expert_cache_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def pin(self, layer, experts, stream=None):
        a, n = _ilist(experts)
        return _chk("expert_cache_pin", _sigs().expert_cache_pin(self.handle, layer, a, n, _cstream(stream)))

    def unpin(self, layer, experts):
        a, n = _ilist(experts)
        return _chk("expert_cache_unpin", _sigs().expert_cache_unpin(self.handle, layer, a, n))

    def evict(self, layer, experts):
        a, n = _ilist(experts)
        return _chk("expert_cache_evict", _sigs().expert_cache_evict(self.handle, layer, a, n))

    def prefetch(self, layer, experts, stream=None):
        a, n = _ilist(experts)
        return _chk("expert_cache_prefetch",
                    _sigs().expert_cache_prefetch(self.handle, layer, a, n, _cstream(stream)))

    def acquire(self, layer, experts, copy_stream=None, compute_stream=None) -> int:
        """Returns the table address (device, or host for the host backend)."""
        a, n = _ilist(experts)
        t = ctypes.c_void_p()
        _chk("expert_cache_acquire", _sigs().expert_cache_acquire(
            self.handle, layer, a, n, _cstream(copy_stream), _cstream(compute_stream), ctypes.byref(t)))
        return t.value

    def release(self, layer, compute_stream=None):
        return _chk("expert_cache_release",
                    _sigs().expert_cache_release(self.handle, layer, _cstream(compute_stream)))

    def learn_pins(self, layer, counts, n_pin, stream=None):
        # 64-bit usage counts saturate at the 32-bit range the call takes
        a, _ = _ilist(min(int(v), 2**31 - 1) for v in counts)
        return _chk("expert_cache_learn_pins",
                    _sigs().expert_cache_learn_pins(self.handle, layer, a, n_pin, _cstream(stream)))

    def resident(self, layer, e) -> bool:
        return bool(_chk("expert_cache_resident", _sigs().expert_cache_resident(self.handle, layer, e)))

    def pinned(self, layer, e) -> bool:
        return bool(_chk("expert_cache_pinned", _sigs().expert_cache_pinned(self.handle, layer, e)))

    def stats(self) -> dict:
        s = CacheStats()
        _chk("expert_cache_stats", _sigs().expert_cache_stats(self.handle, ctypes.byref(s)))
        return s.as_dict()

    def tiered_layer_forward(self, layer, x, Wr, out, ws, ws_pred=None, Wr_next=None,
                             route_counts=None, compute_stream=None, side_stream=None):
        """One tiered decode layer; returns (prefetches started, predicted union size)."""
        d = self.d
        T = _rows(x, "x", d.H)
        _arg(Wr, "Wr", torch.float32, d.E * d.H)
        _arg(Wr_next, "Wr_next", torch.float32, d.E * d.H, optional=True)
        _arg(out, "out", torch.float32, T * d.H)
        _arg(ws, "ws", torch.uint8)
        _arg(ws_pred, "ws_pred", torch.uint8, optional=True)
        _arg(route_counts, "route_counts", torch.int32, d.E, optional=True)
        po = (ctypes.c_int32 * 2)()
        _chk("moe_tiered_layer_forward", _sigs().moe_tiered_layer_forward(
            self.handle, layer, ctypes.byref(self.d), x.shape[0], _ptr(x), _ptr(Wr), _ptr(Wr_next),
            _ptr(out), _ptr(ws), _nbytes(ws), _ptr(ws_pred), _nbytes(ws_pred), _ptr(route_counts),
            _cstream(compute_stream), _cstream(side_stream), po))
        return int(po[0]), int(po[1])


def _cstream(stream):
    if stream is None:
        return None
    if isinstance(stream, torch.cuda.Stream):
        return ctypes.c_void_p(stream.cuda_stream)
    return stream


def moe_layer_route(d: MoeDims, x, Wr, ws, route_counts=None, stream=None):
    _rows(x, "x", d.H)
    _arg(Wr, "Wr", torch.float32, d.E * d.H)
    _arg(ws, "ws", torch.uint8)
    _arg(route_counts, "route_counts", torch.int32, d.E, optional=True)
    _chk("moe_layer_route", _sigs().moe_layer_route(
        ctypes.byref(d), x.shape[0], _ptr(x), _ptr(Wr), _ptr(ws), _nbytes(ws), _ptr(route_counts),
        _stream(stream)))


def moe_read_union(d: MoeDims, T: int, ws, stream=None):
    _arg(ws, "ws", torch.uint8)
    buf = (ctypes.c_int32 * d.E)()
    n = ctypes.c_int32()
    _chk("moe_read_union", _sigs().moe_read_union(ctypes.byref(d), T, _ptr(ws), buf, ctypes.byref(n),
                                                  _stream(stream)))
    return [int(buf[i]) for i in range(n.value)]


def moe_layer_experts(d: MoeDims, T: int, table, out, ws, stream=None):
    if not isinstance(table, int):
        _arg(table, "table", torch.int64, d.E + 1)
    _arg(out, "out", torch.float32, T * d.H)
    _arg(ws, "ws", torch.uint8)
    tp = table if isinstance(table, int) else table.data_ptr()
    _chk("moe_layer_experts", _sigs().moe_layer_experts(
        ctypes.byref(d), T, ctypes.c_void_p(tp), _ptr(out), _ptr(ws), _nbytes(ws), _stream(stream)))


# ----------------------------------------------------------------- route usage on disk
def usage_save(path, counts) -> None:
    """Writes the route-usage record: counts [n_layers][E] of non-negative
    selection counts (the layers' route_counts), atomically (temp + rename)."""
    a = np.asarray(counts)
    if a.ndim != 2 or (a.size and a.min() < 0):
        raise ValueError("counts must be [n_layers][E] non-negative integers")
    a = np.ascontiguousarray(a, dtype=np.uint64)
    _chk("moe_usage_save", _sigs().moe_usage_save(
        os.fsencode(path), a.shape[0], a.shape[1], a.ctypes.data_as(ctypes.POINTER(ctypes.c_uint64))))


def usage_load(path, n_layers: int, E: int, counts=None) -> np.ndarray:
    """Reads a route-usage record [n_layers][E] (uint64).  With `counts` given
    (a uint64 array of that shape) the file's counts are added to it in place
    and it is returned; on any error it is left unchanged."""
    if counts is None:
        out = np.zeros((n_layers, E), dtype=np.uint64)
        acc = 0
    else:
        out = counts
        if out.dtype != np.uint64 or out.shape != (n_layers, E) or not out.flags.c_contiguous:
            raise ValueError("counts must be a contiguous uint64 array [n_layers][E]")
        acc = 1
    _chk("moe_usage_load", _sigs().moe_usage_load(
        os.fsencode(path), n_layers, E, out.ctypes.data_as(ctypes.POINTER(ctypes.c_uint64)), acc))
    return out
