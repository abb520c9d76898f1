"""ctypes binding of libmoe.so (include/moe.h).  Argument marshalling only:
every step of the layer runs in the library's CUDA kernels.  Torch is used for
device memory and streams; the functions take torch tensors and pass their
data pointers and the current CUDA stream.

Importing never falls back to anything else: if libmoe.so is missing or does not
load, the first call raises."""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe.so")

MOE_OK = 0
MOE_PATH_AUTO, MOE_PATH_DECODE, MOE_PATH_PREFILL = 0, 1, 2
MOE_DECODE_T_MAX = 16


class MoeDims(ctypes.Structure):
    _fields_ = [("H", ctypes.c_int32), ("I", ctypes.c_int32), ("E", ctypes.c_int32), ("k", ctypes.c_int32)]


class MoeWsView(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in (
        "status", "xq", "xd", "logits", "idx", "w", "cnt", "off", "uni", "n_uni", "perm", "pos",
        "pair_tok", "hq", "hd")] + [("T_max", ctypes.c_int32)]


class MoeError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn} failed: {status} ({status_string(status)})")
        self.status = status


_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libmoe.so not built ({LIB_PATH}); run "
                               "python -m int4_routed_expert_softmax_b200.build")
        L = ctypes.CDLL(LIB_PATH)
        P, i32, i64, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
        D = ctypes.POINTER(MoeDims)
        sig = {
            "moe_status_string": (ctypes.c_char_p, [ctypes.c_int]),
            "moe_check_dims": (ctypes.c_int, [D]),
            "moe_expert_bytes": (sz, [D]),
            "moe_workspace_bytes": (sz, [D, i32]),
            "moe_workspace_bytes_path": (sz, [D, i32, i32]),
            "moe_workspace_view": (ctypes.c_int, [D, i32, P, ctypes.POINTER(MoeWsView)]),
            "moe_device_sms": (ctypes.c_int, []),
            "moe_set_wait_limit": (i64, [i64]),
            "moe_layer_launches": (ctypes.c_int, [D, i32, i32]),
            "moe_device_binary_version": (ctypes.c_int, []),
            "moe_profile_enable": (ctypes.c_int, [ctypes.c_int]),
            "moe_profile_read": (ctypes.c_int, [ctypes.POINTER(ctypes.c_float), ctypes.c_int]),
            "moe_quant_q8_0": (ctypes.c_int, [P, i64, i32, P, P, P]),
            "moe_router_topk": (ctypes.c_int, [D, i32, P, P, P, P, P, P, P]),
            "moe_bucket": (ctypes.c_int, [D, i32, P, P, P, P, P, P, P]),
            "moe_layer_forward": (ctypes.c_int, [D, i32, P, P, P, P, P, sz, P, i32, P]),
            "moe_layer_forward_host": (ctypes.c_int, [D, i32, P, P, P, P, P, sz, P, i32, P]),
            "moe_layer_forward_static": (ctypes.c_int, [D, i32, P, P, P, P, P, i32, P]),
            "moe_layer_forward_ep": (ctypes.c_int, [D, i32, P, P, P, P, P, sz, P, i32, i32, i32, P]),
            "moe_layer_forward_mxfp4": (ctypes.c_int, [D, i32, P, P, P, P, P, sz, P, P]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _ptr(t: torch.Tensor | None):
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("tensors passed to libmoe must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _arg(t, name: str, dtype, numel: int = 0, cuda: bool = True, optional: bool = False):
    """Checks a tensor before its address crosses the C ABI, which sees only
    pointers: device (or host) memory, dtype, contiguity, and at least `numel`
    elements -- so that a wrong tensor is refused here instead of being read
    or written out of bounds by a kernel."""
    if t is None:
        if optional:
            return
        raise ValueError(f"{name} is required")
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.is_cuda != cuda:
        raise ValueError(f"{name} must be in {'device' if cuda else 'host'} memory")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if t.numel() < numel:
        raise ValueError(f"{name} has {t.numel()} elements, needs at least {numel}")


def _rows(x, name: str, cols: int, cuda: bool = True) -> int:
    """x [T][cols] float32: returns T."""
    _arg(x, name, torch.float32, cuda=cuda)
    if x.dim() != 2 or x.shape[1] != cols:
        raise ValueError(f"{name} must be [T][{cols}], got {tuple(x.shape)}")
    return x.shape[0]


def _stream(stream=None):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _check(fn: str, rc: int):
    if rc != MOE_OK:
        raise MoeError(fn, rc)


def dims(H: int, I: int, E: int, k: int) -> MoeDims:
    return MoeDims(H, I, E, k)


def status_string(status: int) -> str:
    return lib().moe_status_string(status).decode()


def moe_check_dims(d: MoeDims) -> int:
    return lib().moe_check_dims(ctypes.byref(d))


def moe_expert_bytes(d: MoeDims) -> int:
    return int(lib().moe_expert_bytes(ctypes.byref(d)))


def moe_workspace_bytes(d: MoeDims, T_max: int) -> int:
    return int(lib().moe_workspace_bytes(ctypes.byref(d), T_max))


def moe_workspace_bytes_path(d: MoeDims, T_max: int, path: int) -> int:
    return int(lib().moe_workspace_bytes_path(ctypes.byref(d), T_max, path))


def moe_device_sms() -> int:
    return int(lib().moe_device_sms())


def moe_set_wait_limit(cycles: int) -> int:
    """Wait limit (SM clocks) of the kernels' bounded waits for later calls;
    cycles <= 0 restores the default.  Returns the previous limit."""
    return int(lib().moe_set_wait_limit(int(cycles)))


def moe_layer_launches(d: MoeDims, T: int, path: int = MOE_PATH_AUTO) -> int:
    """Kernels one moe_layer_forward call of T tokens enqueues on the current device."""
    return int(lib().moe_layer_launches(ctypes.byref(d), T, path))


def moe_device_binary_version() -> int:
    """SM version the current device's copy of the library's kernels was built
    for (100 = sm_100a), or a negative status."""
    return int(lib().moe_device_binary_version())


def moe_profile_enable(on: bool) -> None:
    _check("moe_profile_enable", lib().moe_profile_enable(1 if on else 0))


def moe_profile_read(max_calls: int = 1024) -> list:
    """Device-stamped ms per recorded call since the last read, oldest first:
    [routing, gate/up, down, whole call] each; clears the history."""
    buf = (ctypes.c_float * (4 * max_calls))()
    n = lib().moe_profile_read(buf, max_calls)
    if n < 0:
        raise MoeError("moe_profile_read", n)
    return [[float(buf[4 * c + j]) for j in range(4)] for c in range(n)]


def moe_quant_q8_0(x: torch.Tensor, q: torch.Tensor, d: torch.Tensor, stream=None):
    _arg(x, "x", torch.float32)
    if x.dim() != 2:
        raise ValueError("x must be [rows][cols]")
    rows, cols = x.shape
    _arg(q, "q", torch.int8, rows * cols)
    _arg(d, "d", torch.float32, rows * (cols // 32))
    _check("moe_quant_q8_0", lib().moe_quant_q8_0(_ptr(x), rows, cols, _ptr(q), _ptr(d), _stream(stream)))


def moe_router_topk(d: MoeDims, x, Wr, idx, w, logits, route_counts=None, stream=None):
    T = _rows(x, "x", d.H)
    _arg(Wr, "Wr", torch.float32, d.E * d.H)
    _arg(idx, "idx", torch.int32, T * d.k)
    _arg(w, "w", torch.float32, T * d.k)
    _arg(logits, "logits", torch.float32, T * d.E)
    _arg(route_counts, "route_counts", torch.int32, d.E, optional=True)
    _check("moe_router_topk", lib().moe_router_topk(
        ctypes.byref(d), x.shape[0], _ptr(x), _ptr(Wr), _ptr(idx), _ptr(w), _ptr(logits),
        _ptr(route_counts), _stream(stream)))


def moe_bucket(d: MoeDims, idx, cnt, off, uni, n_uni, perm, stream=None):
    _arg(idx, "idx", torch.int32)
    if idx.dim() != 2 or idx.shape[1] != d.k:
        raise ValueError(f"idx must be [T][{d.k}], got {tuple(idx.shape)}")
    T = idx.shape[0]
    _arg(cnt, "cnt", torch.int32, d.E)
    _arg(off, "off", torch.int32, d.E + 1)
    _arg(uni, "uni", torch.int32, d.E)
    _arg(n_uni, "n_uni", torch.int32, 1)
    _arg(perm, "perm", torch.int32, T * d.k)
    _check("moe_bucket", lib().moe_bucket(
        ctypes.byref(d), idx.shape[0], _ptr(idx), _ptr(cnt), _ptr(off), _ptr(uni), _ptr(n_uni),
        _ptr(perm), _stream(stream)))


def _layer_args(d: MoeDims, x, Wr, table, out, route_counts, host: bool):
    T = _rows(x, "x", d.H, cuda=not host)
    _arg(out, "out", torch.float32, T * d.H, cuda=not host)
    _arg(Wr, "Wr", torch.float32, d.E * d.H)
    _arg(table, "table", torch.int64, d.E + 1)
    _arg(route_counts, "route_counts", torch.int32, d.E, optional=True)


def moe_layer_forward(d: MoeDims, x, Wr, table, out, ws, route_counts=None,
                      path: int = MOE_PATH_AUTO, stream=None):
    _layer_args(d, x, Wr, table, out, route_counts, host=False)
    _arg(ws, "ws", torch.uint8)
    _check("moe_layer_forward", lib().moe_layer_forward(
        ctypes.byref(d), x.shape[0], _ptr(x), _ptr(Wr), _ptr(table), _ptr(out), _ptr(ws),
        ws.numel() * ws.element_size(), _ptr(route_counts), path, _stream(stream)))


def moe_layer_forward_mxfp4(d: MoeDims, x, Wr, table, out, ws, route_counts=None, stream=None):
    """The layer with MXFP4 expert blobs (decode path: the fused kernel, up to 16 tokens per launch)."""
    T = _rows(x, "x", d.H)
    _arg(Wr, "Wr", torch.float32, d.E * d.H)
    _arg(table, "table", torch.int64, d.E + 1)
    _arg(out, "out", torch.float32, T * d.H)
    _arg(ws, "ws", torch.uint8)
    _arg(route_counts, "route_counts", torch.int32, d.E, optional=True)
    _check("moe_layer_forward_mxfp4", lib().moe_layer_forward_mxfp4(
        ctypes.byref(d), T, _ptr(x), _ptr(Wr), _ptr(table), _ptr(out), _ptr(ws), ws.numel(),
        _ptr(route_counts), _stream(stream)))


def moe_layer_forward_host(d: MoeDims, x_host, Wr, table, out_host, ws, route_counts=None,
                           path: int = MOE_PATH_AUTO, stream=None):
    _layer_args(d, x_host, Wr, table, out_host, route_counts, host=True)
    _arg(ws, "ws", torch.uint8)
    _check("moe_layer_forward_host", lib().moe_layer_forward_host(
        ctypes.byref(d), x_host.shape[0], _ptr(x_host), _ptr(Wr), _ptr(table), _ptr(out_host),
        _ptr(ws), ws.numel() * ws.element_size(), _ptr(route_counts), path, _stream(stream)))


def moe_layer_forward_static(d: MoeDims, x, Wr, table, out, route_counts=None,
                             path: int = MOE_PATH_AUTO, stream=None):
    """moe_layer_forward on the library's static device workspace (no allocation)."""
    _layer_args(d, x, Wr, table, out, route_counts, host=False)
    _check("moe_layer_forward_static", lib().moe_layer_forward_static(
        ctypes.byref(d), x.shape[0], _ptr(x), _ptr(Wr), _ptr(table), _ptr(out), _ptr(route_counts),
        path, _stream(stream)))


def moe_workspace_view(d: MoeDims, T: int, ws: torch.Tensor) -> MoeWsView:
    _arg(ws, "ws", torch.uint8)
    v = MoeWsView()
    _check("moe_workspace_view", lib().moe_workspace_view(ctypes.byref(d), T, _ptr(ws), ctypes.byref(v)))
    return v


# ----------------------------------------------------------------- helpers
def alloc_workspace(d: MoeDims, T_max: int, device="cuda", path: int = MOE_PATH_AUTO) -> torch.Tensor:
    """Device workspace for batches of up to T_max tokens on `path` (256-byte aligned)."""
    n = moe_workspace_bytes_path(d, T_max, path)
    if n == 0:
        raise MoeError("moe_workspace_bytes", -2)
    ws = torch.empty(n + 256, dtype=torch.uint8, device=device)
    off = (-ws.data_ptr()) % 256
    return ws[off:off + n]


def expert_table(blobs: torch.Tensor | list) -> torch.Tensor:
    """Device array of blob pointers (int64) from a [E+1][bytes] uint8 tensor
    or a list of 1-D uint8 device tensors (entry E = shared expert)."""
    if isinstance(blobs, torch.Tensor):
        dev = blobs.device
        ptrs = [blobs[i].data_ptr() for i in range(blobs.shape[0])]
    else:
        dev = blobs[0].device
        ptrs = [b.data_ptr() for b in blobs]
    return torch.tensor(ptrs, dtype=torch.int64, device=dev)


def ws_slice(ws: torch.Tensor, ptr: int, shape, dtype) -> torch.Tensor:
    """The workspace region at device address `ptr` (from moe_workspace_view)
    as a tensor view of `shape` / `dtype`."""
    n = 1
    for s_ in shape:
        n *= s_
    itemsize = torch.empty((), dtype=dtype).element_size()
    off = ptr - ws.data_ptr()
    assert 0 <= off and off + n * itemsize <= ws.numel(), "pointer outside the workspace"
    return ws[off:off + n * itemsize].view(dtype).view(*shape)
