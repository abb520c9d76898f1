"""ctypes wrapper of the CPU oracle (oracle.c).

TEST INFRASTRUCTURE ONLY: only tests/, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / reference leg of ``bench.py`` may import this package.  The
product path (``int4_routed_expert_softmax_b200``) never imports it and shares
no code with it.  What each function computes, and the page passage it follows,
is documented in oracle.h / oracle.c.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SO = os.path.join(_HERE, "liboracle.so")
_SRC = os.path.join(_HERE, "oracle.c")

CFLAGS = ["-O2", "-std=c99", "-Wall", "-Wextra", "-ffp-contract=off", "-fPIC", "-shared"]


def build(force: bool = False) -> str:
    """Compile liboracle.so with gcc (plain C99, one thread, no FP contraction)."""
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < max(
        os.path.getmtime(_SRC), os.path.getmtime(os.path.join(_HERE, "oracle.h"))
    ):
        tmp = _SO + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *CFLAGS, _SRC, "-lm", "-o", tmp])
        os.replace(tmp, _SO)
    return _SO


_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_SO)
        P = ctypes.c_void_p
        i32, i64, f32, sz = ctypes.c_int, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t
        sig = {
            "or_matrix_bytes": (sz, [i32, i32]),
            "or_expert_bytes": (sz, [i32, i32]),
            "or_weight": (i32, [P, i32, i32, i32, i32]),
            "or_scale": (f32, [P, i32, i32, i32, i32]),
            "or_pack_matrix": (None, [P, P, i32, i32, P]),
            "or_half_to_float": (f32, [ctypes.c_uint16]),
            "or_quant_q8_0": (None, [P, i64, P, P]),
            "or_silu": (f32, [f32]),
            "or_silu_n": (None, [P, P, i64]),
            "or_router_logit": (f32, [P, P, i32]),
            "or_router_logits": (None, [P, P, i32, i32, i32, P]),
            "or_topk_softmax": (None, [P, i32, i32, i32, P, P]),
            "or_bucket": (None, [P, i32, i32, i32, P, P, P, P, P]),
            "or_block_dot": (ctypes.c_int32, [P, i32, i32, i32, i32, P]),
            "or_expert_dot": (f32, [P, i32, i32, i32, P, P]),
            "or_expert_ffn": (None, [P, i32, i32, P, P, P, P, P, P, P, P]),
            "or_expert_down": (None, [P, i32, i32, P, P, P]),
            "or_moe_layer": (i32, [i32, i32, i32, i32, i32, P, P, P, P, P]),
            "or_moe_layer_tokens": (i32, [i32, i32, i32, i32, P, P, P, P, i32, P]),
            "or_e2m1_value": (f32, [i32]),
            "or_mx_code": (i32, [P, i32, i32, i32, i32]),
            "or_mx_scale_exp": (i32, [P, i32, i32, i32, i32]),
            "or_mx_weight": (f32, [P, i32, i32, i32, i32]),
            "or_mx_pack_matrix": (None, [P, P, i32, i32, P]),
            "or_mx_block_dot": (ctypes.c_int32, [P, i32, i32, i32, i32, P]),
            "or_mx_expert_dot": (f32, [P, i32, i32, i32, P, P]),
            "or_mx_expert_down": (None, [P, i32, i32, P, P, P]),
            "or_mx_expert_ffn": (None, [P, i32, i32, P, P, P, P, P, P, P, P]),
            "or_moe_layer_mx": (i32, [i32, i32, i32, i32, i32, P, P, P, P, P]),
            "or_moe_layer_tokens_mx": (i32, [i32, i32, i32, i32, P, P, P, P, i32, P]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _p(a: np.ndarray | None):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return ctypes.c_void_p(a.ctypes.data)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


# ---------------------------------------------------------------- container
def matrix_bytes(N: int, K: int) -> int:
    return int(lib().or_matrix_bytes(N, K))


def expert_bytes(H: int, I: int) -> int:
    return int(lib().or_expert_bytes(H, I))


def weight(mat: np.ndarray, N: int, K: int, n: int, k: int) -> int:
    return int(lib().or_weight(_p(mat), N, K, n, k))


def scale(mat: np.ndarray, N: int, K: int, n: int, g: int) -> float:
    return float(lib().or_scale(_p(mat), N, K, n, g))


def pack_matrix(w: np.ndarray, s16: np.ndarray) -> np.ndarray:
    """w int [N][K] in [-8,7], s16 uint16 fp16 bit patterns [N][K/64]."""
    w = _c(w, np.int8)
    s16 = _c(s16, np.uint16)
    N, K = w.shape
    out = np.zeros(matrix_bytes(N, K), np.uint8)
    lib().or_pack_matrix(_p(w), _p(s16), N, K, _p(out))
    return out


def half_to_float(h: int) -> float:
    return float(lib().or_half_to_float(h))


# ---------------------------------------------------------------- Q8_0
def quant_q8_0(x: np.ndarray):
    x = _c(x, np.float32)
    n = x.size
    q = np.zeros(x.shape, np.int8)
    d = np.zeros(x.shape[:-1] + (x.shape[-1] // 32,), np.float32)
    lib().or_quant_q8_0(_p(x), n, _p(q), _p(d))
    return q, d


def silu(x: np.ndarray) -> np.ndarray:
    x = _c(x, np.float32)
    y = np.empty_like(x)
    lib().or_silu_n(_p(x), _p(y), x.size)
    return y


# ---------------------------------------------------------------- router
def router_logits(x: np.ndarray, Wr: np.ndarray) -> np.ndarray:
    x = _c(x, np.float32)
    Wr = _c(Wr, np.float32)
    T, H = x.shape
    E = Wr.shape[0]
    out = np.zeros((T, E), np.float32)
    lib().or_router_logits(_p(x), _p(Wr), T, H, E, _p(out))
    return out


def topk_softmax(logits: np.ndarray, k: int):
    logits = _c(logits, np.float32)
    T, E = logits.shape
    idx = np.zeros((T, k), np.int32)
    w = np.zeros((T, k), np.float32)
    lib().or_topk_softmax(_p(logits), T, E, k, _p(idx), _p(w))
    return idx, w


def bucket(idx: np.ndarray, E: int):
    idx = _c(idx, np.int32)
    T, k = idx.shape
    cnt = np.zeros(E, np.int32)
    off = np.zeros(E + 1, np.int32)
    uni = np.zeros(E, np.int32)
    nu = np.zeros(1, np.int32)
    perm = np.zeros(max(T * k, 1), np.int32)
    lib().or_bucket(_p(idx), T, k, E, _p(cnt), _p(off), _p(uni), _p(nu), _p(perm))
    n = int(nu[0])
    return cnt, off, uni[:n].copy(), n, perm[: T * k].copy()


# ---------------------------------------------------------------- experts
def block_dot(mat, N, K, n, b, q) -> int:
    q = _c(q, np.int8)
    return int(lib().or_block_dot(_p(mat), N, K, n, b, _p(q)))


def expert_dot(mat, N, K, n, q, d) -> float:
    q = _c(q, np.int8)
    d = _c(d, np.float32)
    return float(lib().or_expert_dot(_p(mat), N, K, n, _p(q), _p(d)))


def expert_ffn(blob: np.ndarray, H: int, I: int, xq: np.ndarray, xd: np.ndarray, fmt: str = "int4"):
    """Returns dict g, u, h, hq, hd, y for one token (fmt "int4": int4 gs64
    blob; "mxfp4": MXFP4 blob)."""
    blob = _c(blob, np.uint8)
    xq = _c(xq, np.int8)
    xd = _c(xd, np.float32)
    g = np.zeros(I, np.float32)
    u = np.zeros(I, np.float32)
    h = np.zeros(I, np.float32)
    hq = np.zeros(I, np.int8)
    hd = np.zeros(I // 32, np.float32)
    y = np.zeros(H, np.float32)
    fn = lib().or_mx_expert_ffn if fmt == "mxfp4" else lib().or_expert_ffn
    fn(_p(blob), H, I, _p(xq), _p(xd), _p(g), _p(u), _p(h), _p(hq), _p(hd), _p(y))
    return dict(g=g, u=u, h=h, hq=hq, hd=hd, y=y)


def expert_down(blob: np.ndarray, H: int, I: int, hq: np.ndarray, hd: np.ndarray,
                fmt: str = "int4") -> np.ndarray:
    """y [H] of one expert from given codes hq [I] and scales hd [I/32];
    fmt "int4" (int4 gs64 blob) or "mxfp4" (MXFP4 blob)."""
    blob = _c(blob, np.uint8)
    hq = _c(hq, np.int8)
    hd = _c(hd, np.float32)
    y = np.zeros(H, np.float32)
    fn = lib().or_mx_expert_down if fmt == "mxfp4" else lib().or_expert_down
    fn(_p(blob), H, I, _p(hq), _p(hd), _p(y))
    return y


# ---------------------------------------------------------------- MXFP4 experts
def e2m1_value(code: int) -> float:
    return float(lib().or_e2m1_value(code))


def mx_pack_matrix(codes: np.ndarray, exps: np.ndarray) -> np.ndarray:
    """codes uint8 [N][K] in 0..15 (E2M1), exps uint8 [N][K/32] (E8M0)."""
    codes = _c(codes, np.uint8)
    exps = _c(exps, np.uint8)
    N, K = codes.shape
    out = np.zeros(matrix_bytes(N, K), np.uint8)
    lib().or_mx_pack_matrix(_p(codes), _p(exps), N, K, _p(out))
    return out


def mx_code(mat, N, K, n, k) -> int:
    return int(lib().or_mx_code(_p(mat), N, K, n, k))


def mx_scale_exp(mat, N, K, n, b) -> int:
    return int(lib().or_mx_scale_exp(_p(mat), N, K, n, b))


def mx_weight(mat, N, K, n, k) -> float:
    return float(lib().or_mx_weight(_p(mat), N, K, n, k))


def mx_block_dot(mat, N, K, n, b, q) -> int:
    q = _c(q, np.int8)
    return int(lib().or_mx_block_dot(_p(mat), N, K, n, b, _p(q)))


def mx_expert_dot(mat, N, K, n, q, d) -> float:
    q = _c(q, np.int8)
    d = _c(d, np.float32)
    return float(lib().or_mx_expert_dot(_p(mat), N, K, n, _p(q), _p(d)))


class _Trace(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in
                ("xq", "xd", "logits", "idx", "w", "cnt", "off", "uni", "n_uni", "perm", "hq", "hd", "y")]


def _blob_ptrs(blobs):
    """blobs: uint8 array [E+1][bytes] (C-contiguous) or a list of 1-D uint8 arrays."""
    if isinstance(blobs, np.ndarray) and blobs.ndim == 2:
        arrs = [blobs[i] for i in range(blobs.shape[0])]
    else:
        arrs = list(blobs)
    arrs = [_c(a, np.uint8) for a in arrs]
    ptrs = (ctypes.c_void_p * len(arrs))(*[a.ctypes.data for a in arrs])
    return arrs, ptrs


def moe_layer(x: np.ndarray, Wr: np.ndarray, blobs, H: int, I: int, E: int, k: int,
              trace: bool = False, fmt: str = "int4"):
    """Full layer on every token.  Returns out [T][H] (and the trace dict).
    fmt: "int4" (int4 gs64 blobs) or "mxfp4" (MXFP4 blobs)."""
    x = _c(x, np.float32)
    Wr = _c(Wr, np.float32)
    T = x.shape[0]
    out = np.zeros((T, H), np.float32)
    keep, ptrs = _blob_ptrs(blobs)
    tr = None
    arrays = {}
    if trace:
        arrays = dict(
            xq=np.zeros((T, H), np.int8), xd=np.zeros((T, H // 32), np.float32),
            logits=np.zeros((T, E), np.float32), idx=np.zeros((T, k), np.int32),
            w=np.zeros((T, k), np.float32), cnt=np.zeros(E, np.int32),
            off=np.zeros(E + 1, np.int32), uni=np.zeros(E, np.int32),
            n_uni=np.zeros(1, np.int32), perm=np.zeros(max(T * k, 1), np.int32),
            hq=np.zeros((T, k + 1, I), np.int8), hd=np.zeros((T, k + 1, I // 32), np.float32),
            y=np.zeros((T, k + 1, H), np.float32))
        tr = _Trace(**{n: a.ctypes.data for n, a in arrays.items()})
    fn = lib().or_moe_layer_mx if fmt == "mxfp4" else lib().or_moe_layer
    rc = fn(H, I, E, k, T, _p(x), _p(Wr), ptrs, _p(out), ctypes.byref(tr) if tr is not None else None)
    if rc != 0:
        raise ValueError("oracle rejected the shape")
    del keep
    if trace:
        n = int(arrays["n_uni"][0])
        arrays["uni"] = arrays["uni"][:n]
        arrays["perm"] = arrays["perm"][: T * k]
        arrays["n_uni"] = n
        return out, arrays
    return out


def moe_layer_tokens(x: np.ndarray, Wr: np.ndarray, blobs, H, I, E, k, tokens,
                     fmt: str = "int4") -> np.ndarray:
    """Layer output for the listed token rows only (routing is per token);
    fmt "int4" or "mxfp4" as in moe_layer."""
    x = _c(x, np.float32)
    Wr = _c(Wr, np.float32)
    tok = _c(tokens, np.int32)
    out = np.zeros((tok.size, H), np.float32)
    keep, ptrs = _blob_ptrs(blobs)
    fn = lib().or_moe_layer_tokens_mx if fmt == "mxfp4" else lib().or_moe_layer_tokens
    rc = fn(H, I, E, k, _p(x), _p(Wr), ptrs, _p(tok), tok.size, _p(out))
    del keep
    if rc != 0:
        raise ValueError("oracle rejected the shape")
    return out
