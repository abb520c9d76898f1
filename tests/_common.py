"""Shared helpers of the test suite (not a test module)."""
from __future__ import annotations

import numpy as np
import torch

import moe_inputs as mi
import oracle as orc

REL_L2 = 1e-4      # final outputs: relative L2 error
MAX_ABS = 2e-3     # final outputs: max-abs error as a fraction of rms(reference)


def within_tolerance(got: np.ndarray, ref: np.ndarray):
    """(ok, rel_l2, max_abs / rms) of the stated float tolerance."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    nr = np.linalg.norm(ref)
    rel = float(np.linalg.norm(got - ref) / nr) if nr > 0 else float(np.linalg.norm(got))
    rms = float(np.sqrt(np.mean(ref * ref))) if ref.size else 0.0
    mx = float(np.abs(got - ref).max()) if ref.size else 0.0
    mrel = mx / rms if rms > 0 else mx
    return (rel <= REL_L2 and mrel <= MAX_ABS), rel, mrel


def oracle_layer_from_device(x: torch.Tensor, Wr: torch.Tensor, blobs: torch.Tensor,
                             H, I, E, k, trace=True, tokens=None):
    """Runs the oracle on host copies of the device inputs.  Only the blobs of
    the experts the oracle's own routing selects (and the shared expert) are
    copied back; the oracle never reads the others."""
    xh = x.detach().cpu().numpy()
    wh = Wr.detach().cpu().numpy()
    if tokens is not None:
        xsel = xh[np.asarray(tokens)]
    else:
        xsel = xh
    lg = orc.router_logits(xsel, wh)
    idx, _ = orc.topk_softmax(lg, k)
    need = set(np.unique(idx).tolist()) | {E}
    dummy = np.zeros(16, np.uint8)
    blist = [blobs[e].cpu().numpy() if e in need else dummy for e in range(E + 1)]
    if tokens is not None:
        return orc.moe_layer_tokens(xh, wh, blist, H, I, E, k, tokens)
    return orc.moe_layer(xh, wh, blist, H, I, E, k, trace=trace)


def gpu_layer(w: mi.Workload, x, Wr, blobs, path=0, ws=None):
    """Runs moe_layer_forward; returns (out, ws, dims)."""
    import int4_routed_expert_softmax_b200 as moe
    d = moe.dims(w.H, w.I, w.E, w.k)
    T = x.shape[0]
    if ws is None:
        ws = moe.alloc_workspace(d, T, path=path)
    table = moe.expert_table(blobs)
    out = torch.full((T, w.H), float("nan"), dtype=torch.float32, device=x.device)
    moe.moe_layer_forward(d, x, Wr, table, out, ws, path=path)
    torch.cuda.synchronize()
    return out, ws, d


def ws_trace(ws, d, T):
    """Intermediates of the last forward call, as numpy arrays."""
    import int4_routed_expert_softmax_b200 as moe
    v = moe.moe_workspace_view(d, T, ws)
    H, I, E, k = d.H, d.I, d.E, d.k
    P = T * (k + 1)
    g = lambda p, shape, dt: moe.ws_slice(ws, p, shape, dt).cpu().numpy()
    n_uni = int(g(v.n_uni, (1,), torch.int32)[0])
    return dict(
        status=g(v.status, (4,), torch.int32),
        xq=g(v.xq, (T, H), torch.int8), xd=g(v.xd, (T, H // 32), torch.float32),
        logits=g(v.logits, (T, E), torch.float32), idx=g(v.idx, (T, k), torch.int32),
        w=g(v.w, (T, k), torch.float32), cnt=g(v.cnt, (E,), torch.int32),
        off=g(v.off, (E + 1,), torch.int32), uni=g(v.uni, (E + 1,), torch.int32)[:n_uni],
        n_uni=n_uni, perm=g(v.perm, (T * k,), torch.int32), pos=g(v.pos, (T * k,), torch.int32),
        pair_tok=g(v.pair_tok, (P,), torch.int32),
        hq=g(v.hq, (P, I), torch.int8), hd=g(v.hd, (P, I // 32), torch.float32))


def hq_by_slot(tr_gpu, T, k):
    """GPU per-position h codes rearranged to the oracle's [T][k+1] slot order."""
    P = T * k
    hq = np.zeros((T, k + 1) + tr_gpu["hq"].shape[1:], tr_gpu["hq"].dtype)
    hd = np.zeros((T, k + 1) + tr_gpu["hd"].shape[1:], tr_gpu["hd"].dtype)
    for t in range(T):
        for s in range(k):
            p = tr_gpu["pos"][t * k + s]
            hq[t, s] = tr_gpu["hq"][p]
            hd[t, s] = tr_gpu["hd"][p]
        hq[t, k] = tr_gpu["hq"][P + t]
        hd[t, k] = tr_gpu["hd"][P + t]
    return hq, hd
