"""MXFP4 expert blobs (32 E2M1 codes per E8M0 exponent: the Kimi K3 row of the
model-family table on the colibri deep review page) through the C ABI
(moe_layer_forward_mxfp4, the fused one-token decode kernel) against the
oracle's MXFP4 layer.  Routing does not depend on the weight format and is
checked bit for bit; the h codes within the flip bound; the outputs within
the layer's tolerance (and within 1e-5 of the oracle's down projection of the
path's own h codes)."""
import numpy as np
import pytest
import torch

import moe_inputs as mi
from tests._common import check_traced, oracle_layer_from_device, within_tolerance, ws_trace

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _moe():
    import int4_routed_expert_softmax_b200 as moe
    return moe


def _layer_mx(w, T, seed):
    x = mi.make_x(T, w.H, mi.sub_seed(seed, 0, 1), DEV)
    Wr = mi.make_router(w.E, w.H, mi.sub_seed(seed, 0, 2), DEV)
    blobs = mi.make_blobs_mx(w.H, w.I, w.E + 1, mi.sub_seed(seed, 0, 3), DEV)
    return x, Wr, blobs


def _run(w, x, Wr, blobs, counts=None):
    moe = _moe()
    d = moe.dims(w.H, w.I, w.E, w.k)
    T = x.shape[0]
    ws = moe.alloc_workspace(d, T, path=1)
    out = torch.full((T, w.H), float("nan"), dtype=torch.float32, device=DEV)
    moe.moe_layer_forward_mxfp4(d, x, Wr, moe.expert_table(blobs), out, ws, route_counts=counts)
    torch.cuda.synchronize()
    return out, ws, d


@pytest.mark.parametrize("H,I,E,k", [(256, 128, 16, 2), (1024, 256, 64, 8), (384, 384, 5, 5),
                                     (8192, 4096, 8, 2), (6144, 2048, 256, 8)])
def test_mxfp4_one_token_matches_oracle(H, I, E, k):
    w = mi.Workload("mx", H=H, I=I, E=E, k=k, T=1, seed=700 + E)
    x, Wr, blobs = _layer_mx(w, 1, w.seed)
    out, ws, d = _run(w, x, Wr, blobs)
    ref, tr = oracle_layer_from_device(x, Wr, blobs, H, I, E, k, fmt="mxfp4")
    check_traced(out.cpu().numpy(), ref, ws_trace(ws, d, 1), tr, blobs, w, 1, fmt="mxfp4")


def test_mxfp4_batch_token_by_token():
    moe = _moe()
    w = mi.Workload("mxb", H=1024, I=256, E=64, k=8, T=3, seed=750)
    x, Wr, blobs = _layer_mx(w, 3, w.seed)
    counts = torch.zeros(w.E, dtype=torch.int32, device=DEV)
    out, _, d = _run(w, x, Wr, blobs, counts)
    ref, tr = oracle_layer_from_device(x, Wr, blobs, w.H, w.I, w.E, w.k, fmt="mxfp4")
    ok, rel, mrel = within_tolerance(out.cpu().numpy(), ref)
    assert ok, (rel, mrel)
    assert np.array_equal(counts.cpu().numpy(), np.bincount(tr["idx"].reshape(-1), minlength=w.E))
    again = torch.empty_like(out)
    moe.moe_layer_forward_mxfp4(d, x, Wr, moe.expert_table(blobs), again, moe.alloc_workspace(d, 3, path=1))
    torch.cuda.synchronize()
    assert torch.equal(out, again)          # deterministic
