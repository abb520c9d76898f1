"""Tiered decode through the expert cache (GPU): placement changes speed, never
results -- the tiered output is bitwise the output with every expert resident
(colibri deep review, design rule "never silently change precision or router
semantics") -- plus the oracle on the stacked chain, and the cache's counters."""
import numpy as np
import pytest
import torch

import moe_inputs as mi
import oracle as orc
from tests._common import check_traced, within_tolerance, ws_trace

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _setup(H, I, E, k, L, seed, zipf=None):
    w = mi.Workload("tiered-small", H=H, I=I, E=E, k=k, T=1, layers=L, zipf_s=zipf, seed=seed)
    routers = [mi.make_router(E, H, mi.sub_seed(seed, l, 2), DEV, zipf_s=zipf) for l in range(L)]
    dev_blobs = [mi.make_blobs(H, I, E + 1, mi.sub_seed(seed, l, 3), DEV) for l in range(L)]
    host = [[dev_blobs[l][e].cpu().pin_memory() for e in range(E + 1)] for l in range(L)]
    return w, routers, dev_blobs, host


@pytest.mark.parametrize("per_layer", [12, 40])
def test_tiered_bitwise_equals_resident(per_layer):
    import int4_routed_expert_softmax_b200 as moe
    from int4_routed_expert_softmax_b200 import _cache as C
    H, I, E, k, L, NT = 1024, 256, 64, 8, 3, 12
    w, routers, dev_blobs, host = _setup(H, I, E, k, L, 21, zipf=1.1)
    d = moe.dims(H, I, E, k)
    cache = C.ExpertCache(d, L, host, per_layer * L * w.blob_bytes, C.MOE_CACHE_DEVICE)
    ws = moe.alloc_workspace(d, 1)
    ws_pred = moe.alloc_workspace(d, 1)
    ws_res = moe.alloc_workspace(d, 1)
    tables = [moe.expert_table(b) for b in dev_blobs]
    side = torch.cuda.Stream()
    x0 = mi.make_x(NT, H, 5, "cpu", zipf=True).numpy()
    out_t = torch.empty((1, H), device=DEV)
    out_r = torch.empty((1, H), device=DEV)
    predicted = 0
    for t in range(NT):
        x = x0[t:t + 1]
        for l in range(L):
            xd = torch.from_numpy(x).to(DEV)
            started, npred = cache.tiered_layer_forward(
                l, xd, routers[l], out_t, ws, ws_pred=ws_pred,
                Wr_next=routers[l + 1] if l + 1 < L else None, side_stream=side)
            predicted += npred
            moe.moe_layer_forward(d, xd, routers[l], tables[l], out_r, ws_res)
            torch.cuda.synchronize()
            assert torch.equal(out_t, out_r), (t, l)
            x = mi.chain_next(x, out_t.cpu().numpy(), zipf=True)
    st = cache.stats()
    assert st["misses"] > 0 and st["bytes_h2d"] == (st["misses"] + st["prefetches"]) * w.blob_bytes
    assert predicted > 0
    if per_layer == 12:
        assert st["evictions"] > 0
    cache.close()


def test_tiered_chain_matches_oracle():
    """Two tokens through 3 stacked layers: at every layer the oracle runs on
    the tiered path's own input (the chain of the path's outputs), and the
    call's routing, h codes and outputs are checked against it."""
    import int4_routed_expert_softmax_b200 as moe
    from int4_routed_expert_softmax_b200 import _cache as C
    H, I, E, k, L = 1024, 256, 64, 8, 3
    w, routers, dev_blobs, host = _setup(H, I, E, k, L, 33, zipf=1.1)
    d = moe.dims(H, I, E, k)
    cache = C.ExpertCache(d, L, host, 16 * L * w.blob_bytes, C.MOE_CACHE_DEVICE)
    ws = moe.alloc_workspace(d, 1)
    side = torch.cuda.Stream()
    hb = [np.stack([b.numpy() for b in layer]) for layer in host]
    Wh = [r.cpu().numpy() for r in routers]
    x0 = mi.make_x(2, H, 8, "cpu", zipf=True).numpy()
    out = torch.empty((1, H), device=DEV)
    for t in range(2):
        xg = x0[t:t + 1]
        for l in range(L):
            cache.tiered_layer_forward(l, torch.from_numpy(xg).to(DEV), routers[l], out, ws,
                                       side_stream=side)
            torch.cuda.synchronize()
            got = out.cpu().numpy()
            ref, tr = orc.moe_layer(xg, Wh[l], hb[l], H, I, E, k, trace=True)
            check_traced(got, ref, ws_trace(ws, d, 1), tr, hb[l], w, 1)
            xg = mi.chain_next(xg, got, zipf=True)
    cache.close()


def test_copy_fault_is_reported_and_recoverable():
    """A copy failure injected on the host surfaces as an error status of the
    call (no GPU fault); the cache keeps working afterwards."""
    import int4_routed_expert_softmax_b200 as moe
    from int4_routed_expert_softmax_b200 import _cache as C
    H, I, E, k, L = 512, 256, 16, 2, 1
    w, routers, dev_blobs, host = _setup(H, I, E, k, L, 44)
    d = moe.dims(H, I, E, k)
    cache = C.ExpertCache(d, L, host, 6 * w.blob_bytes, C.MOE_CACHE_DEVICE)
    ws = moe.alloc_workspace(d, 1)
    x = mi.make_x(1, H, 3, DEV)
    out = torch.empty((1, H), device=DEV)
    C.inject_fault(C.MOE_FAULT_COPY, 1, cache)
    with pytest.raises(moe.MoeError) as ex:
        cache.tiered_layer_forward(0, x, routers[0], out, ws)
    assert ex.value.status == -3
    cache.tiered_layer_forward(0, x, routers[0], out, ws)
    ref = torch.empty_like(out)
    moe.moe_layer_forward(d, x, routers[0], moe.expert_table(dev_blobs[0]), ref,
                          moe.alloc_workspace(d, 1))
    torch.cuda.synchronize()
    assert torch.equal(out, ref)
    cache.close()
