"""The fused decode kernel's control words without a memset before the launch.

CTA 0 of the kernel zeroes the grid's arrival counter, the slot counters and
the status word, then publishes the call's sequence number; the other CTAs
wait for it before they touch any of them, and CTA 0 clears it again once all
have arrived.  Checks: a first call on a workspace full of stale bytes equals
a call on a zeroed one bit for bit; a CUDA graph of several calls (the same
sequence numbers on every replay) replays to the eager results bit for bit,
every time; the union kernels' memset path and the fused path share one
workspace in either order; and the MXFP4 token-by-token path, whose later
launches keep the status word, still reports success."""
import numpy as np
import pytest
import torch

import moe_inputs as mi
from tests._common import within_tolerance, oracle_layer_from_device, ws_trace

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _moe():
    import int4_routed_expert_softmax_b200 as moe
    return moe


def _case(name, T):
    if name == "glm":
        return mi.shrink(mi.WORKLOADS["decode"], T=T, seed=900 + T)
    return mi.Workload("ctrl", H=1024, I=256, E=64, k=8, T=T, seed=910 + T)


def _call(d, x, Wr, table, ws, path=0):
    moe = _moe()
    out = torch.full((x.shape[0], d.H), float("nan"), dtype=torch.float32, device=DEV)
    moe.moe_layer_forward(d, x, Wr, table, out, ws, path=path)
    return out


@pytest.mark.parametrize("name,T", [("medium", 1), ("medium", 4), ("glm", 1), ("glm", 3)])
@pytest.mark.parametrize("fill", [0xA5, 0xFF])
def test_first_call_on_a_stale_workspace(name, T, fill):
    moe = _moe()
    w = _case(name, T)
    x, Wr, blobs = mi.make_layer(w, 0, DEV, T=T)
    d = moe.dims(w.H, w.I, w.E, w.k)
    table = moe.expert_table(blobs)
    clean = moe.alloc_workspace(d, T)
    clean.zero_()
    ref = _call(d, x, Wr, table, clean)
    stale = moe.alloc_workspace(d, T)
    stale.fill_(fill)
    got = _call(d, x, Wr, table, stale)
    torch.cuda.synchronize()
    assert ws_trace(stale, d, T)["status"][0] == 0
    assert torch.equal(got, ref)


@pytest.mark.parametrize("name,T", [("medium", 1), ("medium", 3), ("glm", 1), ("glm", 16)])
def test_graph_replays_equal_eager(name, T):
    moe = _moe()
    w = _case(name, T)
    _, Wr, blobs = mi.make_layer(w, 0, DEV, T=T)
    d = moe.dims(w.H, w.I, w.E, w.k)
    table = moe.expert_table(blobs)
    xs = [mi.make_x(T, w.H, mi.sub_seed(w.seed, i, 1), DEV) for i in range(3)]
    ws = moe.alloc_workspace(d, T)
    eager = [_call(d, x, Wr, table, ws) for x in xs]
    torch.cuda.synchronize()
    outs = [torch.empty_like(e) for e in eager]
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):  # warm the launch path on a side stream
        moe.moe_layer_forward(d, xs[0], Wr, table, outs[0], ws)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for x, o in zip(xs, outs):
            moe.moe_layer_forward(d, x, Wr, table, o, ws)
    for _ in range(3):
        for o in outs:
            o.fill_(float("nan"))
        g.replay()
        torch.cuda.synchronize()
        assert ws_trace(ws, d, T)["status"][0] == 0
        for o, e in zip(outs, eager):
            assert torch.equal(o, e)
    # an eager call between replays (a new sequence number) changes nothing
    again = _call(d, xs[1], Wr, table, ws)
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(again, eager[1])
    for o, e in zip(outs, eager):
        assert torch.equal(o, e)
    del g


@pytest.mark.parametrize("T", [1, 4])
def test_union_path_and_fused_path_share_a_workspace(T):
    """The union kernels leave their counters set; the fused kernel after
    them, and they after it, still compute the layer."""
    moe = _moe()
    w = _case("medium", T)
    x, Wr, blobs = mi.make_layer(w, 0, DEV, T=T)
    d = moe.dims(w.H, w.I, w.E, w.k)
    table = moe.expert_table(blobs)
    ws = moe.alloc_workspace(d, T, path=1)
    fused0 = _call(d, x, Wr, table, ws)
    union = _call(d, x, Wr, table, ws, path=1)
    fused1 = _call(d, x, Wr, table, ws)
    union1 = _call(d, x, Wr, table, ws, path=1)
    torch.cuda.synchronize()
    assert torch.equal(fused0, fused1)
    assert torch.equal(union, union1)
    ref = oracle_layer_from_device(x, Wr, blobs, w.H, w.I, w.E, w.k, trace=False)
    ok, rel, mrel = within_tolerance(fused1.cpu().numpy(), ref)
    assert ok, (rel, mrel)


def test_mxfp4_token_by_token_on_a_stale_workspace():
    moe = _moe()
    w = mi.Workload("ctrlmx", H=1024, I=256, E=64, k=8, T=20, seed=930)
    x = mi.make_x(20, w.H, mi.sub_seed(w.seed, 0, 1), DEV)
    Wr = mi.make_router(w.E, w.H, mi.sub_seed(w.seed, 0, 2), DEV)
    blobs = mi.make_blobs_mx(w.H, w.I, w.E + 1, mi.sub_seed(w.seed, 0, 3), DEV)
    d = moe.dims(w.H, w.I, w.E, w.k)
    ws = moe.alloc_workspace(d, 20, path=1)
    ws.fill_(0x5A)
    out = torch.full((20, w.H), float("nan"), device=DEV)
    moe.moe_layer_forward_mxfp4(d, x, Wr, moe.expert_table(blobs), out, ws)
    torch.cuda.synchronize()
    v = moe.moe_workspace_view(d, 20, ws)
    assert moe.ws_slice(ws, v.status, (4,), torch.int32).cpu().numpy()[0] == 0
    ref = oracle_layer_from_device(x, Wr, blobs, w.H, w.I, w.E, w.k, fmt="mxfp4", trace=False)
    ok, rel, mrel = within_tolerance(out.cpu().numpy(), ref)
    assert ok, (rel, mrel)
    assert np.isfinite(out.cpu().numpy()).all()
