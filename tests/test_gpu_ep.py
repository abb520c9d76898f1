"""Expert parallelism through the C ABI (moe_layer_forward_ep) on one GPU: the
ranks of a world are run one after another on the same device and their
partial outputs summed, as the all-reduce of int4_routed_expert_softmax_b200.ep
sums them across GPUs.  Each rank's expert table points every expert it does
not own (and the shared expert, except on rank 0) at a poison blob whose fp16
scales are NaN, so an expert that a rank wrongly reads turns its output NaN.
Checks: the summed partials match moe_layer_forward and the oracle within the
layer's tolerance, the whole range on one rank is moe_layer_forward bit for
bit, and the routing record is the full one on every rank.  Both decode paths
run: one token in the fused kernel, three tokens in the three-kernel path."""
import numpy as np
import pytest
import torch

import moe_inputs as mi
from tests._common import gpu_layer, oracle_layer_from_device, within_tolerance, ws_trace

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _moe():
    import int4_routed_expert_softmax_b200 as moe
    return moe


def _poison_tables(blobs, E, world):
    moe = _moe()
    from int4_routed_expert_softmax_b200 import ep
    poison = torch.full((blobs.shape[1],), 0xFF, dtype=torch.uint8, device=DEV)  # NaN scales
    tables = []
    for r in range(world):
        lo, hi = ep.expert_range(E, world, r)
        ptrs = [blobs[e].data_ptr() if lo <= e < hi else poison.data_ptr() for e in range(E)]
        ptrs.append(blobs[E].data_ptr() if ep.owns_shared(r) else poison.data_ptr())
        tables.append(torch.tensor(ptrs, dtype=torch.int64, device=DEV))
    return tables, poison


@pytest.mark.parametrize("name,T,world", [
    ("medium", 1, 2), ("medium", 1, 4), ("medium", 3, 2), ("medium", 3, 8),
    ("glm", 1, 2), ("glm", 1, 8), ("glm", 4, 4),
])
def test_partials_sum_to_the_layer(name, T, world):
    moe = _moe()
    from int4_routed_expert_softmax_b200 import ep
    if name == "glm":
        w = mi.shrink(mi.WORKLOADS["decode"], T=T, seed=610 + T)
    else:
        w = mi.Workload("ep", H=1024, I=256, E=64, k=8, T=T, seed=620 + T)
    x, Wr, blobs = mi.make_layer(w, 0, DEV, T=T)
    d = moe.dims(w.H, w.I, w.E, w.k)
    full, _, _ = gpu_layer(w, x, Wr, blobs)
    tables, poison = _poison_tables(blobs, w.E, world)
    total = torch.zeros((T, w.H), dtype=torch.float32, device=DEV)
    for r in range(world):
        lo, hi = ep.expert_range(w.E, world, r)
        ws = moe.alloc_workspace(d, T)
        out = torch.full((T, w.H), float("nan"), dtype=torch.float32, device=DEV)
        ep.partial_layer_forward(d, x, Wr, tables[r], out, ws, lo, hi, ep.owns_shared(r))
        torch.cuda.synchronize()
        assert torch.isfinite(out).all(), r
        tr = ws_trace(ws, d, T)
        assert tr["status"][0] == 0, tr["status"]
        if r == 0:
            idx0 = tr["idx"]
        assert np.array_equal(tr["idx"], idx0)                # every rank routes every token alike
        total += out
    got = total.cpu().numpy()
    ok, rel, mrel = within_tolerance(got, full.cpu().numpy())
    assert ok, (rel, mrel)
    ref = oracle_layer_from_device(x, Wr, blobs, w.H, w.I, w.E, w.k, trace=False)
    ok, rel, mrel = within_tolerance(got, ref)
    assert ok, (rel, mrel)


@pytest.mark.parametrize("T", [1, 3])
def test_whole_range_on_one_rank_is_the_layer(T):
    moe = _moe()
    from int4_routed_expert_softmax_b200 import ep
    w = mi.Workload("ep1", H=1024, I=256, E=64, k=8, T=T, seed=630 + T)
    x, Wr, blobs = mi.make_layer(w, 0, DEV, T=T)
    d = moe.dims(w.H, w.I, w.E, w.k)
    full, _, _ = gpu_layer(w, x, Wr, blobs)
    out = torch.empty_like(full)
    ep.partial_layer_forward(d, x, Wr, moe.expert_table(blobs), out, moe.alloc_workspace(d, T), 0, w.E, True)
    torch.cuda.synchronize()
    assert torch.equal(out, full)


def test_rank_without_union_experts_gives_zero_or_shared():
    """An expert range that the tokens never select: the partial is 0 without
    the shared expert, and the shared expert's output with it."""
    moe = _moe()
    from int4_routed_expert_softmax_b200 import ep
    w = mi.Workload("ep0", H=1024, I=256, E=64, k=8, T=1, seed=640)
    x, Wr, blobs = mi.make_layer(w, 0, DEV)
    d = moe.dims(w.H, w.I, w.E, w.k)
    _, ws0, _ = gpu_layer(w, x, Wr, blobs)
    sel = set(ws_trace(ws0, d, 1)["idx"].reshape(-1).tolist())
    free = next(e for e in range(w.E) if e not in sel)
    table = moe.expert_table(blobs)
    out = torch.full((1, w.H), float("nan"), device=DEV)
    ep.partial_layer_forward(d, x, Wr, table, out, moe.alloc_workspace(d, 1), free, free + 1, False)
    torch.cuda.synchronize()
    assert torch.count_nonzero(out) == 0
    ep.partial_layer_forward(d, x, Wr, table, out, moe.alloc_workspace(d, 1), free, free + 1, True)
    torch.cuda.synchronize()
    # the shared expert's output: the layer with every routing weight's expert excluded
    ref = oracle_layer_from_device(x, Wr, blobs, w.H, w.I, w.E, w.k, trace=True)[1]["y"][0, w.k]
    ok, rel, mrel = within_tolerance(out.cpu().numpy()[0], ref)
    assert ok, (rel, mrel)


def test_bad_ranges_are_refused():
    moe = _moe()
    from int4_routed_expert_softmax_b200 import ep
    w = mi.WORKLOADS["tiny"]
    x, Wr, blobs = mi.make_layer(w, 0, DEV)
    d = moe.dims(w.H, w.I, w.E, w.k)
    out = torch.empty((w.T, w.H), device=DEV)
    ws = moe.alloc_workspace(d, w.T)
    for lo, hi in [(-1, 4), (5, 4), (0, w.E + 1)]:
        with pytest.raises(moe.MoeError):
            ep.partial_layer_forward(d, x, Wr, moe.expert_table(blobs), out, ws, lo, hi, True)
