"""Bounded device waits that run out, without a GPU fault (failure handling).

Every wait of a kernel for data is bounded; moe_set_wait_limit shortens the
bound so that the waits of a healthy call run out.  Each case checks that the
call then reports MOE_ERR_TIMEOUT with the detail code of the wait that gave up
in the workspace status word, that the copies and MMAs already issued were
drained (the device stays usable: nothing faults), and that the next call with
the default limit matches the oracle again.  The pages' engine degrades with a
warning instead of crashing when a source fails (tantan.ink page, section
我看到的几个坑); here a device wait that runs out is reported, not trapped."""
import numpy as np
import pytest
import torch

import moe_inputs as mi
from tests._common import check_layer, gpu_layer

pytestmark = pytest.mark.gpu

DEV = "cuda"
SHORT = 200                       # SM clocks: shorter than any copy from HBM takes
MOE_ERR_TIMEOUT = -7
ROUTE_DETAILS = {1, 40, 42, 48}   # the routing kernel's staging wait; the fused kernel's, its grid
                                  # arrival, its wait for CTA 0's zeroed control words
EXPERT_DETAILS = {10, 11, 20, 21}  # gate/up and down: stage landed / stage freed
PREFILL_DETAILS = {31, 32, 33, 34}  # grouped GEMM: operands landed / freed, accumulators


def _moe():
    import int4_routed_expert_softmax_b200 as moe
    return moe


@pytest.fixture(autouse=True)
def default_limit_after():
    yield
    _moe().moe_set_wait_limit(0)


def _status(moe, d, T, ws):
    v = moe.moe_workspace_view(d, T, ws)
    return moe.ws_slice(ws, v.status, (4,), torch.int32).cpu().numpy()


def _medium():
    return mi.Workload("timeout", H=1024, I=256, E=64, k=8, T=1, seed=71)


def test_wait_limit_setter_round_trip():
    moe = _moe()
    default = moe.moe_set_wait_limit(0)
    assert default == 2_000_000_000
    assert moe.moe_set_wait_limit(SHORT) == default
    assert moe.moe_set_wait_limit(-1) == SHORT
    assert moe.moe_set_wait_limit(0) == default


@pytest.mark.parametrize("name", ["tiny", "medium"])
def test_routing_wait_runs_out_then_recovers(name):
    """tiny: four tokens; medium: one token (the auto path's decode kernels)."""
    moe = _moe()
    w = mi.WORKLOADS["tiny"] if name == "tiny" else _medium()
    x, Wr, blobs = mi.make_layer(w, 0, DEV)
    T = x.shape[0]
    ref_out, ws, d = gpu_layer(w, x, Wr, blobs)          # default limit: loads the kernels
    table = moe.expert_table(blobs)
    out = torch.full_like(ref_out, float("nan"))
    moe.moe_set_wait_limit(SHORT)
    moe.moe_layer_forward(d, x, Wr, table, out, ws)
    torch.cuda.synchronize()
    st = _status(moe, d, T, ws)
    assert st[0] == MOE_ERR_TIMEOUT and st[1] in ROUTE_DETAILS, st
    moe.moe_set_wait_limit(0)
    moe.moe_layer_forward(d, x, Wr, table, out, ws)      # the same workspace, reset by the call
    torch.cuda.synchronize()
    assert _status(moe, d, T, ws)[0] == 0
    assert torch.equal(out, ref_out)
    check_layer(w, x, Wr, blobs)


@pytest.mark.parametrize("T", [1, 3])
def test_expert_waits_run_out_then_recover(T):
    """The routing half runs with the default limit, the experts half with the
    short one: the gate/up kernel's waits run out, the down kernel skips."""
    moe = _moe()
    from int4_routed_expert_softmax_b200 import _cache as C
    w = mi.shrink(_medium(), T=T)
    x, Wr, blobs = mi.make_layer(w, 0, DEV, T=T)
    ref_out, ws, d = gpu_layer(w, x, Wr, blobs)
    table = moe.expert_table(blobs)
    out = torch.full_like(ref_out, float("nan"))
    C.moe_layer_route(d, x, Wr, ws)
    moe.moe_set_wait_limit(SHORT)
    C.moe_layer_experts(d, T, table, out, ws)
    torch.cuda.synchronize()
    st = _status(moe, d, T, ws)
    assert st[0] == MOE_ERR_TIMEOUT and st[1] in EXPERT_DETAILS, st
    moe.moe_set_wait_limit(0)
    C.moe_layer_route(d, x, Wr, ws)
    C.moe_layer_experts(d, T, table, out, ws)
    torch.cuda.synchronize()
    assert _status(moe, d, T, ws)[0] == 0
    assert torch.equal(out, ref_out)


def test_prefill_waits_run_out_then_recover():
    moe = _moe()
    w = mi.WORKLOADS["tiny"]
    x, Wr, blobs = mi.make_layer(w, 0, DEV, T=40)
    T = x.shape[0]
    ref_out, ws, d = gpu_layer(w, x, Wr, blobs, path=2)
    table = moe.expert_table(blobs)
    out = torch.zeros_like(ref_out)
    moe.moe_set_wait_limit(SHORT)
    moe.moe_layer_forward(d, x, Wr, table, out, ws, path=2)
    torch.cuda.synchronize()
    st = _status(moe, d, T, ws)
    assert st[0] == MOE_ERR_TIMEOUT and st[1] in PREFILL_DETAILS, st
    moe.moe_set_wait_limit(0)
    moe.moe_layer_forward(d, x, Wr, table, out, ws, path=2)
    torch.cuda.synchronize()
    assert _status(moe, d, T, ws)[0] == 0
    assert torch.equal(out, ref_out)
    check_layer(w, x, Wr, blobs, path=2)


def test_binary_built_for_sm100a():
    """The kernels the device loaded were built for sm_100a (a runtime query,
    no binary tools)."""
    assert _moe().moe_device_binary_version() == 100
