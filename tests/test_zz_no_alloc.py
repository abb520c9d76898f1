"""moe_layer_forward_static: the layer for callers that cannot allocate device
memory (hosts that own and budget all device memory, or paths that must not
allocate once running).  Its workspace is a static device array inside the
library; the test checks, through the C ABI, that two calls in a row give the
output of moe_layer_forward with a caller workspace bit for bit (both run the
same kernels in the same order, and each kernel is deterministic), and that
batches too large for the static workspace are refused on the host.  Kept in
its own file, collected last."""
import ctypes

import numpy as np
import pytest
import torch

import moe_inputs as mi
from tests._common import within_tolerance

DEV = "cuda"


@pytest.mark.gpu
@pytest.mark.parametrize("name,T", [("tiny", 4), ("decode", 1), ("decode", 16)])
def test_static_workspace_entry_matches_workspace_entry(name, T):
    import int4_routed_expert_softmax_b200 as moe
    w = mi.shrink(mi.WORKLOADS[name], seed=300 + T)
    x, Wr, blobs = mi.make_layer(w, 0, DEV, T=T)
    d = moe.dims(w.H, w.I, w.E, w.k)
    table = moe.expert_table(blobs)
    ref = torch.empty((T, w.H), dtype=torch.float32, device=DEV)
    moe.moe_layer_forward(d, x, Wr, table, ref, moe.alloc_workspace(d, T))
    torch.cuda.synchronize()
    ref_h = ref.cpu().numpy()
    for call in range(2):
        out = torch.full((T, w.H), float("nan"), dtype=torch.float32, device=DEV)
        moe.moe_layer_forward_static(d, x, Wr, table, out)
        torch.cuda.synchronize()
        got = out.cpu().numpy()
        ok, rel, mrel = within_tolerance(got, ref_h)
        assert ok, (call, rel, mrel)
        assert np.array_equal(got.view(np.uint32), ref_h.view(np.uint32)), call


def test_static_workspace_refuses_oversized_batches():
    """Host-side size check: no device work is issued for a refused call."""
    import int4_routed_expert_softmax_b200 as moe
    d = moe.dims(8192, 4096, 1024, 32)
    T = 64
    assert moe.moe_workspace_bytes(d, T) > (4 << 20)
    fake = ctypes.c_void_p(4096)
    rc = moe.lib().moe_layer_forward_static(ctypes.byref(d), T, fake, fake, fake, fake, None, 0, None)
    assert rc == -4  # MOE_ERR_WORKSPACE
