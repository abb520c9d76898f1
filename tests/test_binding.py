"""The Python binding refuses wrong tensors before their addresses reach the C
ABI (which sees only pointers): memory space, dtype, contiguity, shape and
minimum size.  Every case raises on the host, so no GPU is needed."""
import pytest
import torch

import int4_routed_expert_softmax_b200 as moe

D = moe.dims(256, 128, 16, 2)


def _host_call(x=None, out=None, Wr=None, table=None):
    x = torch.zeros((4, 256), dtype=torch.float32) if x is None else x
    out = torch.zeros((4, 256), dtype=torch.float32) if out is None else out
    Wr = torch.zeros((16, 256), dtype=torch.float32) if Wr is None else Wr
    table = torch.zeros(17, dtype=torch.int64) if table is None else table
    ws = torch.zeros(1 << 16, dtype=torch.uint8)
    moe.moe_layer_forward_host(D, x, Wr, table, out, ws)


def test_device_entry_refuses_host_tensors():
    x = torch.zeros((4, 256), dtype=torch.float32)
    with pytest.raises(ValueError, match="device memory"):
        moe.moe_layer_forward(D, x, x, x, x, x)
    with pytest.raises(ValueError, match="device memory"):
        moe.moe_quant_q8_0(x, torch.zeros((4, 256), dtype=torch.int8), torch.zeros((4, 8)))


def test_host_entry_checks_host_buffers_first():
    with pytest.raises(ValueError, match="float32"):
        _host_call(x=torch.zeros((4, 256), dtype=torch.float64))
    with pytest.raises(ValueError, match=r"\[T\]\[256\]"):
        _host_call(x=torch.zeros((4, 128), dtype=torch.float32))
    with pytest.raises(ValueError, match="at least 1024"):
        _host_call(out=torch.zeros((3, 256), dtype=torch.float32))
    with pytest.raises(ValueError, match="contiguous"):
        _host_call(x=torch.zeros((256, 4), dtype=torch.float32).t())
    # the router weights must be device memory: reached once the host buffers pass
    with pytest.raises(ValueError, match="Wr must be in device memory"):
        _host_call()
