"""Parity of the prefill path (router GEMM, top-k, bucketing, grouped GEMM over
the expert union on the tensor cores, combine) with the CPU oracle, through the
C ABI with path = MOE_PATH_PREFILL.

Bit-exact: the Q8_0 codes and scales of x, the router logits, the top-k
indices, the bucket counts / offsets / union / permutation; the softmax weights
within 1e-6 relative (CUDA's expf against the C library's).
Final outputs: within rel-L2 <= 1e-4 and max-abs <= 2e-3 * rms(ref).  The
grouped GEMM multiplies the weights by an fp16 hi/lo split of the dequantised
activations (22 significant bits) and accumulates in fp32 in another order
than the oracle, so its sums differ from the oracle's by about 1e-6 relative
and a Q8_0 code of SiLU(g)*u may differ by one where h lies within that of a
half-integer multiple of its block scale; those flips are counted and bounded
(at most 1 in 1000 codes, never by more than one)."""
import numpy as np
import pytest
import torch

import moe_inputs as mi
import oracle as orc
from tests._common import (check_hq, check_layer, check_routing, gpu_layer, hq_by_slot, oracle_layer_from_device,
                           out_from_codes, W_RTOL, within_tolerance, ws_trace)

pytestmark = pytest.mark.gpu

DEV = "cuda"
PREFILL = 2
DECODE = 1


def _moe():
    import int4_routed_expert_softmax_b200 as moe
    return moe


def _check_full(w, x, Wr, blobs):
    out, ref, _ = check_layer(w, x, Wr, blobs, path=PREFILL)
    return out, ref


@pytest.mark.parametrize("T", [1, 4, 37, 300])
def test_prefill_tiny(T):
    """T = 300 puts 300 rows on the shared expert: token tiles of 128, 128, 44."""
    w = mi.WORKLOADS["tiny"]
    x, Wr, blobs = mi.make_layer(w, 0, DEV, T=T)
    _check_full(w, x, Wr, blobs)


@pytest.mark.parametrize("H,I,E,k,T", [
    (384, 384, 5, 5, 40),     # k = E: every expert in the union, ragged group count
    (128, 128, 1, 1, 130),    # one expert with 130 rows: a 2-row token tile
    (1024, 256, 64, 8, 64),
    (256, 128, 16, 2, 17),
    (8192, 4096, 8, 2, 6),    # widest accepted shape
])
def test_prefill_shapes(H, I, E, k, T):
    w = mi.Workload("shape", H=H, I=I, E=E, k=k, T=T, seed=H + I + E + k + T)
    x, Wr, blobs = mi.make_layer(w, 0, DEV)
    _check_full(w, x, Wr, blobs)


def test_prefill_glm_T16_matches_decode_path():
    """One 16-token batch of the GLM-shaped layer on both paths: each within
    the layer's tolerance of the oracle, and of each other."""
    w = mi.WORKLOADS["stacked"]
    x, Wr, blobs = mi.make_layer(w, 1, DEV, T=16)
    out_pf, ref = _check_full(w, x, Wr, blobs)
    out_dc, _, _ = check_layer(w, x, Wr, blobs, path=DECODE)
    ok, rel, mrel = within_tolerance(out_pf.cpu().numpy(), out_dc.cpu().numpy())
    assert ok, (rel, mrel)


def test_prefill_zero_rows_and_repeat():
    w = mi.WORKLOADS["tiny"]
    x, Wr, blobs = mi.make_layer(w, 0, DEV, T=24)
    x[3] = 0.0
    x[17] = 0.0
    out1, _ = _check_full(w, x, Wr, blobs)
    out2, _, _ = gpu_layer(w, x, Wr, blobs, path=PREFILL)
    assert torch.equal(out1, out2)    # no atomics: bitwise reproducible


def test_prefill_glm_full_size_sampled():
    """The benchmarked prefill batch: 2048 tokens, Zipf(1.1)-biased routing over
    256 experts.  Routing and bucketing are checked in full (the oracle router
    on every token); outputs on sampled tokens, including the first and last
    rows of the shared expert's tiles and tokens of the least-used experts."""
    w = mi.WORKLOADS["prefill"]
    x, Wr, blobs = mi.make_layer(w, 0, DEV)
    T = x.shape[0]
    out, ws, d = gpu_layer(w, x, Wr, blobs, path=PREFILL)
    g = ws_trace(ws, d, T)
    assert g["status"][0] == 0, g["status"]
    xh, wh = x.cpu().numpy(), Wr.cpu().numpy()
    xq, xd = orc.quant_q8_0(xh)
    assert np.array_equal(g["xq"], xq)
    assert np.array_equal(g["xd"].view(np.uint32), xd.view(np.uint32))
    lg = orc.router_logits(xh, wh)
    assert np.array_equal(g["logits"].view(np.uint32), lg.view(np.uint32))
    idx, wt = orc.topk_softmax(lg, w.k)
    assert np.array_equal(g["idx"], idx)
    assert np.all(np.abs(g["w"].astype(np.float64) - wt) <= W_RTOL * np.abs(wt.astype(np.float64)))
    cnt, off, uni, n, perm = orc.bucket(idx, w.E)
    assert np.array_equal(g["cnt"], cnt) and np.array_equal(g["off"], off)
    assert g["n_uni"] == n and np.array_equal(g["uni"], uni)
    assert np.array_equal(g["perm"], perm)
    # sampled outputs
    rare = [e for e in uni if cnt[e] <= 2][:2]
    toks = {0, 1, 127, 128, 1023, 2046, 2047}
    for e in rare:
        toks.add(int(perm[off[e]]) // w.k)
    toks = sorted(toks)
    ref = oracle_layer_from_device(x, Wr, blobs, w.H, w.I, w.E, w.k, tokens=toks)
    ok, rel, mrel = within_tolerance(out.cpu().numpy()[toks], ref)
    assert ok, (rel, mrel)


def test_prefill_misaligned_blob_reports_device_error():
    moe = _moe()
    w = mi.WORKLOADS["tiny"]
    x, Wr, blobs = mi.make_layer(w, 0, DEV, T=20)
    d = moe.dims(w.H, w.I, w.E, w.k)
    raw = torch.empty(blobs.numel() + 64, dtype=torch.uint8, device=DEV)
    base = raw[8:8 + blobs.numel()].view(w.E + 1, -1)
    base.copy_(blobs)
    ws = moe.alloc_workspace(d, x.shape[0], path=PREFILL)
    out = torch.zeros((x.shape[0], w.H), device=DEV)
    moe.moe_layer_forward(d, x, Wr, moe.expert_table(base), out, ws, path=PREFILL)
    torch.cuda.synchronize()
    st = moe.ws_slice(ws, moe.moe_workspace_view(d, x.shape[0], ws).status, (4,), torch.int32).cpu()
    assert int(st[0]) == -8   # MOE_ERR_DEVICE


def test_prefill_small_workspace_refused():
    moe = _moe()
    w = mi.WORKLOADS["tiny"]
    x, Wr, blobs = mi.make_layer(w, 0, DEV, T=8)
    d = moe.dims(w.H, w.I, w.E, w.k)
    ws = moe.alloc_workspace(d, 8)               # decode-sized
    out = torch.zeros((8, w.H), device=DEV)
    with pytest.raises(moe.MoeError):
        moe.moe_layer_forward(d, x, Wr, moe.expert_table(blobs), out, ws, path=PREFILL)
