"""Parity of the CUDA path (through the C ABI) with the CPU oracle.

Bit-exact: Q8_0 codes and scales, router logits, top-k indices, bucket counts /
offsets / union / permutation.  Softmax weights within 1e-6 relative (CUDA's
expf against the C library's).  The Q8_0 codes of SiLU(g)*u: at most one in a
thousand differ, by one, from the oracle's -- the kernels sum each row's groups
in their own fixed order, the oracle in plain ascending order, and a code flips
where h lies within that rounding difference of a code boundary.  Final
outputs: within rel-L2 <= 1e-4 and max-abs <= 2e-3 * rms(ref)."""
import numpy as np
import pytest
import torch

import moe_inputs as mi
import oracle as orc
from tests._common import W_RTOL, check_layer, gpu_layer, oracle_layer_from_device, within_tolerance

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _moe():
    import int4_routed_expert_softmax_b200 as moe
    return moe


# ----------------------------------------------------------------- Q8_0
@pytest.mark.parametrize("rows,cols,scale", [(1, 256, 1.0), (7, 6144, 1.0), (33, 384, 1e-3),
                                             (2, 128, 1e4), (1, 32, 0.0)])
def test_quant_q8_0_bit_exact(rows, cols, scale):
    moe = _moe()
    x = mi.make_x(rows, cols, 11 + rows, DEV) * scale
    x[0, :32] = 0.0                       # a zero block
    if rows > 1:
        x[1, 5] = 1e-30                   # tiny amax
    q = torch.empty((rows, cols), dtype=torch.int8, device=DEV)
    d = torch.empty((rows, cols // 32), dtype=torch.float32, device=DEV)
    moe.moe_quant_q8_0(x, q, d)
    torch.cuda.synchronize()
    qo, do = orc.quant_q8_0(x.cpu().numpy())
    assert np.array_equal(q.cpu().numpy(), qo)
    assert np.array_equal(d.cpu().numpy().view(np.uint32), do.view(np.uint32))


# ----------------------------------------------------------------- router
def _weights_close(wt, wo):
    wg = wt.cpu().numpy().astype(np.float64)
    assert np.all(np.abs(wg - wo) <= W_RTOL * np.abs(wo.astype(np.float64))), np.abs(wg - wo).max()


@pytest.mark.parametrize("name,T", [("tiny", 4), ("decode", 1), ("decode", 16), ("decode", 37)])
def test_router_topk_bit_exact(name, T):
    moe = _moe()
    w = mi.WORKLOADS[name]
    x = mi.make_x(T, w.H, 5 + T, DEV)
    Wr = mi.make_router(w.E, w.H, 6, DEV)
    d = moe.dims(w.H, w.I, w.E, w.k)
    idx = torch.empty((T, w.k), dtype=torch.int32, device=DEV)
    wt = torch.empty((T, w.k), dtype=torch.float32, device=DEV)
    lg = torch.empty((T, w.E), dtype=torch.float32, device=DEV)
    cnt = torch.zeros(w.E, dtype=torch.int32, device=DEV)
    moe.moe_router_topk(d, x, Wr, idx, wt, lg, cnt)
    torch.cuda.synchronize()
    lo = orc.router_logits(x.cpu().numpy(), Wr.cpu().numpy())
    io, wo = orc.topk_softmax(lo, w.k)
    assert np.array_equal(lg.cpu().numpy().view(np.uint32), lo.view(np.uint32))
    assert np.array_equal(idx.cpu().numpy(), io)
    _weights_close(wt, wo)
    assert np.array_equal(cnt.cpu().numpy(), np.bincount(io.reshape(-1), minlength=w.E))


@pytest.mark.parametrize("E,k,T", [(512, 8, 5), (256, 16, 3), (1024, 32, 2), (40, 12, 7)])
def test_router_topk_selection_paths(E, k, T):
    # k <= 12 with E <= 256 takes the argmax-rounds selection, the rest the radix selection
    moe = _moe()
    H = 256
    x = mi.make_x(T, H, 21 + E, DEV)
    Wr = mi.make_router(E, H, 22 + k, DEV)
    d = moe.dims(H, 128, E, k)
    idx = torch.empty((T, k), dtype=torch.int32, device=DEV)
    wt = torch.empty((T, k), dtype=torch.float32, device=DEV)
    lg = torch.empty((T, E), dtype=torch.float32, device=DEV)
    moe.moe_router_topk(d, x, Wr, idx, wt, lg)
    torch.cuda.synchronize()
    io, wo = orc.topk_softmax(orc.router_logits(x.cpu().numpy(), Wr.cpu().numpy()), k)
    assert np.array_equal(idx.cpu().numpy(), io)
    _weights_close(wt, wo)


def test_router_ties_lower_index_first():
    moe = _moe()
    H, E, k, T = 256, 16, 4, 3
    Wr = mi.make_router(E, H, 9, DEV)
    Wr[5] = Wr[2]
    Wr[9] = Wr[2]            # experts 2, 5, 9 always tie
    Wr[12] = Wr[3]
    x = mi.make_x(T, H, 10, DEV)
    x[2] = 0.0               # every logit is zero: ties everywhere
    d = moe.dims(H, 128, E, k)
    idx = torch.empty((T, k), dtype=torch.int32, device=DEV)
    wt = torch.empty((T, k), dtype=torch.float32, device=DEV)
    lg = torch.empty((T, E), dtype=torch.float32, device=DEV)
    moe.moe_router_topk(d, x, Wr, idx, wt, lg)
    torch.cuda.synchronize()
    io, wo = orc.topk_softmax(orc.router_logits(x.cpu().numpy(), Wr.cpu().numpy()), k)
    assert np.array_equal(idx.cpu().numpy(), io)
    assert list(io[2]) == [0, 1, 2, 3]
    _weights_close(wt, wo)
    assert np.all(wt.cpu().numpy()[2] == 0.25)   # equal logits: e^0 = 1 exactly


# ----------------------------------------------------------------- bucket
@pytest.mark.parametrize("T,k,E", [(1, 8, 256), (4, 2, 16), (16, 8, 256), (300, 8, 256),
                                   (2048, 8, 256), (5, 3, 3), (64, 1, 1)])
def test_bucket_bit_exact(T, k, E):
    moe = _moe()
    rng = np.random.default_rng(T * 31 + E)
    if T >= 300:   # skewed popularity like the prefill workload
        p = 1.0 / np.arange(1, E + 1) ** 1.1
        p /= p.sum()
        io = np.array([rng.choice(E, size=k, replace=False, p=p) for _ in range(T)], np.int32)
    else:
        io = np.array([rng.permutation(E)[:k] for _ in range(T)], np.int32).reshape(T, k)
    d = moe.dims(128, 128, E, k)
    idx = torch.from_numpy(io).to(DEV)
    cnt = torch.empty(E, dtype=torch.int32, device=DEV)
    off = torch.empty(E + 1, dtype=torch.int32, device=DEV)
    uni = torch.empty(E + 1, dtype=torch.int32, device=DEV)
    nu = torch.empty(1, dtype=torch.int32, device=DEV)
    perm = torch.empty(max(T * k, 1), dtype=torch.int32, device=DEV)
    moe.moe_bucket(d, idx, cnt, off, uni, nu, perm)
    torch.cuda.synchronize()
    c, o, u, n, pm = orc.bucket(io, E)
    assert int(nu.item()) == n
    assert np.array_equal(cnt.cpu().numpy(), c)
    assert np.array_equal(off.cpu().numpy(), o)
    assert np.array_equal(uni.cpu().numpy()[:n], u)
    assert np.array_equal(perm.cpu().numpy()[:T * k], pm)


# ----------------------------------------------------------------- whole layer
def _check_layer(w, x, Wr, blobs, path=0):
    out, ref, _ = check_layer(w, x, Wr, blobs, path=path)
    return out, ref


def test_layer_tiny():
    w = mi.WORKLOADS["tiny"]
    x, Wr, blobs = mi.make_layer(w, 0, DEV)
    _check_layer(w, x, Wr, blobs)


@pytest.mark.parametrize("seed", [0, 1])
def test_layer_decode_glm_T1(seed):
    w = mi.shrink(mi.WORKLOADS["decode"], seed=100 + seed)
    x, Wr, blobs = mi.make_layer(w, 0, DEV)
    _check_layer(w, x, Wr, blobs)


@pytest.mark.parametrize("T", [2, 3, 4, 16])   # 2-3: draft-verification batch sizes
def test_layer_stacked_batches(T):
    w = mi.WORKLOADS["stacked"]
    x, Wr, blobs = mi.make_layer(w, 3, DEV, T=T)
    _check_layer(w, x, Wr, blobs)


@pytest.mark.parametrize("H,I,E,k,T", [
    (384, 384, 5, 5, 3),      # k = E, ragged group count (G = 6 per row)
    (128, 128, 1, 1, 2),      # a single expert
    (256, 128, 16, 2, 1),
    (1024, 256, 64, 8, 16),
    (8192, 4096, 8, 2, 2),    # widest accepted shape
])
def test_layer_shapes(H, I, E, k, T):
    w = mi.Workload("shape", H=H, I=I, E=E, k=k, T=T, seed=H + I + E + k + T)
    x, Wr, blobs = mi.make_layer(w, 0, DEV)
    _check_layer(w, x, Wr, blobs)


def test_layer_zero_rows_and_repeat():
    w = mi.WORKLOADS["tiny"]
    x, Wr, blobs = mi.make_layer(w, 0, DEV)
    x[1] = 0.0                        # all-zero hidden state: every block has d = 0
    out1, _ = _check_layer(w, x, Wr, blobs)
    out2, _, _ = gpu_layer(w, x, Wr, blobs)
    assert torch.equal(out1, out2)    # bitwise reproducible


def test_layer_T0_is_noop():
    moe = _moe()
    w = mi.WORKLOADS["tiny"]
    x, Wr, blobs = mi.make_layer(w, 0, DEV)
    d = moe.dims(w.H, w.I, w.E, w.k)
    ws = moe.alloc_workspace(d, 1)
    out = torch.empty((0, w.H), device=DEV)
    moe.moe_layer_forward(d, x[:0], Wr, moe.expert_table(blobs), out, ws)


def test_layer_chunked_decode_path_T40():
    """T > 16 on the decode path runs in chunks of 16 tokens."""
    w = mi.shrink(mi.WORKLOADS["decode"], seed=77)
    x, Wr, blobs = mi.make_layer(w, 0, DEV, T=40)
    out, ws, d = gpu_layer(w, x, Wr, blobs, path=1)
    toks = [0, 15, 16, 31, 39]
    ref = oracle_layer_from_device(x, Wr, blobs, w.H, w.I, w.E, w.k, tokens=toks)
    got = out.cpu().numpy()[toks]
    ok, rel, mrel = within_tolerance(got, ref)
    assert ok, (rel, mrel)


def test_layer_forward_host_matches_device():
    moe = _moe()
    w = mi.WORKLOADS["tiny"]
    x, Wr, blobs = mi.make_layer(w, 0, DEV)
    out_dev, ws, d = gpu_layer(w, x, Wr, blobs)
    xh = x.cpu().pin_memory()
    oh = torch.empty((x.shape[0], w.H), dtype=torch.float32).pin_memory()
    moe.moe_layer_forward_host(d, xh, Wr, moe.expert_table(blobs), oh, ws)
    torch.cuda.synchronize()
    assert torch.equal(oh, out_dev.cpu())


@pytest.mark.parametrize("pinned", [True, False])
def test_layer_forward_host_decode_T3(pinned):
    """The host-buffer entry on the decode path: pinned buffers go across in
    the staging kernel and the down kernel's own stores; pageable buffers
    through copies.  Both equal the device-buffer call bit for bit."""
    moe = _moe()
    w = mi.shrink(mi.WORKLOADS["decode"], seed=91)
    x, Wr, blobs = mi.make_layer(w, 0, DEV, T=3)
    out_dev, ws, d = gpu_layer(w, x, Wr, blobs)
    xh = x.cpu()
    oh = torch.full((3, w.H), float("nan"), dtype=torch.float32)
    if pinned:
        xh, oh = xh.pin_memory(), oh.pin_memory()
    for _ in range(2):
        moe.moe_layer_forward_host(d, xh, Wr, moe.expert_table(blobs), oh, ws)
        torch.cuda.synchronize()
        assert torch.equal(oh, out_dev.cpu())
        oh.fill_(float("nan"))


def test_route_counts_accumulate():
    moe = _moe()
    w = mi.WORKLOADS["tiny"]
    x, Wr, blobs = mi.make_layer(w, 0, DEV)
    d = moe.dims(w.H, w.I, w.E, w.k)
    ws = moe.alloc_workspace(d, x.shape[0])
    cnt = torch.zeros(w.E, dtype=torch.int32, device=DEV)
    out = torch.empty((x.shape[0], w.H), device=DEV)
    for _ in range(3):
        moe.moe_layer_forward(d, x, Wr, moe.expert_table(blobs), out, ws, route_counts=cnt)
    torch.cuda.synchronize()
    io, _ = orc.topk_softmax(orc.router_logits(x.cpu().numpy(), Wr.cpu().numpy()), w.k)
    assert np.array_equal(cnt.cpu().numpy(), 3 * np.bincount(io.reshape(-1), minlength=w.E))


def test_misaligned_blob_reports_device_error():
    """A 16-byte-misaligned expert pointer is refused by the kernels' own
    check (status word), never dereferenced by a bulk copy."""
    moe = _moe()
    w = mi.WORKLOADS["tiny"]
    x, Wr, blobs = mi.make_layer(w, 0, DEV)
    d = moe.dims(w.H, w.I, w.E, w.k)
    raw = torch.empty(blobs.numel() + 64, dtype=torch.uint8, device=DEV)
    base = raw[8:8 + blobs.numel()].view(w.E + 1, -1)
    base.copy_(blobs)
    ws = moe.alloc_workspace(d, x.shape[0])
    out = torch.zeros((x.shape[0], w.H), device=DEV)
    moe.moe_layer_forward(d, x, Wr, moe.expert_table(base), out, ws)
    torch.cuda.synchronize()
    st = moe.ws_slice(ws, moe.moe_workspace_view(d, x.shape[0], ws).status, (4,), torch.int32).cpu()
    assert int(st[0]) == -8   # MOE_ERR_DEVICE


@pytest.mark.parametrize("path", [1, 2])
def test_profile_records_each_call_and_leaves_output_unchanged(path):
    """Device-stamped per-call timing: one record per call with positive phase
    durations no longer than the call span, and bitwise the same output."""
    moe = _moe()
    w = mi.WORKLOADS["tiny"]
    x, Wr, blobs = mi.make_layer(w, 0, DEV)
    out0, ws, d = gpu_layer(w, x, Wr, blobs, path=path)
    moe.moe_profile_enable(True)
    try:
        out = torch.empty_like(out0)
        for _ in range(3):
            moe.moe_layer_forward(d, x, Wr, moe.expert_table(blobs), out, ws, path=path)
        rec = moe.moe_profile_read(16)
        again = moe.moe_profile_read(16)
    finally:
        moe.moe_profile_enable(False)
    assert torch.equal(out, out0)
    assert len(rec) == 3 and again == []
    for r in rec:
        assert all(v > 0 for v in r), r
        assert max(r[:3]) <= r[3] * (1 + 1e-6), r
        assert r[3] < 1000.0, r       # milliseconds


# ----------------------------------------------------------------- fused one-token kernel
@pytest.mark.parametrize("H,I,E,k,seed", [
    (256, 128, 16, 2, 1),        # tiny shape: most CTAs own no unit and no output row
    (1024, 256, 64, 8, 2),
    (384, 384, 5, 5, 3),         # k = E, ragged group count
    (128, 128, 1, 1, 4),         # a single expert
    (1024, 256, 1024, 32, 5),    # 7 router rows per CTA, k = 32
    (8192, 4096, 8, 2, 6),       # widest shape: down rows in two stages per slot
    (6144, 2048, 256, 8, 7),     # the GLM-5.2 decode layer
])
def test_fused_one_token_equals_three_kernel_path(H, I, E, k, seed):
    """One token runs in the fused cooperative kernel; the same layer split into
    moe_layer_route + moe_layer_experts runs the three-kernel path.  Both use the
    same per-row order, so every output and every intermediate agrees bit for
    bit; the fused call is also checked against the oracle."""
    moe = _moe()
    from int4_routed_expert_softmax_b200 import _cache as C
    w = mi.Workload("fused", H=H, I=I, E=E, k=k, T=1, seed=900 + seed)
    x, Wr, blobs = mi.make_layer(w, 0, DEV)
    d = moe.dims(H, I, E, k)
    assert moe.moe_layer_launches(d, 1) == 1
    assert moe.moe_layer_launches(d, 2) == 1          # one fused launch for the batch, routing included
    assert moe.moe_layer_launches(d, 5) == 1
    assert moe.moe_layer_launches(d, 2, 1) == 3       # MOE_PATH_DECODE: routing, gate/up, down
    out_f, ws_f, _ = gpu_layer(w, x, Wr, blobs)
    ws_s = moe.alloc_workspace(d, 1)
    out_s = torch.full_like(out_f, float("nan"))
    C.moe_layer_route(d, x, Wr, ws_s)
    C.moe_layer_experts(d, 1, moe.expert_table(blobs), out_s, ws_s)
    torch.cuda.synchronize()
    assert torch.equal(out_f, out_s)
    from tests._common import ws_trace
    tf, ts = ws_trace(ws_f, d, 1), ws_trace(ws_s, d, 1)
    for key in ("status", "xq", "xd", "logits", "idx", "w", "cnt", "off", "uni", "perm", "pos", "pair_tok", "hq",
                "hd"):
        assert np.array_equal(tf[key], ts[key]), key
    assert tf["n_uni"] == ts["n_uni"]
    if H * I <= 1024 * 256 or H == 6144:
        _check_layer(w, x, Wr, blobs)


def test_fused_route_counts_and_repeat():
    moe = _moe()
    w = mi.shrink(mi.WORKLOADS["decode"], seed=501)
    x, Wr, blobs = mi.make_layer(w, 0, DEV)
    d = moe.dims(w.H, w.I, w.E, w.k)
    ws = moe.alloc_workspace(d, 1)
    cnt = torch.zeros(w.E, dtype=torch.int32, device=DEV)
    table = moe.expert_table(blobs)
    outs = []
    for _ in range(3):
        out = torch.empty((1, w.H), device=DEV)
        moe.moe_layer_forward(d, x, Wr, table, out, ws, route_counts=cnt)
        outs.append(out)
    torch.cuda.synchronize()
    io, _ = orc.topk_softmax(orc.router_logits(x.cpu().numpy(), Wr.cpu().numpy()), w.k)
    assert np.array_equal(cnt.cpu().numpy(), 3 * np.bincount(io.reshape(-1), minlength=w.E))
    assert torch.equal(outs[0], outs[1]) and torch.equal(outs[0], outs[2])


# ----------------------------------------------------------------- small batches, token by token
@pytest.mark.parametrize("name,T", [("medium", 2), ("medium", 5), ("tiny", 7), ("glm", 4), ("glm", 16)])
def test_batch_token_by_token_equals_union_kernels(name, T):
    """2 <= T <= 16 on the auto path: one fused launch routes the batch and
    streams the tokens' experts one token after the other, writing each pair's
    h codes at its row in the batch's pair order.  MOE_PATH_DECODE runs the
    same batch through the routing kernel and the union's gate/up and down
    kernels.  Both compute every (token, slot) pair with the same per-row code
    and order, so the outputs, the routing record and the h codes agree bit
    for bit."""
    moe = _moe()
    from tests._common import ws_trace
    if name == "glm":
        w = mi.shrink(mi.WORKLOADS["decode"], T=T, seed=950 + T)
    elif name == "tiny":
        w = mi.shrink(mi.WORKLOADS["tiny"], T=T, seed=960 + T)
    else:
        w = mi.Workload("tok", H=1024, I=256, E=64, k=8, T=T, seed=970 + T)
    x, Wr, blobs = mi.make_layer(w, 0, DEV, T=T)
    d = moe.dims(w.H, w.I, w.E, w.k)
    counts = torch.zeros(w.E, dtype=torch.int32, device=DEV)
    table = moe.expert_table(blobs)
    out_a = torch.full((T, w.H), float("nan"), dtype=torch.float32, device=DEV)
    ws_a = moe.alloc_workspace(d, T)
    moe.moe_layer_forward(d, x, Wr, table, out_a, ws_a, route_counts=counts)
    out_b, ws_b, _ = gpu_layer(w, x, Wr, blobs, path=1)
    torch.cuda.synchronize()
    assert torch.equal(out_a, out_b)
    ta, tb = ws_trace(ws_a, d, T), ws_trace(ws_b, d, T)
    for key in ("status", "xq", "xd", "logits", "idx", "w", "cnt", "off", "uni", "perm", "pos", "pair_tok", "hq",
                "hd"):
        assert np.array_equal(ta[key], tb[key]), key
    # the routing kernel counted each selection once
    assert np.array_equal(counts.cpu().numpy(), np.bincount(ta["idx"].reshape(-1), minlength=w.E))
    if name != "glm":
        _check_layer(w, x, Wr, blobs)


def test_profile_ring_full_leaves_later_split_calls_unrecorded():
    """Past the ring's 1024 records a call goes unrecorded, and so does the
    experts half of a split layer (route, then experts): no later call stamps
    into the last record."""
    moe = _moe()
    from int4_routed_expert_softmax_b200 import _cache as C
    w = mi.WORKLOADS["tiny"]
    x, Wr, blobs = mi.make_layer(w, 0, DEV)
    T = x.shape[0]
    _, ws, d = gpu_layer(w, x, Wr, blobs, path=1)
    table = moe.expert_table(blobs)
    out = torch.empty((T, w.H), device=DEV)
    moe.moe_profile_enable(True)
    try:
        for _ in range(1024):
            C.moe_layer_route(d, x, Wr, ws)
            C.moe_layer_experts(d, T, table, out, ws)
        torch.cuda.synchronize()
        torch.cuda._sleep(50_000_000)   # ~25 ms on the stream before the unrecorded calls
        for _ in range(4):
            C.moe_layer_route(d, x, Wr, ws)
            C.moe_layer_experts(d, T, table, out, ws)
        rec = moe.moe_profile_read(1024)
    finally:
        moe.moe_profile_enable(False)
    assert len(rec) == 1024
    spans = [r[3] for r in rec]
    assert max(spans) < 5.0, max(spans)   # milliseconds: no record spans the sleep
