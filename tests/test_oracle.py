"""Pins of the CPU oracle against facts that do not come from the oracle itself:
hand-worked fixtures (tests/golden), exact-integer special cases, brute force on
tiny inputs, closed forms, invariants, and float64 NumPy evaluations within a
stated bound.  Every check here is chosen so that a plausible slip in the oracle
(a dropped term, a wrong sign or index, a transposed operand, a wrong nibble,
the wrong rounding) fails at least one of them.  CPU only."""
import math
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle as orc

GOLD = os.path.join(os.path.dirname(__file__), "golden")
rng = np.random.default_rng(12345)


def _read_fixture(name):
    rows = []
    for line in open(os.path.join(GOLD, name)):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        key, *vals = line.split()
        rows.append((key, vals))
    return rows


def _f16(x):
    return np.asarray(x, np.float16).view(np.uint16)


def _rand_matrix(N, K, scale_ones=False):
    w = rng.integers(-8, 8, size=(N, K)).astype(np.int8)
    if scale_ones:
        s = np.ones((N, K // 64), np.float16)
    else:
        s = np.exp(rng.normal(math.log(0.02), 0.3, size=(N, K // 64))).astype(np.float16)
    return w, s, orc.pack_matrix(w, s.view(np.uint16))


def _ulp_err(got, ref64):
    got = got.astype(np.float64)
    ulp = np.spacing(np.abs(ref64).astype(np.float32)).astype(np.float64)
    return np.abs(got - ref64) / ulp


# ----------------------------------------------------------------- container
def test_int4_layout_hand_worked_row():
    rows = dict(_read_fixture("int4_gs64_row.txt"))
    mat = np.array([int(v, 16) for v in rows["bytes"]], np.uint8)
    w_ref = [int(v) for v in rows["w"]]
    s_ref = [float(v) for v in rows["scale"]]
    assert orc.matrix_bytes(1, 128) == mat.size
    assert [orc.weight(mat, 1, 128, 0, k) for k in range(128)] == w_ref
    assert [orc.scale(mat, 1, 128, 0, g) for g in range(2)] == s_ref


def test_pack_roundtrip_and_sizes():
    w, s, mat = _rand_matrix(8, 256)
    got = np.array([[orc.weight(mat, 8, 256, n, k) for k in range(256)] for n in range(8)])
    assert np.array_equal(got, w)
    gs = np.array([[orc.scale(mat, 8, 256, n, g) for g in range(4)] for n in range(8)], np.float32)
    assert np.array_equal(gs, s.astype(np.float32))
    # repacking the read-back weights reproduces the bytes exactly
    assert np.array_equal(orc.pack_matrix(got, gs.astype(np.float16).view(np.uint16)), mat)
    # 3 matrices of 6144 x 2048 int4 with gs64 fp16 scales: 20,054,016 bytes per expert
    assert orc.expert_bytes(6144, 2048) == 20_054_016
    assert orc.expert_bytes(256, 128) == 52_224


def test_half_to_float_all_patterns():
    pats = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = pats.view(np.float16).astype(np.float32)
    got = np.array([orc.half_to_float(int(p)) for p in pats[::7]], np.float32)
    r = ref[::7]
    fin = np.isfinite(r)
    assert np.array_equal(got[fin], r[fin])
    assert np.array_equal(np.isnan(got), np.isnan(r))


# ----------------------------------------------------------------- Q8_0
def test_q8_0_hand_worked_blocks():
    rows = _read_fixture("q8_0_blocks.txt")
    for i in range(0, len(rows), 3):
        x = np.array([float(v) for v in rows[i][1]], np.float32)
        d_ref = float(rows[i + 1][1][0])
        q_ref = np.array([int(v) for v in rows[i + 2][1]], np.int8)
        q, d = orc.quant_q8_0(x)
        assert float(d[0]) == d_ref
        assert np.array_equal(q, q_ref)


@pytest.mark.parametrize("scale", [1.0, 1e-3, 1e3, 3e-38, 1e30])
def test_q8_0_properties(scale):
    x = (rng.normal(size=(64, 32)) * scale).astype(np.float32)
    x[3] = 0.0                       # all-zero block
    x[5, 7] = -np.abs(x[5]).max() * 2  # negative amax
    q, d = orc.quant_q8_0(x)
    amax = np.abs(x).max(axis=1)
    assert np.array_equal(d[:, 0], (amax / np.float32(127.0)).astype(np.float32))
    for b in range(64):
        if d[b, 0] == 0:
            assert not q[b].any()
            continue
        # the amax element maps to +-127, sign kept
        j = int(np.argmax(np.abs(x[b])))
        assert q[b, j] == np.sign(x[b, j]) * 127
        # each code is the nearest multiple of d (exact rational check, away from ties)
        for i in range(32):
            r = Fraction(float(x[b, i])) / Fraction(float(d[b, 0]))
            frac = abs(r - math.floor(r) - Fraction(1, 2))
            if frac > Fraction(1, 10**4):
                assert q[b, i] == round(r)
            assert abs(int(q[b, i]) - r) <= Fraction(1, 2) + Fraction(1, 10**4)


def test_q8_0_idempotent_on_codes():
    q0 = rng.integers(-127, 128, size=(32, 32)).astype(np.int8)
    q0[:, 0] = 127
    d0 = np.float32(2.0) ** rng.integers(-10, 10, size=(32, 1)).astype(np.float32)
    x = q0.astype(np.float32) * d0   # exact (power-of-two scales)
    q, d = orc.quant_q8_0(x)
    assert np.array_equal(q, q0)
    assert np.array_equal(d, d0)


# ----------------------------------------------------------------- exp / SiLU
def test_silu_closed_forms():
    s = orc.silu(np.array([0.0, -0.0, 20.0, 40.0, 87.0, -120.0, -1e30], np.float32))
    assert s[0] == 0.0 and s[1] == 0.0
    assert s[2] == 20.0 and s[3] == 40.0 and s[4] == 87.0       # 1 + e^-g rounds to 1
    assert s[5] == 0.0 and s[6] == 0.0                          # g / inf
    g = rng.uniform(-60, 60, 200_000).astype(np.float32)
    got = orc.silu(g).astype(np.float64)
    g64 = g.astype(np.float64)
    ref = g64 / (1.0 + np.exp(-g64))
    assert np.all(np.abs(got - ref) <= 4 * np.spacing(np.abs(ref).astype(np.float32)) + 1e-45)
    # SiLU(g) - SiLU(-g) = g (the two halves of the logistic sum to one)
    g2 = rng.uniform(-5, 5, 10_000).astype(np.float32)
    lhs = orc.silu(g2).astype(np.float64) - orc.silu(-g2).astype(np.float64)
    assert np.allclose(lhs, g2.astype(np.float64), rtol=1e-6, atol=1e-6)


# ----------------------------------------------------------------- router
def test_router_integer_inputs_exact():
    H, E, T = 256, 16, 3
    x = rng.integers(-3, 4, size=(T, H)).astype(np.float32)
    Wr = rng.integers(-3, 4, size=(E, H)).astype(np.float32)
    got = orc.router_logits(x, Wr)
    ref = x.astype(np.int64) @ Wr.astype(np.int64).T
    assert np.array_equal(got, ref.astype(np.float32))


def test_router_float_bound():
    H, E, T = 6144, 8, 2
    x = rng.normal(size=(T, H)).astype(np.float32)
    Wr = (rng.normal(size=(E, H)) * 0.02).astype(np.float32)
    got = orc.router_logits(x, Wr).astype(np.float64)
    ref = x.astype(np.float64) @ Wr.astype(np.float64).T
    mag = np.abs(x).astype(np.float64) @ np.abs(Wr).astype(np.float64).T
    # 192 fmaf steps per chain + 5 tree levels, each a relative 2^-24 at most
    assert np.all(np.abs(got - ref) <= (H // 32 + 6) * 2.0**-24 * mag)
    # a one-hot input picks out the column of Wr exactly
    x1 = np.zeros((1, H), np.float32)
    x1[0, 777] = 1.0
    assert np.array_equal(orc.router_logits(x1, Wr)[0], Wr[:, 777])


def test_topk_brute_force_and_ties():
    T, E, k = 50, 16, 4
    lg = rng.normal(size=(T, E)).astype(np.float32)
    lg[::3] = np.round(lg[::3])          # many exact ties
    lg[7] = 0.5                          # every logit tied
    idx, w = orc.topk_softmax(lg, k)
    for t in range(T):
        order = sorted(range(E), key=lambda e: (-float(lg[t, e]), e))[:k]
        assert list(idx[t]) == order
    assert list(idx[7]) == [0, 1, 2, 3]
    assert np.allclose(w[7], 0.25, rtol=0, atol=1e-7)
    assert np.all(np.abs(w.astype(np.float64).sum(1) - 1.0) <= 1e-6)
    assert np.all(np.diff(w, axis=1) <= 0)          # weights follow the logit order
    # weights equal the float64 softmax over the kept logits
    kept = np.take_along_axis(lg, idx, 1).astype(np.float64)
    ref = np.exp(kept - kept.max(1, keepdims=True))
    ref /= ref.sum(1, keepdims=True)
    assert np.allclose(w, ref, rtol=3e-7, atol=1e-9)


def test_topk_special_k():
    lg = rng.normal(size=(10, 12)).astype(np.float32) * 3
    idx, w = orc.topk_softmax(lg, 1)
    assert np.all(w == 1.0) and np.array_equal(idx[:, 0], lg.argmax(1))
    idx, w = orc.topk_softmax(lg, 12)     # k = E: the full softmax
    full = np.exp(lg.astype(np.float64) - lg.max(1, keepdims=True))
    full /= full.sum(1, keepdims=True)
    assert np.allclose(np.take_along_axis(full, idx, 1), w, rtol=1e-6, atol=1e-9)


# ----------------------------------------------------------------- bucket
@pytest.mark.parametrize("T,k,E", [(1, 8, 256), (4, 2, 16), (16, 8, 256), (300, 8, 16), (0, 2, 4), (5, 3, 3)])
def test_bucket_brute_force(T, k, E):
    idx = np.array([rng.permutation(E)[:k] for _ in range(T)], np.int32).reshape(T, k)
    cnt, off, uni, n, perm = orc.bucket(idx, E)
    flat = idx.reshape(-1)
    assert np.array_equal(cnt, np.bincount(flat, minlength=E))
    assert np.array_equal(off, np.concatenate([[0], np.cumsum(cnt)]))
    assert np.array_equal(uni, np.unique(flat))
    assert np.array_equal(perm, np.argsort(flat, kind="stable"))
    assert cnt.sum() == T * k and sorted(perm.tolist()) == list(range(T * k))
    if T:
        assert k <= n <= min(E, T * k)


# ----------------------------------------------------------------- expert dot
def test_expert_dot_integer_exact():
    N, K = 6, 384
    w, s, mat = _rand_matrix(N, K, scale_ones=True)
    q = rng.integers(-127, 128, size=K).astype(np.int8)
    d = np.ones(K // 32, np.float32)
    for n in range(N):
        assert orc.expert_dot(mat, N, K, n, q, d) == float(np.dot(w[n].astype(np.int64), q.astype(np.int64)))
        for b in range(K // 32):
            assert orc.block_dot(mat, N, K, n, b, q) == int(np.dot(w[n, 32 * b:32 * b + 32].astype(np.int64),
                                                                   q[32 * b:32 * b + 32].astype(np.int64)))


@pytest.mark.parametrize("K", [128, 6144])
def test_expert_dot_float_bound(K):
    N = 4
    w, s, mat = _rand_matrix(N, K)
    xq, xd = orc.quant_q8_0(rng.normal(size=K).astype(np.float32))
    deq_w = w.astype(np.float64) * np.repeat(s.astype(np.float64), 64, axis=1)
    deq_x = xq.astype(np.float64) * np.repeat(xd.astype(np.float64), 32)
    for n in range(N):
        got = orc.expert_dot(mat, N, K, n, xq, xd)
        ref = float(deq_w[n] @ deq_x)
        mag = float(np.abs(deq_w[n]) @ np.abs(deq_x))
        assert abs(got - ref) <= (K // 64 + 8) * 2.0**-23 * mag


def test_expert_ffn_vs_float64():
    H, I = 256, 128
    blob = orc_blob(H, I)
    x = rng.normal(size=H).astype(np.float32)
    xq, xd = orc.quant_q8_0(x)
    r = orc.expert_ffn(blob, H, I, xq, xd)
    Wg, Wu, Wd = dequant_blob(blob, H, I)
    xh = xq.astype(np.float64) * np.repeat(xd.astype(np.float64), 32)
    g = Wg @ xh
    u = Wu @ xh
    assert np.allclose(r["g"], g, rtol=1e-5, atol=1e-5 * np.abs(g).max())
    assert np.allclose(r["u"], u, rtol=1e-5, atol=1e-5 * np.abs(u).max())
    h64 = r["g"].astype(np.float64) / (1 + np.exp(-r["g"].astype(np.float64))) * r["u"].astype(np.float64)
    assert np.allclose(r["h"], h64, rtol=1e-6, atol=1e-6 * np.abs(h64).max())
    q2, d2 = orc.quant_q8_0(r["h"])
    assert np.array_equal(q2, r["hq"]) and np.array_equal(d2, r["hd"])
    hh = r["hq"].astype(np.float64) * np.repeat(r["hd"].astype(np.float64), 32)
    y = Wd @ hh
    assert np.allclose(r["y"], y, rtol=1e-5, atol=1e-5 * np.abs(y).max())


def test_expert_down_from_codes_vs_float64():
    """The down projection from given codes: the dequantised matrix times the
    dequantised codes in float64; and the FFN's own y from its own codes."""
    H, I = 256, 128
    blob = orc_blob(H, I)
    _, _, Wd = dequant_blob(blob, H, I)
    hq, hd = orc.quant_q8_0((rng.normal(size=I) * 3).astype(np.float32))
    y = orc.expert_down(blob, H, I, hq, hd)
    ref = Wd @ (hq.astype(np.float64) * np.repeat(hd.astype(np.float64), 32))
    mag = np.abs(Wd) @ np.abs(hq.astype(np.float64) * np.repeat(hd.astype(np.float64), 32))
    assert np.all(np.abs(y - ref) <= (I // 64 + 8) * 2.0**-23 * mag)
    x = rng.normal(size=H).astype(np.float32)
    xq, xd = orc.quant_q8_0(x)
    r = orc.expert_ffn(blob, H, I, xq, xd)
    assert np.array_equal(orc.expert_down(blob, H, I, r["hq"], r["hd"]).view(np.uint32), r["y"].view(np.uint32))


# ----------------------------------------------------------------- layer
def orc_blob(H, I, seed=None):
    parts = []
    for N, K in [(I, H), (I, H), (H, I)]:
        parts.append(_rand_matrix(N, K)[2])
    return np.concatenate(parts)


def dequant_blob(blob, H, I):
    out = []
    o = 0
    for N, K in [(I, H), (I, H), (H, I)]:
        nb = orc.matrix_bytes(N, K)
        mat = blob[o:o + nb]
        o += nb
        packed = mat[: N * K // 2].reshape(N, K // 64, 32)
        lo = (packed & 0xF).astype(np.int64) - 8
        hi = (packed >> 4).astype(np.int64) - 8
        w = np.concatenate([lo, hi], axis=2).reshape(N, K)
        s = mat[N * K // 2:].view(np.float16).reshape(N, K // 64).astype(np.float64)
        out.append(w * np.repeat(s, 64, axis=1))
    return out


def _tiny_layer(T=4, H=256, I=128, E=16, k=2):
    x = rng.normal(size=(T, H)).astype(np.float32)
    Wr = (rng.normal(size=(E, H)) * 0.02).astype(np.float32)
    blobs = np.stack([orc_blob(H, I) for _ in range(E + 1)])
    return x, Wr, blobs


def test_layer_vs_float64_composition():
    H, I, E, k, T = 256, 128, 16, 2, 4
    x, Wr, blobs = _tiny_layer(T, H, I, E, k)
    out, tr = orc.moe_layer(x, Wr, blobs, H, I, E, k, trace=True)
    # routing: float64 logits give the same experts unless a near tie
    lg64 = x.astype(np.float64) @ Wr.astype(np.float64).T
    for t in range(T):
        srt = np.sort(lg64[t])[::-1]
        if srt[k - 1] - srt[k] > 1e-5:
            assert set(tr["idx"][t]) == set(np.argsort(-lg64[t])[:k])
    deq = [dequant_blob(b, H, I) for b in blobs]
    ref = np.zeros((T, H))
    for t in range(T):
        xq, xd = tr["xq"][t], tr["xd"][t]
        xh = xq.astype(np.float64) * np.repeat(xd.astype(np.float64), 32)

        def ffn(e):
            Wg, Wu, Wd = deq[e]
            g, u = Wg @ xh, Wu @ xh
            h = g / (1 + np.exp(-g)) * u
            hq, hd = orc.quant_q8_0(h.astype(np.float32))
            return Wd @ (hq.astype(np.float64) * np.repeat(hd.astype(np.float64), 32))
        ref[t] = ffn(E)
        for s in range(k):
            ref[t] += float(tr["w"][t, s]) * ffn(int(tr["idx"][t, s]))
    rel = np.linalg.norm(out - ref) / np.linalg.norm(ref)
    assert rel < 1e-3, rel


def test_layer_one_hot_combine_and_tokens():
    H, I, E, k, T = 256, 128, 16, 1, 3
    x, Wr, blobs = _tiny_layer(T, H, I, E, k)
    out, tr = orc.moe_layer(x, Wr, blobs, H, I, E, k, trace=True)
    assert np.all(tr["w"] == 1.0)
    for t in range(T):
        ys = tr["y"][t, k]
        ye = tr["y"][t, 0]
        assert np.array_equal(out[t], (ys + ye).astype(np.float32))
    # the token-subset form gives the same rows
    sub = orc.moe_layer_tokens(x, Wr, blobs, H, I, E, k, [2, 0])
    assert np.array_equal(sub, out[[2, 0]])


def test_layer_expert_relabel_invariance():
    H, I, E, k, T = 256, 128, 16, 2, 4
    x, Wr, blobs = _tiny_layer(T, H, I, E, k)
    out = orc.moe_layer(x, Wr, blobs, H, I, E, k)
    p = rng.permutation(E)
    blobs2 = np.concatenate([blobs[:E][p], blobs[E:]])
    out2 = orc.moe_layer(x, Wr[p], blobs2, H, I, E, k)
    assert np.array_equal(out, out2)


def test_layer_rejects_bad_shapes():
    x, Wr, blobs = _tiny_layer(1, 256, 128, 4, 2)
    with pytest.raises(ValueError):
        orc.moe_layer(x[:, :192], Wr[:, :192], blobs, 192, 128, 4, 2)
    with pytest.raises(ValueError):
        orc.moe_layer(x, Wr, blobs, 256, 128, 4, 5)
