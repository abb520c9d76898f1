"""Pins of the oracle's MXFP4 expert format (32 E2M1 codes per E8M0 exponent; the
expert format of the Kimi K3 row of the model-family table on the colibri deep
review page, ai-tools-nav) against facts that do not come from the oracle: the FP4 (E2M1) value
set, a hand-worked row (tests/golden/mxfp4_row.txt), exact-integer special
cases, a cross-format case where int4 gs64 and MXFP4 hold the same weights, and
float64 evaluations within a stated bound.  CPU only."""
import math
import os

import numpy as np
import pytest

import oracle as orc

GOLD = os.path.join(os.path.dirname(__file__), "golden")
rng = np.random.default_rng(2468)

# magnitudes of the E2M1 codes 0..7 (the FP4 value set of the microscaling formats)
E2M1 = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def _fixture(name):
    rows = {}
    for line in open(os.path.join(GOLD, name)):
        line = line.strip()
        if line and not line.startswith("#"):
            key, *vals = line.split()
            rows[key] = vals
    return rows


def _values(codes):
    codes = np.asarray(codes)
    mag = np.array(E2M1)[codes & 7]
    return np.where(codes & 8, -mag, mag)


def _rand_mx(N, K, e_lo=118, e_hi=123):
    codes = rng.integers(0, 16, size=(N, K)).astype(np.uint8)
    exps = rng.integers(e_lo, e_hi + 1, size=(N, K // 32)).astype(np.uint8)
    return codes, exps, orc.mx_pack_matrix(codes, exps)


def _deq(codes, exps):
    return _values(codes) * np.repeat(2.0 ** (exps.astype(np.float64) - 127), 32, axis=1)


def test_e2m1_value_set():
    vals = [orc.e2m1_value(c) for c in range(16)]
    assert vals[:8] == E2M1
    assert all(vals[c + 8] == -vals[c] for c in range(8))
    assert math.copysign(1.0, vals[8]) == -1.0                  # code 8 is -0
    assert all(vals[c] < vals[c + 1] for c in range(7))


def test_hand_worked_row():
    f = _fixture("mxfp4_row.txt")
    mat = np.array([int(v, 16) for v in f["bytes"]], np.uint8)
    assert orc.matrix_bytes(1, 64) == mat.size
    assert [orc.mx_weight(mat, 1, 64, 0, k) for k in range(64)] == [float(v) for v in f["w"]]
    codes = np.array([[k % 16 for k in range(32)] + [7] * 32], np.uint8)
    exps = np.array([[0x7F, 0x7C]], np.uint8)
    assert np.array_equal(orc.mx_pack_matrix(codes, exps), mat)
    q = np.array([int(v) for v in f["q"]], np.int8)
    d = np.array([float(v) for v in f["d"]], np.float32)
    assert [orc.mx_block_dot(mat, 1, 64, 0, b, q) for b in range(2)] == [int(v) for v in f["block_sums"]]
    assert orc.mx_expert_dot(mat, 1, 64, 0, q, d) == float(f["dot"][0])


def test_pack_round_trip_asymmetric():
    N, K = 3, 256
    codes, exps, mat = _rand_mx(N, K)
    for n in range(N):
        assert [orc.mx_code(mat, N, K, n, k) for k in range(K)] == codes[n].tolist()
        assert [orc.mx_scale_exp(mat, N, K, n, b) for b in range(K // 32)] == exps[n].tolist()


def test_block_dot_and_dot_exact_with_unit_scales():
    """With every block exponent 128 (scale 2) and Q8_0 scale 1 the dot is the
    exact integer sum of 2*e2m1*q (float64 of the value set)."""
    N, K = 4, 384
    codes = rng.integers(0, 16, size=(N, K)).astype(np.uint8)
    exps = np.full((N, K // 32), 128, np.uint8)
    mat = orc.mx_pack_matrix(codes, exps)
    q = rng.integers(-127, 128, size=K).astype(np.int8)
    d = np.ones(K // 32, np.float32)
    c2 = (2 * _values(codes)).astype(np.int64)
    for n in range(N):
        for b in range(K // 32):
            assert orc.mx_block_dot(mat, N, K, n, b, q) == int(c2[n, 32 * b:32 * b + 32] @ q[32 * b:32 * b + 32])
        assert orc.mx_expert_dot(mat, N, K, n, q, d) == float(c2[n] @ q.astype(np.int64))


def test_same_weights_in_both_formats_give_the_same_dot():
    """Weights in {0, +-1, +-2, +-3, +-4, +-6} are exact in int4 (scale 1.0) and in
    MXFP4 (code w/2, E = 128); with unit activation scales both dots are the same
    exact integer.  A slip in either container (nibble order, block or exponent
    offset) breaks the equality."""
    N, K = 5, 512
    choices = np.array([0, 1, -1, 2, -2, 3, -3, 4, -4, 6, -6])
    w = rng.choice(choices, size=(N, K)).astype(np.int8)
    int4 = orc.pack_matrix(w, np.full((N, K // 64), 0x3C00, np.uint16))
    half = w.astype(np.float64) / 2
    codes = np.array([[E2M1.index(abs(v)) | (8 if v < 0 else 0) for v in row] for row in half], np.uint8)
    mx = orc.mx_pack_matrix(codes, np.full((N, K // 32), 128, np.uint8))
    q = rng.integers(-127, 128, size=K).astype(np.int8)
    d = np.ones(K // 32, np.float32)
    for n in range(N):
        a = orc.expert_dot(int4, N, K, n, q, d)
        assert a == orc.mx_expert_dot(mx, N, K, n, q, d) == float(w[n].astype(np.int64) @ q.astype(np.int64))


@pytest.mark.parametrize("K", [128, 6144])
def test_dot_float_bound(K):
    N = 4
    codes, exps, mat = _rand_mx(N, K)
    xq, xd = orc.quant_q8_0(rng.normal(size=K).astype(np.float32))
    W = _deq(codes, exps)
    xh = xq.astype(np.float64) * np.repeat(xd.astype(np.float64), 32)
    for n in range(N):
        got = orc.mx_expert_dot(mat, N, K, n, xq, xd)
        mag = float(np.abs(W[n]) @ np.abs(xh))
        assert abs(got - float(W[n] @ xh)) <= (K // 32 + 8) * 2.0**-23 * mag


def _mx_blob(H, I):
    parts, deq = [], []
    for N, K in [(I, H), (I, H), (H, I)]:
        codes, exps, mat = _rand_mx(N, K)
        parts.append(mat)
        deq.append(_deq(codes, exps))
    return np.concatenate(parts), deq


def test_expert_ffn_vs_float64():
    H, I = 256, 128
    blob, (Wg, Wu, Wd) = _mx_blob(H, I)
    assert blob.size == orc.expert_bytes(H, I)
    x = rng.normal(size=H).astype(np.float32)
    xq, xd = orc.quant_q8_0(x)
    r = orc.expert_ffn(blob, H, I, xq, xd, fmt="mxfp4")
    xh = xq.astype(np.float64) * np.repeat(xd.astype(np.float64), 32)
    g, u = Wg @ xh, Wu @ xh
    assert np.allclose(r["g"], g, rtol=1e-5, atol=1e-5 * np.abs(g).max())
    assert np.allclose(r["u"], u, rtol=1e-5, atol=1e-5 * np.abs(u).max())
    q2, d2 = orc.quant_q8_0(r["h"])
    assert np.array_equal(q2, r["hq"]) and np.array_equal(d2, r["hd"])
    y = Wd @ (r["hq"].astype(np.float64) * np.repeat(r["hd"].astype(np.float64), 32))
    assert np.allclose(r["y"], y, rtol=1e-5, atol=1e-5 * np.abs(y).max())


def test_expert_down_from_codes():
    """The down projection from given codes: the FFN's own y from its own codes
    bit for bit, and the dequantised matrix times other codes within the float
    bound of its sum."""
    H, I = 256, 128
    blob, (Wg, Wu, Wd) = _mx_blob(H, I)
    x = rng.normal(size=H).astype(np.float32)
    xq, xd = orc.quant_q8_0(x)
    r = orc.expert_ffn(blob, H, I, xq, xd, fmt="mxfp4")
    assert np.array_equal(orc.expert_down(blob, H, I, r["hq"], r["hd"], fmt="mxfp4").view(np.uint32),
                          r["y"].view(np.uint32))
    hq, hd = orc.quant_q8_0((rng.normal(size=I) * 3).astype(np.float32))
    y = orc.expert_down(blob, H, I, hq, hd, fmt="mxfp4").astype(np.float64)
    hh = hq.astype(np.float64) * np.repeat(hd.astype(np.float64), 32)
    ref, mag = Wd @ hh, np.abs(Wd) @ np.abs(hh)
    assert np.all(np.abs(y - ref) <= (I // 32 + 8) * 2.0**-23 * mag)


def test_layer_vs_float64_and_int4_routing():
    """The MXFP4 layer: the same routing as the int4 layer on the same x and
    router (the experts' format does not enter routing), and its output within
    the float64 evaluation of the same quantised operands."""
    H, I, E, k, T = 256, 128, 8, 2, 3
    x = rng.normal(size=(T, H)).astype(np.float32)
    Wr = (rng.normal(size=(E, H)) * 0.02).astype(np.float32)
    made = [_mx_blob(H, I) for _ in range(E + 1)]
    blobs = np.stack([m[0] for m in made])
    out, tr = orc.moe_layer(x, Wr, blobs, H, I, E, k, trace=True, fmt="mxfp4")
    _, tr4 = orc.moe_layer(x, Wr, blobs, H, I, E, k, trace=True)
    assert np.array_equal(tr["idx"], tr4["idx"]) and np.array_equal(tr["w"], tr4["w"])
    ref = np.zeros((T, H))
    for t in range(T):
        xh = tr["xq"][t].astype(np.float64) * np.repeat(tr["xd"][t].astype(np.float64), 32)

        def ffn(e):
            Wg, Wu, Wd = made[e][1]
            g, u = Wg @ xh, Wu @ xh
            hq, hd = orc.quant_q8_0((g / (1 + np.exp(-g)) * u).astype(np.float32))
            return Wd @ (hq.astype(np.float64) * np.repeat(hd.astype(np.float64), 32))
        ref[t] = ffn(E) + sum(float(tr["w"][t, s]) * ffn(int(tr["idx"][t, s])) for s in range(k))
    assert np.linalg.norm(out - ref) / np.linalg.norm(ref) < 1e-3


def test_seeded_mx_blobs_feed_the_layer():
    """The seeded MXFP4 workload blobs: exponents in range, weights of the int4
    workload's magnitude, and a finite layer output."""
    import moe_inputs as mi
    H, I, E, k, T = 256, 128, 4, 2, 2
    blobs = mi.make_blobs_mx(H, I, E + 1, 11).numpy()
    assert np.array_equal(blobs, mi.make_blobs_mx(H, I, E + 1, 11).numpy())     # seeded
    N, K = I, H
    ex = np.array([orc.mx_scale_exp(blobs[0], N, K, n, b) for n in range(N) for b in range(K // 32)])
    assert ex.min() >= 115 and ex.max() <= 127
    x = rng.normal(size=(T, H)).astype(np.float32)
    Wr = (rng.normal(size=(E, H)) * 0.02).astype(np.float32)
    out = orc.moe_layer(x, Wr, blobs, H, I, E, k, fmt="mxfp4")
    assert np.all(np.isfinite(out)) and np.abs(out).max() > 0


def test_token_subset_equals_full_layer_rows():
    import moe_inputs as mi
    H, I, E, k, T = 256, 128, 4, 2, 5
    blobs = mi.make_blobs_mx(H, I, E + 1, 12).numpy()
    x = rng.normal(size=(T, H)).astype(np.float32)
    Wr = (rng.normal(size=(E, H)) * 0.02).astype(np.float32)
    full = orc.moe_layer(x, Wr, blobs, H, I, E, k, fmt="mxfp4")
    sub = orc.moe_layer_tokens(x, Wr, blobs, H, I, E, k, [4, 0, 2], fmt="mxfp4")
    assert np.array_equal(sub.view(np.uint32), full[[4, 0, 2]].view(np.uint32))
    assert not np.array_equal(full, orc.moe_layer(x, Wr, blobs, H, I, E, k))   # the format matters
