"""The route-usage record on disk (host only): the learned cache's history of
which experts each layer routed to, kept across sessions so that learned pins
survive a restart (tantan.ink page, section 几个关键工程动作)."""
import os

import numpy as np
import pytest

from int4_routed_expert_softmax_b200 import MoeError, dims
from int4_routed_expert_softmax_b200 import _cache as C

NL, E = 3, 16


def _counts(seed):
    rng = np.random.default_rng(seed)
    c = rng.integers(0, 1000, (NL, E)).astype(np.uint64)
    c[1, 3] = np.uint64(1) << np.uint64(40)        # beyond 32 bits
    return c


def test_round_trip_and_accumulate(tmp_path):
    p = str(tmp_path / "usage.bin")
    a, b = _counts(1), _counts(2)
    C.usage_save(p, a)
    assert not os.path.exists(p + ".tmp")
    assert np.array_equal(C.usage_load(p, NL, E), a)
    acc = b.copy()
    C.usage_load(p, NL, E, acc)
    assert np.array_equal(acc, a + b)
    C.usage_save(p, acc)                            # overwrites the earlier record
    assert np.array_equal(C.usage_load(p, NL, E), a + b)


def test_refusals_leave_counts_untouched(tmp_path):
    p = str(tmp_path / "usage.bin")
    a = _counts(3)
    C.usage_save(p, a)
    keep = _counts(4)
    acc = keep.copy()
    with pytest.raises(MoeError) as ex:
        C.usage_load(p, NL, E + 1, np.zeros((NL, E + 1), np.uint64))
    assert ex.value.status == -2                    # written for another shape
    raw = open(p, "rb").read()
    cases = {
        "flipped count byte": raw[:30] + bytes([raw[30] ^ 1]) + raw[31:],
        "truncated": raw[:-3],
        "trailing byte": raw + b"\0",
        "bad magic": b"X" + raw[1:],
    }
    for name, data in cases.items():
        open(p, "wb").write(data)
        with pytest.raises(MoeError) as ex:
            C.usage_load(p, NL, E, acc)
        assert ex.value.status == C.MOE_ERR_IO, name
        assert np.array_equal(acc, keep), name
    with pytest.raises(MoeError) as ex:
        C.usage_load(str(tmp_path / "missing.bin"), NL, E)
    assert ex.value.status == C.MOE_ERR_IO
    with pytest.raises(ValueError):
        C.usage_save(p, np.array([[-1, 2]]))


def test_learned_pins_survive_a_restart(tmp_path):
    """Session 1 records route counts and saves them; session 2 loads the record
    into a fresh cache and pins the same experts session 1 would."""
    H, I, K = 128, 128, 2
    blob = 3 * H * I // 2 + 3 * H * I // 32
    rng = np.random.default_rng(5)
    host = [[rng.integers(0, 256, blob, dtype=np.uint8) for _ in range(E + 1)] for _ in range(NL)]
    counts = np.zeros((NL, E), np.uint64)
    for _ in range(200):                            # session 1's routing
        layer = int(rng.integers(0, NL))
        for e in rng.choice(E, size=K, replace=False, p=np.arange(E, 0, -1) / (E * (E + 1) / 2)):
            counts[layer, e] += 1
    p = str(tmp_path / "usage.bin")
    C.usage_save(p, counts)
    n_pin = 4
    first = C.ExpertCache(dims(H, I, E, K), NL, host, 8 * NL * blob, C.MOE_CACHE_HOST)
    second = C.ExpertCache(dims(H, I, E, K), NL, host, 8 * NL * blob, C.MOE_CACHE_HOST)
    loaded = C.usage_load(p, NL, E)
    for layer in range(NL):
        first.learn_pins(layer, counts[layer], n_pin)
        second.learn_pins(layer, loaded[layer], n_pin)
        top = sorted(range(E), key=lambda e: (-int(counts[layer, e]), e))[:n_pin]
        for e in range(E):
            assert second.pinned(layer, e) == first.pinned(layer, e) == (e in top)
    first.close()
    second.close()
