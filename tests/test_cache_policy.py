"""The expert cache's policy on its host backend (no GPU): residency against an
independent LRU-with-pins model, blob contents behind the returned table,
learned pins, prefetch accounting, and host-side fault injection (failing
copies, failing pool allocation, capacity exhaustion)."""
import ctypes
import random

import numpy as np
import pytest

from int4_routed_expert_softmax_b200 import _cache as C
from int4_routed_expert_softmax_b200 import dims

H, I, E, K, L = 128, 128, 12, 2, 2


def _blob_bytes():
    return 3 * H * I // 2 + 3 * H * I // 32


@pytest.fixture()
def host_blobs():
    rng = np.random.default_rng(7)
    return [[rng.integers(0, 256, _blob_bytes(), dtype=np.uint8) for _ in range(E + 1)] for _ in range(L)]


def make(host_blobs, per_layer):
    return C.ExpertCache(dims(H, I, E, K), L, host_blobs, per_layer * L * _blob_bytes(), C.MOE_CACHE_HOST)


class LruModel:
    """Reference: per-layer LRU with pins; the current request is protected."""

    def __init__(self, cap):
        self.cap = cap
        self.order = []          # most recent first
        self.pinned = set()

    def acquire(self, want):
        hits = misses = 0
        prot = set(want)
        for e in want:
            if e in self.order:
                hits += 1
                self.order.remove(e)
                self.order.insert(0, e)
            else:
                misses += 1
                if len(self.order) >= self.cap:
                    for v in reversed(self.order):
                        if v not in self.pinned and v not in prot:
                            self.order.remove(v)
                            break
                    else:
                        raise RuntimeError("full")
                self.order.insert(0, e)
        return hits, misses


def _want(experts):
    w = []
    for e in experts:
        if e not in w:
            w.append(e)
    if E not in w:
        w.append(E)
    return w


def _table_blob(table_addr, e):
    ptr = ctypes.c_void_p.from_address(table_addr + 8 * e).value
    return None if ptr is None else np.frombuffer(ctypes.string_at(ptr, _blob_bytes()), np.uint8)


def test_geometry_and_contents(host_blobs):
    c = make(host_blobs, 5)
    st = c.stats()
    assert st["slots"] == 10 and st["slots_per_layer"] == 5
    t = c.acquire(1, [3, 7])
    for e in (3, 7, E):
        assert np.array_equal(_table_blob(t, e), host_blobs[1][e])
    assert _table_blob(t, 0) is None
    st = c.stats()
    assert st["misses"] == 3 and st["hits"] == 0 and st["bytes_h2d"] == 3 * _blob_bytes()
    c.close()


@pytest.mark.parametrize("cap", [3, 5, 8])
def test_lru_matches_reference_model(host_blobs, cap):
    c = make(host_blobs, cap)
    rnd = random.Random(cap)
    models = [LruModel(cap) for _ in range(L)]
    hits = misses = 0
    for step in range(300):
        layer = rnd.randrange(L)
        # skewed popularity so that some experts stay hot
        req = rnd.sample(range(E), K) if rnd.random() < 0.3 else rnd.sample(range(4), K)
        want = _want(req)
        h, m = models[layer].acquire(want)
        hits += h
        misses += m
        c.acquire(layer, req)
        for ly in range(L):
            for e in range(E + 1):
                assert c.resident(ly, e) == (e in models[ly].order), (step, ly, e)
    st = c.stats()
    assert st["hits"] == hits and st["misses"] == misses
    assert st["resident"] == sum(len(m.order) for m in models)
    c.close()


def test_pins_survive_and_learned_pins(host_blobs):
    c = make(host_blobs, 6)
    c.pin(0, [5, 6])
    assert c.pinned(0, 5) and c.resident(0, 6)
    for step in range(50):
        c.acquire(0, [step % E, (step + 3) % E])
        assert c.resident(0, 5) and c.resident(0, 6)
    c.evict(0, [5])            # pinned: skipped
    assert c.resident(0, 5)
    c.unpin(0, [5])
    c.evict(0, [5])
    assert not c.resident(0, 5)
    counts = [0] * E
    counts[9], counts[2], counts[4], counts[1] = 50, 30, 30, 1
    c.learn_pins(0, counts, 3)  # the 3 most routed, ties to the lower index: 9, 2, 4
    assert [e for e in range(E) if c.pinned(0, e)] == [2, 4, 9]
    assert c.stats()["pinned"] == 3
    # a full union must always fit: pins beyond slots - (k + 1) are refused
    with pytest.raises(C.MoeError) as ex:
        c.pin(0, [0, 1])
    assert ex.value.status == -5
    c.close()


def test_prefetch_accounting(host_blobs):
    c = make(host_blobs, 6)
    assert c.prefetch(1, [1, 2, 3]) == 3
    assert c.prefetch(1, [1, 2]) == 0          # already resident
    c.acquire(1, [1, 4])
    st = c.stats()
    assert st["prefetches"] == 3 and st["prefetch_hits"] == 1 and st["misses"] == 2  # 4 and shared
    c.acquire(1, [1])
    assert c.stats()["hits"] == 2               # 1 again (now a plain hit) and the shared expert
    c.close()


def test_capacity_exhaustion_is_an_error(host_blobs):
    c = make(host_blobs, 2)
    with pytest.raises(C.MoeError) as ex:
        c.acquire(0, [1, 2])                   # 3 experts with the shared one, 2 slots
    assert ex.value.status == -5
    c.close()


def test_injected_copy_fault_leaves_a_consistent_cache(host_blobs):
    c = make(host_blobs, 4)
    C.inject_fault(C.MOE_FAULT_COPY, 1, c)
    with pytest.raises(C.MoeError) as ex:
        c.acquire(0, [3])
    assert ex.value.status == -3
    assert not c.resident(0, 3)
    st = c.stats()
    assert st["copy_errors"] == 1
    t = c.acquire(0, [3])                       # the next call works, every slot still usable
    assert np.array_equal(_table_blob(t, 3), host_blobs[0][3])
    c.acquire(0, [0, 1])
    c.acquire(0, [5, 6])
    c.close()


def test_injected_alloc_fault(host_blobs):
    C.inject_fault(C.MOE_FAULT_ALLOC, 1)
    with pytest.raises(C.MoeError) as ex:
        make(host_blobs, 4)
    assert ex.value.status == -9
    make(host_blobs, 4).close()                 # one failure only


def test_bad_arguments(host_blobs):
    c = make(host_blobs, 4)
    for call in (lambda: c.acquire(2, [1]), lambda: c.acquire(0, [E + 1]), lambda: c.pin(-1, [0]),
                 lambda: c.prefetch(0, [-3])):
        with pytest.raises(C.MoeError) as ex:
            call()
        assert ex.value.status == -1
    c.close()
