"""Host logic of the prefix cache: key -> pool slot bookkeeping and LRU
eviction, driven with a fake data mover over numpy arrays (no GPU)."""
import numpy as np
import pytest

from linear_attention_recurrent_lq_b200.prefix_cache import PrefixCache


class FakeMover:
    """Serving buffer and pool as [slots, bytes] arrays; records each call."""

    def __init__(self, serve_slots, pool_slots, nbytes=8):
        rng = np.random.default_rng(0)
        self.serve = rng.integers(0, 255, (serve_slots, nbytes), dtype=np.uint8)
        self.pool = np.zeros((pool_slots, nbytes), np.uint8)
        self.calls = []

    def __call__(self, to_pool, dst, src):
        self.calls.append((to_pool, list(dst), list(src)))
        a, b = (self.pool, self.serve) if to_pool else (self.serve, self.pool)
        for d, s in zip(dst, src):
            a[d] = b[s]


def test_store_then_restore_moves_the_bytes_back():
    m = FakeMover(6, 3)
    c = PrefixCache(3, m)
    snap = m.serve.copy()
    slots = c.store([("a", 1), ("b", 4)])
    assert sorted(slots) == [0, 1] and len(c) == 2
    assert m.calls == [(True, slots, [1, 4])]  # one copy for the batch
    m.serve[:] = 0
    assert c.restore([("b", 0), ("zz", 2), ("a", 5)]) == [True, False, True]
    np.testing.assert_array_equal(m.serve[0], snap[4])
    np.testing.assert_array_equal(m.serve[5], snap[1])
    assert not m.serve[2].any()  # a miss leaves the slot alone
    assert (c.hits, c.misses) == (2, 1)


def test_lru_eviction_order():
    m = FakeMover(8, 2)
    c = PrefixCache(2, m)
    c.store([("a", 0)])
    c.store([("b", 1)])
    c.restore([("a", 2)])          # a becomes most recent
    c.store([("c", 3)])            # evicts b
    assert c.keys() == ["a", "c"] and "b" not in c
    assert c.evictions == 1
    # c reuses b's pool slot
    assert m.calls[-1][1] == [1]
    c.store([("d", 4)])            # evicts a
    assert c.keys() == ["c", "d"]


def test_batch_never_evicts_its_own_keys():
    m = FakeMover(8, 3)
    c = PrefixCache(3, m)
    c.store([("a", 0), ("b", 1), ("c", 2)])
    # a is the least recent, but it is part of this batch: b goes instead
    slots = c.store([("a", 3), ("d", 4)])
    assert "a" in c and "d" in c and "b" not in c
    assert len(set(slots)) == 2
    np.testing.assert_array_equal(m.pool[slots[0]], m.serve[3])
    np.testing.assert_array_equal(m.pool[slots[1]], m.serve[4])


def test_overwrite_keeps_the_slot_and_drop_frees_it():
    m = FakeMover(4, 2)
    c = PrefixCache(2, m)
    (s0,) = c.store([("a", 0)])
    (s1,) = c.store([("a", 1)])
    assert s0 == s1 and len(c) == 1
    np.testing.assert_array_equal(m.pool[s0], m.serve[1])
    assert c.drop("a") and not c.drop("a")
    assert len(c) == 0
    c.store([("x", 2), ("y", 3)])
    assert c.evictions == 0


def test_bad_batches_rejected():
    c = PrefixCache(2, FakeMover(4, 2))
    with pytest.raises(ValueError):
        c.store([("a", 0), ("a", 1)])
    with pytest.raises(ValueError):
        c.store([("a", 0), ("b", 1), ("c", 2)])
    with pytest.raises(ValueError):
        PrefixCache(0, FakeMover(1, 1))


def test_random_workload_matches_a_reference_lru():
    """Against a plain list-based LRU over a random mix of stores and restores."""
    rng = np.random.default_rng(7)
    cap = 4
    m = FakeMover(16, cap)
    c = PrefixCache(cap, m)
    ref = []  # keys, least recent first
    content = {}
    for _ in range(400):
        key = int(rng.integers(0, 10))
        slot = int(rng.integers(0, 16))
        if rng.random() < 0.5:
            m.serve[slot] = rng.integers(0, 255, m.serve.shape[1], dtype=np.uint8)
            c.store([(key, slot)])
            content[key] = m.serve[slot].copy()
            if key in ref:
                ref.remove(key)
            elif len(ref) == cap:
                content.pop(ref.pop(0))
            ref.append(key)
        else:
            hit = c.restore([(key, slot)])[0]
            assert hit == (key in ref)
            if hit:
                ref.remove(key)
                ref.append(key)
                np.testing.assert_array_equal(m.serve[slot], content[key])
        assert c.keys() == ref
