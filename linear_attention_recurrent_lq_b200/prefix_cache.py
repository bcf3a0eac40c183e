"""Prefix cache of recurrent states for a continuous-batching server.

A recurrent head's whole context is its state, so caching a shared prompt
prefix means keeping a copy of the state blobs reached at the end of that
prefix.  Snapshots live in a pool buffer of ``capacity`` slots with the same
blob layout as the serving state; ``store`` copies serving slots into the
pool and ``restore`` copies them back, both through ``lq_copy_slots`` (the
bytes move as they are, so a restored sequence continues bit for bit).  When
the pool is full, the least recently used snapshot is evicted.

Taking snapshots right after a window flush (count = 0) keeps them smallest
in meaning, but any blob can be stored: pending pairs are part of its bytes.
"""
from __future__ import annotations

from collections import OrderedDict
from typing import Callable, Hashable, Sequence

# copy(dst_is_pool, dst_slots, src_slots): move whole slots (all heads)
# between the serving buffer and the pool, pairwise.
CopyFn = Callable[[bool, Sequence[int], Sequence[int]], None]


class PrefixCache:
    """Key -> pool slot map with LRU eviction over a fixed pool of slots.

    ``copy`` is the data mover; by default it is built by :meth:`for_state`
    from the library's slot copy.  The bookkeeping is host-side only.
    """

    def __init__(self, capacity: int, copy: CopyFn):
        if capacity <= 0:
            raise ValueError("capacity must be positive")
        self.capacity = capacity
        self._copy = copy
        self._slot_of: OrderedDict[Hashable, int] = OrderedDict()  # oldest first
        self._free = list(range(capacity - 1, -1, -1))
        self.hits = self.misses = self.evictions = 0

    @classmethod
    def for_state(cls, state, capacity: int) -> "PrefixCache":
        """A cache whose pool sits on the device of ``state`` (an LQState).
        Copies run on the current stream, in order with the decode calls
        that use the default stream argument."""
        import torch

        from . import binding as B
        cfg = state.cfg
        pool = torch.empty(capacity * cfg.num_heads * state.blob_bytes, dtype=torch.uint8,
                           device=state.buf.device)

        def copy(to_pool, dst, src):
            dev = state.buf.device
            d = torch.tensor(list(dst), dtype=torch.int32).to(dev, non_blocking=True)
            s = torch.tensor(list(src), dtype=torch.int32).to(dev, non_blocking=True)
            if to_pool:
                B.lq_copy_slots(cfg, pool, capacity, d, state.buf, cfg.num_slots, s)
            else:
                B.lq_copy_slots(cfg, state.buf, cfg.num_slots, d, pool, capacity, s)

        cache = cls(capacity, copy)
        cache.pool = pool
        return cache

    def __len__(self) -> int:
        return len(self._slot_of)

    def __contains__(self, key: Hashable) -> bool:
        return key in self._slot_of

    def keys(self) -> list:
        """Cached keys, least recently used first."""
        return list(self._slot_of)

    def _take_slot(self) -> int:
        if self._free:
            return self._free.pop()
        key, slot = self._slot_of.popitem(last=False)
        self.evictions += 1
        return slot

    def store(self, items: Sequence[tuple[Hashable, int]]) -> list[int]:
        """Snapshot serving slots: items are (key, serving slot).  A key that
        is cached already is overwritten in place.  Returns the pool slot of
        each item.  One copy call moves the whole batch."""
        keys = [k for k, _ in items]
        if len(set(keys)) != len(keys):
            raise ValueError("duplicate key in one store")
        if len(keys) > self.capacity:
            raise ValueError(f"{len(keys)} snapshots do not fit a pool of {self.capacity}")
        # keys of this batch that are cached already must not be evicted by
        # the others: refresh them first
        for k in keys:
            if k in self._slot_of:
                self._slot_of.move_to_end(k)
        pool_slots = []
        for k in keys:
            slot = self._slot_of.get(k)
            if slot is None:
                slot = self._take_slot()
            self._slot_of[k] = slot
            self._slot_of.move_to_end(k)
            pool_slots.append(slot)
        if items:
            self._copy(True, pool_slots, [s for _, s in items])
        return pool_slots

    def restore(self, items: Sequence[tuple[Hashable, int]]) -> list[bool]:
        """Bring cached snapshots back: items are (key, serving slot).  Returns
        per item whether it was a hit (a miss leaves that slot alone)."""
        hit, dst, src = [], [], []
        for k, serve in items:
            slot = self._slot_of.get(k)
            hit.append(slot is not None)
            if slot is None:
                self.misses += 1
                continue
            self.hits += 1
            self._slot_of.move_to_end(k)
            dst.append(serve)
            src.append(slot)
        if dst:
            self._copy(False, dst, src)
        return hit

    def drop(self, key: Hashable) -> bool:
        """Forget a snapshot (its pool slot becomes free)."""
        slot = self._slot_of.pop(key, None)
        if slot is None:
            return False
        self._free.append(slot)
        return True
