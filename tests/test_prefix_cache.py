"""The serving prefix cache's index (CPU): the reference model in
oracle/prefix_cache.py against hand-worked cases, and the native index in
libkda.so against the model, answer for answer, on random prompt streams that
share prefixes (lookups, inserts, evictions)."""
import ctypes
import os
import sys

import numpy as np
import pytest

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

from decode_kda_chunked_b200 import _lib  # noqa: E402
from oracle.prefix_cache import PrefixCacheModel  # noqa: E402


def test_model_hand_worked():
    """Blocks of 2 ids, 3 slots; every answer worked out by hand from the rules."""
    m = PrefixCacheModel(2, 3)
    assert m.insert([1, 2, 3, 4, 5]) == (2, [0, 1])
    assert m.lookup([1, 2, 3, 4, 9]) == (4, 1)
    assert m.lookup([1, 2, 7, 7], max_tokens=3) == (2, 0)
    assert m.insert([5, 6]) == (1, [2])
    # no slot free: the least recently used prefixes go, longest first
    assert m.insert([7, 8, 9, 10]) == (2, [1, 0])
    assert m.lookup([1, 2, 3, 4]) == (0, -1)
    assert m.lookup([7, 8, 9, 10, 11]) == (4, 0)
    assert m.lookup([5, 6]) == (2, 2)
    # a block before first_block must be cached already
    assert m.insert([1, 2, 3, 4, 5, 6], first_block=1) == (0, [-1, -1, -1])
    assert len(m) == 3


def test_model_never_evicts_its_own_prompt():
    m = PrefixCacheModel(2, 2)
    assert m.insert([1, 2, 3, 4, 5, 6]) == (2, [0, 1, -1])
    assert m.lookup([1, 2, 3, 4, 5, 6]) == (4, 1)


class Native:
    """The libkda.so index behind the model's interface."""

    def __init__(self, block, n_slots):
        self.block = block
        self.h = _lib.kda_prefix_cache_create(block, n_slots)

    def lookup(self, ids, max_tokens=None):
        return _lib.kda_prefix_cache_lookup(self.h, ids, max_tokens)

    def insert(self, ids, first_block=0):
        k, out = _lib.kda_prefix_cache_insert(self.h, ids, first_block)
        return k, [int(x) for x in out[:len(ids) // self.block]]

    def __len__(self):
        return _lib.kda_prefix_cache_size(self.h)

    def close(self):
        _lib.kda_prefix_cache_destroy(self.h)


@pytest.mark.parametrize("block,n_slots,seed", [(2, 3, 0), (4, 5, 1), (3, 16, 2), (512, 6, 3)])
def test_native_index_matches_model(block, n_slots, seed):
    rng = np.random.default_rng(seed)
    model, native = PrefixCacheModel(block, n_slots), Native(block, n_slots)
    # a few stems that prompts extend, so prefixes are shared and partly diverge
    stems = [list(rng.integers(0, 50, size=block * int(rng.integers(1, 5)))) for _ in range(5)]
    try:
        for step in range(300):
            stem = stems[int(rng.integers(0, len(stems)))]
            cut = int(rng.integers(0, len(stem) + 1))
            tail = list(rng.integers(0, 50, size=int(rng.integers(0, 3 * block))))
            ids = [int(x) for x in stem[:cut] + tail]
            if rng.random() < 0.5:
                mt = None if rng.random() < 0.5 else int(rng.integers(0, len(ids) + 1))
                assert native.lookup(ids, mt) == model.lookup(ids, mt), (step, ids, mt)
            else:
                fb = 0 if rng.random() < 0.7 else int(rng.integers(0, len(ids) // block + 1))
                assert native.insert(ids, fb) == model.insert(ids, fb), (step, ids, fb)
            assert len(native) == len(model)
    finally:
        native.close()


def test_native_index_rejects_invalid_args():
    lib = _lib.load()
    assert not lib.kda_prefix_cache_create(0, 4)
    assert not lib.kda_prefix_cache_create(512, 0)
    h = lib.kda_prefix_cache_create(512, 4)
    slot = ctypes.c_int32(7)
    assert lib.kda_prefix_cache_lookup(None, None, 0, 0, ctypes.byref(slot)) == -1
    assert lib.kda_prefix_cache_lookup(h, None, 5, 5, ctypes.byref(slot)) == -1
    assert lib.kda_prefix_cache_lookup(h, None, 0, 0, ctypes.byref(slot)) == 0 and slot.value == -1
    ids = (ctypes.c_int32 * 1024)(*range(1024))
    assert lib.kda_prefix_cache_insert(h, ids, 1024, 0, None) == -1   # slots_out required
    assert lib.kda_prefix_cache_insert(h, ids, 1024, -1, None) == -1
    assert lib.kda_prefix_cache_size(None) == -1
    lib.kda_prefix_cache_destroy(h)


def test_state_copies_reject_invalid_args():
    lib = _lib.load()
    F = 1 << 40
    # misaligned pool, dk*dv not a multiple of 4, overlapping pool and dst
    assert lib.kda_state_gather(F + 4, 4, F + (1 << 30), 2, 2, 128, 128, F + (2 << 30), None) == 1
    assert lib.kda_state_gather(F, 4, F + (1 << 30), 2, 1, 1, 3, F + (2 << 30), None) == 1
    assert lib.kda_state_gather(F, 4, F + (1 << 30), 2, 2, 128, 128, F + 4096, None) == 1
    assert lib.kda_state_scatter(F, F + (1 << 30), 2, 2, 128, 128, F + 4096, 4, None) == 1
    assert lib.kda_state_gather(F, 4, None, 0, 2, 128, 128, None, None) == 0   # nothing to do
