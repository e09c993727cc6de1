"""Reference model of the serving prefix cache (test infrastructure, like the rest
of ``oracle/``: only the tests may use it).

The serving cache keeps states at block boundaries of prompts, and a new request
resumes from the longest cached boundary of its prompt ("Kimi K3 开源日来了",
Infra section, second layer).  This model states the cache's bookkeeping as
plainly as possible: a prefix is cached exactly when the tuple of ALL its token
ids is a key of a dict (no hashing, so no collisions), each key owns one slot,
and the order of use is an explicit list.  The native index in libkda.so keys by
chained block hashes instead and must give the same answers:

  * lookup(ids, max_tokens): the longest prefix of ids that ends on a block
    boundary, is at most max_tokens long and whose every block-aligned prefix is
    cached (the native index walks block by block from the start); its length and
    slot.  The walked prefixes become the most recently used, the shortest first
    in the order (so longer prefixes of a chain are evicted before shorter ones).
  * insert(ids, first_block): for blocks j = 0, 1, ...: a cached prefix is
    marked used; an uncached one before first_block stops the walk; otherwise it
    takes the lowest free slot, else the slot of the least recently used prefix
    (which it evicts), unless that prefix was walked by this very call, which
    stops the walk.  Returns the number of leading cached blocks and the slot per
    block to fill (-1 for none).
"""
from __future__ import annotations


class PrefixCacheModel:
    def __init__(self, block: int, n_slots: int):
        self.block = int(block)
        self.n_slots = int(n_slots)
        self.slot_of = {}      # prefix tuple -> slot
        self.order = []        # prefix tuples, most recently used first
        self.free = list(range(self.n_slots))

    def _use(self, keys):
        """Move keys to the front so keys[0] ends first (most recent)."""
        for key in reversed(keys):
            self.order.remove(key)
            self.order.insert(0, key)

    def lookup(self, ids, max_tokens=None):
        ids = [int(x) for x in ids]
        limit = len(ids) if max_tokens is None else min(len(ids), int(max_tokens))
        walked, slot = [], -1
        end = self.block
        while end <= limit:
            key = tuple(ids[:end])
            if key not in self.slot_of:
                break
            walked.append(key)
            slot = self.slot_of[key]
            end += self.block
        self._use(walked)
        return len(walked) * self.block, slot

    def insert(self, ids, first_block: int = 0):
        ids = [int(x) for x in ids]
        nb = len(ids) // self.block
        out = [-1] * nb
        walked = []
        j = 0
        while j < nb:
            key = tuple(ids[:(j + 1) * self.block])
            if key in self.slot_of:
                walked.append(key)
                self._use([key])
                j += 1
                continue
            if j < first_block:
                break
            if self.free:
                slot = min(self.free)
                self.free.remove(slot)
            else:
                victim = self.order[-1]
                if victim in walked:
                    break
                slot = self.slot_of.pop(victim)
                self.order.pop()
            self.slot_of[key] = slot
            self.order.insert(0, key)
            out[j] = slot
            walked.append(key)
            j += 1
        self._use(walked)
        return j, out

    def __len__(self):
        return len(self.slot_of)
