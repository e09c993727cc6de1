"""Prefix-cache resume for serving: requests whose prompts start with a cached
prefix resume from the stored state after it.

The serving cache keeps sparse state snapshots at 512-token block boundaries
and resumes a request from the longest cached one ("Kimi K3 开源日来了", Infra
section, second layer).  The index (chained block hashes of token ids, LRU
eviction) is native code in libkda.so; the states live in a device pool owned
here, and the copies between the pool and the prefill's dense initial states
and snapshots are the library's gather / scatter kernels.  Nothing here
computes any part of KDA.

Flow for a batch of prompts (token ids on the host):

    cache = PrefixCache(n_slots, H, dk, dv)
    plan = cache.plan(prompts)              # cached prefix length and slot per prompt
    # the caller builds q, k, v, g, beta for each prompt's tokens plan[r][0]: only
    out = cache.prefill(prompts, plan, q, k, v, g, beta)   # resumes, then caches
"""
from __future__ import annotations

import torch

from ._lib import (kda_prefix_cache_create, kda_prefix_cache_destroy,
                   kda_prefix_cache_insert, kda_prefix_cache_lookup, kda_prefix_cache_size,
                   kda_state_gather, kda_state_scatter)

BLOCK_TOKENS = 512


class PrefixCache:
    """Host index (libkda.so) over a device pool of fp32 states [n_slots, H, dk, dv]."""

    def __init__(self, n_slots: int, H: int, dk: int, dv: int, block_tokens: int = BLOCK_TOKENS,
                 device="cuda"):
        self.block = int(block_tokens)
        self.handle = kda_prefix_cache_create(self.block, n_slots)
        self.pool = torch.zeros((n_slots, H, dk, dv), dtype=torch.float32, device=device)

    def close(self):
        if getattr(self, "handle", None):
            kda_prefix_cache_destroy(self.handle)
            self.handle = None

    def __del__(self):
        self.close()

    def __len__(self):
        return kda_prefix_cache_size(self.handle)

    def lookup(self, ids, max_tokens=None):
        """(cached prefix length, pool slot or -1) of one prompt."""
        return kda_prefix_cache_lookup(self.handle, ids, max_tokens)

    def plan(self, prompts):
        """Per prompt, the longest cached prefix that leaves at least one token to
        run (its output is the prompt's last position) and its slot."""
        return [self.lookup(p, max(len(p) - 1, 0)) for p in prompts]

    def gather(self, slots, stream=None):
        """Dense states [n, H, dk, dv] of the given pool slots (zeros for -1)."""
        dev = self.pool.device
        s = torch.as_tensor(slots, dtype=torch.int32).to(dev)
        out = torch.empty((s.numel(),) + tuple(self.pool.shape[1:]), dtype=torch.float32,
                          device=dev)
        return kda_state_gather(self.pool, s, out, stream=stream)

    def prefill(self, prompts, plan, q, k, v, g, beta, out_dtype=torch.float32, stream=None,
                g_logits=None):
        """Prefill of every prompt's uncached tokens from its cached state, then the
        new block-boundary states into the cache.

        q, k, v, g (or g_logits), beta: the packed inputs of tokens plan[r][0]: of
        each prompt r, in prompt order.  Returns the ``prefill`` dict for those
        tokens (o, final_state, snapshots) plus ``cached`` (tokens skipped per
        prompt)."""
        from . import prefill as _prefill
        dev = k.device
        cached = [int(m) for m, _ in plan]
        runs = [len(p) - m for p, m in zip(prompts, cached)]
        cu = [0]
        for n in runs:
            cu.append(cu[-1] + n)
        s0 = self.gather([s for _, s in plan], stream=stream)
        out = _prefill(q, k, v, g, beta, torch.tensor(cu, dtype=torch.int32, device=dev),
                       initial_state=s0, snapshot_stride=self.block, out_dtype=out_dtype,
                       cu_seqlens_host=cu, stream=stream, g_logits=g_logits)
        # snapshot row -> pool slot; a slot given out twice keeps only its last use
        rows = []
        for r, p in enumerate(prompts):
            first = cached[r] // self.block
            _, slots = kda_prefix_cache_insert(self.handle, p, first)
            n_snap = runs[r] // self.block
            rows.extend(int(slots[first + j]) for j in range(n_snap))
        seen = set()
        for i in range(len(rows) - 1, -1, -1):
            if rows[i] < 0:
                continue
            if rows[i] in seen:
                rows[i] = -1
            else:
                seen.add(rows[i])
        if any(x >= 0 for x in rows):
            kda_state_scatter(out["snapshots"], torch.tensor(rows, dtype=torch.int32, device=dev),
                              self.pool, stream=stream)
        out["cached"] = cached
        return out
