"""Shared helpers for the parity tests: tolerance metric and oracle sampling.

Tolerance metric (applied per output tensor): max_i |x_i - ref_i| / max_i |ref_i|,
with limits 2e-3 for bf16 inputs with fp32 accumulation and 1e-5 for fp32
inputs.  A purely elementwise relative error is unusable near zeros.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle

TOL_BF16 = 2e-3
TOL_F32 = 1e-5


def rel_err(x, ref) -> float:
    x = x.detach().double().cpu().numpy() if isinstance(x, torch.Tensor) else np.asarray(x)
    ref = ref.detach().double().cpu().numpy() if isinstance(ref, torch.Tensor) else np.asarray(ref)
    assert x.shape == ref.shape, (x.shape, ref.shape)
    if ref.size == 0:
        return 0.0
    den = np.max(np.abs(ref))
    num = np.max(np.abs(x - ref))
    return float(num / den) if den > 0 else float(num)


def oracle_chain(inp, r: int, h: int, stride: int = 0, want_o: bool = True):
    """Oracle for one (request, head) chain of a PrefillInputs (any device)."""
    cu = [int(x) for x in inp.cu_seqlens.cpu().tolist()]
    lo, hi = cu[r], cu[r + 1]
    sl = lambda t: t[lo:hi, h:h + 1].cpu()
    s0 = None if inp.initial_state is None else inp.initial_state[r:r + 1, h:h + 1].cpu()
    out = oracle.prefill(sl(inp.q), sl(inp.k), sl(inp.v), sl(inp.g), inp.beta[lo:hi, h:h + 1].cpu(),
                         np.array([0, hi - lo]), s0, snapshot_stride=stride, want_o=want_o,
                         n_threads=1)
    return out


def oracle_chains(inp, pairs, stride: int = 0, want_o: bool = True):
    """Oracle for several (request, head) chains at once: the chains are packed
    as separate one-head requests into one oracle call, so its thread pool runs
    them in parallel.  Returns {(r, h): dict(o, final_state, snapshots)}."""
    cu = [int(x) for x in inp.cu_seqlens.cpu().tolist()]
    parts = {n: [] for n in ("q", "k", "v", "g", "beta", "s0")}
    lens = []
    for (r, h) in pairs:
        lo, hi = cu[r], cu[r + 1]
        lens.append(hi - lo)
        for n in ("q", "k", "v", "g"):
            parts[n].append(getattr(inp, n)[lo:hi, h:h + 1].cpu().double())
        parts["beta"].append(inp.beta[lo:hi, h:h + 1].cpu().double())
        if inp.initial_state is not None:
            parts["s0"].append(inp.initial_state[r:r + 1, h:h + 1].cpu().double())
    cat = {n: torch.cat(v, 0) for n, v in parts.items() if v}
    pcu = np.concatenate([[0], np.cumsum(lens)])
    res = oracle.prefill(cat["q"], cat["k"], cat["v"], cat["g"], cat["beta"], pcu,
                         cat.get("s0"), snapshot_stride=stride, want_o=want_o)
    out = {}
    cs = res["cu_snapshots"]
    for i, rh in enumerate(pairs):
        out[rh] = {"o": None if res["o"] is None else res["o"][pcu[i]:pcu[i + 1], 0],
                   "final_state": res["final_state"][i, 0],
                   "snapshots": res["snapshots"][cs[i]:cs[i + 1], 0]}
    return out
