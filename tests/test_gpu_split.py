"""GPU: the context-parallel split that kda_prefill_chunked takes when few chains
are live (include/kda.h, kda_prefill_chunked), against the fp64 oracle and
against the same call unsplit (KDA_NO_SPLIT=1)."""
import ctypes

import numpy as np
import pytest
import torch

import decode_kda_chunked_b200 as kda
from decode_kda_chunked_b200 import _lib
from decode_kda_chunked_b200 import inputs as I
from kda_testing import TOL_BF16, oracle_chains, rel_err

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _segments(x, stride):
    """The split kda.prefill's call gets (the same arguments, outputs included)."""
    T, H, dk = x.k.shape
    host = torch.tensor([0] + list(np.cumsum(x.lengths)), dtype=torch.int32)
    o = torch.empty(T, H, dk, device=DEV)
    fin = torch.empty(x.n_req, H, dk, dk, device=DEV)
    cu_snap = snaps = None
    if stride:
        offs = kda.snapshot_offsets(x.lengths, stride)
        cu_snap = torch.tensor(offs, dtype=torch.int32, device=DEV)
        snaps = torch.empty(max(offs[-1], 1), H, dk, dk, device=DEV)
    return kda.kda_prefill_split_segments(x.q, x.k, x.v, x.g, x.beta, x.cu_seqlens, o,
                                          x.initial_state, fin, stride, cu_snap, snaps,
                                          cu_seqlens_host=host)


def _run(x, stride, **kw):
    out = kda.prefill(x.q, x.k, x.v, x.g, x.beta, x.cu_seqlens, initial_state=x.initial_state,
                      snapshot_stride=stride, cu_seqlens_host=[0] + list(np.cumsum(x.lengths)),
                      **kw)
    assert kda.kda_get_device_status() == 0
    return out


def _check_oracle(inp, out, stride, pairs):
    ref = oracle_chains(inp, pairs, stride)
    cu = [0] + list(np.cumsum(inp.lengths))
    cs = out["cu_snapshots"].cpu().tolist() if stride else None
    for (r, h), rr in ref.items():
        lo, hi = cu[r], cu[r + 1]
        assert rel_err(out["o"][lo:hi, h].float().cpu(), rr["o"]) <= TOL_BF16, (r, h)
        assert rel_err(out["final_state"][r, h], rr["final_state"]) <= TOL_BF16, (r, h)
        if stride:
            assert rel_err(out["snapshots"][cs[r]:cs[r + 1], h], rr["snapshots"]) <= TOL_BF16


def test_single_sequence_is_split_and_matches_the_oracle():
    """B=1, H=32, T=8,192 (32 chains): four segments of the one sequence."""
    inp = I.single_seq()
    x = inp.to(DEV)
    assert _segments(x, 512) == 4
    out = _run(x, 512)
    _check_oracle(inp, out, 512, [(0, h) for h in (0, 9, 21, 31)])


def test_split_equals_unsplit(monkeypatch):
    """Two requests with initial states and snapshots; bf16 o too."""
    inp = I.make_prefill_inputs([5000, 3100], H=8, dk=128, dv=128, seed=71, s0_std=0.1,
                                gate_scale=0.3)
    x = inp.to(DEV)
    assert _segments(x, 512) > 2
    split = _run(x, 512)
    split16 = _run(x, 512, out_dtype=torch.bfloat16)
    monkeypatch.setenv("KDA_NO_SPLIT", "1")
    assert _segments(x, 512) == 0
    whole = _run(x, 512)
    for n in ("o", "final_state", "snapshots"):
        assert rel_err(split[n], whole[n]) <= TOL_BF16, n
    assert rel_err(split16["o"].float(), whole["o"]) <= 4e-3
    monkeypatch.delenv("KDA_NO_SPLIT")
    _check_oracle(inp, split, 512, [(0, 3), (1, 6)])


def test_split_with_final_state_in_place_and_gate_logits():
    """final_state aliasing initial_state, and bf16 gate logits, through the split."""
    inp = I.make_prefill_inputs([6000], H=4, dk=128, dv=128, seed=73, s0_std=0.1)
    x = inp.to(DEV)
    assert _segments(x, 0) > 1
    ref = _run(x, 0)
    state = x.initial_state.clone()
    o = torch.empty_like(ref["o"])
    kda.kda_prefill_chunked(x.q, x.k, x.v, x.g, x.beta, x.cu_seqlens, o, state, state,
                            cu_seqlens_host=torch.tensor([0, 6000], dtype=torch.int32))
    assert kda.kda_get_device_status() == 0
    assert torch.equal(o, ref["o"])
    assert torch.equal(state, ref["final_state"])
    # the same sequence with bf16 gate logits whose gate equals x.g up to bf16 rounding
    logits = torch.randn(6000, 4, 128, generator=torch.Generator().manual_seed(5)).bfloat16()
    g = (-5.0 * torch.sigmoid(logits.float())).to(DEV)
    a = kda.prefill(x.q, x.k, x.v, g, x.beta, x.cu_seqlens, initial_state=x.initial_state,
                    cu_seqlens_host=[0, 6000])
    b = kda.prefill(x.q, x.k, x.v, None, x.beta, x.cu_seqlens, initial_state=x.initial_state,
                    cu_seqlens_host=[0, 6000], g_logits=logits.to(DEV))
    assert kda.kda_get_device_status() == 0
    assert rel_err(b["o"], a["o"]) <= TOL_BF16
    assert rel_err(b["final_state"], a["final_state"]) <= TOL_BF16
