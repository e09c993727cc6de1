"""The allocation-free prefill entry point, kda_prefill_chunked_noalloc.

Some callers cannot give the library a device workspace: an engine that
hands all device memory to its own pools at start-up, a plug-in host with no
way to request scratch, or latency-critical code that cannot afford a
cudaMalloc.  For them, kda_prefill_chunked_noalloc keeps its scratch (the
longest-first order of the requests) in a fixed 64 KiB array inside
libkda.so.

These tests call it through the C ABI and compare it with the workspace entry
point, kda_prefill_chunked, on two calls in a row with different batches (the
second call must not see anything left over from the first).  The two entry
points run the same deterministic schedule and kernels, so their results must
agree bit for bit: a stale or partly written order in the shared scratch would
show up as a difference.  This file is
collected last so that, when it fails, a run that stops at the first failure
has already run every other test; it also passes when run alone in a fresh
process, where its first call does the per-device set-up.
"""
import ctypes

import numpy as np
import pytest
import torch

import decode_kda_chunked_b200 as kda
from decode_kda_chunked_b200 import _lib
from decode_kda_chunked_b200 import inputs as I

pytestmark = pytest.mark.gpu
DEV = "cuda"
STRIDE = 128


def _outputs(x):
    T, H, dk = x.k.shape
    offs = kda.snapshot_offsets(x.lengths, STRIDE)
    return {"o": torch.empty(T, H, dk, device=DEV),
            "final": torch.empty(x.n_req, H, dk, dk, device=DEV),
            "cu_snap": torch.tensor(offs, dtype=torch.int32, device=DEV),
            "snaps": torch.empty(max(offs[-1], 1), H, dk, dk, device=DEV)}


def _args(x, out):
    host = torch.tensor([0] + list(np.cumsum(x.lengths)), dtype=torch.int32)
    a = _lib.make_prefill_args(x.q, x.k, x.v, x.g, x.beta, x.cu_seqlens, out["o"],
                               x.initial_state, out["final"], STRIDE, out["cu_snap"],
                               out["snaps"], host)
    return a, host


def _with_workspace(x):
    out = _outputs(x)
    a, host = _args(x, out)
    lib = _lib.load()
    need = lib.kda_prefill_workspace_size(ctypes.byref(a))
    ws = torch.empty(max(need, 256), dtype=torch.uint8, device=DEV)
    stream = torch.cuda.current_stream().cuda_stream or None
    assert lib.kda_prefill_chunked(ctypes.byref(a), ws.data_ptr(), ws.numel(), stream) == 0
    torch.cuda.synchronize()
    return out


def _without_allocation(x):
    out = _outputs(x)
    a, host = _args(x, out)
    stream = torch.cuda.current_stream().cuda_stream or None
    assert _lib.load().kda_prefill_chunked_noalloc(ctypes.byref(a), stream) == 0
    torch.cuda.synchronize()
    return out


def test_noalloc_matches_workspace_entry_point_twice(monkeypatch):
    # the allocation-free entry point never takes the context-parallel split of few-chain
    # calls (its scratch has no room for segment states), so the workspace entry point
    # is compared with the split switched off: then both run the same kernel
    monkeypatch.setenv("KDA_NO_SPLIT", "1")
    batches = [I.make_prefill_inputs([300, 64, 1, 777, 129, 0, 512], H=4, dk=128, dv=128,
                                     seed=23, s0_std=0.1).to(DEV),
               I.make_prefill_inputs([1000, 65, 2049], H=2, dk=128, dv=128, seed=24,
                                     s0_std=0.1).to(DEV)]
    for x in batches:  # two calls in a row, different batches
        ref = _with_workspace(x)
        got = _without_allocation(x)
        n_snap = int(ref["cu_snap"][-1])
        assert torch.equal(got["o"], ref["o"])
        assert torch.equal(got["final"], ref["final"])
        assert torch.equal(got["snaps"][:n_snap], ref["snaps"][:n_snap])
    assert kda.kda_get_device_status() == 0


def test_noalloc_rejects_more_requests_than_its_scratch_holds():
    lib = _lib.load()
    a = _lib.PrefillArgs()
    a.n_req = 16385  # KDA_NOALLOC_MAX_REQUESTS + 1
    a.total_tokens, a.H, a.dk, a.dv = 16385, 1, 128, 128
    assert lib.kda_prefill_chunked_noalloc(ctypes.byref(a), None) == 6  # KDA_ERR_WORKSPACE
