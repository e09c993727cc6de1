"""Host side of the context-parallel split of few-chain prefill calls (no GPU
needed): which calls are split, into how many segments, and the workspace the
split asks for.  KDA_TEST_SM_COUNT stands in for the device's SM count."""
import ctypes

import pytest

from decode_kda_chunked_b200 import _lib

GB = 1 << 32  # fake device addresses, 4 GiB apart: aligned, never dereferenced


def _args(lengths, H, stride=0, dk=128):
    a = _lib.PrefillArgs()
    T = sum(lengths)
    a.n_req, a.total_tokens, a.H, a.dk, a.dv = len(lengths), T, H, dk, dk
    a.in_dtype, a.out_dtype = 0, 1  # bf16 in, fp32 out
    names = ["q", "k", "v", "g", "beta", "cu_seqlens", "o", "final_state"]
    if stride:
        names += ["cu_snapshots", "snapshots"]
        a.snapshot_stride = stride
    for i, n in enumerate(names):
        setattr(a, n, GB * (i + 1))
    cu = [0]
    for L in lengths:
        cu.append(cu[-1] + L)
    host = (ctypes.c_int32 * len(cu))(*cu)
    a.cu_seqlens_host = ctypes.cast(host, ctypes.c_void_p).value
    return a, host


def _segments(monkeypatch, lengths, H, stride=0, sms=148, dk=128):
    monkeypatch.setenv("KDA_TEST_SM_COUNT", str(sms))
    a, host = _args(lengths, H, stride, dk)
    lib = _lib.load()
    n = lib.kda_prefill_split_segments(ctypes.byref(a))
    ws = lib.kda_prefill_workspace_size(ctypes.byref(a))
    return n, ws


def test_single_sequence_fills_one_wave_per_pass(monkeypatch):
    # 32 chains on 148 SMs: at most 148 // 32 = 4 segments per head in each pass.  Pass 1
    # runs the first segment's prefill beside the local states of the three middle ones;
    # pass 2 runs the other four segments: 5 segments of 1,664 tokens (the last 1,536)
    n, ws = _segments(monkeypatch, [8192], H=32)
    assert n == 5
    state = 32 * 128 * 128 * 4
    assert ws >= 3 * 5 * state  # S_loc, M and start states of every segment


def test_split_switch_and_unsupported_calls(monkeypatch):
    monkeypatch.setenv("KDA_NO_SPLIT", "1")
    assert _segments(monkeypatch, [8192], H=32)[0] == 0
    monkeypatch.delenv("KDA_NO_SPLIT")
    assert _segments(monkeypatch, [8192], H=32, dk=64)[0] == 0  # no tensor-core kernel
    assert _segments(monkeypatch, [8192], H=32, sms=0)[0] == 0  # no device


def test_many_chains_are_not_split(monkeypatch):
    # 64 requests x 32 heads = 2,048 chains fill the GPU already
    n, ws = _segments(monkeypatch, [1100] * 64, H=32)
    assert n == 0
    assert ws == 64 * 4  # just the longest-first order


def test_splits_that_do_not_pay_are_not_taken(monkeypatch):
    # segments (but a request's last) hold at least 1,024 tokens, and a two-way split
    # costs about as much as the unsplit chain (local states of the first half, then
    # the second half)
    assert _segments(monkeypatch, [1500], H=2)[0] == 0
    assert _segments(monkeypatch, [1500], H=2, stride=512)[0] == 0  # 1,024 + 476
    assert _segments(monkeypatch, [2048], H=2)[0] == 0
    assert _segments(monkeypatch, [3072], H=2)[0] == 3


def test_few_heads_split_down_to_the_minimum_segment(monkeypatch):
    # 2 chains: up to 74 segments, but segments keep at least 1,024 tokens
    assert _segments(monkeypatch, [8192], H=2)[0] == 8


def test_longest_request_is_split_first(monkeypatch):
    # 16 heads: up to 148 // 16 = 9 segments per head in each pass.  The 9,000-token
    # request takes the first three extra segments (pieces 4,512, 3,008, 2,272), the
    # 3,000-token one the next (1,504), then 9,000 again (1,824, 1,504), at a tie the
    # first request (3 x 1,024), then 9,000 (1,312, 1,152): pass 1 holds 2 + 7 = 9
    # segments per head, pass 2 the 2 + 7 others
    assert _segments(monkeypatch, [3000, 9000], H=16)[0] == 11
    # 32 heads: 4 segments per head in each pass; two requests in three segments each
    # (first segments of 3,008 tokens in pass 1, the other four in pass 2)
    assert _segments(monkeypatch, [9000, 9000], H=32)[0] == 6
    assert _segments(monkeypatch, [9000], H=32)[0] == 5
    # too many chains for any split
    assert _segments(monkeypatch, [3000, 9000], H=64)[0] == 0


def test_snapshot_stride_aligns_segments(monkeypatch):
    # segments start on multiples of the stride; with 4,096 they must hold 4,096 tokens
    assert _segments(monkeypatch, [8192], H=32, stride=512)[0] == 4  # 2,048 each
    assert _segments(monkeypatch, [8192], H=32, stride=4096)[0] == 0  # only two parts
    assert _segments(monkeypatch, [16384], H=16, stride=4096)[0] == 4
