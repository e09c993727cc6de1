"""Context parallelism across ranks, host side (CPU, gloo): the split plan,
the send buffer's (0, I) padding, the one all-gather of (S_loc, M) and the
unpacking into sequence order.  The oracle stands in for the kernels (see
cp_worker.py); results are checked against the unsplit oracle run, which the
split reaches exactly in exact arithmetic (KDA context parallelism, "Kimi K3
开源日来了", Infra section, first layer)."""
import json
import os
import socket
import subprocess
import sys

import numpy as np
import pytest
import torch

import oracle
from decode_kda_chunked_b200 import context_parallel as cp
from decode_kda_chunked_b200 import inputs as I

HERE = os.path.dirname(os.path.abspath(__file__))


def test_plan_layout():
    p = cp.plan_context_parallel([256, 256, 100], 128, 64)
    assert p.world == 3 and p.n_max == 2
    assert p.seg_bounds == ((0, 128, 256), (0, 128, 256), (0, 100))
    assert [p.n_local(r) for r in range(3)] == [2, 2, 1]
    assert [p.token_offset(r) for r in range(3)] == [0, 256, 512]
    assert [p.first_slot(r) for r in range(3)] == [0, 2, 4]
    e = cp.plan_context_parallel([0, 192], 64, 0)
    assert e.seg_bounds == ((0,), (0, 64, 128, 192)) and e.n_max == 3


@pytest.mark.parametrize("bad", [
    dict(rank_tokens=[100, 128], seg_len=64, stride=0),     # ragged slice before the last rank
    dict(rank_tokens=[128], seg_len=96, stride=0),          # segment not a multiple of 64
    dict(rank_tokens=[128], seg_len=128, stride=96),        # stride not a multiple of 64
    dict(rank_tokens=[256], seg_len=128, stride=256),       # stride does not divide seg_len
    dict(rank_tokens=[], seg_len=64, stride=0),
    dict(rank_tokens=[64, -64], seg_len=64, stride=0),
])
def test_plan_rejects_splits_that_break_boundaries(bad):
    with pytest.raises(ValueError):
        cp.plan_context_parallel(bad["rank_tokens"], bad["seg_len"], bad["stride"])


def test_send_buffer_padding_is_the_combine_identity():
    p = cp.plan_context_parallel([128, 64], 64, 64)
    buf, s_loc, m = cp.send_buffer(p, 1, 2, 4, "cpu")
    assert buf.shape == (2, 2, 2, 4, 4) and s_loc.shape == (1, 2, 4, 4) and m.shape == (1, 2, 4, 4)
    assert torch.equal(buf[0, 1], torch.zeros(2, 4, 4))
    assert torch.equal(buf[1, 1], torch.eye(4).expand(2, 4, 4))
    # the views alias the buffer: a kernel writing them fills the send buffer
    s_loc.fill_(3.0)
    assert torch.equal(buf[0, 0], torch.full((2, 4, 4), 3.0))


def test_unpack_gathered_orders_segments_by_rank_then_slot():
    p = cp.plan_context_parallel([128, 128, 64], 64, 0)
    H, d = 1, 2
    bufs = []
    for r in range(3):
        b = torch.zeros(2, p.n_max, H, d, d)
        for s in range(p.n_max):
            b[0, s] = 10 * r + s          # S_loc tag
            b[1, s] = -(10 * r + s)       # M tag
        bufs.append(b.view(-1, H, d, d))
    s_loc, m = cp.unpack_gathered(p, torch.cat(bufs, 0))
    assert s_loc[:, 0, 0, 0].tolist() == [0, 1, 10, 11, 20, 21]
    assert m[:, 0, 0, 0].tolist() == [0, -1, -10, -11, -20, -21]
    assert s_loc.is_contiguous() and m.is_contiguous()


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("rank_tokens,seg_len,stride", [
    ([256, 192], 64, 64),        # uneven segment counts: padding on rank 1
    ([128, 128, 100], 128, 64),  # three ranks, ragged tail
    ([0, 192], 64, 64),          # an empty rank contributes only padding
])
def test_gloo_ranks_match_unsplit_oracle(tmp_path, rank_tokens, seg_len, stride):
    H, d, seed = 2, 8, 5
    spec = json.dumps(dict(rank_tokens=rank_tokens, seg_len=seg_len, stride=stride, H=H, d=d,
                           seed=seed))
    env = dict(os.environ, MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_free_port()),
               OMP_NUM_THREADS="1")
    procs = [subprocess.Popen([sys.executable, os.path.join(HERE, "cp_worker.py"), "--rank",
                               str(r), "--spec", spec, "--out", str(tmp_path)], env=env,
                              stdout=subprocess.PIPE, stderr=subprocess.STDOUT)
             for r in range(len(rank_tokens))]
    for p in procs:
        out, _ = p.communicate(timeout=180)
        assert p.returncode == 0, out.decode()[-2000:]
    res = [np.load(tmp_path / f"rank{r}.npz") for r in range(len(rank_tokens))]

    x = I.make_prefill_inputs([sum(rank_tokens)], H, d, d, dtype=torch.float32, seed=seed,
                              s0_std=0.1)
    full = oracle.prefill(x.q, x.k, x.v, x.g, x.beta, np.array([0, x.total_tokens]),
                          x.initial_state, snapshot_stride=stride)
    o = np.concatenate([r["o"] for r in res], 0)
    snaps = np.concatenate([r["snaps"] for r in res], 0)
    scale = lambda a: max(np.abs(a).max(), 1e-30)
    # the exchange carries fp32 (S_loc, M); everything else is fp64
    assert np.abs(o - full["o"]).max() / scale(full["o"]) < 1e-5
    assert snaps.shape == full["snapshots"].shape
    assert np.abs(snaps - full["snapshots"]).max() / scale(full["snapshots"]) < 1e-5
    for r in res:  # every rank holds the whole sequence's final state
        assert np.abs(r["fin"] - full["final_state"][0]).max() / scale(full["final_state"]) < 1e-5
