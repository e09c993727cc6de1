"""GPU parity of context parallelism across ranks (decode_kda_chunked_b200.context_parallel)
against the unsplit fp64 oracle.

One device stands in for several ranks by running every rank's phase 1,
stacking the send buffers exactly as the all-gather lays them out, and running
every rank's phase 2: no two processes share the GPU and no kernel waits on
another.  A single-rank NCCL process group then runs the public entry point
with its real all-gather."""
import datetime
import os
import socket

import numpy as np
import pytest
import torch

import oracle
from decode_kda_chunked_b200 import context_parallel as cp
from decode_kda_chunked_b200 import inputs as I
from kda_testing import TOL_BF16, TOL_F32, rel_err

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _full_oracle(x, stride):
    return oracle.prefill(x.q, x.k, x.v, x.g, x.beta, np.array([0, x.total_tokens]),
                          x.initial_state, snapshot_stride=stride)


@pytest.mark.parametrize("rank_tokens,seg_len,stride,d,dtype,tol", [
    ([512, 512, 300], 256, 128, 128, torch.bfloat16, TOL_BF16),   # tensor-core kernels
    ([0, 384, 192], 128, 64, 128, torch.bfloat16, TOL_BF16),      # empty first rank, padding
    ([256, 130], 128, 128, 64, torch.float32, TOL_F32),           # fp32 SIMT kernels
])
def test_emulated_ranks_match_unsplit_oracle(rank_tokens, seg_len, stride, d, dtype, tol):
    H = 2
    inp = I.make_prefill_inputs([sum(rank_tokens)], H, d, d, dtype=dtype, seed=41, s0_std=0.1,
                                gate_scale=0.3)
    x = inp.to(DEV)
    plan = cp.plan_context_parallel(rank_tokens, seg_len, stride)
    slices = []
    for r in range(plan.world):
        lo = plan.token_offset(r)
        sl = slice(lo, lo + rank_tokens[r])
        slices.append([t[sl] for t in (x.q, x.k, x.v, x.g, x.beta)])
    sends = [cp.local_pass(plan, r, *slices[r][1:]) for r in range(plan.world)]
    gathered = torch.cat([s.view(-1, H, d, d) for s in sends], 0)
    outs = [cp.finish_pass(plan, r, gathered, *slices[r], initial_state=x.initial_state[0])
            for r in range(plan.world)]
    torch.cuda.synchronize()

    full = _full_oracle(inp, stride)
    o = torch.cat([out["o"] for out in outs], 0)
    snaps = torch.cat([out["snapshots"] for out in outs if out["snapshots"] is not None], 0)
    assert rel_err(o, full["o"]) <= tol
    assert rel_err(snaps, full["snapshots"]) <= tol
    for out in outs:
        assert rel_err(out["final_state"], full["final_state"][0]) <= tol


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_single_rank_nccl_group_runs_the_all_gather():
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_free_port()))
    dist.init_process_group("nccl", rank=0, world_size=1, timeout=datetime.timedelta(seconds=60),
                            device_id=torch.device("cuda", torch.cuda.current_device()))
    try:
        H, d, T = 2, 128, 1000
        inp = I.make_prefill_inputs([T], H, d, d, dtype=torch.bfloat16, seed=43, s0_std=0.1,
                                    gate_scale=0.3)
        x = inp.to(DEV)
        out = cp.context_parallel_prefill(x.q, x.k, x.v, x.g, x.beta, [T], 256, 128,
                                          initial_state=x.initial_state[0])
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    full = _full_oracle(inp, 128)
    assert rel_err(out["o"], full["o"]) <= TOL_BF16
    assert rel_err(out["snapshots"], full["snapshots"]) <= TOL_BF16
    assert rel_err(out["final_state"], full["final_state"][0]) <= TOL_BF16
