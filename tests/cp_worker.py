"""One rank of the CPU (gloo) context-parallel test.

Drives the host side of decode_kda_chunked_b200.context_parallel -- the plan,
the send buffer with its (0, I) padding, the one all-gather and the unpacking
into sequence order -- with the fp64 oracle standing in for the two kernels
(local state + transition, and the prefill), so the exchange logic is checked
without a GPU.  Every rank regenerates the same seeded sequence and keeps its
own slice.  Writes o, snapshots and the final state of its slice to
<out>/rank<r>.npz.
"""
import argparse
import datetime
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402
import torch.distributed as dist  # noqa: E402

import oracle  # noqa: E402
from decode_kda_chunked_b200 import context_parallel as cp  # noqa: E402
from decode_kda_chunked_b200 import inputs as I  # noqa: E402


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--rank", type=int, required=True)
    ap.add_argument("--spec", required=True)  # json: rank_tokens, seg_len, stride, H, d, seed
    ap.add_argument("--out", required=True)
    a = ap.parse_args()
    spec = json.loads(a.spec)
    rank_tokens, H, d = spec["rank_tokens"], spec["H"], spec["d"]
    world = len(rank_tokens)
    dist.init_process_group("gloo", rank=a.rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    plan = cp.plan_context_parallel(rank_tokens, spec["seg_len"], spec["stride"])
    x = I.make_prefill_inputs([sum(rank_tokens)], H, d, d, dtype=torch.float32,
                              seed=spec["seed"], s0_std=0.1)
    lo = plan.token_offset(a.rank)
    sl = slice(lo, lo + rank_tokens[a.rank])
    q, k, v, g, beta = (t[sl] for t in (x.q, x.k, x.v, x.g, x.beta))

    buf, s_loc, m = cp.send_buffer(plan, a.rank, H, d, "cpu")
    n = plan.n_local(a.rank)
    if n:  # stand-in for kda_chunk_local_state
        rs, rm = oracle.chunk_local_state(k, v, g, beta, np.array(plan.seg_bounds[a.rank]))
        s_loc.copy_(torch.from_numpy(rs))
        m.copy_(torch.from_numpy(rm))
    gathered = cp.exchange(plan, buf)
    all_loc, all_m = cp.unpack_gathered(plan, gathered)
    # stand-in for kda_state_combine, then for the prefill of the rank's segments
    s_in, s_fin = oracle.state_combine(all_loc.numpy(), all_m.numpy(), x.initial_state[0])
    first = plan.first_slot(a.rank)
    own = s_in[first:first + n]
    if n:
        res = oracle.prefill(q, k, v, g, beta, np.array(plan.seg_bounds[a.rank]), own,
                             snapshot_stride=plan.snapshot_stride)
        o, snaps = res["o"], res["snapshots"]
    else:
        o, snaps = np.zeros((0, H, d)), np.zeros((0, H, d, d))
    np.savez(os.path.join(a.out, f"rank{a.rank}.npz"), o=o, snaps=snaps, fin=s_fin,
             n_local=n, n_max=plan.n_max)
    dist.destroy_process_group()


if __name__ == "__main__":
    main()
