"""KDA context parallelism across ranks: one long sequence split over devices.

Source: KDA context parallelism ("Kimi K3 开源日来了", Infra section, first
layer; section 三.1 of the CSDN post on the Kimi K3 technical report).  A
segment's effect on the recurrent state is affine in the state that enters
it: running the segment from a start state X gives M X + S_loc, where S_loc is
the state the segment reaches from zero and M = A_L ... A_1 is the product of
its per-token transitions.  Each rank computes (S_loc, M) for its own
segments, the ranks exchange those fixed-size pairs once, and every rank then
knows the exact start state of each of its segments.

The path on each rank, with every arithmetic step in libkda.so:

  phase 1  ``kda_chunk_local_state`` over the rank's segments, written straight
           into the send buffer ``[2, n_max, H, d, d]`` (S_loc block, M block);
           slots past the rank's own segments hold (0, I), an exact no-op of
           the combine.
  exchange one all-gather of the send buffers (2 * n_max * H * d * d fp32 per
           rank) -- the only collective.
  phase 2  ``kda_state_combine`` over all gathered segments in sequence order
           (every rank runs the same short serial scan, so every rank also
           holds the global final state), then ``kda_prefill_chunked`` over the
           rank's own segments from their recovered start states.

Rank r holds the contiguous token slice ``[sum(rank_tokens[:r]), +rank_tokens[r])``.
Every rank but the last holds a multiple of ``seg_len`` tokens, so segment
boundaries -- and snapshot boundaries, ``seg_len`` being a multiple of the
snapshot stride -- fall at the same global positions as in one unsplit run.

The two phases are separate functions so the host logic can be driven
without a process group (one device standing in for several ranks by
stacking their send buffers) and tested on the CPU with stand-in compute.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch

from ._lib import CHUNK, kda_chunk_local_state, kda_state_combine


@dataclass(frozen=True)
class CpPlan:
    """Segment layout of a context-parallel run, identical on every rank."""
    rank_tokens: tuple      # tokens held by each rank
    seg_len: int
    snapshot_stride: int
    seg_bounds: tuple       # per rank: local segment boundaries (0 .. rank_tokens[r])
    n_max: int              # segments per rank in the exchange (the largest count)

    @property
    def world(self) -> int:
        return len(self.rank_tokens)

    def n_local(self, rank: int) -> int:
        return len(self.seg_bounds[rank]) - 1

    def token_offset(self, rank: int) -> int:
        return sum(self.rank_tokens[:rank])

    def first_slot(self, rank: int) -> int:
        """Index of the rank's first segment among the gathered slots."""
        return rank * self.n_max


def plan_context_parallel(rank_tokens, seg_len: int, snapshot_stride: int = 0) -> CpPlan:
    """Validate a split and lay out its segments.  Raises ValueError on a split
    whose segment or snapshot boundaries would not match the unsplit run."""
    rank_tokens = tuple(int(t) for t in rank_tokens)
    if not rank_tokens:
        raise ValueError("rank_tokens must list at least one rank")
    if seg_len <= 0 or seg_len % CHUNK:
        raise ValueError(f"seg_len must be a positive multiple of {CHUNK}")
    if snapshot_stride < 0 or (snapshot_stride and (snapshot_stride % CHUNK or seg_len % snapshot_stride)):
        raise ValueError("snapshot_stride must be 0 or a multiple of 64 dividing seg_len")
    if any(t < 0 for t in rank_tokens):
        raise ValueError("token counts must be non-negative")
    if any(t % seg_len for t in rank_tokens[:-1]):
        raise ValueError("every rank but the last must hold a multiple of seg_len tokens")
    bounds = tuple(tuple(list(range(0, t, seg_len)) + [t]) if t else (0,) for t in rank_tokens)
    n_max = max(len(b) - 1 for b in bounds)
    return CpPlan(rank_tokens, seg_len, snapshot_stride, bounds, n_max)


def send_buffer(plan: CpPlan, rank: int, H: int, d: int, device) -> tuple:
    """The rank's send buffer [2, n_max, H, d, d] fp32 and the (S_loc, M) views
    of its own segments; padding slots hold S_loc = 0, M = I."""
    buf = torch.empty((2, plan.n_max, H, d, d), dtype=torch.float32, device=device)
    n = plan.n_local(rank)
    if n < plan.n_max:
        buf[0, n:].zero_()
        buf[1, n:].copy_(torch.eye(d, dtype=torch.float32, device=device).expand(plan.n_max - n, H, d, d))
    return buf, buf[0, :n], buf[1, :n]


def local_pass(plan: CpPlan, rank: int, k, v, g, beta, stream=None) -> torch.Tensor:
    """Phase 1 on this rank's slice (k, v, g: [T_r, H, d]; beta: [T_r, H]):
    returns the send buffer filled with the rank's (S_loc, M)."""
    T, H, d = k.shape
    if T != plan.rank_tokens[rank]:
        raise ValueError(f"rank {rank} holds {T} tokens, the plan says {plan.rank_tokens[rank]}")
    if v.shape[2] != d:
        raise ValueError("context parallelism needs dk == dv")
    buf, s_loc, m = send_buffer(plan, rank, H, d, k.device)
    if plan.n_local(rank):
        bounds = list(plan.seg_bounds[rank])
        kda_chunk_local_state(k, v, g, beta, torch.tensor(bounds, dtype=torch.int32, device=k.device),
                              s_loc, m, seg_cu_host=torch.tensor(bounds, dtype=torch.int32),
                              stream=stream)
    return buf


def unpack_gathered(plan: CpPlan, gathered: torch.Tensor) -> tuple:
    """[world * 2 * n_max, H, d, d] (rank-major, as the all-gather lays it out)
    -> contiguous (S_loc, M), each [world * n_max, H, d, d] in sequence order."""
    w, n = plan.world, plan.n_max
    g6 = gathered.view(w, 2, n, *gathered.shape[1:])
    return (g6[:, 0].reshape(w * n, *gathered.shape[1:]).contiguous(),
            g6[:, 1].reshape(w * n, *gathered.shape[1:]).contiguous())


def exchange(plan: CpPlan, send: torch.Tensor, group=None) -> torch.Tensor:
    """The one collective: all-gather of every rank's send buffer (skipped only
    for a single rank with no process group)."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        if plan.world != 1:
            raise RuntimeError("a multi-rank plan needs an initialised process group")
        return send.view(-1, *send.shape[2:])
    if dist.get_world_size(group) != plan.world:
        raise ValueError("the process group size differs from the plan's rank count")
    out = torch.empty((plan.world * send.shape[0] * send.shape[1], *send.shape[2:]),
                      dtype=send.dtype, device=send.device)
    dist.all_gather_into_tensor(out, send.view(-1, *send.shape[2:]).contiguous(), group=group)
    return out


def finish_pass(plan: CpPlan, rank: int, gathered, q, k, v, g, beta, initial_state=None,
                out_dtype=torch.float32, stream=None) -> dict:
    """Phase 2: combine over all gathered segments, then the chunked prefill of
    this rank's segments from their start states.

    Returns dict(o [T_r, H, dv], snapshots [T_r // stride, H, d, d] or None,
    final_state [H, d, d] (the whole sequence's), s_in [n_local, H, d, d])."""
    from . import prefill
    s_loc, m = unpack_gathered(plan, gathered)
    H, d = s_loc.shape[1], s_loc.shape[2]
    s_in = torch.empty_like(s_loc)
    s_final = torch.empty((H, d, d), dtype=torch.float32, device=s_loc.device)
    kda_state_combine(s_loc, m, initial_state, s_in, s_final, stream=stream)
    n = plan.n_local(rank)
    first = plan.first_slot(rank)
    own_in = s_in[first:first + n]
    T = plan.rank_tokens[rank]
    if n == 0:
        return {"o": torch.empty((0, H, v.shape[2]), dtype=out_dtype, device=s_loc.device),
                "snapshots": None, "final_state": s_final, "s_in": own_in}
    bounds = list(plan.seg_bounds[rank])
    out = prefill(q, k, v, g, beta, torch.tensor(bounds, dtype=torch.int32, device=k.device),
                  initial_state=own_in.contiguous(), snapshot_stride=plan.snapshot_stride,
                  out_dtype=out_dtype, want_final=False, cu_seqlens_host=bounds, stream=stream)
    snaps = out["snapshots"]
    if snaps is not None and snaps.shape[0] != (T // plan.snapshot_stride):
        raise RuntimeError("snapshot count of the rank's slice does not tile the sequence")
    return {"o": out["o"], "snapshots": snaps, "final_state": s_final, "s_in": own_in}


def context_parallel_prefill(q, k, v, g, beta, rank_tokens, seg_len: int,
                             snapshot_stride: int = 512, initial_state=None,
                             out_dtype=torch.float32, group=None, stream=None) -> dict:
    """One long sequence split over the ranks of ``group`` (one process per GPU).

    q, k, v, g: this rank's token slice [T_r, H, d]; beta [T_r, H];
    rank_tokens: every rank's T_r (the same list on every rank);
    initial_state: [H, d, d] start state of the whole sequence, on every rank
    (or None for zeros).  Returns this rank's o and snapshots (global snapshot
    rows ``sum(rank_tokens[:r]) // stride`` onwards), and the whole sequence's
    final state on every rank.  Everything, the collective included, is
    ordered on ``stream`` (torch's current stream when None)."""
    import contextlib

    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        rank = dist.get_rank(group)
    else:
        rank = 0
    plan = plan_context_parallel(rank_tokens, seg_len, snapshot_stride)
    ctx = torch.cuda.stream(stream) if stream is not None else contextlib.nullcontext()
    with ctx:
        send = local_pass(plan, rank, k, v, g, beta)
        gathered = exchange(plan, send, group)
        return finish_pass(plan, rank, gathered, q, k, v, g, beta, initial_state=initial_state,
                           out_dtype=out_dtype)
