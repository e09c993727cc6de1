"""decode_kda_chunked_b200: Kimi Delta Attention (KDA) on NVIDIA B200 (sm_100a).

The compute lives in libkda.so (C ABI in include/kda.h); this package is its
Python binding.  The same-named functions (``kda_prefill_chunked``,
``kda_chunk_local_state``, ``kda_state_combine``, ``kda_decode_step``) take
caller-allocated torch CUDA tensors; the short helpers below (``prefill``,
``long_context_prefill``, ``decode_step``) only allocate the outputs with
torch and call them.  PyTorch provides device memory and streams; nothing
here computes any part of KDA.
"""
from __future__ import annotations

import torch

from ._lib import (CHUNK, KdaError, kda_chunk_local_state, kda_decode_step,  # noqa: F401
                   kda_get_device_status, kda_prefill_backward,
                   kda_prefill_backward_workspace_size, kda_prefill_chunked,
                   kda_prefill_workspace_size, kda_prefill_split_segments, make_backward_args,
                   kda_prefill_uses_tensor_cores, kda_snapshot_count, kda_state_combine,
                   kda_status_string, kda_version, load, make_prefill_args)

__all__ = ["kda_prefill_chunked", "kda_chunk_local_state", "kda_state_combine",
           "kda_decode_step", "kda_snapshot_count", "kda_get_device_status",
           "kda_status_string", "kda_version", "kda_prefill_workspace_size", "KdaError",
           "kda_prefill_uses_tensor_cores", "kda_prefill_backward",
           "kda_prefill_backward_workspace_size", "kda_prefill_split_segments",
           "prefill", "prefill_backward", "long_context_prefill", "decode_step",
           "snapshot_offsets", "load", "PrefixCache"]


def snapshot_offsets(lengths, stride: int) -> list:
    """cu_snapshots as a host list: prefix sums of floor(L_r / stride)."""
    out = [0]
    for L in lengths:
        out.append(out[-1] + (int(L) // stride if stride > 0 else 0))
    return out


def _host_lengths(cu_seqlens, cu_seqlens_host):
    cu = cu_seqlens_host if cu_seqlens_host is not None else cu_seqlens.detach().cpu()
    cu = [int(x) for x in (cu.tolist() if isinstance(cu, torch.Tensor) else cu)]
    return cu, [b - a for a, b in zip(cu[:-1], cu[1:])]


def prefill(q, k, v, g, beta, cu_seqlens, initial_state=None, snapshot_stride: int = 0,
            out_dtype=torch.float32, want_final: bool = True, cu_seqlens_host=None,
            stream=None, g_logits=None) -> dict:
    """Chunked prefill over packed requests; allocates o / final / snapshots.
    The gate is ``g`` (fp32 log alpha) or, with ``g=None``, ``g_logits`` (bf16
    logits x, log alpha = -5 sigmoid(x) computed in the kernels).

    Returns dict(o, final_state, snapshots, cu_snapshots)."""
    T, H, dk = k.shape
    dv = v.shape[2]
    dev = k.device
    cu_host, lengths = _host_lengths(cu_seqlens, cu_seqlens_host)
    n_req = len(lengths)
    o = torch.empty((T, H, dv), dtype=out_dtype, device=dev)
    fin = torch.empty((n_req, H, dk, dv), dtype=torch.float32, device=dev) if want_final else None
    cu_snap = snaps = None
    if snapshot_stride > 0:
        offs = snapshot_offsets(lengths, snapshot_stride)
        cu_snap = torch.tensor(offs, dtype=torch.int32, device=dev)
        # at least one row so the pointer is valid even when no request reaches the stride
        snaps = torch.empty((max(offs[-1], 1), H, dk, dv), dtype=torch.float32, device=dev)
    kda_prefill_chunked(q, k, v, g, beta, cu_seqlens, o, initial_state, fin, snapshot_stride,
                        cu_snap, snaps, cu_seqlens_host=torch.tensor(cu_host, dtype=torch.int32),
                        stream=stream, g_logits=g_logits)
    if snaps is not None:
        snaps = snaps[:offs[-1]]
    return {"o": o, "final_state": fin, "snapshots": snaps, "cu_snapshots": cu_snap}


def prefill_backward(q, k, v, g, beta, cu_seqlens, d_o=None, d_final=None, initial_state=None,
                     want_initial: bool = True, cu_seqlens_host=None, stream=None,
                     g_logits=None) -> dict:
    """Gradients of sum(d_o * o) + sum(d_final * final_state) of ``prefill`` for the
    same inputs; allocates the fp32 gradients and the workspace.  With ``g_logits``
    (and ``g=None``) the returned ``dg`` is the gradient of the logits.

    Returns dict(dq, dk, dv, dg, dbeta, d_initial)."""
    T, H, dk = k.shape
    dv = v.shape[2]
    dev = k.device
    cu_host, lengths = _host_lengths(cu_seqlens, cu_seqlens_host)
    f32 = dict(dtype=torch.float32, device=dev)
    dq, dk_, dg = (torch.empty((T, H, dk), **f32) for _ in range(3))
    dv_ = torch.empty((T, H, dv), **f32)
    db = torch.empty((T, H), **f32)
    d0 = torch.empty((len(lengths), H, dk, dv), **f32) if want_initial else None
    kda_prefill_backward(q, k, v, g, beta, cu_seqlens, torch.tensor(cu_host, dtype=torch.int32),
                         dq, dk_, dv_, dg, db, initial_state=initial_state, d_o=d_o,
                         d_final=d_final, d_initial=d0, stream=stream, g_logits=g_logits)
    return {"dq": dq, "dk": dk_, "dv": dv_, "dg": dg, "dbeta": db, "d_initial": d0}


def long_context_prefill(q, k, v, g, beta, seg_len: int, snapshot_stride: int = 512,
                         initial_state=None, out_dtype=torch.float32, stream=None,
                         g_logits=None) -> dict:
    """One long sequence split into segments of ``seg_len`` tokens (KDA context
    parallelism on one device): local zero-start states and transitions per
    segment, an exact combine, then the chunked prefill of every segment from
    its recovered start state.  ``seg_len`` must be a multiple of 64 and of
    ``snapshot_stride`` so per-segment snapshots tile the sequence.

    q, k, g: [T, H, d]; v: [T, H, d]; beta: [T, H]; initial_state: [H, d, d] or None.
    Returns dict(o, final_state [H,d,d], snapshots, s_in, s_loc, m)."""
    T, H, dk = k.shape
    dv = v.shape[2]
    dev = k.device
    if seg_len <= 0 or seg_len % CHUNK or (snapshot_stride and seg_len % snapshot_stride):
        raise ValueError("seg_len must be a positive multiple of 64 and of snapshot_stride")
    bounds = list(range(0, T, seg_len)) + [T]
    n_seg = len(bounds) - 1
    seg_cu = torch.tensor(bounds, dtype=torch.int32, device=dev)
    s_loc = torch.empty((n_seg, H, dk, dv), dtype=torch.float32, device=dev)
    m = torch.empty((n_seg, H, dk, dk), dtype=torch.float32, device=dev)
    kda_chunk_local_state(k, v, g, beta, seg_cu, s_loc, m,
                          seg_cu_host=torch.tensor(bounds, dtype=torch.int32), stream=stream,
                          g_logits=g_logits)
    s_in = torch.empty_like(s_loc)
    kda_state_combine(s_loc, m, initial_state, s_in, None, stream=stream)
    out = prefill(q, k, v, g, beta, seg_cu, initial_state=s_in,
                  snapshot_stride=snapshot_stride, out_dtype=out_dtype,
                  cu_seqlens_host=bounds, stream=stream, g_logits=g_logits)
    return {"o": out["o"], "final_state": out["final_state"][-1], "snapshots": out["snapshots"],
            "s_in": s_in, "s_loc": s_loc, "m": m}


def decode_step(q, k, v, g, beta, state, slot=None, out_dtype=torch.float32, stream=None):
    """One token per request; ``state`` is updated in place.  Returns o [N, H, dv]."""
    o = torch.empty((k.shape[0], k.shape[1], v.shape[2]), dtype=out_dtype, device=k.device)
    return kda_decode_step(q, k, v, g, beta, state, o, slot, stream=stream)


from .prefix_cache import PrefixCache  # noqa: E402  (needs prefill above)
