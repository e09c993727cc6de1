"""KDA oracle: fp64 CPU reference for Kimi Delta Attention (test infrastructure).

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library
``libkda.so`` and ``decode_kda_chunked_b200``) never imports it, and the two
share no code: this package wraps ``kda_oracle.c`` (plain C, fp64, one token
at a time) through ctypes and works on numpy float64 arrays.

Every function cites the passage it follows in the C source.  The recurrence
is the delta rule with a channel-wise forget gate (CSDN post on the Kimi K3
technical report, section 一.1):

    S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T,
    o_t = S_t^T q_t,   alpha_t = exp(g_t).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kda_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libkda_oracle.so")
_lib = None
_lock = threading.Lock()

_D = ctypes.POINTER(ctypes.c_double)
_I64 = ctypes.POINTER(ctypes.c_int64)


def build(src: str = _SRC, out: str = _LIB_PATH, extra_flags=()) -> str:
    """Compile the C oracle with gcc into a shared library and return its path."""
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-pthread", *extra_flags,
           src, "-o", out, "-lm"]
    subprocess.run(cmd, check=True)
    return out


def _needs_build() -> bool:
    return (not os.path.exists(_LIB_PATH)
            or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC))


def load(path: str | None = None):
    """Load (building first when stale) the oracle library; returns the ctypes handle."""
    global _lib
    if path is not None:
        return _bind(ctypes.CDLL(path))
    with _lock:
        if _lib is None:
            if _needs_build():
                build()
            _lib = _bind(ctypes.CDLL(_LIB_PATH))
    return _lib


def _bind(lib):
    lib.oracle_kda_prefill.restype = ctypes.c_int
    lib.oracle_kda_prefill.argtypes = [
        ctypes.c_int, _I64, ctypes.c_int, ctypes.c_int, ctypes.c_int,
        _D, _D, _D, _D, _D, _D, ctypes.c_int, _D, _D, _D, ctypes.c_int]
    lib.oracle_kda_decode_step.restype = ctypes.c_int
    lib.oracle_kda_decode_step.argtypes = [
        ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
        _D, _D, _D, _D, _D, _D, _I64, _D, ctypes.c_int]
    lib.oracle_kda_chunk_local_state.restype = ctypes.c_int
    lib.oracle_kda_chunk_local_state.argtypes = [
        ctypes.c_int, _I64, ctypes.c_int, ctypes.c_int, ctypes.c_int,
        _D, _D, _D, _D, _D, _D, ctypes.c_int]
    lib.oracle_kda_state_combine.restype = ctypes.c_int
    lib.oracle_kda_state_combine.argtypes = [
        ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
        _D, _D, _D, _D, _D]
    lib.oracle_kda_prefill_backward.restype = ctypes.c_int
    lib.oracle_kda_prefill_backward.argtypes = [
        ctypes.c_int, _I64, ctypes.c_int, ctypes.c_int, ctypes.c_int,
        _D, _D, _D, _D, _D, _D, _D, _D, _D, _D, _D, _D, _D, _D, ctypes.c_int]
    lib.oracle_snapshot_count.restype = ctypes.c_long
    lib.oracle_snapshot_count.argtypes = [ctypes.c_long, ctypes.c_long]
    return lib


def _f64(x):
    """Exact widening to a C-contiguous float64 array (None passes through)."""
    if x is None:
        return None
    try:  # torch tensors (bf16/fp32) widen exactly through float64
        import torch
        if isinstance(x, torch.Tensor):
            x = x.detach().to("cpu", torch.float64).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _i64(x):
    try:
        import torch
        if isinstance(x, torch.Tensor):
            x = x.detach().cpu().numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(np.asarray(x, dtype=np.int64))


def _p(a, typ=_D):
    return None if a is None else a.ctypes.data_as(typ)


def default_threads() -> int:
    return max(1, os.cpu_count() or 1)


def snapshot_counts(cu_seqlens, stride: int) -> np.ndarray:
    """floor(L_r / stride) per request (0 when stride == 0)."""
    cu = _i64(cu_seqlens)
    lens = cu[1:] - cu[:-1]
    return lens // stride if stride > 0 else np.zeros_like(lens)


def gate_from_logits(x):
    """log(alpha) = -5 sigmoid(x) of gate logits x, in fp64.

    The lower-bounded decay of KDA (CSDN post on the Kimi K3 technical report,
    section 一.1): alpha >= exp(-5) for every logit, the bound every workload's
    gate is drawn under.  The pages give the bound, not the squashing function;
    the logistic sigmoid scaled to [-5, 0] is the plainest map onto that range."""
    x = _f64(x)
    with np.errstate(over="ignore"):
        return -5.0 / (1.0 + np.exp(-x))


def gate_logit_slope(x):
    """d log(alpha) / dx of ``gate_from_logits``: -5 sigmoid(x) (1 - sigmoid(x))."""
    x = _f64(x)
    with np.errstate(over="ignore"):
        s = 1.0 / (1.0 + np.exp(-x))
    return -5.0 * s * (1.0 - s)


def _gate(g, g_logits):
    if (g is None) == (g_logits is None):
        raise ValueError("give exactly one of g and g_logits")
    return _f64(g) if g is not None else gate_from_logits(g_logits)


def prefill(q, k, v, g, beta, cu_seqlens, initial_state=None, snapshot_stride: int = 0,
            want_o: bool = True, n_threads: int | None = None, lib=None, g_logits=None):
    """Token-by-token KDA over packed varlen requests.

    q, k, g: [T, H, dk]; v: [T, H, dv]; beta: [T, H]; cu_seqlens: [n_req + 1];
    initial_state: [n_req, H, dk, dv] or None (zeros).  With ``g=None``, the gate
    is ``gate_from_logits(g_logits)``.
    Returns dict(o=[T,H,dv] or None, final_state=[n_req,H,dk,dv],
    snapshots=[n_snap,H,dk,dv], cu_snapshots=[n_req+1]).
    """
    lib = lib or load()
    g = _gate(g, g_logits)
    q, k, v, g, beta = (_f64(a) for a in (q, k, v, g, beta))
    s0 = _f64(initial_state)
    cu = _i64(cu_seqlens)
    T, H, dk = k.shape
    dv = v.shape[2]
    n_req = cu.shape[0] - 1
    counts = snapshot_counts(cu, snapshot_stride)
    cu_snap = np.concatenate([[0], np.cumsum(counts)]).astype(np.int64)
    o = np.zeros((T, H, dv)) if want_o else None
    fin = np.zeros((n_req, H, dk, dv))
    snaps = np.zeros((int(cu_snap[-1]), H, dk, dv)) if snapshot_stride > 0 else None
    rc = lib.oracle_kda_prefill(
        n_req, _p(cu, _I64), H, dk, dv, _p(q), _p(k), _p(v), _p(g), _p(beta), _p(s0),
        int(snapshot_stride), _p(o), _p(fin), _p(snaps) if snaps is not None and snaps.size else None,
        int(n_threads or default_threads()))
    if rc != 0:
        raise ValueError(f"oracle_kda_prefill failed with code {rc}")
    return {"o": o, "final_state": fin,
            "snapshots": snaps if snaps is not None else np.zeros((0, H, dk, dv)),
            "cu_snapshots": cu_snap}


def prefill_backward(q, k, v, g, beta, cu_seqlens, initial_state=None, d_o=None,
                     d_final=None, n_threads: int | None = None, lib=None, g_logits=None):
    """Gradients of L = sum(d_o * o) + sum(d_final * final_state) of the prefill
    map, by reverse mode through the recurrence's defining lines
    (``oracle_kda_prefill_backward`` in kda_oracle.c).

    Returns dict(dq, dk, dv, dg, dbeta, d_initial) shaped like the inputs
    (d_initial [n_req, H, dk, dv]).  d_o / d_final / initial_state may be None.
    With ``g=None`` the gate is ``gate_from_logits(g_logits)`` and ``dg`` is the
    gradient of the logits (the chain rule through ``gate_logit_slope``)."""
    lib = lib or load()
    g = _gate(g, g_logits)
    q, k, v, g, beta = (_f64(a) for a in (q, k, v, g, beta))
    s0, do, dfin = _f64(initial_state), _f64(d_o), _f64(d_final)
    cu = _i64(cu_seqlens)
    T, H, dk = k.shape
    dv = v.shape[2]
    n_req = cu.shape[0] - 1
    out = {"dq": np.zeros((T, H, dk)), "dk": np.zeros((T, H, dk)), "dv": np.zeros((T, H, dv)),
           "dg": np.zeros((T, H, dk)), "dbeta": np.zeros((T, H)),
           "d_initial": np.zeros((n_req, H, dk, dv))}
    rc = lib.oracle_kda_prefill_backward(
        n_req, _p(cu, _I64), H, dk, dv, _p(q), _p(k), _p(v), _p(g), _p(beta), _p(s0), _p(do),
        _p(dfin), _p(out["dq"]), _p(out["dk"]), _p(out["dv"]), _p(out["dg"]), _p(out["dbeta"]),
        _p(out["d_initial"]), int(n_threads or default_threads()))
    if rc != 0:
        raise ValueError(f"oracle_kda_prefill_backward failed with code {rc}")
    if g_logits is not None:
        out["dg"] = out["dg"] * gate_logit_slope(g_logits)
    return out


def decode_step(q, k, v, g, beta, state, slot=None, n_threads: int | None = None, lib=None):
    """One KDA step for N requests.  ``state`` [P, H, dk, dv] is updated IN PLACE
    (it must already be a contiguous float64 numpy array); returns o [N, H, dv]."""
    lib = lib or load()
    q, k, v, g, beta = (_f64(a) for a in (q, k, v, g, beta))
    if not (isinstance(state, np.ndarray) and state.dtype == np.float64
            and state.flags["C_CONTIGUOUS"]):
        raise TypeError("state must be a C-contiguous float64 numpy array (updated in place)")
    N, H, dk = k.shape
    dv = v.shape[2]
    sl = _i64(slot) if slot is not None else None
    o = np.zeros((N, H, dv))
    rc = lib.oracle_kda_decode_step(N, H, dk, dv, _p(q), _p(k), _p(v), _p(g), _p(beta),
                                    _p(state), _p(sl, _I64), _p(o),
                                    int(n_threads or default_threads()))
    if rc != 0:
        raise ValueError(f"oracle_kda_decode_step failed with code {rc}")
    return o


def chunk_local_state(k, v, g, beta, seg_cu, n_threads: int | None = None, lib=None,
                      g_logits=None):
    """Per segment and head: (S_loc [n_seg,H,dk,dv], M [n_seg,H,dk,dk]).  With
    ``g=None`` the gate is ``gate_from_logits(g_logits)``."""
    lib = lib or load()
    g = _gate(g, g_logits)
    k, v, g, beta = (_f64(a) for a in (k, v, g, beta))
    seg = _i64(seg_cu)
    _, H, dk = k.shape
    dv = v.shape[2]
    n_seg = seg.shape[0] - 1
    s_loc = np.zeros((n_seg, H, dk, dv))
    m = np.zeros((n_seg, H, dk, dk))
    rc = lib.oracle_kda_chunk_local_state(n_seg, _p(seg, _I64), H, dk, dv, _p(k), _p(v),
                                          _p(g), _p(beta), _p(s_loc), _p(m),
                                          int(n_threads or default_threads()))
    if rc != 0:
        raise ValueError(f"oracle_kda_chunk_local_state failed with code {rc}")
    return s_loc, m


def state_combine(s_loc, m, s_init=None, lib=None):
    """Serial combine: returns (S_in [n_seg,H,dk,dv], S_final [H,dk,dv])."""
    lib = lib or load()
    s_loc, m, s_init = _f64(s_loc), _f64(m), _f64(s_init)
    n_seg, H, dk, dv = s_loc.shape
    s_in = np.zeros_like(s_loc)
    s_fin = np.zeros((H, dk, dv))
    rc = lib.oracle_kda_state_combine(n_seg, H, dk, dv, _p(s_loc), _p(m), _p(s_init),
                                      _p(s_in), _p(s_fin))
    if rc != 0:
        raise ValueError(f"oracle_kda_state_combine failed with code {rc}")
    return s_in, s_fin
