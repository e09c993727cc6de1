"""ctypes binding of libkda.so (include/kda.h): argument marshalling only.

Every compute step runs in the CUDA kernels of libkda.so.  This module turns
torch tensors into the raw device pointers and sizes of the C ABI, passes the
current CUDA stream, and raises on any non-zero status.  If the library is not
built, importing the entry points raises immediately: there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libkda.so")

KDA_BF16, KDA_F32 = 0, 1
CHUNK = 64
STATUS_NAMES = {0: "KDA_OK", 1: "KDA_ERR_INVALID_ARG", 2: "KDA_ERR_UNSUPPORTED",
                3: "KDA_ERR_CUDA", 4: "KDA_ERR_GATE_RANGE", 5: "KDA_ERR_TIMEOUT",
                6: "KDA_ERR_WORKSPACE"}

_vp = ctypes.c_void_p
_i32 = ctypes.c_int32


class PrefillArgs(ctypes.Structure):
    _fields_ = [("n_req", _i32), ("total_tokens", _i32), ("H", _i32), ("dk", _i32), ("dv", _i32),
                ("in_dtype", ctypes.c_int), ("out_dtype", ctypes.c_int),
                ("q", _vp), ("k", _vp), ("v", _vp), ("g", _vp), ("beta", _vp),
                ("cu_seqlens", _vp), ("cu_seqlens_host", _vp), ("initial_state", _vp),
                ("o", _vp), ("final_state", _vp), ("snapshot_stride", _i32),
                ("cu_snapshots", _vp), ("snapshots", _vp), ("g_logits", _vp)]


class LocalStateArgs(ctypes.Structure):
    _fields_ = [("n_seg", _i32), ("total_tokens", _i32), ("H", _i32), ("dk", _i32), ("dv", _i32),
                ("in_dtype", ctypes.c_int), ("k", _vp), ("v", _vp), ("g", _vp), ("beta", _vp),
                ("seg_cu", _vp), ("seg_cu_host", _vp), ("s_loc", _vp), ("m", _vp),
                ("g_logits", _vp)]


class DecodeArgs(ctypes.Structure):
    _fields_ = [("n", _i32), ("H", _i32), ("dk", _i32), ("dv", _i32),
                ("in_dtype", ctypes.c_int), ("out_dtype", ctypes.c_int),
                ("q", _vp), ("k", _vp), ("v", _vp), ("g", _vp), ("beta", _vp),
                ("state", _vp), ("n_slots", _i32), ("slot", _vp), ("o", _vp)]


class BackwardArgs(ctypes.Structure):
    _fields_ = [("n_req", _i32), ("total_tokens", _i32), ("H", _i32), ("dk", _i32), ("dv", _i32),
                ("in_dtype", ctypes.c_int), ("q", _vp), ("k", _vp), ("v", _vp), ("g", _vp),
                ("beta", _vp), ("cu_seqlens", _vp), ("cu_seqlens_host", _vp),
                ("initial_state", _vp), ("d_o", _vp), ("d_final", _vp), ("d_q", _vp),
                ("d_k", _vp), ("d_v", _vp), ("d_g", _vp), ("d_beta", _vp), ("d_initial", _vp),
                ("g_logits", _vp)]


class KdaError(RuntimeError):
    def __init__(self, fn: str, code: int):
        super().__init__(f"{fn} returned {STATUS_NAMES.get(code, code)}")
        self.code = code


_lib = None
_lock = threading.Lock()

EXPORTS = ("kda_prefill_workspace_size", "kda_prefill_chunked", "kda_local_state_workspace_size",
           "kda_chunk_local_state", "kda_state_combine", "kda_decode_step", "kda_snapshot_count",
           "kda_get_device_status", "kda_status_string", "kda_version",
           "kda_prefill_uses_tensor_cores", "kda_prefill_chunked_noalloc",
           "kda_prefill_backward_workspace_size", "kda_prefill_backward",
           "kda_prefix_cache_create", "kda_prefix_cache_destroy", "kda_prefix_cache_lookup",
           "kda_prefix_cache_insert", "kda_prefix_cache_size", "kda_state_gather",
           "kda_state_scatter", "kda_prefill_split_segments")


def load(path: str = LIB_PATH):
    """Load libkda.so (raises if it was not built -- there is no fallback)."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(path):
            raise RuntimeError(
                f"libkda.so not found at {path}; build it with "
                "`python -m decode_kda_chunked_b200.build` (nvcc, sm_100a)")
        lib = ctypes.CDLL(path)
        P = ctypes.POINTER
        lib.kda_prefill_workspace_size.restype = ctypes.c_size_t
        lib.kda_prefill_workspace_size.argtypes = [P(PrefillArgs)]
        lib.kda_prefill_chunked.restype = ctypes.c_int
        lib.kda_prefill_chunked.argtypes = [P(PrefillArgs), _vp, ctypes.c_size_t, _vp]
        lib.kda_prefill_split_segments.restype = _i32
        lib.kda_prefill_split_segments.argtypes = [P(PrefillArgs)]
        lib.kda_local_state_workspace_size.restype = ctypes.c_size_t
        lib.kda_local_state_workspace_size.argtypes = [P(LocalStateArgs)]
        lib.kda_chunk_local_state.restype = ctypes.c_int
        lib.kda_chunk_local_state.argtypes = [P(LocalStateArgs), _vp, ctypes.c_size_t, _vp]
        lib.kda_state_combine.restype = ctypes.c_int
        lib.kda_state_combine.argtypes = [_vp, _vp, _vp, _i32, _i32, _i32, _i32, _vp, _vp, _vp]
        lib.kda_decode_step.restype = ctypes.c_int
        lib.kda_decode_step.argtypes = [P(DecodeArgs), _vp]
        lib.kda_snapshot_count.restype = _i32
        lib.kda_snapshot_count.argtypes = [_i32, _i32]
        lib.kda_get_device_status.restype = ctypes.c_int
        lib.kda_get_device_status.argtypes = [_vp]
        lib.kda_status_string.restype = ctypes.c_char_p
        lib.kda_status_string.argtypes = [ctypes.c_int]
        lib.kda_version.restype = _i32
        lib.kda_version.argtypes = []
        lib.kda_prefill_chunked_noalloc.restype = ctypes.c_int
        lib.kda_prefill_chunked_noalloc.argtypes = [P(PrefillArgs), _vp]
        lib.kda_prefill_backward_workspace_size.restype = ctypes.c_size_t
        lib.kda_prefill_backward_workspace_size.argtypes = [P(BackwardArgs)]
        lib.kda_prefill_backward.restype = ctypes.c_int
        lib.kda_prefill_backward.argtypes = [P(BackwardArgs), _vp, ctypes.c_size_t, _vp]
        lib.kda_prefill_uses_tensor_cores.restype = _i32
        lib.kda_prefill_uses_tensor_cores.argtypes = [_i32, _i32, ctypes.c_int]
        lib.kda_prefix_cache_create.restype = _vp
        lib.kda_prefix_cache_create.argtypes = [_i32, _i32]
        lib.kda_prefix_cache_destroy.restype = None
        lib.kda_prefix_cache_destroy.argtypes = [_vp]
        lib.kda_prefix_cache_lookup.restype = _i32
        lib.kda_prefix_cache_lookup.argtypes = [_vp, _vp, _i32, _i32, P(_i32)]
        lib.kda_prefix_cache_insert.restype = _i32
        lib.kda_prefix_cache_insert.argtypes = [_vp, _vp, _i32, _i32, _vp]
        lib.kda_prefix_cache_size.restype = _i32
        lib.kda_prefix_cache_size.argtypes = [_vp]
        lib.kda_state_gather.restype = ctypes.c_int
        lib.kda_state_gather.argtypes = [_vp, _i32, _vp, _i32, _i32, _i32, _i32, _vp, _vp]
        lib.kda_state_scatter.restype = ctypes.c_int
        lib.kda_state_scatter.argtypes = [_vp, _vp, _i32, _i32, _i32, _i32, _vp, _i32, _vp]
        _lib = lib
        return lib


# ----------------------------------------------------------------------------
# marshalling helpers
# ----------------------------------------------------------------------------

def _ptr(t) -> int | None:
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("tensors passed to libkda must be contiguous")
    return t.data_ptr()


def _dtype(t) -> int:
    if t.dtype == torch.bfloat16:
        return KDA_BF16
    if t.dtype == torch.float32:
        return KDA_F32
    raise TypeError(f"unsupported dtype {t.dtype}; use bfloat16 or float32")


def _stream(stream) -> int | None:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream or None
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream or None
    return int(stream) or None


def _check(fn: str, code: int):
    if code != 0:
        raise KdaError(fn, code)


def _host_i32(x):
    """A contiguous CPU int32 tensor (kept alive by the caller) or None."""
    if x is None:
        return None
    if isinstance(x, torch.Tensor):
        return x.detach().to("cpu", torch.int32).contiguous()
    return torch.tensor(list(x), dtype=torch.int32)


# ----------------------------------------------------------------------------
# entry points (same names as the C ABI)
# ----------------------------------------------------------------------------

def make_prefill_args(q, k, v, g, beta, cu_seqlens, o, initial_state=None, final_state=None,
                      snapshot_stride=0, cu_snapshots=None, snapshots=None,
                      cu_seqlens_host=None, g_logits=None):
    T, H, dk = k.shape
    dv = v.shape[2]
    a = PrefillArgs()
    a.n_req = cu_seqlens.numel() - 1
    a.total_tokens = T
    a.H, a.dk, a.dv = H, dk, dv
    a.in_dtype = _dtype(k)
    a.out_dtype = _dtype(o)
    a.q, a.k, a.v, a.g, a.beta = _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta)
    a.cu_seqlens = _ptr(cu_seqlens)
    a.cu_seqlens_host = _ptr(cu_seqlens_host)
    a.initial_state = _ptr(initial_state)
    a.o = _ptr(o)
    a.final_state = _ptr(final_state)
    a.snapshot_stride = int(snapshot_stride)
    a.cu_snapshots = _ptr(cu_snapshots)
    a.snapshots = _ptr(snapshots)
    a.g_logits = _ptr(g_logits)
    return a


def kda_prefill_workspace_size(args: PrefillArgs) -> int:
    return int(load().kda_prefill_workspace_size(ctypes.byref(args)))


def kda_prefill_chunked(q, k, v, g, beta, cu_seqlens, o, initial_state=None, final_state=None,
                        snapshot_stride=0, cu_snapshots=None, snapshots=None,
                        cu_seqlens_host=None, workspace=None, stream=None, g_logits=None):
    """Chunked prefill into caller-provided outputs (see include/kda.h).

    All tensors are CUDA tensors except ``cu_seqlens_host`` (optional CPU int32).
    ``workspace`` is a uint8 CUDA tensor of at least kda_prefill_workspace_size
    bytes; when None it is allocated here through torch (plumbing only)."""
    lib = load()
    host = _host_i32(cu_seqlens_host)
    a = make_prefill_args(q, k, v, g, beta, cu_seqlens, o, initial_state, final_state,
                          snapshot_stride, cu_snapshots, snapshots, host, g_logits)
    need = int(lib.kda_prefill_workspace_size(ctypes.byref(a)))
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=k.device)
    ws_ptr = _ptr(workspace) if workspace is not None else None
    ws_bytes = workspace.numel() if workspace is not None else 0
    _check("kda_prefill_chunked",
           lib.kda_prefill_chunked(ctypes.byref(a), ws_ptr, ws_bytes, _stream(stream)))
    return o


def kda_prefill_split_segments(q, k, v, g, beta, cu_seqlens, o, initial_state=None,
                               final_state=None, snapshot_stride=0, cu_snapshots=None,
                               snapshots=None, cu_seqlens_host=None, g_logits=None) -> int:
    """Segments kda_prefill_chunked would run for these arguments after its
    context-parallel split of few-chain calls; 0 when it would not split."""
    host = _host_i32(cu_seqlens_host)
    a = make_prefill_args(q, k, v, g, beta, cu_seqlens, o, initial_state, final_state,
                          snapshot_stride, cu_snapshots, snapshots, host, g_logits)
    return int(load().kda_prefill_split_segments(ctypes.byref(a)))


def make_backward_args(q, k, v, g, beta, cu_seqlens, cu_seqlens_host, d_q, d_k, d_v, d_g, d_beta,
                       initial_state=None, d_o=None, d_final=None, d_initial=None,
                       g_logits=None):
    T, H, dk = k.shape
    a = BackwardArgs()
    a.n_req = cu_seqlens.numel() - 1
    a.total_tokens = T
    a.H, a.dk, a.dv = H, dk, v.shape[2]
    a.in_dtype = _dtype(k)
    a.q, a.k, a.v, a.g, a.beta = _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta)
    a.cu_seqlens, a.cu_seqlens_host = _ptr(cu_seqlens), _ptr(cu_seqlens_host)
    a.initial_state, a.d_o, a.d_final = _ptr(initial_state), _ptr(d_o), _ptr(d_final)
    a.d_q, a.d_k, a.d_v, a.d_g, a.d_beta = _ptr(d_q), _ptr(d_k), _ptr(d_v), _ptr(d_g), _ptr(d_beta)
    a.d_initial = _ptr(d_initial)
    a.g_logits = _ptr(g_logits)
    return a


def kda_prefill_backward_workspace_size(args: BackwardArgs) -> int:
    return int(load().kda_prefill_backward_workspace_size(ctypes.byref(args)))


def kda_prefill_backward(q, k, v, g, beta, cu_seqlens, cu_seqlens_host, d_q, d_k, d_v, d_g,
                         d_beta, initial_state=None, d_o=None, d_final=None, d_initial=None,
                         workspace=None, stream=None, g_logits=None):
    """Gradients of sum(d_o * o) + sum(d_final * final_state) of the prefill into
    caller-provided fp32 outputs (see include/kda.h).  ``cu_seqlens_host`` (CPU
    int32) is required; ``workspace`` (uint8 CUDA tensor) is allocated through
    torch when None."""
    lib = load()
    host = _host_i32(cu_seqlens_host)
    a = make_backward_args(q, k, v, g, beta, cu_seqlens, host, d_q, d_k, d_v, d_g, d_beta,
                           initial_state, d_o, d_final, d_initial, g_logits)
    need = int(lib.kda_prefill_backward_workspace_size(ctypes.byref(a)))
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=k.device)
    ws_ptr = _ptr(workspace) if workspace is not None else None
    ws_bytes = workspace.numel() if workspace is not None else 0
    _check("kda_prefill_backward",
           lib.kda_prefill_backward(ctypes.byref(a), ws_ptr, ws_bytes, _stream(stream)))
    return d_q, d_k, d_v, d_g, d_beta, d_initial


def kda_chunk_local_state(k, v, g, beta, seg_cu, s_loc, m, seg_cu_host=None, stream=None,
                          g_logits=None):
    lib = load()
    T, H, dk = k.shape
    a = LocalStateArgs()
    a.n_seg = seg_cu.numel() - 1
    a.total_tokens = T
    a.H, a.dk, a.dv = H, dk, v.shape[2]
    a.in_dtype = _dtype(k)
    a.k, a.v, a.g, a.beta = _ptr(k), _ptr(v), _ptr(g), _ptr(beta)
    a.seg_cu = _ptr(seg_cu)
    host = _host_i32(seg_cu_host)
    a.seg_cu_host = _ptr(host)
    a.s_loc, a.m = _ptr(s_loc), _ptr(m)
    a.g_logits = _ptr(g_logits)
    _check("kda_chunk_local_state",
           lib.kda_chunk_local_state(ctypes.byref(a), None, 0, _stream(stream)))
    return s_loc, m


def kda_state_combine(s_loc, m, s_init, s_in, s_final, stream=None):
    lib = load()
    n_seg, H, dk, dv = s_loc.shape
    _check("kda_state_combine",
           lib.kda_state_combine(_ptr(s_loc), _ptr(m), _ptr(s_init), n_seg, H, dk, dv,
                                 _ptr(s_in), _ptr(s_final), _stream(stream)))
    return s_in, s_final


def make_decode_args(q, k, v, g, beta, state, o, slot=None):
    N, H, dk = k.shape
    a = DecodeArgs()
    a.n, a.H, a.dk, a.dv = N, H, dk, v.shape[2]
    a.in_dtype = _dtype(k)
    a.out_dtype = _dtype(o)
    a.q, a.k, a.v, a.g, a.beta = _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta)
    a.state = _ptr(state)
    a.n_slots = state.shape[0]
    a.slot = _ptr(slot)
    a.o = _ptr(o)
    return a


def kda_decode_step(q, k, v, g, beta, state, o, slot=None, stream=None):
    """One decode step; ``state`` [n_slots, H, dk, dv] fp32 is updated in place."""
    lib = load()
    a = make_decode_args(q, k, v, g, beta, state, o, slot)
    _check("kda_decode_step", lib.kda_decode_step(ctypes.byref(a), _stream(stream)))
    return o


def kda_snapshot_count(length: int, stride: int) -> int:
    return int(load().kda_snapshot_count(int(length), int(stride)))


def kda_get_device_status(stream=None) -> int:
    """Synchronise, then read and clear the device status word; returns the code."""
    return int(load().kda_get_device_status(_stream(stream)))


def kda_status_string(code: int) -> str:
    return load().kda_status_string(int(code)).decode()


def kda_version() -> int:
    return int(load().kda_version())


def kda_prefill_uses_tensor_cores(dk: int, dv: int, in_dtype: int = KDA_BF16) -> bool:
    return bool(load().kda_prefill_uses_tensor_cores(int(dk), int(dv), int(in_dtype)))


# ----------------------------------------------------------------------------
# prefix cache over state snapshots (host index + device pool copies)
# ----------------------------------------------------------------------------

def kda_prefix_cache_create(block_tokens: int, n_slots: int) -> int:
    h = load().kda_prefix_cache_create(int(block_tokens), int(n_slots))
    if not h:
        raise ValueError("kda_prefix_cache_create: block_tokens and n_slots must be > 0")
    return h


def kda_prefix_cache_destroy(handle: int) -> None:
    load().kda_prefix_cache_destroy(handle)


def _host_ids(tokens):
    t = torch.as_tensor(tokens, dtype=torch.int32).contiguous().cpu()
    return t, (t.data_ptr() if t.numel() else None)


def kda_prefix_cache_lookup(handle: int, tokens, max_tokens: int | None = None):
    """(cached prefix length in tokens, slot or -1) for host token ids."""
    t, p = _host_ids(tokens)
    n = t.numel()
    slot = _i32(-1)
    m = load().kda_prefix_cache_lookup(handle, p, n, n if max_tokens is None else int(max_tokens),
                                       ctypes.byref(slot))
    if m < 0:
        raise ValueError("kda_prefix_cache_lookup: invalid arguments")
    return int(m), int(slot.value)


def kda_prefix_cache_insert(handle: int, tokens, first_block: int = 0):
    """(leading blocks cached afterwards, slots to fill per block: list, -1 = none)."""
    t, p = _host_ids(tokens)
    n = t.numel()
    out = torch.full((max(n, 1),), -1, dtype=torch.int32)
    k = load().kda_prefix_cache_insert(handle, p, n, int(first_block), out.data_ptr())
    if k < 0:
        raise ValueError("kda_prefix_cache_insert: invalid arguments")
    return int(k), out


def kda_prefix_cache_size(handle: int) -> int:
    return int(load().kda_prefix_cache_size(handle))


def kda_state_gather(pool, slots, dst, stream=None):
    """dst[i] = pool[slots[i]] (zeros for slots[i] < 0); slots: CUDA int32."""
    n_slots, H, dk, dv = pool.shape
    _check("kda_state_gather", load().kda_state_gather(
        _ptr(pool), n_slots, _ptr(slots), slots.numel(), H, dk, dv, _ptr(dst), _stream(stream)))
    return dst


def kda_state_scatter(src, slots, pool, stream=None):
    """pool[slots[i]] = src[i] where slots[i] >= 0; slots: CUDA int32."""
    n_slots, H, dk, dv = pool.shape
    _check("kda_state_scatter", load().kda_state_scatter(
        _ptr(src), _ptr(slots), slots.numel(), H, dk, dv, _ptr(pool), n_slots, _stream(stream)))
    return pool
