"""The C ABI on the host (no GPU needed): the library loads, exports every
function include/kda.h declares, and rejects invalid arguments before
launching anything."""
import ctypes
import os
import re

import pytest
import torch

import decode_kda_chunked_b200 as kda
from decode_kda_chunked_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "kda.h")

FAKE = 1 << 20  # aligned, never dereferenced: validation fails before any launch


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"^\s*[A-Za-z_][\w\s\*]*?\b(kda_\w+)\s*\(", src, flags=re.M)
    return sorted(set(names))


def test_library_exports_every_declared_function():
    lib = ctypes.CDLL(_lib.LIB_PATH)
    names = declared_functions()
    assert len(names) >= 10, names
    for n in names:
        assert hasattr(lib, n), f"libkda.so does not export {n}"
    assert set(names) == set(_lib.EXPORTS)


def test_version_and_status_strings():
    assert kda.kda_version() == 100
    assert kda.kda_status_string(0) == "KDA_OK"
    assert kda.kda_status_string(6) == "KDA_ERR_WORKSPACE"
    assert kda.kda_status_string(99) == "KDA_ERR_UNKNOWN"


@pytest.mark.parametrize("L,stride,exp", [(0, 512, 0), (511, 512, 0), (512, 512, 1),
                                           (1100, 512, 2), (1024, 0, 0), (64, 64, 1)])
def test_snapshot_count(L, stride, exp):
    assert kda.kda_snapshot_count(L, stride) == exp


def _args(**over):
    a = _lib.PrefillArgs()
    a.n_req, a.total_tokens, a.H, a.dk, a.dv = 2, 128, 2, 128, 128
    a.in_dtype, a.out_dtype = 0, 1
    base = FAKE
    for i, n in enumerate(("q", "k", "v", "g", "beta", "cu_seqlens", "o")):
        setattr(a, n, base + (i << 24))
    for k_, v_ in over.items():
        setattr(a, k_, v_)
    return a


def _prefill(a, ws=None, ws_bytes=0):
    return _lib.load().kda_prefill_chunked(ctypes.byref(a), ws, ws_bytes, None)


@pytest.mark.parametrize("over,code", [
    ({"dk": 96, "dv": 96}, 2), ({"dk": 128, "dv": 64}, 2), ({"H": 0}, 1), ({"n_req": -1}, 1),
    ({"snapshot_stride": 100}, 1), ({"snapshot_stride": 512}, 1),  # no snapshot buffers
    ({"q": FAKE + 4}, 1), ({"o": None}, 1), ({"in_dtype": 7}, 1),
    ({"o": FAKE + (2 << 24)}, 1),  # o overlaps v
    ({"g_logits": FAKE + (9 << 24)}, 1),                          # both gate forms
    ({"g": None}, 1),                                             # no gate at all
    ({"g": None, "g_logits": FAKE + (9 << 24) + 2}, 1),           # logits misaligned
    ({"g": None, "g_logits": FAKE + (6 << 24) - 4096}, 1),        # o overlaps the logits
])
def test_prefill_rejects_invalid_args(over, code):
    assert _prefill(_args(**over)) == code


def test_gate_logits_are_an_accepted_gate():
    """With g NULL and bf16 logits given, the arguments are valid (the size query
    succeeds, as it does for fp32 g)."""
    lib = _lib.load()
    a = _args(g=None, g_logits=FAKE + (9 << 24))
    assert lib.kda_prefill_workspace_size(ctypes.byref(a)) > 0
    b = _bwd_args(g=None, g_logits=FAKE + (21 << 24))
    assert lib.kda_prefill_backward_workspace_size(ctypes.byref(b)) > 0
    assert lib.kda_prefill_backward_workspace_size(
        ctypes.byref(_bwd_args(g_logits=FAKE + (21 << 24)))) == 0   # both gate forms


def test_prefill_rejects_bad_host_seqlens():
    bad = (ctypes.c_int32 * 3)(0, 100, 90)      # decreasing
    assert _prefill(_args(cu_seqlens_host=ctypes.addressof(bad))) == 1
    short = (ctypes.c_int32 * 3)(0, 50, 100)    # does not end at total_tokens
    assert _prefill(_args(cu_seqlens_host=ctypes.addressof(short))) == 1


def test_prefill_workspace_contract():
    a = _args()
    lib = _lib.load()
    need = lib.kda_prefill_workspace_size(ctypes.byref(a))
    assert need > 0 and need % 256 == 0
    assert _prefill(a, None, 0) == 6                  # missing workspace
    assert _prefill(a, FAKE + 16, need) == 6          # not 256-byte aligned
    assert _prefill(a, FAKE, need - 1) == 6           # too small
    one = _args(n_req=1)
    assert lib.kda_prefill_workspace_size(ctypes.byref(one)) == 0
    assert lib.kda_prefill_workspace_size(ctypes.byref(_args(dk=96, dv=96))) == 0


def test_empty_batch_is_a_no_op():
    assert _prefill(_args(n_req=0, total_tokens=0)) == 0


def test_decode_rejects_invalid_args():
    lib = _lib.load()
    a = _lib.DecodeArgs()
    a.n, a.H, a.dk, a.dv, a.in_dtype, a.out_dtype = 4, 2, 128, 128, 0, 1
    for i, n in enumerate(("q", "k", "v", "g", "beta", "state", "o")):
        setattr(a, n, FAKE + (i << 24))
    a.n_slots = 3                                          # fewer slots than requests
    assert lib.kda_decode_step(ctypes.byref(a), None) == 1
    a.n_slots = 4
    a.dk = a.dv = 32
    assert lib.kda_decode_step(ctypes.byref(a), None) == 2
    a.dk = a.dv = 128
    a.o = a.state                                          # o overlaps the state pool
    assert lib.kda_decode_step(ctypes.byref(a), None) == 1
    a.n = 0
    assert lib.kda_decode_step(ctypes.byref(a), None) == 0


def test_combine_and_local_state_reject_invalid_args():
    lib = _lib.load()
    assert lib.kda_state_combine(FAKE, FAKE + (1 << 24), None, 0, 2, 128, 128, FAKE + (2 << 24),
                                 None, None) == 1
    assert lib.kda_state_combine(FAKE, FAKE + (1 << 24), None, 3, 2, 96, 96, FAKE + (2 << 24),
                                 None, None) == 2
    assert lib.kda_state_combine(FAKE, FAKE + (1 << 24), None, 3, 2, 128, 128, FAKE,
                                 None, None) == 1   # output overlaps input
    a = _lib.LocalStateArgs()
    a.n_seg, a.total_tokens, a.H, a.dk, a.dv, a.in_dtype = 2, 128, 2, 128, 128, 0
    for i, n in enumerate(("k", "v", "g", "beta", "seg_cu", "s_loc", "m")):
        setattr(a, n, FAKE + (i << 24))
    bad = (ctypes.c_int32 * 3)(0, 100, 64)
    a.seg_cu_host = ctypes.addressof(bad)
    assert lib.kda_chunk_local_state(ctypes.byref(a), None, 0, None) == 1
    a.seg_cu_host = None
    a.g_logits = FAKE + (9 << 24)                          # both gate forms
    assert lib.kda_chunk_local_state(ctypes.byref(a), None, 0, None) == 1
    a.g_logits = None
    a.m = a.s_loc
    assert lib.kda_chunk_local_state(ctypes.byref(a), None, 0, None) == 1


def test_binding_rejects_unsupported_dtype():
    x = torch.zeros(4, 1, 64, dtype=torch.float16)
    with pytest.raises(TypeError):
        _lib._dtype(x)


def test_missing_library_fails_loudly(tmp_path):
    saved = _lib._lib
    try:
        _lib._lib = None
        with pytest.raises(RuntimeError, match="libkda.so not found"):
            _lib.load(str(tmp_path / "nope.so"))
    finally:
        _lib._lib = saved


_CU_BWD = (ctypes.c_int32 * 3)(0, 64, 128)


def _bwd_args(**over):
    a = _lib.BackwardArgs()
    a.n_req, a.total_tokens, a.H, a.dk, a.dv, a.in_dtype = 2, 128, 2, 128, 128, 0
    names = ("q", "k", "v", "g", "beta", "cu_seqlens", "d_o", "d_q", "d_k", "d_v", "d_g",
             "d_beta")
    for i, n in enumerate(names):
        setattr(a, n, FAKE + (i << 24))
    a.cu_seqlens_host = ctypes.addressof(_CU_BWD)
    for k_, v_ in over.items():
        setattr(a, k_, v_)
    return a


def _backward(a, ws=None, ws_bytes=0):
    return _lib.load().kda_prefill_backward(ctypes.byref(a), ws, ws_bytes, None)


@pytest.mark.parametrize("over,code", [
    ({"cu_seqlens_host": None}, 1),                # the host offsets are required
    ({"dk": 96, "dv": 96}, 2), ({"H": 0}, 1), ({"in_dtype": 7}, 1),
    ({"d_q": None}, 1), ({"d_k": FAKE + 4}, 1),
    ({"d_v": FAKE + (2 << 24)}, 1),                # d_v overlaps v
    ({"d_g": FAKE + (7 << 24)}, 1),                # d_g overlaps d_q
    ({"total_tokens": 100}, 1),                    # host offsets end elsewhere
    ({"g": None}, 1),                              # no gate at all
    ({"g": None, "g_logits": FAKE + (21 << 24) + 8}, 1),   # logits misaligned
    ({"g": None, "g_logits": FAKE + (10 << 24)}, 1),       # d_g overlaps the logits
])
def test_backward_rejects_invalid_args(over, code):
    assert _backward(_bwd_args(**over)) == code


def test_backward_workspace_contract():
    lib = _lib.load()
    a = _bwd_args()
    need = lib.kda_prefill_backward_workspace_size(ctypes.byref(a))
    assert need > 0 and need % 256 == 0
    assert _backward(a, None, 0) == 6
    assert _backward(a, FAKE + (20 << 24) + 16, need) == 6
    assert _backward(a, FAKE + (20 << 24), need - 1) == 6
    assert _backward(a, FAKE + (7 << 24), need) == 1      # workspace overlaps d_q
    # one more chunk (65 tokens in the second request) needs more workspace
    cu = (ctypes.c_int32 * 3)(0, 64, 129)
    b = _bwd_args(total_tokens=129, cu_seqlens_host=ctypes.addressof(cu))
    assert lib.kda_prefill_backward_workspace_size(ctypes.byref(b)) > need
    assert lib.kda_prefill_backward_workspace_size(ctypes.byref(_bwd_args(dk=96, dv=96))) == 0
    assert _backward(_bwd_args(n_req=0, total_tokens=0)) == 0
