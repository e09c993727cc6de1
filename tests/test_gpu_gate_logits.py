"""GPU parity of the fused gate activation: bf16 gate logits x are given instead of
fp32 log alpha, and the kernels compute log(alpha) = -5 sigmoid(x) as they load the
tiles.  Every path (tensor-core prefill, SIMT prefill, context-parallel local
state, backward) is checked against the fp64 oracle on the same logits, with the
tolerance metric of the other parity tests (max |x - ref| / max |ref| per tensor:
2e-3 for bf16 inputs, 1e-5 for fp32 inputs)."""
import numpy as np
import pytest
import torch

import decode_kda_chunked_b200 as kda
import oracle
from decode_kda_chunked_b200 import inputs as I
from kda_testing import TOL_BF16, TOL_F32, rel_err

pytestmark = pytest.mark.gpu
DEV = "cuda"
PATHS = [(128, torch.bfloat16, TOL_BF16), (64, torch.float32, TOL_F32),
         (64, torch.bfloat16, TOL_BF16), (128, torch.float32, TOL_F32)]
PATH_IDS = ["bf16-d128-tc", "fp32-d64", "bf16-d64", "fp32-d128"]


def _status_ok():
    st = kda.kda_get_device_status()
    assert st == 0, kda.kda_status_string(st)


def _prefill_pair(inp, stride=64):
    x = inp.to(DEV)
    out = kda.prefill(x.q, x.k, x.v, None, x.beta, x.cu_seqlens, initial_state=x.initial_state,
                      snapshot_stride=stride, cu_seqlens_host=inp.cu_seqlens,
                      g_logits=x.g_logits)
    torch.cuda.synchronize()
    _status_ok()
    ref = oracle.prefill(inp.q, inp.k, inp.v, None, inp.beta, inp.cu_seqlens.numpy(),
                         inp.initial_state, snapshot_stride=stride, g_logits=inp.g_logits)
    return out, ref


@pytest.mark.parametrize("d,dtype,tol", PATHS, ids=PATH_IDS)
def test_prefill_with_gate_logits_matches_oracle(d, dtype, tol):
    # ragged tails, a one-token request, several chunks and one snapshot-crossing request
    inp = I.make_prefill_inputs([100, 64, 1, 190, 513], H=2, dk=d, dv=d, dtype=dtype, seed=61,
                                s0_std=0.1, gate_logits=True)
    assert inp.g is None and inp.g_logits.dtype == torch.bfloat16
    out, ref = _prefill_pair(inp)
    for name in ("o", "final_state", "snapshots"):
        assert rel_err(out[name], ref[name]) <= tol, (name, rel_err(out[name], ref[name]))


def test_extreme_gate_logits():
    """Logits far out on both sides saturate the gate at 0 (alpha = 1) and -5
    (alpha = exp(-5)); the kernels reach the same limits as the oracle."""
    inp = I.make_prefill_inputs([300, 77], H=2, dk=128, dv=128, seed=62, s0_std=0.1,
                                gate_logits=True)
    gen = torch.Generator().manual_seed(63)
    choice = torch.tensor([-120.0, -30.0, -2.0, 0.0, 2.0, 30.0, 120.0])
    idx = torch.randint(0, len(choice), inp.g_logits.shape, generator=gen)
    inp.g_logits = choice[idx].to(torch.bfloat16).contiguous()
    out, ref = _prefill_pair(inp)
    for name in ("o", "final_state", "snapshots"):
        assert rel_err(out[name], ref[name]) <= TOL_BF16, (name, rel_err(out[name], ref[name]))


def test_gate_logits_on_the_headline_shape_sampled():
    """The varlen workload (64 requests, H=32, d=128) with bf16 logits: every
    final state of a sample of (request, head) chains against the oracle."""
    inp = I.varlen(gate_logits=True)
    x = inp.to(DEV)
    out = kda.prefill(x.q, x.k, x.v, None, x.beta, x.cu_seqlens,
                      cu_seqlens_host=inp.cu_seqlens, g_logits=x.g_logits)
    torch.cuda.synchronize()
    _status_ok()
    cu = inp.cu_seqlens.tolist()
    rng = np.random.default_rng(64)
    for r, h in zip(rng.choice(64, 6, replace=False), rng.choice(32, 6)):
        lo, hi = cu[r], cu[r + 1]
        sl = lambda t: t[lo:hi, h:h + 1]
        ref = oracle.prefill(sl(inp.q), sl(inp.k), sl(inp.v), None, inp.beta[lo:hi, h:h + 1],
                             np.array([0, hi - lo]), None, g_logits=sl(inp.g_logits))
        assert rel_err(out["final_state"][r, h], ref["final_state"][0, 0]) <= TOL_BF16, (r, h)
        assert rel_err(out["o"][lo:hi, h], ref["o"][:, 0]) <= TOL_BF16, (r, h)


@pytest.mark.parametrize("d,dtype,tol", PATHS[:2], ids=PATH_IDS[:2])
def test_context_parallel_with_gate_logits(d, dtype, tol):
    """Local states and transitions with logits, combined, equal the unsplit oracle."""
    inp = I.make_prefill_inputs([1024], H=2, dk=d, dv=d, dtype=dtype, seed=65, s0_std=0.1,
                                gate_logits=True)
    x = inp.to(DEV)
    out = kda.long_context_prefill(x.q, x.k, x.v, None, x.beta, seg_len=256,
                                   snapshot_stride=256, initial_state=x.initial_state[0],
                                   g_logits=x.g_logits)
    torch.cuda.synchronize()
    _status_ok()
    ref = oracle.prefill(inp.q, inp.k, inp.v, None, inp.beta, inp.cu_seqlens.numpy(),
                         inp.initial_state, snapshot_stride=256, g_logits=inp.g_logits)
    assert rel_err(out["o"], ref["o"]) <= tol
    assert rel_err(out["final_state"], ref["final_state"][0]) <= tol
    assert rel_err(out["snapshots"], ref["snapshots"]) <= tol


@pytest.mark.parametrize("d,dtype,tol", PATHS, ids=PATH_IDS)
def test_backward_with_gate_logits_matches_oracle(d, dtype, tol):
    """dg is the gradient of the logits: the oracle's dL/dg times the gate's slope."""
    inp = I.make_prefill_inputs([100, 64, 1, 190], H=2, dk=d, dv=d, dtype=dtype, seed=66,
                                s0_std=0.1, gate_logits=True)
    gen = torch.Generator().manual_seed(67)
    T, n = inp.total_tokens, inp.n_req
    d_o = torch.randn((T, 2, d), generator=gen)
    d_fin = torch.randn((n, 2, d, d), generator=gen)
    x = inp.to(DEV)
    got = kda.prefill_backward(x.q, x.k, x.v, None, x.beta, x.cu_seqlens, d_o=d_o.to(DEV),
                               d_final=d_fin.to(DEV), initial_state=x.initial_state,
                               cu_seqlens_host=inp.cu_seqlens, g_logits=x.g_logits)
    torch.cuda.synchronize()
    _status_ok()
    ref = oracle.prefill_backward(inp.q, inp.k, inp.v, None, inp.beta, inp.cu_seqlens.numpy(),
                                  inp.initial_state, d_o, d_fin, g_logits=inp.g_logits)
    for name in ("dq", "dk", "dv", "dg", "dbeta", "d_initial"):
        assert rel_err(got[name], ref[name]) <= tol, (name, rel_err(got[name], ref[name]))
