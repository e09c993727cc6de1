"""GPU parity of kda_prefill_chunked against the fp64 oracle (through the C ABI).

Small cases compare every output element; the full-size workloads compare
sampled (request, head) chains that the oracle recomputes one by one.  The
launch configuration is the one bench.py times (same entry point, same
dtypes, fp32 outputs).
"""
import os
import random

import numpy as np
import pytest
import torch

import decode_kda_chunked_b200 as kda
from decode_kda_chunked_b200 import inputs as I
from kda_testing import TOL_BF16, TOL_F32, oracle_chains, rel_err

pytestmark = pytest.mark.gpu
DEV = "cuda"


def run_prefill(inp, stride=0, out_dtype=torch.float32):
    x = inp.to(DEV)
    out = kda.prefill(x.q, x.k, x.v, x.g, x.beta, x.cu_seqlens, initial_state=x.initial_state,
                      snapshot_stride=stride, out_dtype=out_dtype,
                      cu_seqlens_host=[0] + list(np.cumsum(x.lengths)))
    assert kda.kda_get_device_status() == 0
    return out


def check_all_chains(inp, out, stride, tol, pairs=None):
    cu = [int(c) for c in inp.cu_seqlens.cpu().tolist()]
    H = inp.k.shape[1]
    pairs = pairs or [(r, h) for r in range(inp.n_req) for h in range(H)]
    ref = oracle_chains(inp, pairs, stride)
    cs = out["cu_snapshots"].cpu().tolist() if out["cu_snapshots"] is not None else None
    worst = {"o": 0.0, "final": 0.0, "snap": 0.0}
    o_gpu = out["o"].float().cpu()
    for (r, h), rr in ref.items():
        lo, hi = cu[r], cu[r + 1]
        if hi > lo:
            worst["o"] = max(worst["o"], rel_err(o_gpu[lo:hi, h], rr["o"]))
        worst["final"] = max(worst["final"], rel_err(out["final_state"][r, h], rr["final_state"]))
        if stride:
            sn = out["snapshots"][cs[r]:cs[r + 1], h]
            assert sn.shape[0] == rr["snapshots"].shape[0]
            if sn.shape[0]:
                worst["snap"] = max(worst["snap"], rel_err(sn, rr["snapshots"]))
    for k_, v_ in worst.items():
        assert v_ <= tol, f"{k_} rel err {v_:.3e} > {tol:.1e}"
    return worst


# --------------------------------------------------------------------------
# small cases: every element
# --------------------------------------------------------------------------

def test_oracle_scale_fp32():
    """B=1, H=2, T=256, d=64, fp32 inputs, zero initial state: tolerance 1e-5."""
    inp = I.oracle_scale()
    out = run_prefill(inp)
    check_all_chains(inp, out, 0, TOL_F32)


RAGGED = [1, 63, 64, 65, 127, 128, 200, 0, 513]


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32], ids=["bf16", "fp32"])
def test_ragged_varlen(d, dtype):
    inp = I.make_prefill_inputs(RAGGED, H=3, dk=d, dv=d, dtype=dtype, seed=7, s0_std=0.1)
    out = run_prefill(inp, stride=64)
    check_all_chains(inp, out, 64, TOL_F32 if dtype == torch.float32 else TOL_BF16)


RAGGED_32 = [31, 32, 33, 95, 96, 97, 160, 1, 0, 64]


def test_ragged_around_32_token_chunks():
    """The tensor-core kernel works in 32-token chunks: lengths one short of, at and
    one past chunk ends, with snapshots every 64 tokens (every second chunk end)."""
    inp = I.make_prefill_inputs(RAGGED_32, H=2, dk=128, dv=128, seed=8, s0_std=0.1)
    out = run_prefill(inp, stride=64)
    check_all_chains(inp, out, 64, TOL_BF16)


def test_weak_decay_long_memory():
    """Weak gates keep long-range state alive, so errors carried across many
    chunks show up (the standard -5 sigmoid gates forget within a few tokens)."""
    inp = I.make_prefill_inputs([1000, 777], H=2, dk=128, dv=128, dtype=torch.bfloat16, seed=3,
                                s0_std=0.1, gate_scale=0.02)
    out = run_prefill(inp, stride=128)
    check_all_chains(inp, out, 128, TOL_BF16)


def test_tensor_core_and_simt_kernels_agree(monkeypatch):
    """bf16 inputs with d=128 run on the tcgen05 kernel; KDA_FORCE_SIMT=1 runs the
    fp32 SIMT kernel on the same inputs.  Both must agree within tolerance."""
    assert kda.kda_prefill_uses_tensor_cores(128, 128)
    inp = I.make_prefill_inputs([333, 64, 700], H=3, dk=128, dv=128, seed=29, s0_std=0.1,
                                gate_scale=0.5)
    tc = run_prefill(inp, stride=64)
    monkeypatch.setenv("KDA_FORCE_SIMT", "1")
    assert not kda.kda_prefill_uses_tensor_cores(128, 128)
    simt = run_prefill(inp, stride=64)
    for n in ("o", "final_state", "snapshots"):
        assert rel_err(tc[n], simt[n]) <= TOL_BF16, n


def test_bf16_output():
    inp = I.make_prefill_inputs([300, 64], H=2, dk=128, dv=128, seed=5, s0_std=0.1)
    out = run_prefill(inp, out_dtype=torch.bfloat16)
    ref = oracle_chains(inp, [(0, 0), (1, 1)])
    # bf16 storage alone costs up to 2^-9 relative per element
    assert rel_err(out["o"][:300, 0].float(), ref[(0, 0)]["o"]) <= 2 * TOL_BF16
    assert rel_err(out["final_state"][1, 1], ref[(1, 1)]["final_state"]) <= TOL_BF16


def test_empty_requests_keep_initial_state():
    inp = I.make_prefill_inputs([0, 5, 0], H=2, dk=64, dv=64, dtype=torch.float32, seed=9,
                                s0_std=1.0)
    out = run_prefill(inp)
    s0 = inp.initial_state.to(DEV)
    assert torch.equal(out["final_state"][0], s0[0])
    assert torch.equal(out["final_state"][2], s0[2])


def test_final_state_in_place():
    inp = I.make_prefill_inputs([130, 70], H=2, dk=128, dv=128, seed=11, s0_std=0.1).to(DEV)
    ref = kda.prefill(inp.q, inp.k, inp.v, inp.g, inp.beta, inp.cu_seqlens,
                      initial_state=inp.initial_state)
    state = inp.initial_state.clone()
    o = torch.empty_like(ref["o"])
    kda.kda_prefill_chunked(inp.q, inp.k, inp.v, inp.g, inp.beta, inp.cu_seqlens, o,
                            initial_state=state, final_state=state)
    torch.cuda.synchronize()
    assert torch.equal(state, ref["final_state"])
    assert torch.equal(o, ref["o"])


def test_snapshot_tagging_exact():
    """beta=1, alpha=1, one-hot keys: each write replaces one state row, so a
    snapshot names exactly which positions it has seen.  Values are small
    integers (exact in bf16), so the chunked kernel must reproduce them bit for bit."""
    d, stride = 128, 64
    lengths = [130, 64, 300, 63]
    T = sum(lengths)
    cu = np.concatenate([[0], np.cumsum(lengths)])
    k = torch.zeros(T, 1, d)
    v = torch.zeros(T, 1, d)
    for r, L in enumerate(lengths):
        for p in range(L):
            k[cu[r] + p, 0, p % d] = 1.0
            v[cu[r] + p, 0, 0] = (p % 128) + 1
            v[cu[r] + p, 0, 1] = (p // 128) + 1
            v[cu[r] + p, 0, 2] = r + 1
    inp = I.PrefillInputs(k.clone().bfloat16(), k.bfloat16(), v.bfloat16(), torch.zeros(T, 1, d),
                          torch.ones(T, 1), torch.tensor(cu, dtype=torch.int32), lengths, None)
    out = run_prefill(inp, stride=stride)
    snaps = out["snapshots"].cpu()
    idx = 0
    for r, L in enumerate(lengths):
        for j in range(1, L // stride + 1):
            n = j * stride
            exp_ = torch.zeros(d, d)
            for p in range(n):
                exp_[p % d, 0] = (p % 128) + 1
                exp_[p % d, 1] = (p // 128) + 1
                exp_[p % d, 2] = r + 1
            assert torch.equal(snaps[idx, 0], exp_), (r, j)
            idx += 1
    assert idx == snaps.shape[0]


def test_varlen_isolation_bitexact():
    lengths = [200, 64, 1, 333]
    inp = I.make_prefill_inputs(lengths, H=2, dk=128, dv=128, seed=13, s0_std=0.1)
    packed = run_prefill(inp, stride=64)
    cu = [0] + list(np.cumsum(lengths))
    for r in (0, 3):
        lo, hi = cu[r], cu[r + 1]
        alone_in = I.PrefillInputs(inp.q[lo:hi], inp.k[lo:hi], inp.v[lo:hi], inp.g[lo:hi],
                                   inp.beta[lo:hi], torch.tensor([0, hi - lo], dtype=torch.int32),
                                   [hi - lo], inp.initial_state[r:r + 1])
        alone = run_prefill(alone_in, stride=64)
        assert torch.equal(alone["o"], packed["o"][lo:hi])
        assert torch.equal(alone["final_state"][0], packed["final_state"][r])
        cs = packed["cu_snapshots"].tolist()
        assert torch.equal(alone["snapshots"], packed["snapshots"][cs[r]:cs[r + 1]])
    # scrambling the other requests changes nothing for request 0
    scr = I.make_prefill_inputs(lengths, H=2, dk=128, dv=128, seed=99, s0_std=0.1)
    lo, hi = cu[0], cu[1]
    for n in ("q", "k", "v", "g", "beta"):
        getattr(scr, n)[lo:hi] = getattr(inp, n)[lo:hi]
    scr.initial_state[0] = inp.initial_state[0]
    other = run_prefill(scr, stride=64)
    assert torch.equal(other["o"][lo:hi], packed["o"][lo:hi])


def test_deterministic():
    inp = I.make_prefill_inputs([700, 129], H=4, dk=128, dv=128, seed=17, s0_std=0.1)
    a = run_prefill(inp, stride=128)
    b = run_prefill(inp, stride=128)
    for n in ("o", "final_state", "snapshots"):
        assert torch.equal(a[n], b[n])


def test_resume_from_snapshot_bitexact():
    """prefill(0..L) == prefill(512j..L) started from snapshot j."""
    L, stride = 1500, 512
    inp = I.make_prefill_inputs([L], H=2, dk=128, dv=128, seed=19, s0_std=0.1, gate_scale=0.05)
    full = run_prefill(inp, stride=stride)
    for j in (1, 2):
        cut = j * stride
        part_in = I.PrefillInputs(inp.q[cut:], inp.k[cut:], inp.v[cut:], inp.g[cut:],
                                  inp.beta[cut:], torch.tensor([0, L - cut], dtype=torch.int32),
                                  [L - cut], full["snapshots"][j - 1:j].cpu())
        part = run_prefill(part_in)
        assert torch.equal(part["o"], full["o"][cut:])
        assert torch.equal(part["final_state"], full["final_state"])


def test_validation_mode_flags_gate_range():
    inp = I.make_prefill_inputs([70], H=1, dk=64, dv=64, dtype=torch.float32, seed=21)
    inp.g[3, 0, 5] = -6.0  # below the lower bound
    os.environ["KDA_VALIDATE"] = "1"
    try:
        x = inp.to(DEV)
        kda.prefill(x.q, x.k, x.v, x.g, x.beta, x.cu_seqlens)
        assert kda.kda_get_device_status() == 4  # KDA_ERR_GATE_RANGE
        assert kda.kda_get_device_status() == 0  # cleared by the read
    finally:
        del os.environ["KDA_VALIDATE"]


def test_invalid_args_launch_nothing():
    x = I.make_prefill_inputs([64], H=1, dk=128, dv=128, seed=1).to(DEV)
    o = torch.full((64, 1, 128), 7.0, device=DEV)
    with pytest.raises(kda.KdaError) as ei:
        kda.kda_prefill_chunked(x.q, x.k, x.v, x.g, x.beta, x.cu_seqlens, o, snapshot_stride=100)
    assert ei.value.code == 1
    torch.cuda.synchronize()
    assert torch.all(o == 7.0)


# --------------------------------------------------------------------------
# full-size workloads: sampled chains
# --------------------------------------------------------------------------

@pytest.mark.slow
def test_single_sequence_full_size():
    """B=1, H=32, T=8192, d=128, bf16, N(0, 0.1) initial state; 6 heads sampled."""
    inp = I.single_seq(device=DEV)
    out = run_prefill(inp.to(DEV), stride=512)
    check_all_chains(inp, out, 512, TOL_BF16, pairs=[(0, h) for h in (0, 5, 11, 17, 26, 31)])


@pytest.mark.slow
def test_varlen_full_size():
    """64 requests, log-uniform lengths on [128, 4096], H=32, d=128: 24 chains sampled,
    including the longest and the shortest request."""
    inp = I.varlen(device=DEV)
    out = run_prefill(inp, stride=512)
    lens = inp.lengths
    rng = random.Random(0)
    reqs = {int(np.argmax(lens)), int(np.argmin(lens))} | set(rng.sample(range(len(lens)), 10))
    pairs = [(r, rng.randrange(32)) for r in sorted(reqs)] + [(int(np.argmax(lens)), 31)]
    pairs = sorted(set(pairs))[:24]
    check_all_chains(inp, out, 512, TOL_BF16, pairs=pairs)
