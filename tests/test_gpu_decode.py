"""GPU parity of kda_decode_step against the fp64 oracle (through the C ABI)."""
import numpy as np
import pytest
import torch

import decode_kda_chunked_b200 as kda
import oracle
from decode_kda_chunked_b200 import inputs as I
from kda_testing import TOL_BF16, TOL_F32, rel_err

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _step_inputs(x, t):
    return [getattr(x, n)[t].to(DEV).contiguous() for n in ("q", "k", "v", "g", "beta")]


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32], ids=["bf16", "fp32"])
def test_decode_small_every_element(d, dtype):
    steps, N, H = 20, 5, 3
    x = I.decode(steps, N=N, H=H, d=d, dtype=dtype, seed=3)
    state = x.state.to(DEV).clone()
    ref_state = np.ascontiguousarray(x.state.double().numpy())
    tol = TOL_F32 if dtype == torch.float32 else TOL_BF16
    for t in range(steps):
        q, k, v, g, b = _step_inputs(x, t)
        o = kda.decode_step(q, k, v, g, b, state)
        ref_o = oracle.decode_step(x.q[t], x.k[t], x.v[t], x.g[t], x.beta[t], ref_state)
        assert rel_err(o, ref_o) <= tol
    assert rel_err(state, ref_state) <= tol
    assert kda.kda_get_device_status() == 0


def test_decode_slots_touch_only_their_states():
    N, H, d, pool = 4, 2, 128, 9
    x = I.decode(1, N=pool, H=H, d=d, seed=5)
    slot = torch.tensor([7, 0, 3, 5], dtype=torch.int32)
    state = x.state.to(DEV).clone()
    before = state.clone()
    q, k, v, g, b = [t[:N] for t in _step_inputs(x, 0)]
    o = kda.decode_step(q, k, v, g, b, state, slot=slot.to(DEV))
    ref_state = np.ascontiguousarray(x.state.double().numpy())
    ref_o = oracle.decode_step(x.q[0, :N], x.k[0, :N], x.v[0, :N], x.g[0, :N], x.beta[0, :N],
                               ref_state, slot=slot.numpy())
    for s in range(pool):
        if s not in slot.tolist():
            assert torch.equal(state[s], before[s])
    assert rel_err(state, ref_state) <= TOL_BF16
    assert rel_err(o, ref_o) <= TOL_BF16


def test_decode_matches_prefill():
    """L decode steps of N requests equal a prefill of the N packed requests."""
    L, N, H, d = 70, 3, 2, 128
    x = I.decode(L, N=N, H=H, d=d, seed=8)
    state = x.state.to(DEV).clone()
    outs = []
    for t in range(L):
        q, k, v, g, b = _step_inputs(x, t)
        outs.append(kda.decode_step(q, k, v, g, b, state))
    dec_o = torch.stack(outs, 0)  # [L, N, H, d]
    perm = lambda t: t.transpose(0, 1).reshape(L * N, *t.shape[2:]).contiguous().to(DEV)
    cu = torch.arange(0, (N + 1) * L, L, dtype=torch.int32, device=DEV)
    pf = kda.prefill(perm(x.q), perm(x.k), perm(x.v), perm(x.g), perm(x.beta), cu,
                     initial_state=x.state.to(DEV))
    assert rel_err(dec_o.transpose(0, 1).reshape(L * N, H, d), pf["o"]) <= TOL_BF16
    assert rel_err(state, pf["final_state"]) <= TOL_BF16


@pytest.mark.slow
def test_decode_full_size_1000_steps():
    """256 requests x 32 heads x 128x128 fp32 states, 1,000 steps; 16 states tracked
    by the oracle at every step, and the whole state pool checked against the
    oracle's tracked states at the end."""
    steps, N, H, d = 1000, 256, 32, 128
    x = I.decode(steps, N=N, H=H, d=d, device=DEV, seed=0)
    state = x.state.clone()
    rng = np.random.default_rng(0)
    picks = sorted({(int(rng.integers(N)), int(rng.integers(H))) for _ in range(16)})
    nn = np.array([p[0] for p in picks])
    hh = np.array([p[1] for p in picks])
    ref_state = np.ascontiguousarray(x.state[nn, hh].double().cpu().numpy()[:, None])
    cpu = {n: getattr(x, n)[:, nn, hh].cpu() for n in ("q", "k", "v", "g", "beta")}
    worst = 0.0
    for t in range(steps):
        q, k, v, g, b = (getattr(x, n)[t] for n in ("q", "k", "v", "g", "beta"))
        o = kda.decode_step(q, k, v, g, b, state)
        ref_o = oracle.decode_step(cpu["q"][t][:, None], cpu["k"][t][:, None],
                                   cpu["v"][t][:, None], cpu["g"][t][:, None],
                                   cpu["beta"][t][:, None], ref_state)
        if t % 50 == 0 or t == steps - 1:
            worst = max(worst, rel_err(o[nn, hh], ref_o[:, 0]))
    assert worst <= TOL_BF16
    assert rel_err(state[nn, hh], ref_state[:, 0]) <= TOL_BF16
    assert kda.kda_get_device_status() == 0
