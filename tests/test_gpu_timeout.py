"""The timeout path of the tensor-core prefill, made to run on purpose.

Every wait inside the kernel is bounded.  A wait that runs out makes the CTA give
up: it lets the loads and products it already issued land, releases its tensor
memory, returns, and leaves KDA_ERR_TIMEOUT in the device status word.  The test
shortens the limit to 1 ns through KDA_TEST_WAIT_LIMIT_NS, which exists only for
this purpose, so the control warp's first wait for the workers' operands (and
the workers' first waits) cannot be met in time while the chunk's first tile
loads are still in flight.  Nothing faults or hangs: the wait gives up by
design.  Then a normal call on the same context must give the oracle's result.
"""
import numpy as np
import pytest
import torch

import decode_kda_chunked_b200 as kda
from decode_kda_chunked_b200 import inputs as I
from kda_testing import TOL_BF16, oracle_chains, rel_err

pytestmark = pytest.mark.gpu
DEV = "cuda"
KDA_ERR_TIMEOUT = 5


def _run(x):
    return kda.prefill(x.q, x.k, x.v, x.g, x.beta, x.cu_seqlens, initial_state=x.initial_state,
                       snapshot_stride=64, cu_seqlens_host=[0] + list(np.cumsum(x.lengths)))


def test_wait_that_runs_out_reports_timeout_and_the_next_call_is_exact(monkeypatch):
    inp = I.make_prefill_inputs([300, 64, 129], H=2, dk=128, dv=128, seed=41, s0_std=0.1)
    x = inp.to(DEV)
    assert kda.kda_prefill_uses_tensor_cores(128, 128)
    assert kda.kda_get_device_status() == 0
    monkeypatch.setenv("KDA_TEST_WAIT_LIMIT_NS", "1")
    _run(x)
    torch.cuda.synchronize()  # the kernel returned
    assert kda.kda_get_device_status() == KDA_ERR_TIMEOUT
    monkeypatch.delenv("KDA_TEST_WAIT_LIMIT_NS")
    assert kda.kda_get_device_status() == 0  # reading the status cleared it
    out = _run(x)
    assert kda.kda_get_device_status() == 0
    pairs = [(r, h) for r in range(inp.n_req) for h in range(2)]
    ref = oracle_chains(inp, pairs, 64)
    cu = [0] + list(np.cumsum(inp.lengths))
    for (r, h), rr in ref.items():
        assert rel_err(out["o"][cu[r]:cu[r + 1], h], rr["o"]) <= TOL_BF16
        assert rel_err(out["final_state"][r, h], rr["final_state"]) <= TOL_BF16
