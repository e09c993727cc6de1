"""GPU parity of the context-parallel path: kda_chunk_local_state,
kda_state_combine and the segment-wise prefill, against the fp64 oracle and
against the unsplit GPU run."""
import numpy as np
import pytest
import torch

import decode_kda_chunked_b200 as kda
import oracle
from decode_kda_chunked_b200 import inputs as I
from kda_testing import TOL_BF16, TOL_F32, oracle_chains, rel_err

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.mark.parametrize("d,dtype,tol", [(128, torch.bfloat16, TOL_BF16),
                                         (64, torch.float32, TOL_F32)])
def test_local_state_and_transition(d, dtype, tol):
    seg = [0, 192, 200, 512, 900]           # ragged segments, one of 8 tokens
    T, H = seg[-1], 2
    inp = I.make_prefill_inputs([T], H=H, dk=d, dv=d, dtype=dtype, seed=31, gate_scale=0.05)
    x = inp.to(DEV)
    n = len(seg) - 1
    s_loc = torch.empty(n, H, d, d, device=DEV)
    m = torch.empty(n, H, d, d, device=DEV)
    kda.kda_chunk_local_state(x.k, x.v, x.g, x.beta, torch.tensor(seg, dtype=torch.int32,
                                                                 device=DEV), s_loc, m,
                              seg_cu_host=seg)
    ref_s, ref_m = oracle.chunk_local_state(inp.k, inp.v, inp.g, inp.beta, np.array(seg))
    assert rel_err(s_loc, ref_s) <= tol
    assert rel_err(m, ref_m) <= tol
    assert kda.kda_get_device_status() == 0


def test_combine_against_oracle():
    n, H, d = 5, 3, 128
    g = torch.Generator().manual_seed(0)
    s_loc = torch.randn(n, H, d, d, generator=g)
    m = torch.randn(n, H, d, d, generator=g) / d ** 0.5
    s0 = torch.randn(H, d, d, generator=g)
    s_in = torch.empty(n, H, d, d, device=DEV)
    s_fin = torch.empty(H, d, d, device=DEV)
    kda.kda_state_combine(s_loc.to(DEV), m.to(DEV), s0.to(DEV), s_in, s_fin)
    ref_in, ref_fin = oracle.state_combine(s_loc, m, s0)
    assert rel_err(s_in, ref_in) <= TOL_F32
    assert rel_err(s_fin, ref_fin) <= TOL_F32


@pytest.mark.parametrize("gate_scale", [5.0, 0.05])
def test_split_and_combine_equals_unsplit(gate_scale):
    T, H, d, seg_len, stride = 4096, 2, 128, 1024, 512
    inp = I.make_prefill_inputs([T], H=H, dk=d, dv=d, seed=33, gate_scale=gate_scale)
    x = inp.to(DEV)
    s0 = 0.1 * torch.randn(H, d, d, device=DEV)
    kcp = kda.long_context_prefill(x.q, x.k, x.v, x.g, x.beta, seg_len, stride, initial_state=s0)
    inp.initial_state = s0[None].cpu()
    ref = oracle_chains(inp, [(0, h) for h in range(H)], stride)
    for h in range(H):
        assert rel_err(kcp["o"][:, h], ref[(0, h)]["o"]) <= TOL_BF16
        assert rel_err(kcp["final_state"][h], ref[(0, h)]["final_state"]) <= TOL_BF16
        assert rel_err(kcp["snapshots"][:, h], ref[(0, h)]["snapshots"]) <= TOL_BF16
    assert kda.kda_get_device_status() == 0


def test_weak_decay_split_over_sixteen_segments():
    """16 segments of 64 tokens under weak decay (log alpha = -0.05 sigmoid): a
    segment's 64 keys leave half of the 128 key directions untouched by the delta
    rule, where its transition M only decays (by about exp(-1.6)), so M stays far
    from 0 and the combine carries real state across every segment boundary.
    Checked against the oracle over the whole sequence."""
    T, H, d, seg_len, stride = 16 * 64, 2, 128, 64, 64
    inp = I.make_prefill_inputs([T], H=H, dk=d, dv=d, seed=35, gate_scale=0.05)
    x = inp.to(DEV)
    s0 = 0.1 * torch.randn(H, d, d, device=DEV, generator=torch.Generator(DEV).manual_seed(5))
    kcp = kda.long_context_prefill(x.q, x.k, x.v, x.g, x.beta, seg_len, stride, initial_state=s0)
    # the transitions of the later segments are far from zero: the combine matters
    assert float(kcp["m"][1:].abs().amax()) > 0.05
    inp.initial_state = s0[None].cpu()
    ref = oracle_chains(inp, [(0, h) for h in range(H)], stride)
    for h in range(H):
        assert rel_err(kcp["o"][:, h], ref[(0, h)]["o"]) <= TOL_BF16
        assert rel_err(kcp["final_state"][h], ref[(0, h)]["final_state"]) <= TOL_BF16
        assert rel_err(kcp["snapshots"][:, h], ref[(0, h)]["snapshots"]) <= TOL_BF16
    assert kda.kda_get_device_status() == 0


@pytest.mark.slow
def test_million_token_context():
    """B=1, H=16, T=1,048,576, d=128: 16 segments of 65,536 tokens combined
    exactly; snapshots every 512 tokens.  Checked against the unsplit GPU run
    over the whole sequence, against the oracle over the whole sequence for one
    head, and on the first two segments of a second head."""
    inp = I.million(device=DEV)
    seg_len, stride = 65536, 512
    kcp = kda.long_context_prefill(inp.q, inp.k, inp.v, inp.g, inp.beta, seg_len, stride)
    full = kda.prefill(inp.q, inp.k, inp.v, inp.g, inp.beta, inp.cu_seqlens,
                       snapshot_stride=stride)
    torch.cuda.synchronize()
    assert rel_err(kcp["o"], full["o"]) <= TOL_BF16
    assert rel_err(kcp["final_state"], full["final_state"][0]) <= TOL_BF16
    assert rel_err(kcp["snapshots"], full["snapshots"]) <= TOL_BF16
    # the oracle over the whole sequence for head 3 (about 1.2e11 fp64 FLOPs), and on a
    # prefix of two segments for head 9
    full_ref = oracle_chains(inp, [(0, 3)], stride)[(0, 3)]
    assert rel_err(kcp["o"][:, 3], full_ref["o"]) <= TOL_BF16
    assert rel_err(kcp["final_state"][3], full_ref["final_state"]) <= TOL_BF16
    assert rel_err(kcp["snapshots"][:, 3], full_ref["snapshots"]) <= TOL_BF16
    Tp = 2 * seg_len
    pre = I.PrefillInputs(inp.q[:Tp], inp.k[:Tp], inp.v[:Tp], inp.g[:Tp], inp.beta[:Tp],
                          torch.tensor([0, Tp], dtype=torch.int32), [Tp], None)
    ref = oracle_chains(pre, [(0, 9)], stride)
    assert rel_err(kcp["o"][:Tp, 9], ref[(0, 9)]["o"]) <= TOL_BF16
    assert rel_err(kcp["snapshots"][:Tp // stride, 9], ref[(0, 9)]["snapshots"]) <= TOL_BF16
    assert kda.kda_get_device_status() == 0
