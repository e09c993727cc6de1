"""GPU parity of the prefill backward (kda_prefill_backward) against the fp64
oracle's reverse-mode derivative, element by element, plus determinism and
varlen isolation.  Tolerance metric as for the forward: max |x - ref| /
max |ref| per gradient tensor, 2e-3 for bf16 inputs, 1e-5 for fp32 inputs."""
import numpy as np
import pytest
import torch

import decode_kda_chunked_b200 as kda
import oracle
from decode_kda_chunked_b200 import inputs as I
from kda_testing import TOL_BF16, TOL_F32, rel_err

pytestmark = pytest.mark.gpu
DEV = "cuda"
GRADS = ("dq", "dk", "dv", "dg", "dbeta")


def _case(lengths, H, d, dtype, seed, gate_scale=5.0, s0=True, cot_o=True, cot_fin=True):
    inp = I.make_prefill_inputs(lengths, H, d, d, dtype=dtype, seed=seed,
                                s0_std=0.1 if s0 else None, gate_scale=gate_scale)
    gen = torch.Generator().manual_seed(seed + 1000)
    T, n = inp.total_tokens, len(lengths)
    d_o = torch.randn((T, H, d), generator=gen) if cot_o else None
    d_fin = torch.randn((n, H, d, d), generator=gen) if cot_fin else None
    return inp, d_o, d_fin


def _run_gpu(inp, d_o, d_fin):
    x = inp.to(DEV)
    out = kda.prefill_backward(x.q, x.k, x.v, x.g, x.beta, x.cu_seqlens,
                               d_o=None if d_o is None else d_o.to(DEV),
                               d_final=None if d_fin is None else d_fin.to(DEV),
                               initial_state=x.initial_state, cu_seqlens_host=inp.cu_seqlens)
    torch.cuda.synchronize()
    return out


def _run_oracle(inp, d_o, d_fin):
    return oracle.prefill_backward(inp.q, inp.k, inp.v, inp.g, inp.beta,
                                   inp.cu_seqlens.numpy(), inp.initial_state, d_o, d_fin)


@pytest.mark.parametrize("d,dtype,tol", [(128, torch.bfloat16, TOL_BF16),
                                         (64, torch.float32, TOL_F32),
                                         (64, torch.bfloat16, TOL_BF16),
                                         (128, torch.float32, TOL_F32)],
                         ids=["bf16-d128", "fp32-d64", "bf16-d64", "fp32-d128"])
@pytest.mark.parametrize("gate_scale", [5.0, 0.05], ids=["strong_decay", "weak_decay"])
def test_backward_matches_oracle(d, dtype, tol, gate_scale):
    # ragged tails, a one-token request and several chunks per request
    inp, d_o, d_fin = _case([100, 64, 1, 190], H=2, d=d, dtype=dtype, seed=51,
                            gate_scale=gate_scale)
    got = _run_gpu(inp, d_o, d_fin)
    ref = _run_oracle(inp, d_o, d_fin)
    for name in GRADS + ("d_initial",):
        assert rel_err(got[name], ref[name]) <= tol, (name, rel_err(got[name], ref[name]))


@pytest.mark.parametrize("cot_o,cot_fin", [(True, False), (False, True)],
                         ids=["only_dO", "only_dS_final"])
def test_backward_single_cotangent(cot_o, cot_fin):
    # weak decay: with strong decay a final-state cotangent alone reaches the early
    # tokens only as values far below the fp32 range (about 1e-114 here)
    inp, d_o, d_fin = _case([130, 70], H=2, d=128, dtype=torch.bfloat16, seed=53,
                            gate_scale=0.05, cot_o=cot_o, cot_fin=cot_fin)
    got = _run_gpu(inp, d_o, d_fin)
    ref = _run_oracle(inp, d_o, d_fin)
    for name in GRADS + ("d_initial",):
        assert rel_err(got[name], ref[name]) <= TOL_BF16, name


def test_backward_empty_request_and_zero_start():
    # an empty request: its initial-state gradient is d_final itself
    inp, d_o, d_fin = _case([65, 0, 128], H=2, d=128, dtype=torch.bfloat16, seed=55, s0=False)
    got = _run_gpu(inp, d_o, d_fin)
    ref = _run_oracle(inp, d_o, d_fin)
    for name in GRADS + ("d_initial",):
        assert rel_err(got[name], ref[name]) <= TOL_BF16, name
    assert torch.equal(got["d_initial"][1].cpu(), d_fin[1])


def test_backward_is_deterministic_and_isolated():
    lengths = [150, 77, 200]
    inp, d_o, d_fin = _case(lengths, H=2, d=128, dtype=torch.bfloat16, seed=57)
    a = _run_gpu(inp, d_o, d_fin)
    b = _run_gpu(inp, d_o, d_fin)
    for name in GRADS + ("d_initial",):
        assert torch.equal(a[name], b[name]), name
    # request 1 alone gives bit-identical gradients
    lo, hi = 150, 227
    alone = I.PrefillInputs(inp.q[lo:hi], inp.k[lo:hi], inp.v[lo:hi], inp.g[lo:hi],
                            inp.beta[lo:hi], torch.tensor([0, hi - lo], dtype=torch.int32),
                            [hi - lo], inp.initial_state[1:2], inp.meta)
    c = _run_gpu(alone, d_o[lo:hi], d_fin[1:2])
    for name in GRADS:
        assert torch.equal(c[name], a[name][lo:hi]), name
    assert torch.equal(c["d_initial"][0], a["d_initial"][1])


def test_backward_through_the_simt_forward(monkeypatch):
    """bf16 d=128 with the forward's SIMT kernel forced: the same gradients
    (the chunk-start states differ only by the forward kernels' rounding)."""
    inp, d_o, d_fin = _case([129, 64], H=1, d=128, dtype=torch.bfloat16, seed=59)
    ref = _run_oracle(inp, d_o, d_fin)
    monkeypatch.setenv("KDA_FORCE_SIMT", "1")
    got = _run_gpu(inp, d_o, d_fin)
    for name in GRADS + ("d_initial",):
        assert rel_err(got[name], ref[name]) <= TOL_BF16, name


@pytest.mark.slow
def test_backward_varlen_full_size():
    """The headline workload (64 requests, lengths log-uniform on [128, 4096], H=32,
    d=128) at full size, in the launch configuration bench.py times; the oracle's
    derivative on 6 sampled chains (the longest and shortest request and 4 random
    (request, head) pairs), each packed as a one-head request."""
    import random
    inp = I.varlen(device=DEV)
    T, H, d, n = inp.total_tokens, 32, 128, inp.n_req
    gen = torch.Generator().manual_seed(61)
    d_o = torch.randn((T, H, d), generator=gen)
    d_fin = torch.randn((n, H, d, d), generator=gen)
    got = kda.prefill_backward(inp.q, inp.k, inp.v, inp.g, inp.beta, inp.cu_seqlens,
                               d_o=d_o.to(DEV), d_final=d_fin.to(DEV),
                               cu_seqlens_host=inp.cu_seqlens.cpu())
    torch.cuda.synchronize()
    lens = inp.lengths
    rng = random.Random(1)
    pairs = [(int(np.argmax(lens)), 3), (int(np.argmin(lens)), 17)]
    pairs += [(rng.randrange(n), rng.randrange(H)) for _ in range(4)]
    cu = [int(c) for c in inp.cu_seqlens.cpu().tolist()]
    parts = {k: [] for k in ("q", "k", "v", "g", "beta", "d_o")}
    for (r, h) in pairs:
        lo, hi = cu[r], cu[r + 1]
        for name in ("q", "k", "v", "g"):
            parts[name].append(getattr(inp, name)[lo:hi, h:h + 1].cpu())
        parts["beta"].append(inp.beta[lo:hi, h:h + 1].cpu())
        parts["d_o"].append(d_o[lo:hi, h:h + 1])
    cat = {k: torch.cat(v, 0) for k, v in parts.items()}
    pcu = np.concatenate([[0], np.cumsum([cu[r + 1] - cu[r] for r, _ in pairs])])
    dfin = torch.stack([d_fin[r, h:h + 1] for r, h in pairs], 0)
    ref = oracle.prefill_backward(cat["q"], cat["k"], cat["v"], cat["g"], cat["beta"], pcu,
                                  None, cat["d_o"], dfin)
    for c, (r, h) in enumerate(pairs):
        lo, hi = cu[r], cu[r + 1]
        plo, phi = int(pcu[c]), int(pcu[c + 1])
        for name in GRADS:
            g_gpu = got[name][lo:hi, h]
            g_ref = ref[name][plo:phi, 0]
            assert rel_err(g_gpu, g_ref) <= TOL_BF16, (name, r, h, rel_err(g_gpu, g_ref))
        # with strong decay a whole request's decay can take dS_0 below the fp32 range
        d0_ref = np.asarray(ref["d_initial"][c, 0])
        d0 = got["d_initial"][r, h].double().cpu().numpy()
        if np.abs(d0_ref).max() < 1e-30:
            assert np.abs(d0).max() < 1e-30, (r, h)
        else:
            assert rel_err(d0, d0_ref) <= TOL_BF16, (r, h)
