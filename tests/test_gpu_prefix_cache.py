"""GPU: the state pool copies (gather / scatter) bit-exact against plain indexing, a
slot past the pool reported instead of touched, and a prefix-cache resume (two
batches of prompts that share prefixes) equal to the fp64 oracle's run over the
whole prompts."""
import numpy as np
import pytest
import torch

import decode_kda_chunked_b200 as kda
import oracle
from decode_kda_chunked_b200 import _lib
from decode_kda_chunked_b200 import inputs as I
from kda_testing import TOL_BF16, rel_err

pytestmark = pytest.mark.gpu
DEV = "cuda"


def test_gather_and_scatter_are_exact_copies():
    gen = torch.Generator(device=DEV).manual_seed(5)
    pool = torch.randn((6, 2, 64, 64), generator=gen, device=DEV)
    slots = torch.tensor([3, -1, 0, 5, 3], dtype=torch.int32, device=DEV)
    dst = torch.full((5, 2, 64, 64), 7.0, device=DEV)
    _lib.kda_state_gather(pool, slots, dst)
    src = torch.randn((4, 2, 64, 64), generator=gen, device=DEV)
    pool2 = pool.clone()
    _lib.kda_state_scatter(src, torch.tensor([1, -1, 4, 2], dtype=torch.int32, device=DEV), pool2)
    torch.cuda.synchronize()
    assert kda.kda_get_device_status() == 0
    for i, s in enumerate([3, -1, 0, 5, 3]):
        ref = pool[s] if s >= 0 else torch.zeros_like(pool[0])
        assert torch.equal(dst[i], ref), i
    ref_pool = pool.clone()
    ref_pool[1], ref_pool[4], ref_pool[2] = src[0], src[2], src[3]
    assert torch.equal(pool2, ref_pool)


def test_slot_past_the_pool_is_reported_and_not_touched():
    pool = torch.zeros((4, 2, 64, 64), device=DEV)
    dst = torch.full((2, 2, 64, 64), 3.0, device=DEV)
    _lib.kda_state_gather(pool, torch.tensor([1, 4], dtype=torch.int32, device=DEV), dst)
    assert kda.kda_get_device_status() == 1          # KDA_ERR_INVALID_ARG
    assert torch.equal(dst[1], torch.full_like(dst[1], 3.0))
    assert torch.equal(dst[0], torch.zeros_like(dst[0]))
    src = torch.ones((1, 2, 64, 64), device=DEV)
    _lib.kda_state_scatter(src, torch.tensor([9], dtype=torch.int32, device=DEV), pool)
    assert kda.kda_get_device_status() == 1
    assert torch.equal(pool, torch.zeros_like(pool))


@pytest.mark.parametrize("d,dtype", [(128, torch.bfloat16), (64, torch.bfloat16)],
                         ids=["d128-tc", "d64-simt"])
def test_resume_through_the_cache_matches_oracle(d, dtype):
    H, vocab = 2, 4096
    table = I.token_table(vocab, H, d, d, dtype=dtype, seed=71)
    table_dev = table.to(DEV)
    rng = np.random.default_rng(72)
    new = lambda n: [int(x) for x in rng.integers(0, vocab, size=n)]
    A, B = new(1300), new(700)
    cache = kda.PrefixCache(n_slots=8, H=H, dk=d, dv=d, device=DEV)

    def run(prompts, expect_cached):
        plan = cache.plan(prompts)
        assert [m for m, _ in plan] == expect_cached
        x = I.prompt_inputs(table_dev, [p[m:] for p, (m, _) in zip(prompts, plan)])
        out = cache.prefill(prompts, plan, x.q, x.k, x.v, x.g, x.beta)
        torch.cuda.synchronize()
        assert kda.kda_get_device_status() == 0
        full = I.prompt_inputs(table, prompts)
        ref = oracle.prefill(full.q, full.k, full.v, full.g, full.beta, full.cu_seqlens.numpy())
        cu_run = x.cu_seqlens.tolist()
        cu_full = full.cu_seqlens.tolist()
        for r, (m, _) in enumerate(plan):
            got_o = out["o"][cu_run[r]:cu_run[r + 1]]
            ref_o = ref["o"][cu_full[r] + m:cu_full[r + 1]]
            assert rel_err(got_o, ref_o) <= TOL_BF16, (r, rel_err(got_o, ref_o))
            assert rel_err(out["final_state"][r], ref["final_state"][r]) <= TOL_BF16, r

    run([A, B], [0, 0])
    assert len(cache) == 3                       # A: 2 blocks, B: 1 block
    A2, C, D = A[:1024] + new(200), B[:512] + new(300), new(600)
    # A itself: at least one token must run, so 1,024 of its 1,300 come from the cache
    run([A2, C, D, A], [1024, 512, 0, 1024])
    assert len(cache) == 4                       # only D brings a block not seen before
