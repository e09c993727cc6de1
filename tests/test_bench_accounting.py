"""The bench's algorithmic work per unit (CPU): each count against its derivation
from the tensors the path must read and write and the products it must form.  These
are the numerators of every roofline fraction bench.py reports."""
import os
import sys

import pytest

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

import bench  # noqa: E402

D, C = 128, 64


def test_prefill_flops_per_token_head():
    # per chunk: A and P (half of C^2 d each), T K and T V (half of C^2 d each), P U (half
    # of C^2 d), and the three dense C d^2 state products: O, U and the state update,
    # 2 FLOPs per multiply-add, divided over the C tokens of the chunk
    per_chunk_macs = 5 * (C * C * D) // 2 + 3 * C * D * D
    assert bench.prefill_flops_per_token_head(D, D) == 2 * per_chunk_macs // C == 139_264


def test_prefill_bytes_per_token_head():
    # q, k, v bf16 (3 x 256 B), g fp32 (512 B), beta fp32 (4 B), o fp32 (512 B)
    assert bench.prefill_bytes(1, 1, D, D, 1, final=False) == 3 * 2 * D + 4 * D + 4 + 4 * D == 1_796
    # bf16 gate logits instead of fp32 g: 256 B fewer
    assert bench.prefill_bytes(1, 1, D, D, 1, final=False, gate_bytes=2) == 1_540
    # a final state written: one 128 x 128 fp32 state per (request, head)
    assert bench.prefill_bytes(1, 1, D, D, 1, final=True) - 1_796 == D * D * 4
    # an initial state read as well
    assert bench.prefill_bytes(1, 1, D, D, 1, initial=True, final=True) - 1_796 == 2 * D * D * 4


def test_decode_bytes_per_state():
    # the fp32 state read and written, q, k, v bf16, g fp32, beta fp32, o fp32
    assert bench.decode_bytes(1, 1, D) == 2 * D * D * 4 + 3 * D * 2 + 4 * D + 4 + 4 * D == 132_868
    assert bench.decode_bytes(256, 32, D) == 256 * 32 * 132_868


def test_backward_counts():
    # reads q, k, v (bf16), g, beta, dO; writes dq, dk, dv, dg (fp32), dbeta
    assert bench.backward_bytes(1, 1, D, 0) == 3 * 2 * D + 4 * D + 4 + 4 * D + 4 * 4 * D + 4 == 3_848
    # plus per chain: the initial state and dS_final read, dS_0 written
    assert bench.backward_bytes(1, 1, D, 1) - 3_848 == 3 * D * D * 4
    # 7 C d^2 + 7 C^2 d multiply-adds per chunk, over C tokens, plus the forward recompute
    assert bench.backward_flops_per_token_head(D) == 2 * (7 * D * D + 7 * C * D) + 139_264 == 483_328


def test_fp32_cuda_core_peak():
    assert bench.simt_fp32_peak_tflops(1965.0) == pytest.approx(74.44992)


def test_traffic_record_matches_the_kernel_source():
    """The committed ncu DRAM record applies to the current prefill kernel source, so
    the bench reports its traffic instead of null."""
    t = bench.measured_traffic(1_000_000)
    assert t is not None and 0.9e6 < t < 1.1e6
