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


def test_kcp_bytes_count_each_input_once():
    # pass 1 reads k, v (bf16), g and beta once per token-head: 1,028 B at d = 128, and
    # writes (S_loc, M) per segment-head; pass 2 is the prefill with fp32 o from the
    # recovered start states; snapshots every 512 tokens
    T, H, n_seg = 65536, 1, 1
    pass1 = T * H * 1_028 + 2 * n_seg * H * D * D * 4
    pass2 = T * H * 1_796 + n_seg * H * D * D * 4
    snaps = (T // 512) * H * D * D * 4
    assert bench.kcp_bytes(T, H, D, n_seg) == pass1 + pass2 + snaps
    # the million-token workload: about 17.2 GB + 30.1 GB + 2.15 GB
    assert 49.4e9 < bench.kcp_bytes(1 << 20, 16, D, 16) < 49.6e9


def test_launcher_command_is_one_node_torchrun():
    cmd = bench.torchrun_command(4, ["--gpus", "4", "--steps", "2"], 29511)
    assert cmd[1:4] == ["-m", "torch.distributed.run", "--nnodes=1"]
    assert "--nproc-per-node=4" in cmd and "--master-addr=127.0.0.1" in cmd
    assert "--master-port=29511" in cmd
    assert cmd[-4:] == ["--gpus", "4", "--steps", "2"]


def test_gpus_flag_starts_that_many_ranks():
    """`bench.py --gpus 2` outside any launcher starts two ranks itself; the ranks
    join one process group (gloo here, NCCL on GPUs) and rank 0 reports the group
    size and the max over ranks of a per-rank value."""
    import json
    import subprocess
    env = {k: v for k, v in os.environ.items()
           if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK", "MASTER_ADDR", "MASTER_PORT")}
    out = subprocess.run([sys.executable, bench.__file__, "--gpus", "2", "--dist-check"],
                         env=env, capture_output=True, text=True, timeout=300)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [json.loads(x) for x in out.stdout.splitlines() if x.startswith("{")]
    assert len(lines) == 1
    rec = lines[0]
    assert rec["n_gpus"] == 2
    assert rec["process_group"] == {"backend": "gloo", "size": 2}
    assert rec["max_over_ranks"] == 1.0


def test_world_size_must_match_the_gpus_flag():
    import subprocess
    env = dict(os.environ, WORLD_SIZE="1", RANK="0", LOCAL_RANK="0")
    out = subprocess.run([sys.executable, bench.__file__, "--gpus", "3", "--dist-check"],
                         env=env, capture_output=True, text=True, timeout=120)
    assert out.returncode != 0 and "--gpus 3" in out.stderr
