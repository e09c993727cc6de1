"""Per-phase cycle profile of the tensor-core chunked prefill.

    python -m decode_kda_chunked_b200.phase_profile [--requests N] [--steps K]

Builds the diagnostic library libkda_phase.so (the same sources compiled with
KDA_PHASE_PROFILE: worker thread 0 of every CTA reads clock64 at each step of the
chunk loop), runs the varlen prefill workload (64 requests, lengths log-uniform on
[128, 4096], H=32, d=128, bf16 q/k/v, fp32 g, beta and o) through it, and prints
the mean cycles per 32-token chunk of each step of both worker groups (group A:
gate, row operands, A|P read-out, solve; group B: state scaling, Khat^T, outputs,
V^T), each with its share of the group's time.  The counters
perturb the timing slightly; the table shows where a chunk's time goes, the
bench measures how long it takes.  Needs a CUDA device.
"""
from __future__ import annotations

import argparse
import ctypes
import json

# group A (worker thread 0) and group B (worker thread 256) steps, by counter slot
PHASES = {0: "A wait: O^T, Y^T of chunk m-1", 1: "A wait: tiles of m+1",
          2: "A gate (cumulative) of m+1",
          3: "A rows (L, R', gamma Q/K)", 4: "A wait: A|P", 5: "A read (A, P)",
          7: "A solve: diagonal blocks", 6: "A solve: block below the diagonal",
          8: "B wait: O^T, Y^T", 9: "B scale S^T", 10: "B wait: next gate", 11: "B Khat^T",
          12: "B wait: last products", 13: "B out (o, snapshots)", 14: "B V^T"}
# group A (worker thread 0) and group B (worker thread 256), slots in loop order
GROUPS = (("A", (0, 1, 2, 3, 4, 5, 7, 6)), ("B", range(8, 15)))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--requests", type=int, default=None, help="first N requests only")
    ap.add_argument("--steps", type=int, default=3)
    args = ap.parse_args()

    import torch

    from . import _lib, build
    from . import inputs as I
    path = build.build(phase_profile=True)
    lib = _lib.load(path)
    lib.kda_phase_cycles.restype = ctypes.c_int
    lib.kda_phase_cycles.argtypes = [ctypes.POINTER(ctypes.c_ulonglong), ctypes.c_int, ctypes.c_int]
    dev = torch.device("cuda", 0)
    if args.requests is None:
        x = I.varlen(device=dev)
    else:
        x = I.make_prefill_inputs(I.varlen_lengths(0)[:args.requests], H=32, dk=128, dv=128,
                                  seed=0, device=dev)
    from . import prefill
    buf = (ctypes.c_ulonglong * 16)()
    prefill(x.q, x.k, x.v, x.g, x.beta, x.cu_seqlens, cu_seqlens_host=x.cu_seqlens.cpu())
    torch.cuda.synchronize()
    assert lib.kda_phase_cycles(buf, 16, 1) == 0  # clear after the warm-up call
    for _ in range(args.steps):
        prefill(x.q, x.k, x.v, x.g, x.beta, x.cu_seqlens, cu_seqlens_host=x.cu_seqlens.cpu())
    torch.cuda.synchronize()
    assert lib.kda_phase_cycles(buf, 16, 0) == 0
    chunks = buf[15]
    out = {}
    print(f"{chunks // args.steps} chunks of 32 tokens per call")
    for grp, slots in GROUPS:
        total = sum(buf[k] for k in slots)
        print(f"group {grp}: {total / chunks:.0f} cycles per chunk")
        rows = [{"phase": PHASES[k], "cycles_per_chunk": buf[k] / chunks,
                 "share": buf[k] / total if total else 0.0} for k in slots]
        for rw in rows:
            print(f"  {rw['phase']:<32} {rw['cycles_per_chunk']:8.0f}  {100 * rw['share']:5.1f} %")
        out[grp] = {"cycles_per_chunk": total / chunks, "phases": rows}
    print(json.dumps(out))


if __name__ == "__main__":
    main()
