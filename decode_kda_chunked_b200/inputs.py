"""Seeded synthetic inputs for KDA workloads.

This module only draws random numbers and lays them out; it holds none of
the method's arithmetic, imports neither the CUDA binding nor the oracle, and
feeds both.  Draw order within one workload is fixed: q, k, v, g, beta,
initial state.

Distributions (the five standard workloads below):
  * q, k ~ N(0, 1), L2-normalised per (token, head) in fp32, then cast to the
    input dtype (round-to-nearest-even for bf16);
  * v ~ N(0, 1), cast to the input dtype;
  * beta = sigmoid(N(0, 1)) per (token, head), fp32;
  * g = log alpha = -5 * sigmoid(N(0, 1)) per (token, head, channel), fp32,
    so alpha >= exp(-5) (the lower-bounded decay of KDA, CSDN post on the
    Kimi K3 technical report, section 一.1);
  * initial states ~ N(0, std) fp32 where a workload asks for one.

With ``gate_logits=True`` the gate's N(0, 1) draw is kept as bf16 logits
``g_logits`` instead (for the fused gate activation, which applies
-5 * sigmoid itself) and ``g`` is None; every other draw is unchanged.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

GATE_LOWER = -5.0  # log alpha >= -5 in every standard workload


@dataclass
class PrefillInputs:
    q: torch.Tensor            # [T, H, dk]
    k: torch.Tensor            # [T, H, dk]
    v: torch.Tensor            # [T, H, dv]
    g: torch.Tensor            # [T, H, dk] fp32 log alpha
    beta: torch.Tensor         # [T, H] fp32
    cu_seqlens: torch.Tensor   # [n_req + 1] int32 (same device as the tensors)
    lengths: list              # host copy of the request lengths
    initial_state: torch.Tensor | None  # [n_req, H, dk, dv] fp32 or None
    meta: dict = field(default_factory=dict)
    g_logits: torch.Tensor | None = None  # [T, H, dk] bf16 gate logits (g is None then)

    @property
    def total_tokens(self) -> int:
        return int(sum(self.lengths))

    @property
    def n_req(self) -> int:
        return len(self.lengths)

    def to(self, device) -> "PrefillInputs":
        mv = lambda t: None if t is None else t.to(device)
        return PrefillInputs(mv(self.q), mv(self.k), mv(self.v), mv(self.g), mv(self.beta),
                             mv(self.cu_seqlens), list(self.lengths), mv(self.initial_state),
                             dict(self.meta), mv(self.g_logits))


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _unit_rows(shape, gen, device, dtype):
    x = torch.randn(shape, generator=gen, device=device, dtype=torch.float32)
    x = x / x.norm(dim=-1, keepdim=True)
    return x.to(dtype)


def make_prefill_inputs(lengths, H: int, dk: int, dv: int, dtype=torch.bfloat16,
                        seed: int = 0, s0_std: float | None = None, device="cpu",
                        gate_scale: float = -GATE_LOWER,
                        gate_logits: bool = False) -> PrefillInputs:
    """Packed varlen inputs for ``len(lengths)`` requests of the given lengths."""
    lengths = [int(x) for x in lengths]
    T = sum(lengths)
    gen = _gen(seed, device)
    q = _unit_rows((T, H, dk), gen, device, dtype)
    k = _unit_rows((T, H, dk), gen, device, dtype)
    v = torch.randn((T, H, dv), generator=gen, device=device, dtype=torch.float32).to(dtype)
    z = torch.randn((T, H, dk), generator=gen, device=device, dtype=torch.float32)
    x = z.to(torch.bfloat16).contiguous() if gate_logits else None
    g = None if gate_logits else (-gate_scale * torch.sigmoid(z)).contiguous()
    beta = torch.sigmoid(torch.randn((T, H), generator=gen, device=device, dtype=torch.float32))
    s0 = None
    if s0_std is not None:
        s0 = s0_std * torch.randn((len(lengths), H, dk, dv), generator=gen, device=device,
                                  dtype=torch.float32)
    cu = torch.tensor([0] + list(_cumsum(lengths)), dtype=torch.int32, device=device)
    return PrefillInputs(q, k, v, g, beta.contiguous(), cu, lengths, s0,
                         {"seed": seed, "dtype": str(dtype).replace("torch.", "")}, x)


def _cumsum(xs):
    s = 0
    for x in xs:
        s += x
        yield s


def loguniform_lengths(n: int, lo: int, hi: int, seed: int = 0) -> list:
    """n lengths drawn log-uniform on [lo, hi] (CPU generator, so identical on every box)."""
    gen = _gen(seed, "cpu")
    u = torch.rand(n, generator=gen, dtype=torch.float64)
    lens = torch.floor(torch.exp(math.log(lo) + u * (math.log(hi) - math.log(lo))))
    return [int(min(max(x, lo), hi)) for x in lens.tolist()]


# --------------------------------------------------------------------------
# The five standard workloads.
# --------------------------------------------------------------------------

WORKLOADS = {
    "oracle_scale": "B=1, H=2, T=256, d_k=d_v=64, fp32 q/k/v, zero initial state, seed 0",
    "single_seq": "B=1, H=32, T=8192, d_k=d_v=128, bf16 q/k/v, fp32 g/beta, "
                  "initial state N(0, 0.1) fp32, seed 0",
    "varlen": "64 requests, lengths log-uniform on [128, 4096] (seed 0), H=32, "
              "d_k=d_v=128, bf16 q/k/v, fp32 g/beta, zero initial states, final states out",
    "million": "B=1, H=16, T=1,048,576, d_k=d_v=128, bf16 q/k/v, fp32 g/beta, "
               "16 segments of 65,536 tokens, fp32 snapshots every 512 tokens",
    "decode": "256 requests x H=32 fp32 states of 128x128 ~ N(0, 0.05), one bf16 "
              "token per request per step",
}


def oracle_scale(device="cpu", seed: int = 0) -> PrefillInputs:
    return make_prefill_inputs([256], H=2, dk=64, dv=64, dtype=torch.float32, seed=seed,
                               s0_std=None, device=device)


def single_seq(device="cpu", seed: int = 0, T: int = 8192) -> PrefillInputs:
    return make_prefill_inputs([T], H=32, dk=128, dv=128, dtype=torch.bfloat16, seed=seed,
                               s0_std=0.1, device=device)


VARLEN_N, VARLEN_LO, VARLEN_HI = 64, 128, 4096


def varlen_lengths(seed: int = 0) -> list:
    return loguniform_lengths(VARLEN_N, VARLEN_LO, VARLEN_HI, seed)


def varlen(device="cpu", seed: int = 0, gate_logits: bool = False) -> PrefillInputs:
    return make_prefill_inputs(varlen_lengths(seed), H=32, dk=128, dv=128,
                               dtype=torch.bfloat16, seed=seed, s0_std=None, device=device,
                               gate_logits=gate_logits)


MILLION_T, MILLION_SEGMENTS, SNAPSHOT_STRIDE = 1 << 20, 16, 512


def million(device="cpu", seed: int = 0, T: int = MILLION_T, H: int = 16) -> PrefillInputs:
    return make_prefill_inputs([T], H=H, dk=128, dv=128, dtype=torch.bfloat16, seed=seed,
                               s0_std=None, device=device)


@dataclass
class DecodeInputs:
    q: torch.Tensor        # [steps, N, H, dk]
    k: torch.Tensor
    v: torch.Tensor        # [steps, N, H, dv]
    g: torch.Tensor        # [steps, N, H, dk]
    beta: torch.Tensor     # [steps, N, H]
    state: torch.Tensor    # [N, H, dk, dv] fp32


def decode(steps: int, N: int = 256, H: int = 32, d: int = 128, device="cpu", seed: int = 0,
           state_std: float = 0.05, dtype=torch.bfloat16) -> DecodeInputs:
    """``steps`` tokens for each of N requests plus their initial fp32 states."""
    gen = _gen(seed, device)
    q = _unit_rows((steps, N, H, d), gen, device, dtype)
    k = _unit_rows((steps, N, H, d), gen, device, dtype)
    v = torch.randn((steps, N, H, d), generator=gen, device=device,
                    dtype=torch.float32).to(dtype)
    g = GATE_LOWER * torch.sigmoid(torch.randn((steps, N, H, d), generator=gen, device=device,
                                               dtype=torch.float32))
    beta = torch.sigmoid(torch.randn((steps, N, H), generator=gen, device=device,
                                     dtype=torch.float32))
    state = state_std * torch.randn((N, H, d, d), generator=gen, device=device,
                                    dtype=torch.float32)
    return DecodeInputs(q, k, v, g, beta, state)


# --------------------------------------------------------------------------
# Prompts as token ids (prefix-cache workloads): the inputs of a token are a
# fixed row per id, so prompts that share a prefix share its inputs.
# --------------------------------------------------------------------------

def token_table(vocab: int, H: int, dk: int, dv: int, dtype=torch.bfloat16, seed: int = 0,
                device="cpu", gate_logits: bool = False) -> PrefillInputs:
    """Per token id t < vocab, the inputs of one token (row t of every tensor),
    drawn like any workload; a stand-in for a model's per-token projections."""
    return make_prefill_inputs([vocab], H, dk, dv, dtype=dtype, seed=seed, device=device,
                               gate_logits=gate_logits)


def prompt_inputs(table: PrefillInputs, prompts) -> PrefillInputs:
    """Packed inputs of the given prompts (sequences of token ids): rows of ``table``."""
    lengths = [len(p) for p in prompts]
    dev = table.k.device
    ids = torch.tensor([int(t) for p in prompts for t in p], dtype=torch.long, device=dev)
    pick = lambda x: None if x is None else x[ids].contiguous()
    cu = torch.tensor([0] + list(_cumsum(lengths)), dtype=torch.int32, device=dev)
    return PrefillInputs(pick(table.q), pick(table.k), pick(table.v), pick(table.g),
                         pick(table.beta), cu, lengths, None, dict(table.meta),
                         pick(table.g_logits))
