"""Seeded synthetic inputs for the gated delta rule with a QDQ state.

This module only draws random inputs; it holds none of the recurrence's or the
codecs' arithmetic, so both the CUDA path and the CPU oracle can take their
inputs from it without sharing any of the method.

Distributions follow the workload descriptions of the GatedDeltaNet / KDA
state-QAT pages (the "linear_attention" QAT series): q and k are standard
normal and L2-normalised per (token, head) over the key axis, v is standard
normal, beta = sigmoid(N(0, 1)), and the log-gate is g = log sigmoid(N(3, 1))
(natural log, so the decay is alpha = exp(g) in (0, 1)); for KDA the gate is
drawn per key channel.  Random initial states are N(0, 0.05^2) in fp32.

Draw order for one case, all from one ``torch.Generator('cpu')`` seeded with
``case.seed``: lengths (packed cases only), q, k, v, beta-logit, gate-logit,
initial state, then the decode tokens' q, k, v, beta-logit and gate-logit,
each drawn for all decode steps at once ([steps, n_seq, H, ...]).  Every
draw is fp32 on the CPU; q/k/v are cast to the case's dtype at the end.
"""

from __future__ import annotations

import dataclasses
from typing import Optional

import torch

__all__ = ["Case", "CONFIGS", "generate", "small_case"]


@dataclasses.dataclass(frozen=True)
class Case:
    """One workload: shapes, dtypes, gate kind, codec and random recipe.

    ``T`` is the tokens per sequence for a dense ``[B, T, H, d]`` layout; a
    packed case sets ``lengths`` (or ``varlen_max`` to draw them) instead and
    uses ``[1, sum(lengths), H, d]`` with int32 ``cu_seqlens``.
    """

    name: str
    n_seq: int
    H: int
    d_k: int
    d_v: int
    T: int = 0
    varlen_max: int = 0
    lengths: Optional[tuple] = None
    dtype: str = "bf16"          # dtype of q, k, v and o: "bf16" or "f32"
    gate: str = "scalar"         # "scalar" (GDN) or "per_key" (KDA)
    qdq: str = "fp8_tile64"      # "none", "fp8_tile64", "int8_g32"
    state: str = "zero"          # "zero" or "normal" (N(0, state_std^2))
    state_std: float = 0.05
    decode_steps: int = 0
    seed: int = 1000

    @property
    def varlen(self) -> bool:
        return self.varlen_max > 0 or self.lengths is not None


# The five workloads of the method's benchmark description.
CONFIGS = {
    "tiny": Case("tiny", n_seq=1, H=2, d_k=64, d_v=64, T=64, dtype="f32",
                 gate="scalar", qdq="int8_g32", state="zero",
                 decode_steps=64, seed=1000),
    "gdn_prefill": Case("gdn_prefill", n_seq=4, H=16, d_k=128, d_v=128,
                        T=4096, dtype="bf16", gate="scalar",
                        qdq="fp8_tile64", state="zero", seed=1001),
    "kda_prefill": Case("kda_prefill", n_seq=2, H=32, d_k=128, d_v=128,
                        T=8192, dtype="bf16", gate="per_key",
                        qdq="int8_g32", state="zero", seed=1002),
    "serving_decode": Case("serving_decode", n_seq=256, H=32, d_k=128,
                           d_v=128, T=0, dtype="bf16", gate="scalar",
                           qdq="int8_g32", state="normal", decode_steps=512,
                           seed=1003),
    "varlen": Case("varlen", n_seq=64, H=16, d_k=128, d_v=128,
                   varlen_max=4096, dtype="bf16", gate="scalar",
                   qdq="fp8_tile64", state="normal", decode_steps=32,
                   seed=1004),
}


def small_case(base: str, **over) -> Case:
    """A smaller case with the same distributions as ``CONFIGS[base]``."""
    return dataclasses.replace(CONFIGS[base], **over)


_TORCH_DTYPE = {"bf16": torch.bfloat16, "f32": torch.float32}


def _unit_normal_rows(gen: torch.Generator, shape) -> torch.Tensor:
    x = torch.randn(shape, generator=gen, dtype=torch.float32)
    return x / x.norm(dim=-1, keepdim=True)


def _log_gate(gen: torch.Generator, shape) -> torch.Tensor:
    # log sigmoid(x), x ~ N(3, 1): evaluated in fp64, stored as fp32.
    x = torch.randn(shape, generator=gen, dtype=torch.float32) + 3.0
    return torch.nn.functional.logsigmoid(x.double()).float()


def _beta(gen: torch.Generator, shape) -> torch.Tensor:
    return torch.sigmoid(torch.randn(shape, generator=gen, dtype=torch.float32))


def generate(case: Case) -> dict:
    """Draw every input of ``case`` on the CPU.

    Returns a dict with ``q, k, v`` ([B, T, H, d] dense or [1, total, H, d]
    packed, in the case dtype), ``g`` (fp32, [..., H] or [..., H, d_k]),
    ``beta`` (fp32 [..., H]), ``state_in`` (fp32 [n_seq, H, d_k, d_v] or
    None for a zero state), ``cu_seqlens`` (int32 [n_seq + 1] or None),
    ``lengths`` (list of int), and, when the case has decode steps,
    ``dec_q, dec_k, dec_v`` ([steps, n_seq, H, d]), ``dec_g``, ``dec_beta``.
    """
    gen = torch.Generator("cpu")
    gen.manual_seed(case.seed)
    dt = _TORCH_DTYPE[case.dtype]
    H, dk, dv = case.H, case.d_k, case.d_v

    if case.lengths is not None:
        lengths = [int(x) for x in case.lengths]
    elif case.varlen_max > 0:
        lengths = torch.randint(1, case.varlen_max + 1, (case.n_seq,),
                                generator=gen).tolist()
    else:
        lengths = [case.T] * case.n_seq

    if case.varlen:
        lead = (1, sum(lengths))
        cu = torch.zeros(case.n_seq + 1, dtype=torch.int32)
        cu[1:] = torch.cumsum(torch.tensor(lengths, dtype=torch.int64), 0).to(torch.int32)
    else:
        lead = (case.n_seq, case.T)
        cu = None

    out = {"lengths": lengths, "cu_seqlens": cu}
    out["q"] = _unit_normal_rows(gen, lead + (H, dk)).to(dt)
    out["k"] = _unit_normal_rows(gen, lead + (H, dk)).to(dt)
    out["v"] = torch.randn(lead + (H, dv), generator=gen, dtype=torch.float32).to(dt)
    out["beta"] = _beta(gen, lead + (H,))
    gshape = lead + ((H, dk) if case.gate == "per_key" else (H,))
    out["g"] = _log_gate(gen, gshape)
    if case.state == "normal":
        out["state_in"] = torch.randn((case.n_seq, H, dk, dv), generator=gen,
                                      dtype=torch.float32) * case.state_std
    else:
        out["state_in"] = None

    if case.decode_steps > 0:
        S, N = case.decode_steps, case.n_seq
        gs = (S, N, H, dk) if case.gate == "per_key" else (S, N, H)
        out["dec_q"] = _unit_normal_rows(gen, (S, N, H, dk)).to(dt)
        out["dec_k"] = _unit_normal_rows(gen, (S, N, H, dk)).to(dt)
        out["dec_v"] = torch.randn((S, N, H, dv), generator=gen, dtype=torch.float32).to(dt)
        out["dec_beta"] = _beta(gen, (S, N, H))
        out["dec_g"] = _log_gate(gen, gs)
    return out
