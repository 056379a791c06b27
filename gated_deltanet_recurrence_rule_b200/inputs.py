"""Seeded synthetic inputs for the gated delta rule workloads.

This module only draws random numbers and shapes them; it holds none of the
recurrence arithmetic.  The oracle and the CUDA path read the same tensors it
returns, so both see identical bf16 / fp32 bits.

Recipe (all draws on the CPU from one ``torch.Generator`` seeded per
workload, in this order):
  q, k ~ N(0, 1) in fp32, L2-normalised per (token, head) over the head dim,
         then cast to the input dtype (round to nearest even);
  v    ~ N(0, 1) cast to the input dtype;
  beta = sigmoid(N(0, 1)) fp32, one per (token, V head);
  g    = -softplus(N(mu, 1)) fp32 (log of the decay alpha; mu = 0, or -2 for
         the slow-decay long-context workload);
  initial states ~ N(0, std^2) fp32 when requested (std = 0.02).
Keys are normalised because the pages describe k_t as the normalized key
("Inside Qwen3.8-27B ...", section "Gated DeltaNet Mechanics"); the head
layout 16 QK / 48 V heads at head dim 128 is from "Qwen 3.8 27B Review ...",
section "3. Architecture: Gated DeltaNet Hybrid + FP8 Quantization".
"""
from __future__ import annotations

from dataclasses import dataclass

import torch
import torch.nn.functional as F

DTYPES = {"bf16": torch.bfloat16, "fp32": torch.float32}


@dataclass(frozen=True)
class Workload:
    name: str
    lengths: tuple          # sequence lengths (prefill) ; () for decode
    Hqk: int
    Hv: int
    D: int
    dtype: str              # "bf16" | "fp32"
    seed: int
    g_mu: float = 0.0
    init_std: float = 0.0   # 0 -> no initial state (zeros)
    batch: int = 0          # decode: sequences per step
    steps: int = 0          # decode: consecutive steps

    @property
    def total_tokens(self) -> int:
        return int(sum(self.lengths))


def varlen_lengths(num_seqs: int = 32, lo: int = 1024, hi: int = 32768, seed: int = 4):
    gen = torch.Generator().manual_seed(seed)
    return tuple(int(x) for x in torch.randint(lo, hi + 1, (num_seqs,), generator=gen))


WORKLOADS = {
    # small case the oracle finishes in seconds (fp32)
    "tiny": Workload("tiny", (256,), 2, 6, 64, "fp32", 0),
    # one Qwen3.8-27B-shaped DeltaNet layer, 8k-token prefill
    "prefill8k": Workload("prefill8k", (8192,), 16, 48, 128, "bf16", 1),
    # batched decode, 64 sequences x 1000 steps, fp32 state ~N(0, 0.02^2)
    "decode64": Workload("decode64", (), 16, 48, 128, "bf16", 2, init_std=0.02, batch=64,
                         steps=1000),
    # 262,144-token prefill, slow decay, nonzero initial state
    "long262k": Workload("long262k", (262144,), 16, 48, 128, "bf16", 3, g_mu=-2.0, init_std=0.02),
    # 32 packed sequences, lengths uniform in [1024, 32768]
    "varlen32": Workload("varlen32", varlen_lengths(), 16, 48, 128, "bf16", 4, init_std=0.02),
}


def _unit_rows(x: torch.Tensor) -> torch.Tensor:
    return x / x.norm(dim=-1, keepdim=True).clamp_min(1e-30)


def prefill_inputs(lengths, Hqk, Hv, D, dtype="bf16", seed=0, g_mu=0.0, init_std=0.0,
                   Dv=None):
    """Packed-sequence inputs.  Returns a dict of CPU tensors:
    q, k [T, Hqk, D]; v [T, Hv, Dv]; g, beta [T, Hv] fp32; cu_seqlens [N+1] int32;
    initial_state [N, Hv, Dv, D] fp32 or None."""
    Dv = D if Dv is None else Dv
    dt = DTYPES[dtype]
    lengths = [int(x) for x in lengths]
    T, N = sum(lengths), len(lengths)
    gen = torch.Generator().manual_seed(seed)
    q = _unit_rows(torch.randn(T, Hqk, D, generator=gen)).to(dt)
    k = _unit_rows(torch.randn(T, Hqk, D, generator=gen)).to(dt)
    v = torch.randn(T, Hv, Dv, generator=gen).to(dt)
    beta = torch.sigmoid(torch.randn(T, Hv, generator=gen))
    g = -F.softplus(torch.randn(T, Hv, generator=gen) + g_mu)
    cu = torch.zeros(N + 1, dtype=torch.int32)
    if N:
        cu[1:] = torch.cumsum(torch.tensor(lengths, dtype=torch.int64), 0).to(torch.int32)
    s0 = None
    if init_std > 0:
        s0 = torch.randn(N, Hv, Dv, D, generator=gen) * init_std
    return {"q": q, "k": k, "v": v, "g": g.contiguous(), "beta": beta.contiguous(),
            "cu_seqlens": cu, "initial_state": s0}


def decode_inputs(batch, Hqk, Hv, D, steps=1, dtype="bf16", seed=0, init_std=0.02, Dv=None):
    """Decode inputs for ``steps`` consecutive single-token steps.  Returns CPU
    tensors q, k [steps, B, Hqk, D]; v [steps, B, Hv, Dv]; g, beta
    [steps, B, Hv] fp32; state [B, Hv, Dv, D] fp32."""
    Dv = D if Dv is None else Dv
    dt = DTYPES[dtype]
    gen = torch.Generator().manual_seed(seed)
    state = torch.randn(batch, Hv, Dv, D, generator=gen) * init_std
    q = _unit_rows(torch.randn(steps, batch, Hqk, D, generator=gen)).to(dt)
    k = _unit_rows(torch.randn(steps, batch, Hqk, D, generator=gen)).to(dt)
    v = torch.randn(steps, batch, Hv, Dv, generator=gen).to(dt)
    beta = torch.sigmoid(torch.randn(steps, batch, Hv, generator=gen))
    g = -F.softplus(torch.randn(steps, batch, Hv, generator=gen))
    return {"q": q, "k": k, "v": v, "g": g.contiguous(), "beta": beta.contiguous(),
            "state": state}


def workload_inputs(w: Workload):
    if w.batch:
        return decode_inputs(w.batch, w.Hqk, w.Hv, w.D, steps=w.steps, dtype=w.dtype,
                             seed=w.seed, init_std=w.init_std)
    return prefill_inputs(w.lengths, w.Hqk, w.Hv, w.D, dtype=w.dtype, seed=w.seed,
                          g_mu=w.g_mu, init_std=w.init_std)
