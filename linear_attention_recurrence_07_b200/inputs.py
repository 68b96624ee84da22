"""Seeded synthetic inputs for the Gated DeltaNet token mixer.

This module only draws random numbers and lays them out; it holds none of the
method's arithmetic, so both the CUDA library's tests and the CPU oracle can
be fed from it.  The shapes follow the model described in "Qwen3.8-Flash-Next
技术总结 -- Qwen4 架构的探路者", section 2.1 "Gated DeltaNet" (48 V heads sharing
16 QK heads, head dim 128) and section 一 (native context 262,144 tokens).

Recipe (one torch generator per call, seeded, drawn in this order):
  q, k  ~ N(0, 1), then divided by their L2 norm over the head dimension (in
          fp32, before the cast to the storage dtype)
  v     ~ N(0, 1)
  alpha = exp(U(lo, hi))                      (forget gate in (0, 1))
  beta  = sigmoid(N(0, 1))                    (write strength)
  S0    ~ N(0, s0_std) in fp32, or None when s0_std == 0
"""
from dataclasses import dataclass, field
from typing import Optional

import torch


@dataclass(frozen=True)
class Workload:
    """One synthetic workload: shapes, dtypes and the input distributions."""
    name: str
    B: int
    T: int
    Hqk: int
    Hv: int
    dk: int = 128
    dv: int = 128
    dtype: torch.dtype = torch.bfloat16       # dtype of q, k, v and o
    log_alpha: tuple = (-0.1, -0.001)         # U(lo, hi) for log alpha
    s0_std: float = 0.0                       # std of the initial state; 0 -> S0 = None
    seed: int = 20260
    chunk: int = 64
    decode_steps: int = 0                     # > 0: a decode workload of this many steps
    extra: dict = field(default_factory=dict)

    @property
    def tokens(self) -> int:
        return self.B * self.T


# The workloads the library is checked and measured on.
PREFILL_SMALL_FP32 = Workload("gdn_prefill_small_fp32", B=1, T=256, Hqk=2, Hv=6,
                              dtype=torch.float32, seed=20260)
PREFILL_4K = Workload("gdn_prefill_B1_T4096", B=1, T=4096, Hqk=16, Hv=48, seed=20261)
PREFILL_BATCH8_8K = Workload("gdn_prefill_B8_T8192_S0", B=8, T=8192, Hqk=16, Hv=48,
                             s0_std=0.02, seed=20262)
PREFILL_256K = Workload("gdn_prefill_B1_T262144", B=1, T=262144, Hqk=16, Hv=48,
                        log_alpha=(-0.02, -0.0005), seed=20263)
DECODE_B256 = Workload("gdn_decode_B256", B=256, T=1, Hqk=16, Hv=48, s0_std=0.02,
                       seed=20264, decode_steps=1000)
# Multi-token decode (draft verification): 4 tokens for each of 256 sequences, with
# the state after every token kept.
VERIFY_B256_N4 = Workload("gdn_verify_B256_n4", B=256, T=4, Hqk=16, Hv=48, s0_std=0.02,
                          seed=20265)

# Packed prefill of 24 sequences of mixed lengths (64 .. 8192 tokens, seeded),
# continuous batching of prompts; extra: lengths drawn by varlen_lengths.
PREFILL_VARLEN = Workload("gdn_prefill_varlen_N24", B=24, T=0, Hqk=16, Hv=48, s0_std=0.02,
                          seed=20266, extra={"lo": 64, "hi": 8192})

WORKLOADS = {w.name: w for w in (PREFILL_SMALL_FP32, PREFILL_4K, PREFILL_BATCH8_8K,
                                  PREFILL_256K, DECODE_B256, VERIFY_B256_N4, PREFILL_VARLEN)}


def _generator(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _unit_rows(shape, g, device, dtype):
    x = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    x = x / x.norm(dim=-1, keepdim=True)
    return x.to(dtype)


def prefill_inputs(B: int, T: int, Hqk: int, Hv: int, dk: int = 128, dv: int = 128,
                   dtype=torch.bfloat16, log_alpha=(-0.1, -0.001), s0_std: float = 0.0,
                   seed: int = 0, device="cpu"):
    """Returns dict(q, k, v, alpha, beta, S0) in the library's layouts:
    q, k [B, T, Hqk, dk] and v [B, T, Hv, dv] in ``dtype``; alpha, beta
    [B, T, Hv] fp32; S0 [B, Hv, dk, dv] fp32 or None."""
    g = _generator(device, seed)
    q = _unit_rows((B, T, Hqk, dk), g, device, dtype)
    k = _unit_rows((B, T, Hqk, dk), g, device, dtype)
    v = torch.randn((B, T, Hv, dv), generator=g, device=device, dtype=torch.float32).to(dtype)
    lo, hi = log_alpha
    la = torch.rand((B, T, Hv), generator=g, device=device, dtype=torch.float32) * (hi - lo) + lo
    alpha = torch.exp(la)
    beta = torch.sigmoid(torch.randn((B, T, Hv), generator=g, device=device, dtype=torch.float32))
    S0 = None
    if s0_std > 0:
        S0 = torch.randn((B, Hv, dk, dv), generator=g, device=device, dtype=torch.float32) * s0_std
    return dict(q=q.contiguous(), k=k.contiguous(), v=v.contiguous(),
                alpha=alpha.contiguous(), beta=beta.contiguous(), S0=S0)


def workload_inputs(w: Workload, device="cpu", T: Optional[int] = None, B: Optional[int] = None):
    """Prefill inputs of workload ``w`` (optionally with a shorter T or B, same seed)."""
    return prefill_inputs(B if B is not None else w.B, T if T is not None else w.T,
                          w.Hqk, w.Hv, w.dk, w.dv, w.dtype, w.log_alpha, w.s0_std,
                          w.seed, device)


def decode_state(w: Workload, device="cpu", B: Optional[int] = None):
    """Initial recurrent state [B, Hv, dk, dv] fp32 ~ N(0, s0_std) for a decode workload."""
    B = B if B is not None else w.B
    g = _generator(device, w.seed)
    return torch.randn((B, w.Hv, w.dk, w.dv), generator=g, device=device,
                       dtype=torch.float32) * w.s0_std


def decode_inputs(w: Workload, step: int, device="cpu", B: Optional[int] = None):
    """Token inputs of decode step ``step``: q, k [B, Hqk, dk], v [B, Hv, dv] in
    ``w.dtype``; alpha, beta [B, Hv] fp32.  Seed = w.seed + 1 + step."""
    B = B if B is not None else w.B
    d = prefill_inputs(B, 1, w.Hqk, w.Hv, w.dk, w.dv, w.dtype, w.log_alpha, 0.0,
                       w.seed + 1 + step, device)
    return dict(q=d["q"][:, 0].contiguous(), k=d["k"][:, 0].contiguous(),
                v=d["v"][:, 0].contiguous(), alpha=d["alpha"][:, 0].contiguous(),
                beta=d["beta"][:, 0].contiguous())


def varlen_lengths(n: int, lo: int, hi: int, seed: int):
    """n sequence lengths, uniform integers in [lo, hi] (seeded, CPU generator)."""
    g = torch.Generator().manual_seed(seed)
    return torch.randint(lo, hi + 1, (n,), generator=g).tolist()


def varlen_inputs(lengths, Hqk: int, Hv: int, dk: int = 128, dv: int = 128,
                  dtype=torch.bfloat16, log_alpha=(-0.1, -0.001), s0_std: float = 0.0,
                  seed: int = 0, device="cpu"):
    """Packed prefill inputs: q, k [T_total, Hqk, dk], v [T_total, Hv, dv], alpha,
    beta [T_total, Hv], S0 [N, Hv, dk, dv] or None, cu_seqlens [N + 1] int32, for
    sequences of the given lengths laid out back to back."""
    T = int(sum(lengths))
    d = prefill_inputs(1, max(T, 1), Hqk, Hv, dk, dv, dtype, log_alpha, 0.0, seed, device)
    out = {key: d[key][0, :T].contiguous() for key in ("q", "k", "v", "alpha", "beta")}
    g = _generator(device, seed + 1)
    out["S0"] = (torch.randn((len(lengths), Hv, dk, dv), generator=g, device=device,
                             dtype=torch.float32) * s0_std) if s0_std > 0 else None
    cu = torch.zeros(len(lengths) + 1, dtype=torch.int32)
    cu[1:] = torch.cumsum(torch.tensor(lengths, dtype=torch.int64), 0).to(torch.int32)
    out["cu_seqlens"] = cu.to(device)
    return out


def varlen_workload_inputs(w: Workload, device="cpu"):
    """Inputs of a packed-prefill workload (lengths from w.extra, seeded)."""
    lengths = varlen_lengths(w.B, w.extra["lo"], w.extra["hi"], w.seed)
    return varlen_inputs(lengths, w.Hqk, w.Hv, w.dk, w.dv, w.dtype, w.log_alpha, w.s0_std,
                         w.seed, device)
