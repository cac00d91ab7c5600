"""Seeded synthetic inputs for the KDA recurrence.

This module is the only code that the CUDA path and the CPU oracle have in
common. It draws random tensors and shapes them like the workloads the Kimi
Linear pages discuss (long contexts at H=32 heads of width 128, a large decode
batch, variable-length packing); it holds none of the recurrence's arithmetic.

Recipe for every preset (all draws from one ``torch.Generator`` seeded per
preset, in the fixed order q, k, v, beta, log_alpha, S0):
  * q, k ~ N(0, 1), then L2-normalised per (token, head) in fp32, then cast to
    the preset's dtype (the kernels do not normalise; after a bf16 cast the norm
    is 1 only to bf16 precision, and the oracle reads the same rounded values);
  * v ~ N(0, 1), cast to the preset's dtype;
  * beta = sigmoid(N(0, 1)) in fp32, one per (token, head);
  * log_alpha = -softplus(N(0, 1) + shift) in fp32, one per (token, head, key
    channel); shift 0 (fast decay), -2 (medium) or -3 (slow);
  * S0 ~ N(0, std) in fp32 (std 0.01 for prefill, 0.05 for the decode state) or
    absent (zero state).
"""
from __future__ import annotations

from dataclasses import dataclass

import torch


@dataclass(frozen=True)
class Preset:
    name: str
    B: int
    T: int
    H: int
    d: int
    dtype: torch.dtype
    gate_shift: float
    s0_std: float          # 0.0 means no S0 (zero state)
    seed: int
    n_varlen: int = 0      # >0: this many packed sequences (B must be 1)
    varlen_min: int = 0
    varlen_max: int = 0

    @property
    def scale(self) -> float:
        return self.d ** -0.5


# Named workloads. "tiny" is small enough for the oracle to finish in
# milliseconds; the others are the full-size prefill/decode workloads.
TINY = Preset("tiny_fp32_B1_H2_T64_d32", 1, 64, 2, 32, torch.float32, 0.0, 0.0, 1)
CHUNKED = Preset("chunked_bf16_B4_H16_T4096_d128", 4, 4096, 16, 128, torch.bfloat16,
                 -2.0, 0.01, 2)
LONG = Preset("long_bf16_B1_H32_T131072_d128", 1, 131072, 32, 128, torch.bfloat16,
              -3.0, 0.0, 3)
VARLEN = Preset("varlen_bf16_N8_H32_d128", 1, 0, 32, 128, torch.bfloat16, -2.0, 0.01, 5,
                n_varlen=8, varlen_min=1024, varlen_max=65536)


@dataclass(frozen=True)
class DecodePreset:
    name: str
    N: int
    H: int
    d: int
    dtype: torch.dtype
    gate_shift: float
    s_std: float
    seed: int
    steps: int
    step_seed0: int

    @property
    def scale(self) -> float:
        return self.d ** -0.5


DECODE = DecodePreset("decode_bf16_N256_H32_d128", 256, 32, 128, torch.bfloat16, -2.0,
                      0.05, 4, 1000, 4000)

PRESETS = {p.name: p for p in (TINY, CHUNKED, LONG, VARLEN)}


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def _unit(x: torch.Tensor) -> torch.Tensor:
    return x / x.norm(dim=-1, keepdim=True).clamp_min(1e-6)


def varlen_lengths(n: int, lo: int, hi: int, seed: int) -> list[int]:
    """n sequence lengths drawn uniformly from [lo, hi] (inclusive)."""
    g = _gen(seed, "cpu")
    return [int(x) for x in torch.randint(lo, hi + 1, (n,), generator=g)]


def cu_seqlens_from_lengths(lengths) -> torch.Tensor:
    cu = [0]
    for n in lengths:
        cu.append(cu[-1] + int(n))
    return torch.tensor(cu, dtype=torch.int32)


def make_prefill(B: int, T: int, H: int, d: int, dtype=torch.bfloat16, gate_shift=0.0,
                 s0_std=0.0, seed=0, lengths=None, device="cpu", dv: int | None = None):
    """Draw one prefill problem. With ``lengths`` the tokens are packed into a
    single [1, sum(lengths), H, d] batch and ``cu_seqlens`` is returned.

    Returns a dict with q, k, v, log_alpha, beta, S0 (or None), cu_seqlens (or
    None) and scale.
    """
    dv = d if dv is None else dv
    g = _gen(seed, device)
    if lengths is not None:
        B, T = 1, int(sum(lengths))
        n_seq = len(lengths)
        cu = cu_seqlens_from_lengths(lengths)
    else:
        n_seq, cu = B, None
    f32 = dict(device=device, dtype=torch.float32)
    q = _unit(torch.randn(B, T, H, d, generator=g, **f32)).to(dtype)
    k = _unit(torch.randn(B, T, H, d, generator=g, **f32)).to(dtype)
    v = torch.randn(B, T, H, dv, generator=g, **f32).to(dtype)
    beta = torch.sigmoid(torch.randn(B, T, H, generator=g, **f32))
    log_alpha = -torch.nn.functional.softplus(
        torch.randn(B, T, H, d, generator=g, **f32) + gate_shift)
    S0 = (torch.randn(n_seq, H, d, dv, generator=g, **f32) * s0_std) if s0_std > 0 else None
    return dict(q=q, k=k, v=v, log_alpha=log_alpha, beta=beta, S0=S0,
                cu_seqlens=None if cu is None else cu.to(device), scale=d ** -0.5)


def make_preset(p: Preset, device="cpu"):
    """Draw the full problem of a named prefill preset."""
    lengths = None
    if p.n_varlen:
        lengths = varlen_lengths(p.n_varlen, p.varlen_min, p.varlen_max, p.seed)
    return make_prefill(p.B, p.T, p.H, p.d, p.dtype, p.gate_shift, p.s0_std, p.seed,
                        lengths=lengths, device=device)


def make_decode_state(N: int, H: int, d: int, std: float, seed: int, device="cpu",
                      dv: int | None = None) -> torch.Tensor:
    """The recurrent state S [N, H, d, dv] ~ N(0, std) in fp32."""
    dv = d if dv is None else dv
    g = _gen(seed, device)
    return torch.randn(N, H, d, dv, generator=g, device=device, dtype=torch.float32) * std


def make_decode_token(N: int, H: int, d: int, dtype=torch.bfloat16, gate_shift=-2.0,
                      seed=0, device="cpu", dv: int | None = None):
    """One decode token for each of N sequences: q, k, log_alpha [N,H,d];
    v [N,H,dv]; beta [N,H]."""
    dv = d if dv is None else dv
    g = _gen(seed, device)
    f32 = dict(device=device, dtype=torch.float32)
    q = _unit(torch.randn(N, H, d, generator=g, **f32)).to(dtype)
    k = _unit(torch.randn(N, H, d, generator=g, **f32)).to(dtype)
    v = torch.randn(N, H, dv, generator=g, **f32).to(dtype)
    beta = torch.sigmoid(torch.randn(N, H, generator=g, **f32))
    log_alpha = -torch.nn.functional.softplus(torch.randn(N, H, d, generator=g, **f32)
                                              + gate_shift)
    return dict(q=q, k=k, v=v, log_alpha=log_alpha, beta=beta)
