"""Seeded synthetic inputs for KDA prefill and decode workloads.

This module only draws and shapes random tensors; it contains none of the
method's arithmetic. Both the CUDA path's tests and the CPU oracle take their
inputs from here.

Every (batch, head) slice of a prefill workload, every head of a decode state
and every decode step has its own torch CPU generator, seeded from the
workload seed and the slice index. Any slice can therefore be regenerated on
its own, bit-identical to what the full tensor holds, which lets tests check
sampled heads of full-size runs against the oracle.

Distributions (per token, per head):
  q, k  ~ N(0, 1), then L2-normalised over the key dimension (in fp32)
  v     ~ N(0, 1)
  beta  = sigmoid(N(0, 1))
  log_alpha = -U(lo, hi), per key channel
  S0    ~ N(0, s0_std) fp32 (second parameter read as a standard deviation)
bf16 workloads round q, k, v, log_alpha and beta to bf16 after drawing them.
"""
from __future__ import annotations

import dataclasses

import torch


@dataclasses.dataclass(frozen=True)
class PrefillConfig:
    name: str
    B: int
    H: int
    T: int
    dk: int
    dv: int
    C: int
    dtype: str          # "f32" or "bf16": dtype of q, k, v, log_alpha, beta, o
    la_lo: float        # log_alpha = -U(la_lo, la_hi)
    la_hi: float
    s0_std: float       # 0 => S0 = 0
    seed: int

    def replace(self, **kw) -> "PrefillConfig":
        return dataclasses.replace(self, **kw)

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16


@dataclasses.dataclass(frozen=True)
class DecodeConfig:
    name: str
    N: int
    H: int
    dk: int
    dv: int
    steps: int
    dtype: str
    la_lo: float
    la_hi: float
    s_std: float
    seed: int

    def replace(self, **kw) -> "DecodeConfig":
        return dataclasses.replace(self, **kw)

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16


# The five workloads of this path.
SMALL_F32 = PrefillConfig("prefill_b1_h1_t256_d64_f32", 1, 1, 256, 64, 64, 64, "f32", 0.001, 0.1, 0.0, 0)
B2_H16_T4K = PrefillConfig("prefill_b2_h16_t4096_d128_bf16", 2, 16, 4096, 128, 128, 64, "bf16", 0.001, 0.1, 0.01, 1)
B4_H32_T8K = PrefillConfig("prefill_b4_h32_t8192_d128_bf16_strong_decay", 4, 32, 8192, 128, 128, 64, "bf16",
                           0.01, 1.0, 0.0, 2)
B1_H32_T128K = PrefillConfig("prefill_b1_h32_t131072_d128_bf16", 1, 32, 131072, 128, 128, 64, "bf16",
                             0.0001, 0.05, 0.0, 3)
DECODE_N256_H32 = DecodeConfig("decode_n256_h32_d128_bf16_1000_steps", 256, 32, 128, 128, 1000, "bf16",
                               0.001, 0.1, 0.1, 4)

PREFILL_CONFIGS = [SMALL_F32, B2_H16_T4K, B4_H32_T8K, B1_H32_T128K]


def _gen(*key: int) -> torch.Generator:
    s = 0x9E3779B97F4A7C15
    for x in key:
        s = (s * 6364136223846793005 + (int(x) & 0xFFFFFFFF) + 1442695040888963407) & 0xFFFFFFFFFFFFFFFF
    g = torch.Generator(device="cpu")
    g.manual_seed(s & 0x7FFFFFFFFFFFFFFF)
    return g


def _unit(x: torch.Tensor) -> torch.Tensor:
    return x / x.norm(dim=-1, keepdim=True).clamp_min(1e-30)


def prefill_head(cfg: PrefillConfig, b: int, h: int) -> dict:
    """Inputs of one (b, h) slice: q,k,log_alpha [T,dk], v [T,dv], beta [T]
    in cfg's dtype, and S0 [dk,dv] fp32 (zeros when s0_std == 0)."""
    g = _gen(cfg.seed, 1, b, h)
    T, dk, dv = cfg.T, cfg.dk, cfg.dv
    q = _unit(torch.randn(T, dk, generator=g))
    k = _unit(torch.randn(T, dk, generator=g))
    v = torch.randn(T, dv, generator=g)
    la = -(cfg.la_lo + (cfg.la_hi - cfg.la_lo) * torch.rand(T, dk, generator=g))
    beta = torch.sigmoid(torch.randn(T, generator=g))
    if cfg.s0_std > 0:
        S0 = cfg.s0_std * torch.randn(dk, dv, generator=g)
    else:
        S0 = torch.zeros(dk, dv)
    dt = cfg.torch_dtype
    return dict(q=q.to(dt), k=k.to(dt), v=v.to(dt), log_alpha=la.to(dt), beta=beta.to(dt), S0=S0)


def prefill_inputs(cfg: PrefillConfig, heads=None) -> dict:
    """Full prefill inputs on the CPU: q,k,log_alpha [B,T,H,dk], v [B,T,H,dv],
    beta [B,T,H] in cfg's dtype, S0 [B,H,dk,dv] fp32 (or None when zero).

    With heads = [(b, h), ...] the result holds only those slices, stacked as
    a batch of single-head sequences: shapes [n,T,1,*] and S0 [n,1,dk,dv]."""
    dt = cfg.torch_dtype
    if heads is None:
        heads_ = [(b, h) for b in range(cfg.B) for h in range(cfg.H)]
        Bo, Ho = cfg.B, cfg.H
    else:
        heads_ = list(heads)
        Bo, Ho = len(heads_), 1
    T, dk, dv = cfg.T, cfg.dk, cfg.dv
    q = torch.empty(Bo, T, Ho, dk, dtype=dt)
    k = torch.empty(Bo, T, Ho, dk, dtype=dt)
    la = torch.empty(Bo, T, Ho, dk, dtype=dt)
    v = torch.empty(Bo, T, Ho, dv, dtype=dt)
    beta = torch.empty(Bo, T, Ho, dtype=dt)
    S0 = torch.zeros(Bo, Ho, dk, dv)
    for i, (b, h) in enumerate(heads_):
        bo, ho = (b, h) if heads is None else (i, 0)
        x = prefill_head(cfg, b, h)
        q[bo, :, ho] = x["q"]
        k[bo, :, ho] = x["k"]
        la[bo, :, ho] = x["log_alpha"]
        v[bo, :, ho] = x["v"]
        beta[bo, :, ho] = x["beta"]
        S0[bo, ho] = x["S0"]
    return dict(q=q, k=k, v=v, log_alpha=la, beta=beta, S0=S0 if cfg.s0_std > 0 else None)


def decode_state(cfg: DecodeConfig, heads=None) -> torch.Tensor:
    """Initial decode state S [N,H,dk,dv] fp32, or [n,1,dk,dv] for the listed
    (n, h) heads."""
    if heads is None:
        g = _gen(cfg.seed, 2)
        return cfg.s_std * torch.randn(cfg.N, cfg.H, cfg.dk, cfg.dv, generator=g)
    full = decode_state(cfg)
    return torch.stack([full[n, h] for (n, h) in heads]).unsqueeze(1)


def decode_step_inputs(cfg: DecodeConfig, step: int) -> dict:
    """Inputs of one decode step: q,k,log_alpha [N,H,dk], v [N,H,dv], beta [N,H]."""
    g = _gen(cfg.seed, 3, step)
    N, H, dk, dv = cfg.N, cfg.H, cfg.dk, cfg.dv
    q = _unit(torch.randn(N, H, dk, generator=g))
    k = _unit(torch.randn(N, H, dk, generator=g))
    v = torch.randn(N, H, dv, generator=g)
    la = -(cfg.la_lo + (cfg.la_hi - cfg.la_lo) * torch.rand(N, H, dk, generator=g))
    beta = torch.sigmoid(torch.randn(N, H, generator=g))
    dt = cfg.torch_dtype
    return dict(q=q.to(dt), k=k.to(dt), v=v.to(dt), log_alpha=la.to(dt), beta=beta.to(dt))


def varlen_lengths(n: int, mean: int, seed: int, zero_frac: float = 0.0) -> list:
    """A seeded length mix for packed batches: lengths ~ U(1, 2*mean - 1),
    with about `zero_frac` of them set to 0 (empty sequences)."""
    g = _gen(seed, 7)
    ls = torch.randint(1, 2 * mean, (n,), generator=g)
    z = torch.rand(n, generator=g) < zero_frac
    return [0 if zz else int(x) for x, zz in zip(ls.tolist(), z.tolist())]


def varlen_inputs(cfg: PrefillConfig, lengths) -> dict:
    """Packed inputs for sequences of the given lengths: sequence n, head h is
    prefill_head(cfg with T = lengths[n], n, h). Shapes: q,k,log_alpha
    [total_T,H,dk], v [total_T,H,dv], beta [total_T,H], S0 [N,H,dk,dv] fp32
    (None when s0_std == 0), cu_seqlens int32 [N+1]."""
    lengths = [int(x) for x in lengths]
    N, H, dk, dv, dt = len(lengths), cfg.H, cfg.dk, cfg.dv, cfg.torch_dtype
    cu = [0]
    for L in lengths:
        cu.append(cu[-1] + L)
    TT = cu[-1]
    q = torch.empty(TT, H, dk, dtype=dt)
    k = torch.empty(TT, H, dk, dtype=dt)
    la = torch.empty(TT, H, dk, dtype=dt)
    v = torch.empty(TT, H, dv, dtype=dt)
    beta = torch.empty(TT, H, dtype=dt)
    S0 = torch.zeros(N, H, dk, dv)
    for n, L in enumerate(lengths):
        cn = cfg.replace(T=L)
        for h in range(H):
            x = prefill_head(cn, n, h)
            a, b = cu[n], cu[n + 1]
            q[a:b, h], k[a:b, h], la[a:b, h] = x["q"], x["k"], x["log_alpha"]
            v[a:b, h], beta[a:b, h] = x["v"], x["beta"]
            S0[n, h] = x["S0"]
    return dict(q=q, k=k, v=v, log_alpha=la, beta=beta, S0=S0 if cfg.s0_std > 0 else None,
                cu_seqlens=torch.tensor(cu, dtype=torch.int32))


def bwd_cotangents(cfg: PrefillConfig, with_dST: bool = True) -> dict:
    """Seeded upstream gradients for a backward pass over cfg's prefill:
    dO ~ N(0, 1) [B,T,H,dv] in cfg's dtype, dS_T ~ N(0, 1) fp32 [B,H,dk,dv]
    (None without it)."""
    g = _gen(cfg.seed, 9)
    dO = torch.randn(cfg.B, cfg.T, cfg.H, cfg.dv, generator=g).to(cfg.torch_dtype)
    dST = torch.randn(cfg.B, cfg.H, cfg.dk, cfg.dv, generator=g) if with_dST else None
    return {"dO": dO, "dST": dST}
