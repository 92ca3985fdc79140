"""Seeded synthetic inputs for the KDA recurrence.

This module only draws random numbers in the distributions the benchmark
workloads name; it holds none of the recurrence's arithmetic.  Both the CUDA
path (through its Python binding) and the fp64 oracle consume exactly the
tensors produced here.

Recipe (per (token, head) unless stated):
  q, k      ~ N(0, 1), L2-normalised over the head dimension in fp32, then
              rounded to the I/O dtype (bf16 round-to-nearest-even);
  v         ~ N(0, 1), rounded to the I/O dtype;
  log_alpha = -softplus(x + gate_shift), x ~ N(0, 1), per channel, fp32;
  beta      = sigmoid(N(0, 1)), fp32, one per (token, head);
  h0        ~ N(0, h0_std^2) fp32 (zeros when h0_std == 0);
  scale     = 1 / sqrt(dk).
"""
import math
from dataclasses import dataclass, field
from typing import List, Optional

import numpy as np
import torch


@dataclass
class PrefillConfig:
    name: str
    B: int
    T: int
    H: int
    dk: int
    dv: int
    io_dtype: str            # "f32" or "bf16"
    seed: int
    gate_shift: float = 0.0
    h0_std: float = 0.0
    lengths: Optional[List[int]] = None   # packed variable-length sequences (B must be 1)

    @property
    def N(self) -> int:
        return len(self.lengths) if self.lengths is not None else self.B

    @property
    def tokens(self) -> int:
        return self.B * self.T


@dataclass
class DecodeConfig:
    name: str
    N: int
    H: int
    dk: int
    dv: int
    steps: int
    seed: int
    io_dtype: str = "bf16"
    state_std: float = 0.02
    gate_shift: float = 0.0


def varlen_lengths(seed: int = 4, n: int = 16, total: int = 1 << 20,
                   lo: int = 2048, hi: int = 262144) -> List[int]:
    """n lengths drawn log-uniform in [lo, hi], rescaled to sum exactly to `total`.

    Draw u ~ U(ln lo, ln hi), L = round(e^u); rescale by total / sum(L); clip to
    [lo, hi]; then hand the integer residual to the unclipped sequences, largest
    first, repeating until the sum is exact.
    """
    rng = np.random.default_rng(seed)
    u = rng.uniform(math.log(lo), math.log(hi), size=n)
    L = np.round(np.exp(u)).astype(np.int64)
    L = np.round(L * (total / L.sum())).astype(np.int64)
    for _ in range(1000):
        L = np.clip(L, lo, hi)
        resid = int(total - L.sum())
        if resid == 0:
            break
        free = [i for i in np.argsort(-L) if (lo < L[i] < hi) or (resid > 0 and L[i] == lo)
                or (resid < 0 and L[i] == hi)]
        if not free:
            raise ValueError("cannot meet the requested total within [lo, hi]")
        share = resid // len(free) if abs(resid) >= len(free) else (1 if resid > 0 else -1)
        for i in free:
            if resid == 0:
                break
            step = share if abs(share) <= abs(resid) else resid
            L[i] += step
            resid -= step
    assert int(L.sum()) == total
    return [int(x) for x in L]


# The five benchmark workloads (shapes of Kimi Linear's KDA layers, H=32 and d=128
# where the workload is the full-size one).
TINY = PrefillConfig("tiny_fp32_B1_H2_T256_d64", 1, 256, 2, 64, 64, "f32", seed=0)
SINGLE = PrefillConfig("prefill_B1_H16_T4096_d128_bf16", 1, 4096, 16, 128, 128, "bf16",
                       seed=1, h0_std=0.02)
BATCHED = PrefillConfig("prefill_B8_H32_T8192_d128_bf16", 8, 8192, 32, 128, 128, "bf16",
                        seed=2, gate_shift=-2.0)
DECODE = DecodeConfig("decode_N256_H32_d128_bf16_x1000", 256, 32, 128, 128, 1000, seed=3)


def varlen_config() -> PrefillConfig:
    L = varlen_lengths()
    return PrefillConfig("varlen16_2p20tok_H32_d128_bf16", 1, sum(L), 32, 128, 128, "bf16",
                         seed=4, lengths=L)


def _tdtype(io_dtype: str):
    return {"f32": torch.float32, "bf16": torch.bfloat16}[io_dtype]


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _unit_rows(x: torch.Tensor) -> torch.Tensor:
    return x / x.norm(dim=-1, keepdim=True)


def _fill_normal(shape, gen, device, block=1 << 26):
    """N(0,1) fp32 of `shape`, drawn in slabs along the first axis to bound temporaries."""
    out = torch.empty(shape, dtype=torch.float32, device=device)
    if out.numel() == 0:
        return out
    flat = out.view(shape[0], -1)
    rows_per = max(1, block // max(1, flat.shape[1]))
    for r in range(0, flat.shape[0], rows_per):
        flat[r:r + rows_per].normal_(generator=gen)
    return out


def make_prefill(cfg: PrefillConfig, device="cpu") -> dict:
    """All inputs of one forward call for `cfg`, as torch tensors on `device`."""
    gen = _gen(cfg.seed, device)
    dt = _tdtype(cfg.io_dtype)
    B, T, H, dk, dv = cfg.B, cfg.T, cfg.H, cfg.dk, cfg.dv
    out = {}
    for name, d, unit in (("q", dk, True), ("k", dk, True), ("v", dv, False)):
        x = _fill_normal((B * T, H, d), gen, device)
        if unit:
            # normalise slab by slab to avoid a second full-size temporary
            for r in range(0, B * T, 1 << 16):
                x[r:r + (1 << 16)] = _unit_rows(x[r:r + (1 << 16)])
        out[name] = x.to(dt).view(B, T, H, d)
        del x
    x = _fill_normal((B * T, H, dk), gen, device)
    for r in range(0, B * T, 1 << 16):
        x[r:r + (1 << 16)] = -torch.nn.functional.softplus(x[r:r + (1 << 16)] + cfg.gate_shift)
    out["log_alpha"] = x.view(B, T, H, dk)
    out["beta"] = torch.sigmoid(torch.randn((B, T, H), generator=gen, device=device))
    N = cfg.N
    if cfg.h0_std > 0:
        out["h0"] = torch.randn((N, H, dk, dv), generator=gen, device=device) * cfg.h0_std
    else:
        out["h0"] = None
    if cfg.lengths is not None:
        cu = np.concatenate([[0], np.cumsum(cfg.lengths)]).astype(np.int32)
        out["cu_seqlens"] = torch.from_numpy(cu).to(device)
    else:
        out["cu_seqlens"] = None
    out["scale"] = 1.0 / math.sqrt(dk)
    return out


def make_decode_step(cfg: DecodeConfig, gen: torch.Generator, device="cpu") -> dict:
    """Inputs of one decode step (fresh q, k, v, gates for every sequence)."""
    dt = _tdtype(cfg.io_dtype)
    N, H, dk, dv = cfg.N, cfg.H, cfg.dk, cfg.dv
    q = _unit_rows(torch.randn((N, H, dk), generator=gen, device=device)).to(dt)
    k = _unit_rows(torch.randn((N, H, dk), generator=gen, device=device)).to(dt)
    v = torch.randn((N, H, dv), generator=gen, device=device).to(dt)
    g = -torch.nn.functional.softplus(
        torch.randn((N, H, dk), generator=gen, device=device) + cfg.gate_shift)
    b = torch.sigmoid(torch.randn((N, H), generator=gen, device=device))
    return {"q": q, "k": k, "v": v, "log_alpha": g, "beta": b}


def make_decode_state(cfg: DecodeConfig, gen: torch.Generator, device="cpu") -> torch.Tensor:
    return torch.randn((cfg.N, cfg.H, cfg.dk, cfg.dv), generator=gen, device=device) * cfg.state_std


def decode_generator(cfg: DecodeConfig, device="cpu") -> torch.Generator:
    return _gen(cfg.seed, device)


def small_prefill(B=1, T=200, H=2, dk=64, dv=64, io_dtype="f32", seed=0, gate_shift=0.0,
                  h0_std=0.0, lengths=None) -> PrefillConfig:
    """A parity-test-sized workload with the same distributions."""
    if lengths is not None:
        B, T = 1, int(sum(lengths))
    return PrefillConfig(f"small_B{B}_T{T}_H{H}_dk{dk}_dv{dv}_{io_dtype}", B, T, H, dk, dv,
                         io_dtype, seed, gate_shift, h0_std, lengths)


def scalar_gates(B: int, T: int, H: int, seed: int, gate_shift: float = 0.0,
                 device="cpu") -> torch.Tensor:
    """Gated DeltaNet gates: log a = -softplus(N(0,1) + gate_shift), one per (token, head)."""
    gen = _gen(seed + 1000, device)
    x = torch.randn((B, T, H), generator=gen, device=device)
    return -torch.nn.functional.softplus(x + gate_shift)
