"""Seeded synthetic inputs for the WavePrune attention workloads.

This module only draws random numbers and fixes shapes. It holds none of the
method's arithmetic (no frequencies, cutoffs, rotations or attention), so both
the fp64 oracle and the CUDA library can be fed from it without sharing code.

Recipe (the same for every workload):
  * a CPU ``torch.Generator`` seeded with ``1000 + index`` (index = the 1-based
    position of the workload in ``WORKLOADS``);
  * fp32 N(0, 1) draws, rounded to bf16 with round-to-nearest-even;
  * the Qwen3-8B-shaped workload multiplies Q and K by per-head-dim scales drawn
    log-uniform in [0.5, 2] (one independent draw per dim index for Q and one
    for K, shared by all tokens and heads) before rounding;
  * decode lengths are drawn uniform in [Lmin, Lmax] (inclusive).

Q/K drawn here are the *pre-rotation* projections: the rotation is part of the
path under test.  A decode KV cache holds keys that a model would already have
rotated; an i.i.d. N(0, 1) vector rotated by any angle is again i.i.d. N(0, 1),
so the cache is drawn directly.

The shapes follow the pages' kernel benchmark setup (bf16, GQA 32 query heads /
8 KV heads, head dim 128, RoPE base 1e6, causal) of the WavePrune reading
notes, section 3.4 "系统实验与消融" and Table 11.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

INTERLEAVED = 0
HALF_SPLIT = 1


@dataclass(frozen=True)
class Workload:
    name: str
    kind: str                 # "prefill" or "decode"
    B: int
    Hq: int
    Hkv: int
    d: int
    theta: float
    layout: int
    N: int = 0                # prefill sequence length
    scale_all: float = 1.0    # uniform frequency scale (1/4 = position interpolation by 4)
    perdim_scale: bool = False
    Lmin: int = 0             # decode length range
    Lmax: int = 0
    sampled_rows: int = 0     # oracle rows per head for long contexts (0 = all rows)
    index: int = 0

    @property
    def seed(self) -> int:
        return 1000 + self.index


WORKLOADS = [
    Workload("tiny", "prefill", B=1, Hq=2, Hkv=2, d=64, theta=1e4, layout=INTERLEAVED, N=256, index=1),
    Workload("qwen3_8b_4k", "prefill", B=2, Hq=32, Hkv=8, d=128, theta=1e6, layout=HALF_SPLIT, N=4096,
             perdim_scale=True, index=2),
    Workload("long_32k", "prefill", B=1, Hq=32, Hkv=8, d=128, theta=1e6, layout=HALF_SPLIT, N=32768,
             sampled_rows=256, index=3),
    Workload("decode_32k", "decode", B=16, Hq=32, Hkv=8, d=128, theta=1e6, layout=HALF_SPLIT,
             Lmin=16384, Lmax=32768, index=4),
    Workload("scaled_128k", "prefill", B=1, Hq=32, Hkv=8, d=128, theta=1e6, layout=HALF_SPLIT, N=131072,
             scale_all=0.25, sampled_rows=128, index=5),
]
BY_NAME = {w.name: w for w in WORKLOADS}


def workload(name: str) -> Workload:
    return BY_NAME[name]


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    return g


def _normal_bf16(g: torch.Generator, shape, scale: torch.Tensor | None = None) -> torch.Tensor:
    x = torch.randn(shape, generator=g, dtype=torch.float32)
    if scale is not None:
        x.mul_(scale)
    return x.to(torch.bfloat16)


def _log_uniform(g: torch.Generator, n: int, lo: float, hi: float) -> torch.Tensor:
    u = torch.rand(n, generator=g, dtype=torch.float64)
    return torch.exp(math.log(lo) + u * (math.log(hi) - math.log(lo))).to(torch.float32)


def prefill_inputs(w: Workload, B: int | None = None, N: int | None = None, seed: int | None = None):
    """Pre-rotation bf16 Q [B,N,Hq,d], K [B,N,Hkv,d] and V [B,N,Hkv,d] on the CPU.

    ``B``/``N``/``seed`` override the workload's own values (used for small
    parity cases with the same distribution)."""
    B = w.B if B is None else B
    N = w.N if N is None else N
    g = _gen(w.seed if seed is None else seed)
    sq = sk = None
    if w.perdim_scale:
        sq = _log_uniform(g, w.d, 0.5, 2.0)
        sk = _log_uniform(g, w.d, 0.5, 2.0)
    q = _normal_bf16(g, (B, N, w.Hq, w.d), sq)
    k = _normal_bf16(g, (B, N, w.Hkv, w.d), sk)
    v = _normal_bf16(g, (B, N, w.Hkv, w.d))
    return q, k, v


def decode_inputs(w: Workload, B: int | None = None, Lmax: int | None = None, Lmin: int | None = None,
                  seed: int | None = None):
    """Decode inputs: pre-rotation query q [B,Hq,d] (bf16), KV caches
    [B,Hkv,Lmax,d] (bf16, keys already rotated) and lengths [B] (int32)."""
    B = w.B if B is None else B
    Lmax = w.Lmax if Lmax is None else Lmax
    Lmin = w.Lmin if Lmin is None else Lmin
    g = _gen(w.seed if seed is None else seed)
    lens = torch.randint(Lmin, Lmax + 1, (B,), generator=g, dtype=torch.int64).to(torch.int32)
    q = _normal_bf16(g, (B, w.Hq, w.d))
    kc = _normal_bf16(g, (B, w.Hkv, Lmax, w.d))
    vc = _normal_bf16(g, (B, w.Hkv, Lmax, w.d))
    return q, kc, vc, lens


def sample_rows(w: Workload, per_head: int, N: int | None = None, seed: int | None = None):
    """Sampled query rows for long contexts: ``per_head`` distinct row indices
    for every (batch, query head), drawn uniformly, plus the last row (the
    longest one) so the full key range is always exercised. Returns int64
    tensors (b, h, i), each of length B*Hq*per_head."""
    N = w.N if N is None else N
    g = _gen((w.seed if seed is None else seed) + 7919)
    bs, hs, is_ = [], [], []
    for b in range(w.B):
        for h in range(w.Hq):
            rows = torch.randperm(N, generator=g)[: per_head - 1]
            rows = torch.cat([rows, torch.tensor([N - 1])]).sort().values
            bs.append(torch.full_like(rows, b))
            hs.append(torch.full_like(rows, h))
            is_.append(rows)
    return torch.cat(bs), torch.cat(hs), torch.cat(is_)
