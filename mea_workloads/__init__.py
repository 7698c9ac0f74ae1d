"""Seeded synthetic inputs for memory-efficient attention — shared by tests and bench.

This module only draws random inputs and segment lengths; it holds none of the attention
arithmetic. Both the CUDA path's tests/bench and the CPU oracle consume what it produces.

Workloads (shapes from the pages; values synthetic, ~N(0, 1); seed = 1000 + workload index):

0. packed varlen: seqlens [37, 120, 8, 200] (365 tokens), 8 heads, D=64, fp16, scale 1/8,
   non-causal and causal — the packed example of the 7minutos page, section 4.
1. GQA BMGHK: B=2, M=256, G=2 KV heads, 4 query heads per group, D=64, fp16, scale 1/8 — the
   grouped example of the same page, section 5 (viewed packed as 2 segments of 256 tokens).
2. packed causal GQA + ALiBi: bf16, 32 query / 8 KV heads, D=128, segment lengths drawn
   U[64, 4096] until the sum reaches 32768, the last one truncated so the total is exactly 32768,
   ALiBi slopes 2^(-8(h+1)/32), scale 1/sqrt(128).
3. long causal prefill: bf16, one segment of 16384 tokens, 64 query / 8 KV heads, D=128, no ALiBi.
4. split-KV decode: bf16, 64 requests x 1 query token, KV lengths U[512, 32768], 64 query / 8 KV
   heads, D=128, causal (all keys visible to the newest token).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import List, Optional

import numpy as np
import torch


@dataclass
class Workload:
    index: int
    name: str
    dtype: torch.dtype
    n_heads_q: int
    n_heads_kv: int
    head_dim: int
    seqlens_q: List[int]
    seqlens_k: List[int]
    causal_passes: List[bool]
    alibi: bool
    scale: float
    decode: bool = False
    extra: dict = field(default_factory=dict)

    @property
    def seed(self) -> int:
        return 1000 + self.index

    @property
    def total_q(self) -> int:
        return int(sum(self.seqlens_q))

    @property
    def total_k(self) -> int:
        return int(sum(self.seqlens_k))


def cu_seqlens(seqlens) -> torch.Tensor:
    """Prefix sums [0, l0, l0+l1, ...] as int32 (host tensor)."""
    out = torch.zeros(len(seqlens) + 1, dtype=torch.int32)
    if len(seqlens):
        out[1:] = torch.cumsum(torch.tensor(list(seqlens), dtype=torch.int64), 0).to(torch.int32)
    return out


def packed_segment_lengths(seed: int, lo: int = 64, hi: int = 4096, total: int = 32768):
    """Integers U[lo, hi] (inclusive) drawn until their sum reaches `total`; the last one is cut
    so that the lengths sum to exactly `total` (it may end up shorter than `lo`)."""
    rng = np.random.default_rng(seed)
    out, acc = [], 0
    while acc < total:
        x = int(rng.integers(lo, hi, endpoint=True))
        x = min(x, total - acc)
        out.append(x)
        acc += x
    return out


def decode_kv_lengths(seed: int, n: int = 64, lo: int = 512, hi: int = 32768):
    rng = np.random.default_rng(seed)
    return [int(x) for x in rng.integers(lo, hi, size=n, endpoint=True)]


def alibi_slope_values(n_heads: int) -> torch.Tensor:
    """The workloads' ALiBi slopes 2^(-8(h+1)/H), h = 0..H-1, as fp32 inputs."""
    return torch.tensor([2.0 ** (-8.0 * (h + 1) / n_heads) for h in range(n_heads)],
                        dtype=torch.float32)


def workload(index: int) -> Workload:
    if index == 0:
        s = [37, 120, 8, 200]
        return Workload(0, "packed varlen [37,120,8,200] x 8 heads, D=64, fp16", torch.float16,
                        8, 8, 64, s, s, [False, True], False, 1.0 / 8.0)
    if index == 1:
        s = [256, 256]
        return Workload(1, "GQA BMGHK B=2 M=256 G=2 Hq=4 D=64, fp16", torch.float16,
                        8, 2, 64, s, s, [False, True], False, 1.0 / 8.0,
                        extra={"bmghk": (2, 256, 2, 4, 64)})
    if index == 2:
        s = packed_segment_lengths(1002)
        return Workload(2, "packed causal GQA 32/8 + ALiBi, D=128, bf16, U[64,4096] -> 32768",
                        torch.bfloat16, 32, 8, 128, s, s, [True], True, 1.0 / math.sqrt(128))
    if index == 3:
        s = [16384]
        return Workload(3, "causal prefill 16384 tokens, GQA 64/8, D=128, bf16", torch.bfloat16,
                        64, 8, 128, s, s, [True], False, 1.0 / math.sqrt(128))
    if index == 4:
        lk = decode_kv_lengths(1004)
        return Workload(4, "split-KV decode 64 x 1 token, KV U[512,32768], GQA 64/8, D=128, bf16",
                        torch.bfloat16, 64, 8, 128, [1] * len(lk), lk, [True], False,
                        1.0 / math.sqrt(128), decode=True)
    raise ValueError(f"no workload {index}")


def randn(shape, seed: int, dtype: torch.dtype, device="cpu") -> torch.Tensor:
    """~N(0,1) values drawn in fp32 from a seeded generator, then cast to `dtype`."""
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return torch.randn(shape, generator=g, dtype=torch.float32, device=device).to(dtype)


def make_qkv(seqlens_q, seqlens_k, n_heads_q, n_heads_kv, head_dim, dtype, seed: int,
             device="cpu"):
    """Packed q [T_q, Hq, D], k/v [T_k, Hkv, D] from one seed (three derived streams)."""
    tq, tk = int(sum(seqlens_q)), int(sum(seqlens_k))
    q = randn((tq, n_heads_q, head_dim), seed * 3 + 0, dtype, device)
    k = randn((tk, n_heads_kv, head_dim), seed * 3 + 1, dtype, device)
    v = randn((tk, n_heads_kv, head_dim), seed * 3 + 2, dtype, device)
    return q, k, v


def sample_rows(seed: int, n: int, n_heads: int, total: int, must_tokens=()):
    """A seeded sample of (head, token) pairs; every token in `must_tokens` appears once."""
    rng = np.random.default_rng(seed + 7)
    rows = [(int(rng.integers(0, n_heads)), int(t)) for t in must_tokens if 0 <= t < total]
    while len(rows) < n:
        rows.append((int(rng.integers(0, n_heads)), int(rng.integers(0, total))))
    return rows
