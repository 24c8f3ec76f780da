"""Seeded synthetic inputs for varlen attention: sequence lengths, cumulative
offsets and bf16 N(0,1) tensors.

This module holds no attention arithmetic. It is the one piece shared by the
oracle tests, the GPU parity tests and the benchmark, so that every side sees
the same bytes. Everything here is numpy; tensors are returned as raw bf16
bit patterns (``uint16``) so that no consumer has to trust a conversion it did
not make itself.

Workload shapes follow the pages:
  * "Mecanismo cu_seqlens en FlashAttention", section "Ejemplo de uso con
    PyTorch": two sequences, cu_seqlens_q = [0, 200, 1024],
    cu_seqlens_k = [0, 300, 1024], 12 heads, head_dim 64, scale 1/8.
  * "FlashAttention-2 GPU work partitioning", section "Qué significa la mejora
    de aproximadamente dos veces": 16k tokens per batch, sequence lengths from
    512 to about 16k, head dims 64 and 128, causal and non-causal.
"""
from __future__ import annotations

from dataclasses import dataclass, field
import math

import numpy as np

TOTAL_TOKENS = 16384


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to bf16 with round-to-nearest-even; returns uint16 bits.

    Inputs are finite N(0,1) draws, so no NaN handling is needed.
    """
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    rounding = ((b >> 16) & 1) + np.uint32(0x7FFF)
    return ((b + rounding) >> 16).astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to float32."""
    return (np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def bf16_normal(rng: np.random.Generator, shape) -> np.ndarray:
    """N(0,1) drawn in float32, rounded RNE to bf16 (uint16 bits)."""
    return f32_to_bf16_bits(rng.standard_normal(size=shape, dtype=np.float32))


def lengths_uniform(seed: int, total: int, lo: int, hi: int) -> list[int]:
    """Draw i.i.d. lengths from U{lo..hi} until the running sum reaches
    ``total``; the last length is clipped so the sum is exactly ``total``."""
    rng = np.random.default_rng(seed)
    out: list[int] = []
    s = 0
    while s < total:
        n = int(rng.integers(lo, hi + 1))
        n = min(n, total - s)
        out.append(n)
        s += n
    return out


def cu_from_lengths(lengths) -> np.ndarray:
    """Cumulative offsets, length batch+1, int32 (page 1, "Estructuras de
    datos clave")."""
    cu = np.zeros(len(lengths) + 1, dtype=np.int64)
    cu[1:] = np.cumsum(np.asarray(lengths, dtype=np.int64))
    return cu.astype(np.int32)


@dataclass
class Workload:
    """One synthetic varlen attention problem."""
    name: str
    cu_q: np.ndarray
    cu_k: np.ndarray
    heads: int
    head_dim: int
    scale: float
    causal: bool
    seed: int
    with_grad: bool = False
    heads_k: int | None = None  # key/value heads (grouped-query attention); None: = heads
    _tensors: dict = field(default_factory=dict, repr=False)

    @property
    def kv_heads(self) -> int:
        return self.heads if self.heads_k is None else self.heads_k

    @property
    def batch(self) -> int:
        return len(self.cu_q) - 1

    @property
    def total_q(self) -> int:
        return int(self.cu_q[-1])

    @property
    def total_k(self) -> int:
        return int(self.cu_k[-1])

    @property
    def max_seqlen_q(self) -> int:
        return int(np.max(np.diff(self.cu_q))) if self.batch else 0

    @property
    def max_seqlen_k(self) -> int:
        return int(np.max(np.diff(self.cu_k))) if self.batch else 0

    def tensors(self) -> dict:
        """q, dout as bf16 bits [tokens, heads, head_dim]; k, v as
        [tokens, kv_heads, head_dim]. Drawn in the order q, k, v, dout."""
        if not self._tensors:
            rng = np.random.default_rng(self.seed)
            H, Hk, d = self.heads, self.kv_heads, self.head_dim
            self._tensors["q"] = bf16_normal(rng, (self.total_q, H, d))
            self._tensors["k"] = bf16_normal(rng, (self.total_k, Hk, d))
            self._tensors["v"] = bf16_normal(rng, (self.total_k, Hk, d))
            self._tensors["dout"] = bf16_normal(rng, (self.total_q, H, d))
        return self._tensors


def make_workload(name: str, lengths_q, lengths_k=None, heads=1, head_dim=64,
                  causal=False, seed=0, scale=None, with_grad=False, heads_k=None) -> Workload:
    lengths_k = lengths_q if lengths_k is None else lengths_k
    if scale is None:
        scale = 1.0 / math.sqrt(head_dim)
    return Workload(name, cu_from_lengths(lengths_q), cu_from_lengths(lengths_k), heads,
                    head_dim, float(scale), bool(causal), int(seed), with_grad, heads_k)


def decode_workload(batch: int, keys: int, heads: int = 32, heads_k: int = 8, head_dim: int = 128,
                    seed: int = 9) -> Workload:
    """Token-by-token decoding: one query token per sequence against ``keys``
    cached keys each (packed), grouped heads, causal (the single query is the
    last position, so it sees every key). The split-KV benchmark lines and
    their parity test use these inputs."""
    return make_workload(f"decode-{batch}x{keys}-h{heads}-kv{heads_k}-d{head_dim}", [1] * batch, [keys] * batch,
                         heads=heads, head_dim=head_dim, causal=True, seed=seed, heads_k=heads_k)


def standard_workload(n: int, causal: bool | None = None, head_dim: int | None = None) -> Workload:
    """The five standard workloads, numbered 1..5.

    1  two sequences, cu_q=[0,200,1024], cu_k=[0,300,1024], H=12, d=64,
       scale 1/8, non-causal (page 1's usage example, read as packed).
    2  8 x 2048 fixed length, H=16, d=128, causal or non-causal.
    3  16384 tokens, lengths U{128..4096}, H=32, d=128, causal.
    4  1 x 16384, H=16, d=64 or 128, causal.
    5  16384 tokens, lengths U{512..8192}, H=16, d=128, causal, fwd+bwd.
    """
    if n == 1:
        w = make_workload("varlen-2seq-h12-d64", [200, 824], [300, 724], heads=12,
                          head_dim=64, causal=False, seed=1, scale=1.0 / 8.0)
        w.cu_q = np.array([0, 200, 1024], dtype=np.int32)
        w.cu_k = np.array([0, 300, 1024], dtype=np.int32)
        return w
    if n == 2:
        c = True if causal is None else causal
        return make_workload(f"fixed-8x2048-h16-d128-{'causal' if c else 'full'}",
                             [2048] * 8, heads=16, head_dim=128, causal=c, seed=2)
    if n == 3:
        lens = lengths_uniform(3, TOTAL_TOKENS, 128, 4096)
        return make_workload("packed-16k-U128..4096-h32-d128-causal", lens, heads=32,
                             head_dim=128, causal=True, seed=3)
    if n == 4:
        d = 128 if head_dim is None else head_dim
        return make_workload(f"long-1x16384-h16-d{d}-causal", [16384], heads=16,
                             head_dim=d, causal=True, seed=4)
    if n == 5:
        lens = lengths_uniform(5, TOTAL_TOKENS, 512, 8192)
        return make_workload("varlen-16k-U512..8192-h16-d128-causal-fwdbwd", lens,
                             heads=16, head_dim=128, causal=True, seed=5, with_grad=True)
    raise ValueError(f"no standard workload {n}")
