"""Seeded synthetic workloads for the quantized KV cache.

This module only draws inputs: it holds none of the method's arithmetic
(no quantization, no layout, no attention).  Both the CUDA path and the CPU
oracle are fed from it.

Recipe (all draws from numpy.random.default_rng(seed), PCG64, in this order):
  1. outlier key channels: 4 distinct channels per kv head (choice without
     replacement), fixed for every token of the workload (keys carry
     persistent outlier channels across positions);
  2. lengths: per-sequence residual fill r ~ U{0..R-1} (fixed-T workloads) or
     sequence lengths L ~ U[lo, hi] (the continuous-batching mix);
  3. K: standard normal float32 [sum(L)][H_kv][D], then x20 on the outlier
     channels (in fp32), then round-to-nearest-even to bf16;
  4. V: standard normal float32, bf16;
  5. q: standard normal float32 [B][H_q][D], bf16;
  6. per decode step: new K [B][H_kv][D] (with the same outliers), new V, new q.
Tokens are laid out sequence-major (all tokens of sequence 0, then 1, ...), the
order a bulk prefill appends them in.
"""
from dataclasses import dataclass, field
from typing import List, Optional

import numpy as np
import torch


def to_bf16_bits(x32: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bit patterns (uint16), round to nearest even (torch CPU)."""
    t = torch.from_numpy(np.ascontiguousarray(x32, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


@dataclass
class CacheFormat:
    """A KV-cache storage format (argument bundle for both implementations)."""
    bits: int
    asym: int
    k_axis: int          # 0: keys grouped per token; 1: keys grouped per channel
    g_k: int
    g_v: int
    scale_fp32: int
    residual: int        # R (0 for per-token keys, == g_k for per-channel keys)
    page: int            # P tokens per block
    fp8: int = 0         # 1: FP8 E4M3 elements with one scale per kv head


@dataclass
class Workload:
    name: str
    seed: int
    fmt: CacheFormat
    batch: int
    h_q: int
    h_kv: int
    d_h: int
    lengths: List[int]               # tokens per sequence after the prefill
    outliers: int = 4                # outlier key channels per kv head
    outlier_gain: float = 20.0
    steps: int = 0                   # decode steps (one appended token per sequence)
    layers_reported: int = 1         # layer count used for the memory report
    note: str = ""
    extra: dict = field(default_factory=dict)


def _lengths_fixed(rng, batch, T, R):
    if R > 0:
        return [T + int(r) for r in rng.integers(0, R, size=batch)]
    return [T] * batch


# The five workloads, with the pages' geometry (H_kv=8, d_h=128, ...).
def workload(idx: int) -> Workload:
    if idx == 1:
        f = CacheFormat(bits=8, asym=0, k_axis=0, g_k=128, g_v=128, scale_fp32=1, residual=0, page=512)
        return Workload("tiny-int8-contiguous", 0, f, batch=1, h_q=1, h_kv=1, d_h=128,
                        lengths=[512], outliers=0,
                        note="1 sequence, H_q=H_kv=1, T=512, INT8 per-token G=128 fp32 scale, one block")
    if idx == 2:
        f = CacheFormat(bits=8, asym=0, k_axis=0, g_k=128, g_v=128, scale_fp32=0, residual=0, page=16)
        return Workload("int8-paged-gqa", 1, f, batch=8, h_q=32, h_kv=8, d_h=128,
                        lengths=[4096] * 8,
                        note="B=8, T=4096, INT8 per-token G=128 fp16 scales, P=16 shuffled")
    if idx == 3:
        f = CacheFormat(bits=4, asym=0, k_axis=1, g_k=64, g_v=64, scale_fp32=0, residual=64, page=16)
        return Workload("int4-kivi", 2, f, batch=16, h_q=32, h_kv=8, d_h=128,
                        lengths=[], layers_reported=32,
                        note="B=16, T=8192 + residual U{0..63}, INT4 sym, K per-channel G=64, V per-token G=64")
    if idx == 4:
        f = CacheFormat(bits=2, asym=1, k_axis=1, g_k=32, g_v=32, scale_fp32=0, residual=32, page=16)
        return Workload("int2-asym-128k", 3, f, batch=1, h_q=32, h_kv=8, d_h=128,
                        lengths=[131072 + 31],
                        note="B=1, T=131072 + 31 residual, INT2 asym G=32 (fp16 scale + zero)")
    if idx == 5:
        f = CacheFormat(bits=4, asym=0, k_axis=1, g_k=64, g_v=64, scale_fp32=0, residual=64, page=16)
        return Workload("continuous-batching-int4", 4, f, batch=64, h_q=32, h_kv=8, d_h=128,
                        lengths=[], steps=100,
                        note="64 sequences, L ~ U[512, 32768], INT4 as the KIVI workload, 100 steps")
    raise ValueError(idx)


class Draws:
    """Materialised seeded inputs of a workload."""

    def __init__(self, w: Workload, length_override: Optional[List[int]] = None,
                 steps: Optional[int] = None):
        self.w = w
        rng = np.random.default_rng(w.seed)
        self.rng = rng
        D, H = w.d_h, w.h_kv
        # 1. outlier channels
        self.outlier_channels = np.zeros((H, w.outliers), dtype=np.int64)
        for h in range(H):
            if w.outliers:
                self.outlier_channels[h] = np.sort(rng.choice(D, size=w.outliers, replace=False))
        # 2. lengths
        if length_override is not None:
            self.lengths = list(length_override)
        elif w.name == "int4-kivi":
            self.lengths = _lengths_fixed(rng, w.batch, 8192, w.fmt.residual)
        elif w.name == "continuous-batching-int4":
            self.lengths = [int(x) for x in rng.integers(512, 32768 + 1, size=w.batch)]
        else:
            self.lengths = list(w.lengths)
        n = int(sum(self.lengths))
        # 3-5. prefill K, V and the first query
        self.k = self._keys(n)
        self.v = to_bf16_bits(rng.standard_normal((n, H, D), dtype=np.float32))
        self.q = to_bf16_bits(rng.standard_normal((w.batch, w.h_q, D), dtype=np.float32))
        self.seq_ids = np.repeat(np.arange(w.batch, dtype=np.int32),
                                 np.asarray(self.lengths, dtype=np.int64))
        self.steps = w.steps if steps is None else steps

    def _keys(self, n: int) -> np.ndarray:
        w = self.w
        k = self.rng.standard_normal((n, w.h_kv, w.d_h), dtype=np.float32)
        for h in range(w.h_kv):
            for c in self.outlier_channels[h]:
                k[:, h, c] *= np.float32(w.outlier_gain)
        return to_bf16_bits(k)

    def step(self):
        """Inputs of one decode step: (k_new, v_new, q), each bf16 bits."""
        w = self.w
        k = self._keys(w.batch)
        v = to_bf16_bits(self.rng.standard_normal((w.batch, w.h_kv, w.d_h), dtype=np.float32))
        q = to_bf16_bits(self.rng.standard_normal((w.batch, w.h_q, w.d_h), dtype=np.float32))
        return k, v, q


def random_bf16(rng, shape, scale: float = 1.0) -> np.ndarray:
    """Generic seeded bf16 normal draws (small parity cases)."""
    return to_bf16_bits(rng.standard_normal(shape, dtype=np.float32) * np.float32(scale))
