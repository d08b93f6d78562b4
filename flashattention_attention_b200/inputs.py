"""Seeded synthetic inputs shared by the tests, the bench and the oracle checks.

This module draws random numbers and lays them out; it holds none of the
attention or quantisation arithmetic.  Draws use numpy's PCG64
(``numpy.random.default_rng(seed)``) in a fixed order: sequence lengths first
(when the workload has any), then Q, then K, then V, each from
``standard_normal`` in float64, narrowed to fp32 and then rounded to bf16
(round to nearest even) when the workload is bf16.

The workloads mirror the shapes the fkl_python PR #6 verification speaks of
(dense d64 causal, ragged lengths, int8-KV decode) at the sizes of the
benchmarked configurations: a tiny fp32 causal case, a causal GQA prefill,
an int8-KV decode with per-sequence cache lengths, a varlen causal prefill
with a sliding window and a fused epilogue, and a long-context causal
prefill over an int8 KV cache.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import List, Optional, Tuple

import numpy as np
import torch


def normal(rng: np.random.Generator, shape, dtype: torch.dtype) -> torch.Tensor:
    """iid N(0,1) drawn in float64, narrowed to fp32, then to ``dtype`` (CPU)."""
    x = torch.from_numpy(rng.standard_normal(size=shape)).to(torch.float32)
    return x if dtype == torch.float32 else x.to(dtype)


def cu_from_lengths(lengths) -> torch.Tensor:
    """int32 cumulative offsets [B+1] of a list of lengths."""
    cu = np.zeros(len(lengths) + 1, dtype=np.int64)
    cu[1:] = np.cumsum(np.asarray(lengths, dtype=np.int64))
    return torch.from_numpy(cu.astype(np.int32))


@dataclass
class Workload:
    name: str
    dtype: torch.dtype
    batch: int
    hq: int
    hkv: int
    d: int
    causal: bool
    window: int
    scale: float
    epilogue: List[Tuple[str, float]] = field(default_factory=list)
    seqlen_q: int = 0
    seqlen_k: int = 0
    lengths: Optional[List[int]] = None     # varlen sequence lengths or decode cache lengths
    kv_int8: bool = False
    cache_capacity: int = 0
    q: Optional[torch.Tensor] = None
    k: Optional[torch.Tensor] = None
    v: Optional[torch.Tensor] = None


def dense_prefill(name, *, batch, hq, hkv, s_q, s_k, d, dtype, causal, window=0,
                  epilogue=(), seed=0, kv_int8=False) -> Workload:
    """Dense layout: q [batch*hq, s_q, d], k/v [batch*hkv, s_k, d]."""
    rng = np.random.default_rng(seed)
    w = Workload(name, dtype, batch, hq, hkv, d, causal, window, 1.0 / float(np.sqrt(d)),
                 list(epilogue), s_q, s_k, kv_int8=kv_int8)
    w.q = normal(rng, (batch * hq, s_q, d), dtype)
    w.k = normal(rng, (batch * hkv, s_k, d), dtype)
    w.v = normal(rng, (batch * hkv, s_k, d), dtype)
    return w


def varlen_prefill(name, *, lengths, hq, hkv, d, dtype, causal, window=0,
                   epilogue=(), seed=0) -> Workload:
    """Varlen self-attention: q [hq, total, d], k/v [hkv, total, d] with
    sequence b at rows cu[b]:cu[b+1] of every head plane."""
    rng = np.random.default_rng(seed)
    total = int(sum(lengths))
    w = Workload(name, dtype, len(lengths), hq, hkv, d, causal, window,
                 1.0 / float(np.sqrt(d)), list(epilogue), lengths=list(map(int, lengths)))
    w.q = normal(rng, (hq, total, d), dtype)
    w.k = normal(rng, (hkv, total, d), dtype)
    w.v = normal(rng, (hkv, total, d), dtype)
    return w


def varlen_lengths(seed: int, n: int, lo: int, hi: int) -> List[int]:
    """n lengths uniform in [lo, hi] (inclusive) drawn first from ``seed``."""
    return [int(x) for x in np.random.default_rng(seed).integers(lo, hi + 1, n)]


def decode_cache(name, *, lengths, hq, hkv, d, capacity, seed=0, kv_int8=True,
                 window=0, epilogue=()) -> Workload:
    """Decode: q [B*hq, 1, d] bf16; k/v caches [B*hkv, capacity, d] bf16 with
    keys 0..L_b-1 of sequence b drawn N(0,1) and the unused tail zero.
    Draw order: q, then for each (b, kv-head) the L_b keys of K, then the
    same for V."""
    rng = np.random.default_rng(seed)
    batch = len(lengths)
    w = Workload(name, torch.bfloat16, batch, hq, hkv, d, True, window,
                 1.0 / float(np.sqrt(d)), list(epilogue), seqlen_q=1,
                 lengths=list(map(int, lengths)), kv_int8=kv_int8,
                 cache_capacity=capacity)
    w.q = normal(rng, (batch * hq, 1, d), torch.bfloat16)
    caches = []
    for _ in range(2):
        c = torch.zeros((batch * hkv, capacity, d), dtype=torch.bfloat16)
        for b in range(batch):
            for h in range(hkv):
                c[b * hkv + h, :lengths[b]] = normal(rng, (lengths[b], d), torch.bfloat16)
        caches.append(c)
    w.k, w.v = caches
    return w


# --- the benchmarked workloads ------------------------------------------------

def tiny_fp32_causal(seed=0) -> Workload:
    """fp32, (batch*heads=2, seq=64, d=64), causal, scale 1/8, no epilogue."""
    return dense_prefill("tiny_fp32_causal_bh2_s64_d64", batch=1, hq=2, hkv=2, s_q=64,
                         s_k=64, d=64, dtype=torch.float32, causal=True, seed=seed)


def gqa_causal_prefill(seed=0, batch=4, s=4096) -> Workload:
    """bf16 causal GQA prefill, B=4, Hq=32, Hkv=8, S=4096, d=128."""
    return dense_prefill(f"gqa_causal_prefill_b{batch}_hq32_hkv8_s{s}_d128_bf16",
                         batch=batch, hq=32, hkv=8, s_q=s, s_k=s, d=128,
                         dtype=torch.bfloat16, causal=True, seed=seed)


def ring_cp_last_rank(seed=0, batch=4, block=4096, ranks=4) -> Workload:
    """The last rank of a `ranks`-way context-parallel causal prefill: its
    query block q [batch*32, block, 128] and the K/V of all ranks
    [batch*8, ranks*block, 128] (block r = positions r*block..), bf16."""
    return dense_prefill(f"ring_cp{ranks}_last_rank_b{batch}_hq32_hkv8_block{block}_d128_bf16",
                         batch=batch, hq=32, hkv=8, s_q=block, s_k=ranks * block, d=128,
                         dtype=torch.bfloat16, causal=True, seed=seed)


def int8kv_decode(seed=0, batch=16, lo=1024, hi=32768, capacity=32768) -> Workload:
    """s_q=1 decode, B=16, Hq=32, Hkv=8, d=128, cache lengths U[1024, 32768]."""
    lengths = np.random.default_rng(seed).integers(lo, hi + 1, batch)
    return decode_cache(f"int8kv_decode_b{batch}_hq32_hkv8_d128_cap{capacity}",
                        lengths=lengths, hq=32, hkv=8, d=128, capacity=capacity,
                        seed=seed + 1, kv_int8=True)


def varlen_window_prefill(seed=0, n=8, lo=33, hi=8192) -> Workload:
    """8 packed sequences, lengths U[33, 8192], Hq=32, Hkv=8, d=64, causal,
    window 1024, epilogue [Mul(2.0), Add(0.5)]."""
    lengths = varlen_lengths(seed, n, lo, hi)
    return varlen_prefill(f"varlen_causal_window1024_{n}seq_hq32_hkv8_d64_bf16",
                          lengths=lengths, hq=32, hkv=8, d=64, dtype=torch.bfloat16,
                          causal=True, window=1024, epilogue=[("mul", 2.0), ("add", 0.5)],
                          seed=seed + 1)


def int8kv_long_prefill(seed=0, s=16384) -> Workload:
    """B=1, Hq=64, Hkv=8, S=16384, d=128, causal, int8 KV, epilogue [Mul(0.5)]."""
    return dense_prefill(f"int8kv_causal_prefill_b1_hq64_hkv8_s{s}_d128", batch=1, hq=64,
                         hkv=8, s_q=s, s_k=s, d=128, dtype=torch.bfloat16, causal=True,
                         epilogue=[("mul", 0.5)], seed=seed, kv_int8=True)


def rotation_signs(d: int, seed: int = 0) -> torch.Tensor:
    """The random +-1 signs of a TurboQuant rotation (fp32 [d]), drawn from
    numpy's PCG64 with the given seed (the method's random draw, passed in)."""
    return torch.from_numpy(np.random.default_rng(seed).choice(np.array([-1.0, 1.0], np.float32), d))

