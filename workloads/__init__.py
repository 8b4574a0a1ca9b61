"""Seeded synthetic workloads for compact-KV decode attention.

This module draws random numbers and fixes shapes; it holds none of the method's
arithmetic (no attention, no compaction, no quantisation). Both sides of every
parity check take their inputs from here: the CPU oracle under ``oracle/`` and
the CUDA library under ``compressed_decode_attention_fdms_b200/``.

The workloads stand in for the decode benchmark of the FastDMS announcement
(aiwitness.kr/community/1t3vlrx, the KV-memory table: ctx_len 8192, gen_len 128,
concurrency 1 and 8, Llama-3.2-1B and Qwen3-8B shapes). No model, checkpoint or
dataset is used: keys, values and queries are Gaussian, and the learned per-head
eviction decision of DMS is replaced by a Bernoulli keep bit per (token, kv head)
with a per-head rate.

Recipe (every tensor is regenerated from (seed, tag, layer, seq, step)):

* K, V: N(0, 1) per element, times a per-(layer, kv head, channel) scale drawn
  from U[0.5, 2] when the workload asks for one (independent vectors for K and
  V, shared across sequences), rounded to bf16 (round to nearest even).
* q: N(0, 1) rounded to bf16, fresh per (layer, step).
* keep: 1 with probability ``rate[layer, seq, kv_head]`` for every token,
  decode tokens included. The always-visible recent window is a property of the
  cache (``window``), not of the mask.
* Context lengths: fixed, or U[lo, hi] (integers) per sequence.
* Dense outliers: exactly round(frac * L * B * Hkv) (layer, seq, head) triples,
  chosen by a seeded permutation, get rate 1.
"""
from __future__ import annotations

import dataclasses
from dataclasses import dataclass, field
from typing import Optional, Sequence

import numpy as np
import torch

__all__ = [
    "Workload", "WORKLOADS", "get", "scaled",
    "context_lengths", "keep_rates", "channel_scales",
    "prefill_inputs", "decode_inputs", "decode_query",
]

# tags keep the random streams of different tensors apart
_TAG_K, _TAG_V, _TAG_KEEP, _TAG_Q, _TAG_CTX, _TAG_RATE, _TAG_CSCALE, _TAG_DENSE = range(1, 9)


@dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    layers: int
    q_heads: int
    kv_heads: int
    head_dim: int
    kv_dtype: str                    # "bf16" or "fp8_e4m3"
    window: int                      # always-visible recent window W
    period: int                      # compaction period P (1 = every step)
    steps: int                       # decode steps after the prefill
    ctx: int = 8192                  # prefill length (fixed)
    ctx_range: Optional[tuple] = None  # (lo, hi): per-sequence U[lo, hi] instead of ctx
    rate: Optional[float] = None     # one keep rate for every head
    rate_range: tuple = (0.05, 0.30)  # else U[lo, hi]
    rate_per_seq: bool = True        # rate per (layer, seq, head) (else per (layer, head))
    dense_frac: float = 0.0          # fraction of (layer, seq, head) triples with rate 1
    channel_scale: bool = False      # per-(layer, head, channel) U[0.5, 2] on K and V
    seed: int = 0xFD45

    @property
    def group(self) -> int:
        return self.q_heads // self.kv_heads

    @property
    def max_ctx(self) -> int:
        return self.ctx_range[1] if self.ctx_range else self.ctx

    @property
    def max_seq_len(self) -> int:
        return self.max_ctx + self.steps


# The five workloads. Seeds are 0xFD45 + index.
WORKLOADS = {
    "tiny": Workload("tiny", batch=1, layers=1, q_heads=4, kv_heads=2, head_dim=64,
                     kv_dtype="bf16", window=16, period=1, steps=8, ctx=512, rate=0.25,
                     seed=0xFD45 + 0),
    "llama1b_c1": Workload("llama1b_c1", batch=1, layers=16, q_heads=32, kv_heads=8,
                           head_dim=64, kv_dtype="bf16", window=256, period=1, steps=128,
                           ctx=8192, rate_range=(0.05, 0.30), rate_per_seq=False,
                           channel_scale=True, seed=0xFD45 + 1),
    "llama1b_c8": Workload("llama1b_c8", batch=8, layers=16, q_heads=32, kv_heads=8,
                           head_dim=64, kv_dtype="bf16", window=256, period=1, steps=128,
                           ctx=8192, rate_range=(0.05, 0.30), channel_scale=True,
                           seed=0xFD45 + 2),
    "qwen8b_c8_fp8": Workload("qwen8b_c8_fp8", batch=8, layers=36, q_heads=32, kv_heads=8,
                              head_dim=128, kv_dtype="fp8_e4m3", window=256, period=1,
                              steps=128, ctx=8192, rate_range=(0.06, 0.20),
                              seed=0xFD45 + 3),
    # the Qwen3-8B c=8 FP8 workload with the per-block FP8 scale reading (each sealed
    # 64-slot block's own maxima; the staged block and the ring in bf16)
    "qwen8b_c8_fp8_block": Workload("qwen8b_c8_fp8_block", batch=8, layers=36, q_heads=32,
                                    kv_heads=8, head_dim=128, kv_dtype="fp8_e4m3_block",
                                    window=256, period=1, steps=128, ctx=8192,
                                    rate_range=(0.06, 0.20), seed=0xFD45 + 3),
    "qwen8b_long_fp8": Workload("qwen8b_long_fp8", batch=32, layers=36, q_heads=32,
                                kv_heads=8, head_dim=128, kv_dtype="fp8_e4m3", window=256,
                                period=64, steps=256, ctx_range=(1024, 32768),
                                rate_range=(0.03, 0.25), dense_frac=0.10,
                                seed=0xFD45 + 4),
}


def get(name: str) -> Workload:
    return WORKLOADS[name]


def scaled(wl: Workload, **changes) -> Workload:
    """A copy of ``wl`` with some fields changed (smaller test shapes)."""
    return dataclasses.replace(wl, **changes)


def _seed(*parts: int) -> int:
    ss = np.random.SeedSequence([int(p) & 0xFFFFFFFF for p in parts])
    return int(ss.generate_state(1, dtype=np.uint64)[0] & 0x7FFFFFFFFFFFFFFF)


def _gen(device, *parts: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(_seed(*parts))
    return g


def context_lengths(wl: Workload) -> np.ndarray:
    """Prefill length of each sequence, int64 [B]."""
    if wl.ctx_range is None:
        return np.full(wl.batch, wl.ctx, dtype=np.int64)
    rng = np.random.default_rng(_seed(wl.seed, _TAG_CTX))
    lo, hi = wl.ctx_range
    return rng.integers(lo, hi + 1, size=wl.batch).astype(np.int64)


def keep_rates(wl: Workload) -> np.ndarray:
    """Keep probability per (layer, seq, kv head), float64 [L][B][Hkv]."""
    L, B, H = wl.layers, wl.batch, wl.kv_heads
    if wl.rate is not None:
        rates = np.full((L, B, H), float(wl.rate))
    else:
        rng = np.random.default_rng(_seed(wl.seed, _TAG_RATE))
        lo, hi = wl.rate_range
        if wl.rate_per_seq:
            rates = rng.uniform(lo, hi, size=(L, B, H))
        else:
            rates = np.broadcast_to(rng.uniform(lo, hi, size=(L, 1, H)), (L, B, H)).copy()
    if wl.dense_frac > 0:
        n = int(round(wl.dense_frac * L * B * H))
        rng = np.random.default_rng(_seed(wl.seed, _TAG_DENSE))
        idx = rng.permutation(L * B * H)[:n]
        rates.reshape(-1)[idx] = 1.0
    return rates


def channel_scales(wl: Workload, layer: int):
    """(c_K, c_V): float32 [Hkv][D] each; ones when the workload has no channel scale."""
    shape = (wl.kv_heads, wl.head_dim)
    if not wl.channel_scale:
        one = torch.ones(shape, dtype=torch.float32)
        return one, one
    g = _gen("cpu", wl.seed, _TAG_CSCALE, layer)
    ck = torch.rand(shape, generator=g, dtype=torch.float32) * 1.5 + 0.5
    cv = torch.rand(shape, generator=g, dtype=torch.float32) * 1.5 + 0.5
    return ck, cv


def _kv_rows(wl, layer, seq, step, n, device, tag, cscale):
    g = _gen(device, wl.seed, tag, layer, seq, step)
    x = torch.randn((n, wl.kv_heads, wl.head_dim), generator=g, device=device,
                    dtype=torch.float32)
    if wl.channel_scale:
        x.mul_(cscale.to(device))
    return x.to(torch.bfloat16)


def _keep_rows(wl, layer, seq, step, n, rates, device):
    g = _gen(device, wl.seed, _TAG_KEEP, layer, seq, step)
    u = torch.rand((n, wl.kv_heads), generator=g, device=device, dtype=torch.float64)
    r = torch.as_tensor(rates[layer, seq], dtype=torch.float64, device=device)
    return (u < r).to(torch.uint8)


def prefill_inputs(wl: Workload, layer: int, device="cpu", seqs: Optional[Sequence[int]] = None):
    """Prefill tokens of one layer.

    Returns a dict with ``k``/``v`` bf16 [B][max_new][Hkv][D], ``keep`` uint8
    [B][max_new][Hkv] and ``n_new`` int32 [B] (rows past ``n_new[b]`` are zero).
    ``seqs`` restricts generation to some sequences (the others get n_new = 0);
    each sequence's values do not depend on which others are generated.
    """
    ctx = context_lengths(wl)
    rates = keep_rates(wl)
    ck, cv = channel_scales(wl, layer)
    seqs = range(wl.batch) if seqs is None else list(seqs)
    max_new = int(max(ctx[list(seqs)])) if len(seqs) else 0
    shape = (wl.batch, max_new, wl.kv_heads, wl.head_dim)
    k = torch.zeros(shape, dtype=torch.bfloat16, device=device)
    v = torch.zeros(shape, dtype=torch.bfloat16, device=device)
    keep = torch.zeros(shape[:3], dtype=torch.uint8, device=device)
    n_new = torch.zeros(wl.batch, dtype=torch.int32)
    for b in seqs:
        n = int(ctx[b])
        k[b, :n] = _kv_rows(wl, layer, b, -1, n, device, _TAG_K, ck)
        v[b, :n] = _kv_rows(wl, layer, b, -1, n, device, _TAG_V, cv)
        keep[b, :n] = _keep_rows(wl, layer, b, -1, n, rates, device)
        n_new[b] = n
    return {"k": k, "v": v, "keep": keep, "n_new": n_new.to(device), "max_new": max_new}


def decode_inputs(wl: Workload, layer: int, step: int, device="cpu"):
    """One decode token per sequence for one layer: k, v [B][1][Hkv][D], keep [B][1][Hkv]."""
    rates = keep_rates(wl)
    ck, cv = channel_scales(wl, layer)
    shape = (wl.batch, 1, wl.kv_heads, wl.head_dim)
    g = _gen(device, wl.seed, _TAG_K, layer, step, 0x5EED)
    k = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    v = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    if wl.channel_scale:
        k.mul_(ck.to(device))
        v.mul_(cv.to(device))
    u = torch.rand(shape[:3], generator=g, device=device, dtype=torch.float64)
    r = torch.as_tensor(rates[layer], dtype=torch.float64, device=device)  # [B][Hkv]
    keep = (u < r[:, None, :]).to(torch.uint8)
    n_new = torch.ones(wl.batch, dtype=torch.int32, device=device)
    return {"k": k.to(torch.bfloat16), "v": v.to(torch.bfloat16), "keep": keep,
            "n_new": n_new, "max_new": 1}


def decode_query(wl: Workload, layer: int, step: int, device="cpu"):
    """Query of one decode step: bf16 [B][Hq][D], N(0, 1)."""
    g = _gen(device, wl.seed, _TAG_Q, layer, step)
    q = torch.randn((wl.batch, wl.q_heads, wl.head_dim), generator=g, device=device,
                    dtype=torch.float32)
    return q.to(torch.bfloat16)
