"""Seeded synthetic inputs for decode attention, shared by the tests, the bench
and the oracle's callers.

This module holds none of the attention arithmetic: it draws random numbers,
rounds them to the storage type and counts bytes.  The workloads follow the
shapes the pages discuss — the paper's decoder (d_model 1024, h = 8,
d_k = d_v = 128, length 128, from "Fast Transformer Decoding" study notes §6.1)
and long-context MQA / GQA / MHA serving batches — with N(0, 1) values, because
no trained weights or datasets are involved.

Draw order for a workload and a seed (NumPy ``Generator(PCG64(seed))``):
lens, K cache, V cache, q, k_new, v_new.  Values are drawn in float32 and, for
bf16 workloads, rounded to bf16 with round-to-nearest-even.  Cache rows at or
past a sequence's valid length hold NaN in correctness runs so that any read of
a masked row shows up in the result.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace

import numpy as np

BF16_NAN_BITS = 0x7FC0


def f32_to_bf16_bits(x):
    """float32 array -> bf16 bit patterns (uint16), round to nearest even.
    NaN stays NaN (quiet).  Works in fixed-size chunks with reused buffers so
    multi-GB caches do not allocate GB-sized temporaries."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.reshape(-1).view(np.uint32)
    out = np.empty(u.shape, dtype=np.uint16)
    chunk = 1 << 22
    tmp = np.empty(min(chunk, u.size), dtype=np.uint32)
    for s in range(0, u.size, chunk):
        e = min(u.size, s + chunk)
        t = tmp[: e - s]
        np.right_shift(u[s:e], 16, out=t)
        np.bitwise_and(t, 1, out=t)
        np.add(t, u[s:e], out=t)
        np.add(t, 0x7FFF, out=t)          # no wrap: the largest non-NaN pattern is 0xFF800000
        np.right_shift(t, 16, out=t)
        out[s:e] = t
        nan = np.isnan(x.reshape(-1)[s:e])
        if nan.any():
            out[s:e][nan] = BF16_NAN_BITS
    return out.reshape(x.shape)


def bf16_bits_to_f32(bits):
    """bf16 bit patterns (uint16) -> float32 values (exact)."""
    bits = np.ascontiguousarray(bits, dtype=np.uint16)
    return (bits.astype(np.uint32) << 16).view(np.float32)


@dataclass(frozen=True)
class Workload:
    """One decode-attention problem: b sequences, h query heads sharing g K/V
    heads, head sizes d_k / d_v, a cache of m_max rows per sequence and valid
    lengths drawn uniformly from [len_lo, len_hi]."""
    name: str
    b: int
    h: int
    g: int
    d_k: int
    d_v: int
    m_max: int
    len_lo: int
    len_hi: int
    dtype: str            # "f32" or "bf16": q, caches and o share it
    scale: float          # multiplies q·k
    q_std: float = 1.0
    steps: int = 1        # >1: the cache grows by one row per step from len 1
    description: str = ""

    @property
    def elem_bytes(self) -> int:
        return 4 if self.dtype == "f32" else 2

    @property
    def heads_per_group(self) -> int:
        return self.h // self.g

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


_S128 = 1.0 / math.sqrt(128.0)

WORKLOADS = {
    "tiny_mqa_f32": Workload(
        "tiny_mqa_f32", b=1, h=4, g=1, d_k=32, d_v=32, m_max=64, len_lo=64, len_hi=64,
        dtype="f32", scale=1.0 / math.sqrt(32.0),
        description="tiny MQA, fp32: b=1 h=4 g=1 d=32, 64 valid rows, one append + one decode"),
    "paper_mqa_b128_m128": Workload(
        "paper_mqa_b128_m128", b=128, h=8, g=1, d_k=128, d_v=128, m_max=128, len_lo=1, len_hi=128,
        dtype="bf16", scale=_S128, steps=128,
        description="paper-shaped MQA decoder: b=128 h=8 g=1 d=128, 128 steps, cache grows 1..128"),
    "long_mqa_b64_m8k": Workload(
        "long_mqa_b64_m8k", b=64, h=32, g=1, d_k=128, d_v=128, m_max=8192, len_lo=1024, len_hi=8192,
        dtype="bf16", scale=1.0, q_std=_S128,
        description="long-context MQA serving batch: b=64 h=32 g=1 d=128 m_max=8192, lens U[1024,8192]"),
    "long_mqa_d64_b64_m8k": Workload(
        "long_mqa_d64_b64_m8k", b=64, h=32, g=1, d_k=64, d_v=64, m_max=8192, len_lo=1024, len_hi=8192,
        dtype="bf16", scale=1.0, q_std=1.0 / math.sqrt(64.0),
        description="long-context MQA batch with head size 64: b=64 h=32 g=1 d=64 m_max=8192, lens U[1024,8192]"),
    "gqa8_b32_m32k": Workload(
        "gqa8_b32_m32k", b=32, h=64, g=8, d_k=128, d_v=128, m_max=32768, len_lo=8192, len_hi=32768,
        dtype="bf16", scale=_S128,
        description="GQA-8: b=32 h=64 g=8 d=128 m_max=32768, lens U[8192,32768]"),
    "mha_b16_m16k": Workload(
        "mha_b16_m16k", b=16, h=32, g=32, d_k=128, d_v=128, m_max=16384, len_lo=16384, len_hi=16384,
        dtype="bf16", scale=_S128,
        description="MHA point (g=h=32): b=16 d=128 m=16384 all valid"),
    "mqa_b16_m16k": Workload(
        "mqa_b16_m16k", b=16, h=32, g=1, d_k=128, d_v=128, m_max=16384, len_lo=16384, len_hi=16384,
        dtype="bf16", scale=_S128,
        description="MQA on the MHA point's shapes (g=1): b=16 h=32 d=128 m=16384 all valid"),
}


def draw_lens(wl: Workload, rng) -> np.ndarray:
    return rng.integers(wl.len_lo, wl.len_hi + 1, size=wl.b, endpoint=False).astype(np.int32)


def host_inputs(wl: Workload, seed: int, nan_tail: bool = True, lens=None):
    """All inputs of one decode step of ``wl`` on the host.

    Returns a dict with
      lens  int32 [b]                 (valid rows per sequence after the append)
      k, v  [b, m_max, g, d]          cache (bf16 bits as uint16, or float32)
      q     [b, h, d_k]
      k_new, v_new [b, g, d]          the step's K/V, to be written at row lens-1
    and the same arrays as float32 values under the keys ``*_f32``.
    """
    rng = np.random.Generator(np.random.PCG64(seed))
    drawn = draw_lens(wl, rng)
    lens = drawn if lens is None else np.asarray(lens, dtype=np.int32)
    shape_k = (wl.b, wl.m_max, wl.g, wl.d_k)
    shape_v = (wl.b, wl.m_max, wl.g, wl.d_v)
    k = rng.standard_normal(shape_k, dtype=np.float32)
    v = rng.standard_normal(shape_v, dtype=np.float32)
    q = rng.standard_normal((wl.b, wl.h, wl.d_k), dtype=np.float32) * np.float32(wl.q_std)
    k_new = rng.standard_normal((wl.b, wl.g, wl.d_k), dtype=np.float32)
    v_new = rng.standard_normal((wl.b, wl.g, wl.d_v), dtype=np.float32)
    if nan_tail:
        rows = np.arange(wl.m_max)[None, :] >= lens[:, None]          # [b, m_max]
        k[rows] = np.nan
        v[rows] = np.nan
    out = {"lens": lens}
    for name, arr in (("k", k), ("v", v), ("q", q), ("k_new", k_new), ("v_new", v_new)):
        if wl.dtype == "bf16":
            bits = f32_to_bf16_bits(arr)
            out[name] = bits
            out[name + "_f32"] = bf16_bits_to_f32(bits)
        else:
            out[name] = arr
            out[name + "_f32"] = arr
    return out


def device_inputs(wl: Workload, seed: int, device, copies: int = 1, chunk_rows: int = 1 << 22):
    """Large inputs generated on the device with torch's seeded generator
    (plumbing only: torch allocates and fills the buffers).  Used where the
    host would need many GB for the full-size workloads.  Returns a dict with
    lens (int32, from NumPy with the same seed), and torch tensors q, k_new,
    v_new and ``copies`` K/V cache pairs (lists) in the workload's dtype.
    Cache rows past lens hold N(0,1) values like the rest."""
    import torch

    rng = np.random.Generator(np.random.PCG64(seed))
    lens = draw_lens(wl, rng)
    tdt = torch.float32 if wl.dtype == "f32" else torch.bfloat16
    gen = torch.Generator(device=device)
    gen.manual_seed(int(seed) * 1000003 + 17)

    def randn(shape, std=1.0):
        out = torch.empty(shape, dtype=tdt, device=device)
        flat = out.view(-1)
        n = flat.numel()
        for s in range(0, n, chunk_rows):
            e = min(n, s + chunk_rows)
            tmp = torch.randn(e - s, generator=gen, device=device, dtype=torch.float32)
            if std != 1.0:
                tmp.mul_(std)
            flat[s:e].copy_(tmp)
        return out

    ks, vs = [], []
    for _ in range(copies):
        ks.append(randn((wl.b, wl.m_max, wl.g, wl.d_k)))
        vs.append(randn((wl.b, wl.m_max, wl.g, wl.d_v)))
    q = randn((wl.b, wl.h, wl.d_k), wl.q_std)
    k_new = randn((wl.b, wl.g, wl.d_k))
    v_new = randn((wl.b, wl.g, wl.d_v))
    return {"lens": lens, "k": ks, "v": vs, "q": q, "k_new": k_new, "v_new": v_new}


# ---------------------------------------------------------------- byte counts

def kv_cache_bytes(b: int, m: int, g: int, d_k: int, d_v: int, elem_bytes: int) -> int:
    """Bytes of a K+V cache of b sequences, m rows, g K/V heads: the quantity the
    MQA/MHA comparison is about (2·T·n_h·d_h versus 2·T·d_h per sequence)."""
    return b * m * g * (d_k + d_v) * elem_bytes


def decode_algorithmic_bytes(wl: Workload, lens, window: int = 0) -> int:
    """Bytes one decode must move at minimum: every attended K and V row once
    (the valid rows, or the newest ``window`` of them), q read once, o written
    once.  Masked rows and split partials not counted."""
    lens = np.asarray(lens, dtype=np.int64)
    if window > 0:
        lens = np.minimum(lens, window)
    kv = int(lens.sum()) * wl.g * (wl.d_k + wl.d_v) * wl.elem_bytes
    qo = wl.b * wl.h * (wl.d_k + wl.d_v) * wl.elem_bytes
    return kv + qo


def append_algorithmic_bytes(wl: Workload) -> int:
    """Bytes of one append: the new K/V read once and written once."""
    return 2 * wl.b * wl.g * (wl.d_k + wl.d_v) * wl.elem_bytes


def decode_flops(wl: Workload, lens) -> int:
    """2·d_k FLOPs per (head, row) for q·k plus 2·d_v for the weighted V."""
    lens = np.asarray(lens, dtype=np.int64)
    return int(lens.sum()) * wl.h * 2 * (wl.d_k + wl.d_v)


@dataclass(frozen=True)
class PrefillWorkload:
    """One batched (prefill) attention problem: b sequences of n tokens each,
    packed, h query heads sharing g K/V heads of size d, causal or not."""
    name: str
    b: int
    n: int
    h: int
    g: int
    d: int
    causal: bool
    scale: float
    description: str = ""

    @property
    def total(self) -> int:
        return self.b * self.n


PREFILL_WORKLOADS = {
    "prefill_mqa_b8_n4096": PrefillWorkload(
        "prefill_mqa_b8_n4096", b=8, n=4096, h=32, g=1, d=128, causal=True, scale=_S128,
        description="MQA prompt prefill: 8 sequences x 4096 tokens, h=32 g=1 d=128, causal"),
    "prefill_gqa8_b4_n8192": PrefillWorkload(
        "prefill_gqa8_b4_n8192", b=4, n=8192, h=64, g=8, d=128, causal=True, scale=_S128,
        description="GQA-8 prompt prefill: 4 sequences x 8192 tokens, h=64 g=8 d=128, causal"),
}


def prefill_flops(wl: PrefillWorkload) -> int:
    """2 h d FLOPs for q.k and 2 h d for p.v per attended (query, key) pair."""
    pairs = wl.n * (wl.n + 1) // 2 if wl.causal else wl.n * wl.n
    return 4 * wl.h * wl.d * pairs * wl.b


def prefill_device_inputs(wl: PrefillWorkload, seed: int, device):
    """q [T,h,d], k/v [T,g,d] bf16 N(0,1) from torch's seeded generator, and
    cu_seqlens int32 [b+1] for equal-length packed sequences."""
    import torch
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    T = wl.total
    out = {}
    for name, heads in (("q", wl.h), ("k", wl.g), ("v", wl.g)):
        out[name] = torch.randn((T, heads, wl.d), generator=gen, device=device, dtype=torch.float32).to(torch.bfloat16)
    out["cu"] = torch.arange(0, T + 1, wl.n, dtype=torch.int32, device=device)
    return out


@dataclass(frozen=True)
class BeamWorkload:
    """One decode step of W beams per sequence sharing a prefix: b sequences,
    prefix lengths U[lp_lo, lp_hi] (cache m_p rows), suffix lengths
    U[ls_lo, ls_hi] per beam (cache m_s rows)."""
    name: str
    b: int
    W: int
    h: int
    g: int
    d: int
    m_p: int
    lp_lo: int
    lp_hi: int
    m_s: int
    ls_lo: int
    ls_hi: int
    scale: float
    description: str = ""


BEAM_WORKLOADS = {
    "beam4_mqa_b64_p8k": BeamWorkload(
        "beam4_mqa_b64_p8k", b=64, W=4, h=8, g=1, d=128, m_p=8192, lp_lo=4096, lp_hi=8192, m_s=128, ls_lo=1,
        ls_hi=128, scale=_S128,
        description="beam-4 MQA decoder (the paper's h=8, d=128): 64 sequences x 4 beams, prefixes U[4096,8192], "
                    "suffixes U[1,128]"),
}


def beam_device_inputs(wl: BeamWorkload, seed: int, device):
    """q [b,W,h,d], prefix caches [b,m_p,g,d], suffix caches [b*W,m_s,g,d] (bf16
    N(0,1), torch's seeded generator) and the two length arrays (int32)."""
    import torch
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    rng = np.random.Generator(np.random.PCG64(seed))
    lp = rng.integers(wl.lp_lo, wl.lp_hi + 1, size=wl.b).astype(np.int32)
    ls = rng.integers(wl.ls_lo, wl.ls_hi + 1, size=wl.b * wl.W).astype(np.int32)

    def rnd(shape):
        return torch.randn(shape, generator=gen, device=device, dtype=torch.float32).to(torch.bfloat16)

    return {"q": rnd((wl.b, wl.W, wl.h, wl.d)), "pk": rnd((wl.b, wl.m_p, wl.g, wl.d)),
            "pv": rnd((wl.b, wl.m_p, wl.g, wl.d)), "sk": rnd((wl.b * wl.W, wl.m_s, wl.g, wl.d)),
            "sv": rnd((wl.b * wl.W, wl.m_s, wl.g, wl.d)), "lp": lp, "ls": ls}


def beam_algorithmic_bytes(wl: BeamWorkload, lp, ls) -> int:
    """Every prefix row once (shared by the beams), every suffix row once, q and o."""
    rows = int(np.asarray(lp, dtype=np.int64).sum() + np.asarray(ls, dtype=np.int64).sum())
    return rows * wl.g * 2 * wl.d * 2 + wl.b * wl.W * wl.h * 2 * wl.d * 2
