"""Seeded synthetic inputs for HGA routed attention (shared by the CUDA path's
tests/bench and by the CPU oracle's tests).

This module holds NO step of the routed-attention method itself (no summary,
score, selection or softmax).  It only draws the inputs the method consumes:
projected, RoPE-applied Q/K/V of one attention layer, optionally with planted
"needle" groups, rounded to the storage dtype.

Recipe (one layer, head-major K/V like a KV cache):
  * Q ~ N(0,1) of shape [Tq][Hq][d] for positions q0..T-1, then K ~ N(0,1) and
    V ~ N(0,1) of shape [Hkv][T][d], all drawn in float32 from
    numpy.random.Generator(PCG64(seed)) in that order (seed 0 by default).
  * RoPE (rotate-half pairing of dims i and i+d/2, inverse frequencies
    theta**(-2i/d), absolute positions, angles in float64) is applied to Q and K.
    The pages ("Long-Context Fine-Tuning with Limited VRAM", abstract of the HGA
    paper) call the summaries "RoPE-aware"; the inputs of the path are
    post-RoPE projections, so RoPE belongs to input preparation.
  * Needles (optional): n_needles per KV head, drawn from a second stream
    PCG64(seed + 1).  Each picks one 8-token group j and a later query block b*
    of the segment for which j's chunk lies strictly between the sink and the
    local window of b*; the group's 8 post-RoPE keys are replaced by
    0.8 * mean(post-RoPE q over b*'s rows and the query heads of that KV head)
    + 0.2 * N(0, I).  V is left as drawn.
  * Finally everything is rounded once (round-to-nearest-even) to the storage
    dtype: bfloat16 or float32.

The workloads below are the five shapes the path is measured and checked on:
Qwen3-style attention shapes (the pages evaluate Qwen3-8B and
Qwen3-30B-A3B), routing with 64-token chunks and 8-token groups (page
"Long-Context Fine-Tuning with Limited VRAM", section 2.1 and Table 1).
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import numpy as np
import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    """One routed-attention problem: shapes, routing budget and input recipe."""
    name: str
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    T: int                # total context length (keys 0..T-1)
    q0: int               # first query position; the query segment is [q0, T)
    rope_theta: float
    sink: int
    local: int
    top_chunks: int       # <= 0 means "all"
    top_groups: int       # <= 0 means "all"
    dtype: str = "bf16"   # "bf16" or "fp32"
    chunk: int = 64
    group: int = 8
    qblock: int = 64
    n_needles: int = 0    # planted needle groups per KV head
    seed: int = 0

    @property
    def Tq(self) -> int:
        return self.T - self.q0

    @property
    def G(self) -> int:
        return self.n_q_heads // self.n_kv_heads

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


# The five measured/checked workloads.
TINY_FP32 = Workload("tiny_fp32_1k", 2, 1, 64, 1024, 0, 1e6, 64, 128, 4, 8,
                     dtype="fp32")
QWEN3_8B_16K = Workload("qwen3_8b_prefill_16k", 32, 8, 128, 16384, 0, 1e6, 64,
                        256, 16, 32, n_needles=32)
QWEN3_30B_64K = Workload("qwen3_30b_a3b_64k_last2k", 32, 4, 128, 65536, 63488,
                         1e7, 64, 512, 32, 64, n_needles=32)
TIERED_128K = Workload("qwen3_8b_tiered_128k_last4k", 32, 8, 128, 131072,
                       126976, 1e6, 64, 512, 32, 64, n_needles=32)
SWEEP_32K = Workload("qwen3_8b_sweep_32k", 32, 8, 128, 32768, 0, 1e6, 64, 256,
                     16, 32, n_needles=32)
SWEEP_BUDGETS = (4, 8, 16, 64, 0)   # top-chunks; top-groups = 2x (0 = all)

WORKLOADS = {w.name: w for w in
             (TINY_FP32, QWEN3_8B_16K, QWEN3_30B_64K, TIERED_128K, SWEEP_32K)}


def _rope_tables(positions: np.ndarray, d: int, theta: float):
    half = d // 2
    inv_freq = theta ** (-(np.arange(half, dtype=np.float64) * 2.0) / d)
    ang = positions.astype(np.float64)[:, None] * inv_freq[None, :]
    return np.cos(ang), np.sin(ang)


def _apply_rope(x: np.ndarray, cos: np.ndarray, sin: np.ndarray) -> np.ndarray:
    """x [..., P, d] float64 with cos/sin [P, d/2]; rotate-half pairing."""
    half = x.shape[-1] // 2
    x1 = x[..., :half]
    x2 = x[..., half:]
    out = np.empty_like(x)
    out[..., :half] = x1 * cos - x2 * sin
    out[..., half:] = x2 * cos + x1 * sin
    return out


def _round(x: np.ndarray, dtype: str) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return t.to(torch.bfloat16) if dtype == "bf16" else t.clone()


@dataclasses.dataclass
class Inputs:
    """CPU tensors in the storage dtype, laid out as the C ABI expects:
    q [Tq][Hq][d], k and v [Hkv][T][d]; needles is a list of (h, group, block)."""
    w: Workload
    q: torch.Tensor
    k: torch.Tensor
    v: torch.Tensor
    needles: list


def make_inputs(w: Workload, seed: Optional[int] = None) -> Inputs:
    seed = w.seed if seed is None else seed
    rng = np.random.Generator(np.random.PCG64(seed))
    Hq, Hkv, d, T, q0 = w.n_q_heads, w.n_kv_heads, w.head_dim, w.T, w.q0
    q = rng.standard_normal((w.Tq, Hq, d), dtype=np.float32)
    k = rng.standard_normal((Hkv, T, d), dtype=np.float32)
    v = rng.standard_normal((Hkv, T, d), dtype=np.float32)

    cos_q, sin_q = _rope_tables(np.arange(q0, T), d, w.rope_theta)
    # q is [Tq][Hq][d]: rotate with the position axis first.
    q64 = _apply_rope(q.astype(np.float64).transpose(1, 0, 2), cos_q, sin_q)
    q64 = q64.transpose(1, 0, 2)
    cos_k, sin_k = _rope_tables(np.arange(T), d, w.rope_theta)
    k_out = np.empty((Hkv, T, d), dtype=np.float32)
    for h in range(Hkv):
        k_out[h] = _apply_rope(k[h].astype(np.float64), cos_k, sin_k)
    del k

    needles = []
    if w.n_needles > 0:
        needles = _plant_needles(w, q64, k_out, seed + 1)

    qt = _round(q64, w.dtype)
    kt = _round(k_out, w.dtype)
    vt = _round(v, w.dtype)
    return Inputs(w, qt, kt, vt, needles)


def make_q_before(w: Workload, seed: Optional[int] = None) -> torch.Tensor:
    """The qblock queries at positions q0 - qblock .. q0 - 1, [qblock][Hq][d]
    in the storage dtype: standard normal rows rotated at their positions,
    drawn from their own stream (seed + 2).  All zero when q0 < qblock (no
    earlier positions exist).  They feed the strictly causal routing
    variant, which routes the segment's first block on them."""
    seed = w.seed if seed is None else seed
    B, Hq, d = w.qblock, w.n_q_heads, w.head_dim
    if w.q0 < B:
        return _round(np.zeros((B, Hq, d)), w.dtype)
    rng = np.random.Generator(np.random.PCG64(seed + 2))
    q = rng.standard_normal((B, Hq, d), dtype=np.float32)
    cos_q, sin_q = _rope_tables(np.arange(w.q0 - B, w.q0), d, w.rope_theta)
    q64 = _apply_rope(q.astype(np.float64).transpose(1, 0, 2), cos_q, sin_q)
    return _round(q64.transpose(1, 0, 2), w.dtype)


def _plant_needles(w: Workload, q64: np.ndarray, k_out: np.ndarray,
                   seed: int) -> list:
    """Replace the keys of n_needles groups per KV head in k_out (in place)."""
    rng = np.random.Generator(np.random.PCG64(seed))
    C, g, B, G = w.chunk, w.group, w.qblock, w.G
    n_blocks = (w.Tq + B - 1) // B
    out = []
    for h in range(w.n_kv_heads):
        # For each group, the latest block that may route to it: group j's chunk
        # c must satisfy sink/C <= c < (b0 - local)/C for that block's b0.
        last_b0 = w.q0 + (n_blocks - 1) * B
        hi_chunk = (last_b0 - w.local) // C          # exclusive
        lo_chunk = w.sink // C
        if hi_chunk <= lo_chunk:
            continue
        for _ in range(w.n_needles):
            c = int(rng.integers(lo_chunk, hi_chunk))
            j = c * (C // g) + int(rng.integers(0, C // g))
            # blocks b with (b0 - local)/C > c  <=>  b0 > c*C + local
            first_b0 = c * C + w.local + C
            b_first = max(0, -(-(first_b0 - w.q0) // B))
            b_star = int(rng.integers(b_first, n_blocks))
            b0 = w.q0 + b_star * B
            rows = q64[b0 - w.q0: min(b0 + B, w.T) - w.q0, h * G:(h + 1) * G, :]
            mean_q = rows.reshape(-1, w.head_dim).mean(axis=0)
            noise = rng.standard_normal((g, w.head_dim))
            k_out[h, j * g:(j + 1) * g, :] = 0.8 * mean_q[None, :] + 0.2 * noise
            out.append((h, j, b_star))
    return out


def to_f64(t: torch.Tensor) -> np.ndarray:
    """Exact float64 copy of a storage-dtype tensor (bf16 and fp32 widen exactly)."""
    return t.detach().to(torch.float64).cpu().numpy()
