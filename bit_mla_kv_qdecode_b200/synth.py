"""Seeded synthetic inputs for the low-bit MLA decode workloads.

This module only draws inputs. It holds none of the method's arithmetic (no
quantizer, no packing, no attention), so both the CUDA path and the CPU oracle
can consume what it produces without sharing any of the computation.

Workloads (shapes and value distributions of the QuantMLA setting: an MLA
cache with a 512-wide content latent c_kv and a 64-wide decoupled RoPE key
k_r, "QuantMLA" abstract, arxivdaily.com/papers/2609.36760):

  0  tiny:      B=1,   H=16,  s_q=1, T=1024,            INT4/INT4 g64, contiguous
  1  dsv3:      B=32,  H=128, s_q=1, T=4096,            INT4/INT4 g64, paged
  2  mixed:     B=64,  H=128, s_q=1, T~U[2048,16384],   INT2 g32 / INT4 g64, 1% outliers x8
  3  long:      B=4,   H=128, s_q=1, T=131072,          INT4/INT4 g64, 32 splits (+ BF16 run)
  4  mtp:       B=128, H=128, s_q=2 causal, T~U[1024,32768], INT2 g32 / INT4 g64, append 2
  5  membound:  B=64,  H=16,  s_q=1, T=32768,           INT4/INT4 g64 (memory-bound supplement)

Value recipe, per workload with seed = workload index:
  * per-channel magnitudes mag_j = exp(N(0, 0.5^2)) for the 576 concatenated
    [c_kv | k_r] channels, shared by every token of every request;
  * outliers (workload 2): round(1% * 576) = 6 channels drawn without
    replacement among the 576 get mag_j *= 8;
  * cache values x[t, j] = N(0,1) * mag_j, rounded to bf16;
  * queries q_c, q_r are bf16 N(0,1);
  * ragged lengths are integer-uniform on the inclusive range;
  * block table: a random permutation of the pool's pages, handed out in
    request order (workload 0: the identity, i.e. a contiguous cache).

Every request draws from its own stream (seed, 1, b), so any request's tokens
can be regenerated on their own, without the rest of the batch.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np

D_C = 512
D_R = 64
D_QK = D_C + D_R
PAGE = 64


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    index: int
    B: int
    H: int
    s_q: int
    t_lo: int
    t_hi: int
    bits_c: int
    group_c: int
    bits_r: int
    group_r: int
    paged: bool
    outlier_frac: float
    n_new: int
    num_splits: int  # 0 = let the library choose
    bf16_compare: bool = False

    @property
    def seed(self) -> int:
        return self.index

    @property
    def scale(self) -> float:
        # 1/sqrt(d_nope + d_rope) with the DeepSeek-V3 head dims 128 + 64
        return 1.0 / math.sqrt(192.0)

    def scaled(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS = [
    Workload("tiny", 0, 1, 16, 1, 1024, 1024, 4, 64, 4, 64, False, 0.0, 1, 0),
    Workload("dsv3", 1, 32, 128, 1, 4096, 4096, 4, 64, 4, 64, True, 0.0, 1, 0),
    Workload("mixed", 2, 64, 128, 1, 2048, 16384, 2, 32, 4, 64, True, 0.01, 1, 0),
    Workload("long", 3, 4, 128, 1, 131072, 131072, 4, 64, 4, 64, True, 0.0, 1, 32, True),
    Workload("mtp", 4, 128, 128, 2, 1024, 32768, 2, 32, 4, 64, True, 0.0, 2, 0),
    Workload("membound", 5, 64, 16, 1, 32768, 32768, 4, 64, 4, 64, True, 0.0, 1, 0),
]


def workload(i_or_name) -> Workload:
    for w in WORKLOADS:
        if w.index == i_or_name or w.name == i_or_name:
            return w
    raise KeyError(i_or_name)


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (nearest, ties to even); return uint16 bits."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32)
    # 32-bit arithmetic: the sum stays below 2^32 for every finite or infinite
    # input (only NaN payloads with all high bits set could carry out)
    u = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    return u.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def channel_magnitudes(w: Workload) -> np.ndarray:
    rng = np.random.default_rng([w.seed, 3])
    mag = np.exp(rng.normal(0.0, 0.5, D_QK))
    n_out = int(round(w.outlier_frac * D_QK))
    if n_out:
        idx = rng.choice(D_QK, n_out, replace=False)
        mag[idx] *= 8.0
    return mag.astype(np.float32)


def seq_lens(w: Workload) -> np.ndarray:
    """Keys visible to the last query of each request (after the step's append)."""
    if w.t_lo == w.t_hi:
        return np.full(w.B, w.t_lo, dtype=np.int32)
    rng = np.random.default_rng([w.seed, 0])
    return rng.integers(w.t_lo, w.t_hi + 1, size=w.B).astype(np.int32)


def cache_tokens_bf16(w: Workload, b: int, n_tokens: int, mag=None) -> np.ndarray:
    """uint16 bf16 bits [n_tokens, 576] of request b's tokens 0..n_tokens-1."""
    if mag is None:
        mag = channel_magnitudes(w)
    rng = np.random.default_rng([w.seed, 1, b])
    x = rng.standard_normal((n_tokens, D_QK), dtype=np.float32)
    x *= mag[None, :]
    return f32_to_bf16_bits(x)


def queries_bf16(w: Workload):
    """(q_c bits [B, s_q, H, 512], q_r bits [B, s_q, H, 64]) as uint16 bf16."""
    rng = np.random.default_rng([w.seed, 2])
    q = rng.standard_normal((w.B, w.s_q, w.H, D_QK), dtype=np.float32)
    qb = f32_to_bf16_bits(q)
    return np.ascontiguousarray(qb[..., :D_C]), np.ascontiguousarray(qb[..., D_C:])


def pages_per_request(lens: np.ndarray, headroom: int = 0) -> np.ndarray:
    return ((np.asarray(lens, dtype=np.int64) + headroom + PAGE - 1) // PAGE).astype(np.int32)


def block_table(w: Workload, lens: np.ndarray, headroom: int = 0):
    """(table int32 [B, max_pages], num_pages). Unused entries are -1."""
    ppr = pages_per_request(lens, headroom)
    num_pages = int(ppr.sum())
    maxp = int(ppr.max()) if len(ppr) else 0
    table = np.full((len(ppr), max(maxp, 1)), -1, dtype=np.int32)
    if w.paged:
        perm = np.random.default_rng([w.seed, 4]).permutation(num_pages).astype(np.int32)
    else:
        perm = np.arange(num_pages, dtype=np.int32)
    off = 0
    for b, n in enumerate(ppr):
        table[b, :n] = perm[off:off + n]
        off += n
    return table, num_pages
