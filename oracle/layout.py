"""Oracle page layout and paged cache writer/reader.

The method stores a packed physical cache with metadata (QuantMLA,
arxivdaily.com/papers/2609.36760, English abstract: "physical cache layout";
QuantMLA podcast episode, researchpod.app, passage on what the compression
figure counts). The pages give no byte layout; this module defines the one the
library uses (version 1), structure-of-arrays per 64-token page, every segment
16-byte aligned:

  [content codes : P x d_c*b_c/8 B][rope codes : P x d_r*b_r/8 B]
  [content (s,z) fp16 pairs : P x d_c/g_c x 4 B][rope (s,z) : P x d_r/g_r x 4 B]

Logical token t of request b lives in page block_table[b][t // P], slot t % P.
A token's codes are one contiguous row of its segment; its metadata likewise.
"""
from __future__ import annotations

import dataclasses

import numpy as np

from . import quant


def _align16(n: int) -> int:
    return (n + 15) // 16 * 16


@dataclasses.dataclass(frozen=True)
class Desc:
    d_c: int = 512
    d_r: int = 64
    bits_c: int = 4
    group_c: int = 64
    bits_r: int = 4
    group_r: int = 64
    page_size: int = 64

    @property
    def code_row_c(self) -> int:
        return self.d_c * self.bits_c // 8

    @property
    def code_row_r(self) -> int:
        return self.d_r * self.bits_r // 8

    @property
    def groups_c(self) -> int:
        return self.d_c // self.group_c

    @property
    def groups_r(self) -> int:
        return self.d_r // self.group_r

    def offsets(self):
        """(content codes, rope codes, content meta, rope meta, page bytes)."""
        p = self.page_size
        o_cc = 0
        o_rc = _align16(o_cc + p * self.code_row_c)
        o_cm = _align16(o_rc + p * self.code_row_r)
        o_rm = _align16(o_cm + p * self.groups_c * 4)
        end = _align16(o_rm + p * self.groups_r * 4)
        return o_cc, o_rc, o_cm, o_rm, end

    @property
    def page_bytes(self) -> int:
        return self.offsets()[4]


def new_pool(desc: Desc, num_pages: int) -> np.ndarray:
    return np.zeros((num_pages, desc.page_bytes), dtype=np.uint8)


def encode_tokens(desc: Desc, c_f32, kr_f32):
    """Quantize and pack tokens: returns per-token byte rows of the four segments."""
    uc, sc, zc = quant.quantize_groups(c_f32, desc.bits_c, desc.group_c)
    ur, sr, zr = quant.quantize_groups(kr_f32, desc.bits_r, desc.group_r)
    return (quant.pack_codes(uc, desc.bits_c), quant.pack_codes(ur, desc.bits_r),
            quant.meta_bytes(sc, zc), quant.meta_bytes(sr, zr))


def append(desc: Desc, pool, table, lens_before, c_new_f32, kr_new_f32):
    """Write new tokens [B, n, d] at positions lens_before[b] + j. In place."""
    o_cc, o_rc, o_cm, o_rm, _ = desc.offsets()
    p = desc.page_size
    B, n = c_new_f32.shape[:2]
    if B == 0 or n == 0:
        return pool
    rows = encode_tokens(desc, c_new_f32.reshape(B * n, desc.d_c),
                         kr_new_f32.reshape(B * n, desc.d_r))
    widths = (desc.code_row_c, desc.code_row_r, desc.groups_c * 4, desc.groups_r * 4)
    bases = (o_cc, o_rc, o_cm, o_rm)
    for b in range(B):
        for j in range(n):
            t = int(lens_before[b]) + j
            page = int(table[b][t // p])
            slot = t % p
            for seg, base, w in zip(rows, bases, widths):
                pool[page, base + slot * w: base + (slot + 1) * w] = seg[b * n + j]
    return pool


def gather_tokens(desc: Desc, pool, table_row, n_tokens: int):
    """Dequantized (C [T, d_c], R [T, d_r]) float64 of one request's first n_tokens."""
    o_cc, o_rc, o_cm, o_rm, _ = desc.offsets()
    p = desc.page_size
    t = np.arange(n_tokens)
    pages = np.asarray(table_row, dtype=np.int64)[t // p]
    slots = t % p

    def seg(base, width):
        idx = base + slots[:, None] * width + np.arange(width)[None, :]
        return pool[pages[:, None], idx]

    uc = quant.unpack_codes(seg(o_cc, desc.code_row_c), desc.bits_c, desc.d_c)
    ur = quant.unpack_codes(seg(o_rc, desc.code_row_r), desc.bits_r, desc.d_r)
    sc, zc = quant.meta_from_bytes(seg(o_cm, desc.groups_c * 4), desc.groups_c)
    sr, zr = quant.meta_from_bytes(seg(o_rm, desc.groups_r * 4), desc.groups_r)
    return (quant.dequantize_groups(uc, sc, zc, desc.group_c),
            quant.dequantize_groups(ur, sr, zr, desc.group_r))


def bf16_pool_gather(pool_f32, table_row, n_tokens: int, page_size: int = 64, d_c: int = 512):
    """Unquantized pool float [num_pages, P, d_c + d_r] -> (C, R) float64 of one request."""
    t = np.arange(n_tokens)
    pages = np.asarray(table_row, dtype=np.int64)[t // page_size]
    rows = np.asarray(pool_f32)[pages, t % page_size].astype(np.float64)
    return rows[:, :d_c], rows[:, d_c:]
