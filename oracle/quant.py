"""Oracle quantizer: per-token, per-group asymmetric round-to-nearest.

Source: QuantMLA (arxivdaily.com/papers/2609.36760), English abstract -- joint
INT4 caching of the content and RoPE caches, or INT2 content with INT4 RoPE;
QuantMLA podcast episode (researchpod.app), passage on baselines -- the
comparison methods share one round-to-nearest quantizer with QuantMLA. The
pages give no formula; the plainest reading, used here:

  for one token's channel group x[0..g) and b bits, qmax = 2^b - 1:
    mn = min(x) + 0, mx = max(x)                (exact on the bf16 inputs; +0
                                                 makes a -0.0 minimum +0.0)
    s  = fp16( fp32( fp32(mx - mn) / qmax ) )   (IEEE fp32 ops, then RN to fp16)
    z  = fp16( mn )
    u  = 0                                       if s == 0
         clamp( rint( fp32( fp32(x - z) / s ) ), 0, qmax )   otherwise
    x_hat = u * s + z

Readings: the zero-point is a float offset equal to the group minimum (the
workload stores "fp16 scale + zero"); encode uses the rounded fp16 s and z so
encode and decode agree; ties round half to even; a constant group has s == 0
and decodes exactly to z; the clamp absorbs fp16 rounding of s and z; groups
run along channels within a token starting at channel 0.

Decisions (the integer codes) are taken in fp32, the precision the CUDA
kernel uses, so the two agree bit for bit. Dequantization is float64, where it
is exact (u*s has at most 15 significant bits; fp16 exponents span < 40).

Bit packing (a reading; the pages are silent): little-endian within a byte,
element j of a token's code row at byte floor(j*b/8), bit (j*b) mod 8. So for
INT4 the even channel is the low nibble; for INT2 channel 4i+k sits at bits
2k..2k+1 of byte i.
"""
from __future__ import annotations

import numpy as np


def qmax_of(bits: int) -> int:
    return (1 << bits) - 1


def quantize_groups(x, bits: int, group: int):
    """Quantize float32 values x [N, D] per (token, group).

    Returns (codes uint8 [N, D], s fp16 [N, D/group], z fp16 [N, D/group]).
    """
    x = np.asarray(x, dtype=np.float32)
    n, d = x.shape
    if d % group:
        raise ValueError("channel count must be a multiple of the group size")
    xg = x.reshape(n, d // group, group)
    # adding +0 turns a minimum of -0.0 into +0.0, so the zero-point of a
    # group whose minimum is a signed zero does not depend on which zero a
    # min-reduction happens to return
    mn = np.add(xg.min(axis=-1), np.float32(0), dtype=np.float32)
    mx = xg.max(axis=-1)
    qmax = np.float32(qmax_of(bits))
    rng_ = np.subtract(mx, mn, dtype=np.float32)
    s32 = np.divide(rng_, qmax, dtype=np.float32)
    s16 = s32.astype(np.float16)
    z16 = mn.astype(np.float16)
    s = s16.astype(np.float32)[..., None]
    z = z16.astype(np.float32)[..., None]
    diff = np.subtract(xg, z, dtype=np.float32)
    with np.errstate(divide="ignore", invalid="ignore"):
        t = np.divide(diff, s, dtype=np.float32)
    u = np.where(s == 0, np.float32(0), np.clip(np.rint(t), np.float32(0), qmax))
    return u.astype(np.uint8).reshape(n, d), s16, z16


def dequantize_groups(codes, s16, z16, group: int) -> np.ndarray:
    """x_hat = u*s + z in float64, [N, D]."""
    codes = np.asarray(codes)
    n, d = codes.shape
    u = codes.astype(np.float64).reshape(n, d // group, group)
    s = np.asarray(s16, dtype=np.float16).astype(np.float64)[..., None]
    z = np.asarray(z16, dtype=np.float16).astype(np.float64)[..., None]
    return (u * s + z).reshape(n, d)


def pack_codes(codes, bits: int) -> np.ndarray:
    """uint8 codes [N, D] -> packed bytes [N, D*bits/8]."""
    codes = np.asarray(codes, dtype=np.uint8)
    per = 8 // bits
    n, d = codes.shape
    if d % per:
        raise ValueError("channel count must fill whole bytes")
    out = np.zeros((n, d // per), dtype=np.uint8)
    for k in range(per):
        out |= (codes[:, k::per] & qmax_of(bits)) << np.uint8(bits * k)
    return out


def unpack_codes(packed, bits: int, d: int) -> np.ndarray:
    packed = np.asarray(packed, dtype=np.uint8)
    per = 8 // bits
    n = packed.shape[0]
    out = np.empty((n, d), dtype=np.uint8)
    for k in range(per):
        out[:, k::per] = (packed >> np.uint8(bits * k)) & np.uint8(qmax_of(bits))
    return out


def meta_bytes(s16, z16) -> np.ndarray:
    """(s, z) pairs [N, G] -> bytes [N, G*4]: fp16 s at +0, fp16 z at +2, little-endian."""
    s = np.asarray(s16, dtype=np.float16).view(np.uint16)
    z = np.asarray(z16, dtype=np.float16).view(np.uint16)
    pair = np.stack([s, z], axis=-1).astype("<u2")
    n = pair.shape[0]
    return pair.view(np.uint8).reshape(n, -1)


def meta_from_bytes(raw, groups: int):
    raw = np.ascontiguousarray(np.asarray(raw, dtype=np.uint8))
    n = raw.shape[0]
    pair = raw.reshape(n, groups * 4).view("<u2").reshape(n, groups, 2)
    return pair[..., 0].copy().view(np.float16), pair[..., 1].copy().view(np.float16)
