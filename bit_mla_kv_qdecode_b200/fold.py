"""Offline folding of QuantMLA's path-specific transforms into MLA weights.

This runs once, before serving, on the weights; nothing here is on the decode
path (the decode kernels see only the already-transformed cache and queries).

QuantMLA (arxivdaily.com/papers/2609.36760, abstract; podcast episode,
researchpod.app, the passages on the transformation spaces) transforms each
cache path so that full-precision computation is unchanged and the transform
fuses into existing parameters:

* Content path: c' = T c with T = D R (channel scaling D, rotation R). The
  cache stores c'. The down-projection absorbs T (W_DKV' = T W_DKV) and every
  consumer of c absorbs T^-1 (W_UK' = W_UK T^-1, W_UV' = W_UV T^-1), so keys,
  values and scores are unchanged.
* RoPE path: M acts inside each rotary pair as a 2-D rotation and one shared
  scale, M = (+)_i s_i R(phi_i). Such an M commutes with RoPE (2-D rotations
  commute; the scale is uniform in the pair), so it folds into the key
  projection before RoPE (W_KR' = M W_KR) and the query side takes the
  reciprocal M^-T = (+)_i s_i^-1 R(phi_i) (W_QR' = M^-T W_QR), preserving every
  positional score q_r . k_r.

Learning the transforms (the pages' function-aligned objectives) needs model
weights and calibration data and is not done here; callers pass the
transforms. Float64 numpy throughout.
"""
from __future__ import annotations

import numpy as np


def rotary_pairs(d: int, convention: str = "interleaved") -> np.ndarray:
    """Index pairs [d/2, 2] a rotary embedding rotates together: (2i, 2i+1)
    ("interleaved") or (i, i + d/2) ("half")."""
    if d % 2:
        raise ValueError("rotary width must be even")
    i = np.arange(d // 2)
    if convention == "interleaved":
        return np.stack([2 * i, 2 * i + 1], axis=1)
    if convention == "half":
        return np.stack([i, i + d // 2], axis=1)
    raise ValueError(f"unknown rotary convention {convention!r}")


def rope(x: np.ndarray, pos, base: float = 10000.0, convention: str = "interleaved") -> np.ndarray:
    """Rotary embedding of x [..., d] at integer positions pos (broadcast over
    the leading axes): pair i turns by pos * base^(-2i/d)."""
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    pr = rotary_pairs(d, convention)
    theta = np.asarray(pos, dtype=np.float64)[..., None] * base ** (-2.0 * np.arange(d // 2) / d)
    cos, sin = np.cos(theta), np.sin(theta)
    out = x.copy()
    a, b = x[..., pr[:, 0]], x[..., pr[:, 1]]
    out[..., pr[:, 0]] = a * cos - b * sin
    out[..., pr[:, 1]] = a * sin + b * cos
    return out


def content_transform(rotation: np.ndarray, scale: np.ndarray) -> np.ndarray:
    """T = diag(scale) @ rotation for the content latent (rotation orthogonal,
    scale positive)."""
    rotation = np.asarray(rotation, dtype=np.float64)
    scale = np.asarray(scale, dtype=np.float64)
    if rotation.shape != (scale.size, scale.size):
        raise ValueError("rotation must be square with one scale per channel")
    if not np.allclose(rotation @ rotation.T, np.eye(scale.size), atol=1e-10):
        raise ValueError("rotation must be orthogonal")
    if np.any(scale <= 0):
        raise ValueError("scales must be positive")
    return scale[:, None] * rotation


def rope_pair_transform(angles: np.ndarray, scales: np.ndarray, convention: str = "interleaved") -> np.ndarray:
    """M = (+)_i s_i R(phi_i) acting on the rotary pairs of a d_r = 2 * len(angles) vector."""
    angles = np.asarray(angles, dtype=np.float64)
    scales = np.asarray(scales, dtype=np.float64)
    if angles.shape != scales.shape or np.any(scales <= 0):
        raise ValueError("one angle and one positive scale per rotary pair")
    d = 2 * angles.size
    pr = rotary_pairs(d, convention)
    M = np.zeros((d, d))
    c, s = np.cos(angles) * scales, np.sin(angles) * scales
    M[pr[:, 0], pr[:, 0]] = c
    M[pr[:, 0], pr[:, 1]] = -s
    M[pr[:, 1], pr[:, 0]] = s
    M[pr[:, 1], pr[:, 1]] = c
    return M


def fold_content(W_dkv: np.ndarray, W_uk: np.ndarray, W_uv: np.ndarray, T: np.ndarray):
    """Fold the content transform: returns (T W_dkv, W_uk T^-1, W_uv T^-1).

    W_dkv [d_c, d_model] produces the latent; W_uk [H, d_h, d_c] and
    W_uv [H, d_v, d_c] up-project it per head."""
    Tinv = np.linalg.inv(np.asarray(T, dtype=np.float64))
    return T @ W_dkv, np.asarray(W_uk, dtype=np.float64) @ Tinv, np.asarray(W_uv, dtype=np.float64) @ Tinv


def fold_rope(W_kr: np.ndarray, W_qr: np.ndarray, M: np.ndarray):
    """Fold the RoPE-path transform: returns (M W_kr, M^-T W_qr).

    W_kr [d_r, d_model] is the shared decoupled key projection (before RoPE),
    W_qr [H, d_r, d_q] the per-head decoupled query projection (before RoPE)."""
    Minv_t = np.linalg.inv(np.asarray(M, dtype=np.float64)).T
    return M @ W_kr, Minv_t @ np.asarray(W_qr, dtype=np.float64)
