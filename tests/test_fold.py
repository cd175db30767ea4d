"""Offline transform folding (CPU): equivalence on random synthetic weights.

The transforms change what the cache stores, never what attention computes at
full precision. Checked against an explicit, non-absorbed MLA layer written
out here, and through the oracle's absorbed-MQA decode.
"""
import numpy as np
import pytest

from bit_mla_kv_qdecode_b200 import fold
from oracle import attention

D_MODEL, D_C, D_R, H, D_H, D_V, D_Q = 48, 32, 8, 3, 16, 12, 24


def _orth(rng, n):
    q, r = np.linalg.qr(rng.standard_normal((n, n)))
    return q * np.sign(np.diag(r))


def _weights(rng):
    return dict(W_dkv=rng.standard_normal((D_C, D_MODEL)) / 7, W_uk=rng.standard_normal((H, D_H, D_C)) / 6,
                W_uv=rng.standard_normal((H, D_V, D_C)) / 6, W_kr=rng.standard_normal((D_R, D_MODEL)) / 7,
                W_uq=rng.standard_normal((H, D_H, D_Q)) / 5, W_qr=rng.standard_normal((H, D_R, D_Q)) / 5)


def _mla_layer(W, h, cq, convention):
    """Textbook MLA: per-head keys/values up-projected from the latent, decoupled
    RoPE key shared by the heads, causal softmax. h [T, D_MODEL], cq [s_q, D_Q]
    (queries at positions T - s_q + i). Returns per-head outputs [s_q, H, D_V]
    and the cache (c [T, D_C], k_r [T, D_R])."""
    T, s_q = h.shape[0], cq.shape[0]
    c = h @ W["W_dkv"].T
    kr = fold.rope(h @ W["W_kr"].T, np.arange(T), convention=convention)
    scale = 1.0 / np.sqrt(D_H + D_R)
    out = np.zeros((s_q, H, D_V))
    for i in range(s_q):
        pos = T - s_q + i
        for hh in range(H):
            k = c @ W["W_uk"][hh].T
            v = c @ W["W_uv"][hh].T
            q = W["W_uq"][hh] @ cq[i]
            qr = fold.rope(W["W_qr"][hh] @ cq[i], pos, convention=convention)
            s = (k @ q + kr @ qr) * scale
            s[pos + 1:] = -np.inf
            p = np.exp(s - s.max())
            out[i, hh] = (p / p.sum()) @ v
    return out, c, kr


@pytest.mark.parametrize("convention", ["interleaved", "half"])
def test_pair_transform_commutes_with_rope(convention):
    rng = np.random.default_rng(31)
    M = fold.rope_pair_transform(rng.uniform(-np.pi, np.pi, D_R // 2), rng.uniform(0.3, 3.0, D_R // 2),
                                 convention)
    x = rng.standard_normal((5, D_R))
    pos = np.array([0, 1, 17, 1000, 65535])
    assert np.allclose(fold.rope(x @ M.T, pos, convention=convention),
                       fold.rope(x, pos, convention=convention) @ M.T, atol=1e-12)
    # negative control: a scale that differs inside a pair breaks the commutation
    Mb = M.copy()
    a = fold.rotary_pairs(D_R, convention)[0, 0]
    Mb[:, a] *= 1.5
    assert not np.allclose(fold.rope(x @ Mb.T, pos, convention=convention),
                           fold.rope(x, pos, convention=convention) @ Mb.T, atol=1e-6)


@pytest.mark.parametrize("convention", ["interleaved", "half"])
@pytest.mark.parametrize("s_q", [1, 3])
def test_folded_layer_is_equivalent(convention, s_q):
    rng = np.random.default_rng(32 + s_q)
    W = _weights(rng)
    T = fold.content_transform(_orth(rng, D_C), rng.uniform(0.2, 5.0, D_C))
    M = fold.rope_pair_transform(rng.uniform(-np.pi, np.pi, D_R // 2), rng.uniform(0.2, 5.0, D_R // 2),
                                 convention)
    F = dict(W)
    F["W_dkv"], F["W_uk"], F["W_uv"] = fold.fold_content(W["W_dkv"], W["W_uk"], W["W_uv"], T)
    F["W_kr"], F["W_qr"] = fold.fold_rope(W["W_kr"], W["W_qr"], M)
    h = rng.standard_normal((40, D_MODEL))
    cq = rng.standard_normal((s_q, D_Q))
    o, c, kr = _mla_layer(W, h, cq, convention)
    of, cf, krf = _mla_layer(F, h, cq, convention)
    assert np.allclose(of, o, rtol=1e-10, atol=1e-12)
    # the cache does change: content c' = T c, RoPE key k_r' = M k_r (after RoPE)
    assert np.allclose(cf, c @ T.T, atol=1e-12) and not np.allclose(cf, c, atol=1e-3)
    assert np.allclose(krf, kr @ M.T, atol=1e-12)


def test_absorbed_decode_over_the_folded_cache():
    # decode in the library's form -- q_c = W_uk'^T q per head against the
    # transformed latent, output W_uv' o_latent -- with the oracle's absorbed
    # attention, against the explicit layer on the original weights
    rng = np.random.default_rng(40)
    W = _weights(rng)
    T = fold.content_transform(_orth(rng, D_C), rng.uniform(0.2, 5.0, D_C))
    M = fold.rope_pair_transform(rng.uniform(-np.pi, np.pi, D_R // 2), rng.uniform(0.2, 5.0, D_R // 2))
    F = dict(W)
    F["W_dkv"], F["W_uk"], F["W_uv"] = fold.fold_content(W["W_dkv"], W["W_uk"], W["W_uv"], T)
    F["W_kr"], F["W_qr"] = fold.fold_rope(W["W_kr"], W["W_qr"], M)
    h = rng.standard_normal((33, D_MODEL))
    cq = rng.standard_normal((1, D_Q))
    o_ref, _, _ = _mla_layer(W, h, cq, "interleaved")
    c = h @ F["W_dkv"].T
    kr = fold.rope(h @ F["W_kr"].T, np.arange(33))
    qc = np.stack([F["W_uk"][hh].T @ (F["W_uq"][hh] @ cq[0]) for hh in range(H)])
    qr = np.stack([fold.rope(F["W_qr"][hh] @ cq[0], 32) for hh in range(H)])
    o_lat, _ = attention.attend(qc, qr, c, kr, 1.0 / np.sqrt(D_H + D_R), np.full(H, 33))
    o = np.stack([F["W_uv"][hh] @ o_lat[hh] for hh in range(H)])
    assert np.allclose(o, o_ref[0], rtol=1e-10, atol=1e-12)


def test_invalid_transforms_are_rejected():
    rng = np.random.default_rng(41)
    with pytest.raises(ValueError):
        fold.content_transform(rng.standard_normal((4, 4)), np.ones(4))  # not orthogonal
    with pytest.raises(ValueError):
        fold.content_transform(np.eye(4), np.array([1.0, -1.0, 1.0, 1.0]))  # non-positive scale
    with pytest.raises(ValueError):
        fold.rope_pair_transform(np.zeros(3), np.zeros(3))
