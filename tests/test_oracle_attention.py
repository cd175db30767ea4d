"""Pins for the oracle's absorbed-MQA attention, split-KV merge and paging (CPU).

The central pin is explicit, non-absorbed MLA: per-head keys and values are
built by up-projecting the latent with random W_UK / W_UV and attended the
textbook way; the absorbed oracle must give the same result once its latent
output is projected by W_UV. The rest are closed forms and invariants.
"""
import numpy as np
import pytest

from oracle import attention, layout

SCALE = 1.0 / np.sqrt(192.0)


def _rand(rng, *shape):
    return rng.standard_normal(shape)


def test_absorbed_matches_explicit_mla():
    rng = np.random.default_rng(0)
    H, T, d_nope, d_c, d_r, d_v = 3, 70, 128, 512, 64, 128
    W_UK = _rand(rng, H, d_nope, d_c) / np.sqrt(d_c)
    W_UV = _rand(rng, H, d_v, d_c) / np.sqrt(d_c)
    q_nope = _rand(rng, H, d_nope)
    q_rope = _rand(rng, H, d_r)
    C = _rand(rng, T, d_c)
    R = _rand(rng, T, d_r)
    # explicit multi-head attention with per-head up-projected keys/values
    ref_out, ref_lse = [], []
    for h in range(H):
        K = np.concatenate([C @ W_UK[h].T, R], axis=1)       # [T, 192]
        V = C @ W_UV[h].T                                     # [T, 128]
        q = np.concatenate([q_nope[h], q_rope[h]])            # [192]
        s = (K @ q) * SCALE
        w = np.exp(s - s.max())
        ref_out.append((w / w.sum()) @ V)
        ref_lse.append(s.max() + np.log(w.sum()))
    # absorbed: q_c = W_UK^T q_nope, all heads attend the shared latent
    q_c = np.einsum("hnc,hn->hc", W_UK, q_nope)
    o_lat, lse = attention.attend(q_c, q_rope, C, R, SCALE, np.full(H, T))
    out = np.einsum("hvc,hc->hv", W_UV, o_lat)
    np.testing.assert_allclose(out, np.array(ref_out), rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(lse, np.array(ref_lse), rtol=1e-13)


def test_weights_sum_to_one_and_shift_invariance():
    rng = np.random.default_rng(1)
    rows, T = 5, 90
    qc, qr = _rand(rng, rows, 512), _rand(rng, rows, 64)
    C, R = _rand(rng, T, 512), _rand(rng, T, 64)
    L = np.array([90, 1, 45, 64, 65])
    p = attention.softmax_weights(qc, qr, C, R, SCALE, L)
    np.testing.assert_allclose(p.sum(1), 1.0, rtol=0, atol=1e-12)
    assert np.all(p[1, 1:] == 0) and np.all(p[2, 45:] == 0)
    o, _ = attention.attend(qc, qr, C, R, SCALE, L)
    # shifting every RoPE key by one vector u shifts each head's scores by a
    # constant (q_r . u * scale), so the weights and the output stay the same
    u = _rand(rng, 64) * 3
    o2, _ = attention.attend(qc, qr, C, R + u[None, :], SCALE, L)
    np.testing.assert_allclose(o2, o, rtol=1e-11, atol=1e-12)


def test_single_key_zero_query_and_dominant_key():
    rng = np.random.default_rng(2)
    C, R = _rand(rng, 40, 512), _rand(rng, 40, 64)
    qc, qr = _rand(rng, 1, 512), _rand(rng, 1, 64)
    o, lse = attention.attend(qc, qr, C, R, SCALE, [1])
    assert np.array_equal(o[0], C[0])
    np.testing.assert_allclose(lse[0], SCALE * (qc[0] @ C[0] + qr[0] @ R[0]), rtol=1e-14)
    o, lse = attention.attend(np.zeros((1, 512)), np.zeros((1, 64)), C, R, SCALE, [40])
    np.testing.assert_allclose(o[0], C.mean(0), rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(lse[0], np.log(40.0), rtol=1e-14)
    # raise key 17's score 50 above every other: its weight is 1 - O(40 e^-50)
    s = SCALE * (C @ qc[0] + R @ qr[0])
    boost = (s.max() - s[17] + 50.0) / SCALE / (qr[0] @ qr[0])
    R2 = R.copy()
    R2[17] += boost * qr[0]
    o, _ = attention.attend(qc, qr, C, R2, SCALE, [40])
    np.testing.assert_allclose(o[0], C[17], rtol=1e-12, atol=1e-12)


def test_empty_rows():
    rng = np.random.default_rng(3)
    C, R = _rand(rng, 10, 512), _rand(rng, 10, 64)
    o, lse = attention.attend(_rand(rng, 2, 512), _rand(rng, 2, 64), C, R, SCALE, [0, 3])
    assert np.all(o[0] == 0) and lse[0] == -np.inf and np.isfinite(lse[1])
    o, lse = attention.attend(_rand(rng, 2, 512), _rand(rng, 2, 64), C[:0], R[:0], SCALE, [0, 0])
    assert np.all(o == 0) and np.all(lse == -np.inf)


def test_causal_rows():
    # query i of s_q sits at position seq_len - s_q + i and sees keys up to it
    for seq_len, s_q in [(10, 2), (1, 2), (64, 3), (5, 1)]:
        for i in range(s_q):
            pos = seq_len - s_q + i
            assert attention.visible_keys(seq_len, s_q, i) == len(range(0, pos + 1))
    rng = np.random.default_rng(4)
    T, H = 77, 4
    C, R = _rand(rng, T, 512), _rand(rng, T, 64)
    qc, qr = _rand(rng, 2, H, 512), _rand(rng, 2, H, 64)
    rq_c, rq_r, L = attention.request_rows(qc, qr, T)
    o, _ = attention.attend(rq_c, rq_r, C, R, SCALE, L)
    o0, _ = attention.attend(qc[0], qr[0], C[:T - 1], R[:T - 1], SCALE, np.full(H, T - 1))
    o1, _ = attention.attend(qc[1], qr[1], C, R, SCALE, np.full(H, T))
    np.testing.assert_allclose(o[:H], o0, rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(o[H:], o1, rtol=1e-13, atol=1e-15)


def test_combine_closed_form():
    a, b = np.ones((1, 1, 4)), 3 * np.ones((1, 1, 4))
    o, lse = attention.combine(np.concatenate([a, b]), np.array([[0.7], [0.7]]))
    np.testing.assert_allclose(o, 2.0 * np.ones((1, 4)), rtol=1e-15)
    np.testing.assert_allclose(lse, [0.7 + np.log(2.0)], rtol=1e-15)
    # an empty chunk carries no weight; all chunks empty -> 0, -inf
    o, lse = attention.combine(np.concatenate([a, b]), np.array([[0.1], [-np.inf]]))
    assert np.array_equal(o, a[0]) and lse[0] == 0.1
    o, lse = attention.combine(np.concatenate([a, b]), np.full((2, 1), -np.inf))
    assert np.all(o == 0) and lse[0] == -np.inf


@pytest.mark.parametrize("chunk", [1, 17, 64, 100, 1000])
def test_split_kv_equals_unsplit(chunk):
    rng = np.random.default_rng(5)
    T = 150
    C, R = _rand(rng, T, 512), _rand(rng, T, 64)
    qc, qr = _rand(rng, 4, 512), _rand(rng, 4, 64)
    L = np.array([150, 149, 64, 0])
    o, lse = attention.attend(qc, qr, C, R, SCALE, L)
    o2, lse2 = attention.attend_chunked(qc, qr, C, R, SCALE, L, chunk)
    np.testing.assert_allclose(o2, o, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(lse2[:3], lse[:3], rtol=1e-13)
    assert lse2[3] == -np.inf and np.all(o2[3] == 0)


def test_paging_invariance_and_pool_decode():
    desc = layout.Desc()
    rng = np.random.default_rng(6)
    B, H, s_q = 2, 4, 2
    lens = np.array([130, 64])
    c = (rng.standard_normal((B, 130, 512)).astype(np.float32).view(np.uint32) & 0xFFFF0000).view(np.float32)
    r = (rng.standard_normal((B, 130, 64)).astype(np.float32).view(np.uint32) & 0xFFFF0000).view(np.float32)
    qc, qr = _rand(rng, B, s_q, H, 512), _rand(rng, B, s_q, H, 64)
    outs = []
    for table in (np.array([[0, 1, 2], [3, -1, -1]]), np.array([[3, 0, 2], [1, -1, -1]])):
        pool = layout.new_pool(desc, 4)
        for b in range(B):
            layout.append(desc, pool, table[b:b + 1], [0], c[b:b + 1, :lens[b]], r[b:b + 1, :lens[b]])
        outs.append(attention.qdecode(desc, pool, table, lens, qc, qr, SCALE))
    assert np.array_equal(outs[0][0], outs[1][0]) and np.array_equal(outs[0][1], outs[1][1])
    # and the pool decode equals attending the dequantized tokens directly
    from oracle import quant
    for b in range(B):
        T = lens[b]
        u, s, z = quant.quantize_groups(c[b, :T], 4, 64)
        Ch = quant.dequantize_groups(u, s, z, 64)
        u, s, z = quant.quantize_groups(r[b, :T], 4, 64)
        Rh = quant.dequantize_groups(u, s, z, 64)
        rq_c, rq_r, L = attention.request_rows(qc[b], qr[b], T)
        o, lse = attention.attend(rq_c, rq_r, Ch, Rh, SCALE, L)
        assert np.array_equal(outs[0][0][b].reshape(s_q * H, -1), o)


def _bf16(x):
    return (np.asarray(x, np.float32).view(np.uint32) & 0xFFFF0000).view(np.float32)


@pytest.mark.parametrize("s_q", [1, 2])
def test_hybrid_cache_equals_position_ordered_decode(s_q):
    # The hybrid decode attends [history ; protected] with its own visibility
    # rule. Restated independently: lay the tokens out by position -- sink
    # (first k protected tokens), history, window (rest of the protected
    # segment) -- each with its stored precision, and apply the ordinary causal
    # rule L = T - s_q + 1 + i. Both must agree.
    desc = layout.Desc()
    rng = np.random.default_rng(21)
    B, H, k = 2, 3, 64
    hist = np.array([128, 0])
    win = np.array([70, 5])
    prot = k + win
    T = hist + prot
    c = _bf16(rng.standard_normal((B, T.max(), 512)))
    r = _bf16(rng.standard_normal((B, T.max(), 64)))
    qc, qr = _rand(rng, B, s_q, H, 512), _rand(rng, B, s_q, H, 64)
    pool = layout.new_pool(desc, 4)
    table = np.array([[0, 1], [2, 3]])
    prot_pool = np.zeros((6, 64, 576), np.float32)
    prot_table = np.array([[0, 1, 2], [3, 4, 5]])
    for b in range(B):
        hist_tok = slice(k, k + hist[b])
        prot_tok = np.r_[0:k, k + hist[b]:T[b]]
        if hist[b]:
            layout.append(desc, pool, table[b:b + 1], [0], c[b:b + 1, hist_tok], r[b:b + 1, hist_tok])
        rows = np.concatenate([c[b, prot_tok], r[b, prot_tok]], axis=1)
        for j in range(prot[b]):
            prot_pool[prot_table[b][j // 64], j % 64] = rows[j]
    o, lse = attention.hybrid_decode(desc, pool, table, hist, prot_pool, prot_table, prot, qc, qr, SCALE)
    for b in range(B):
        C = c[b, :T[b]].astype(np.float64).copy()
        R = r[b, :T[b]].astype(np.float64).copy()
        if hist[b]:
            from oracle import quant
            u, s, z = quant.quantize_groups(c[b, k:k + hist[b]], 4, 64)
            C[k:k + hist[b]] = quant.dequantize_groups(u, s, z, 64)
            u, s, z = quant.quantize_groups(r[b, k:k + hist[b]], 4, 64)
            R[k:k + hist[b]] = quant.dequantize_groups(u, s, z, 64)
        rq_c, rq_r, L = attention.request_rows(qc[b], qr[b], T[b])
        ob, lb = attention.attend(rq_c, rq_r, C, R, SCALE, L)
        assert np.allclose(o[b].reshape(s_q * H, -1), ob, rtol=1e-12, atol=1e-12)
        assert np.allclose(lse[b].reshape(-1), lb, rtol=1e-12, atol=1e-12)


def test_hybrid_cache_degenerate_segments():
    # no history: the BF16 decode of the protected segment; no protected
    # keys at s_q = 1: the quantized decode of the history
    desc = layout.Desc()
    rng = np.random.default_rng(22)
    B, H, s_q = 1, 4, 1
    c = _bf16(rng.standard_normal((B, 200, 512)))
    r = _bf16(rng.standard_normal((B, 200, 64)))
    qc, qr = _rand(rng, B, s_q, H, 512), _rand(rng, B, s_q, H, 64)
    prot_pool = np.zeros((4, 64, 576), np.float32)
    for j in range(200):
        prot_pool[j // 64, j % 64] = np.concatenate([c[0, j], r[0, j]])
    pt = np.array([[0, 1, 2, 3]])
    pool = layout.new_pool(desc, 4)
    layout.append(desc, pool, pt, [0], c, r)
    o, lse = attention.hybrid_decode(desc, pool, pt, [0], prot_pool, pt, [200], qc, qr, SCALE)
    o2, lse2 = attention.decode_bf16(prot_pool, pt, [200], qc, qr, SCALE)
    assert np.array_equal(o, o2) and np.array_equal(lse, lse2)
    o, lse = attention.hybrid_decode(desc, pool, pt, [200], prot_pool, pt, [0], qc, qr, SCALE)
    o3, lse3 = attention.qdecode(desc, pool, pt, [200], qc, qr, SCALE)
    assert np.array_equal(o, o3) and np.array_equal(lse, lse3)
