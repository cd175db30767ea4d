"""Oracle attention: dequantize-then-attend in float64, absorbed MQA form.

Sources:
* Group-Query Latent Attention abstract (thelatestinai.com/papers/2607.27269):
  MLA compresses keys and values into one low-rank latent, and its trained
  weights expose a single decoding path, an absorbed MQA form -- every head
  attends the same shared latent.
* QuantMLA (arxivdaily.com/papers/2609.36760), English abstract: the cache has
  a content path and a decoupled RoPE path; the native kernel unpacks and
  dequantizes inside the attention computation.

For request b, query i in [0, s_q) and head h (readings, stated once here):

  L_{b,i} = seq_len_b - s_q + 1 + i        query i sits at position
                                            seq_len_b - s_q + i and sees keys
                                            0..its own position (causal)
  S_t     = scale * (q_c . c_hat_t + q_r . kr_hat_t),   t < L_{b,i}
  p_t     = exp(S_t - max S) / sum_t exp(S_t - max S)
  o       = sum_t p_t c_hat_t               (latent-space output, 512 wide)
  lse     = max S + ln sum_t exp(S_t - max S)

k_r in the cache and q_r arrive already rotated (RoPE applied upstream, the
learned transforms folded offline), so no rotation happens here. A row that
sees no key has o = 0 and lse = -inf. scale multiplies the sum of both dot
products.
"""
from __future__ import annotations

import numpy as np

from . import layout


def visible_keys(seq_len: int, s_q: int, i: int) -> int:
    return max(0, int(seq_len) - s_q + 1 + i)


def attend(qc, qr, C, R, scale: float, L):
    """Rows of queries against one request's keys.

    qc [rows, d_c], qr [rows, d_r], C [T, d_c], R [T, d_r] (any float),
    L [rows] visible-key counts. Returns (o float64 [rows, d_c], lse [rows]).
    """
    qc = np.asarray(qc, dtype=np.float64)
    qr = np.asarray(qr, dtype=np.float64)
    C = np.asarray(C, dtype=np.float64)
    R = np.asarray(R, dtype=np.float64)
    L = np.asarray(L, dtype=np.int64)
    rows = qc.shape[0]
    T = C.shape[0]
    o = np.zeros((rows, C.shape[1]), dtype=np.float64)
    lse = np.full(rows, -np.inf, dtype=np.float64)
    if T == 0 or rows == 0:
        return o, lse
    S = (qc @ C.T + qr @ R.T) * float(scale)
    valid = np.arange(T)[None, :] < L[:, None]
    S = np.where(valid, S, -np.inf)
    live = L > 0
    if not live.any():
        return o, lse
    m = S[live].max(axis=1, keepdims=True)
    p = np.exp(S[live] - m)
    l_ = p.sum(axis=1, keepdims=True)
    o[live] = (p @ C) / l_
    lse[live] = (m + np.log(l_))[:, 0]
    return o, lse


def softmax_weights(qc, qr, C, R, scale: float, L):
    """The probabilities p [rows, T] that ``attend`` uses (for invariant checks)."""
    qc = np.asarray(qc, dtype=np.float64)
    qr = np.asarray(qr, dtype=np.float64)
    S = (qc @ np.asarray(C, np.float64).T + qr @ np.asarray(R, np.float64).T) * float(scale)
    T = S.shape[1]
    S = np.where(np.arange(T)[None, :] < np.asarray(L)[:, None], S, -np.inf)
    m = S.max(axis=1, keepdims=True)
    p = np.exp(S - m)
    return p / p.sum(axis=1, keepdims=True)


def request_rows(qc_b, qr_b, seq_len: int):
    """Flatten one request's queries [s_q, H, d] into rows r = i*H + h with their L."""
    s_q, H = qc_b.shape[:2]
    L = np.repeat([visible_keys(seq_len, s_q, i) for i in range(s_q)], H)
    return qc_b.reshape(s_q * H, -1), qr_b.reshape(s_q * H, -1), L


def qdecode(desc: layout.Desc, pool, table, seq_lens, qc, qr, scale: float, requests=None):
    """Decode over an oracle-packed pool.

    qc [B, s_q, H, d_c], qr [B, s_q, H, d_r] (float values of the bf16 inputs).
    Returns o float64 [B, s_q, H, d_c] and lse [B, s_q, H] for the requested
    batch rows (all by default; other rows stay zero / -inf).
    """
    B, s_q, H = qc.shape[:3]
    o = np.zeros((B, s_q, H, desc.d_c))
    lse = np.full((B, s_q, H), -np.inf)
    for b in (range(B) if requests is None else requests):
        T = int(seq_lens[b])
        C, R = layout.gather_tokens(desc, pool, table[b], T)
        rq_c, rq_r, L = request_rows(qc[b], qr[b], T)
        ob, lb = attend(rq_c, rq_r, C, R, scale, L)
        o[b] = ob.reshape(s_q, H, -1)
        lse[b] = lb.reshape(s_q, H)
    return o, lse


def decode_bf16(pool_f32, table, seq_lens, qc, qr, scale: float, requests=None, page_size=64):
    """Unquantized decode over a pool of bf16 values [num_pages, P, d_c + d_r]."""
    B, s_q, H, d_c = qc.shape
    o = np.zeros((B, s_q, H, d_c))
    lse = np.full((B, s_q, H), -np.inf)
    for b in (range(B) if requests is None else requests):
        T = int(seq_lens[b])
        C, R = layout.bf16_pool_gather(pool_f32, table[b], T, page_size, d_c)
        rq_c, rq_r, L = request_rows(qc[b], qr[b], T)
        ob, lb = attend(rq_c, rq_r, C, R, scale, L)
        o[b] = ob.reshape(s_q, H, -1)
        lse[b] = lb.reshape(s_q, H)
    return o, lse


def hybrid_decode(desc: layout.Desc, pool, table, hist_lens, prot_pool_f32, prot_table, prot_lens, qc, qr,
                  scale: float, requests=None, page_size=64):
    """Decode over a hybrid cache: BF16 protection of the earliest tokens and a
    recent window, the history between them quantized; the history stays
    visible, only its storage precision differs (QuantMLA podcast episode,
    researchpod.app, the passage on keeping history uncompressed).
    Per request b (readings, stated here): the protected segment holds
    prot_lens[b] tokens of a BF16 pool in position order -- the sink, then the
    window, the newest s_q keys last; the quantized pool holds the hist_lens[b]
    history tokens, all older than every query. Query i sees every history key
    and the first prot_lens[b] - s_q + 1 + i protected keys. One softmax over
    both segments. qc, qr as in ``qdecode``; prot_pool_f32 [num_pages, P, d_c + d_r].
    """
    B, s_q, H = qc.shape[:3]
    o = np.zeros((B, s_q, H, desc.d_c))
    lse = np.full((B, s_q, H), -np.inf)
    for b in (range(B) if requests is None else requests):
        Th, Tp = int(hist_lens[b]), int(prot_lens[b])
        Ch, Rh = layout.gather_tokens(desc, pool, table[b], Th)
        Cp, Rp = layout.bf16_pool_gather(prot_pool_f32, prot_table[b], Tp, page_size, desc.d_c)
        rq_c, rq_r, Lp = request_rows(qc[b], qr[b], Tp)
        ob, lb = attend(rq_c, rq_r, np.concatenate([Ch, Cp]), np.concatenate([Rh, Rp]), scale, Th + Lp)
        o[b] = ob.reshape(s_q, H, -1)
        lse[b] = lb.reshape(s_q, H)
    return o, lse


def combine(o_parts, lse_parts):
    """Merge split-KV partial results.

    o_parts [n, rows, d], lse_parts [n, rows]; each partial is normalised
    within its own key chunk. lse = log sum_j exp(lse_j); o = sum_j
    exp(lse_j - lse) o_j. Chunks with lse_j = -inf carry weight 0; a row
    whose every chunk is empty gives o = 0, lse = -inf.
    """
    o_parts = np.asarray(o_parts, dtype=np.float64)
    lse_parts = np.asarray(lse_parts, dtype=np.float64)
    n, rows, d = o_parts.shape
    o = np.zeros((rows, d))
    lse = np.full(rows, -np.inf)
    m = lse_parts.max(axis=0)
    live = np.isfinite(m)
    if not live.any():
        return o, lse
    w = np.exp(lse_parts[:, live] - m[live][None, :])
    tot = w.sum(axis=0)
    lse[live] = m[live] + np.log(tot)
    o[live] = np.einsum("nr,nrd->rd", w / tot[None, :], o_parts[:, live])
    return o, lse


def attend_chunked(qc, qr, C, R, scale: float, L, chunk: int):
    """Attend each key chunk [k*chunk, (k+1)*chunk) alone, then ``combine``."""
    T = C.shape[0]
    L = np.asarray(L)
    parts_o, parts_l = [], []
    for t0 in range(0, max(T, 1), chunk):
        t1 = min(T, t0 + chunk)
        Lc = np.clip(L - t0, 0, t1 - t0)
        o, l_ = attend(qc, qr, C[t0:t1], R[t0:t1], scale, Lc)
        parts_o.append(o)
        parts_l.append(l_)
    return combine(np.stack(parts_o), np.stack(parts_l))
