"""Helpers shared by the GPU parity tests: build a workload on the device
through the library's own append, and the matching oracle values on the host.

Inputs come only from ``bit_mla_kv_qdecode_b200.synth``; expected values come
only from ``oracle``. Nothing read back from the device feeds the oracle.
"""
from __future__ import annotations

import dataclasses

import numpy as np
import torch

from bit_mla_kv_qdecode_b200 import api, synth
from oracle import attention, quant

RTOL_RMS = 2e-3    # max |o - o_ref| <= 2e-3 * RMS(o_ref)  (fp32 output)
LSE_ATOL = 2e-3    # |lse - lse_ref| in natural-log units


def bits_to_torch(bits: np.ndarray, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(device).view(torch.bfloat16)


@dataclasses.dataclass
class Case:
    w: synth.Workload
    lens: np.ndarray          # keys visible to the last query of each request
    table: np.ndarray
    num_pages: int
    qc_bits: np.ndarray
    qr_bits: np.ndarray
    mag: np.ndarray
    n_history: np.ndarray     # tokens cached before the step's append

    @property
    def desc(self):
        w = self.w
        return api.make_desc(w.bits_c, w.group_c, w.bits_r, w.group_r, num_pages=self.num_pages)

    def tokens(self, b: int) -> np.ndarray:
        return synth.cache_tokens_bf16(self.w, b, int(self.lens[b]), self.mag)

    @property
    def max_seq_len(self) -> int:
        return int(self.lens.max()) if len(self.lens) else 0


def make_case(w: synth.Workload, lens=None) -> Case:
    lens = synth.seq_lens(w) if lens is None else np.asarray(lens, dtype=np.int32)
    table, num_pages = synth.block_table(w, lens)
    qc, qr = synth.queries_bf16(w)
    n_hist = np.maximum(lens - w.n_new, 0).astype(np.int32)
    return Case(w, lens, table, num_pages, qc, qr, synth.channel_magnitudes(w), n_hist)


def fill_pool(case: Case, quantized=True, upto="all", chunk=8192):
    """Device pool holding each request's tokens [0, n) with n = lens or n_history."""
    dev = "cuda"
    table_t = torch.from_numpy(case.table).to(dev)
    pool = api.new_qcache_pool(case.desc) if quantized else api.new_bf16_pool(case.num_pages)
    for b in range(case.w.B):
        n = int(case.lens[b] if upto == "all" else case.n_history[b])
        if n == 0:
            continue
        toks = case.tokens(b)[:n]
        for t0 in range(0, n, chunk):
            part = toks[t0:t0 + chunk]
            c = bits_to_torch(part[None, :, :512])
            r = bits_to_torch(part[None, :, 512:])
            lb = torch.tensor([t0], dtype=torch.int32, device=dev)
            if quantized:
                api.mla_qcache_append(case.desc, pool, table_t[b:b + 1], lb, c, r)
            else:
                api.mla_bf16cache_append(pool, table_t[b:b + 1], lb, c, r)
    return pool, table_t


def oracle_request(case: Case, b: int, quantized=True):
    """(C_hat, R_hat) float64 of request b's visible tokens, via the oracle quantizer."""
    x = synth.bf16_bits_to_f32(case.tokens(b))
    if not quantized:
        return x[:, :512].astype(np.float64), x[:, 512:].astype(np.float64)
    w = case.w
    u, s, z = quant.quantize_groups(x[:, :512], w.bits_c, w.group_c)
    C = quant.dequantize_groups(u, s, z, w.group_c)
    u, s, z = quant.quantize_groups(x[:, 512:], w.bits_r, w.group_r)
    R = quant.dequantize_groups(u, s, z, w.group_r)
    return C, R


def _oracle_rows(case: Case, b: int, C, R, heads=None):
    """Oracle (o [s_q, H', 512], lse [s_q, H']) of request b over its dequantized keys,
    for every head or only the listed ones."""
    w = case.w
    qc = synth.bf16_bits_to_f32(case.qc_bits[b])
    qr = synth.bf16_bits_to_f32(case.qr_bits[b])
    if heads is not None:
        qc, qr = qc[:, heads], qr[:, heads]
    nh = qc.shape[1]
    rq_c, rq_r, L = attention.request_rows(qc, qr, int(case.lens[b]))
    o, lse = attention.attend(rq_c, rq_r, C, R, w.scale, L)
    return o.reshape(w.s_q, nh, -1), lse.reshape(w.s_q, nh)


def oracle_decode(case: Case, requests, quantized=True, heads=None):
    """{b: (o [s_q, H', 512], lse [s_q, H'])} for the listed requests (H' = len(heads))."""
    return {b: _oracle_rows(case, b, *oracle_request(case, b, quantized), heads=heads) for b in requests}


def fill_pool_with_reference(case: Case, heads, upto="all", chunk=8192, all_heads=()):
    """fill_pool and oracle_decode(heads=...) over every request in one pass: each
    request's tokens are drawn once, appended through the library (its first n
    tokens, n = lens or n_history) and quantized by the oracle (all lens tokens).
    Returns (pool, table, ref over `heads` for every request, ref over every head
    for the requests listed in all_heads)."""
    dev = "cuda"
    w = case.w
    table_t = torch.from_numpy(case.table).to(dev)
    pool = api.new_qcache_pool(case.desc)
    ref, ref_all = {}, {}
    for b in range(w.B):
        toks = case.tokens(b)
        n = int(case.lens[b] if upto == "all" else case.n_history[b])
        for t0 in range(0, n, chunk):
            part = toks[t0:min(t0 + chunk, n)]
            lb = torch.tensor([t0], dtype=torch.int32, device=dev)
            api.mla_qcache_append(case.desc, pool, table_t[b:b + 1], lb, bits_to_torch(part[None, :, :512]),
                                  bits_to_torch(part[None, :, 512:]))
        x = synth.bf16_bits_to_f32(toks)
        u, s, z = quant.quantize_groups(x[:, :512], w.bits_c, w.group_c)
        C = quant.dequantize_groups(u, s, z, w.group_c)
        u, s, z = quant.quantize_groups(x[:, 512:], w.bits_r, w.group_r)
        R = quant.dequantize_groups(u, s, z, w.group_r)
        ref[b] = _oracle_rows(case, b, C, R, heads=heads)
        if b in all_heads:
            ref_all[b] = _oracle_rows(case, b, C, R)
    return pool, table_t, ref, ref_all


def device_queries(case: Case):
    return bits_to_torch(case.qc_bits), bits_to_torch(case.qr_bits)


def parity(out: torch.Tensor, lse: torch.Tensor, ref: dict, bf16_out=False, heads=None):
    """Return (err / RMS, max |lse diff|) over the requests in ref (and, when given,
    only the listed heads, as oracle_decode(heads=...) computed them); assert nothing."""
    o_dev = out.float().cpu().numpy()
    l_dev = lse.cpu().numpy() if lse is not None else None
    if heads is not None:
        o_dev = o_dev[:, :, heads]
        l_dev = l_dev[:, :, heads] if l_dev is not None else None
    refs = np.concatenate([ref[b][0].reshape(-1) for b in ref])
    rms = float(np.sqrt(np.mean(refs ** 2))) if refs.size else 1.0
    worst, lworst = 0.0, 0.0
    for b, (o_ref, lse_ref) in ref.items():
        diff = np.abs(o_dev[b].astype(np.float64) - o_ref)
        if bf16_out:
            diff = np.maximum(diff - half_ulp_bf16(o_ref), 0.0)
        worst = max(worst, float(diff.max()) / rms if diff.size else 0.0)
        if l_dev is not None:
            fin = np.isfinite(lse_ref)
            assert np.array_equal(np.isfinite(l_dev[b]), fin), "lse -inf pattern differs"
            if fin.any():
                lworst = max(lworst, float(np.abs(l_dev[b][fin] - lse_ref[fin]).max()))
    return worst, lworst


def half_ulp_bf16(x: np.ndarray) -> np.ndarray:
    """Half a bf16 ulp of |x| (8 significant bits)."""
    ax = np.abs(x)
    e = np.floor(np.log2(np.where(ax > 0, ax, 1.0)))
    return np.where(ax > 0, 2.0 ** (e - 8), 0.0)
