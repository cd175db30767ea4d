"""GPU tests of mla_qdecode_fused_append: the step's cache append fused into the decode.

The fused call must leave the pool byte-identical to mla_qcache_append followed
by mla_qdecode, and return bit-identical outputs (both read the same bytes with
the same kernel); the output also meets the oracle bar.
"""
import numpy as np
import pytest
import torch

from bit_mla_kv_qdecode_b200 import MLA_DECODE_FORCE_SIMT, api, synth
from tests import mla_cases as mc

pytestmark = pytest.mark.gpu

CASES = [
    # (bits_c, group_c, bits_r, group_r, H, s_q, n_new, lens, num_splits, flags)
    (4, 64, 4, 64, 128, 1, 1, [1, 64, 65, 1000], 0, 0),
    (2, 32, 4, 64, 128, 2, 2, [2, 65, 66, 300, 4096], 0, 0),       # new tokens straddle a page edge (63, 64)
    (2, 32, 4, 64, 128, 2, 2, [130, 777], 3, 0),                    # split plan: the last split writes
    (4, 64, 4, 64, 64, 3, 3, [5, 200], 1, 0),                       # 192 rows: two row tiles both write
    (4, 64, 4, 64, 16, 1, 1, [1024, 7], 0, 0),                      # s_q*H <= 16: fused into the small-row kernel
    (4, 64, 4, 64, 8, 2, 2, [64, 65, 700], 3, 0),                   # small-row kernel, tokens straddle a page edge
    (2, 32, 4, 64, 16, 1, 1, [300, 9], 0, 0),                       # s_q*H <= 16, INT2 g32: fused into the small-row kernel
    (2, 64, 2, 32, 8, 2, 2, [64, 65, 129], 2, 0),                   # small-row kernel, INT2 RoPE, page edge
    (4, 64, 4, 64, 128, 1, 2, [90, 3], 2, MLA_DECODE_FORCE_SIMT),   # SIMT path: append kernel, then decode
]


def _new_tokens(case):
    w = case.w
    c = np.zeros((w.B, w.n_new, 512), dtype=np.uint16)
    r = np.zeros((w.B, w.n_new, 64), dtype=np.uint16)
    for b in range(w.B):
        toks = case.tokens(b)[case.n_history[b]:]
        c[b], r[b] = toks[:, :512], toks[:, 512:]
    return mc.bits_to_torch(c), mc.bits_to_torch(r)


@pytest.mark.parametrize("spec", CASES)
def test_fused_matches_append_then_decode(spec):
    bc, gc, br, gr, H, s_q, n_new, lens, num_splits, flags = spec
    w = synth.workload(4).scaled(B=len(lens), H=H, s_q=s_q, n_new=n_new, bits_c=bc, group_c=gc, bits_r=br,
                                 group_r=gr)
    case = mc.make_case(w, lens=lens)
    assert np.all(case.lens - case.n_history == n_new)
    pool0, table_t = mc.fill_pool(case, upto="history")
    c_new, kr_new = _new_tokens(case)
    qc, qr = mc.device_queries(case)
    lens_t = torch.from_numpy(case.lens).cuda()
    hist_t = torch.from_numpy(case.n_history).cuda()
    res = []
    for fused in (False, True):
        pool = pool0.clone()
        lse = torch.empty((w.B, w.s_q, w.H), dtype=torch.float32, device="cuda")
        if fused:
            out, _ = api.mla_qdecode_fused_append(case.desc, pool, table_t, lens_t, case.max_seq_len, c_new, kr_new,
                                                  qc, qr, w.scale, out_dtype=torch.float32, lse=lse,
                                                  num_splits=num_splits, flags=flags)
        else:
            api.mla_qcache_append(case.desc, pool, table_t, hist_t, c_new, kr_new)
            out, _ = api.mla_qdecode(case.desc, pool, table_t, lens_t, case.max_seq_len, qc, qr, w.scale,
                                     out_dtype=torch.float32, lse=lse, num_splits=num_splits, flags=flags)
        torch.cuda.synchronize()
        assert api.mla_get_device_status() == 0
        res.append((pool, out, lse))
    (pa, oa, la), (pb, ob, lb) = res
    assert torch.equal(pa, pb), "pool bytes differ"
    assert torch.equal(oa, ob) and torch.equal(la, lb), "outputs differ"
    ref = mc.oracle_decode(case, range(w.B))
    err, lerr = mc.parity(ob, lb, ref)
    assert err <= mc.RTOL_RMS and lerr <= mc.LSE_ATOL, (err, lerr)


def test_fused_length_below_n_new_is_flagged():
    w = synth.workload(1).scaled(B=2, n_new=2)
    case = mc.make_case(w, lens=[70, 40])
    pool, table_t = mc.fill_pool(case, upto="history")
    c_new, kr_new = _new_tokens(case)
    qc, qr = mc.device_queries(case)
    bad = torch.tensor([70, 1], dtype=torch.int32, device="cuda")  # request 1 holds fewer keys than new tokens
    api.mla_qdecode_fused_append(case.desc, pool, table_t, bad, case.max_seq_len, c_new, kr_new, qc, qr, w.scale)
    torch.cuda.synchronize()
    assert api.mla_get_device_status() == api._lib.MLA_ERR_INVALID_ARG
    assert api.mla_get_device_status() == 0  # reading clears it


def test_fused_full_size_mtp_every_request():
    """The benchmark's timed call on the full speculative-verify workload (128
    requests, 128 heads, 2 causal queries, ragged 1K..32K keys, INT2/INT4, 2 new
    tokens per request): auto split plan, bf16 output, checked against the oracle
    on every request (a fixed head subset) and on two requests in full. The plain
    decode over the pool the fused call left must then give the same bits."""
    heads = [0, 45, 90, 127]
    w = synth.workload(4)
    case = mc.make_case(w)
    pool, table_t, ref, ref_all = mc.fill_pool_with_reference(case, heads, upto="history", all_heads=(0, 77))
    c_new, kr_new = _new_tokens(case)
    qc, qr = mc.device_queries(case)
    lens_t = torch.from_numpy(case.lens).cuda()
    lse = torch.empty((w.B, w.s_q, w.H), dtype=torch.float32, device="cuda")
    out, _ = api.mla_qdecode_fused_append(case.desc, pool, table_t, lens_t, case.max_seq_len, c_new, kr_new,
                                          qc, qr, w.scale, out_dtype=torch.bfloat16, lse=lse,
                                          num_splits=w.num_splits)
    torch.cuda.synchronize()
    assert api.mla_get_device_status() == 0
    err, lerr = mc.parity(out, lse, ref, bf16_out=True, heads=heads)
    assert err <= mc.RTOL_RMS and lerr <= mc.LSE_ATOL, (err, lerr)
    err, lerr = mc.parity(out, lse, ref_all, bf16_out=True)
    assert err <= mc.RTOL_RMS and lerr <= mc.LSE_ATOL, (err, lerr)
    lse2 = torch.empty_like(lse)
    out2, _ = api.mla_qdecode(case.desc, pool, table_t, lens_t, case.max_seq_len, qc, qr, w.scale,
                              out_dtype=torch.bfloat16, lse=lse2, num_splits=w.num_splits)
    torch.cuda.synchronize()
    assert torch.equal(out, out2) and torch.equal(lse, lse2)
