"""GPU parity of the decode path against the float64 oracle.

Bar (fp32 output): max |o - o_ref| <= 2e-3 * RMS(o_ref) over the checked
rows; bf16 output adds half a bf16 ulp of the value. lse within 2e-3.
"""
import numpy as np
import pytest
import torch

from bit_mla_kv_qdecode_b200 import MLA_DECODE_FORCE_SIMT, api, synth
from tests import mla_cases as mc

pytestmark = pytest.mark.gpu

KERNELS = [0, MLA_DECODE_FORCE_SIMT]


def run_decode(case, pool, table_t, flags=0, num_splits=0, out_dtype=torch.float32, quantized=True,
               lens=None):
    w = case.w
    qc, qr = mc.device_queries(case)
    lens_t = torch.from_numpy(case.lens if lens is None else lens).cuda()
    lse = torch.empty((w.B, w.s_q, w.H), dtype=torch.float32, device="cuda")
    if quantized:
        out, _ = api.mla_qdecode(case.desc, pool, table_t, lens_t, case.max_seq_len, qc, qr, w.scale,
                                 out_dtype=out_dtype, lse=lse, num_splits=num_splits, flags=flags)
    else:
        out, _ = api.mla_decode_bf16(pool, table_t, lens_t, case.max_seq_len, qc, qr, w.scale,
                                     out_dtype=out_dtype, lse=lse, num_splits=num_splits, flags=flags)
    torch.cuda.synchronize()
    return out, lse


def check(case, out, lse, requests, quantized=True, bf16_out=False):
    ref = mc.oracle_decode(case, requests, quantized)
    err, lerr = mc.parity(out, lse, ref, bf16_out=bf16_out)
    assert err <= mc.RTOL_RMS, f"max err {err:.3e} x RMS"
    assert lerr <= mc.LSE_ATOL, f"lse err {lerr:.3e}"
    return err


SMALL = [
    # (bits_c, group_c, bits_r, group_r, H, s_q, lens)
    (4, 64, 4, 64, 128, 1, [1, 63, 64, 65, 200, 1000]),
    (2, 32, 4, 64, 128, 1, [130, 1, 777]),
    (2, 32, 4, 64, 128, 2, [2, 65, 300, 1024]),
    (4, 64, 4, 64, 16, 1, [1024, 5]),
    (4, 32, 2, 64, 32, 2, [100, 129]),
    (2, 64, 2, 32, 64, 1, [640, 64]),
    (4, 64, 4, 64, 8, 3, [3, 70]),
    # at most 16 query rows: the warp-level MMA kernel, every format
    (4, 64, 4, 64, 16, 1, [1, 63, 64, 65, 200, 1000]),
    (4, 64, 4, 64, 8, 2, [2, 65, 300, 4096]),
    (4, 64, 4, 64, 5, 3, [100, 1, 129]),
    (4, 64, 4, 64, 1, 1, [33, 640]),
    (2, 32, 4, 64, 16, 1, [1, 65, 1000]),
    (2, 32, 4, 64, 8, 2, [2, 130, 777]),
    (4, 32, 2, 64, 16, 1, [100, 129]),
    (2, 64, 2, 32, 5, 3, [640, 64, 3]),
    (4, 32, 4, 32, 16, 1, [300, 63]),
    (2, 32, 2, 32, 16, 1, [64, 1, 500]),
    (2, 64, 4, 64, 3, 1, [257]),
]


@pytest.mark.parametrize("flags", KERNELS)
@pytest.mark.parametrize("spec", SMALL)
@pytest.mark.parametrize("num_splits", [1, 3, 0])
def test_decode_small_cases(spec, num_splits, flags):
    bc, gc, br, gr, H, s_q, lens = spec
    w = synth.workload(2).scaled(B=len(lens), H=H, s_q=s_q, bits_c=bc, group_c=gc, bits_r=br, group_r=gr)
    case = mc.make_case(w, lens=lens)
    pool, table_t = mc.fill_pool(case)
    out, lse = run_decode(case, pool, table_t, flags=flags, num_splits=num_splits)
    assert api.mla_get_device_status() == 0
    check(case, out, lse, range(w.B))


@pytest.mark.parametrize("flags", KERNELS)
def test_decode_bf16_output(flags):
    w = synth.workload(1).scaled(B=3)
    case = mc.make_case(w, lens=[64, 500, 1])
    pool, table_t = mc.fill_pool(case)
    out, lse = run_decode(case, pool, table_t, flags=flags, out_dtype=torch.bfloat16)
    assert out.dtype == torch.bfloat16
    check(case, out, lse, range(w.B), bf16_out=True)


@pytest.mark.parametrize("flags", KERNELS)
@pytest.mark.parametrize("num_splits", [1, 4])
def test_bf16_cache_decode(flags, num_splits):
    w = synth.workload(3).scaled(B=3, s_q=2)
    case = mc.make_case(w, lens=[65, 1000, 2])
    pool, table_t = mc.fill_pool(case, quantized=False)
    out, lse = run_decode(case, pool, table_t, flags=flags, num_splits=num_splits, quantized=False)
    check(case, out, lse, range(w.B), quantized=False)


BF16_SMALL = [
    # (H, s_q, lens): at most 16 query rows, the warp-level MMA kernel for the BF16 cache
    (16, 1, [1, 31, 32, 33, 63, 64, 65, 1000]),
    (8, 2, [2, 65, 300, 4096]),
    (5, 3, [100, 1, 129]),
    (1, 1, [33, 640]),
]


@pytest.mark.parametrize("spec", BF16_SMALL)
@pytest.mark.parametrize("num_splits", [1, 3, 0])
def test_bf16_cache_small_rows(spec, num_splits):
    H, s_q, lens = spec
    w = synth.workload(3).scaled(B=len(lens), H=H, s_q=s_q)
    case = mc.make_case(w, lens=lens)
    pool, table_t = mc.fill_pool(case, quantized=False)
    out, lse = run_decode(case, pool, table_t, num_splits=num_splits, quantized=False)
    assert api.mla_get_device_status() == 0
    check(case, out, lse, range(w.B), quantized=False)


def test_empty_request_and_length_errors():
    w = synth.workload(1).scaled(B=3)
    case = mc.make_case(w, lens=[0, 70, 0])
    pool, table_t = mc.fill_pool(case)
    for splits in (1, 2):
        out, lse = run_decode(case, pool, table_t, num_splits=splits)
        o = out.cpu().numpy()
        assert np.all(o[0] == 0) and np.all(o[2] == 0)
        assert np.all(np.isneginf(lse.cpu().numpy()[[0, 2]]))
        check(case, out, lse, [1])
    assert api.mla_get_device_status() == 0
    # a device length above max_seq_len is clamped and flagged, never read past
    bad = case.lens.copy()
    bad[1] = 10_000
    run_decode(case, pool, table_t, lens=bad)
    assert api.mla_get_device_status() == api._lib.MLA_ERR_INVALID_ARG


@pytest.mark.parametrize("quantized", [True, False])
@pytest.mark.parametrize("H", [16, 128])
@pytest.mark.parametrize("flags", KERNELS)
@pytest.mark.parametrize("bad_entry", ["past_pool", "unused"])
def test_bad_table_entry_is_flagged(quantized, H, flags, bad_entry):
    # One block-table entry inside request 1's pages names no page of the
    # pool (past its end, or the -1 of an unused slot). Every kernel path
    # (small-row and tensor-core, quantized and BF16, and the SIMT kernel)
    # skips that page without reading it, flags the call in the device status
    # word, and leaves the other requests exact.
    w = synth.workload(1).scaled(B=3, H=H)
    case = mc.make_case(w, lens=[200, 300, 130])
    pool, table_t = mc.fill_pool(case, quantized=quantized)
    assert api.mla_get_device_status() == 0
    bad = table_t.clone()
    bad[1, 2] = case.num_pages + 7 if bad_entry == "past_pool" else -1
    out, lse = run_decode(case, pool, bad, flags=flags, quantized=quantized)
    assert api.mla_get_device_status() == api._lib.MLA_ERR_INVALID_ARG
    assert api.mla_get_device_status() == 0  # reading clears it
    check(case, out, lse, [0, 2], quantized=quantized)


def test_determinism_and_paging_invariance():
    w = synth.workload(2).scaled(B=3, H=128)
    lens = [333, 1024, 65]
    paged = mc.make_case(w, lens=lens)
    flat = mc.make_case(w.scaled(paged=False), lens=lens)
    assert not np.array_equal(paged.table, flat.table)
    outs = []
    for case in (paged, flat):
        pool, table_t = mc.fill_pool(case)
        outs.append(run_decode(case, pool, table_t, num_splits=2))
    again = run_decode(paged, *mc.fill_pool(paged), num_splits=2)
    for a, b in ((outs[0], again), (outs[0], outs[1])):
        assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def test_split_counts_agree():
    w = synth.workload(3).scaled(B=1, t_lo=8192, t_hi=8192)
    case = mc.make_case(w)
    pool, table_t = mc.fill_pool(case)
    ref = mc.oracle_decode(case, [0])
    errs = []
    for splits in (1, 7, 32, 128):
        out, lse = run_decode(case, pool, table_t, num_splits=splits)
        errs.append(mc.parity(out, lse, ref)[0])
    assert max(errs) <= mc.RTOL_RMS, errs


# Full-size workloads in the launch configuration the benchmark times (auto
# split plan, bf16 output), oracle on a sample of requests. The ragged
# workloads (2 and 4) are checked on every request below.
FULL = {0: [0], 1: [0, 31], 3: [2], 5: [3]}

# A fixed subset of heads for the every-request checks: the oracle's cost grows
# with the heads it evaluates, while the kernels treat every head alike (the
# first and last rows of each 128-row tile are among them).
HEADS = [0, 45, 90, 127]


@pytest.mark.parametrize("idx", [2, 4])
def test_full_size_every_request(idx):
    w = synth.workload(idx)
    case = mc.make_case(w)
    pool, table_t, ref, ref_all = mc.fill_pool_with_reference(case, HEADS, all_heads=(5, w.B - 1))
    out, lse = run_decode(case, pool, table_t, num_splits=w.num_splits, out_dtype=torch.bfloat16)
    assert api.mla_get_device_status() == 0
    assert len(ref) == w.B
    err, lerr = mc.parity(out, lse, ref, bf16_out=True, heads=HEADS)
    assert err <= mc.RTOL_RMS and lerr <= mc.LSE_ATOL, (err, lerr)
    err, lerr = mc.parity(out, lse, ref_all, bf16_out=True)
    assert err <= mc.RTOL_RMS and lerr <= mc.LSE_ATOL, (err, lerr)


@pytest.mark.parametrize("idx", sorted(FULL))
def test_full_size_workloads(idx):
    w = synth.workload(idx)
    case = mc.make_case(w)
    pool, table_t = mc.fill_pool(case)
    out, lse = run_decode(case, pool, table_t, num_splits=w.num_splits, out_dtype=torch.bfloat16)
    assert api.mla_get_device_status() == 0
    check(case, out, lse, FULL[idx], bf16_out=True)
    if w.bf16_compare or w.s_q * w.H <= 16:  # the BF16 comparison decode of these shapes too
        del pool
        pool_b, _ = mc.fill_pool(case, quantized=False)
        out, lse = run_decode(case, pool_b, table_t, num_splits=w.num_splits, out_dtype=torch.bfloat16,
                              quantized=False)
        check(case, out, lse, FULL[idx], quantized=False, bf16_out=True)


@pytest.mark.parametrize("fmt", [(2, 32, 4, 64), (4, 32, 2, 32)])
def test_small_rows_full_length_other_formats(fmt):
    # The memory-bound shape (16 query rows, 32,768 keys, paged) in formats
    # other than INT4/INT4 g64, on the small-row kernel with its auto split
    # plan; four requests, every one checked.
    bc, gc, br, gr = fmt
    w = synth.workload(5).scaled(B=4, bits_c=bc, group_c=gc, bits_r=br, group_r=gr)
    case = mc.make_case(w)
    pool, table_t = mc.fill_pool(case)
    out, lse = run_decode(case, pool, table_t, out_dtype=torch.bfloat16)
    assert api.mla_get_device_status() == 0
    check(case, out, lse, range(w.B), bf16_out=True)


def test_long_request_chunk_cap():
    # 32,768 keys asked for as one split: the library raises the split count so
    # that no accumulator sums more than 8,192 keys, which keeps the error well
    # inside the bound (one 32K-key chunk measured 1.75e-3 x RMS)
    w = synth.workload(3).scaled(B=1, t_lo=32768, t_hi=32768)
    assert api.mla_decode_num_splits(1, 1, 128, 32768, 1) == 4
    case = mc.make_case(w)
    pool, table_t = mc.fill_pool(case)
    out, lse = run_decode(case, pool, table_t, num_splits=1)
    err = check(case, out, lse, [0])
    assert err < 1e-3, err


def test_skewed_batch_takes_units_longest_first():
    # One 32,768-key request among 199 short ones (1..399 keys), 128 heads:
    # the split plan's grid runs in several waves, so the tensor-core kernel
    # takes its units from the device-built work list, longest first. Every
    # request matches the oracle, and a second run repeats the first bit for
    # bit (the order decides only which cluster runs a unit).
    lens = [32768] + [int(x) for x in np.random.default_rng(11).integers(1, 400, size=199)]
    w = synth.workload(2).scaled(B=200, H=128, s_q=1)  # INT2 g32 content / INT4 g64 rope
    case = mc.make_case(w, lens=lens)
    n = api.mla_decode_num_splits(w.B, 1, w.H, case.max_seq_len, 0)
    parts = w.B * n * w.H
    partials = ((parts * 4 + 255) // 256) * 256 + parts * 2048
    assert n > 1 and api.mla_decode_workspace_bytes(w.B, 1, w.H, case.max_seq_len, 0) == partials + w.B * n * 4
    pool, table_t, ref, ref_all = mc.fill_pool_with_reference(case, HEADS, all_heads=(0, 7))
    out, lse = run_decode(case, pool, table_t)
    assert api.mla_get_device_status() == 0
    err, lerr = mc.parity(out, lse, ref, heads=HEADS)
    assert err <= mc.RTOL_RMS and lerr <= mc.LSE_ATOL, (err, lerr)
    err, lerr = mc.parity(out, lse, ref_all)
    assert err <= mc.RTOL_RMS and lerr <= mc.LSE_ATOL, (err, lerr)
    again = run_decode(case, pool, table_t)
    assert torch.equal(out, again[0]) and torch.equal(lse, again[1])
