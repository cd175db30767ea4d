"""The allocation-free decode entry point, called through the C ABI.

mla_qdecode_noalloc serves callers that may not call cudaMalloc when they
decode (fixed device-memory budgets, plug-ins whose host framework owns all
device memory, code where an allocation could synchronise the device). It
takes its split-KV scratch from an array compiled into the library, so its
results must equal those of mla_qdecode given a caller-allocated workspace.
This file is named to be collected last, so a run that stops at the first
failure has already run every other test; it also passes on its own.
"""
import ctypes

import numpy as np
import pytest
import torch

from bit_mla_kv_qdecode_b200 import _lib, api, synth
from tests import mla_cases as mc

pytestmark = pytest.mark.gpu


def _noalloc(lib, case, pool, table_t, lens_t, qc, qr, out, lse, splits):
    w = case.w
    return lib.mla_qdecode_noalloc(
        ctypes.byref(case.desc), pool.data_ptr(), table_t.data_ptr(), table_t.shape[1], lens_t.data_ptr(),
        case.max_seq_len, qc.data_ptr(), qr.data_ptr(), w.B, w.s_q, w.H, w.scale, splits, out.data_ptr(),
        1, lse.data_ptr(), 0, torch.cuda.current_stream().cuda_stream)


@pytest.mark.parametrize("idx,lens,splits", [(1, [1000, 77, 513], 3), (4, [300, 65], 2), (3, [8192], 32)])
def test_noalloc_matches_workspace_decode_on_two_calls(idx, lens, splits):
    w = synth.workload(idx).scaled(B=len(lens))
    case = mc.make_case(w, lens=lens)
    pool, table_t = mc.fill_pool(case)
    qc, qr = mc.device_queries(case)
    lens_t = torch.from_numpy(case.lens).cuda()
    shape = (w.B, w.s_q, w.H)
    assert api.mla_decode_workspace_bytes(w.B, w.s_q, w.H, case.max_seq_len, splits) > 0  # scratch is used
    ref_lse = torch.empty(shape, dtype=torch.float32, device="cuda")
    ref, _ = api.mla_qdecode(case.desc, pool, table_t, lens_t, case.max_seq_len, qc, qr, w.scale,
                             out_dtype=torch.float32, lse=ref_lse, num_splits=splits)
    torch.cuda.synchronize()
    ref_np = ref.cpu().numpy().astype(np.float64)
    rms = float(np.sqrt(np.mean(ref_np ** 2)))
    lib = _lib.load()
    for call in range(2):
        out = torch.full((*shape, 512), float("nan"), dtype=torch.float32, device="cuda")
        lse = torch.full(shape, float("nan"), dtype=torch.float32, device="cuda")
        assert _noalloc(lib, case, pool, table_t, lens_t, qc, qr, out, lse, splits) == _lib.MLA_OK
        torch.cuda.synchronize()
        err = float(np.abs(out.cpu().numpy() - ref_np).max()) / rms
        assert err <= mc.RTOL_RMS, (call, err)
        assert float((lse - ref_lse).abs().max()) <= mc.LSE_ATOL, call
    assert api.mla_get_device_status() == 0


def test_noalloc_rejects_shapes_beyond_its_scratch():
    lib = _lib.load()
    B, H, T, splits = 64, 128, 65536, 32
    need = lib.mla_decode_workspace_bytes(B, 1, H, T, splits)
    assert need > _lib.MLA_QDECODE_NOALLOC_SCRATCH_BYTES
    desc = _lib.make_desc(4, 64, 4, 64, num_pages=B * T // 64)
    fake = 0x10000000  # never dereferenced: the size check comes before any launch
    st = lib.mla_qdecode_noalloc(ctypes.byref(desc), fake, fake, T // 64, fake, T, fake, fake, B, 1, H, 0.1,
                                 splits, fake, 1, None, 0, None)
    assert st == _lib.MLA_ERR_WORKSPACE
