"""The device-side timeout path of the tensor-core decode, run without a fault.

MLA_DECODE_TEST_STALL makes the kernel's page producer never load one chunk
and shortens every bounded wait to 1 ms: the consumers' waits run out, the
kernel records MLA_ERR_TIMEOUT, drains its copies and MMAs and exits. The
call must return, the status word must report the timeout (and read as clear
afterwards), and the next normal call must reproduce a clean run bit for bit.
"""
import pytest
import torch

from bit_mla_kv_qdecode_b200 import api, synth
from bit_mla_kv_qdecode_b200._lib import MLA_DECODE_TEST_STALL, MLA_ERR_TIMEOUT
from tests import mla_cases as mc

pytestmark = pytest.mark.gpu


def _decode(case, pool, table_t, flags, num_splits):
    w = case.w
    qc, qr = mc.device_queries(case)
    lens_t = torch.from_numpy(case.lens).cuda()
    lse = torch.full((w.B, w.s_q, w.H), 7.0, dtype=torch.float32, device="cuda")
    out = torch.full((w.B, w.s_q, w.H, 512), 7.0, dtype=torch.float32, device="cuda")
    api.mla_qdecode(case.desc, pool, table_t, lens_t, case.max_seq_len, qc, qr, w.scale, out=out, lse=lse,
                    num_splits=num_splits, flags=flags)
    torch.cuda.synchronize()
    return out, lse


@pytest.mark.parametrize("num_splits", [1, 2])
@pytest.mark.parametrize("quantized", [True, False])
def test_timeout_reports_and_next_call_is_clean(num_splits, quantized):
    w = synth.workload(2).scaled(B=2, H=128, s_q=1)
    case = mc.make_case(w, lens=[300, 1000])
    pool, table_t = mc.fill_pool(case, quantized=quantized)
    if not quantized:
        def run(flags):
            w_ = case.w
            qc, qr = mc.device_queries(case)
            lens_t = torch.from_numpy(case.lens).cuda()
            lse = torch.full((w_.B, w_.s_q, w_.H), 7.0, dtype=torch.float32, device="cuda")
            out = torch.full((w_.B, w_.s_q, w_.H, 512), 7.0, dtype=torch.float32, device="cuda")
            api.mla_decode_bf16(pool, table_t, lens_t, case.max_seq_len, qc, qr, w_.scale, out=out, lse=lse,
                                num_splits=num_splits, flags=flags)
            torch.cuda.synchronize()
            return out, lse
    else:
        def run(flags):
            return _decode(case, pool, table_t, flags, num_splits)
    ref = run(0)
    assert api.mla_get_device_status() == 0
    run(MLA_DECODE_TEST_STALL)  # returns: every wait is bounded
    assert api.mla_get_device_status() == MLA_ERR_TIMEOUT
    assert api.mla_get_device_status() == 0  # reading clears the word
    again = run(0)
    assert api.mla_get_device_status() == 0
    assert torch.equal(ref[0], again[0]) and torch.equal(ref[1], again[1])
    if quantized:
        err, lerr = mc.parity(again[0], again[1], mc.oracle_decode(case, [0, 1]))
        assert err <= mc.RTOL_RMS and lerr <= mc.LSE_ATOL
