"""GPU parity of the cache writer: packed bytes must equal the oracle's, bit for bit."""
import numpy as np
import pytest
import torch

from bit_mla_kv_qdecode_b200 import api, synth
from oracle import layout
from tests import mla_cases as mc

pytestmark = pytest.mark.gpu

BIT_COMBOS = [(4, 64, 4, 64), (2, 32, 4, 64), (4, 32, 2, 64), (2, 64, 2, 32), (4, 64, 2, 32), (2, 32, 4, 32)]


def _oracle_pool(case, desc_np, upto_lens):
    pool = layout.new_pool(desc_np, case.num_pages)
    for b in range(case.w.B):
        n = int(upto_lens[b])
        if n:
            x = synth.bf16_bits_to_f32(case.tokens(b)[:n])
            layout.append(desc_np, pool, case.table[b:b + 1], [0], x[None, :, :512], x[None, :, 512:])
    return pool


@pytest.mark.parametrize("bc,gc,br,gr", BIT_COMBOS)
def test_append_bytes_equal_oracle(bc, gc, br, gr):
    w = synth.workload(1).scaled(B=4, bits_c=bc, group_c=gc, bits_r=br, group_r=gr)
    case = mc.make_case(w, lens=[130, 64, 1, 257])
    pool, _ = mc.fill_pool(case, chunk=100)  # several appends per request, ragged
    assert api.mla_get_device_status() == 0
    ref = _oracle_pool(case, layout.Desc(bits_c=bc, group_c=gc, bits_r=br, group_r=gr), case.lens)
    got = pool.cpu().numpy()
    assert got.shape == ref.shape
    assert np.array_equal(got, ref)


def test_append_extreme_values_bit_exact():
    # fp16-range extremes, fp16-subnormal groups, constant groups and signed zeros
    w = synth.workload(0).scaled(B=1)
    case = mc.make_case(w, lens=[8])
    toks = np.zeros((8, 576), dtype=np.float32)
    rng = np.random.default_rng(9)
    toks[0] = rng.standard_normal(576) * 30000.0
    toks[1] = 1e-6 * (1 + rng.random(576))
    toks[2] = 0.5
    toks[3, :] = -0.0
    toks[3, 7] = 0.25
    toks[4] = rng.standard_normal(576) * np.exp(rng.normal(0, 3, 576))
    toks[5, :64] = 65280.0   # the largest bf16 value within fp16's range
    toks[5, 64:] = -65280.0
    toks[6] = np.where(rng.random(576) < 0.5, -1e-7, 3e-8)
    toks[7] = rng.standard_normal(576)
    bits = synth.f32_to_bf16_bits(np.clip(toks, -65280, 65280))
    x = synth.bf16_bits_to_f32(bits)
    for bc, gc, br, gr in BIT_COMBOS:
        desc = api.make_desc(bc, gc, br, gr, num_pages=1)
        pool = api.new_qcache_pool(desc)
        table = torch.zeros((1, 1), dtype=torch.int32, device="cuda")
        api.mla_qcache_append(desc, pool, table, torch.zeros(1, dtype=torch.int32, device="cuda"),
                              mc.bits_to_torch(bits[None, :, :512]), mc.bits_to_torch(bits[None, :, 512:]))
        d_np = layout.Desc(bits_c=bc, group_c=gc, bits_r=br, group_r=gr)
        ref = layout.new_pool(d_np, 1)
        layout.append(d_np, ref, np.zeros((1, 1), np.int32), [0], x[None, :, :512], x[None, :, 512:])
        assert np.array_equal(pool.cpu().numpy(), ref), (bc, gc, br, gr)


@pytest.mark.parametrize("idx", [1, 4])
def test_append_step_full_size(idx):
    """The timed step's append (config sizes, one call for the whole batch)."""
    w = synth.workload(idx)
    case = mc.make_case(w)
    desc = case.desc
    pool = api.new_qcache_pool(desc)
    table_t = torch.from_numpy(case.table).cuda()
    B, n = w.B, w.n_new
    new = np.stack([synth.cache_tokens_bf16(w, b, int(case.lens[b]), case.mag)[-n:] for b in range(B)])
    lens_before = torch.from_numpy(case.n_history).cuda()
    api.mla_qcache_append(desc, pool, table_t, lens_before, mc.bits_to_torch(new[:, :, :512]),
                          mc.bits_to_torch(new[:, :, 512:]))
    assert api.mla_get_device_status() == 0
    d_np = layout.Desc(bits_c=w.bits_c, group_c=w.group_c, bits_r=w.bits_r, group_r=w.group_r)
    touched = sorted({int(case.table[b][(int(case.n_history[b]) + j) // 64]) for b in range(B) for j in range(n)})
    ref = np.zeros((case.num_pages, d_np.page_bytes), dtype=np.uint8)
    x = synth.bf16_bits_to_f32(new)
    layout.append(d_np, ref, case.table, case.n_history, x[:, :, :512], x[:, :, 512:])
    got = pool[torch.tensor(touched, device="cuda")].cpu().numpy()
    assert np.array_equal(got, ref[touched])
    # nothing else was written
    assert int(pool.sum(dtype=torch.int64).item()) == int(ref[touched].astype(np.int64).sum())


def test_append_noop_and_bad_table_entry():
    desc = api.make_desc(4, 64, 4, 64, num_pages=2)
    pool = api.new_qcache_pool(desc)
    dev = "cuda"
    c = torch.ones((1, 1, 512), dtype=torch.bfloat16, device=dev)
    r = torch.ones((1, 1, 64), dtype=torch.bfloat16, device=dev)
    api.mla_qcache_append(desc, pool, torch.zeros((1, 1), dtype=torch.int32, device=dev),
                          torch.zeros(1, dtype=torch.int32, device=dev), c[:, :0], r[:, :0])
    assert api.mla_get_device_status() == 0
    # table entry outside the pool: nothing is written, the status word says so once
    api.mla_qcache_append(desc, pool, torch.full((1, 1), 7, dtype=torch.int32, device=dev),
                          torch.zeros(1, dtype=torch.int32, device=dev), c, r)
    assert api.mla_get_device_status() == api._lib.MLA_ERR_INVALID_ARG
    assert api.mla_get_device_status() == 0
    # position past the table row
    api.mla_qcache_append(desc, pool, torch.zeros((1, 1), dtype=torch.int32, device=dev),
                          torch.full((1,), 64, dtype=torch.int32, device=dev), c, r)
    assert api.mla_get_device_status() == api._lib.MLA_ERR_INVALID_ARG
    assert int(pool.sum().item()) == 0
