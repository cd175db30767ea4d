"""Pins for the oracle quantizer, packer and page layout (CPU only).

Each test checks the oracle against something other than itself: hand-derived
worked examples, a per-element brute-force quantizer written as plain loops,
closed-form round-trip bounds and byte offsets derived from the layout rule.
"""
import numpy as np
import pytest

from oracle import layout, quant


def test_page_bytes_closed_form():
    # INT4/INT4 g64: 64*256 codes + 64*32 rope codes + 64*8*4 meta + 64*1*4 meta
    d44 = layout.Desc()
    assert d44.offsets() == (0, 16384, 16384 + 2048, 16384 + 2048 + 2048, 20736)
    # INT2 g32 content / INT4 g64 rope: 64*128 + 64*32 + 64*16*4 + 64*4
    d24 = layout.Desc(bits_c=2, group_c=32)
    assert d24.offsets() == (0, 8192, 8192 + 2048, 8192 + 2048 + 4096, 14592)
    # bytes per token against BF16's 1152: 3.556x and 5.053x
    assert d44.page_bytes / 64 == 324 and d24.page_bytes / 64 == 228


def test_worked_example_int4_bytes():
    # x_k = z + (k mod 16) * s with s = 0.125, z = -1 (both exact in fp16 and
    # bf16): the range is 15 s, so s and z are recovered exactly and the codes
    # are 0..15 in order. Even channel = low nibble -> 0x10, 0x32, ..., 0xFE.
    x = (-1.0 + (np.arange(64) % 16) * 0.125).astype(np.float32)[None, :]
    u, s, z = quant.quantize_groups(x, 4, 64)
    assert float(s[0, 0]) == 0.125 and float(z[0, 0]) == -1.0
    assert list(u[0]) == [k % 16 for k in range(64)]
    packed = quant.pack_codes(u, 4)[0]
    assert list(packed[:8]) == [0x10, 0x32, 0x54, 0x76, 0x98, 0xBA, 0xDC, 0xFE]
    assert list(packed) == list(packed[:8]) * 4
    xh = quant.dequantize_groups(u, s, z, 64)
    assert np.array_equal(xh, x.astype(np.float64))


def test_worked_example_int2_bytes():
    # s = 0.5, z = -1: codes 0,1,2,3 repeating; channel 4i+k at bits 2k -> 0xE4.
    x = (-1.0 + (np.arange(32) % 4) * 0.5).astype(np.float32)[None, :]
    u, s, z = quant.quantize_groups(x, 2, 32)
    assert float(s[0, 0]) == 0.5 and float(z[0, 0]) == -1.0
    assert list(quant.pack_codes(u, 2)[0]) == [0xE4] * 8
    assert np.array_equal(quant.dequantize_groups(u, s, z, 32), x.astype(np.float64))


def test_meta_byte_order():
    s = np.array([[1.0]], dtype=np.float16)   # 0x3C00
    z = np.array([[-2.0]], dtype=np.float16)  # 0xC000
    assert list(quant.meta_bytes(s, z)[0]) == [0x00, 0x3C, 0x00, 0xC0]
    s2, z2 = quant.meta_from_bytes(quant.meta_bytes(s, z), 1)
    assert s2[0, 0] == s[0, 0] and z2[0, 0] == z[0, 0]


def _brute_quantize(x, bits, group):
    """Element-by-element restatement with numpy float32 scalars and Python loops."""
    f32 = np.float32
    qmax = (1 << bits) - 1
    n, d = x.shape
    codes = np.zeros((n, d), dtype=np.uint8)
    ss = np.zeros((n, d // group), dtype=np.float16)
    zz = np.zeros((n, d // group), dtype=np.float16)
    for i in range(n):
        for g in range(d // group):
            vals = [f32(x[i, g * group + j]) for j in range(group)]
            lo, hi = f32(min(vals) + f32(0)), max(vals)
            s = np.float16(f32(f32(hi - lo) / f32(qmax)))
            z = np.float16(lo)
            ss[i, g], zz[i, g] = s, z
            for j, v in enumerate(vals):
                if f32(s) == 0:
                    c = 0
                else:
                    t = f32(f32(v - f32(z)) / f32(s))
                    c = min(max(round(float(t)), 0), qmax)  # round(): ties to even
                codes[i, g * group + j] = c
    return codes, ss, zz


@pytest.mark.parametrize("bits,group", [(4, 64), (2, 32), (4, 32), (2, 64)])
def test_vectorised_matches_brute_force(bits, group):
    rng = np.random.default_rng(7)
    mag = np.exp(rng.normal(0, 0.5, 128)).astype(np.float32)
    x = (rng.standard_normal((6, 128)).astype(np.float32) * mag)
    x[2, :group] = 0.75           # a constant group
    x[3, 5] = 40.0                # an outlier
    # a group below fp16's normal range: fp16(min) != min there, so the
    # zero-point's rounding to fp16 changes the codes
    x[4, group:2 * group] = 1e-6 * (1.0 + rng.random(group).astype(np.float32))
    x = (x.astype(np.float32).view(np.uint32) & 0xFFFF0000).view(np.float32)  # bf16 values
    u, s, z = quant.quantize_groups(x, bits, group)
    ub, sb, zb = _brute_quantize(x, bits, group)
    assert np.array_equal(u, ub)
    assert np.array_equal(s.view(np.uint16), sb.view(np.uint16))
    assert np.array_equal(z.view(np.uint16), zb.view(np.uint16))


@pytest.mark.parametrize("bits,group", [(4, 64), (2, 32)])
def test_roundtrip_error_bound(bits, group):
    rng = np.random.default_rng(11)
    n, d = 300, 512
    mag = np.exp(rng.normal(0, 0.5, d)).astype(np.float32)
    mag[rng.choice(d, 5, replace=False)] *= 8
    x = (rng.standard_normal((n, d)).astype(np.float32) * mag)
    x = (x.view(np.uint32) & 0xFFFF0000).view(np.float32)
    u, s, z = quant.quantize_groups(x, bits, group)
    assert u.max() <= (1 << bits) - 1
    xh = quant.dequantize_groups(u, s, z, group)
    qmax = (1 << bits) - 1
    xg = x.astype(np.float64).reshape(n, d // group, group)
    mn, mx = xg.min(-1), xg.max(-1)
    s64, z64 = s.astype(np.float64), z.astype(np.float64)
    bound = (s64 / 2 + np.abs(mn - z64) + qmax * np.abs((mx - mn) / qmax - s64)
             + 4 * 2.0 ** -24 * (np.abs(xg).max(-1) + np.abs(z64) + qmax * s64))
    err = np.abs(xh.reshape(n, d // group, group) - xg).max(-1)
    assert np.all(err <= bound)
    # the group minimum always encodes to code 0
    am = xg.argmin(-1)
    ug = u.reshape(n, d // group, group)
    assert np.all(np.take_along_axis(ug, am[..., None], -1) == 0)


def test_signed_zero_minimum_gives_positive_zero_point():
    x = np.zeros((2, 64), dtype=np.float32)
    x[0, 3] = -0.0
    x[1, :] = -0.0
    x[1, 7] = 0.5
    _, _, z = quant.quantize_groups(x, 4, 64)
    assert np.all(z.view(np.uint16) == 0)


def test_constant_group_decodes_exactly():
    x = np.full((3, 64), 1.5, dtype=np.float32)
    x[1] = -0.25
    u, s, z = quant.quantize_groups(x, 4, 64)
    assert np.all(u == 0) and np.all(s.astype(np.float32) == 0)
    assert np.array_equal(quant.dequantize_groups(u, s, z, 64), x.astype(np.float64))


@pytest.mark.parametrize("bits", [2, 4, 8])
def test_pack_unpack_identity(bits):
    rng = np.random.default_rng(bits)
    codes = rng.integers(0, 1 << bits, size=(17, 64)).astype(np.uint8)
    assert np.array_equal(quant.unpack_codes(quant.pack_codes(codes, bits), bits, 64), codes)


def test_page_writer_offsets_and_reader():
    desc = layout.Desc(bits_c=2, group_c=32)
    rng = np.random.default_rng(3)
    T = 130  # three pages, ragged tail
    c = (rng.standard_normal((1, T, 512)).astype(np.float32).view(np.uint32) & 0xFFFF0000).view(np.float32)
    r = (rng.standard_normal((1, T, 64)).astype(np.float32).view(np.uint32) & 0xFFFF0000).view(np.float32)
    table = np.array([[2, 0, 1]], dtype=np.int32)
    pool = layout.new_pool(desc, 3)
    layout.append(desc, pool, table, [0], c[:, :100], r[:, :100])
    layout.append(desc, pool, table, [100], c[:, 100:], r[:, 100:])
    # token 70 -> page table[0][1] = 0, slot 6: its content codes row is bytes
    # [6*128, 7*128) of page 0, its rope meta 4 bytes at 8192+2048+4096+6*4
    uc, sc, zc = quant.quantize_groups(c[0, 70:71], 2, 32)
    ur, sr, zr = quant.quantize_groups(r[0, 70:71], 4, 64)
    assert np.array_equal(pool[0, 6 * 128:7 * 128], quant.pack_codes(uc, 2)[0])
    off = 8192 + 2048 + 4096 + 6 * 4
    assert np.array_equal(pool[0, off:off + 4], quant.meta_bytes(sr, zr)[0])
    C, R = layout.gather_tokens(desc, pool, table[0], T)
    u, s, z = quant.quantize_groups(c[0], 2, 32)
    assert np.array_equal(C, quant.dequantize_groups(u, s, z, 32))
    u, s, z = quant.quantize_groups(r[0], 4, 64)
    assert np.array_equal(R, quant.dequantize_groups(u, s, z, 64))


def test_batched_append_uses_each_requests_table():
    # Layout rule: token t of request b lives in page block_table[b][t // P],
    # slot t % P. One append call for two requests with different histories:
    # request 1's new tokens must land in its own pages (byte check at a
    # hand-computed offset), and request 0's pages must hold only its tokens.
    desc = layout.Desc()
    rng = np.random.default_rng(11)
    c = (rng.standard_normal((2, 3, 512)).astype(np.float32).view(np.uint32) & 0xFFFF0000).view(np.float32)
    r = (rng.standard_normal((2, 3, 64)).astype(np.float32).view(np.uint32) & 0xFFFF0000).view(np.float32)
    table = np.array([[1, 3], [2, 0]], dtype=np.int32)
    pool = layout.new_pool(desc, 4)
    layout.append(desc, pool, table, [62, 5], c, r)
    # request 1, new token 0 is t = 5 -> page table[1][0] = 2, slot 5
    uc, _, _ = quant.quantize_groups(c[1, 0:1], 4, 64)
    assert np.array_equal(pool[2, 5 * 256:6 * 256], quant.pack_codes(uc, 4)[0])
    # request 0, new token 2 is t = 64 -> page table[0][1] = 3, slot 0
    uc, _, _ = quant.quantize_groups(c[0, 2:3], 4, 64)
    assert np.array_equal(pool[3, 0:256], quant.pack_codes(uc, 4)[0])
    # page 0 (request 1's second page) is untouched
    assert not pool[0].any()
    for b, t0 in ((0, 62), (1, 5)):
        C, _ = layout.gather_tokens(desc, pool, table[b], t0 + 3)
        u, s, z = quant.quantize_groups(c[b], 4, 64)
        assert np.array_equal(C[t0:t0 + 3], quant.dequantize_groups(u, s, z, 64))
