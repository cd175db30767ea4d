"""CPU model of the small-row kernel's code-to-MMA-fragment mappings (csrc/decode_small.cu).

The kernel turns packed codes into warp-level MMA operands with byte permutes
(PTX prmt) and shifts. This test restates those steps in Python, feeds them
bytes packed by the oracle's pack_codes (the layout's packing order), and checks
that every score B-fragment half holds the code of the channel its Q fragment
pairs with, and that every output N-tile column reads the code of the channel
the epilogue writes, for INT4 and INT2 codes in groups of 32 and 64. An N-tile
must also lie in one scale group (its weight operand carries one scale).
"""
import numpy as np
import pytest

from oracle import quant


def prmt(a, b, sel):
    """PTX prmt.b32 (default mode): byte i of the result is selected by nibble i of sel."""
    src = [(a >> (8 * i)) & 0xFF for i in range(4)] + [(b >> (8 * i)) & 0xFF for i in range(4)]
    out = 0
    for i in range(4):
        s = (sel >> (4 * i)) & 0xF
        byte = src[s & 7]
        if s & 8:
            byte = 0xFF if byte & 0x80 else 0
        out |= byte << (8 * i)
    return out


def byte_pairs(a, b, hb4):
    m01, m23 = prmt(a, b, 0x5140), prmt(a, b, 0x7362)
    return [prmt(m01, hb4, 0x4140), prmt(m01, hb4, 0x4342), prmt(m23, hb4, 0x4140), prmt(m23, hb4, 0x4342)]


def u32(b, off):
    return int.from_bytes(b[off:off + 4], "little")


def u16(b, off):
    return int.from_bytes(b[off:off + 2], "little")


def qk_codes(p, bits, gs):
    bf = [[0, 0] for _ in range(gs // 16)]
    if bits == 4:
        words = [u32(p, 0), u32(p, 4)] if gs == 64 else [u32(p, 0)]
        for i, w in enumerate(words):
            q = byte_pairs(w & 0x0F0F0F0F, (w >> 4) & 0x0F0F0F0F, 0x43434343)
            bf[2 * i], bf[2 * i + 1] = [q[0], q[1]], [q[2], q[3]]
    else:
        w = u32(p, 0) if gs == 64 else u16(p, 0)
        p01 = byte_pairs(w & 0x03030303, (w >> 2) & 0x03030303, 0x43434343)
        p23 = byte_pairs((w >> 4) & 0x03030303, (w >> 6) & 0x03030303, 0x43434343)
        for s in range(gs // 16):
            bf[s] = [p01[s], p23[s]]
    return bf


def spread_crumbs(x):
    x = (x | (x << 8)) & 0x00FF00FF
    x = (x | (x << 4)) & 0x0F0F0F0F
    return (x | (x << 2)) & 0x33333333


def pv_codes(p, n, bits, gs):
    if bits == 4 and gs == 64:
        return u32(p, 4 * n)
    if bits == 4:
        return u16(p, 2 * n) | (u16(p, 16 + 2 * n) << 16)
    if gs == 64:
        return spread_crumbs(u16(p, 2 * n))
    return spread_crumbs(p[n] | (p[8 + n] << 8))


def pv_channel(j, n, gs):
    return 8 * n + j if gs == 64 else 32 * (j >> 2) + 4 * n + (j & 3)


def sel_pair(j):
    return j | ((8 | j) << 4) | ((4 + j) << 8) | ((12 + j) << 12)


@pytest.mark.parametrize("bits", [2, 4])
@pytest.mark.parametrize("gs", [32, 64])
def test_fragment_maps(bits, gs):
    rng = np.random.default_rng(bits * 100 + gs)
    qmax = (1 << bits) - 1
    for _ in range(20):
        codes = rng.integers(0, qmax + 1, size=(2, 512)).astype(np.uint8)
        packed = quant.pack_codes(codes, bits)
        row, row2 = bytes(packed[0]), bytes(packed[1])
        # scores: group g, lane kp; K-step s pairs channels (GS/4) kp + 4s + {0,1} / {2,3}
        for g in range(512 // gs):
            for kp in range(4):
                off = g * (gs * bits // 8) + kp * (gs * bits // 32)
                bf = qk_codes(row[off:], bits, gs)
                for s in range(gs // 16):
                    c0 = g * gs + (gs // 4) * kp + 4 * s
                    for h in range(2):
                        assert bf[s][h] & 0xFFFF == 0x4300 | int(codes[0, c0 + 2 * h])      # bf16 128 + u
                        assert bf[s][h] >> 16 == 0x4300 | int(codes[0, c0 + 2 * h + 1])
        # output: warp w, lane column n, N-tile j; B pair = (key a, key b) as fp16 [u, 0x00]
        for w in range(8):
            wa = [pv_codes(r[8 * bits * w:], n, bits, gs) for r in (row, row2) for n in range(8)]
            for n in range(8):
                lo_a, hi_a = wa[n] & 0x0F0F0F0F, (wa[n] >> 4) & 0x0F0F0F0F
                lo_b, hi_b = wa[8 + n] & 0x0F0F0F0F, (wa[8 + n] >> 4) & 0x0F0F0F0F
                for j in range(8):
                    pair = prmt(hi_a, hi_b, sel_pair(j >> 1)) if j & 1 else prmt(lo_a, lo_b, sel_pair(j >> 1))
                    ch = 64 * w + pv_channel(j, n, gs)
                    assert pair & 0xFFFF == int(codes[0, ch])
                    assert pair >> 16 == int(codes[1, ch])
    # an N-tile lies in one scale group: tiles 0-3 / 4-7 of a warp for groups of 32
    for w in range(8):
        for j in range(8):
            groups = {(64 * w + pv_channel(j, n, gs)) // gs for n in range(8)}
            assert groups == {(64 * w) // gs + j // (8 // (64 // gs))}
    # the epilogue's channel map is a bijection onto the warp's 64 channels
    assert sorted(pv_channel(j, n, gs) for j in range(8) for n in range(8)) == list(range(64))
