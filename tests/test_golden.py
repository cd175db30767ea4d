"""The oracle's quantizer, packer and page layout against the hand-derived
fixtures in tests/golden/ (each file states its derivation and citation)."""
import os

import numpy as np

from oracle import layout, quant

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _rows(name):
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                yield [c.strip() for c in line.split("|")]


def test_quant_worked_examples():
    rows = list(_rows("quant_worked_examples.txt"))
    assert len(rows) == 2
    for name, bits, group, xdef, s_ref, z_ref, packed_hex in rows:
        bits, group = int(bits), int(group)
        z0, step, period, n = xdef.split()
        k = np.arange(int(n))
        x = (float(z0) + (k % int(period)) * float(step)).astype(np.float32)[None, :]
        u, s, z = quant.quantize_groups(x, bits, group)
        assert float(s[0, 0]) == float(s_ref) and float(z[0, 0]) == float(z_ref), name
        assert list(quant.pack_codes(u, bits)[0]) == [int(h, 16) for h in packed_hex.split()], name
        assert np.array_equal(quant.dequantize_groups(u, s, z, group), x.astype(np.float64)), name


def test_page_layout_v1():
    rows = list(_rows("page_layout_v1.txt"))
    assert len(rows) == 2
    for bc, gc, br, gr, offs in rows:
        d = layout.Desc(bits_c=int(bc), group_c=int(gc), bits_r=int(br), group_r=int(gr))
        assert d.offsets() == tuple(int(v) for v in offs.split())


def test_library_layout_matches_golden():
    # the C library's segment offsets (host arithmetic, no GPU) against the same fixture
    import ctypes

    from bit_mla_kv_qdecode_b200 import _lib
    from bit_mla_kv_qdecode_b200 import build as _build
    _build.build()
    lib = _lib.load()
    for bc, gc, br, gr, offs in _rows("page_layout_v1.txt"):
        d = _lib.make_desc(int(bc), int(gc), int(br), int(gr))
        out = (ctypes.c_size_t * 5)()
        assert lib.mla_qcache_segment_offsets(ctypes.byref(d), out) == 0
        assert list(out) == [int(v) for v in offs.split()]
