"""C-ABI checks that need no GPU: symbols, layout arithmetic, argument errors.

Every call here returns before the library touches a device (validation runs
first), so no compute happens; fake device addresses are never dereferenced.
"""
import ctypes
import os
import re

import pytest

from bit_mla_kv_qdecode_b200 import _lib
from bit_mla_kv_qdecode_b200 import build as _build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    _build.build()
    return _lib.load()


def declared_functions():
    names = []
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names += re.findall(r"^\s*(?:const\s+)?[A-Za-z_][\w\s\*]*?\b(mla_\w+)\s*\(", src, flags=re.M)
    return sorted(set(names))


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert len(names) >= 11, names
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(_lib.SIGNATURES), "binding and header disagree"


def test_layout_arithmetic(lib):
    d44 = _lib.make_desc(4, 64, 4, 64)
    d24 = _lib.make_desc(2, 32, 4, 64)
    assert lib.mla_qcache_page_bytes(ctypes.byref(d44)) == 20736
    assert lib.mla_qcache_page_bytes(ctypes.byref(d24)) == 14592
    out = (ctypes.c_size_t * 5)()
    assert lib.mla_qcache_segment_offsets(ctypes.byref(d24), out) == 0
    assert list(out) == [0, 8192, 10240, 14336, 14592]
    assert lib.mla_qcache_layout_version() == 1


def test_desc_validation(lib):
    assert lib.mla_qcache_check_desc(None) == _lib.MLA_ERR_INVALID_ARG
    assert lib.mla_qcache_check_desc(ctypes.byref(_lib.make_desc(3, 64))) == _lib.MLA_ERR_UNSUPPORTED
    assert lib.mla_qcache_check_desc(ctypes.byref(_lib.make_desc(4, 48))) == _lib.MLA_ERR_INVALID_ARG
    assert lib.mla_qcache_check_desc(ctypes.byref(_lib.make_desc(4, 64, d_c=256))) == _lib.MLA_ERR_UNSUPPORTED
    assert lib.mla_qcache_check_desc(ctypes.byref(_lib.make_desc(4, 64, page_size=32))) == _lib.MLA_ERR_UNSUPPORTED
    assert lib.mla_qcache_page_bytes(ctypes.byref(_lib.make_desc(8, 64))) == 0
    for code in range(7):
        assert lib.mla_status_string(code)
    assert b"unknown" in lib.mla_status_string(99)


def test_split_plan_and_workspace(lib):
    # explicit split count: 128K tokens = 2048 pages into 32 chunks of 64 pages
    assert lib.mla_decode_num_splits(4, 1, 128, 131072, 32) == 32
    ws = lib.mla_decode_workspace_bytes(4, 1, 128, 131072, 32)
    parts = 4 * 32 * 128
    assert ws == ((parts * 4 + 255) // 256) * 256 + parts * 512 * 4
    # requests for more splits than pages are capped
    assert lib.mla_decode_num_splits(1, 1, 16, 100, 50) == 2
    assert lib.mla_decode_workspace_bytes(1, 1, 16, 64, 1) == 0
    n = lib.mla_decode_num_splits(32, 1, 128, 4096, 0)
    assert 1 <= n <= 64
    # no chunk sums more than 8,192 keys: explicit requests are raised, automatic plans respect it
    assert lib.mla_decode_num_splits(1, 1, 128, 8192, 1) == 1
    assert lib.mla_decode_num_splits(1, 1, 128, 8193, 1) == 2
    assert lib.mla_decode_num_splits(1, 1, 128, 32768, 1) == 4
    assert lib.mla_decode_num_splits(1, 1, 128, 32768, 8) == 8
    for B, T in ((1, 1 << 20), (128, 32768), (4, 131072), (64, 16384)):
        n = lib.mla_decode_num_splits(B, 1, 128, T, 0)
        pages = (T + 63) // 64
        assert (pages + n - 1) // n <= 128, (B, T, n)


FAKE = 0x10000000  # never dereferenced: every call below fails validation first


def test_append_argument_errors(lib):
    d = ctypes.byref(_lib.make_desc(4, 64, num_pages=4))
    # B == 0 and n_new == 0 are no-ops
    assert lib.mla_qcache_append(d, None, None, 1, None, None, None, 0, 5, None) == 0
    assert lib.mla_qcache_append(d, None, None, 1, None, None, None, 5, 0, None) == 0
    assert lib.mla_qcache_append(d, None, FAKE, 1, FAKE, FAKE, FAKE, 1, 1, None) == _lib.MLA_ERR_INVALID_ARG
    assert lib.mla_qcache_append(d, FAKE + 16, FAKE, 1, FAKE, FAKE, FAKE, 1, 1, None) == _lib.MLA_ERR_INVALID_ARG
    assert lib.mla_qcache_append(d, FAKE, FAKE, 1, FAKE, FAKE, FAKE, -1, 1, None) == _lib.MLA_ERR_INVALID_ARG
    bad = ctypes.byref(_lib.make_desc(3, 64, num_pages=4))
    assert lib.mla_qcache_append(bad, FAKE, FAKE, 1, FAKE, FAKE, FAKE, 1, 1, None) == _lib.MLA_ERR_UNSUPPORTED
    assert lib.mla_bf16cache_append(FAKE, 4, 32, FAKE, 1, FAKE, FAKE, FAKE, 1, 1, None) == _lib.MLA_ERR_UNSUPPORTED


def _qdecode(lib, **kw):
    a = dict(desc=ctypes.byref(_lib.make_desc(4, 64, num_pages=8)), pool=FAKE, table=FAKE, maxp=4, lens=FAKE,
             max_seq_len=256, qc=FAKE, qr=FAKE, B=2, s_q=1, H=16, scale=0.1, splits=1, ws=None, ws_bytes=0,
             out=FAKE, out_dtype=0, lse=None, flags=0, stream=None)
    a.update(kw)
    return lib.mla_qdecode(a["desc"], a["pool"], a["table"], a["maxp"], a["lens"], a["max_seq_len"], a["qc"],
                           a["qr"], a["B"], a["s_q"], a["H"], a["scale"], a["splits"], a["ws"], a["ws_bytes"],
                           a["out"], a["out_dtype"], a["lse"], a["flags"], a["stream"])


def test_decode_argument_errors(lib):
    E = _lib
    assert _qdecode(lib, B=0) == E.MLA_OK
    assert _qdecode(lib, qc=None) == E.MLA_ERR_INVALID_ARG
    assert _qdecode(lib, out=FAKE + 4) == E.MLA_ERR_INVALID_ARG       # out not 16-byte aligned
    assert _qdecode(lib, s_q=0) == E.MLA_ERR_INVALID_ARG
    assert _qdecode(lib, out_dtype=2) == E.MLA_ERR_INVALID_ARG
    assert _qdecode(lib, scale=float("nan")) == E.MLA_ERR_INVALID_ARG
    assert _qdecode(lib, flags=8) == E.MLA_ERR_INVALID_ARG
    assert _qdecode(lib, max_seq_len=257) == E.MLA_ERR_CAPACITY        # > 4 pages * 64
    assert _qdecode(lib, splits=4) == E.MLA_ERR_WORKSPACE              # 4 splits need workspace
    need = lib.mla_decode_workspace_bytes(2, 1, 16, 256, 4)
    assert _qdecode(lib, splits=4, ws=FAKE, ws_bytes=need - 1) == E.MLA_ERR_WORKSPACE
    assert _qdecode(lib, desc=ctypes.byref(_lib.make_desc(4, 64, bits_r=8))) == E.MLA_ERR_UNSUPPORTED
    assert _qdecode(lib, B=70000) == E.MLA_ERR_UNSUPPORTED
    assert lib.mla_decode_bf16(FAKE, 8, 64, FAKE, 4, FAKE, 300, FAKE, FAKE, 2, 1, 16, 0.1, 1, None, 0, FAKE, 0,
                               None, 0, None) == E.MLA_ERR_CAPACITY
    assert lib.mla_get_device_status(None, None) == E.MLA_ERR_INVALID_ARG


def test_cache_capacity_closed_forms(lib):
    # host arithmetic only: bytes per request in whole pages, and requests per budget
    from bit_mla_kv_qdecode_b200 import api
    T = 131072
    d44 = api.make_desc(4, 64, 4, 64, num_pages=7)  # num_pages is ignored
    d24 = api.make_desc(2, 32, 4, 64)
    assert api.mla_cache_bytes_per_request(None, T) == T * 1152
    assert api.mla_cache_bytes_per_request(d44, T) == T * 324  # 2048 pages x 20,736 B
    assert api.mla_cache_bytes_per_request(d24, T) == T * 228
    assert api.mla_cache_bytes_per_request(d44, 65) == 2 * 20736  # whole pages
    # hybrid: sink 64 + window 128..191 in BF16 pages, history 64 * floor((T - 192) / 64) quantized
    hist = (T - 192) // 64 * 64
    assert hist == T - 192
    assert api.mla_cache_bytes_per_request(d44, T, 64, 128) == (hist // 64) * 20736 + (1 + 2) * 64 * 1152
    assert api.mla_cache_bytes_per_request(d44, 100, 64, 128) == 2 * 64 * 1152  # all protected
    assert api.mla_cache_bytes_per_request(d44, 1000, 64, 128) == 12 * 20736 + (1 + 3) * 64 * 1152
    ratio = api.mla_cache_bytes_per_request(None, T) / api.mla_cache_bytes_per_request(d44, T, 64, 128)
    assert 3.54 < ratio < 3.556
    # requests per budget: floor(budget / bytes)
    budget = 140 * 10 ** 9
    assert api.mla_cache_max_requests(None, T, budget) == budget // (T * 1152)
    assert api.mla_cache_max_requests(d44, T, budget) == budget // (T * 324)
    assert api.mla_cache_max_requests(d24, T, budget) == budget // (T * 228)
    # invalid: sink not a whole number of pages, negative sizes, protection without a desc, empty request
    assert api.mla_cache_bytes_per_request(d44, T, 10, 0) == 0
    assert api.mla_cache_bytes_per_request(d44, -1) == 0
    assert api.mla_cache_bytes_per_request(None, T, 64, 0) == 0
    assert api.mla_cache_max_requests(d44, 0, budget) == -1


def test_fused_append_argument_errors(lib):
    E = _lib
    d = ctypes.byref(_lib.make_desc(4, 64, num_pages=8))

    def call(pool=FAKE, cn=FAKE, kn=FAKE, n=1, B=2, flags=0):
        return lib.mla_qdecode_fused_append(d, pool, FAKE, 4, FAKE, 256, cn, kn, n, FAKE, FAKE, B, 1, 128, 0.1, 1,
                                            None, 0, FAKE, 0, None, flags, None)

    assert call(n=-1) == E.MLA_ERR_INVALID_ARG
    assert call(cn=None) == E.MLA_ERR_INVALID_ARG
    assert call(kn=FAKE + 8) == E.MLA_ERR_INVALID_ARG                 # not 16-byte aligned
    assert call(pool=None) == E.MLA_ERR_INVALID_ARG
    assert call(B=0) == E.MLA_OK
    assert call(B=0, n=0, cn=None, kn=None) == E.MLA_OK


def test_hybrid_and_noalloc_argument_errors(lib):
    E = _lib
    d = ctypes.byref(_lib.make_desc(4, 64, num_pages=8))

    def hybrid(B=2, s_q=1, H=16, out=FAKE, ws=FAKE, ws_bytes=1 << 30, out_dtype=0, desc=d):
        return lib.mla_qdecode_hybrid(desc, FAKE, FAKE, 4, FAKE, 128, FAKE, 4, FAKE, 4, FAKE, 128, FAKE, FAKE,
                                      B, s_q, H, 0.1, ws, ws_bytes, out, out_dtype, None, None)

    assert hybrid(B=0) == E.MLA_OK
    assert hybrid(s_q=0) == E.MLA_ERR_INVALID_ARG
    assert hybrid(out_dtype=3) == E.MLA_ERR_INVALID_ARG
    assert hybrid(out=None) == E.MLA_ERR_INVALID_ARG
    assert hybrid(ws=None) == E.MLA_ERR_WORKSPACE
    assert hybrid(ws_bytes=16) == E.MLA_ERR_WORKSPACE
    assert hybrid(B=60000, s_q=4, H=16384) == E.MLA_ERR_UNSUPPORTED
    assert hybrid(desc=ctypes.byref(_lib.make_desc(3, 64))) == E.MLA_ERR_UNSUPPORTED
    # page moves: B == 0 is a no-op; missing pointers are argument errors
    assert lib.mla_qcache_append_bf16_pages(d, FAKE, FAKE, 4, FAKE, FAKE, 4, FAKE, 0, None) == E.MLA_OK
    assert lib.mla_qcache_append_bf16_pages(d, FAKE, FAKE, 4, FAKE, FAKE, 4, None, 2, None) == E.MLA_ERR_INVALID_ARG
    # allocation-free decode: its argument errors come before any device work
    assert lib.mla_qdecode_noalloc(d, FAKE, FAKE, 4, FAKE, 256, FAKE, FAKE, -1, 1, 16, 0.1, 0, FAKE, 0, None, 0,
                                   None) == E.MLA_ERR_INVALID_ARG
    assert lib.mla_qdecode_noalloc(d, FAKE, FAKE, 4, FAKE, 256, FAKE, FAKE, 2, 0, 16, 0.1, 0, FAKE, 0, None, 0,
                                   None) == E.MLA_ERR_INVALID_ARG
    # a plan whose split scratch exceeds the fixed array is refused, not truncated
    big = lib.mla_qdecode_noalloc(d, FAKE, FAKE, 4096, FAKE, 262144, FAKE, FAKE, 64, 1, 128, 0.1, 32, FAKE, 0, None,
                                  0, None)
    assert big == E.MLA_ERR_WORKSPACE


def test_workspace_holds_the_work_list_of_multi_wave_split_plans():
    # A split plan for the tensor-core kernel whose units (request, split,
    # 128-row tile) exceed two waves of the 74 two-CTA cluster slots of a
    # 148-SM device takes them from a device-built list, one int32 per unit,
    # placed after the split partials.
    lib = _lib.load()
    B, s_q, H, T = 128, 2, 128, 32770
    n = lib.mla_decode_num_splits(B, s_q, H, T, 0)
    rows = s_q * H
    parts = B * n * rows
    partials = ((parts * 4 + 255) // 256) * 256 + parts * 512 * 4
    units = B * n * ((rows + 127) // 128)
    assert n > 1 and units > 148
    assert lib.mla_decode_workspace_bytes(B, s_q, H, T, 0) == partials + units * 4
    # one wave or less (here 4 x 32 units), or a small-row plan: no list
    parts = 4 * 32 * 128
    assert lib.mla_decode_workspace_bytes(4, 1, 128, 131072, 32) == ((parts * 4 + 255) // 256) * 256 + parts * 2048
    n16 = lib.mla_decode_num_splits(300, 1, 16, 32768, 0)
    parts = 300 * n16 * 16
    assert lib.mla_decode_workspace_bytes(300, 1, 16, 32768, 0) == ((parts * 4 + 255) // 256) * 256 + parts * 2048
