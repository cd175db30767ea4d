"""ctypes binding of the C ABI in include/mla_qcache.h (same names, same arguments).

Argument marshalling only: every step of the decode path runs in the CUDA
library. Pointers are passed as integers (device addresses, e.g. from
``torch.Tensor.data_ptr()``) and streams as ``cudaStream_t`` integers. Loading
fails loudly if the library has not been built.
"""
from __future__ import annotations

import ctypes
import os

from . import build as _build

_c_int, _c_size, _c_void, _c_float, _c_uint = ctypes.c_int, ctypes.c_size_t, ctypes.c_void_p, ctypes.c_float, ctypes.c_uint

MLA_OK = 0
MLA_ERR_INVALID_ARG = 1
MLA_ERR_UNSUPPORTED = 2
MLA_ERR_CAPACITY = 3
MLA_ERR_WORKSPACE = 4
MLA_ERR_CUDA = 5
MLA_ERR_TIMEOUT = 6

MLA_DECODE_DEFAULT = 0
MLA_DECODE_FORCE_SIMT = 1
MLA_DECODE_FAST_UNCOMPENSATED = 2
MLA_DECODE_TEST_STALL = 4  # tests only: runs the device-side timeout path

MLA_QDECODE_NOALLOC_SCRATCH_BYTES = 64 << 20


class mla_qcache_desc(ctypes.Structure):
    _fields_ = [(n, _c_int) for n in ("d_c", "d_r", "bits_c", "group_c", "bits_r", "group_r",
                                      "page_size", "num_pages")]


_P = ctypes.POINTER(mla_qcache_desc)

# name -> (restype, argtypes); mirrors include/mla_qcache.h
SIGNATURES = {
    "mla_status_string": (ctypes.c_char_p, [_c_int]),
    "mla_qcache_layout_version": (_c_int, []),
    "mla_qcache_check_desc": (_c_int, [_P]),
    "mla_qcache_page_bytes": (_c_size, [_P]),
    "mla_qcache_segment_offsets": (_c_int, [_P, ctypes.POINTER(_c_size)]),
    "mla_qcache_append": (_c_int, [_P, _c_void, _c_void, _c_int, _c_void, _c_void, _c_void, _c_int, _c_int,
                                   _c_void]),
    "mla_bf16cache_append": (_c_int, [_c_void, _c_int, _c_int, _c_void, _c_int, _c_void, _c_void, _c_void,
                                      _c_int, _c_int, _c_void]),
    "mla_decode_num_splits": (_c_int, [_c_int, _c_int, _c_int, _c_int, _c_int]),
    "mla_decode_workspace_bytes": (_c_size, [_c_int, _c_int, _c_int, _c_int, _c_int]),
    "mla_qdecode": (_c_int, [_P, _c_void, _c_void, _c_int, _c_void, _c_int, _c_void, _c_void, _c_int, _c_int,
                             _c_int, _c_float, _c_int, _c_void, _c_size, _c_void, _c_int, _c_void, _c_uint,
                             _c_void]),
    "mla_qdecode_fused_append": (_c_int, [_P, _c_void, _c_void, _c_int, _c_void, _c_int, _c_void, _c_void, _c_int,
                                          _c_void, _c_void, _c_int, _c_int, _c_int, _c_float, _c_int, _c_void,
                                          _c_size, _c_void, _c_int, _c_void, _c_uint, _c_void]),
    "mla_decode_bf16": (_c_int, [_c_void, _c_int, _c_int, _c_void, _c_int, _c_void, _c_int, _c_void, _c_void,
                                 _c_int, _c_int, _c_int, _c_float, _c_int, _c_void, _c_size, _c_void, _c_int,
                                 _c_void, _c_uint, _c_void]),
    "mla_qdecode_noalloc": (_c_int, [_P, _c_void, _c_void, _c_int, _c_void, _c_int, _c_void, _c_void, _c_int,
                                     _c_int, _c_int, _c_float, _c_int, _c_void, _c_int, _c_void, _c_uint, _c_void]),
    "mla_qcache_append_bf16_pages": (_c_int, [_P, _c_void, _c_void, _c_int, _c_void, _c_void, _c_int, _c_void,
                                              _c_int, _c_void]),
    "mla_qdecode_hybrid_workspace_bytes": (_c_size, [_c_int, _c_int, _c_int, _c_int, _c_int]),
    "mla_qdecode_hybrid": (_c_int, [_P, _c_void, _c_void, _c_int, _c_void, _c_int, _c_void, _c_int, _c_void,
                                    _c_int, _c_void, _c_int, _c_void, _c_void, _c_int, _c_int, _c_int, _c_float,
                                    _c_void, _c_size, _c_void, _c_int, _c_void, _c_void]),
    "mla_cache_bytes_per_request": (_c_size, [_P, ctypes.c_long, _c_int, _c_int]),
    "mla_cache_max_requests": (ctypes.c_long, [_P, ctypes.c_long, _c_int, _c_int, _c_size]),
    "mla_get_device_status": (_c_int, [ctypes.POINTER(_c_int), _c_void]),
}

_lib = None


def lib_path() -> str:
    return _build.LIB_PATH


def load():
    """Load the built library (building it first only if MLA_BUILD_ON_IMPORT=1)."""
    global _lib
    if _lib is not None:
        return _lib
    path = lib_path()
    if not os.path.exists(path):
        if os.environ.get("MLA_BUILD_ON_IMPORT") == "1":
            _build.build()
        else:
            raise ImportError(
                f"CUDA library {path} is missing: build it with "
                "`python -m bit_mla_kv_qdecode_b200.build` (there is no CPU fallback)")
    lib = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def status_string(code: int) -> str:
    return load().mla_status_string(int(code)).decode()


class MlaError(RuntimeError):
    def __init__(self, fn: str, code: int):
        self.code = int(code)
        super().__init__(f"{fn} failed: {status_string(code)}")


def check(fn: str, code: int) -> None:
    if code != MLA_OK:
        raise MlaError(fn, code)


def make_desc(bits_c=4, group_c=64, bits_r=4, group_r=64, num_pages=0, d_c=512, d_r=64, page_size=64):
    return mla_qcache_desc(d_c, d_r, bits_c, group_c, bits_r, group_r, page_size, num_pages)
