"""Low-bit (INT4 / INT2) MLA KV-cache decode for NVIDIA B200 (sm_100a).

The compute lives in a CUDA library with a C ABI (include/mla_qcache.h);
``bit_mla_kv_qdecode_b200.api`` binds it for PyTorch tensors and
``bit_mla_kv_qdecode_b200._lib`` is the raw ctypes binding.
"""
from ._lib import (MLA_DECODE_DEFAULT, MLA_DECODE_FAST_UNCOMPENSATED, MLA_DECODE_FORCE_SIMT,  # noqa: F401
                   MlaError, make_desc, mla_qcache_desc)

__all__ = ["api", "synth", "make_desc", "mla_qcache_desc", "MlaError", "MLA_DECODE_DEFAULT",
           "MLA_DECODE_FORCE_SIMT", "MLA_DECODE_FAST_UNCOMPENSATED"]
