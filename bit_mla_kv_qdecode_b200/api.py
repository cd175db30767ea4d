"""PyTorch-facing binding of the C ABI (include/mla_qcache.h).

The functions carry the C entry points' names and only marshal arguments:
they check dtypes, devices and contiguity, allocate outputs and workspace
through PyTorch when the caller passes none, and hand raw pointers plus the
current CUDA stream to the library. Nothing is computed here.
"""
from __future__ import annotations

import ctypes

import torch

from . import _lib
from ._lib import MlaError, check, make_desc, mla_qcache_desc  # noqa: F401

D_C, D_R, PAGE = 512, 64, 64


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _need(t: torch.Tensor, name: str, dtype, shape=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    return t.data_ptr()


def mla_qcache_page_bytes(desc: mla_qcache_desc) -> int:
    return int(_lib.load().mla_qcache_page_bytes(ctypes.byref(desc)))


def mla_qcache_segment_offsets(desc: mla_qcache_desc):
    out = (ctypes.c_size_t * 5)()
    check("mla_qcache_segment_offsets", _lib.load().mla_qcache_segment_offsets(ctypes.byref(desc), out))
    return tuple(int(v) for v in out)


def new_qcache_pool(desc: mla_qcache_desc, device="cuda") -> torch.Tensor:
    """uint8 pool [num_pages, page_bytes] (PyTorch allocations are 256-byte aligned)."""
    return torch.zeros((desc.num_pages, mla_qcache_page_bytes(desc)), dtype=torch.uint8, device=device)


def new_bf16_pool(num_pages: int, device="cuda") -> torch.Tensor:
    return torch.zeros((num_pages, PAGE, D_C + D_R), dtype=torch.bfloat16, device=device)


def mla_qcache_append(desc, pool, block_table, seq_lens_before, c_new, kr_new, stream=None) -> None:
    B, n = c_new.shape[0], c_new.shape[1]
    args = (_need(pool, "pool", torch.uint8), _need(block_table, "block_table", torch.int32),
            block_table.shape[1], _need(seq_lens_before, "seq_lens_before", torch.int32, (B,)),
            _need(c_new, "c_new", torch.bfloat16, (B, n, D_C)), _need(kr_new, "kr_new", torch.bfloat16, (B, n, D_R)))
    check("mla_qcache_append",
          _lib.load().mla_qcache_append(ctypes.byref(desc), *args, B, n, _stream(stream)))


def mla_bf16cache_append(pool, block_table, seq_lens_before, c_new, kr_new, stream=None) -> None:
    B, n = c_new.shape[0], c_new.shape[1]
    check("mla_bf16cache_append", _lib.load().mla_bf16cache_append(
        _need(pool, "pool", torch.bfloat16), pool.shape[0], pool.shape[1],
        _need(block_table, "block_table", torch.int32), block_table.shape[1],
        _need(seq_lens_before, "seq_lens_before", torch.int32, (B,)),
        _need(c_new, "c_new", torch.bfloat16, (B, n, D_C)), _need(kr_new, "kr_new", torch.bfloat16, (B, n, D_R)),
        B, n, _stream(stream)))


def mla_decode_num_splits(B, s_q, H, max_seq_len, num_splits=0) -> int:
    return int(_lib.load().mla_decode_num_splits(B, s_q, H, max_seq_len, num_splits))


def mla_decode_workspace_bytes(B, s_q, H, max_seq_len, num_splits=0) -> int:
    return int(_lib.load().mla_decode_workspace_bytes(B, s_q, H, max_seq_len, num_splits))


def _decode_io(q_c, q_r, out, out_dtype, lse, workspace, max_seq_len, num_splits):
    B, s_q, H = q_c.shape[:3]
    qc = _need(q_c, "q_c", torch.bfloat16, (B, s_q, H, D_C))
    qr = _need(q_r, "q_r", torch.bfloat16, (B, s_q, H, D_R))
    if out is None:
        out = torch.empty((B, s_q, H, D_C), dtype=out_dtype, device=q_c.device)
    if out.dtype not in (torch.bfloat16, torch.float32):
        raise TypeError("out must be bfloat16 or float32")
    po = _need(out, "out", out.dtype, (B, s_q, H, D_C))
    pl = None
    if lse is not None:
        pl = _need(lse, "lse", torch.float32, (B, s_q, H))
    need = mla_decode_workspace_bytes(B, s_q, H, max_seq_len, num_splits)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=q_c.device)
    pw, nw = (None, 0) if workspace is None else (_need(workspace, "workspace", torch.uint8), workspace.numel())
    return (B, s_q, H), qc, qr, out, po, pl, pw, nw, int(out.dtype == torch.float32), workspace


def mla_qdecode(desc, pool, block_table, seq_lens, max_seq_len, q_c, q_r, scale, *, out=None,
                out_dtype=torch.bfloat16, lse=None, num_splits=0, workspace=None, flags=0, stream=None):
    """Returns (out, lse). See include/mla_qcache.h for the contract."""
    (B, s_q, H), qc, qr, out, po, pl, pw, nw, f32, _ = _decode_io(
        q_c, q_r, out, out_dtype, lse, workspace, max_seq_len, num_splits)
    B_ = seq_lens.shape[0]
    if B_ != B:
        raise ValueError("seq_lens must have one entry per request")
    check("mla_qdecode", _lib.load().mla_qdecode(
        ctypes.byref(desc), _need(pool, "pool", torch.uint8), _need(block_table, "block_table", torch.int32),
        block_table.shape[1], _need(seq_lens, "seq_lens", torch.int32), int(max_seq_len), qc, qr, B, s_q, H,
        float(scale), int(num_splits), pw, nw, po, f32, pl, int(flags), _stream(stream)))
    return out, lse


def mla_qdecode_noalloc(desc, pool, block_table, seq_lens, max_seq_len, q_c, q_r, scale, out, lse=None, *,
                        num_splits=0, flags=0, stream=None):
    """mla_qdecode without a workspace argument, for callers that cannot
    allocate: the split-KV scratch is a fixed array inside the library (see
    include/mla_qcache.h). `out` must be given; nothing is allocated here."""
    B, s_q, H = q_c.shape[:3]
    f32 = {torch.float32: 1, torch.bfloat16: 0}[out.dtype]
    check("mla_qdecode_noalloc", _lib.load().mla_qdecode_noalloc(
        ctypes.byref(desc), _need(pool, "pool", torch.uint8), _need(block_table, "block_table", torch.int32),
        block_table.shape[1], _need(seq_lens, "seq_lens", torch.int32, (B,)), int(max_seq_len),
        _need(q_c, "q_c", torch.bfloat16, (B, s_q, H, D_C)), _need(q_r, "q_r", torch.bfloat16, (B, s_q, H, D_R)),
        B, s_q, H, float(scale), int(num_splits), _need(out, "out", out.dtype, (B, s_q, H, D_C)), f32,
        None if lse is None else _need(lse, "lse", torch.float32, (B, s_q, H)), int(flags), _stream(stream)))
    return out, lse


def mla_qdecode_fused_append(desc, pool, block_table, seq_lens, max_seq_len, c_new, kr_new, q_c, q_r, scale, *,
                             out=None, out_dtype=torch.bfloat16, lse=None, num_splits=0, workspace=None, flags=0,
                             stream=None):
    """Append the step's new tokens (c_new [B, n, 512], kr_new [B, n, 64]; seq_lens count them) and
    decode, in one call. Returns (out, lse). See include/mla_qcache.h for the contract."""
    (B, s_q, H), qc, qr, out, po, pl, pw, nw, f32, _ = _decode_io(
        q_c, q_r, out, out_dtype, lse, workspace, max_seq_len, num_splits)
    if seq_lens.shape[0] != B or c_new.shape[0] != B:
        raise ValueError("seq_lens and c_new must have one entry per request")
    n = c_new.shape[1]
    check("mla_qdecode_fused_append", _lib.load().mla_qdecode_fused_append(
        ctypes.byref(desc), _need(pool, "pool", torch.uint8), _need(block_table, "block_table", torch.int32),
        block_table.shape[1], _need(seq_lens, "seq_lens", torch.int32), int(max_seq_len),
        _need(c_new, "c_new", torch.bfloat16, (B, n, D_C)), _need(kr_new, "kr_new", torch.bfloat16, (B, n, D_R)), n,
        qc, qr, B, s_q, H, float(scale), int(num_splits), pw, nw, po, f32, pl, int(flags), _stream(stream)))
    return out, lse


def mla_decode_bf16(pool, block_table, seq_lens, max_seq_len, q_c, q_r, scale, *, out=None,
                    out_dtype=torch.bfloat16, lse=None, num_splits=0, workspace=None, flags=0, stream=None):
    (B, s_q, H), qc, qr, out, po, pl, pw, nw, f32, _ = _decode_io(
        q_c, q_r, out, out_dtype, lse, workspace, max_seq_len, num_splits)
    check("mla_decode_bf16", _lib.load().mla_decode_bf16(
        _need(pool, "pool", torch.bfloat16), pool.shape[0], pool.shape[1],
        _need(block_table, "block_table", torch.int32), block_table.shape[1],
        _need(seq_lens, "seq_lens", torch.int32), int(max_seq_len), qc, qr, B, s_q, H, float(scale),
        int(num_splits), pw, nw, po, f32, pl, int(flags), _stream(stream)))
    return out, lse


def mla_qcache_append_bf16_pages(desc, pool, block_table, seq_lens_before, bf16_pool, src_pages, stream=None) -> None:
    """Quantize whole BF16 pages (src_pages[b] of bf16_pool, or -1) into the quantized cache at
    positions seq_lens_before[b] .. + 63. See include/mla_qcache.h."""
    B = src_pages.shape[0]
    check("mla_qcache_append_bf16_pages", _lib.load().mla_qcache_append_bf16_pages(
        ctypes.byref(desc), _need(pool, "pool", torch.uint8), _need(block_table, "block_table", torch.int32),
        block_table.shape[1], _need(seq_lens_before, "seq_lens_before", torch.int32, (B,)),
        _need(bf16_pool, "bf16_pool", torch.bfloat16), bf16_pool.shape[0],
        _need(src_pages, "src_pages", torch.int32, (B,)), B, _stream(stream)))


def mla_qdecode_hybrid_workspace_bytes(B, s_q, H, max_hist_len, max_prot_len) -> int:
    return int(_lib.load().mla_qdecode_hybrid_workspace_bytes(B, s_q, H, max_hist_len, max_prot_len))


def mla_qdecode_hybrid(desc, pool, block_table, hist_lens, max_hist_len, bf16_pool, prot_table, prot_lens,
                       max_prot_len, q_c, q_r, scale, *, out=None, out_dtype=torch.bfloat16, lse=None,
                       workspace=None, stream=None):
    """Decode over a hybrid cache (quantized history + BF16 sink and window). Returns (out, lse)."""
    B, s_q, H = q_c.shape[:3]
    qc = _need(q_c, "q_c", torch.bfloat16, (B, s_q, H, D_C))
    qr = _need(q_r, "q_r", torch.bfloat16, (B, s_q, H, D_R))
    if out is None:
        out = torch.empty((B, s_q, H, D_C), dtype=out_dtype, device=q_c.device)
    po = _need(out, "out", out.dtype, (B, s_q, H, D_C))
    pl = None if lse is None else _need(lse, "lse", torch.float32, (B, s_q, H))
    need = mla_qdecode_hybrid_workspace_bytes(B, s_q, H, max_hist_len, max_prot_len)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q_c.device)
    check("mla_qdecode_hybrid", _lib.load().mla_qdecode_hybrid(
        ctypes.byref(desc), _need(pool, "pool", torch.uint8), _need(block_table, "block_table", torch.int32),
        block_table.shape[1], _need(hist_lens, "hist_lens", torch.int32, (B,)), int(max_hist_len),
        _need(bf16_pool, "bf16_pool", torch.bfloat16), bf16_pool.shape[0],
        _need(prot_table, "prot_table", torch.int32), prot_table.shape[1],
        _need(prot_lens, "prot_lens", torch.int32, (B,)), int(max_prot_len), qc, qr, B, s_q, H, float(scale),
        _need(workspace, "workspace", torch.uint8), workspace.numel(), po, int(out.dtype == torch.float32), pl,
        _stream(stream)))
    return out, lse


def mla_cache_bytes_per_request(desc, seq_len, sink=0, window=0) -> int:
    """Bytes one request holds (desc None: the BF16 cache). See include/mla_qcache.h."""
    return int(_lib.load().mla_cache_bytes_per_request(None if desc is None else ctypes.byref(desc),
                                                       int(seq_len), int(sink), int(window)))


def mla_cache_max_requests(desc, seq_len, budget_bytes, sink=0, window=0) -> int:
    return int(_lib.load().mla_cache_max_requests(None if desc is None else ctypes.byref(desc), int(seq_len),
                                                  int(sink), int(window), int(budget_bytes)))


def mla_get_device_status(stream=None) -> int:
    v = ctypes.c_int(0)
    check("mla_get_device_status", _lib.load().mla_get_device_status(ctypes.byref(v), _stream(stream)))
    return int(v.value)
