// C ABI of the low-bit MLA decode library: argument validation, split
// planning, dispatch to the kernels, and the per-device status word.
// Declarations and the contract of every entry point: include/mla_qcache.h.
#include <math.h>
#include <stddef.h>
#include <stdint.h>

#include <algorithm>
#include <mutex>

#include "mla_common.cuh"
#include "mla_internal.h"

namespace {

// First error recorded by any kernel on this device since the last read.
__device__ int g_device_status;

constexpr int kMaxDevices = 64;
std::mutex g_status_mu;
int* g_status_ptr[kMaxDevices] = {};

// Device address of g_device_status on the current device (looked up once per
// device; cudaGetSymbolAddress needs that device current).
int* status_ptr() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lk(g_status_mu);
  if (!g_status_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_device_status) != cudaSuccess) return nullptr;
    g_status_ptr[dev] = static_cast<int*>(p);
  }
  return g_status_ptr[dev];
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

size_t align_up(size_t n, size_t a) { return (n + a - 1) / a * a; }

bool supported_bits(int b) { return b == 2 || b == 4; }
bool supported_group(int g) { return g == 32 || g == 64; }

int device_sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
    cudaGetLastError();  // clear a sticky "no device" from the query
    return 148;          // B200
  }
  return n;
}

struct SplitPlan {
  int n_split;
  int chunk_pages;
};

// Split each request's pages into n page-aligned chunks. No chunk holds more
// than kMaxChunkPages pages: the tensor cores' fp32 accumulation loses
// accuracy in proportion to the keys one accumulator sums (measured on B200
// at about 5e-8 x RMS per key), so 8,192 keys keep the output within about
// 4.5e-4 x RMS of exact, a fourfold margin on the stated bound. An explicit
// request is honoured (capped at the page count) when it meets that limit and
// raised to it otherwise. The automatic choice models the decode time of the
// longest request as waves(n) * (pages / n), where a wave is one work unit
// (128 query rows of one request and one split) on each 2-CTA cluster slot --
// or, for at most 16 query rows, one request and split on each of two CTA
// slots per SM (the small-row kernel) -- and picks the smallest n within 3% of
// the best, with chunks of at least 4 pages for the tensor-core kernel (a unit
// costs it about two pages of set-up and epilogue) and of at least one page
// for the small-row kernel.
constexpr int kMaxChunkPages = 128;

SplitPlan plan_splits(int B, int s_q, int H, int max_seq_len, int requested) {
  const int pages = std::max(1, (max_seq_len + mla::kPage - 1) / mla::kPage);
  const int n_min = (pages + kMaxChunkPages - 1) / kMaxChunkPages;
  int n;
  if (requested > 0) {
    n = std::max(std::min(requested, pages), n_min);
  } else {
    const bool small = static_cast<long>(s_q) * H <= mla::kSmallRows;
    const long units = static_cast<long>(std::max(B, 1)) * (small ? 1 : (static_cast<long>(s_q) * H + 127) / 128);
    const long slots = std::max(1, small ? 2 * device_sm_count() : device_sm_count() / 2);
    const int n_max = std::max(n_min, std::min(small ? pages : pages / 4, 64));
    double best = 1e30;
    n = n_min;
    for (int c = n_min; c <= n_max; ++c) {
      const long waves = (units * c + slots - 1) / slots;
      const double cost = static_cast<double>(waves) * ((pages + c - 1) / c) + 2.0 * waves;  // + per-unit overhead
      if (cost < best * 0.97) {
        best = cost;
        n = c;
      }
    }
  }
  const int chunk = (pages + n - 1) / n;
  return SplitPlan{(pages + chunk - 1) / chunk, chunk};
}

// Units of the tensor-core kernel (request, split, 128-row tile).
long tc_units(int B, int rows, const SplitPlan& p) {
  return static_cast<long>(B) * p.n_split * ((rows + 127) / 128);
}

// Whether the tensor-core kernel takes its units from a device-built work
// list, longest first: for split plans whose grid runs in more than two waves
// of its 2-CTA cluster slots, where the order of the units decides the tail.
bool use_worklist(int B, int rows, const SplitPlan& p) {
  if (rows <= mla::kSmallRows || p.n_split <= 1 || p.chunk_pages > mla::kMaxWorklistChunkPages) return false;
  const long units = tc_units(B, rows, p);
  return units > 2L * (device_sm_count() / 2) && units <= (1L << 24);
}

// Bytes of the split partials (lse, then o), 256-byte aligned.
size_t partials_bytes(int B, int rows, const SplitPlan& p) {
  const size_t parts = static_cast<size_t>(B) * p.n_split * rows;
  return align_up(parts * sizeof(float), 256) + align_up(parts * mla::kDc * sizeof(float), 256);
}

// Workspace of a decode: the split partials, then the work list (int32 per unit) when used.
size_t workspace_for(int B, int rows, const SplitPlan& p) {
  if (p.n_split <= 1) return 0;
  size_t bytes = partials_bytes(B, rows, p);
  if (use_worklist(B, rows, p)) bytes += static_cast<size_t>(tc_units(B, rows, p)) * sizeof(int);
  return bytes;
}

mla_status from_cuda(cudaError_t e) { return e == cudaSuccess ? MLA_OK : MLA_ERR_CUDA; }

// Hybrid decode workspace: the two segments' fp32 results and lse, then the
// scratch their decodes share (they run one after the other on one stream).
struct HybridWorkspace {
  size_t off_o_hist, off_l_hist, off_o_prot, off_l_prot, off_inner, inner, total;
};

HybridWorkspace hybrid_workspace(int B, int s_q, int H, int max_hist_len, int max_prot_len) {
  const size_t rows = static_cast<size_t>(B) * s_q * H;
  HybridWorkspace w{};
  w.off_o_hist = 0;
  w.off_l_hist = align_up(w.off_o_hist + rows * mla::kDc * sizeof(float), 256);
  w.off_o_prot = align_up(w.off_l_hist + rows * sizeof(float), 256);
  w.off_l_prot = align_up(w.off_o_prot + rows * mla::kDc * sizeof(float), 256);
  w.off_inner = align_up(w.off_l_prot + rows * sizeof(float), 256);
  w.inner = std::max(workspace_for(B, s_q * H, plan_splits(B, 1, s_q * H, max_hist_len, 0)),
                     workspace_for(B, s_q * H, plan_splits(B, s_q, H, max_prot_len, 0)));
  w.total = w.off_inner + w.inner;
  return w;
}

struct DecodeCommon {
  const void* pool;
  int num_pages;
  const int32_t* block_table;
  int max_pages_per_seq;
  const int32_t* seq_lens;
  int max_seq_len;
  const void* q_c;
  const void* q_r;
  int B, s_q, H;
  float scale;
  int num_splits;
  void* workspace;
  size_t workspace_bytes;
  void* out;
  int out_dtype;
  float* lse;
  unsigned flags;
  cudaStream_t stream;
  // fused append (quantized cache): new tokens, the last n_new of seq_lens[b]
  const void* c_new;
  const void* kr_new;
  int n_new;
};

mla_status run_decode(const DecodeCommon& c, bool quantized, const mla_qcache_desc* desc) {
  if (c.B < 0 || c.s_q < 1 || c.H < 1 || c.num_pages < 0 || c.max_seq_len < 0 || c.num_splits < 0)
    return MLA_ERR_INVALID_ARG;
  if (c.out_dtype != 0 && c.out_dtype != 1) return MLA_ERR_INVALID_ARG;
  if (!isfinite(c.scale)) return MLA_ERR_INVALID_ARG;
  if (c.flags & ~(MLA_DECODE_FORCE_SIMT | MLA_DECODE_FAST_UNCOMPENSATED | MLA_DECODE_TEST_STALL))
    return MLA_ERR_INVALID_ARG;
  if (c.n_new < 0 || (c.n_new > 0 && (!quantized || !c.c_new || !c.kr_new))) return MLA_ERR_INVALID_ARG;
  if (c.n_new > 0 && (!aligned(c.c_new, 16) || !aligned(c.kr_new, 16) || !c.pool)) return MLA_ERR_INVALID_ARG;
  if (static_cast<long>(c.B) * c.n_new > (1L << 26)) return MLA_ERR_UNSUPPORTED;
  if (c.B == 0) return MLA_OK;
  if (c.B > 65535 || static_cast<long>(c.s_q) * c.H > (1 << 20)) return MLA_ERR_UNSUPPORTED;
  if (!c.block_table || !c.seq_lens || !c.q_c || !c.q_r || !c.out) return MLA_ERR_INVALID_ARG;
  if (c.num_pages > 0 && !c.pool) return MLA_ERR_INVALID_ARG;
  if (c.max_pages_per_seq < 1) return MLA_ERR_INVALID_ARG;
  if (static_cast<long>(c.max_seq_len) > static_cast<long>(c.max_pages_per_seq) * mla::kPage)
    return MLA_ERR_CAPACITY;
  if (!aligned(c.q_c, 16) || !aligned(c.q_r, 16) || !aligned(c.out, 16) || (c.pool && !aligned(c.pool, 256)) ||
      !aligned(c.lse, 4))
    return MLA_ERR_INVALID_ARG;
  const int rows = c.s_q * c.H;
  const SplitPlan plan = plan_splits(c.B, c.s_q, c.H, c.max_seq_len, c.num_splits);
  if (plan.n_split > 65535) return MLA_ERR_UNSUPPORTED;
  const size_t need = workspace_for(c.B, rows, plan);
  if (need > 0 && (!c.workspace || c.workspace_bytes < need || !aligned(c.workspace, 256)))
    return MLA_ERR_WORKSPACE;

  int* status = status_ptr();
  if (!status) return MLA_ERR_CUDA;

  mla::DecodeLaunch L{};
  L.pool = c.pool;
  L.quantized = quantized;
  if (quantized) {
    L.bits_c = desc->bits_c;
    L.group_c = desc->group_c;
    L.bits_r = desc->bits_r;
    L.group_r = desc->group_r;
  }
  L.num_pages = c.num_pages;
  L.table = c.block_table;
  L.max_pages = c.max_pages_per_seq;
  L.seq_lens = c.seq_lens;
  L.max_seq_len = c.max_seq_len;
  L.q_c = c.q_c;
  L.q_r = c.q_r;
  L.B = c.B;
  L.s_q = c.s_q;
  L.H = c.H;
  L.scale = c.scale;
  L.n_split = plan.n_split;
  L.chunk_pages = plan.chunk_pages;
  if (plan.n_split > 1) {
    const size_t parts = static_cast<size_t>(c.B) * plan.n_split * rows;
    L.lse_part = static_cast<float*>(c.workspace);
    L.o_part = reinterpret_cast<float*>(static_cast<char*>(c.workspace) + align_up(parts * sizeof(float), 256));
    if (use_worklist(c.B, rows, plan))
      L.worklist = reinterpret_cast<int*>(static_cast<char*>(c.workspace) + partials_bytes(c.B, rows, plan));
  }
  L.out = c.out;
  L.out_f32 = c.out_dtype;
  L.lse = c.lse;
  L.flags = c.flags;
  L.status = status;
  L.stream = c.stream;

  // A fused append runs inside the tensor-core and small-row kernels; the
  // SIMT kernel gets the append kernel launched first (lengths here already
  // count the new tokens).
  auto append_first = [&]() -> cudaError_t {
    mla::AppendLaunch A{const_cast<void*>(c.pool), c.num_pages, c.block_table, c.max_pages_per_seq, c.seq_lens,
                        c.c_new, c.kr_new, c.B, c.n_new, L.bits_c, L.group_c, L.bits_r, L.group_r,
                        nullptr, 0, nullptr, status, c.stream, -c.n_new};
    return mla::launch_qcache_append(A);
  };
  cudaError_t e = cudaErrorNotSupported;
  if (!(c.flags & MLA_DECODE_FORCE_SIMT)) {
    if (c.n_new > 0) {
      L.c_new = c.c_new;
      L.kr_new = c.kr_new;
      L.n_new = c.n_new;
    }
    e = mla::launch_decode_small(L);
    if (e == cudaErrorNotSupported) {
      cudaGetLastError();
      e = mla::launch_decode_tc(L);  // returns NotSupported before launching anything
    }
  }
  if (e == cudaErrorNotSupported) {
    cudaGetLastError();
    if (L.n_new > 0) {  // neither the small-row nor the tensor-core kernel took the fused append
      L.n_new = 0;
      if (append_first() != cudaSuccess) return MLA_ERR_CUDA;
    } else if (c.n_new > 0 && (c.flags & MLA_DECODE_FORCE_SIMT)) {
      if (append_first() != cudaSuccess) return MLA_ERR_CUDA;
    }
    e = mla::launch_decode_simt(L);
  }
  if (e != cudaSuccess) return MLA_ERR_CUDA;
  if (plan.n_split > 1) return from_cuda(mla::launch_combine(L));
  return MLA_OK;
}

}  // namespace

extern "C" {

const char* mla_status_string(mla_status s) {
  switch (s) {
    case MLA_OK: return "MLA_OK";
    case MLA_ERR_INVALID_ARG: return "MLA_ERR_INVALID_ARG: invalid argument";
    case MLA_ERR_UNSUPPORTED: return "MLA_ERR_UNSUPPORTED: shape or bit width not supported by this build";
    case MLA_ERR_CAPACITY: return "MLA_ERR_CAPACITY: sequence does not fit its block-table row";
    case MLA_ERR_WORKSPACE: return "MLA_ERR_WORKSPACE: workspace missing, too small or misaligned";
    case MLA_ERR_CUDA: return "MLA_ERR_CUDA: a CUDA call failed";
    case MLA_ERR_TIMEOUT: return "MLA_ERR_TIMEOUT: a bounded device-side wait ran out";
  }
  return "unknown mla_status";
}

int mla_qcache_layout_version(void) { return MLA_QCACHE_LAYOUT_VERSION; }

mla_status mla_qcache_check_desc(const mla_qcache_desc* d) {
  if (!d) return MLA_ERR_INVALID_ARG;
  if (d->d_c <= 0 || d->d_r <= 0 || d->bits_c <= 0 || d->bits_r <= 0 || d->group_c <= 0 || d->group_r <= 0 ||
      d->page_size <= 0 || d->num_pages < 0)
    return MLA_ERR_INVALID_ARG;
  if (d->d_c % d->group_c || d->d_r % d->group_r) return MLA_ERR_INVALID_ARG;
  if (d->d_c != mla::kDc || d->d_r != mla::kDr || d->page_size != mla::kPage) return MLA_ERR_UNSUPPORTED;
  if (!supported_bits(d->bits_c) || !supported_bits(d->bits_r) || !supported_group(d->group_c) ||
      !supported_group(d->group_r))
    return MLA_ERR_UNSUPPORTED;
  return MLA_OK;
}

mla_status mla_qcache_segment_offsets(const mla_qcache_desc* d, size_t out[5]) {
  if (!out) return MLA_ERR_INVALID_ARG;
  const mla_status st = mla_qcache_check_desc(d);
  if (st != MLA_OK) return st;
  const size_t P = d->page_size;
  out[0] = 0;
  out[1] = align_up(out[0] + P * (d->d_c * d->bits_c / 8), 16);
  out[2] = align_up(out[1] + P * (d->d_r * d->bits_r / 8), 16);
  out[3] = align_up(out[2] + P * (d->d_c / d->group_c) * 4, 16);
  out[4] = align_up(out[3] + P * (d->d_r / d->group_r) * 4, 16);
  return MLA_OK;
}

size_t mla_qcache_page_bytes(const mla_qcache_desc* d) {
  size_t off[5];
  return mla_qcache_segment_offsets(d, off) == MLA_OK ? off[4] : 0;
}

mla_status mla_qcache_append(const mla_qcache_desc* desc, void* pool, const int32_t* block_table,
                             int max_pages_per_seq, const int32_t* seq_lens_before, const void* c_new,
                             const void* kr_new, int B, int n_new, mla_stream_t stream) {
  const mla_status st = mla_qcache_check_desc(desc);
  if (st != MLA_OK) return st;
  if (B < 0 || n_new < 0) return MLA_ERR_INVALID_ARG;
  if (B == 0 || n_new == 0) return MLA_OK;
  if (!pool || !block_table || !seq_lens_before || !c_new || !kr_new || max_pages_per_seq < 1)
    return MLA_ERR_INVALID_ARG;
  if (!aligned(pool, 256) || !aligned(c_new, 16) || !aligned(kr_new, 16)) return MLA_ERR_INVALID_ARG;
  if (static_cast<long>(B) * n_new > (1L << 26)) return MLA_ERR_UNSUPPORTED;
  int* status = status_ptr();
  if (!status) return MLA_ERR_CUDA;
  mla::AppendLaunch L{pool, desc->num_pages, block_table, max_pages_per_seq, seq_lens_before, c_new, kr_new,
                      B, n_new, desc->bits_c, desc->group_c, desc->bits_r, desc->group_r,
                      nullptr, 0, nullptr, status, reinterpret_cast<cudaStream_t>(stream)};
  return from_cuda(mla::launch_qcache_append(L));
}

mla_status mla_qcache_append_bf16_pages(const mla_qcache_desc* desc, void* pool, const int32_t* block_table,
                                        int max_pages_per_seq, const int32_t* seq_lens_before,
                                        const void* bf16_pool, int bf16_num_pages, const int32_t* src_pages, int B,
                                        mla_stream_t stream) {
  const mla_status st = mla_qcache_check_desc(desc);
  if (st != MLA_OK) return st;
  if (B < 0 || bf16_num_pages < 0) return MLA_ERR_INVALID_ARG;
  if (B == 0) return MLA_OK;
  if (!pool || !block_table || !seq_lens_before || !src_pages || max_pages_per_seq < 1) return MLA_ERR_INVALID_ARG;
  if (bf16_num_pages > 0 && !bf16_pool) return MLA_ERR_INVALID_ARG;
  if (!aligned(pool, 256) || !aligned(bf16_pool, 16)) return MLA_ERR_INVALID_ARG;
  if (B > (1 << 20)) return MLA_ERR_UNSUPPORTED;
  int* status = status_ptr();
  if (!status) return MLA_ERR_CUDA;
  mla::AppendLaunch L{pool, desc->num_pages, block_table, max_pages_per_seq, seq_lens_before, nullptr, nullptr,
                      B, mla::kPage, desc->bits_c, desc->group_c, desc->bits_r, desc->group_r,
                      bf16_pool, bf16_num_pages, src_pages, status, reinterpret_cast<cudaStream_t>(stream)};
  return from_cuda(mla::launch_qcache_append(L));
}

mla_status mla_bf16cache_append(void* pool, int num_pages, int page_size, const int32_t* block_table,
                                int max_pages_per_seq, const int32_t* seq_lens_before, const void* c_new,
                                const void* kr_new, int B, int n_new, mla_stream_t stream) {
  if (page_size != mla::kPage) return page_size > 0 ? MLA_ERR_UNSUPPORTED : MLA_ERR_INVALID_ARG;
  if (B < 0 || n_new < 0 || num_pages < 0) return MLA_ERR_INVALID_ARG;
  if (B == 0 || n_new == 0) return MLA_OK;
  if (!pool || !block_table || !seq_lens_before || !c_new || !kr_new || max_pages_per_seq < 1)
    return MLA_ERR_INVALID_ARG;
  if (!aligned(pool, 256) || !aligned(c_new, 16) || !aligned(kr_new, 16)) return MLA_ERR_INVALID_ARG;
  if (static_cast<long>(B) * n_new > (1L << 26)) return MLA_ERR_UNSUPPORTED;
  int* status = status_ptr();
  if (!status) return MLA_ERR_CUDA;
  mla::AppendLaunch L{pool, num_pages, block_table, max_pages_per_seq, seq_lens_before, c_new, kr_new,
                      B, n_new, 0, 0, 0, 0, nullptr, 0, nullptr, status, reinterpret_cast<cudaStream_t>(stream)};
  return from_cuda(mla::launch_bf16cache_append(L));
}

int mla_decode_num_splits(int B, int s_q, int H, int max_seq_len, int num_splits) {
  if (B < 0 || s_q < 1 || H < 1 || max_seq_len < 0 || num_splits < 0) return 0;
  if (static_cast<long>(s_q) * H > (1 << 20)) return 0;  // beyond what a decode accepts; s_q * H must not overflow
  return plan_splits(B, s_q, H, max_seq_len, num_splits).n_split;
}

size_t mla_decode_workspace_bytes(int B, int s_q, int H, int max_seq_len, int num_splits) {
  if (B <= 0 || s_q < 1 || H < 1 || max_seq_len < 0 || num_splits < 0) return 0;
  if (static_cast<long>(s_q) * H > (1 << 20)) return 0;  // beyond what a decode accepts; s_q * H must not overflow
  return workspace_for(B, s_q * H, plan_splits(B, s_q, H, max_seq_len, num_splits));
}

mla_status mla_qdecode(const mla_qcache_desc* desc, const void* pool, const int32_t* block_table,
                       int max_pages_per_seq, const int32_t* seq_lens, int max_seq_len, const void* q_c,
                       const void* q_r, int B, int s_q, int H, float scale, int num_splits, void* workspace,
                       size_t workspace_bytes, void* out, int out_dtype, float* lse, unsigned flags,
                       mla_stream_t stream) {
  const mla_status st = mla_qcache_check_desc(desc);
  if (st != MLA_OK) return st;
  DecodeCommon c{pool, desc->num_pages, block_table, max_pages_per_seq, seq_lens, max_seq_len, q_c, q_r,
                 B, s_q, H, scale, num_splits, workspace, workspace_bytes, out, out_dtype, lse, flags,
                 reinterpret_cast<cudaStream_t>(stream)};
  return run_decode(c, true, desc);
}

mla_status mla_qdecode_fused_append(const mla_qcache_desc* desc, void* pool, const int32_t* block_table,
                                    int max_pages_per_seq, const int32_t* seq_lens, int max_seq_len,
                                    const void* c_new, const void* kr_new, int n_new, const void* q_c,
                                    const void* q_r, int B, int s_q, int H, float scale, int num_splits,
                                    void* workspace, size_t workspace_bytes, void* out, int out_dtype, float* lse,
                                    unsigned flags, mla_stream_t stream) {
  const mla_status st = mla_qcache_check_desc(desc);
  if (st != MLA_OK) return st;
  if (n_new < 0 || (n_new > 0 && !pool)) return MLA_ERR_INVALID_ARG;
  DecodeCommon c{pool, desc->num_pages, block_table, max_pages_per_seq, seq_lens, max_seq_len, q_c, q_r,
                 B, s_q, H, scale, num_splits, workspace, workspace_bytes, out, out_dtype, lse, flags,
                 reinterpret_cast<cudaStream_t>(stream), c_new, kr_new, n_new};
  return run_decode(c, true, desc);
}

mla_status mla_decode_bf16(const void* pool, int num_pages, int page_size, const int32_t* block_table,
                           int max_pages_per_seq, const int32_t* seq_lens, int max_seq_len, const void* q_c,
                           const void* q_r, int B, int s_q, int H, float scale, int num_splits, void* workspace,
                           size_t workspace_bytes, void* out, int out_dtype, float* lse, unsigned flags,
                           mla_stream_t stream) {
  if (page_size != mla::kPage) return page_size > 0 ? MLA_ERR_UNSUPPORTED : MLA_ERR_INVALID_ARG;
  DecodeCommon c{pool, num_pages, block_table, max_pages_per_seq, seq_lens, max_seq_len, q_c, q_r,
                 B, s_q, H, scale, num_splits, workspace, workspace_bytes, out, out_dtype, lse, flags,
                 reinterpret_cast<cudaStream_t>(stream)};
  return run_decode(c, false, nullptr);
}

size_t mla_qdecode_hybrid_workspace_bytes(int B, int s_q, int H, int max_hist_len, int max_prot_len) {
  if (B <= 0 || s_q < 1 || H < 1 || max_hist_len < 0 || max_prot_len < 0) return 0;
  return hybrid_workspace(B, s_q, H, max_hist_len, max_prot_len).total;
}

mla_status mla_qdecode_hybrid(const mla_qcache_desc* desc, const void* pool, const int32_t* block_table,
                              int max_pages_per_seq, const int32_t* hist_lens, int max_hist_len,
                              const void* bf16_pool, int bf16_num_pages, const int32_t* prot_table,
                              int prot_max_pages, const int32_t* prot_lens, int max_prot_len, const void* q_c,
                              const void* q_r, int B, int s_q, int H, float scale, void* workspace,
                              size_t workspace_bytes, void* out, int out_dtype, float* lse, mla_stream_t stream) {
  const mla_status st = mla_qcache_check_desc(desc);
  if (st != MLA_OK) return st;
  if (B < 0 || s_q < 1 || H < 1 || max_hist_len < 0 || max_prot_len < 0) return MLA_ERR_INVALID_ARG;
  if (out_dtype != 0 && out_dtype != 1) return MLA_ERR_INVALID_ARG;
  if (B == 0) return MLA_OK;
  if (static_cast<long>(B) * s_q * H > 0x7FFFFFFFL) return MLA_ERR_UNSUPPORTED;  // rows of the merge
  if (!out || !q_c || !q_r || !aligned(out, 16) || !aligned(lse, 4)) return MLA_ERR_INVALID_ARG;
  const HybridWorkspace hw = hybrid_workspace(B, s_q, H, max_hist_len, max_prot_len);
  if (!workspace || workspace_bytes < hw.total || !aligned(workspace, 256)) return MLA_ERR_WORKSPACE;
  char* base = static_cast<char*>(workspace);
  float* o_hist = reinterpret_cast<float*>(base + hw.off_o_hist);
  float* l_hist = reinterpret_cast<float*>(base + hw.off_l_hist);
  float* o_prot = reinterpret_cast<float*>(base + hw.off_o_prot);
  float* l_prot = reinterpret_cast<float*>(base + hw.off_l_prot);
  void* inner = hw.inner ? base + hw.off_inner : nullptr;
  const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  // history: every key is older than every query, so its rows are decoded as
  // s_q * H rows of one query position (no causal offset)
  DecodeCommon ch{pool, desc->num_pages, block_table, max_pages_per_seq, hist_lens, max_hist_len, q_c, q_r,
                  B, 1, s_q * H, scale, 0, inner, hw.inner, o_hist, 1, l_hist, 0, s};
  mla_status r = run_decode(ch, true, desc);
  if (r != MLA_OK) return r;
  // protected segment: position order, the newest s_q keys last (causal)
  DecodeCommon cp{bf16_pool, bf16_num_pages, prot_table, prot_max_pages, prot_lens, max_prot_len, q_c, q_r,
                  B, s_q, H, scale, 0, inner, hw.inner, o_prot, 1, l_prot, 0, s};
  r = run_decode(cp, false, nullptr);
  if (r != MLA_OK) return r;
  return from_cuda(mla::launch_merge2(o_hist, l_hist, o_prot, l_prot, B * s_q * H, out, out_dtype, lse, s));
}

size_t mla_cache_bytes_per_request(const mla_qcache_desc* desc, long seq_len, int sink, int window) {
  constexpr size_t kBf16Page = static_cast<size_t>(mla::kPage) * mla::kDqk * 2;
  if (seq_len < 0 || sink < 0 || window < 0 || sink % mla::kPage != 0) return 0;
  auto pages = [](long n) { return static_cast<size_t>((n + mla::kPage - 1) / mla::kPage); };
  if (!desc) {
    if (sink || window) return 0;
    return pages(seq_len) * kBf16Page;
  }
  mla_qcache_desc d = *desc;
  d.num_pages = 0;
  const size_t qpage = mla_qcache_page_bytes(&d);
  if (qpage == 0) return 0;
  if (sink == 0 && window == 0) return pages(seq_len) * qpage;
  const long hist = std::max(0L, (seq_len - sink - window) / mla::kPage * mla::kPage);
  const long prot_sink = std::min<long>(sink, seq_len);
  const long prot_window = seq_len - prot_sink - hist;
  return pages(hist) * qpage + (pages(prot_sink) + pages(prot_window)) * kBf16Page;
}

long mla_cache_max_requests(const mla_qcache_desc* desc, long seq_len, int sink, int window,
                            size_t budget_bytes) {
  const size_t per = mla_cache_bytes_per_request(desc, seq_len, sink, window);
  if (per == 0) return -1;  // invalid arguments, or an empty request (no bound)
  return static_cast<long>(budget_bytes / per);
}

mla_status mla_get_device_status(int* status, mla_stream_t stream) {
  if (!status) return MLA_ERR_INVALID_ARG;
  *status = MLA_OK;
  if (!status_ptr()) return MLA_ERR_CUDA;
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return MLA_ERR_CUDA;
  int v = 0;
  const int zero = 0;
  if (cudaMemcpyFromSymbol(&v, g_device_status, sizeof(int)) != cudaSuccess) return MLA_ERR_CUDA;
  if (cudaMemcpyToSymbol(g_device_status, &zero, sizeof(int)) != cudaSuccess) return MLA_ERR_CUDA;
  *status = v;
  return MLA_OK;
}

}  // extern "C"
