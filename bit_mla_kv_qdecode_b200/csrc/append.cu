// Cache writer: quantize + pack + paged scatter of new tokens, one warp per
// token (the per-token writer is in append_token.cuh).
#include "append_token.cuh"
#include "mla_common.cuh"
#include "mla_internal.h"
#include "sm100_ptx.cuh"

namespace mla {

template <int BITS_C, int G_C, int BITS_R, int G_R>
__global__ void __launch_bounds__(256)
qcache_append_kernel(uint8_t* __restrict__ pool, int num_pages, const int32_t* __restrict__ table,
                     int max_pages, const int32_t* __restrict__ lens_before,
                     const __nv_bfloat16* __restrict__ c_new, const __nv_bfloat16* __restrict__ kr_new,
                     const __nv_bfloat16* __restrict__ src_pool, int src_num_pages,
                     const int32_t* __restrict__ src_pages, int n_tokens, int n_new, int lens_offset,
                     int* status) {
  using G = QGeom<BITS_C, G_C, BITS_R, G_R>;
  ptx::griddep_launch_dependents();  // a decode launched as a programmatic dependent may be scheduled now
  const int lane = threadIdx.x & 31;
  const int tok = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  if (tok >= n_tokens) return;
  const int b = tok / n_new, j = tok - b * n_new;
  // token source: the dense arrays, or row j of BF16 page src_pages[b] ([64][576], content then RoPE)
  const __nv_bfloat16* c_src;
  const __nv_bfloat16* kr_src;
  if (!src_pages) {
    c_src = c_new + static_cast<size_t>(tok) * kDc;
    kr_src = kr_new + static_cast<size_t>(tok) * kDr;
  } else {
    const int sp = __ldg(src_pages + b);
    if (sp < 0) return;  // this request moves nothing
    if (sp >= src_num_pages) {
      if (lane == 0) record_error(status, MLA_ERR_INVALID_ARG);
      return;
    }
    c_src = src_pool + (static_cast<size_t>(sp) * kPage + j) * kDqk;
    kr_src = c_src + kDc;
  }
  const int t = __ldg(lens_before + b) + lens_offset + j;
  const int page = lookup_page(table, max_pages, num_pages, b, t);
  if (page < 0) {
    if (lane == 0) record_error(status, MLA_ERR_INVALID_ARG);
    return;
  }
  quantize_token_warp<BITS_C, G_C, BITS_R, G_R>(pool + static_cast<size_t>(page) * G::kPageBytes, t % kPage,
                                                 c_src, kr_src, lane);
}

// Unquantized comparison cache: copy each token's 576 bf16 channels.
__global__ void __launch_bounds__(256)
bf16cache_append_kernel(__nv_bfloat16* __restrict__ pool, int num_pages, const int32_t* __restrict__ table,
                        int max_pages, const int32_t* __restrict__ lens_before,
                        const __nv_bfloat16* __restrict__ c_new, const __nv_bfloat16* __restrict__ kr_new,
                        int n_tokens, int n_new, int* status) {
  ptx::griddep_launch_dependents();
  const int lane = threadIdx.x & 31;
  const int tok = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  if (tok >= n_tokens) return;
  const int b = tok / n_new, j = tok - b * n_new;
  const int t = __ldg(lens_before + b) + j;
  const int page = lookup_page(table, max_pages, num_pages, b, t);
  if (page < 0) {
    if (lane == 0) record_error(status, MLA_ERR_INVALID_ARG);
    return;
  }
  uint4* dst = reinterpret_cast<uint4*>(pool + (static_cast<size_t>(page) * kPage + t % kPage) * kDqk);
  const uint4* sc = reinterpret_cast<const uint4*>(c_new + static_cast<size_t>(tok) * kDc);
  const uint4* sr = reinterpret_cast<const uint4*>(kr_new + static_cast<size_t>(tok) * kDr);
  dst[lane] = __ldg(sc + lane);
  dst[lane + 32] = __ldg(sc + lane + 32);
  if (lane < 8) dst[64 + lane] = __ldg(sr + lane);
}

template <int BC, int GC, int BR, int GR>
static cudaError_t launch_append_t(const AppendLaunch& L) {
  const int n_tokens = L.B * L.n_new;
  const int blocks = (n_tokens + 7) / 8;
  qcache_append_kernel<BC, GC, BR, GR><<<blocks, 256, 0, L.stream>>>(
      static_cast<uint8_t*>(L.pool), L.num_pages, L.table, L.max_pages, L.lens_before,
      static_cast<const __nv_bfloat16*>(L.c_new), static_cast<const __nv_bfloat16*>(L.kr_new),
      static_cast<const __nv_bfloat16*>(L.src_pool), L.src_num_pages, L.src_pages, n_tokens, L.n_new, L.lens_offset,
      L.status);
  return cudaGetLastError();
}

cudaError_t launch_qcache_append(const AppendLaunch& L) {
  // bits in {2,4} x group in {32,64} for both paths
#define MLA_APPEND_CASE(BC, GC, BR, GR)                                                   \
  if (L.bits_c == BC && L.group_c == GC && L.bits_r == BR && L.group_r == GR)           \
    return launch_append_t<BC, GC, BR, GR>(L);
#define MLA_APPEND_R(BC, GC) \
  MLA_APPEND_CASE(BC, GC, 4, 64) MLA_APPEND_CASE(BC, GC, 4, 32) MLA_APPEND_CASE(BC, GC, 2, 64) MLA_APPEND_CASE(BC, GC, 2, 32)
  MLA_APPEND_R(4, 64)
  MLA_APPEND_R(4, 32)
  MLA_APPEND_R(2, 64)
  MLA_APPEND_R(2, 32)
#undef MLA_APPEND_R
#undef MLA_APPEND_CASE
  return cudaErrorInvalidValue;
}

cudaError_t launch_bf16cache_append(const AppendLaunch& L) {
  const int n_tokens = L.B * L.n_new;
  const int blocks = (n_tokens + 7) / 8;
  bf16cache_append_kernel<<<blocks, 256, 0, L.stream>>>(
      static_cast<__nv_bfloat16*>(L.pool), L.num_pages, L.table, L.max_pages, L.lens_before,
      static_cast<const __nv_bfloat16*>(L.c_new), static_cast<const __nv_bfloat16*>(L.kr_new),
      n_tokens, L.n_new, L.status);
  return cudaGetLastError();
}

}  // namespace mla
