// Cache writer: quantize + pack + paged scatter of new tokens.
//
// QuantMLA (arxivdaily.com/papers/2609.36760, English abstract) keeps the
// content and RoPE caches in INT4 (or INT2 content) and never holds a
// full-history high-precision copy, so every new token is quantized as it is
// written. One warp handles one token: lane l owns content channels
// [16l, 16l+16) and RoPE channels {2l, 2l+1}; a group's min/max is a shuffle
// reduction over the lanes that share it. All arithmetic is IEEE fp32 with
// explicit round-to-nearest intrinsics so codes match a plain fp32 reference
// bit for bit.
#include "mla_common.cuh"
#include "mla_internal.h"
#include "sm100_ptx.cuh"

namespace mla {

template <int BITS>
__device__ __forceinline__ uint32_t quantize_code(float x, float s, float z) {
  constexpr float qmax = static_cast<float>((1 << BITS) - 1);
  if (s == 0.0f) return 0u;
  float t = rintf(__fdiv_rn(__fsub_rn(x, z), s));
  t = fminf(fmaxf(t, 0.0f), qmax);
  return static_cast<uint32_t>(t);
}

// Group scale and zero-point from the group's min and max.
template <int BITS>
__device__ __forceinline__ void group_params(float mn, float mx, __half& s16, __half& z16) {
  constexpr float qmax = static_cast<float>((1 << BITS) - 1);
  mn = __fadd_rn(mn, 0.0f);  // a -0.0 minimum becomes +0.0
  s16 = __float2half_rn(__fdiv_rn(__fsub_rn(mx, mn), qmax));
  z16 = __float2half_rn(mn);
}

template <int BITS_C, int G_C, int BITS_R, int G_R>
__global__ void __launch_bounds__(256)
qcache_append_kernel(uint8_t* __restrict__ pool, int num_pages, const int32_t* __restrict__ table,
                     int max_pages, const int32_t* __restrict__ lens_before,
                     const __nv_bfloat16* __restrict__ c_new, const __nv_bfloat16* __restrict__ kr_new,
                     const __nv_bfloat16* __restrict__ src_pool, int src_num_pages,
                     const int32_t* __restrict__ src_pages, int n_tokens, int n_new, int* status) {
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
  const int t = __ldg(lens_before + b) + j;
  const int page = lookup_page(table, max_pages, num_pages, b, t);
  if (page < 0) {
    if (lane == 0) record_error(status, MLA_ERR_INVALID_ARG);
    return;
  }
  const int slot = t % kPage;
  uint8_t* pg = pool + static_cast<size_t>(page) * G::kPageBytes;

  // ---- content path: 16 channels per lane ----
  const uint4* src = reinterpret_cast<const uint4*>(c_src) + 2 * lane;
  const uint4 v0 = __ldg(src), v1 = __ldg(src + 1);
  const uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
  float x[16];
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    x[2 * k] = bf16_lo(w[k]);
    x[2 * k + 1] = bf16_hi(w[k]);
  }
  float mn = x[0], mx = x[0];
#pragma unroll
  for (int k = 1; k < 16; ++k) {
    mn = fminf(mn, x[k]);
    mx = fmaxf(mx, x[k]);
  }
  constexpr int kLanesC = G_C / 16;  // lanes sharing one content group
#pragma unroll
  for (int o = 1; o < kLanesC; o <<= 1) {
    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  }
  __half s16, z16;
  group_params<BITS_C>(mn, mx, s16, z16);
  const float s = __half2float(s16), z = __half2float(z16);
  uint32_t packed[2] = {0u, 0u};
#pragma unroll
  for (int k = 0; k < 16; ++k) {
    const uint32_t u = quantize_code<BITS_C>(x[k], s, z);
    const int bit = k * BITS_C;
    packed[bit >> 5] |= u << (bit & 31);
  }
  uint8_t* crow = pg + G::kOffCC + slot * G::kRowC;
  if constexpr (BITS_C == 4) {
    reinterpret_cast<uint2*>(crow)[lane] = make_uint2(packed[0], packed[1]);
  } else {
    reinterpret_cast<uint32_t*>(crow)[lane] = packed[0];
  }
  if ((lane % kLanesC) == 0) {
    const uint32_t meta = static_cast<uint32_t>(__half_as_ushort(s16)) |
                          (static_cast<uint32_t>(__half_as_ushort(z16)) << 16);
    reinterpret_cast<uint32_t*>(pg + G::kOffCM + slot * G::kGroupsC * 4)[lane / kLanesC] = meta;
  }

  // ---- RoPE path: 2 channels per lane ----
  const uint32_t rw = __ldg(reinterpret_cast<const uint32_t*>(kr_src) + lane);
  const float r0 = bf16_lo(rw), r1 = bf16_hi(rw);
  float rmn = fminf(r0, r1), rmx = fmaxf(r0, r1);
  constexpr int kLanesR = G_R / 2;
#pragma unroll
  for (int o = 1; o < kLanesR; o <<= 1) {
    rmn = fminf(rmn, __shfl_xor_sync(0xffffffffu, rmn, o));
    rmx = fmaxf(rmx, __shfl_xor_sync(0xffffffffu, rmx, o));
  }
  __half rs16, rz16;
  group_params<BITS_R>(rmn, rmx, rs16, rz16);
  const float rs = __half2float(rs16), rz = __half2float(rz16);
  const uint32_t rbits = quantize_code<BITS_R>(r0, rs, rz) | (quantize_code<BITS_R>(r1, rs, rz) << BITS_R);
  uint8_t* rrow = pg + G::kOffRC + slot * G::kRowR;
  if constexpr (BITS_R == 4) {
    rrow[lane] = static_cast<uint8_t>(rbits);
  } else {
    const uint32_t nb = __shfl_down_sync(0xffffffffu, rbits, 1);
    if ((lane & 1) == 0) rrow[lane >> 1] = static_cast<uint8_t>(rbits | (nb << 4));
  }
  if ((lane % kLanesR) == 0) {
    const uint32_t meta = static_cast<uint32_t>(__half_as_ushort(rs16)) |
                          (static_cast<uint32_t>(__half_as_ushort(rz16)) << 16);
    reinterpret_cast<uint32_t*>(pg + G::kOffRM + slot * G::kGroupsR * 4)[lane / kLanesR] = meta;
  }
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
      static_cast<const __nv_bfloat16*>(L.src_pool), L.src_num_pages, L.src_pages, n_tokens, L.n_new, L.status);
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
