// CUDA-core decode: dequantize-then-attend in fp32, plus the split-KV combine.
//
// Absorbed MQA form of MLA decode (Group-Query Latent Attention abstract,
// thelatestinai.com/papers/2607.27269): all heads attend one shared latent,
//   score_t = (q_c . c_t + q_r . k_r,t) * scale,  o = sum_t softmax_t c_t.
// The cache is unpacked and dequantized inside the attention loop (QuantMLA,
// arxivdaily.com/papers/2609.36760, English abstract), never materialised.
//
// This kernel is the simple, exact path: a CTA takes 16 query rows of one
// request and one key split, stages 32 dequantized tokens at a time in shared
// memory as fp32 (u*s + z is exact there), and keeps an online softmax in the
// log2 domain. It serves shapes the tensor-core kernel does not cover and
// cross-checks that kernel.
#include <math_constants.h>

#include "mla_common.cuh"
#include "mla_internal.h"
#include "sm100_ptx.cuh"

namespace mla {
namespace {

constexpr int kRowsT = 16;
constexpr int kTokT = 32;
constexpr int kThreads = 256;
constexpr int kStride = kDqk + 1;  // padded fp32 row stride: conflict-free columns

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ void bf16x8_to_f32(uint4 v, float* d) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    d[2 * k] = bf16_lo(w[k]);
    d[2 * k + 1] = bf16_hi(w[k]);
  }
}

// Channels [c0, c0+8) of one cached token, dequantized to fp32.
template <class G>
struct QuantSource {
  __device__ static void load8(const DecodeArgs& a, int page, int slot, int c0, float* d) {
    const uint8_t* pg = a.pool + static_cast<size_t>(page) * G::kPageBytes;
    uint32_t meta, w;
    int bits, c;
    if (c0 < kDc) {
      c = c0;
      bits = G::kBitsC;
      meta = __ldg(reinterpret_cast<const uint32_t*>(pg + G::kOffCM + slot * G::kGroupsC * 4) + c / G::kGroupC);
      const uint8_t* row = pg + G::kOffCC + slot * G::kRowC;
      w = (bits == 4) ? __ldg(reinterpret_cast<const uint32_t*>(row + c / 2))
                      : __ldg(reinterpret_cast<const uint16_t*>(row + c / 4));
    } else {
      c = c0 - kDc;
      bits = G::kBitsR;
      meta = __ldg(reinterpret_cast<const uint32_t*>(pg + G::kOffRM + slot * G::kGroupsR * 4) + c / G::kGroupR);
      const uint8_t* row = pg + G::kOffRC + slot * G::kRowR;
      w = (bits == 4) ? __ldg(reinterpret_cast<const uint32_t*>(row + c / 2))
                      : __ldg(reinterpret_cast<const uint16_t*>(row + c / 4));
    }
    const float s = half_bits_to_float(meta), z = half_bits_to_float(meta >> 16);
    const uint32_t mask = (1u << bits) - 1u;
#pragma unroll
    for (int k = 0; k < 8; ++k) d[k] = fmaf(static_cast<float>((w >> (k * bits)) & mask), s, z);
  }
};

struct Bf16Source {
  __device__ static void load8(const DecodeArgs& a, int page, int slot, int c0, float* d) {
    const uint4* p = reinterpret_cast<const uint4*>(
        reinterpret_cast<const __nv_bfloat16*>(a.pool) + (static_cast<size_t>(page) * kPage + slot) * kDqk + c0);
    bf16x8_to_f32(__ldg(p), d);
  }
};

template <class Src>
__global__ void __launch_bounds__(kThreads) decode_simt_kernel(DecodeArgs a) {
  ptx::griddep_wait();
  ptx::griddep_launch_dependents();
  extern __shared__ float smem[];
  float* sQ = smem;                    // [16][577]
  float* sK = sQ + kRowsT * kStride;   // [32][577]
  float* sP = sK + kTokT * kStride;    // [16][32]
  float* sAlpha = sP + kRowsT * kTokT; // [16]
  float* sML = sAlpha + kRowsT;        // [16][2]

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int b = blockIdx.z, split = blockIdx.y, r0 = blockIdx.x * kRowsT;
  const int T = checked_len(a, b);
  const int pages_b = (T + kPage - 1) / kPage;
  const int p_begin = split * a.chunk_pages;
  if (a.n_split > 1 && p_begin >= pages_b) return;  // empty split; the combine skips it
  const int t_begin = min(p_begin * kPage, T);
  const int t_end = min(T, (p_begin + a.chunk_pages) * kPage);

  for (int idx = tid; idx < kRowsT * (kDqk / 8); idx += kThreads) {
    const int r = idx / (kDqk / 8), c8 = idx % (kDqk / 8), row = r0 + r;
    float v[8];
    if (row < a.rows) {
      const size_t qrow = static_cast<size_t>(b) * a.rows + row;
      const uint4* s = (c8 < kDc / 8) ? reinterpret_cast<const uint4*>(a.q_c + qrow * kDc) + c8
                                      : reinterpret_cast<const uint4*>(a.q_r + qrow * kDr) + (c8 - kDc / 8);
      bf16x8_to_f32(__ldg(s), v);
    } else {
#pragma unroll
      for (int k = 0; k < 8; ++k) v[k] = 0.0f;
    }
#pragma unroll
    for (int k = 0; k < 8; ++k) sQ[r * kStride + c8 * 8 + k] = v[k];
  }

  float m_run[2] = {-CUDART_INF_F, -CUDART_INF_F}, l_run[2] = {0.0f, 0.0f};
  float acc[2][kRowsT];
#pragma unroll
  for (int k = 0; k < 2; ++k)
#pragma unroll
    for (int r = 0; r < kRowsT; ++r) acc[k][r] = 0.0f;
  const int my_r = tid >> 4, my_t = tid & 15;
  const int my_row = r0 + my_r;
  const int my_L = my_row < a.rows ? row_visible(T, a.s_q, a.H, my_row) : 0;
  __syncthreads();

  for (int t0 = t_begin; t0 < t_end; t0 += kTokT) {
    const int page = lookup_page(a.table, a.max_pages, a.num_pages, b, t0);
    if (page < 0 && tid == 0) record_error(a.status, MLA_ERR_INVALID_ARG);
    for (int idx = tid; idx < kTokT * (kDqk / 8); idx += kThreads) {
      const int tt = idx / (kDqk / 8), c8 = idx % (kDqk / 8);
      float v[8];
      if (page >= 0 && t0 + tt < t_end) {
        Src::load8(a, page, (t0 + tt) % kPage, c8 * 8, v);
      } else {
#pragma unroll
        for (int k = 0; k < 8; ++k) v[k] = 0.0f;
      }
#pragma unroll
      for (int k = 0; k < 8; ++k) sK[tt * kStride + c8 * 8 + k] = v[k];
    }
    __syncthreads();

    {  // scores, log2 domain
      const float* q = sQ + my_r * kStride;
      const float* k0 = sK + my_t * kStride;
      const float* k1 = sK + (my_t + 16) * kStride;
      float d0 = 0.0f, d1 = 0.0f;
#pragma unroll 8
      for (int c = 0; c < kDqk; ++c) {
        const float qv = q[c];
        d0 = fmaf(qv, k0[c], d0);
        d1 = fmaf(qv, k1[c], d1);
      }
      const bool ok = page >= 0;
      sP[my_r * kTokT + my_t] = (ok && t0 + my_t < my_L && t0 + my_t < t_end) ? d0 * a.scale_log2 : -CUDART_INF_F;
      sP[my_r * kTokT + my_t + 16] =
          (ok && t0 + my_t + 16 < my_L && t0 + my_t + 16 < t_end) ? d1 * a.scale_log2 : -CUDART_INF_F;
    }
    __syncthreads();

#pragma unroll
    for (int k = 0; k < 2; ++k) {  // online softmax; warp w owns rows 2w, 2w+1
      const int r = 2 * warp + k;
      const float v = sP[r * kTokT + lane];
      const float m_new = fmaxf(m_run[k], warp_max(v));
      float alpha = 1.0f, p = 0.0f;
      if (m_new != -CUDART_INF_F) {
        alpha = exp2f(m_run[k] - m_new);
        p = exp2f(v - m_new);
      }
      l_run[k] = l_run[k] * alpha + warp_sum(p);
      m_run[k] = m_new;
      sP[r * kTokT + lane] = p;
      if (lane == 0) sAlpha[r] = alpha;
    }
    __syncthreads();

#pragma unroll
    for (int kk = 0; kk < 2; ++kk) {
      const int j = tid + kk * kThreads;
#pragma unroll
      for (int r = 0; r < kRowsT; ++r) acc[kk][r] *= sAlpha[r];
      for (int tt = 0; tt < kTokT; ++tt) {
        const float kv = sK[tt * kStride + j];
#pragma unroll
        for (int r = 0; r < kRowsT; ++r) acc[kk][r] = fmaf(sP[r * kTokT + tt], kv, acc[kk][r]);
      }
    }
    __syncthreads();
  }

  if (lane == 0) {
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      sML[(2 * warp + k) * 2] = m_run[k];
      sML[(2 * warp + k) * 2 + 1] = l_run[k];
    }
  }
  __syncthreads();
#pragma unroll
  for (int r = 0; r < kRowsT; ++r) {
    const int row = r0 + r;
    if (row >= a.rows) break;
    const float m = sML[r * 2], l = sML[r * 2 + 1];
    const float inv = l > 0.0f ? 1.0f / l : 0.0f;
    const float lse = l > 0.0f ? (m + log2f(l)) * kLn2 : -CUDART_INF_F;
    const size_t qrow = static_cast<size_t>(b) * a.rows + row;
#pragma unroll
    for (int kk = 0; kk < 2; ++kk) {
      const int j = tid + kk * kThreads;
      const float o = acc[kk][r] * inv;
      if (a.n_split == 1) {
        if (a.out_f32)
          static_cast<float*>(a.out)[qrow * kDc + j] = o;
        else
          static_cast<__nv_bfloat16*>(a.out)[qrow * kDc + j] = __float2bfloat16_rn(o);
      } else {
        a.o_part[((static_cast<size_t>(b) * a.n_split + split) * a.rows + row) * kDc + j] = o;
      }
    }
    if (tid == 0) {
      if (a.n_split == 1) {
        if (a.lse) a.lse[qrow] = lse;
      } else {
        a.lse_part[(static_cast<size_t>(b) * a.n_split + split) * a.rows + row] = lse;
      }
    }
  }
}

// Split-KV merge: lse = log sum_j exp(lse_j), o = sum_j exp(lse_j - lse) o_j.
// Splits past the request's last page were never written and are not read;
// splits that saw no key carry lse_j = -inf and weight 0. Launched as a
// programmatic dependent of the decode kernel: it waits for that grid's
// results before its first read.
//
// A warp merges 512 / kParts channels of one output row: lane l holds the
// 16-byte pieces 32 q + l (q < 4 / kParts) of its part in every split. The
// loads of kGroup splits (their lse and their pieces) are issued together and
// merged online against a running maximum, so a row of up to kGroup splits
// costs one round trip to memory. kParts = 4 spreads a small batch over more
// warps and keeps sixteen splits in flight (one piece each); large batches
// take a whole row per warp (fewer, longer warps; four splits of four pieces).
constexpr int kCombineWarps = 8;
template <int kParts, int kGroup>
__global__ void __launch_bounds__(32 * kCombineWarps) combine_kernel(DecodeArgs a) {
  ptx::griddep_wait();
  ptx::griddep_launch_dependents();
  constexpr int kVec = 4 / kParts;  // 16-byte pieces per lane and split
  const int lane = threadIdx.x & 31;
  const long gw = static_cast<long>(blockIdx.x) * kCombineWarps + (threadIdx.x >> 5);
  if (gw >= static_cast<long>(a.B) * a.rows * kParts) return;
  const int part = static_cast<int>(gw % kParts);
  const long rw = gw / kParts;
  const int b = static_cast<int>(rw / a.rows), row = static_cast<int>(rw % a.rows);
  const int T = checked_len(a, b);
  const int pages_b = (T + kPage - 1) / kPage;
  const int n_b = min(a.n_split, (pages_b + a.chunk_pages - 1) / a.chunk_pages);
  const size_t base = static_cast<size_t>(b) * a.n_split;
  const float* lse_p = a.lse_part + base * a.rows + row;  // split j at [j * rows]
  const float4* o_p =
      reinterpret_cast<const float4*>(a.o_part + (base * a.rows + row) * kDc) + part * 32 * kVec + lane;
  const size_t o_stride = static_cast<size_t>(a.rows) * (kDc / 4);  // float4 per split
  float m = -CUDART_INF_F, tot = 0.0f;
  float4 acc[kVec];
#pragma unroll
  for (int q = 0; q < kVec; ++q) acc[q] = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int j = 0; j < n_b; j += kGroup) {
    float l[kGroup];
    float4 v[kGroup][kVec];
#pragma unroll
    for (int u = 0; u < kGroup; ++u) {
      const bool in = j + u < n_b;
      l[u] = in ? lse_p[static_cast<size_t>(j + u) * a.rows] : -CUDART_INF_F;
#pragma unroll
      for (int q = 0; q < kVec; ++q)
        v[u][q] = in ? o_p[static_cast<size_t>(j + u) * o_stride + 32 * q] : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    float mg = l[0];
#pragma unroll
    for (int u = 1; u < kGroup; ++u) mg = fmaxf(mg, l[u]);
    if (mg == -CUDART_INF_F) continue;  // no split of this group saw a key (same values in every lane)
    if (mg > m) {  // the running maximum moves: rescale what is merged so far
      const float f = (m == -CUDART_INF_F) ? 0.0f : exp2f((m - mg) * kLog2e);
      tot *= f;
#pragma unroll
      for (int q = 0; q < kVec; ++q) {
        acc[q].x *= f;
        acc[q].y *= f;
        acc[q].z *= f;
        acc[q].w *= f;
      }
      m = mg;
    }
#pragma unroll
    for (int u = 0; u < kGroup; ++u) {
      const float w = exp2f((l[u] - m) * kLog2e);  // lse -inf -> 0
      tot += w;
#pragma unroll
      for (int q = 0; q < kVec; ++q) {
        acc[q].x = fmaf(w, v[u][q].x, acc[q].x);
        acc[q].y = fmaf(w, v[u][q].y, acc[q].y);
        acc[q].z = fmaf(w, v[u][q].z, acc[q].z);
        acc[q].w = fmaf(w, v[u][q].w, acc[q].w);
      }
    }
  }
  const float inv = tot > 0.0f ? 1.0f / tot : 0.0f;
  const size_t qrow = static_cast<size_t>(b) * a.rows + row;
#pragma unroll
  for (int q = 0; q < kVec; ++q) {
    const int piece = part * 32 * kVec + 32 * q + lane;
    const float4 r = make_float4(acc[q].x * inv, acc[q].y * inv, acc[q].z * inv, acc[q].w * inv);
    if (a.out_f32) {
      reinterpret_cast<float4*>(static_cast<float*>(a.out) + qrow * kDc)[piece] = r;
    } else {
      const __nv_bfloat162 h0 = __floats2bfloat162_rn(r.x, r.y), h1 = __floats2bfloat162_rn(r.z, r.w);
      reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(a.out) + qrow * kDc)[piece] =
          make_uint2(*reinterpret_cast<const uint32_t*>(&h0), *reinterpret_cast<const uint32_t*>(&h1));
    }
  }
  if (part == 0 && lane == 0 && a.lse) a.lse[qrow] = tot > 0.0f ? m + logf(tot) : -CUDART_INF_F;
}

template <class Src>
cudaError_t launch_simt_t(const DecodeArgs& args, cudaStream_t stream) {
  const size_t smem = (kRowsT * kStride + kTokT * kStride + kRowsT * kTokT + kRowsT + 2 * kRowsT) * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(decode_simt_kernel<Src>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  dim3 grid((args.rows + kRowsT - 1) / kRowsT, args.n_split, args.B);
  return launch_dependent(decode_simt_kernel<Src>, grid, dim3(kThreads), smem, stream, args);
}

}  // namespace

DecodeArgs make_decode_args(const DecodeLaunch& L) {
  DecodeArgs a;
  a.pool = static_cast<const uint8_t*>(L.pool);
  a.table = L.table;
  a.seq_lens = L.seq_lens;
  a.q_c = static_cast<const __nv_bfloat16*>(L.q_c);
  a.q_r = static_cast<const __nv_bfloat16*>(L.q_r);
  a.out = L.out;
  a.lse = L.lse;
  a.o_part = L.o_part;
  a.lse_part = L.lse_part;
  a.status = L.status;
  a.max_pages = L.max_pages;
  a.num_pages = L.num_pages;
  a.max_seq_len = L.max_seq_len;
  a.B = L.B;
  a.s_q = L.s_q;
  a.H = L.H;
  a.rows = L.s_q * L.H;
  a.n_split = L.n_split;
  a.chunk_pages = L.chunk_pages;
  a.out_f32 = L.out_f32;
  a.scale_log2 = L.scale * kLog2e;
  a.c_new = static_cast<const __nv_bfloat16*>(L.c_new);
  a.kr_new = static_cast<const __nv_bfloat16*>(L.kr_new);
  a.n_new = L.n_new;
  a.flags = L.flags;
  a.worklist = L.worklist;
  return a;
}

cudaError_t launch_decode_simt(const DecodeLaunch& L) {
  const DecodeArgs a = make_decode_args(L);
  if (!L.quantized) return launch_simt_t<Bf16Source>(a, L.stream);
#define MLA_SIMT_CASE(BC, GC, BR, GR)                                               \
  if (L.bits_c == BC && L.group_c == GC && L.bits_r == BR && L.group_r == GR)     \
    return launch_simt_t<QuantSource<QGeom<BC, GC, BR, GR>>>(a, L.stream);
#define MLA_SIMT_R(BC, GC) \
  MLA_SIMT_CASE(BC, GC, 4, 64) MLA_SIMT_CASE(BC, GC, 4, 32) MLA_SIMT_CASE(BC, GC, 2, 64) MLA_SIMT_CASE(BC, GC, 2, 32)
  MLA_SIMT_R(4, 64)
  MLA_SIMT_R(4, 32)
  MLA_SIMT_R(2, 64)
  MLA_SIMT_R(2, 32)
#undef MLA_SIMT_R
#undef MLA_SIMT_CASE
  return cudaErrorInvalidValue;
}

cudaError_t launch_combine(const DecodeLaunch& L) {
  const DecodeArgs a = make_decode_args(L);
  const long rows = static_cast<long>(a.B) * a.rows;
  // fewer rows than 16 whole-row warps for each SM: split each row over four warps
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
      sms <= 0) {
    cudaGetLastError();
    sms = 148;
  }
  const bool quarter = rows < 16L * sms;
  const long blocks = (rows * (quarter ? 4 : 1) + kCombineWarps - 1) / kCombineWarps;
  if (blocks > 0x7FFFFFFFL) return cudaErrorInvalidValue;
  const dim3 grid(static_cast<unsigned>(blocks)), block(32 * kCombineWarps);
  return quarter ? launch_dependent(combine_kernel<4, 16>, grid, block, 0, L.stream, a)
                 : launch_dependent(combine_kernel<1, 4>, grid, block, 0, L.stream, a);
}

}  // namespace mla
