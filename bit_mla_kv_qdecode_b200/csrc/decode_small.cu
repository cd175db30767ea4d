// Decode for few query rows (s_q * H <= 16) on warp-level tensor-core MMAs
// (mma.sync m16n8k16). With 16 rows a 128-row tcgen05 tile would be 7/8
// padding, so this kernel keeps the rows at the MMA's native M = 16 and lets
// the tokens carry the N and K dimensions. Every cache format: INT4 or INT2
// codes, groups of 32 or 64 channels, for the content and the RoPE part.
//
// Absorbed MQA decode over the low-bit latent cache: scores
// (q_c . c_hat_t + q_r . kr_hat_t) * scale, softmax, output sum_t p_t c_hat_t
// (Group-Query Latent Attention abstract: one absorbed decoding path over the
// shared latent; QuantMLA abstract: dequantization inside the attention).
//
// Scores are exact in the codes. For a group with scale s and zero z,
// q . c_hat = s * (q . (u + 128)) + (z - 128 s) * sum(q): the MMA takes the
// integer codes as bf16 values u + 128 (exact, built by byte permutes), q is
// bf16, products are exact and accumulate in fp32; s and z are applied per
// (token, group) in fp32 afterwards, so every group has its own MMA chain. The
// output is exact in the codes as well: for a group, sum_t p_t c_hat_t =
// sum_t (p_t s_t) u_t + sum_t p_t z_t. The MMA takes the codes as the exact
// fp16 values u * 2^-24 (the subnormal whose bits are [u, 0x00]) and the
// weights w_t = p_t s_t as an fp16 hi + lo pair (22 significant bits, two
// MMAs); the epilogue scales by 2^24 and adds sum_t p_t z_t, accumulated in
// fp32 per (row, group). An output N-tile of 8 channels lies in one group, so
// one weight operand serves it.
//
// One CTA per (request, split): whole 64-token pages are bulk-copied into a
// 4-stage ring (issued by one thread, three pages ahead); eight warps split each page's tokens for
// the scores (8 keys each) and its channels for the output (64 channels each,
// the accumulators stay in registers). One named barrier per page hands the
// weights and per-warp maxima across; the running maximum is lazy (it moves
// only when a score exceeds it by more than 2^8), so the common page needs no
// rescale.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <math_constants.h>

#include "append_token.cuh"
#include "mla_common.cuh"
#include "mla_internal.h"
#include "sm100_ptx.cuh"

namespace mla {
namespace small {

constexpr int kWarps = 8;                    // compute warps
constexpr int kThreads = 32 * kWarps;
constexpr int kNS = 4;                       // page stages
constexpr int kRows = 16;                    // MMA M
constexpr int kKSteps = kDqk / 16;           // 36 score K-steps: the content groups', then the RoPE groups'
constexpr float kRescaleLog2 = 8.0f;
constexpr uint64_t kWaitLimitNs = 2000000000ull;
constexpr unsigned kFull = 0xffffffffu;
constexpr int kPRow = (kPage + 8) * 4;       // weight tile row stride (bytes): 64 fp32 + pad
constexpr int kPTile = kRows * kPRow;
constexpr int kORow = kDc + 4;               // epilogue output tile row stride (floats)
constexpr float kCodeScale = 16777216.0f;    // 2^24: the output MMA sees the codes as u * 2^-24

template <class G>
struct Layout {
  static constexpr int kGroups = G::kGroupsC + G::kGroupsR;   // scale groups of a token
  static constexpr int kStage = (G::kPageBytes + 127) / 128 * 128;
  static constexpr int kOffQ = kNS * kStage;                  // Q A-fragments [K-step][lane] x 16 B
  static constexpr int kOffQSum = kOffQ + kKSteps * 32 * 16;  // [group][row] float
  static constexpr int kOffP = kOffQSum + kGroups * kRows * 4;    // [2][16 rows][kPRow] fp32 weights
  static constexpr int kOffM = kOffP + 2 * kPTile;                // [2][16 rows][8 warps] float maxima
  static constexpr int kOffL = kOffM + 2 * kRows * kWarps * 4;    // [16 rows][8 warps] float row sums
  static constexpr int kOffBar = kOffL + kRows * kWarps * 4;      // full[kNS]
  static constexpr int kOffMisc = kOffBar + kNS * 8;              // abort flag, stage page ids
  static constexpr int kBytes = kOffMisc + 64;
  static_assert(kRows * kORow * 4 <= kNS * kStage, "epilogue tile reuses the page stages");
  static_assert(kOffQ % 16 == 0 && kOffP % 16 == 0 && kOffM % 16 == 0 && kOffBar % 8 == 0, "alignment");
};

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

// Byte j of a -> byte 0, byte j of b -> byte 2; bytes 1 and 3 replicate the
// sign bit of those bytes, which is 0 for the small code values used here.
__host__ __device__ constexpr uint32_t sel_pair(int j) {
  return static_cast<uint32_t>(j | ((8 | j) << 4) | ((4 + j) << 8) | ((12 + j) << 12));
}

// Four 16-bit operand pairs from two words a, b of one small code per byte
// (values 0..15): pair j = (a.byte j, b.byte j), each completed with the high
// byte hb (0x43: bf16 128 + u). Three byte permutes per two pairs: interleave
// first, then merge the constant.
__device__ __forceinline__ void byte_pairs(uint32_t a, uint32_t b, uint32_t hb4, uint32_t (&p)[4]) {
  const uint32_t m01 = prmt(a, b, 0x5140u), m23 = prmt(a, b, 0x7362u);  // [a0 b0 a1 b1], [a2 b2 a3 b3]
  p[0] = prmt(m01, hb4, 0x4140u);  // [a0, hb, b0, hb]
  p[1] = prmt(m01, hb4, 0x4342u);  // [a1, hb, b1, hb]
  p[2] = prmt(m23, hb4, 0x4140u);
  p[3] = prmt(m23, hb4, 0x4342u);
}

__device__ __forceinline__ void mma_bf16_frag(float (&d)[4], const uint4& a, uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a.x), "r"(a.y), "r"(a.z), "r"(a.w), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void mma_f16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void named_barrier_compute() {
  asm volatile("bar.sync 1, %0;" ::"n"(kWarps * 32) : "memory");
}

__device__ __forceinline__ uint32_t h2_bits(__half2 h) { return *reinterpret_cast<uint32_t*>(&h); }
__device__ __forceinline__ __half2 bits_h2(uint32_t u) { return *reinterpret_cast<__half2*>(&u); }

// fp16 hi + lo of two fp32 values (hi = RN(x), lo = RN(x - hi)).
__device__ __forceinline__ void split_h2(float x0, float x1, uint32_t& hi, uint32_t& lo) {
  const __half2 h = __floats2half2_rn(x0, x1);
  const float2 hf = __half22float2(h);
  hi = h2_bits(h);
  lo = h2_bits(__floats2half2_rn(x0 - hf.x, x1 - hf.y));
}

// Score B fragments of one group for this lane: the lane's GS/4 contiguous
// channels of its key (GS * BITS / 32 bytes at p), K-step s taking channels
// 4s + {0, 1} (b[s][0]) and 4s + {2, 3} (b[s][1]) as bf16 128 + u.
template <int BITS, int GS>
__device__ __forceinline__ void qk_codes(const uint8_t* p, uint32_t (&bf)[GS / 16][2]) {
  constexpr uint32_t kHB = 0x43434343u;
  if constexpr (BITS == 4) {
    // byte i holds channels 2i (low nibble) and 2i + 1: K-step s uses bytes 2s, 2s + 1
    uint32_t cw[GS / 32];
    if constexpr (GS == 64) {
      const uint2 v = *reinterpret_cast<const uint2*>(p);
      cw[0] = v.x;
      cw[1] = v.y;
    } else {
      cw[0] = *reinterpret_cast<const uint32_t*>(p);
    }
#pragma unroll
    for (int i = 0; i < GS / 32; ++i) {
      uint32_t q[4];
      byte_pairs(cw[i] & 0x0F0F0F0Fu, (cw[i] >> 4) & 0x0F0F0F0Fu, kHB, q);
      bf[2 * i][0] = q[0];
      bf[2 * i][1] = q[1];
      bf[2 * i + 1][0] = q[2];
      bf[2 * i + 1][1] = q[3];
    }
  } else {
    // byte s holds channels 4s .. 4s + 3 in bits 0-1, 2-3, 4-5, 6-7
    const uint32_t cw = GS == 64 ? *reinterpret_cast<const uint32_t*>(p)
                                 : static_cast<uint32_t>(*reinterpret_cast<const uint16_t*>(p));
    uint32_t p01[4], p23[4];
    byte_pairs(cw & 0x03030303u, (cw >> 2) & 0x03030303u, kHB, p01);
    byte_pairs((cw >> 4) & 0x03030303u, (cw >> 6) & 0x03030303u, kHB, p23);
#pragma unroll
    for (int st = 0; st < GS / 16; ++st) {
      bf[st][0] = p01[st];
      bf[st][1] = p23[st];
    }
  }
}

// Partial scores of one group: (s * D + (z - 128 s) * sum(q)) for this lane's
// accumulator entries (rows r, r + 8; keys tl0, tl0 + 1) added into sc.
// codes: the lane's bytes of key 8w + r; qf: the group's first Q fragment of
// this lane; meta: (s, z) of key tl0 (key tl0 + 1 at + meta_stride); qs: the
// group's q sums of row r (row r + 8 at + 8).
template <int BITS, int GS>
__device__ __forceinline__ void qk_group(const uint8_t* codes, const uint4* qf, const uint8_t* meta, int meta_stride,
                                         const float* qs, float (&sc)[4]) {
  uint32_t bq[GS / 16][2];
  qk_codes<BITS, GS>(codes, bq);
  float d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int ks = 0; ks < GS / 16; ++ks) mma_bf16_frag(d, qf[ks * 32], bq[ks][0], bq[ks][1]);
  const uint32_t m0 = *reinterpret_cast<const uint32_t*>(meta);
  const uint32_t m1 = *reinterpret_cast<const uint32_t*>(meta + meta_stride);
  const float2 sz0 = __half22float2(bits_h2(m0)), sz1 = __half22float2(bits_h2(m1));  // (s, z)
  const float e0 = fmaf(-128.0f, sz0.x, sz0.y), e1 = fmaf(-128.0f, sz1.x, sz1.y);
  const float qa = qs[0], qb = qs[8];
  sc[0] = fmaf(sz0.x, d[0], fmaf(e0, qa, sc[0]));
  sc[1] = fmaf(sz1.x, d[1], fmaf(e1, qa, sc[1]));
  sc[2] = fmaf(sz0.x, d[2], fmaf(e0, qb, sc[2]));
  sc[3] = fmaf(sz1.x, d[3], fmaf(e1, qb, sc[3]));
}

// Spread the eight 2-bit fields of x (bits 2j, 2j + 1) to nibbles (bits 4j, 4j + 1).
__device__ __forceinline__ uint32_t spread_crumbs(uint32_t x) {
  x = (x | (x << 8)) & 0x00FF00FFu;
  x = (x | (x << 4)) & 0x0F0F0F0Fu;
  return (x | (x << 2)) & 0x33333333u;
}

// Output codes of one key for lane column n of the warp's 64 channels (content
// codes of the key at p): nibble j is the code of output N-tile j's column n.
// Groups of 64: tile j column n is channel 8n + j; groups of 32: tiles 0-3
// take the first group (channel 4n + j), tiles 4-7 the second (4n + j - 4).
template <int BITS, int GS>
__device__ __forceinline__ uint32_t pv_codes(const uint8_t* p, int n) {
  if constexpr (BITS == 4 && GS == 64) {
    return *reinterpret_cast<const uint32_t*>(p + 4 * n);
  } else if constexpr (BITS == 4) {
    return static_cast<uint32_t>(*reinterpret_cast<const uint16_t*>(p + 2 * n)) |
           (static_cast<uint32_t>(*reinterpret_cast<const uint16_t*>(p + 16 + 2 * n)) << 16);
  } else if constexpr (GS == 64) {
    return spread_crumbs(*reinterpret_cast<const uint16_t*>(p + 2 * n));
  } else {
    return spread_crumbs(static_cast<uint32_t>(p[n]) | (static_cast<uint32_t>(p[8 + n]) << 8));
  }
}

// Channel (of the warp's 64) of output N-tile j, column n.
template <int GS>
__device__ __forceinline__ int pv_channel(int j, int n) {
  return GS == 64 ? 8 * n + j : 32 * (j >> 2) + 4 * n + (j & 3);
}

template <int BITS_C, int G_C, int BITS_R, int G_R>
__global__ void __launch_bounds__(kThreads, 2) decode_small_kernel(const DecodeArgs a) {
  using G = QGeom<BITS_C, G_C, BITS_R, G_R>;
  using Lo = Layout<G>;
  static_assert(Lo::kGroups * kRows <= 2 * kThreads, "q sums: at most two (group, row) entries per thread");
  // launched as a programmatic dependent: wait for the previous grid before any read
  ptx::griddep_wait();
  ptx::griddep_launch_dependents();
  extern __shared__ __align__(128) uint8_t smem[];
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + Lo::kOffBar);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Lo::kOffMisc);
  volatile int* stage_page = reinterpret_cast<volatile int*>(smem + Lo::kOffMisc + 16);  // [kNS]

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int b = blockIdx.x / a.n_split;
  const int split = blockIdx.x % a.n_split;
  const int T = checked_len(a, b);
  const int pages_b = (T + kPage - 1) / kPage;
  const int p_begin = split * a.chunk_pages;
  const int p_end = min(pages_b, p_begin + a.chunk_pages);
  const int n_pages = max(0, p_end - p_begin);
  const int t_end = min(T, p_end * kPage);  // keys this unit may see
  if (a.n_split > 1 && p_begin >= pages_b) return;  // split past the last page: never read by the merge

  if (tid == 0) {
    for (int s = 0; s < kNS; ++s) ptx::mbar_init(&full[s], 1);
    *abort_flag = 0;
    ptx::fence_mbar_init_cluster();
  }
  __syncthreads();

  // Fused append (mla_qdecode_fused_append): the step's n_new new tokens are
  // the last n_new of the T positions. The unit whose key range holds them
  // quantizes them into the pool (one warp per token, the append kernel's
  // writer) before it copies any page; the proxy fence and the barrier order
  // those writes before the bulk copies. Units of other key ranges never read
  // those bytes.
  if (a.n_new > 0) {
    if (T < a.n_new) {
      if (tid == 0) record_error(a.status, MLA_ERR_INVALID_ARG);
    } else {
      const int t_new = T - a.n_new;
      for (int t = max(t_new, p_begin * kPage) + warp; t < t_end; t += kWarps) {
        const int page = lookup_page(a.table, a.max_pages, a.num_pages, b, t);
        if (page < 0) {
          if (lane == 0) record_error(a.status, MLA_ERR_INVALID_ARG);
          continue;
        }
        const size_t src = static_cast<size_t>(b) * a.n_new + (t - t_new);
        quantize_token_warp<BITS_C, G_C, BITS_R, G_R>(
            const_cast<uint8_t*>(a.pool) + static_cast<size_t>(page) * G::kPageBytes, t % kPage,
            a.c_new + src * kDc, a.kr_new + src * kDr, lane);
      }
      ptx::fence_proxy_async_global();
    }
    __syncthreads();
  }

  // Page k of the unit goes to stage k % kNS. Thread 0 issues pages
  // 0 .. kNS-2 here and page k + kNS - 1 right after page k's named barrier,
  // when every warp is past the output MMAs of page k - 1, the last reader of
  // that stage. A missing page arrives without bytes; its keys are masked.
  int n_issued = 0;
  auto entry_of = [&](int k) { return k < n_pages ? table_entry(a.table, a.max_pages, b, (p_begin + k) * kPage) : -1; };
  auto issue_page = [&](int k, int page) {  // page: the block-table entry of unit page k
    if (k >= n_pages) return;
    const int s = k % kNS;
    if (page_valid(page, a.num_pages)) {
      stage_page[s] = page;
      ptx::mbar_arrive_expect_tx(&full[s], G::kPageBytes);
      ptx::bulk_load(smem + s * Lo::kStage, a.pool + static_cast<size_t>(page) * G::kPageBytes, G::kPageBytes,
                     &full[s]);
    } else {  // never dereferenced: the page's keys are masked and the call is flagged
      record_error(a.status, MLA_ERR_INVALID_ARG);
      stage_page[s] = -1;
      ptx::mbar_arrive(&full[s]);
    }
    n_issued = k + 1;
  };
  if (tid == 0)
    for (int k = 0; k < kNS - 1; ++k) issue_page(k, entry_of(k));

  {
    // =========================== compute warps ===========================
    const int w = warp;
    const int r = lane >> 2, kp = lane & 3;  // MMA fragment coordinates: row group, k pair
    const bool row_ok0 = r < a.rows, row_ok1 = r + 8 < a.rows;
    const int lim0 = row_ok0 ? min(row_visible(T, a.s_q, a.H, r), t_end) : 0;
    const int lim1 = row_ok1 ? min(row_visible(T, a.s_q, a.H, r + 8), t_end) : 0;

    // Q as A fragments, one 16-byte entry per (K-step, lane); the K-steps run
    // over the content groups, then the RoPE groups, GS/16 per group of GS
    // channels. Within a group, K-step s pairs logical columns {2kp, 2kp+1}
    // with channels (GS/4) kp + 4s + {0,1} and {8+2kp, 9+2kp} with
    // (GS/4) kp + 4s + {2,3}: the code bytes one lane needs for all of the
    // group's K-steps are then contiguous in the token's group.
    {
      const uint32_t* qc = reinterpret_cast<const uint32_t*>(a.q_c);
      const uint32_t* qr = reinterpret_cast<const uint32_t*>(a.q_r);
      uint4* qf = reinterpret_cast<uint4*>(smem + Lo::kOffQ);
      // Every load of the set-up is issued before the first use of any, so
      // the set-up costs one round trip to memory (it precedes the first page).
      constexpr int kEntries = kKSteps * 32;
      constexpr int kPerThread = (kEntries + kWarps * 32 - 1) / (kWarps * 32);
      constexpr int kStepsC = kDc / 16;  // content K-steps
      uint4 fv[kPerThread];
#pragma unroll
      for (int k = 0; k < kPerThread; ++k) {
        const int e = tid + k * kWarps * 32;
        fv[k] = make_uint4(0, 0, 0, 0);
        if (e < kEntries) {
          const int ks = e / 32, ln = e & 31;
          const int er = ln >> 2, ekp = ln & 3;
          const bool rope = ks >= kStepsC;
          const int gs = rope ? G_R : G_C, kr = rope ? ks - kStepsC : ks;
          const int g = kr / (gs / 16), st = kr % (gs / 16);
          const int c = g * gs + (gs / 4) * ekp + 4 * st;  // channel within q_c or q_r
          const bool ok0 = er < a.rows, ok1 = er + 8 < a.rows;
          const size_t q0 = static_cast<size_t>(b) * a.rows + er, q1 = q0 + 8;
          auto ld = [&](bool ok, size_t q, int cc) -> uint32_t {
            if (!ok) return 0u;
            return rope ? __ldg(qr + (q * kDr + cc) / 2) : __ldg(qc + (q * kDc + cc) / 2);
          };
          fv[k] = make_uint4(ld(ok0, q0, c), ld(ok1, q1, c), ld(ok0, q0, c + 2), ld(ok1, q1, c + 2));
        }
      }
      // per (group, row) sums of q, for the zero-point and code-offset term:
      // a group's channels as 16-byte loads, at most two entries per thread
      constexpr int kSumEntries = Lo::kGroups * kRows;
      constexpr int kSumPer = (kSumEntries + kThreads - 1) / kThreads;
      constexpr int kMaxV = (G_C > G_R ? G_C : G_R) / 8;
      uint4 qv[kSumPer][kMaxV];
#pragma unroll
      for (int i = 0; i < kSumPer; ++i) {
        const int e = tid + i * kThreads;
        const int eg = e / kRows, erow = e % kRows;
        const bool ok = e < kSumEntries && erow < a.rows;
        const bool rope = eg >= G::kGroupsC;
        const int nv = (rope ? G_R : G_C) / 8;
        const uint4* q = reinterpret_cast<const uint4*>(
            rope ? a.q_r + (static_cast<size_t>(b) * a.rows + erow) * kDr + G_R * (eg - G::kGroupsC)
                 : a.q_c + (static_cast<size_t>(b) * a.rows + erow) * kDc + G_C * eg);
#pragma unroll
        for (int v = 0; v < kMaxV; ++v) qv[i][v] = (ok && v < nv) ? __ldg(q + v) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int k = 0; k < kPerThread; ++k)
        if (tid + k * kWarps * 32 < kEntries) qf[tid + k * kWarps * 32] = fv[k];
#pragma unroll
      for (int i = 0; i < kSumPer; ++i) {
        const int e = tid + i * kThreads;
        if (e < kSumEntries) {
          float acc = 0.0f;
#pragma unroll
          for (int v = 0; v < kMaxV; ++v) {
            const uint32_t wv[4] = {qv[i][v].x, qv[i][v].y, qv[i][v].z, qv[i][v].w};
#pragma unroll
            for (int x = 0; x < 4; ++x) acc += bf16_lo(wv[x]) + bf16_hi(wv[x]);
          }
          reinterpret_cast<float*>(smem + Lo::kOffQSum)[e] = acc;  // [group][row]
        }
      }
      named_barrier_compute();
    }
    const uint4* qfrag = reinterpret_cast<const uint4*>(smem + Lo::kOffQ);
    const float* qsum = reinterpret_cast<const float*>(smem + Lo::kOffQSum);
    constexpr int kPvGroups = 64 / G_C;  // scale groups among a warp's 64 output channels
    float o[8][4];  // output accumulators of channels 64w .. 64w+63: N-tile j, fragment c (see the epilogue)
#pragma unroll
    for (int j = 0; j < 8; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.0f;
    float m_run[2] = {-CUDART_INF_F, -CUDART_INF_F};  // running maximum (log2 units) of rows r, r+8
    float l_acc[2] = {0.0f, 0.0f};                      // this thread's share of the row sums, scaled to m_run
    float corr[kPvGroups][2] = {};                      // this thread's share of sum p z per group, rows r, r+8
    const float sl2 = a.scale_log2;

    for (int k = 0; k < n_pages; ++k) {
      const int s = k % kNS, pb = k & 1;
      // the entry of the page issued after this page's barrier, loaded now so
      // that the issuing thread does not hold the next barrier up
      const int next_entry = tid == 0 ? entry_of(k + kNS - 1) : -1;
      // on a timeout the loop runs on (every warp keeps the same barrier
      // sequence) with the abort flag set, so later waits return at once
      if (!ptx::mbar_wait(&full[s], (k / kNS) & 1, abort_flag, kWaitLimitNs)) {
        record_error(a.status, MLA_ERR_TIMEOUT);
        *abort_flag = 1;
      }
      const uint8_t* st = smem + s * Lo::kStage;
      const bool page_ok = stage_page[s] >= 0;
      const int P0 = (p_begin + k) * kPage;  // first key of the page

      // ---- scores of this warp's 8 keys (one n-tile): lane (r, kp) feeds key 8w + r ----
      float sc[4] = {0.f, 0.f, 0.f, 0.f};
      const int tlb = 8 * w + r;       // key of this lane's B column
      const int tl0 = 8 * w + 2 * kp;  // keys of this lane's accumulator columns: tl0, tl0 + 1
#pragma unroll
      for (int g = 0; g < G::kGroupsC; ++g)
        qk_group<BITS_C, G_C>(st + G::kOffCC + tlb * G::kRowC + g * (G_C * BITS_C / 8) + kp * (G_C * BITS_C / 32),
                              qfrag + g * (G_C / 16) * 32 + lane, st + G::kOffCM + tl0 * G::kGroupsC * 4 + 4 * g,
                              G::kGroupsC * 4, qsum + g * kRows + r, sc);
#pragma unroll
      for (int g = 0; g < G::kGroupsR; ++g)
        qk_group<BITS_R, G_R>(st + G::kOffRC + tlb * G::kRowR + g * (G_R * BITS_R / 8) + kp * (G_R * BITS_R / 32),
                              qfrag + (kDc / 16 + g * (G_R / 16)) * 32 + lane,
                              st + G::kOffRM + tl0 * G::kGroupsR * 4 + 4 * g, G::kGroupsR * 4,
                              qsum + (G::kGroupsC + g) * kRows + r, sc);

      // ---- masks, this warp's maximum, weights ----
      float mloc[2] = {-CUDART_INF_F, -CUDART_INF_F};
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int lim = (c < 2) ? lim0 : lim1;
        const bool ok = page_ok && (P0 + tl0 + (c & 1)) < lim;
        sc[c] = ok ? sc[c] * sl2 : -CUDART_INF_F;
        mloc[c >> 1] = fmaxf(mloc[c >> 1], sc[c]);
      }
      float mw[2], l_own[2];
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        mloc[i] = fmaxf(mloc[i], __shfl_xor_sync(kFull, mloc[i], 1));
        mloc[i] = fmaxf(mloc[i], __shfl_xor_sync(kFull, mloc[i], 2));
        mw[i] = (mloc[i] > m_run[i] + kRescaleLog2) ? mloc[i] : m_run[i];
      }
      uint8_t* ptile = smem + Lo::kOffP + pb * kPTile;
      {
        const float meff0 = (mw[0] == -CUDART_INF_F) ? 0.0f : mw[0];
        const float meff1 = (mw[1] == -CUDART_INF_F) ? 0.0f : mw[1];
        const float2 p0 = make_float2(exp2f(sc[0] - meff0), exp2f(sc[1] - meff0));
        const float2 p1 = make_float2(exp2f(sc[2] - meff1), exp2f(sc[3] - meff1));
        l_own[0] = p0.x + p0.y;
        l_own[1] = p1.x + p1.y;
        *reinterpret_cast<float2*>(ptile + r * kPRow + tl0 * 4) = p0;
        *reinterpret_cast<float2*>(ptile + (r + 8) * kPRow + tl0 * 4) = p1;
      }
      float* mt = reinterpret_cast<float*>(smem + Lo::kOffM) + pb * kRows * kWarps;
      if (kp == 0) {
        mt[r * kWarps + w] = mw[0];
        mt[(r + 8) * kWarps + w] = mw[1];
      }
      named_barrier_compute();
      if (tid == 0) issue_page(k + kNS - 1, next_entry);

      // ---- new running maximum; rescale O and the row sums when it moved ----
      float mwr[2][kWarps];
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const float4 u = *reinterpret_cast<const float4*>(mt + (r + 8 * i) * kWarps);
        const float4 v = *reinterpret_cast<const float4*>(mt + (r + 8 * i) * kWarps + 4);
        mwr[i][0] = u.x; mwr[i][1] = u.y; mwr[i][2] = u.z; mwr[i][3] = u.w;
        mwr[i][4] = v.x; mwr[i][5] = v.y; mwr[i][6] = v.z; mwr[i][7] = v.w;
      }
      float mnew[2], alpha[2];
      bool uniform = true;  // every warp took its weights against the new maximum (the common case)
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        mnew[i] = m_run[i];
#pragma unroll
        for (int v = 0; v < kWarps; ++v) mnew[i] = fmaxf(mnew[i], mwr[i][v]);
#pragma unroll
        for (int v = 0; v < kWarps; ++v) uniform &= mwr[i][v] == mnew[i];
        alpha[i] = (mnew[i] == -CUDART_INF_F) ? 1.0f : exp2f(m_run[i] - mnew[i]);
        const float own = (mw[i] == -CUDART_INF_F) ? 0.0f : exp2f(mw[i] - mnew[i]);
        l_acc[i] = l_acc[i] * alpha[i] + l_own[i] * own;
#pragma unroll
        for (int pg = 0; pg < kPvGroups; ++pg) corr[pg][i] *= alpha[i];
        m_run[i] = mnew[i];
      }
      if (__any_sync(kFull, alpha[0] != 1.0f || alpha[1] != 1.0f)) {
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          o[j][0] *= alpha[0];
          o[j][1] *= alpha[0];
          o[j][2] *= alpha[1];
          o[j][3] *= alpha[1];
        }
      }
      const bool rescale_w = __any_sync(kFull, !uniform);

      // ---- O[16 rows, channels 64w .. 64w+63] += sum_t p_t c_hat_t over the page ----
      // Lane (r, kp) supplies column r of every N-tile (pv_codes and
      // pv_channel give the channels); an N-tile lies in one scale group. K-step
      // ks takes keys 16ks + [0, 16), scored by warps 2ks and 2ks+1; their
      // weights were taken against those warps' maxima and are scaled to the
      // new one.
#pragma unroll
      for (int ks = 0; ks < 4; ++ks) {
        const int ta = 16 * ks + 2 * kp, tb = ta + 8;  // page-local keys of B rows {0,1} and {8,9}
        // weights in A-fragment order: (r, ta..ta+1), (r+8, ta..), (r, tb..), (r+8, tb..)
        float2 pw[4] = {*reinterpret_cast<const float2*>(ptile + r * kPRow + ta * 4),
                        *reinterpret_cast<const float2*>(ptile + (r + 8) * kPRow + ta * 4),
                        *reinterpret_cast<const float2*>(ptile + r * kPRow + tb * 4),
                        *reinterpret_cast<const float2*>(ptile + (r + 8) * kPRow + tb * 4)};
        if (rescale_w) {  // some warp's maximum differs from the new one: scale its weights
          float fq[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const float mq = mwr[q & 1][2 * ks + (q >> 1)];
            fq[q] = (mq == -CUDART_INF_F) ? 0.0f : exp2f(mq - mnew[q & 1]);
          }
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            pw[q].x *= fq[q];
            pw[q].y *= fq[q];
          }
        }
        // (s, z) of the warp's groups for keys ta, ta+1, tb, tb+1; keys past
        // the end (or of a missing page) get s = z = 0, so garbage never
        // reaches the MMA
        float sv[kPvGroups][4], zv[kPvGroups][4];
        uint32_t wd[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int t = (q < 2 ? ta : tb) + (q & 1);
          const bool ok = page_ok && P0 + t < t_end;
#pragma unroll
          for (int pg = 0; pg < kPvGroups; ++pg) {
            const uint32_t m =
                ok ? *reinterpret_cast<const uint32_t*>(st + G::kOffCM + t * G::kGroupsC * 4 + 4 * (kPvGroups * w + pg))
                   : 0u;
            const float2 sz = __half22float2(bits_h2(m));
            sv[pg][q] = sz.x;
            zv[pg][q] = sz.y;
          }
          wd[q] = pv_codes<BITS_C, G_C>(st + G::kOffCC + t * G::kRowC + 8 * BITS_C * w, r);
        }
        // A = w = p * s as fp16 hi + lo; the zero-point term sum p z in fp32
        uint32_t ah[kPvGroups][4], al[kPvGroups][4];
#pragma unroll
        for (int pg = 0; pg < kPvGroups; ++pg) {
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int k0 = (q < 2) ? 0 : 2;  // keys (ta, ta+1) or (tb, tb+1)
            split_h2(pw[q].x * sv[pg][k0], pw[q].y * sv[pg][k0 + 1], ah[pg][q], al[pg][q]);
            corr[pg][q & 1] = fmaf(pw[q].x, zv[pg][k0], fmaf(pw[q].y, zv[pg][k0 + 1], corr[pg][q & 1]));
          }
        }
        // B: code nibble j of keys (ta, ta+1) and (tb, tb+1). The 16-bit
        // pattern [u, 0x00] is the fp16 value u * 2^-24 (subnormal, exact):
        // one byte permute per pair, no offset to cancel; the epilogue scales
        // by 2^24.
        const uint32_t la0 = wd[0] & 0x0F0F0F0Fu, ha0 = (wd[0] >> 4) & 0x0F0F0F0Fu;
        const uint32_t la1 = wd[1] & 0x0F0F0F0Fu, ha1 = (wd[1] >> 4) & 0x0F0F0F0Fu;
        const uint32_t lb0 = wd[2] & 0x0F0F0F0Fu, hb0 = (wd[2] >> 4) & 0x0F0F0F0Fu;
        const uint32_t lb1 = wd[3] & 0x0F0F0F0Fu, hb1 = (wd[3] >> 4) & 0x0F0F0F0Fu;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int pg = j / (8 / kPvGroups);
          const uint32_t sel = sel_pair(j >> 1);
          const uint32_t b0 = (j & 1) ? prmt(ha0, ha1, sel) : prmt(la0, la1, sel);
          const uint32_t b1 = (j & 1) ? prmt(hb0, hb1, sel) : prmt(lb0, lb1, sel);
          mma_f16(o[j], ah[pg], b0, b1);
          mma_f16(o[j], al[pg], b0, b1);
        }
      }
    }

    // ---- epilogue: row sums across lanes and warps, O / l, lse ----
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      l_acc[i] += __shfl_xor_sync(kFull, l_acc[i], 1);
      l_acc[i] += __shfl_xor_sync(kFull, l_acc[i], 2);
#pragma unroll
      for (int pg = 0; pg < kPvGroups; ++pg) {  // every lane of the row needs the group's full term
        corr[pg][i] += __shfl_xor_sync(kFull, corr[pg][i], 1);
        corr[pg][i] += __shfl_xor_sync(kFull, corr[pg][i], 2);
      }
    }
    float* lt = reinterpret_cast<float*>(smem + Lo::kOffL);
    if (kp == 0) {
      lt[r * kWarps + w] = l_acc[0];
      lt[(r + 8) * kWarps + w] = l_acc[1];
    }
    named_barrier_compute();  // also: every warp is done with the page stages
    float l[2], inv[2];
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const float4 u = *reinterpret_cast<const float4*>(lt + (r + 8 * i) * kWarps);
      const float4 v = *reinterpret_cast<const float4*>(lt + (r + 8 * i) * kWarps + 4);
      l[i] = ((u.x + u.y) + (u.z + u.w)) + ((v.x + v.y) + (v.z + v.w));
      inv[i] = l[i] > 0.0f ? 1.0f / l[i] : 0.0f;
    }
    float* otile = reinterpret_cast<float*>(smem);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int ch = 64 * w + pv_channel<G_C>(j, 2 * kp + e);
        const int pg = j / (8 / kPvGroups);
        otile[r * kORow + ch] = fmaf(o[j][e], kCodeScale, corr[pg][0]) * inv[0];
        otile[(r + 8) * kORow + ch] = fmaf(o[j][2 + e], kCodeScale, corr[pg][1]) * inv[1];
      }
    }
    const size_t part_row0 = (static_cast<size_t>(b) * a.n_split + split) * a.rows;
    if (w == 0 && kp == 0) {
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const int row = r + 8 * i;
        if (row >= a.rows) continue;
        const float lse = l[i] > 0.0f ? (m_run[i] + log2f(l[i])) * kLn2 : -CUDART_INF_F;
        if (a.n_split == 1) {
          if (a.lse) a.lse[static_cast<size_t>(b) * a.rows + row] = lse;
        } else {
          a.lse_part[part_row0 + row] = lse;
        }
      }
    }
    named_barrier_compute();
    {
      const int row = tid >> 4, seg = tid & 15;  // 16 rows x 16 segments of 32 channels
      if (row < a.rows) {
        const float* src = otile + row * kORow + seg * 32;
        if (a.n_split == 1 && !a.out_f32) {
          uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(a.out) +
                                                (static_cast<size_t>(b) * a.rows + row) * kDc + seg * 32);
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            uint32_t wds[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              __nv_bfloat162 h = __floats2bfloat162_rn(src[8 * v + 2 * e], src[8 * v + 2 * e + 1]);
              wds[e] = *reinterpret_cast<uint32_t*>(&h);
            }
            dst[v] = make_uint4(wds[0], wds[1], wds[2], wds[3]);
          }
        } else {
          float* base = (a.n_split == 1) ? static_cast<float*>(a.out) + (static_cast<size_t>(b) * a.rows + row) * kDc
                                         : a.o_part + (part_row0 + row) * kDc;
          float4* dst = reinterpret_cast<float4*>(base + seg * 32);
#pragma unroll
          for (int v = 0; v < 8; ++v) dst[v] = make_float4(src[4 * v], src[4 * v + 1], src[4 * v + 2], src[4 * v + 3]);
        }
      }
    }
  }

  // ---- teardown: after an abort, let every issued page copy land before the CTA exits ----
  __syncthreads();
  if (tid == 0 && *abort_flag) {
    for (int k = max(0, n_issued - kNS); k < n_issued; ++k)
      ptx::mbar_wait(&full[k % kNS], (k / kNS) & 1, nullptr, kWaitLimitNs);
  }
}

template <int BC, int GC, int BR, int GR>
cudaError_t launch_t(const DecodeLaunch& L) {
  using Lo = Layout<QGeom<BC, GC, BR, GR>>;
  auto kern = decode_small_kernel<BC, GC, BR, GR>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Lo::kBytes);
  if (e != cudaSuccess) return e;
  const DecodeArgs a = make_decode_args(L);
  return launch_dependent(kern, dim3(static_cast<unsigned>(L.B * L.n_split)), dim3(kThreads), Lo::kBytes, L.stream,
                          a);
}

}  // namespace small

bool decode_small_supported(const DecodeLaunch& L) {
  auto bits_ok = [](int bits) { return bits == 2 || bits == 4; };
  auto group_ok = [](int g) { return g == 32 || g == 64; };
  return L.quantized && L.s_q * L.H <= small::kRows && L.num_pages >= 1 && bits_ok(L.bits_c) && bits_ok(L.bits_r) &&
         group_ok(L.group_c) && group_ok(L.group_r);
}

cudaError_t launch_decode_small(const DecodeLaunch& L) {
  if (!L.quantized) return launch_decode_small_bf16(L);
  if (!decode_small_supported(L)) return cudaErrorNotSupported;
#define MLA_SMALL_CASE(BC, GC, BR, GR)                                            \
  if (L.bits_c == BC && L.group_c == GC && L.bits_r == BR && L.group_r == GR)   \
    return small::launch_t<BC, GC, BR, GR>(L);
#define MLA_SMALL_R(BC, GC) \
  MLA_SMALL_CASE(BC, GC, 4, 64) MLA_SMALL_CASE(BC, GC, 4, 32) MLA_SMALL_CASE(BC, GC, 2, 64) MLA_SMALL_CASE(BC, GC, 2, 32)
  MLA_SMALL_R(4, 64)
  MLA_SMALL_R(4, 32)
  MLA_SMALL_R(2, 64)
  MLA_SMALL_R(2, 32)
#undef MLA_SMALL_R
#undef MLA_SMALL_CASE
  return cudaErrorNotSupported;
}

}  // namespace mla
