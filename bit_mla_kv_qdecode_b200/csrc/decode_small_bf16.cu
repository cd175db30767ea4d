// Decode of the unquantized BF16 comparison cache for few query rows
// (s_q * H <= 16) on warp-level tensor-core MMAs (mma.sync m16n8k16).
//
// The same absorbed MQA decode as the quantized path (Group-Query Latent
// Attention abstract: one absorbed decoding path over the shared latent):
// scores (q_c . c_t + q_r . kr_t) * scale, softmax, output sum_t p_t c_t, over
// a cache of bf16 rows [pages][64][576] (the in-library BF16 decode the
// quantized one is compared with). At 16 query rows a 128-row tcgen05 tile is
// 7/8 padding; this kernel keeps the rows at the warp-level MMA's M = 16.
//
// Arithmetic. The cache values and the queries are exact bf16 operands, so a
// score needs one MMA term; the weights p are split into bf16 hi + lo (16
// significant bits) and the output takes two terms, P_hi.C + P_lo.C. All
// accumulation is fp32.
//
// One CTA per (request, key split), eight warps, two CTAs per SM (the phases
// of a stage are short and separated by barriers: the other CTA fills the
// gaps), a ring of two stages of 32 tokens (half a page) per CTA. Warp 4
// copies the next stage's rows as soon as the current stage's scores are in,
// with one bulk copy per token into rows padded to 1,168 bytes, so the eight 16-byte row pieces one
// ldmatrix phase reads fall in distinct banks. Per stage: warp w scores key
// tile w & 3 (8 keys) over channel half w >> 2 (18 K-steps); warps 4-7 hand
// their partial sums to warps 0-3 through shared memory, which finish the
// scores, publish per-tile row maxima and, after a barrier, write the
// weights as MMA A fragments; then every warp accumulates the output for its
// 64 channels (8 N-tiles, two 16-key K-steps, two terms). The running maximum
// is lazy: it moves only when a tile's maximum exceeds it by more than 2^8.
#include <cuda_bf16.h>
#include <math_constants.h>

#include "mla_common.cuh"
#include "mla_internal.h"
#include "sm100_ptx.cuh"

namespace mla {
namespace small_bf16 {

constexpr int kWarps = 8;
constexpr int kThreads = 32 * kWarps;
constexpr int kRows = 16;                    // MMA M
constexpr int kTok = 32;                     // tokens per stage (half a page)
constexpr int kNS = 2;                       // stages (two CTAs per SM: four stages in flight per SM)
constexpr int kIssueWarp = 4;                // a warp that idles between the score and maximum barriers
constexpr int kRowBytes = kDqk * 2;          // one token's 576 bf16
constexpr int kRowStride = kRowBytes + 16;   // 1,168: 292 words, 4 (mod 32) banks apart
constexpr int kStage = kTok * kRowStride;
constexpr int kKSteps = kDqk / 16;           // 36
constexpr int kHalfK = kKSteps / 2;          // 18 K-steps per scoring warp
constexpr float kRescaleLog2 = 8.0f;
constexpr uint64_t kWaitLimitNs = 2000000000ull;
constexpr unsigned kFull = 0xffffffffu;

constexpr int kOffQ = kNS * kStage;                   // Q as A fragments: [36 K-steps][32 lanes] x 16 B
constexpr int kOffP = kOffQ + kKSteps * 32 * 16;      // weights as A fragments: [2 K-steps][hi, lo][32 lanes] x 16 B
constexpr int kOffS = kOffP + 2 * 2 * 32 * 16;        // second-half score partials: [4 key tiles][32 lanes] x 16 B
constexpr int kOffM = kOffS + 4 * 32 * 16;            // key-tile row maxima: [16 rows][4 tiles]
constexpr int kOffL = kOffM + kRows * 4 * 4;          // row sums: [16 rows][4 tiles]
constexpr int kOffBar = kOffL + kRows * 4 * 4;        // full[kNS]
constexpr int kOffMisc = kOffBar + kNS * 8;           // abort flag, stage pages
constexpr int kBytes = kOffMisc + 64;
constexpr int kORow = kDc + 4;                        // epilogue output tile row stride (floats)
static_assert(kRows * kORow * 4 <= kNS * kStage, "epilogue tile reuses the stages");
static_assert(kOffQ % 128 == 0 && kOffBar % 8 == 0, "alignment");
static_assert(kRowStride % 16 == 0 && (kRowStride / 4) % 32 == 4, "padded rows: 16-byte aligned, 4 banks apart");

__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint4& a, uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a.x), "r"(a.y), "r"(a.z), "r"(a.w), "r"(b0), "r"(b1));
}

// Four 8x8 b16 matrices; lane l gives the address of row l % 8 of matrix l / 8.
__device__ __forceinline__ void ldsm_x4(uint32_t (&d)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3])
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_trans(uint32_t (&d)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3])
               : "r"(addr));
}

__device__ __forceinline__ void named_barrier() { asm volatile("bar.sync 1, %0;" ::"n"(kThreads) : "memory"); }

__device__ __forceinline__ float ex2_approx(float x) {  // 2^x; -inf -> +0
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// bf16 hi + lo of two fp32 values, packed (lower value in the low half).
__device__ __forceinline__ void split2(float x0, float x1, uint32_t& hi, uint32_t& lo) {
  __nv_bfloat162 h = __floats2bfloat162_rn(x0, x1);
  hi = *reinterpret_cast<uint32_t*>(&h);
  __nv_bfloat162 l = __floats2bfloat162_rn(x0 - bf16_lo(hi), x1 - bf16_hi(hi));
  lo = *reinterpret_cast<uint32_t*>(&l);
}

__global__ void __launch_bounds__(kThreads, 2) decode_small_bf16_kernel(const DecodeArgs a) {
  // launched as a programmatic dependent: wait for the previous grid before any read
  ptx::griddep_wait();
  ptx::griddep_launch_dependents();
  extern __shared__ __align__(128) uint8_t smem[];
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kOffBar);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffMisc);
  volatile int* stage_page = reinterpret_cast<volatile int*>(smem + kOffMisc + 16);  // [kNS]

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int b = blockIdx.x / a.n_split;
  const int split = blockIdx.x % a.n_split;
  const int T = checked_len(a, b);
  const int pages_b = (T + kPage - 1) / kPage;
  const int p_begin = split * a.chunk_pages;
  if (a.n_split > 1 && p_begin >= pages_b) return;  // split past the last page: never read by the merge
  const int p_end = min(pages_b, p_begin + a.chunk_pages);
  const int t_begin = p_begin * kPage;
  const int t_end = min(T, p_end * kPage);  // keys this unit may see
  const int n_st = t_end > t_begin ? (t_end - t_begin + kTok - 1) / kTok : 0;

  if (tid == 0) {
    for (int s = 0; s < kNS; ++s) ptx::mbar_init(&full[s], 1);
    *abort_flag = 0;
    ptx::fence_mbar_init_cluster();
  }
  __syncthreads();

  // Stage k holds tokens t_begin + 32k .. +31, half (k & 1) of one page. The
  // issuing warp copies it: one bulk copy per token into its padded row; rows past the
  // unit's keys, or of a page the table could not name, are zeroed (their
  // weights are 0, and 0 times stale bytes must not meet a NaN). The zeroing
  // stores come before the arrive that opens the stage's phase.
  int n_issued = 0;
  auto page_of = [&](int k) {
    return k < n_st ? lookup_page(a.table, a.max_pages, a.num_pages, b, t_begin + k * kTok) : -1;
  };
  auto issue_stage = [&](int k, int page) {  // the issuing warp, all lanes; page: lookup_page of stage k
    if (k >= n_st) return;
    const int s = k % kNS;
    const int t0 = t_begin + k * kTok;
    const int n_valid = page >= 0 ? min(kTok, t_end - t0) : 0;
    uint8_t* row = smem + s * kStage + lane * kRowStride;
    if (lane >= n_valid) {
#pragma unroll 4
      for (int c = 0; c < kRowBytes / 16; ++c) *reinterpret_cast<uint4*>(row + 16 * c) = make_uint4(0, 0, 0, 0);
    }
    __syncwarp();
    if (lane == 0) {
      stage_page[s] = page;
      if (page < 0) {  // never dereferenced: the stage's keys are masked and the call is flagged
        record_error(a.status, MLA_ERR_INVALID_ARG);
        ptx::mbar_arrive(&full[s]);
      } else {
        ptx::mbar_arrive_expect_tx(&full[s], n_valid * kRowBytes);
      }
    }
    __syncwarp();
    if (lane < n_valid)
      ptx::bulk_load(row,
                     a.pool + (static_cast<size_t>(page) * kPage + (t0 % kPage) + lane) * kRowBytes,
                     kRowBytes, &full[s]);
    n_issued = k + 1;
  };
  if (warp == kIssueWarp)  // every slot is free at the start
    for (int k = 0; k < kNS; ++k) issue_stage(k, page_of(k));

  const int r = lane >> 2, kp = lane & 3;  // MMA fragment coordinates: row group, k pair
  const bool row_ok0 = r < a.rows, row_ok1 = r + 8 < a.rows;
  const int lim0 = row_ok0 ? min(row_visible(T, a.s_q, a.H, r), t_end) : 0;
  const int lim1 = row_ok1 ? min(row_visible(T, a.s_q, a.H, r + 8), t_end) : 0;

  // Q as A fragments: K-step ks covers channels 16ks .. 16ks+15 of the
  // concatenated [q_c | q_r]; lane (r, kp) holds rows r and r+8, channels
  // 16ks + 2kp + {0, 1} and 16ks + 8 + 2kp + {0, 1}. All loads first.
  {
    constexpr int kEntries = kKSteps * 32;
    constexpr int kPerThread = kEntries / kThreads;  // 4.5 -> 5
    uint4 fv[kPerThread + 1];
#pragma unroll
    for (int k = 0; k <= kPerThread; ++k) {
      const int e = tid + k * kThreads;
      fv[k] = make_uint4(0, 0, 0, 0);
      if (e < kEntries) {
        const int ks = e >> 5, ln = e & 31;
        const int er = ln >> 2, ekp = ln & 3;
        auto ld = [&](int row, int ch) -> uint32_t {
          if (row >= a.rows) return 0u;
          const size_t q = static_cast<size_t>(b) * a.rows + row;
          return ch < kDc ? __ldg(reinterpret_cast<const uint32_t*>(a.q_c + q * kDc + ch))
                          : __ldg(reinterpret_cast<const uint32_t*>(a.q_r + q * kDr + (ch - kDc)));
        };
        const int c0 = 16 * ks + 2 * ekp;
        fv[k] = make_uint4(ld(er, c0), ld(er + 8, c0), ld(er, c0 + 8), ld(er + 8, c0 + 8));
      }
    }
    uint4* qf = reinterpret_cast<uint4*>(smem + kOffQ);
#pragma unroll
    for (int k = 0; k <= kPerThread; ++k)
      if (tid + k * kThreads < kEntries) qf[tid + k * kThreads] = fv[k];
  }
  __syncthreads();

  const uint4* qfrag = reinterpret_cast<const uint4*>(smem + kOffQ);
  uint4* pfrag = reinterpret_cast<uint4*>(smem + kOffP);
  float4* spart = reinterpret_cast<float4*>(smem + kOffS);
  float* mtile = reinterpret_cast<float*>(smem + kOffM);
  const int nt = warp & 3, kh = warp >> 2;  // scoring: key tile, channel half
  float o[8][4];  // output accumulators: N-tile j = channels 64 warp + 8j .. +7
#pragma unroll
  for (int j = 0; j < 8; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.0f;
  float m_run[2] = {-CUDART_INF_F, -CUDART_INF_F};  // running maximum (log2 units) of rows r, r+8
  float l_acc[2] = {0.0f, 0.0f};                      // scoring warps: this lane's share of the row sums
  const float sl2 = a.scale_log2;

  for (int k = 0; k < n_st; ++k) {
    const int s = k % kNS;
    // the page of the stage issued after this stage's scores, loaded now so
    // that the issuing warp does not hold the next barrier up
    const int next_page = (warp == kIssueWarp && k > 0) ? page_of(k + kNS - 1) : -1;
    // on a timeout the loop runs on (every warp keeps the same barrier
    // sequence) with the abort flag set, so later waits return at once
    if (!ptx::mbar_wait(&full[s], (k / kNS) & 1, abort_flag, kWaitLimitNs)) {
      record_error(a.status, MLA_ERR_TIMEOUT);
      *abort_flag = 1;
    }
    const uint32_t st = ptx::smem_u32(smem + s * kStage);
    const bool page_ok = stage_page[s] >= 0;
    const int t0 = t_begin + k * kTok;

    // ---- scores of key tile nt over channel half kh ----
    float d[4] = {0.f, 0.f, 0.f, 0.f};
    {
      // ldmatrix rows: keys 8nt + (lane & 7); matrices (K-step, channels
      // 0-7), (K-step, 8-15), (next K-step, 0-7), (next K-step, 8-15).
      // Even and odd K-steps accumulate separately: two chains of 9 MMAs
      // instead of one of 18.
      const uint32_t rowaddr = st + (8 * nt + (lane & 7)) * kRowStride + ((lane >> 3) & 1) * 16 + (lane >> 4) * 32;
      float d1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int kk = 0; kk < kHalfK; kk += 2) {
        const int ks = kh * kHalfK + kk;
        uint32_t bq[4];
        ldsm_x4(bq, rowaddr + ks * 32);
        mma_bf16(d, qfrag[ks * 32 + lane], bq[0], bq[1]);
        mma_bf16(d1, qfrag[(ks + 1) * 32 + lane], bq[2], bq[3]);
      }
#pragma unroll
      for (int c = 0; c < 4; ++c) d[c] += d1[c];
    }
    if (kh == 1) spart[nt * 32 + lane] = make_float4(d[0], d[1], d[2], d[3]);
    named_barrier();
    // every warp is past the output MMAs of stage k-1, the last reader of the
    // ring slot of stage k + kNS - 1 (issued at the start for k = 0); the
    // issuing warp has nothing to do until the next barrier
    if (warp == kIssueWarp && k > 0) issue_stage(k + kNS - 1, next_page);
    if (kh == 0) {
      const float4 p2 = spart[nt * 32 + lane];
      d[0] += p2.x; d[1] += p2.y; d[2] += p2.z; d[3] += p2.w;
      // keys 8nt + 2kp + {0, 1} of the stage, rows r (d0, d1) and r + 8 (d2, d3)
      const int tk = t0 + 8 * nt + 2 * kp;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const bool ok = page_ok && tk + (c & 1) < (c < 2 ? lim0 : lim1);
        d[c] = ok ? d[c] * sl2 : -CUDART_INF_F;
      }
      float m0 = fmaxf(d[0], d[1]), m1 = fmaxf(d[2], d[3]);
      m0 = fmaxf(m0, __shfl_xor_sync(kFull, m0, 1));
      m0 = fmaxf(m0, __shfl_xor_sync(kFull, m0, 2));
      m1 = fmaxf(m1, __shfl_xor_sync(kFull, m1, 1));
      m1 = fmaxf(m1, __shfl_xor_sync(kFull, m1, 2));
      if (kp == 0) {
        mtile[r * 4 + nt] = m0;
        mtile[(r + 8) * 4 + nt] = m1;
      }
    }
    named_barrier();

    // ---- running maximum (every warp takes the same decision per row) ----
    float alpha[2];
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const float4 mt = *reinterpret_cast<const float4*>(mtile + (r + 8 * i) * 4);
      const float mx = fmaxf(fmaxf(mt.x, mt.y), fmaxf(mt.z, mt.w));
      alpha[i] = 1.0f;
      if (mx > -CUDART_INF_F) {
        if (m_run[i] == -CUDART_INF_F) {
          m_run[i] = mx;
        } else if (mx > m_run[i] + kRescaleLog2) {
          alpha[i] = ex2_approx(m_run[i] - mx);
          m_run[i] = mx;
        }
      }
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
    // ---- weights of the scoring warps, as A fragments of the output MMAs ----
    if (kh == 0) {
      const float me0 = m_run[0] == -CUDART_INF_F ? 0.0f : m_run[0];
      const float me1 = m_run[1] == -CUDART_INF_F ? 0.0f : m_run[1];
      const float p0 = ex2_approx(d[0] - me0), p1 = ex2_approx(d[1] - me0);
      const float p2 = ex2_approx(d[2] - me1), p3 = ex2_approx(d[3] - me1);
      l_acc[0] = l_acc[0] * alpha[0] + (p0 + p1);
      l_acc[1] = l_acc[1] * alpha[1] + (p2 + p3);
      uint32_t h01, l01, h23, l23;
      split2(p0, p1, h01, l01);
      split2(p2, p3, h23, l23);
      // K-step nt >> 1 holds key tiles 2(nt >> 1) and 2(nt >> 1) + 1: an even
      // tile fills A words 0 (row r) and 1 (row r+8), an odd tile words 2, 3
      uint32_t* ph = reinterpret_cast<uint32_t*>(pfrag + ((nt >> 1) * 2 + 0) * 32 + lane);
      uint32_t* pl = reinterpret_cast<uint32_t*>(pfrag + ((nt >> 1) * 2 + 1) * 32 + lane);
      ph[2 * (nt & 1)] = h01;
      ph[2 * (nt & 1) + 1] = h23;
      pl[2 * (nt & 1)] = l01;
      pl[2 * (nt & 1) + 1] = l23;
    } else {
      l_acc[0] *= alpha[0];
      l_acc[1] *= alpha[1];
    }
    named_barrier();

    // ---- output: O[16 rows, channels 64 warp .. +63] += P_hi.C + P_lo.C ----
    {
      // ldmatrix.trans rows: keys 16 K-step + (lane & 7) + 8 ((lane >> 3) & 1);
      // matrices (keys 0-7, channels c0..c0+7), (keys 8-15, c0..), (0-7, c0+8..), (8-15, c0+8..)
      const uint32_t rowaddr =
          st + ((lane & 7) + 8 * ((lane >> 3) & 1)) * kRowStride + (64 * warp + 8 * (lane >> 4)) * 2;
#pragma unroll
      for (int kk = 0; kk < 2; ++kk) {
        const uint4 ah = pfrag[(kk * 2 + 0) * 32 + lane];
        const uint4 al = pfrag[(kk * 2 + 1) * 32 + lane];
#pragma unroll
        for (int np = 0; np < 4; ++np) {
          uint32_t bc[4];
          ldsm_x4_trans(bc, rowaddr + kk * 16 * kRowStride + np * 32);
          mma_bf16(o[2 * np], ah, bc[0], bc[1]);
          mma_bf16(o[2 * np], al, bc[0], bc[1]);
          mma_bf16(o[2 * np + 1], ah, bc[2], bc[3]);
          mma_bf16(o[2 * np + 1], al, bc[2], bc[3]);
        }
      }
    }
  }

  // ---- epilogue: row sums across lanes and scoring warps, O / l, lse ----
  float* lt = reinterpret_cast<float*>(smem + kOffL);
  if (kh == 0) {
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      l_acc[i] += __shfl_xor_sync(kFull, l_acc[i], 1);
      l_acc[i] += __shfl_xor_sync(kFull, l_acc[i], 2);
    }
    if (kp == 0) {
      lt[r * 4 + nt] = l_acc[0];
      lt[(r + 8) * 4 + nt] = l_acc[1];
    }
  }
  __syncthreads();  // also: every warp is done with the stages
  float l[2], inv[2];
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const float4 u = *reinterpret_cast<const float4*>(lt + (r + 8 * i) * 4);
    l[i] = (u.x + u.y) + (u.z + u.w);
    inv[i] = l[i] > 0.0f ? 1.0f / l[i] : 0.0f;
  }
  float* otile = reinterpret_cast<float*>(smem);
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int ch = 64 * warp + 8 * j + 2 * kp;
    otile[r * kORow + ch] = o[j][0] * inv[0];
    otile[r * kORow + ch + 1] = o[j][1] * inv[0];
    otile[(r + 8) * kORow + ch] = o[j][2] * inv[1];
    otile[(r + 8) * kORow + ch + 1] = o[j][3] * inv[1];
  }
  const size_t part_row0 = (static_cast<size_t>(b) * a.n_split + split) * a.rows;
  if (warp == 0 && kp == 0) {
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
  __syncthreads();
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

  // ---- teardown: after an abort, let every issued stage copy land before the CTA exits ----
  __syncthreads();
  if (warp == kIssueWarp && lane == 0 && *abort_flag) {
    for (int k = max(0, n_issued - kNS); k < n_issued; ++k)
      ptx::mbar_wait(&full[k % kNS], (k / kNS) & 1, nullptr, kWaitLimitNs);
  }
}

}  // namespace small_bf16

bool decode_small_bf16_supported(const DecodeLaunch& L) {
  return !L.quantized && L.s_q * L.H <= small_bf16::kRows && L.num_pages >= 1;
}

cudaError_t launch_decode_small_bf16(const DecodeLaunch& L) {
  if (!decode_small_bf16_supported(L)) return cudaErrorNotSupported;
  auto kern = small_bf16::decode_small_bf16_kernel;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, small_bf16::kBytes);
  if (e != cudaSuccess) return e;
  const DecodeArgs a = make_decode_args(L);
  return launch_dependent(kern, dim3(static_cast<unsigned>(L.B * L.n_split)), dim3(small_bf16::kThreads),
                          small_bf16::kBytes, L.stream, a);
}

}  // namespace mla
