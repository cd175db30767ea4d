// Tensor-core decode for sm_100a: tcgen05 MMAs with TMEM accumulators over a
// TMA-staged, low-bit quantized latent cache.
//
// Computation (absorbed MQA form of MLA decode, Group-Query Latent Attention
// abstract, thelatestinai.com/papers/2607.27269; unpack + dequant inside the
// attention, QuantMLA abstract, arxivdaily.com/papers/2609.36760):
//   S[r,t] = (q_c[r] . c_hat[t] + q_r[r] . kr_hat[t]) * scale
//   O[r,:] = sum_t softmax_t(S[r,:]) c_hat[t]
// for 128 query rows r (heads x queries of one request) at a time.
//
// Work unit and cluster split. A unit is (request, key split, 128-row tile).
// It runs on a cluster of two CTAs; CTA k owns latent channels
// [256k, 256k+256) and RoPE channels [32k, 32k+32). Each CTA dequantizes only
// its half of every token, computes a partial score over its 288 channels,
// and the two partial scores are exchanged through distributed shared memory
// and added (fp32 addition commutes, so both CTAs hold bit-identical scores
// and take identical softmax decisions). Each CTA then accumulates its own
// 256-wide half of the output: O_half = 128 x 256 fp32 fits TMEM beside the
// score buffers and the query operand.
//
// Precision. The dequantized values u*s+z are split into bf16 hi + bf16 lo
// (both rounded to nearest; 16 significant bits together), and so are the
// softmax weights. Rounding, not truncating, the hi part keeps the dropped
// P_lo*C_lo term zero-mean; with truncated hi parts it is biased and the
// output error grew with the sequence length (measured). Scores use
// Q*C_hi + Q*C_lo (Q is exact in bf16); the output uses P_hi*C_hi + P_lo*C_hi
// + P_hi*C_lo. All accumulation is fp32 in TMEM. This keeps the output within
// 2e-3 of its RMS of the exact float64 result; single bf16 operands would not.
//
// Pipeline. A chunk's operand tile (C_hi, C_lo of this CTA's 288 channels,
// 36 KB) is held from its dequantization until its PV MMAs finish; four
// operand stages, two code stages and one weight tile (rewritten only after
// the previous chunk's PV) fit the shared memory. The softmax step of chunk
// j reads the peer's partial scores of chunk j-1, sends this CTA's partial of
// chunk j, and only then finishes chunk j-1: the copy to the peer is in
// flight during that work (measured 7-12 % faster than finishing chunk j-1
// first, once the fourth operand stage relieved the stage ring).
// Warp roles (512 threads):
//   warp 0      TMA producer: packed codes + metadata of 32-token chunks
//   warp 1      TMEM owner; issues the QK MMAs of even chunks
//   warp 6      issues the PV MMAs
//   warp 7      issues the QK MMAs of odd chunks
//   warps 2-5   unpack + dequantize into bf16 hi/lo operand tiles
//   warps 8-15  two threads per row (warps w and w+4 share a TMEM lane
//               quarter, 16 of each chunk's 32 columns each): score exchange,
//               online softmax, P tiles, output rescaling in TMEM, epilogue
//               (rows staged in shared memory and written by bulk copies)
// Fused append (mla_qdecode_fused_append): before the cluster barrier of the
// set-up, CTA 0's softmax warps quantize the step's new tokens that fall in
// the unit's key range into the pool; the barrier and proxy fences order
// those writes before both CTAs' TMA reads.
// The host caps a unit at 8,192 keys: the fp32 accumulation in TMEM loses
// accuracy in proportion to the keys one accumulator sums.
// Every wait is bounded; a timeout sets MLA_ERR_TIMEOUT and the unit drains
// and exits without touching memory it does not own. The kernel is launched
// as a programmatic dependent and waits (griddepcontrol.wait) before any read.
#include <cuda.h>
#include <math_constants.h>

#include <mutex>

#include "append_token.cuh"
#include "mla_common.cuh"
#include "mla_internal.h"
#include "sm100_ptx.cuh"

namespace mla {
namespace tc {

constexpr int kThreads = 512;
constexpr int kSoftThreads = 256;  // warps 8-15
constexpr int kChunk = 32;            // tokens per pipeline step
constexpr int kRows = 128;            // query rows per unit (MMA M)
constexpr int kHalfC = 256;           // content channels per CTA
constexpr int kHalfR = 32;            // rope channels per CTA
constexpr int kKChunks = (kHalfC + kHalfR) / 8;  // 36 eight-channel chunks per token
constexpr int kNC = 4;                // operand-tile stages
constexpr int kNS = 2;                // TMA code stages
constexpr int kBarCode = kNC > kNS ? kNC : kNS;  // code_full entries (the BF16 cache uses one per operand stage)
static_assert(kChunk == 32, "the PV issue sequence covers two 16-token K-steps");
constexpr float kRescaleLog2 = 8.0f;  // lazy rescale threshold (weights stay <= 2^8)
constexpr uint64_t kWaitLimitNs = 2000000000ull;
constexpr unsigned kFull = 0xffffffffu;

// TMEM columns
constexpr uint32_t kTmemO = 0;        // 256 fp32 columns: this CTA's half of O
constexpr uint32_t kTmemS = 256;      // two 64-column score buffers: [S_hi | S_lo] of 32 tokens
constexpr uint32_t kTmemQ = 384;      // 128 columns: content part of Q (256 bf16 per row)
constexpr uint32_t kTmemCols = 512;

// Shared memory layout (bytes)
// Operand stage: per 8-channel chunk c, the hi and lo core matrices of the 32
// tokens sit side by side ([c][hi/lo][token group][8 rows x 16 B]), so one
// K-major QK operand of N = 64 rows covers C_hi and C_lo of the same tokens.
constexpr int kCChunkStride = 1024;
constexpr int kCLoOff = 512;
constexpr int kCStage = kKChunks * kCChunkStride;
constexpr int kBfChunkStride = 512;  // bf16 cache: C only, [chunk][token group][8 rows x 16 B]
constexpr int kPTile = (kRows / 8) * 4 * 128;      // 8 KB: 16 row groups x 4 token groups x 128 B
// Score-exchange slot: [column half h][row][16 floats]. The four 16-byte
// pieces of row i are stored in the order k ^ ((i >> 1) & 3), so that eight
// consecutive rows' 16-byte accesses cover all 32 banks. The 32 rows one
// softmax warp owns in one half are a contiguous 2048-byte block, sent as one
// bulk copy (the copy moves bytes, so both sides see the same order).
constexpr int kXRowBytes = 64;
constexpr int kXWarpBlock = 32 * kXRowBytes;
constexpr int kXHalf = kRows * kXRowBytes;
constexpr int kXBuf = 2 * kXHalf;
constexpr int kCodeCC = 4096;                      // content codes half (32 tokens x <=128 B)
constexpr int kCodeRC = 1024;                      // rope codes (32 tokens x <=32 B)
constexpr int kCodeCM = 1024;                      // content meta half (32 tokens x <=32 B)
constexpr int kCodeStage = 7168;                   // content codes 1024-aligned at its start; <= 6,400 B used
constexpr int kOffC = 0;
constexpr int kOffP = kOffC + kNC * kCStage;
constexpr int kOffX = kOffP + 2 * kPTile;  // one weight tile (hi, lo): rewritten only after PV of the previous chunk
constexpr int kOffCode = kOffX + 2 * kXBuf;
constexpr int kOffBar = kOffCode + kNS * kCodeStage + kRows * kHalfR * 2;
constexpr int kOffQR = kOffCode + kNS * kCodeStage;  // rope part of Q: 128 rows x 32 bf16, core matrices
constexpr int kQRBytes = kRows * kHalfR * 2;
constexpr int kNumBars = kBarCode + kNS + 3 * kNC + 16 + 12;
constexpr int kOffMisc = kOffQR + kQRBytes + kNumBars * 8;
constexpr int kOffRed = kOffMisc + 64;  // row-pair exchange: [2 parity][2 halves][128] maxima, [2][128] sums
constexpr int kSmemBytes = kOffRed + (2 * 2 * kRows + 2 * kRows) * 4;
// Epilogue staging of the output rows, over the operand stages and weight tiles
// (free once every MMA has completed): [row][2 halves x 512 B] + 16 B of pad,
// so that the 16-byte stores of eight consecutive rows hit distinct banks.
constexpr int kEpiRow = 2 * 512 + 16;
static_assert(kOffC + kRows * kEpiRow <= kOffX, "epilogue staging fits the operand and weight-tile stages");
constexpr int kSmemAlloc = kSmemBytes + 1024;      // slack to align the base to 1024
static_assert(kOffCode % 1024 == 0 && kCodeStage % 1024 == 0, "TMA swizzle needs 1024-byte aligned stages");
static_assert(kSmemAlloc <= 232448, "shared memory budget");
static_assert(kSmemAlloc > 232448 / 2, "one CTA per SM keeps the 512-column TMEM allocation uncontended");

struct TmapSet {
  CUtensorMap cc;  // content codes [pages][64][row_c] bytes, box = half row x 32 tokens
  CUtensorMap rc;  // rope codes    [pages][64][row_r], box = full row x 32 tokens
  CUtensorMap cm;  // content meta  [pages][64][groups_c*4], box = half x 32 tokens
};

struct Bars {
  uint64_t* code_full;   // [kBarCode] TMA -> dequant (quantized: per code stage; BF16: per operand stage)
  uint64_t* code_empty;  // [kNS] dequant -> TMA
  uint64_t* c_full;      // [kNC] dequant -> MMA: channel chunks 0-15 of the stage written
  uint64_t* c_full2;     // [kNC] dequant -> MMA: chunks 16-35 written
  uint64_t* c_empty;     // [kNC] MMA (after PV) -> dequant
  uint64_t* s_full;      // [2] MMA (QK) -> softmax
  uint64_t* s_empty;     // [2] softmax read S -> MMA
  uint64_t* p_full;      // [1] softmax P tile + O rescale -> MMA (one tile buffer; slot 1 unused)
  uint64_t* p_empty;     // [1] MMA (PV) -> softmax
  uint64_t* x_full;      // [2] peer wrote its partial scores into my exchange buffer
  uint64_t* q_full;      // [1] Q in TMEM
  uint64_t* o_full;      // [1] all PV MMAs of the unit done
  uint64_t* qk_drain;    // [1] all QK MMAs of the even-chunk issuer done
  uint64_t* qk_drain2;   // [1] ... of the odd-chunk issuer
  uint64_t* pair_max;    // [4 lane quarters][2 parity] both halves of a row published their chunk maximum
  uint64_t* pair_sum;    // [4] both halves published their row sums (epilogue)
};

__device__ __forceinline__ Bars carve_bars(uint8_t* smem) {
  uint64_t* b = reinterpret_cast<uint64_t*>(smem + kOffBar);
  Bars r;
  r.code_full = b;
  r.code_empty = b + kBarCode;
  r.c_full = b + kBarCode + kNS;
  r.c_empty = b + kBarCode + kNS + kNC;
  uint64_t* p = b + kBarCode + kNS + 2 * kNC;
  r.s_full = p;
  r.s_empty = p + 2;
  r.p_full = p + 4;
  r.p_empty = p + 6;
  r.x_full = p + 8;
  r.q_full = p + 12;
  r.o_full = p + 13;
  r.qk_drain = p + 14;
  r.qk_drain2 = p + 15;
  r.pair_max = p + 16;
  r.pair_sum = p + 24;
  r.c_full2 = p + 28;  // [kNC]
  return r;
}

__device__ __forceinline__ float u2f(uint32_t u) {  // exact for u < 2^23
  return __uint_as_float(u | 0x4B000000u) - 8388608.0f;
}

// bf16 hi/lo of 8 values, packed two per 32-bit word (lower channel in the low half).
__device__ __forceinline__ void split8(const float (&x)[8], uint4& hi, uint4& lo) {
  uint32_t h[4], l[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    __nv_bfloat162 hb = __floats2bfloat162_rn(x[2 * k], x[2 * k + 1]);
    const uint32_t hw = *reinterpret_cast<uint32_t*>(&hb);
    const float h0 = __uint_as_float(hw << 16), h1 = __uint_as_float(hw & 0xFFFF0000u);
    __nv_bfloat162 lb = __floats2bfloat162_rn(x[2 * k] - h0, x[2 * k + 1] - h1);
    h[k] = hw;
    l[k] = *reinterpret_cast<uint32_t*>(&lb);
  }
  hi = make_uint4(h[0], h[1], h[2], h[3]);
  lo = make_uint4(l[0], l[1], l[2], l[3]);
}

template <int BITS>
__device__ __forceinline__ void dequant8(uint32_t w, float s, float z, float (&x)[8]) {
  constexpr uint32_t mask = (1u << BITS) - 1u;
#pragma unroll
  for (int k = 0; k < 8; ++k) x[k] = fmaf(u2f((w >> (k * BITS)) & mask), s, z);
}

__device__ __forceinline__ float ex2_approx(float x) {  // 2^x; -inf -> +0
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// 8 codes of one word -> bf16 hi/lo of u*s+z, with packed fp32x2 arithmetic.
// Code k sits at bits [k*BITS, (k+1)*BITS). Each code is placed in the low
// byte of the float 2^23 (exact integer embedding), the 2^23 is subtracted,
// and u*s+z is one fused multiply-add per pair.
template <int BITS>
__device__ __forceinline__ void dequant_split8(uint32_t w, float2 s2, float2 z2, uint4& hi, uint4& lo) {
  uint32_t b[8];
  if constexpr (BITS == 4) {
    const uint32_t ev = w & 0x0F0F0F0Fu, od = (w >> 4) & 0x0F0F0F0Fu;  // codes 0,2,4,6 / 1,3,5,7 in bytes
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      b[2 * k] = __byte_perm(ev, 0x4B000000u, 0x7650 | k);
      b[2 * k + 1] = __byte_perm(od, 0x4B000000u, 0x7650 | k);
    }
  } else {
    const uint32_t q0 = w & 0x03030303u, q1 = (w >> 2) & 0x03030303u;  // codes 0,4 / 1,5 in bytes 0,1 ...
    const uint32_t q2 = (w >> 4) & 0x03030303u, q3 = (w >> 6) & 0x03030303u;
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      b[4 * k] = __byte_perm(q0, 0x4B000000u, 0x7650 | k);
      b[4 * k + 1] = __byte_perm(q1, 0x4B000000u, 0x7650 | k);
      b[4 * k + 2] = __byte_perm(q2, 0x4B000000u, 0x7650 | k);
      b[4 * k + 3] = __byte_perm(q3, 0x4B000000u, 0x7650 | k);
    }
  }
  const float2 magic = make_float2(-8388608.0f, -8388608.0f);
  uint32_t h[4], l[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    float2 u = __fadd2_rn(make_float2(__uint_as_float(b[2 * k]), __uint_as_float(b[2 * k + 1])), magic);
    const float2 x = __ffma2_rn(u, s2, z2);
    __nv_bfloat162 hb = __floats2bfloat162_rn(x.x, x.y);
    const uint32_t hw = *reinterpret_cast<uint32_t*>(&hb);
    const float2 r = __fadd2_rn(x, make_float2(-__uint_as_float(hw << 16), -__uint_as_float(hw & 0xFFFF0000u)));
    __nv_bfloat162 lb = __floats2bfloat162_rn(r.x, r.y);
    h[k] = hw;
    l[k] = *reinterpret_cast<uint32_t*>(&lb);
  }
  hi = make_uint4(h[0], h[1], h[2], h[3]);
  lo = make_uint4(l[0], l[1], l[2], l[3]);
}

// Multiply one TMEM lane's 128 fp32 output columns at taddr by f
// (warp-collective: each lane scales its own row). Out of line: it runs
// rarely, and inlined its 32-register buffer would crowd the softmax loop.
__device__ __noinline__ void rescale_cols(uint32_t taddr, float f) {
#pragma unroll 1
  for (int c = 0; c < kHalfC / 64; ++c) {
    uint32_t ov[32];
    ptx::tmem_ld32(taddr + c * 32, ov);
    ptx::tmem_ld_wait();
#pragma unroll
    for (int k = 0; k < 32; ++k) ov[k] = __float_as_uint(__uint_as_float(ov[k]) * f);
    ptx::tmem_st32(taddr + c * 32, ov);
  }
}

__device__ __forceinline__ void fail(const DecodeArgs& a, volatile int* abort_flag) {
  record_error(a.status, MLA_ERR_TIMEOUT);
  *abort_flag = 1;
}

// kBF16: the unquantized comparison cache (bf16 [pages][64][576]); the TMA
// writes its rows straight into the operand layout (C_hi, no C_lo), the
// "dequant" warps only zero rows past the end of the keys, scores need one
// term and the output two (P_hi.C + P_lo.C). BITS_*/G_* are unused then.
template <int BITS_C, int G_C, int BITS_R, int G_R, bool kBF16>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    decode_tc_kernel(const DecodeArgs a, const __grid_constant__ TmapSet tm, int row_tiles, int n_terms_qk,
                     int n_terms_pv) {
  using G = QGeom<BITS_C, G_C, BITS_R, G_R>;
  // launched as a programmatic dependent: wait for the previous grid (e.g. the
  // cache append) before any read, then let the combine be scheduled
  ptx::griddep_wait();
  ptx::griddep_launch_dependents();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const Bars bars = carve_bars(smem);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffMisc + 8);
  volatile int* stage_page = reinterpret_cast<volatile int*>(smem + kOffMisc + 16);  // [kBarCode]

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t crank = ptx::cluster_ctarank();
  const uint32_t peer = crank ^ 1u;
  // MLA_DECODE_TEST_STALL (tests only): every wait gives up after 1 ms and the
  // page producer never issues chunk 1, so that the timeout path runs
  const bool test_stall = (a.flags & MLA_DECODE_TEST_STALL) != 0;
  const uint64_t wlim = test_stall ? 1000000ull : kWaitLimitNs;

  // ---- unit: from the work list (longest first) when the plan has one ----
  const int unit = a.worklist ? __ldg(a.worklist + (blockIdx.x >> 1)) : static_cast<int>(blockIdx.x >> 1);
  const int rt = unit % row_tiles;
  const int split = (unit / row_tiles) % a.n_split;
  const int b = unit / (row_tiles * a.n_split);
  const int T = checked_len(a, b);
  const int pages_b = (T + kPage - 1) / kPage;
  const int p_begin = split * a.chunk_pages;
  if (a.n_split > 1 && p_begin >= pages_b) return;  // both CTAs of the cluster leave together
  const int t_begin = min(p_begin * kPage, T);
  const int t_end = min(T, (p_begin + a.chunk_pages) * kPage);
  const int n_chunks = (t_end - t_begin + kChunk - 1) / kChunk;
  const int row0 = rt * kRows;

  if (n_chunks == 0) {  // no keys: o = 0, lse = -inf (single-split plans write the output)
    if (a.n_new > T && tid == 0 && crank == 0) record_error(a.status, MLA_ERR_INVALID_ARG);
    if (tid < kRows) {
      const int row = row0 + tid;
      if (row < a.rows) {
        const size_t qrow = static_cast<size_t>(b) * a.rows + row;
        for (int c = 0; c < kHalfC; ++c) {
          const size_t off = qrow * kDc + crank * kHalfC + c;
          if (a.n_split == 1) {
            if (a.out_f32) static_cast<float*>(a.out)[off] = 0.0f;
            else static_cast<__nv_bfloat16*>(a.out)[off] = __float2bfloat16_rn(0.0f);
          } else {
            a.o_part[((static_cast<size_t>(b) * a.n_split + split) * a.rows + row) * kDc + crank * kHalfC + c] = 0.f;
          }
        }
        if (crank == 0) {
          if (a.n_split == 1) { if (a.lse) a.lse[qrow] = -CUDART_INF_F; }
          else a.lse_part[(static_cast<size_t>(b) * a.n_split + split) * a.rows + row] = -CUDART_INF_F;
        }
      }
    }
    return;
  }

  // ---- setup ----
  if (tid == 0) {
    for (int i = 0; i < kBarCode; ++i) ptx::mbar_init(&bars.code_full[i], 1);
    for (int i = 0; i < kNS; ++i) ptx::mbar_init(&bars.code_empty[i], 128);
    for (int i = 0; i < kNC; ++i) {
      ptx::mbar_init(&bars.c_full[i], 128);
      ptx::mbar_init(&bars.c_full2[i], 128);
      ptx::mbar_init(&bars.c_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      ptx::mbar_init(&bars.s_full[i], 1);
      ptx::mbar_init(&bars.s_empty[i], kSoftThreads);
      ptx::mbar_init(&bars.p_full[i], kSoftThreads);
      ptx::mbar_init(&bars.p_empty[i], 1);
      ptx::mbar_init(&bars.x_full[i], 1);     // armed locally with expect_tx; bytes come from the peer
    }
    ptx::mbar_init(bars.q_full, kSoftThreads);
    ptx::mbar_init(bars.o_full, 1);
    ptx::mbar_init(bars.qk_drain, 1);
    ptx::mbar_init(bars.qk_drain2, 1);
    for (int q = 0; q < 8; ++q) ptx::mbar_init(&bars.pair_max[q], 64);
    for (int q = 0; q < 4; ++q) ptx::mbar_init(&bars.pair_sum[q], 64);
    *abort_flag = 0;
    ptx::fence_mbar_init_cluster();
  }
  if (warp == 0 && lane == 0) {
    ptx::prefetch_tmap(&tm.cc);
    ptx::prefetch_tmap(&tm.rc);
    ptx::prefetch_tmap(&tm.cm);
  }
  if (warp == 1) {
    ptx::tmem_alloc(tmem_slot, kTmemCols);
    ptx::tmem_relinquish();
  }
  if constexpr (!kBF16) {
    // Fused append: the step's n_new new tokens are the last n_new of the T
    // positions. CTA 0 of the pair quantizes those inside this unit's key
    // range into the pool (one warp per token, the same writer as the append
    // kernel) before either CTA loads a page; the proxy fence and the cluster
    // barrier below order those writes before the TMA reads. Row tiles of one
    // request write identical bytes.
    if (a.n_new > 0 && crank == 0 && warp >= 8) {
      if (T < a.n_new) {
        if (tid == 256) record_error(a.status, MLA_ERR_INVALID_ARG);
      } else {
        const int t_new = T - a.n_new;
        for (int t = max(t_new, t_begin) + (warp - 8); t < t_end; t += 8) {
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
    }
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::cluster_sync();  // peer barriers are initialised before any remote arrive; fused-append writes are visible
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // =========================== TMA producer ===========================
    if (lane == 0 && kBF16) {
      // bf16 rows land directly in operand stage j % kNC once PV of chunk j-kNC released it
      int issued[kNC];
      for (int i = 0; i < kNC; ++i) issued[i] = 0;
      for (int j = 0; j < n_chunks; ++j) {
        const int cs = j % kNC;
        if (j >= kNC && !ptx::mbar_wait(&bars.c_empty[cs], ((j - kNC) / kNC) & 1, abort_flag, wlim)) {
          fail(a, abort_flag);
          break;
        }
        if (test_stall && j == 1) continue;  // never issued nor arrived: the consumers' waits run out
        const int t0 = t_begin + j * kChunk;
        const int page = lookup_page(a.table, a.max_pages, a.num_pages, b, t0);
        uint8_t* st = smem + kOffC + cs * kCStage;
        stage_page[cs] = page;
        if (page >= 0) {
          ptx::mbar_arrive_expect_tx(&bars.code_full[cs], kKChunks * kChunk * 16);
          const int slot0 = t0 % kPage;
          ptx::tma_load_4d(st, &tm.cc, 0, slot0, crank * (kHalfC / 8), page, &bars.code_full[cs]);
          ptx::tma_load_4d(st + (kHalfC / 8) * kBfChunkStride, &tm.rc, 0, slot0, kDc / 8 + crank * (kHalfR / 8), page,
                           &bars.code_full[cs]);
        } else {
          record_error(a.status, MLA_ERR_INVALID_ARG);
          ptx::mbar_arrive(&bars.code_full[cs]);
        }
        issued[cs] = j + 1;
      }
      for (int cs = 0; cs < kNC; ++cs)
        if (issued[cs] > 0) ptx::mbar_wait(&bars.code_full[cs], ((issued[cs] - 1) / kNC) & 1, nullptr, wlim);
    } else if (lane == 0) {
      if (a.n_new > 0) ptx::fence_proxy_async_global();  // the fused append's writes precede these TMA reads
      const uint32_t bytes = kChunk * (G::kRowC / 2) + kChunk * G::kRowR + kChunk * (G::kGroupsC * 2) +
                             kChunk * G::kGroupsR * 4;
      int issued[kNS];
      for (int i = 0; i < kNS; ++i) issued[i] = 0;
      for (int j = 0; j < n_chunks; ++j) {
        const int s = j % kNS;
        if (j >= kNS && !ptx::mbar_wait(&bars.code_empty[s], ((j - kNS) / kNS) & 1, abort_flag, wlim)) {
          fail(a, abort_flag);
          break;
        }
        if (test_stall && j == 1) continue;  // never issued nor arrived: the consumers' waits run out
        const int t0 = t_begin + j * kChunk;
        const int page = lookup_page(a.table, a.max_pages, a.num_pages, b, t0);
        uint8_t* st = smem + kOffCode + s * kCodeStage;
        stage_page[s] = page;  // published to the dequant warps by the release-arrive below
        if (page >= 0) {
          ptx::mbar_arrive_expect_tx(&bars.code_full[s], bytes);
          const int slot0 = t0 % kPage;
          ptx::tma_load_3d(st, &tm.cc, crank * (G::kRowC / 2), slot0, page, &bars.code_full[s]);
          ptx::tma_load_3d(st + kCodeCC, &tm.rc, 0, slot0, page, &bars.code_full[s]);
          ptx::tma_load_3d(st + kCodeCC + kCodeRC, &tm.cm, crank * (G::kGroupsC * 2), slot0, page,
                           &bars.code_full[s]);
          const uint8_t* rm = a.pool + static_cast<size_t>(page) * G::kPageBytes + G::kOffRM +
                              static_cast<size_t>(slot0) * G::kGroupsR * 4;
          ptx::bulk_load(st + kCodeCC + kCodeRC + kCodeCM, rm, kChunk * G::kGroupsR * 4, &bars.code_full[s]);
        } else {
          record_error(a.status, MLA_ERR_INVALID_ARG);
          ptx::mbar_arrive(&bars.code_full[s]);
        }
        issued[s] = j + 1;
      }
      // drain copies still in flight before the CTA can exit
      for (int s = 0; s < kNS; ++s)
        if (issued[s] > 0) ptx::mbar_wait(&bars.code_full[s], ((issued[s] - 1) / kNS) & 1, nullptr, wlim);
    }
  } else if (warp == 1 || warp == 7) {
    // =========================== QK issuers ===========================
    // S_j[128 rows x 64] = Q . [C_hi ; C_lo]^T over this CTA's 288 channels:
    // 16 K-steps with the content part of Q in TMEM, 2 with its RoPE part in
    // shared memory. Descriptors are built once; K-steps only move the start
    // address field.
    // Two issuing threads (even / odd chunks) hide the per-instruction issue
    // latency of tcgen05.mma; each owns one of the two score buffers.
    if (lane == 0) {
      const int par = (warp == 1) ? 0 : 1;
      uint64_t* drain = (warp == 1) ? bars.qk_drain : bars.qk_drain2;
      constexpr int cstride = kBF16 ? kBfChunkStride : kCChunkStride;
      const uint32_t idesc = ptx::idesc_bf16_f32(kRows, (!kBF16 && n_terms_qk == 2) ? 2 * kChunk : kChunk, 0, 0);
      const uint64_t b0 = ptx::smem_desc_noswizzle(ptx::smem_u32(smem + kOffC), cstride, 128);
      const uint64_t a_rope = ptx::smem_desc_noswizzle(ptx::smem_u32(smem + kOffQR), 128, 512);
      bool ok = ptx::mbar_wait(bars.q_full, 0, abort_flag, wlim);
      for (int j = par; ok && j < n_chunks; j += 2) {
        const int cs = j % kNC, sb = j & 1;
        if (!ptx::mbar_wait(&bars.c_full[cs], (j / kNC) & 1, abort_flag, wlim) ||
            (j >= 2 && !ptx::mbar_wait(&bars.s_empty[sb], ((j - 2) >> 1) & 1, abort_flag, wlim))) {
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        const uint64_t bs = b0 + static_cast<uint64_t>((cs * kCStage) >> 4);
        const uint32_t d = tmem + kTmemS + sb * 2 * kChunk;
        // K-steps 0-7 read channel chunks 0-15, which the dequant warps
        // publish first (c_full); the rest follow once c_full2 completes
#pragma unroll
        for (int k = 0; k < kHalfC / 16; ++k) {
          if (k == kHalfC / 32) {
            if (!ptx::mbar_wait(&bars.c_full2[cs], (j / kNC) & 1, abort_flag, wlim)) {
              ok = false;
              break;
            }
            ptx::tc_fence_after();
          }
          ptx::mma_ts(d, tmem + kTmemQ + k * 8, bs + static_cast<uint64_t>((k * 2 * cstride) >> 4), idesc,
                      k > 0 ? 1u : 0u);
        }
        if (!ok) break;
#pragma unroll
        for (int k = 0; k < kHalfR / 16; ++k)
          ptx::mma_ss(d, a_rope + static_cast<uint64_t>((k * 256) >> 4),
                      bs + static_cast<uint64_t>(((kHalfC / 8 + 2 * k) * cstride) >> 4), idesc, 1u);
        ptx::mma_commit(&bars.s_full[sb]);
      }
      if (!ok) fail(a, abort_flag);
      ptx::mma_commit(drain);
      ptx::mbar_wait(drain, 0, nullptr, wlim);  // MMAs finish before TMEM is released
    }
  } else if (warp == 6) {
    // =========================== PV issuer ===========================
    // O_half[128 x 256] += P_hi.C_hi + P_lo.C_hi + P_hi.C_lo over the chunk's 32 tokens.
    if (lane == 0) {
      const uint32_t idesc = ptx::idesc_bf16_f32(kRows, kHalfC, 0, 1);
      const uint64_t a0 = ptx::smem_desc_noswizzle(ptx::smem_u32(smem + kOffP), 128, 512);
      const uint64_t b0 = ptx::smem_desc_noswizzle(ptx::smem_u32(smem + kOffC), 128,
                                                   kBF16 ? kBfChunkStride : kCChunkStride);
      bool ok = true;
      for (int j = 0; j < n_chunks; ++j) {
        const int cs = j % kNC;
        if (!ptx::mbar_wait(&bars.p_full[0], j & 1, abort_flag, wlim)) {
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        // Straight-line issue: the issuing thread runs no per-instruction
        // address or predicate arithmetic between the MMAs (measured: such
        // work between two tcgen05.mma instructions slows their issue).
        const uint64_t ap = a0;
        const uint64_t bc = b0 + static_cast<uint64_t>((cs * kCStage) >> 4);
        const uint64_t ap_lo = ap + static_cast<uint64_t>(kPTile >> 4);    // P_lo
        const uint64_t bc_lo = bc + static_cast<uint64_t>(kCLoOff >> 4);   // C_lo
        constexpr uint64_t kK1 = 256 >> 4;                                 // second 16-token K-step
        const uint32_t acc0 = j > 0 ? 1u : 0u;
        const uint32_t o = tmem + kTmemO;
        ptx::mma_ss(o, ap, bc, idesc, acc0);                               // P_hi . C_hi
        ptx::mma_ss(o, ap + kK1, bc + kK1, idesc, 1u);
        if (n_terms_pv >= 2) {                                             // P_lo . C_hi
          ptx::mma_ss(o, ap_lo, bc, idesc, 1u);
          ptx::mma_ss(o, ap_lo + kK1, bc + kK1, idesc, 1u);
        }
        if (n_terms_pv >= 3) {                                             // P_hi . C_lo
          ptx::mma_ss(o, ap, bc_lo, idesc, 1u);
          ptx::mma_ss(o, ap + kK1, bc_lo + kK1, idesc, 1u);
        }
        ptx::mma_commit(&bars.p_empty[0]);
        ptx::mma_commit(&bars.c_empty[cs]);
      }
      if (!ok) fail(a, abort_flag);
      ptx::mma_commit(bars.o_full);
      ptx::mbar_wait(bars.o_full, 0, nullptr, wlim);  // MMAs finish before TMEM is released
    }
  } else if (warp >= 2 && warp < 6) {
    // =========================== dequant ===========================
    const int dq = tid - 64;
    const int tq = dq & 31;       // token within the chunk
    const int qsel = dq >> 5;     // 0..3
    for (int j = 0; kBF16 && j < n_chunks; ++j) {
      // bf16 operands are already in place; rows past the keys (stale pool
      // rows, or a page the table could not name) are zeroed so that 0 * x
      // never meets a NaN or Inf
      const int cs = j % kNC;
      if (!ptx::mbar_wait(&bars.code_full[cs], (j / kNC) & 1, abort_flag, wlim)) { fail(a, abort_flag); break; }
      const int t0 = t_begin + j * kChunk;
      const int lim = stage_page[cs] >= 0 ? t_end - t0 : 0;
      if (lim < kChunk && tq >= lim) {
        uint8_t* st = smem + kOffC + cs * kCStage;
#pragma unroll
        for (int c = 0; c < kKChunks / 4; ++c)
          *reinterpret_cast<uint4*>(st + (qsel * (kKChunks / 4) + c) * kBfChunkStride + tq * 16) = make_uint4(0, 0, 0, 0);
      }
      ptx::fence_proxy_async_smem();
      ptx::mbar_arrive(&bars.c_full[cs]);
      ptx::mbar_arrive(&bars.c_full2[cs]);
    }
    for (int j = 0; !kBF16 && j < n_chunks; ++j) {
      const int s = j % kNS, cs = j % kNC;
      if (!ptx::mbar_wait(&bars.code_full[s], (j / kNS) & 1, abort_flag, wlim)) { fail(a, abort_flag); break; }
      if (j >= kNC && !ptx::mbar_wait(&bars.c_empty[cs], ((j - kNC) / kNC) & 1, abort_flag, wlim)) {
        fail(a, abort_flag);
        break;
      }
      const int t0 = t_begin + j * kChunk;
      const bool valid = (t0 + tq < t_end) && stage_page[s] >= 0;
      const uint8_t* st = smem + kOffCode + s * kCodeStage;
      uint8_t* chi = smem + kOffC + cs * kCStage;
      uint8_t* clo = chi + kCLoOff;
      // content: quads qsel and qsel+4 (32 channels each)
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int q = qsel + 4 * h;
        const uint32_t meta = *reinterpret_cast<const uint32_t*>(st + kCodeCC + kCodeRC +
                                                                 tq * (G::kGroupsC * 2) + ((q * 32) / G_C) * 4);
        const float sc = half_bits_to_float(meta), zc = half_bits_to_float(meta >> 16);
        uint32_t w[4];
        if constexpr (BITS_C == 4) {  // 16 B per quad, 128-byte swizzled rows
          const uint4 v = *reinterpret_cast<const uint4*>(st + tq * 128 + ((q ^ (tq & 7)) * 16));
          w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w;
        } else {                      // 8 B per quad, 64-byte swizzled rows
          const uint2 v = *reinterpret_cast<const uint2*>(st + tq * 64 + ((((q >> 1) ^ ((tq >> 1) & 3)) * 16)) +
                                                           (q & 1) * 8);
          w[0] = v.x & 0xFFFFu; w[1] = v.x >> 16; w[2] = v.y & 0xFFFFu; w[3] = v.y >> 16;
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          uint4 hi = make_uint4(0, 0, 0, 0), lo = hi;
          if (valid) dequant_split8<BITS_C>(w[i], make_float2(sc, sc), make_float2(zc, zc), hi, lo);
          const int off = (4 * q + i) * kCChunkStride + tq * 16;
          *reinterpret_cast<uint4*>(chi + off) = hi;
          *reinterpret_cast<uint4*>(clo + off) = lo;
        }
        if (h == 0) {  // chunks 0-15 of every token are in place: the first QK K-steps may start
          ptx::fence_proxy_async_smem();
          ptx::mbar_arrive(&bars.c_full[cs]);
        }
      }
      {  // rope: 8 channels (chunk qsel of this CTA's 32)
        const uint32_t meta = *reinterpret_cast<const uint32_t*>(st + kCodeCC + kCodeRC + kCodeCM +
                                                                 tq * G::kGroupsR * 4 + (G_R == 64 ? 0 : crank) * 4);
        const float sr = half_bits_to_float(meta), zr = half_bits_to_float(meta >> 16);
        const uint8_t* row = st + kCodeCC + tq * G::kRowR + crank * (G::kRowR / 2);
        const uint32_t w = (BITS_R == 4) ? *reinterpret_cast<const uint32_t*>(row + qsel * 4)
                                         : static_cast<uint32_t>(*reinterpret_cast<const uint16_t*>(row + qsel * 2));
        uint4 hi = make_uint4(0, 0, 0, 0), lo = hi;
        if (valid) dequant_split8<BITS_R>(w, make_float2(sr, sr), make_float2(zr, zr), hi, lo);
        const int off = (32 + qsel) * kCChunkStride + tq * 16;
        *reinterpret_cast<uint4*>(chi + off) = hi;
        *reinterpret_cast<uint4*>(clo + off) = lo;
      }
      ptx::fence_proxy_async_smem();
      ptx::mbar_arrive(&bars.c_full2[cs]);
      ptx::mbar_arrive(&bars.code_empty[s]);
    }
  } else if (warp >= 8) {
    // =========================== softmax / epilogue ===========================
    // Two threads per row: warps w and w+4 read the same TMEM lane quarter;
    // half h owns score columns [16h, 16h+16) of every chunk and output
    // columns [128h, 128h+128) of this CTA's 256. The halves exchange their
    // chunk maximum through shared memory (an mbarrier per lane quarter, so a
    // stalled partner ends in a bounded wait), take identical softmax
    // decisions, and add their partial row sums once, in the epilogue.
    const int h = (warp - 8) >> 2;
    const int quarter = warp & 3;
    const int i = quarter * 32 + lane;  // row within the tile == TMEM lane
    const int row = row0 + i;
    const bool row_ok = row < a.rows;
    const int L = row_ok ? row_visible(T, a.s_q, a.H, row) : 0;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    const size_t qrow = static_cast<size_t>(b) * a.rows + (row_ok ? row : 0);
    float* red_max = reinterpret_cast<float*>(smem + kOffRed);   // [parity][half][row]
    float* red_sum = red_max + 2 * 2 * kRows;                   // [half][row]

    // Q: content half -> TMEM columns [384, 512) (half h stores 64 of its 256
    // channels' worth of columns); RoPE half -> shared memory as K-major core
    // matrices (half h stores chunks 2h, 2h+1). Padding rows get zeros.
    {
      const uint4* qc = reinterpret_cast<const uint4*>(a.q_c + qrow * kDc + crank * kHalfC);
      const uint4* qr = reinterpret_cast<const uint4*>(a.q_r + qrow * kDr + crank * kHalfR);
      // both blocks' loads are issued before the first TMEM store (a single
      // round trip to memory: the stores are barriers to the compiler)
      uint32_t v[2][32];
#pragma unroll
      for (int bb = 0; bb < 2; ++bb)
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const uint4 x = row_ok ? __ldg(qc + (2 * h + bb) * 8 + k) : make_uint4(0, 0, 0, 0);
          v[bb][4 * k] = x.x; v[bb][4 * k + 1] = x.y; v[bb][4 * k + 2] = x.z; v[bb][4 * k + 3] = x.w;
        }
#pragma unroll
      for (int bb = 0; bb < 2; ++bb) ptx::tmem_st32(lane_base + kTmemQ + (2 * h + bb) * 32, v[bb]);
      uint8_t* qrs = smem + kOffQR + (i >> 3) * 512 + (i & 7) * 16;
#pragma unroll
      for (int kk = 0; kk < 2; ++kk) {
        const int kc = 2 * h + kk;
        *reinterpret_cast<uint4*>(qrs + kc * 128) = row_ok ? __ldg(qr + kc) : make_uint4(0, 0, 0, 0);
      }
      ptx::fence_proxy_async_smem();
      ptx::tmem_st_wait();
      ptx::tc_fence_before();
      ptx::mbar_arrive(bars.q_full);
    }

    // Score exchange. Each CTA reads its partial S_j from TMEM, stages it in
    // its own exchange slot (j+1)&1 (whose chunk j-1 entries it has just
    // read), and each warp bulk-copies its 32 rows x 16 columns to the same
    // place in the peer's slot j&1 (the copy engine completes the bytes on
    // the peer's x_full). No release handshake is needed: the peer sends
    // chunk j+1 into the staging slot only after it received chunk j, i.e.
    // after this copy has read the stage.
    const uint32_t xbuf_peer = ptx::mapa(ptx::smem_u32(smem + kOffX), peer);
    const uint32_t xfull_peer = ptx::mapa(ptx::smem_u32(bars.x_full), peer);
    float m_used = -CUDART_INF_F, l_sum = 0.0f;  // l_sum: this half's columns only
    bool o_live = false;  // O has been written by a PV MMA
    bool ok = true;
    uint32_t prev[16];
    int prev_page = -1;

    // Chunk jj's weight tile (my 16 tokens of this row) -> shared memory,
    // once PV of chunk jj-1 has released the one tile buffer (the phase waited
    // for is the latest: PV of chunk jj needs this tile first, so no later
    // phase can have completed). False when the wait gave up.
    auto store_weights = [&](int jj, const uint32_t (&ph)[8], const uint32_t (&pl)[8]) -> bool {
      if (jj >= 1 &&
          !__all_sync(kFull, ptx::mbar_wait(&bars.p_empty[0], (jj - 1) & 1, abort_flag, wlim)))
        return false;
      uint8_t* pt = smem + kOffP + (i >> 3) * 512 + (i & 7) * 16;
#pragma unroll
      for (int kk = 0; kk < 2; ++kk) {
        const int kc = 2 * h + kk;
        *reinterpret_cast<uint4*>(pt + kc * 128) = make_uint4(ph[4 * kk], ph[4 * kk + 1], ph[4 * kk + 2], ph[4 * kk + 3]);
        *reinterpret_cast<uint4*>(pt + kPTile + kc * 128) =
            make_uint4(pl[4 * kk], pl[4 * kk + 1], pl[4 * kk + 2], pl[4 * kk + 3]);
      }
      return true;
    };
    // The O rescale a grown maximum needs, then the release of chunk jj's
    // weight tile to the PV issuer. `fence`: the tile's stores still need the
    // generic -> async proxy fence (a later fence of this thread covers them
    // too). False when a wait gave up.
    auto release_weights = [&](int jj, float alpha, bool rescale, bool fence) -> bool {
      // rescale my half of this row of O in TMEM (warp-collective: lanes that
      // do not need it multiply by 1); O must be quiescent: PV of chunk jj-1 done
      if (__any_sync(kFull, rescale && o_live)) {
        if (!__all_sync(kFull, ptx::mbar_wait(&bars.p_empty[0], (jj - 1) & 1, abort_flag,
                                              wlim)))
          return false;
        ptx::tc_fence_after();
        rescale_cols(lane_base + kTmemO + h * (kHalfC / 2), (rescale && o_live) ? alpha : 1.0f);
        ptx::tmem_st_wait();
      }
      o_live = true;
      if (fence) ptx::fence_proxy_async_smem();
      ptx::tc_fence_before();
      ptx::mbar_arrive(&bars.p_full[0]);
      return true;
    };

    // Step j: first the peer's partial scores of chunk j-1 (sent one step
    // earlier) into registers, then the read and send of this CTA's partial
    // of chunk j (staged in the exchange slot just read), then the softmax of
    // chunk j-1 and its weight tile: the copy to the peer is in flight while
    // this thread finishes the previous chunk.
    for (int j = 0; j <= n_chunks && ok; ++j) {
      float pvv[16];
      if (j >= 1) {
        const int jj = j - 1, pb = jj & 1;
        if (!__all_sync(kFull, ptx::mbar_wait(&bars.x_full[pb], (jj >> 1) & 1, abort_flag, wlim))) {
          ok = false;
          break;
        }
        const float4* xr = reinterpret_cast<const float4*>(smem + kOffX + pb * kXBuf + h * kXHalf + i * kXRowBytes);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float4 pv = xr[k ^ ((i >> 1) & 3)];
          pvv[4 * k] = pv.x; pvv[4 * k + 1] = pv.y; pvv[4 * k + 2] = pv.z; pvv[4 * k + 3] = pv.w;
        }
      }
      uint32_t cur[16];
      int cur_page = -1;
      if (j < n_chunks) {
        const int sb = j & 1;
        // block-table entry of chunk j, checked one step later: issued before the wait to hide the load
        cur_page = table_entry(a.table, a.max_pages, b, t_begin + j * kChunk);
        // wait results are made warp-uniform: the TMEM loads below are warp-collective
        if (!__all_sync(kFull, ptx::mbar_wait(&bars.s_full[sb], (j >> 1) & 1, abort_flag, wlim))) {
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        ptx::tmem_ld16(lane_base + kTmemS + sb * 2 * kChunk + 16 * h, cur);
        if (n_terms_qk == 2) {  // add the C_lo half of the score tile, 8 columns at a time
#pragma unroll
          for (int g = 0; g < 2; ++g) {
            uint32_t lo[8];
            ptx::tmem_ld8(lane_base + kTmemS + sb * 2 * kChunk + kChunk + 16 * h + 8 * g, lo);
            ptx::tmem_ld_wait();
#pragma unroll
            for (int k = 0; k < 8; ++k)
              cur[8 * g + k] = __float_as_uint(__uint_as_float(cur[8 * g + k]) + __uint_as_float(lo[k]));
          }
        }
        ptx::tmem_ld_wait();
        ptx::tc_fence_before();
        ptx::mbar_arrive(&bars.s_empty[sb]);
        // Send my partial scores to the peer, staged in the other exchange
        // slot, whose segment for my row and half I read above (chunk j-1);
        // the peer writes that slot again (chunk j+1) only after this copy
        // has landed, and I restage it only after that.
        const int blk = h * kXHalf + quarter * kXWarpBlock;
        uint8_t* stage = smem + kOffX + (sb ^ 1) * kXBuf + h * kXHalf + i * kXRowBytes;
#pragma unroll
        for (int k = 0; k < 4; ++k)
          *reinterpret_cast<uint4*>(stage + 16 * (k ^ ((i >> 1) & 3))) = make_uint4(cur[4 * k], cur[4 * k + 1], cur[4 * k + 2], cur[4 * k + 3]);
        ptx::fence_proxy_async_smem();
        __syncwarp();
        if (i == 0 && h == 0) ptx::mbar_arrive_expect_tx(&bars.x_full[sb], kXBuf);
        if (lane == 0)
          ptx::bulk_copy_to_peer(xbuf_peer + sb * kXBuf + blk, smem + kOffX + (sb ^ 1) * kXBuf + blk, kXWarpBlock,
                                 xfull_peer + sb * 8);
      }
      if (j >= 1) {
        const int jj = j - 1, pb = jj & 1;
        const int t0 = t_begin + jj * kChunk;
        uint32_t ph[8], pl[8];
        float alpha = 1.0f;
        bool rescale = false;
        // full score = my partial + peer partial, then * scale * log2(e)
        const float2 sc2 = make_float2(a.scale_log2, a.scale_log2);
        float2 sp[8];
#pragma unroll
        for (int k = 0; k < 8; ++k)
          sp[k] = __fmul2_rn(__fadd2_rn(make_float2(__uint_as_float(prev[2 * k]), __uint_as_float(prev[2 * k + 1])),
                                        make_float2(pvv[2 * k], pvv[2 * k + 1])), sc2);
        const int lim = (page_valid(prev_page, a.num_pages) ? min(L, t_end) - t0 : 0) - 16 * h;  // visible columns in my half
        if (lim < 16) {
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            if (2 * k >= lim) sp[k].x = -CUDART_INF_F;
            if (2 * k + 1 >= lim) sp[k].y = -CUDART_INF_F;
          }
        }
        float mt[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) mt[k] = fmaxf(sp[k].x, sp[k].y);
#pragma unroll
        for (int w = 4; w >= 1; w >>= 1)
#pragma unroll
          for (int k = 0; k < w; ++k) mt[k] = fmaxf(mt[k], mt[k + w]);
        // chunk maximum of the whole row: publish mine, wait for the other half's
        red_max[(pb * 2 + h) * kRows + i] = mt[0];
        ptx::mbar_arrive(&bars.pair_max[quarter * 2 + pb]);
        if (!__all_sync(kFull, ptx::mbar_wait(&bars.pair_max[quarter * 2 + pb], (jj >> 1) & 1, abort_flag,
                                              wlim))) {
          ok = false;
          break;
        }
        const float mx = fmaxf(mt[0], red_max[(pb * 2 + (h ^ 1)) * kRows + i]);
        if (mx > -CUDART_INF_F) {
          if (m_used == -CUDART_INF_F) {
            m_used = mx;
          } else if (mx > m_used + kRescaleLog2) {
            alpha = ex2_approx(m_used - mx);
            m_used = mx;
            rescale = true;
          }
        }
        // p = 2^(s - m); rows that have seen no key use m = 0, so every p is 0
        const float m_eff = (m_used == -CUDART_INF_F) ? 0.0f : m_used;
        const float2 negm = make_float2(-m_eff, -m_eff);
        float2 ps[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const float2 d = __fadd2_rn(sp[k], negm);
          const float2 pk = make_float2(ex2_approx(d.x), ex2_approx(d.y));
          ps[k] = pk;
          __nv_bfloat162 hb = __floats2bfloat162_rn(pk.x, pk.y);
          const uint32_t hw = *reinterpret_cast<uint32_t*>(&hb);
          const float2 r = __fadd2_rn(pk, make_float2(-__uint_as_float(hw << 16), -__uint_as_float(hw & 0xFFFF0000u)));
          __nv_bfloat162 lb = __floats2bfloat162_rn(r.x, r.y);
          ph[k] = hw;
          pl[k] = *reinterpret_cast<uint32_t*>(&lb);
        }
#pragma unroll
        for (int w = 4; w >= 1; w >>= 1)
#pragma unroll
          for (int k = 0; k < w; ++k) ps[k] = __fadd2_rn(ps[k], ps[k + w]);
        l_sum = l_sum * alpha + (ps[0].x + ps[0].y);
        if (!store_weights(jj, ph, pl) || !release_weights(jj, alpha, rescale, true)) {
          ok = false;
          break;
        }
      }
#pragma unroll
      for (int k = 0; k < 16; ++k) prev[k] = cur[k];
      prev_page = cur_page;
    }

    // epilogue: row sum = both halves; O / l for my 128 of this CTA's 256 channels
    if (!ok) fail(a, abort_flag);
    red_sum[h * kRows + i] = l_sum;
    ptx::mbar_arrive(&bars.pair_sum[quarter]);
    const bool sums_ready = ptx::mbar_wait(&bars.pair_sum[quarter], 0, abort_flag, wlim);
    const bool o_ready = ptx::mbar_wait(bars.o_full, 0, abort_flag, wlim);
    const int aborted = *abort_flag;
    if (__all_sync(kFull, sums_ready && o_ready && ok && !aborted)) {  // warp-uniform: TMEM loads are collective
      ptx::tc_fence_after();
      const float l_tot = l_sum + red_sum[(h ^ 1) * kRows + i];
      const float inv = l_tot > 0.0f ? 1.0f / l_tot : 0.0f;
      const float lse = l_tot > 0.0f ? (m_used + log2f(l_tot)) * kLn2 : -CUDART_INF_F;
      const size_t part = (static_cast<size_t>(b) * a.n_split + split) * a.rows + row;
      // My 128 channels of the row are staged in shared memory, then written
      // by one bulk copy: whole 128-byte lines, where direct stores would
      // scatter 16-byte pieces over 32 rows per warp instruction.
      const bool bf16_out = (a.n_split == 1 && !a.out_f32);
      uint8_t* srow = smem + kOffC + i * kEpiRow + h * 512;
#pragma unroll 1
      for (int c = 0; c < kHalfC / 64; ++c) {
        uint32_t ov[32];
        ptx::tmem_ld32(lane_base + kTmemO + h * (kHalfC / 2) + c * 32, ov);
        ptx::tmem_ld_wait();
        if (bf16_out) {
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            uint32_t w[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              __nv_bfloat162 hv = __floats2bfloat162_rn(__uint_as_float(ov[8 * k + 2 * e]) * inv,
                                                        __uint_as_float(ov[8 * k + 2 * e + 1]) * inv);
              w[e] = *reinterpret_cast<uint32_t*>(&hv);
            }
            *reinterpret_cast<uint4*>(srow + c * 64 + 16 * k) = make_uint4(w[0], w[1], w[2], w[3]);
          }
        } else {
#pragma unroll
          for (int k = 0; k < 8; ++k)
            *reinterpret_cast<float4*>(srow + c * 128 + 16 * k) =
                make_float4(__uint_as_float(ov[4 * k]) * inv, __uint_as_float(ov[4 * k + 1]) * inv,
                            __uint_as_float(ov[4 * k + 2]) * inv, __uint_as_float(ov[4 * k + 3]) * inv);
        }
      }
      if (row_ok) {
        const int col = crank * kHalfC + h * (kHalfC / 2);
        void* dst = bf16_out ? static_cast<void*>(static_cast<__nv_bfloat16*>(a.out) + qrow * kDc + col)
                             : static_cast<void*>((a.n_split == 1 ? static_cast<float*>(a.out) + qrow * kDc
                                                                  : a.o_part + part * kDc) + col);
        ptx::fence_proxy_async_smem();
        ptx::bulk_store(dst, srow, bf16_out ? 256u : 512u);
        ptx::bulk_commit();
        ptx::bulk_wait_all();  // the copy has read shared memory and written the row before the CTA exits
      }
      if (crank == 0 && h == 0 && row_ok) {
        if (a.n_split == 1) {
          if (a.lse) a.lse[qrow] = lse;
        } else {
          a.lse_part[part] = lse;
        }
      }
    }
  }

  // ---- teardown ----
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, kTmemCols);
  }
  // No remote copy or arrive may target a CTA that has exited. After a clean
  // run every score copy has landed (each one was waited for); after an abort
  // one may still be in flight, so give it time to land before either exits.
  ptx::cluster_sync();
  if (tid == 0 && (*abort_flag || ptx::ld_cluster_s32(ptx::mapa(ptx::smem_u32((const void*)abort_flag), peer)))) {
    const uint64_t t0 = ptx::globaltimer_ns();
    while (ptx::globaltimer_ns() - t0 < 100000ull) {
    }
  }
  ptx::cluster_sync();
}

// ---------------------------------------------------------------- host side

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 3-D byte tensor [pages][64 tokens][width bytes] at base (row stride = width,
// page stride = page_bytes); box = box_w bytes x 32 tokens x 1 page.
bool make_map(CUtensorMap* m, const void* base, int width, int box_w, int page_bytes, int num_pages,
              CUtensorMapSwizzle swz) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(width), static_cast<cuuint64_t>(kPage),
                              static_cast<cuuint64_t>(num_pages)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(width), static_cast<cuuint64_t>(page_bytes)};
  const cuuint32_t box[3] = {static_cast<cuuint32_t>(box_w), static_cast<cuuint32_t>(kChunk), 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 4-D bf16 tensor [pages][64 tokens][72 chunks][8 channels] with the chunk
// dimension outermost-but-one in shared memory: box = 8 channels x 32 tokens
// x box_chunks x 1 page lands as [chunk][token][16 B], i.e. the no-swizzle
// core-matrix layout with a 512-byte chunk stride.
bool make_map_bf16(CUtensorMap* m, const void* base, int num_pages, int box_chunks) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[4] = {8, static_cast<cuuint64_t>(kPage), static_cast<cuuint64_t>(kDqk / 8),
                              static_cast<cuuint64_t>(num_pages)};
  const cuuint64_t strides[3] = {static_cast<cuuint64_t>(kDqk * 2), 16, static_cast<cuuint64_t>(kPage * kDqk * 2)};
  const cuuint32_t box[4] = {8, static_cast<cuuint32_t>(kChunk), static_cast<cuuint32_t>(box_chunks), 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int BC, int GC, int BR, int GR, bool kBF16>
cudaError_t launch_t(const DecodeLaunch& L) {
  using G = QGeom<BC, GC, BR, GR>;
  TmapSet tm;
  const uint8_t* pool = static_cast<const uint8_t*>(L.pool);
  if constexpr (kBF16) {
    if (!make_map_bf16(&tm.cc, pool, L.num_pages, kHalfC / 8) || !make_map_bf16(&tm.rc, pool, L.num_pages, kHalfR / 8))
      return cudaErrorNotSupported;
    tm.cm = tm.rc;
  } else {
    const CUtensorMapSwizzle swz_c = (BC == 4) ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
    if (!make_map(&tm.cc, pool + G::kOffCC, G::kRowC, G::kRowC / 2, G::kPageBytes, L.num_pages, swz_c) ||
        !make_map(&tm.rc, pool + G::kOffRC, G::kRowR, G::kRowR, G::kPageBytes, L.num_pages,
                  CU_TENSOR_MAP_SWIZZLE_NONE) ||
        !make_map(&tm.cm, pool + G::kOffCM, G::kGroupsC * 4, G::kGroupsC * 2, G::kPageBytes, L.num_pages,
                  CU_TENSOR_MAP_SWIZZLE_NONE))
      return cudaErrorNotSupported;
  }
  const DecodeArgs a = make_decode_args(L);
  const int row_tiles = (a.rows + kRows - 1) / kRows;
  const long units = static_cast<long>(a.B) * a.n_split * row_tiles;
  if (units * 2 > 0x7FFFFFFFL) return cudaErrorNotSupported;
  if (L.worklist) {
    const cudaError_t pe = launch_plan_units(L, row_tiles);
    if (pe != cudaSuccess) return pe;
  }
  auto kern = decode_tc_kernel<BC, GC, BR, GR, kBF16>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemAlloc);
  if (e != cudaSuccess) return e;
  const bool fast = (L.flags & MLA_DECODE_FAST_UNCOMPENSATED) != 0;
  const int terms_qk = (kBF16 || fast) ? 1 : 2;
  const int terms_pv = fast ? 1 : (kBF16 ? 2 : 3);
  return launch_dependent(kern, dim3(static_cast<unsigned>(units * 2)), dim3(kThreads), kSmemAlloc, L.stream, a, tm,
                          row_tiles, terms_qk, terms_pv);
}

}  // namespace tc

cudaError_t launch_decode_tc(const DecodeLaunch& L) {
  if (L.num_pages < 1) return cudaErrorNotSupported;
  int dev = 0, major = 0, minor = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess || major != 10 ||
      minor != 0)
    return cudaErrorNotSupported;
  if (!L.quantized) return tc::launch_t<4, 64, 4, 64, true>(L);
#define MLA_TC_CASE(BC, GC, BR, GR)                                              \
  if (L.bits_c == BC && L.group_c == GC && L.bits_r == BR && L.group_r == GR)  \
    return tc::launch_t<BC, GC, BR, GR, false>(L);
#define MLA_TC_R(BC, GC) \
  MLA_TC_CASE(BC, GC, 4, 64) MLA_TC_CASE(BC, GC, 4, 32) MLA_TC_CASE(BC, GC, 2, 64) MLA_TC_CASE(BC, GC, 2, 32)
  MLA_TC_R(4, 64)
  MLA_TC_R(4, 32)
  MLA_TC_R(2, 64)
  MLA_TC_R(2, 32)
#undef MLA_TC_R
#undef MLA_TC_CASE
  return cudaErrorNotSupported;
}

}  // namespace mla
