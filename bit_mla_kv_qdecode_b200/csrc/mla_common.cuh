// Shared definitions of the low-bit MLA decode library (device side).
//
// Cache geometry follows the page layout declared in include/mla_qcache.h:
// per 64-token page, [content codes][rope codes][content (s,z)][rope (s,z)],
// each segment 16-byte aligned; fp16 (s, z) pairs, codes packed little-endian.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "mla_qcache.h"

namespace mla {

constexpr int kDc = 512;   // content latent width
constexpr int kDr = 64;    // decoupled RoPE key width
constexpr int kDqk = kDc + kDr;
constexpr int kPage = 64;  // tokens per page
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// Compile-time geometry of one quantized page.
template <int BITS_C, int G_C, int BITS_R, int G_R>
struct QGeom {
  static constexpr int kBitsC = BITS_C, kGroupC = G_C, kBitsR = BITS_R, kGroupR = G_R;
  static constexpr int kRowC = kDc * BITS_C / 8;  // content code bytes per token
  static constexpr int kRowR = kDr * BITS_R / 8;  // rope code bytes per token
  static constexpr int kGroupsC = kDc / G_C;
  static constexpr int kGroupsR = kDr / G_R;
  static constexpr int kOffCC = 0;
  static constexpr int kOffRC = kOffCC + kPage * kRowC;
  static constexpr int kOffCM = kOffRC + kPage * kRowR;
  static constexpr int kOffRM = kOffCM + kPage * kGroupsC * 4;
  static constexpr int kPageBytes = kOffRM + kPage * kGroupsR * 4;
  static_assert(kOffRC % 16 == 0 && kOffCM % 16 == 0 && kOffRM % 16 == 0 && kPageBytes % 16 == 0,
                "page segments must stay 16-byte aligned");
};

// Record the first error seen on the device; later errors keep the first.
__device__ __forceinline__ void record_error(int* status, int code) {
  if (status) atomicCAS(status, 0, code);
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ float half_bits_to_float(uint32_t h) {
  return __half2float(__ushort_as_half(static_cast<unsigned short>(h & 0xFFFFu)));
}

// Page of token position t of request b, or -1 when the position or table
// entry is out of range (the caller skips such tokens and flags the status).
// The block-table entry for token t, not yet checked against the pool (-1 past
// the table's end): a caller can issue the load early and validate where it uses it.
__device__ __forceinline__ int table_entry(const int32_t* table, int max_pages, int b, int t) {
  int idx = t / kPage;
  if (t < 0 || idx >= max_pages) return -1;
  return __ldg(table + static_cast<size_t>(b) * max_pages + idx);
}

__device__ __forceinline__ bool page_valid(int page, int num_pages) { return page >= 0 && page < num_pages; }

__device__ __forceinline__ int lookup_page(const int32_t* table, int max_pages, int num_pages,
                                           int b, int t) {
  const int page = table_entry(table, max_pages, b, t);
  return page_valid(page, num_pages) ? page : -1;
}

// Arguments shared by the decode kernels.
struct DecodeArgs {
  const uint8_t* pool;       // quantized pool bytes, or bf16 pool
  const int32_t* table;
  const int32_t* seq_lens;
  const __nv_bfloat16* q_c;  // [B, s_q, H, 512]
  const __nv_bfloat16* q_r;  // [B, s_q, H, 64]
  void* out;                 // [B, s_q, H, 512]
  float* lse;                // [B, s_q, H] or null
  float* o_part;             // [B, n_split, rows, 512] (split plans only)
  float* lse_part;           // [B, n_split, rows]
  int* status;
  int max_pages, num_pages, max_seq_len;
  int B, s_q, H, rows;       // rows = s_q * H
  int n_split, chunk_pages;
  int out_f32;
  float scale_log2;          // softmax scale * log2(e)
  const __nv_bfloat16* c_new;   // fused append: [B, n_new, 512] (tensor-core and small-row kernels)
  const __nv_bfloat16* kr_new;  // [B, n_new, 64]
  int n_new;                    // 0: no fused append
  unsigned flags;               // MLA_DECODE_* bits of the call
  const int* worklist;          // tensor-core kernel: unit index per cluster, or null (index order)
};

// Keys visible to flattened row r = i*H + h of a request holding T keys.
__device__ __forceinline__ int row_visible(int T, int s_q, int H, int r) {
  int v = T - s_q + 1 + r / H;
  return v < 0 ? 0 : v;
}

// Clamp a device-side sequence length into [0, max_seq_len], flagging bad ones.
__device__ __forceinline__ int checked_len(const DecodeArgs& a, int b) {
  int T = __ldg(a.seq_lens + b);
  int cap = a.max_seq_len;
  if (T < 0 || T > cap) {
    record_error(a.status, MLA_ERR_INVALID_ARG);
    T = T < 0 ? 0 : cap;
  }
  return T;
}

}  // namespace mla
