// Quantize + pack one token into its page slot, one warp per token: the
// writer shared by the append kernel and by the decode kernel's fused append.
//
// QuantMLA (arxivdaily.com/papers/2609.36760, English abstract) keeps the
// content and RoPE caches in INT4 (or INT2 content) and never holds a
// full-history high-precision copy, so every new token is quantized as it is
// written. Lane l owns content channels [16l, 16l+16) and RoPE channels
// {2l, 2l+1}; a group's min/max is a shuffle reduction over the lanes that
// share it. All arithmetic is IEEE fp32 with explicit round-to-nearest
// intrinsics so codes match a plain fp32 reference bit for bit.
#pragma once

#include "mla_common.cuh"

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

// Writes token (c_src [512], kr_src [64], bf16) into slot `slot` of page `pg`:
// content codes, content (s,z), RoPE codes, RoPE (s,z). All 32 lanes call it.
template <int BITS_C, int G_C, int BITS_R, int G_R>
__device__ __forceinline__ void quantize_token_warp(uint8_t* pg, int slot, const __nv_bfloat16* c_src,
                                                    const __nv_bfloat16* kr_src, int lane) {
  using G = QGeom<BITS_C, G_C, BITS_R, G_R>;

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

}  // namespace mla
