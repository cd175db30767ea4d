// Merge of two normalised partial attention results over disjoint key sets:
// the BF16-protected segment (earliest tokens and the recent window) and the
// quantized history of a hybrid cache (QuantMLA podcast episode: history stays
// visible, only its storage precision differs). With lse_j = log sum of the
// segment's weights, one softmax over the union is
//   lse = log(e^{lse_a} + e^{lse_b}),  o = e^{lse_a - lse} o_a + e^{lse_b - lse} o_b.
#include <cuda_bf16.h>
#include <math_constants.h>

#include "mla_common.cuh"
#include "mla_internal.h"

namespace mla {
namespace {

__global__ void __launch_bounds__(128) merge2_kernel(const float* __restrict__ o_a, const float* __restrict__ l_a,
                                                     const float* __restrict__ o_b, const float* __restrict__ l_b,
                                                     void* out, int out_f32, float* lse) {
  const size_t row = blockIdx.x;
  const int tid = threadIdx.x;  // 4 of the row's 512 channels each
  const float la = l_a[row], lb = l_b[row];
  const float m = fmaxf(la, lb);
  float wa = 0.0f, wb = 0.0f, tot = 0.0f;
  if (m != -CUDART_INF_F) {
    wa = expf(la - m);
    wb = expf(lb - m);
    tot = wa + wb;
    wa /= tot;
    wb /= tot;
  }
  const float4 a = reinterpret_cast<const float4*>(o_a + row * kDc)[tid];
  const float4 b = reinterpret_cast<const float4*>(o_b + row * kDc)[tid];
  const float4 o = make_float4(fmaf(wa, a.x, wb * b.x), fmaf(wa, a.y, wb * b.y), fmaf(wa, a.z, wb * b.z),
                               fmaf(wa, a.w, wb * b.w));
  if (out_f32) {
    reinterpret_cast<float4*>(static_cast<float*>(out) + row * kDc)[tid] = o;
  } else {
    __nv_bfloat162* dst = reinterpret_cast<__nv_bfloat162*>(static_cast<__nv_bfloat16*>(out) + row * kDc) + 2 * tid;
    dst[0] = __floats2bfloat162_rn(o.x, o.y);
    dst[1] = __floats2bfloat162_rn(o.z, o.w);
  }
  if (tid == 0 && lse) lse[row] = tot > 0.0f ? m + logf(tot) : -CUDART_INF_F;
}

}  // namespace

cudaError_t launch_merge2(const float* o_a, const float* l_a, const float* o_b, const float* l_b, int rows,
                          void* out, int out_f32, float* lse, cudaStream_t stream) {
  if (rows <= 0) return cudaSuccess;
  merge2_kernel<<<rows, 128, 0, stream>>>(o_a, l_a, o_b, l_b, out, out_f32, lse);
  return cudaGetLastError();
}

}  // namespace mla
