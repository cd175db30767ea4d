// Internal launch interface between the C ABI (api.cu) and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

namespace mla {

// Launch `kern` as a programmatic dependent of the previous work in `stream`:
// its blocks may be scheduled while that work drains, and the kernel itself
// waits (griddepcontrol.wait) before reading anything.
template <typename... KArgs, typename... Args>
cudaError_t launch_dependent(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                             Args&&... args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

struct AppendLaunch {
  void* pool;
  int num_pages;
  const int32_t* table;
  int max_pages;
  const int32_t* lens_before;
  const void* c_new;
  const void* kr_new;
  int B, n_new;
  int bits_c, group_c, bits_r, group_r;
  // optional token source for the quantized append: row j of BF16 page
  // src_pages[b] of src_pool ([pages][64][576]) instead of c_new / kr_new
  const void* src_pool;
  int src_num_pages;
  const int32_t* src_pages;
  int* status;
  cudaStream_t stream;
  // position of new token j of request b: lens_before[b] + lens_offset + j
  // (-n_new when the lengths passed already count the new tokens)
  int lens_offset;
};

cudaError_t launch_qcache_append(const AppendLaunch& L);
cudaError_t launch_bf16cache_append(const AppendLaunch& L);

// One decode call, after validation and split planning.
struct DecodeLaunch {
  const void* pool;
  bool quantized;
  int bits_c, group_c, bits_r, group_r;
  int num_pages;
  const int32_t* table;
  int max_pages;
  const int32_t* seq_lens;
  int max_seq_len;
  const void* q_c;
  const void* q_r;
  int B, s_q, H;
  float scale;
  int n_split, chunk_pages;
  float* o_part;   // workspace (n_split > 1)
  float* lse_part;
  void* out;
  int out_f32;
  float* lse;
  unsigned flags;
  int* status;
  cudaStream_t stream;
  // fused append (tensor-core and small-row kernels): bf16 c_new [B, n_new, 512] and
  // kr_new [B, n_new, 64] are the last n_new of seq_lens[b] positions; each
  // unit quantizes those in its key range into the pool before reading it
  const void* c_new;
  const void* kr_new;
  int n_new;
  // tensor-core kernel with a split plan over a multi-wave grid: the order in
  // which clusters take their units (unit indices, longest first), built on
  // the device by launch_plan_units in the caller's workspace; null: index order
  int* worklist;
};

struct DecodeArgs;
DecodeArgs make_decode_args(const DecodeLaunch& L);

cudaError_t launch_decode_simt(const DecodeLaunch& L);
// out = log-sum-exp merge of two normalised partial results (fp32 [rows][512]
// each, natural-log lse; -inf carries weight 0), as bf16 (out_f32 = 0) or fp32.
cudaError_t launch_merge2(const float* o_a, const float* l_a, const float* o_b, const float* l_b, int rows,
                          void* out, int out_f32, float* lse, cudaStream_t stream);
cudaError_t launch_combine(const DecodeLaunch& L);
// Largest chunk (in pages) a work list handles: the split planner's cap.
constexpr int kMaxWorklistChunkPages = 128;
// Fill L.worklist (when set) with the tensor-core kernel's unit indices,
// longest unit first (one block; launched as a programmatic dependent).
cudaError_t launch_plan_units(const DecodeLaunch& L, int row_tiles);
// Returns cudaErrorNotSupported when the tensor-core kernel has no variant for
// the shape; the caller then uses the SIMT kernel.
cudaError_t launch_decode_tc(const DecodeLaunch& L);
// Warp-level MMA kernels for s_q * H <= 16 rows (quantized: INT4 g64 content
// and RoPE; or the BF16 cache); cudaErrorNotSupported for other shapes and formats.
cudaError_t launch_decode_small(const DecodeLaunch& L);
bool decode_small_supported(const DecodeLaunch& L);
// Warp-level MMA kernel for s_q * H <= 16 rows over the BF16 comparison cache.
cudaError_t launch_decode_small_bf16(const DecodeLaunch& L);
bool decode_small_bf16_supported(const DecodeLaunch& L);
// Query rows up to which a decode unit is one CTA of the small-row kernel.
constexpr int kSmallRows = 16;

}  // namespace mla
