// Decode entry point for callers that cannot allocate device memory.
//
// Some callers of a decode library are not allowed to call cudaMalloc at the
// moment they decode: a serving loop that owns a fixed device-memory budget
// and forbids allocation after start-up, a plug-in running inside a host
// framework that hands out all device memory itself, or latency-critical code
// where an allocation could synchronise the device. mla_qdecode asks such a
// caller for a workspace when it splits the keys; this file gives them a
// variant that takes its split-KV scratch from a fixed array compiled into the
// library instead.
//
// The scratch is a file-scope __device__ array. Every GPU that loads the
// library holds MLA_QDECODE_NOALLOC_SCRATCH_BYTES of it until the process
// exits. Host code cannot use the array's name as a device address, so the
// address is looked up with cudaGetSymbolAddress once per device, with that
// device current, on the first call made on that device.
#include <mutex>

#include "mla_common.cuh"
#include "mla_qcache.h"

namespace {

constexpr size_t kScratchBytes = MLA_QDECODE_NOALLOC_SCRATCH_BYTES;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch[kMaxDevices] = {};

// Device address of the scratch array on the current device (set up once per device).
mla_status scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return MLA_ERR_CUDA;
  }
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_scratch[dev]) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || !p) {
      cudaGetLastError();
      return MLA_ERR_CUDA;
    }
    g_scratch[dev] = p;
  }
  *out = g_scratch[dev];
  return MLA_OK;
}

}  // namespace

extern "C" mla_status mla_qdecode_noalloc(const mla_qcache_desc* desc, const void* pool, const int32_t* block_table,
                                          int max_pages_per_seq, const int32_t* seq_lens, int max_seq_len,
                                          const void* q_c, const void* q_r, int B, int s_q, int H, float scale,
                                          int num_splits, void* out, int out_dtype, float* lse, unsigned flags,
                                          mla_stream_t stream) {
  if (B < 0 || s_q < 1 || H < 1 || max_seq_len < 0 || num_splits < 0) return MLA_ERR_INVALID_ARG;
  // The split partials of every request are written by the decode kernel of
  // the same call before the combine kernel reads them, so the scratch needs
  // no clearing between calls.
  const size_t need = mla_decode_workspace_bytes(B, s_q, H, max_seq_len, num_splits);
  if (need > kScratchBytes) return MLA_ERR_WORKSPACE;
  void* ws = nullptr;
  if (need > 0) {
    const mla_status st = scratch_address(&ws);
    if (st != MLA_OK) return st;
  }
  return mla_qdecode(desc, pool, block_table, max_pages_per_seq, seq_lens, max_seq_len, q_c, q_r, B, s_q, H, scale,
                     num_splits, ws, need, out, out_dtype, lse, flags, stream);
}
