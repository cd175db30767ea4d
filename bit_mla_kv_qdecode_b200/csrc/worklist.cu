// Work partition of a split decode: the order in which the tensor-core decode
// kernel's clusters take their units (request, key split, 128-row tile).
//
// A split plan cuts every request's keys into page-aligned chunks of the same
// length (chunk_pages), so a ragged batch has units of every size from one
// page to a full chunk, and requests shorter than the longest have empty
// trailing splits. The hardware hands out CTAs (here: clusters) in index
// order as slots free up; taking the units longest first (a largest-first
// list schedule) keeps the short units for the tail, where they fill the
// slots the long ones leave, instead of a few long units running alone at the
// end. Sizes come from the device-side lengths, so the list is built on the
// device: one block counts the units per size (in pages, one bucket per page
// count), prefix-sums the counts in descending size order and scatters every
// unit index into its bucket. The order within a bucket is unspecified; it
// changes which slot runs a unit, never what the unit computes.
#include "mla_common.cuh"
#include "mla_internal.h"
#include "sm100_ptx.cuh"

namespace mla {

namespace {

constexpr int kPlanThreads = 1024;
constexpr int kMaxBuckets = kMaxWorklistChunkPages + 1;

__global__ void __launch_bounds__(kPlanThreads) plan_units_kernel(const int32_t* seq_lens, int max_seq_len, int B,
                                                                 int n_split, int chunk_pages, int row_tiles,
                                                                 int* worklist) {
  // launched as a programmatic dependent: the lengths may come from the previous kernel
  ptx::griddep_wait();
  ptx::griddep_launch_dependents();
  __shared__ int cnt[kMaxBuckets];
  const int tid = threadIdx.x;
  const int per_b = n_split * row_tiles;
  const int units = B * per_b;
  const int nb = chunk_pages + 1;
  for (int k = tid; k < nb; k += kPlanThreads) cnt[k] = 0;
  __syncthreads();
  // bucket 0 holds the units of chunk_pages pages, bucket chunk_pages the empty ones
  auto bucket = [&](int u) -> int {
    const int b = u / per_b;
    const int split = (u / row_tiles) % n_split;
    int T = __ldg(seq_lens + b);
    T = T < 0 ? 0 : (T > max_seq_len ? max_seq_len : T);  // the decode kernel flags bad lengths itself
    const int pages = (T + kPage - 1) / kPage - split * chunk_pages;
    return chunk_pages - (pages < 0 ? 0 : (pages > chunk_pages ? chunk_pages : pages));
  };
  for (int u = tid; u < units; u += kPlanThreads) atomicAdd(&cnt[bucket(u)], 1);
  __syncthreads();
  if (tid == 0) {
    int run = 0;
    for (int k = 0; k < nb; ++k) {
      const int c = cnt[k];
      cnt[k] = run;
      run += c;
    }
  }
  __syncthreads();
  for (int u = tid; u < units; u += kPlanThreads) worklist[atomicAdd(&cnt[bucket(u)], 1)] = u;
}

}  // namespace

cudaError_t launch_plan_units(const DecodeLaunch& L, int row_tiles) {
  if (!L.worklist) return cudaSuccess;
  if (L.chunk_pages < 1 || L.chunk_pages > kMaxWorklistChunkPages) return cudaErrorInvalidValue;
  return launch_dependent(plan_units_kernel, dim3(1), dim3(kPlanThreads), 0, L.stream, L.seq_lens, L.max_seq_len,
                          L.B, L.n_split, L.chunk_pages, row_tiles, L.worklist);
}

}  // namespace mla
