// Tensor-core (tcgen05 / TMEM) decode kernel for sm_100a.
#include "mla_common.cuh"
#include "mla_internal.h"

namespace mla {

cudaError_t launch_decode_tc(const DecodeLaunch&) { return cudaErrorNotSupported; }

}  // namespace mla
