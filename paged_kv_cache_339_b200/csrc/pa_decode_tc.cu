// Tensor-core decode (placeholder until the tcgen05 kernel lands).
#include "pa_common.cuh"
#include "pa_internal.h"

namespace pa {
bool tc_supported(int, int, int) { return false; }
cudaError_t tc_num_ctas(int, int, int*) { return cudaErrorInvalidValue; }
cudaError_t launch_decode_tc(const DecodeParams&, int, cudaStream_t) { return cudaErrorInvalidValue; }
}  // namespace pa
