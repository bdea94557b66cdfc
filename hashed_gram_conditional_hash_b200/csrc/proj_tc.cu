// Tensor-core (tcgen05) projection engine: not yet enabled in this build.
#include "engram_internal.cuh"

namespace engram {

bool tc_projection_supported(int, int, engram_dtype) { return false; }

cudaError_t launch_proj_tc(const ProjParams&, cudaStream_t) { return cudaErrorNotSupported; }

}  // namespace engram
