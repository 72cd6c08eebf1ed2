// Tensor-core (tcgen05) GEMM: placeholder until the sm_100a kernel lands;
// every GEMM currently takes the CUDA-core path.
#include "internal.cuh"

namespace dust {

bool tc_gemm_supported(const GemmDesc&, const EpiDesc&) { return false; }

cudaError_t launch_gemm_tc(cudaStream_t, const GemmDesc&, const EpiDesc&, int) {
  return cudaErrorNotSupported;
}

}  // namespace dust
