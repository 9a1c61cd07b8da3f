// tcgen05 GEMM (placeholder until the tensor-core kernel lands).
#include "launch.h"
bool gemm_tc_supported(int, int, int, long, bool, long, bool) { return false; }
cudaError_t launch_gemm_tc(int, int, int, const bf16*, long, bool, const bf16*, long, bool,
                           const EpiParams<bf16>&, int, unsigned*, cudaStream_t) {
  return cudaErrorNotSupported;
}
