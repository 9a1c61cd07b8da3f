// bf16 tensor-core attention (placeholder until the kernel lands).
#include "launch.h"
bool attn_mma_supported(int) { return false; }
cudaError_t launch_attn_fwd_mma(const bf16*, bf16*, float*, const int*, int, int, int, int, cudaStream_t) {
  return cudaErrorNotSupported;
}
cudaError_t launch_attn_bwd_mma(const bf16*, const bf16*, const bf16*, const float*, float*, const int*, bf16*,
                                int, int, int, int, cudaStream_t) {
  return cudaErrorNotSupported;
}
