// Tensor-core GEMM (tcgen05): not built yet; every request takes the CUDA-core GEMM.
#include "kernels.h"

namespace attn {
bool gemm_tc_supported(int, int, int, int) { return false; }
cudaError_t launch_gemm_tc(const void*, const void*, void*, int, int, int, cudaStream_t) {
  return cudaErrorNotSupported;
}
}  // namespace attn
