// Tensor-core prefill (tcgen05 + TMEM + TMA): not built yet; every request takes the
// CUDA-core kernel.
#include "kernels.h"

namespace attn {
bool prefill_tc_supported(const PrefillParams&, int) { return false; }
cudaError_t launch_prefill_tc(const PrefillParams&, cudaStream_t) { return cudaErrorNotSupported; }
}  // namespace attn
