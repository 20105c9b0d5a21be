// tcgen05 / TMA / TMEM prefill kernel (placeholder until the kernel lands).
#include "common.cuh"

namespace sdpa15 {
bool prefill_supported(const Params&, int) { return false; }
cudaError_t launch_prefill(const Params&, int, cudaStream_t) { return cudaErrorNotSupported; }
}  // namespace sdpa15
