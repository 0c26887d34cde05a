// Tensor-core expert path (placeholder until the tcgen05 kernels land).
#include "prefill.h"

namespace jmoe {
bool prefill_available() { return false; }
cudaError_t launch_prefill(const PrefillArgs&, cudaStream_t) { return cudaErrorNotSupported; }
}  // namespace jmoe
