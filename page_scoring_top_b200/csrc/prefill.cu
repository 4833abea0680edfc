// prefill.cu -- tensor-core (tcgen05) scoring of multi-token prefill chunks.
#include "kernels.h"

namespace idx {

bool prefill_supported(int, int, int, int64_t) { return false; }

cudaError_t launch_prefill(const PrefillArgs&, int, cudaStream_t) { return cudaErrorNotSupported; }

}  // namespace idx
