// Tensor-core (tcgen05 / TMEM / TMA) path: placeholder until the kernel lands.
#include <cuda_runtime.h>

#include "llattn_internal.h"

namespace llattn {

bool tc_supports(int, int, int, int) { return false; }
size_t tc_workspace_bytes(int, int, int, int, int, int) { return 0; }
cudaError_t tc_forward(const Problem&, int, void*, cudaStream_t) { return cudaErrorNotSupported; }

}  // namespace llattn
