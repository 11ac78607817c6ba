// Tensor-core (tcgen05 / TMEM / TMA) hybrid attention for bf16 on sm_100a.
#include <cuda_runtime.h>

#include "hyat_internal.h"

namespace hyat {

bool attn_tc_supported(int, int) { return false; }

cudaError_t launch_attn_tc(const AttnArgs&, int, cudaStream_t) { return cudaErrorNotSupported; }

}  // namespace hyat
