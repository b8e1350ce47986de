// kda_fused.cuh -- the fused persistent sm_100a kernel (placeholder until it lands).
#pragma once
#include "kda_internal.h"

namespace kda {

bool fused_supported(float) { return false; }

cudaError_t launch_fused(const StagedArgs&, cudaStream_t) { return cudaErrorNotSupported; }

}  // namespace kda
