// tcgen05 (5th-generation tensor core) decode kernel for the bf16 workloads.
#pragma once

#include "common.cuh"

namespace mla {

constexpr bool kTcDecodeAvailable = false;

inline cudaError_t launch_tc_decode(const RunParams&, cudaStream_t) { return cudaErrorNotSupported; }

}  // namespace mla
