// chunk_tc.cuh -- tensor-core (tcgen05) chunked prefill for bf16 inputs.
#pragma once

#include "chunk_simt.cuh"

namespace dr {

inline bool tc_supported(int, int) { return false; }
inline cudaError_t tc_dispatch(int, int, bool, const PrefillArgs &, int, cudaStream_t) {
  return cudaErrorNotSupported;
}

}  // namespace dr
