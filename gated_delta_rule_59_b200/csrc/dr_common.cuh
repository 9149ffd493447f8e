// dr_common.cuh -- small device helpers shared by the delta-rule kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "dr.h"

namespace dr {

// Device status word of the library (one per device).  Kernels OR error codes
// into it (DR_ERR_SHAPE for malformed cu_seqlens, DR_ERR_TIMEOUT for a bounded
// wait that gave up); dr_get_device_status() reads and clears it.
__device__ int g_device_status;

__device__ __forceinline__ void raise_status(int code) { atomicOr(&g_device_status, 1 << code); }

template <typename T>
struct io;
template <>
struct io<float> {
  static __device__ __forceinline__ float ld(const float *p) { return *p; }
  static __device__ __forceinline__ void st(float *p, float x) { *p = x; }
};
template <>
struct io<__nv_bfloat16> {
  static __device__ __forceinline__ float ld(const __nv_bfloat16 *p) { return __bfloat162float(*p); }
  static __device__ __forceinline__ void st(__nv_bfloat16 *p, float x) { *p = __float2bfloat16_rn(x); }
};

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

// Sequence bounds of work unit n.  Returns false (and raises DR_ERR_SHAPE) when
// cu_seqlens is malformed for this sequence.
__device__ __forceinline__ bool seq_bounds(const int32_t *cu_seqlens, int n, int n_seqs, int T,
                                           int &batch, int &bos, int &eos) {
  if (cu_seqlens == nullptr) {
    batch = n;
    bos = 0;
    eos = T;
    return true;
  }
  batch = 0;
  bos = cu_seqlens[n];
  eos = cu_seqlens[n + 1];
  if (bos < 0 || eos < bos || eos > T || (n == 0 && bos != 0) || (n == n_seqs - 1 && eos != T)) {
    raise_status(DR_ERR_SHAPE);
    return false;
  }
  return true;
}

// First chunk-state row of sequence n: the number of 64-token chunks (a ragged last one
// included) of the sequences before it, a sequence of length <= 0 counting none.  Without
// cu_seqlens every sequence has T tokens.  Called by a whole, converged warp.
__device__ __forceinline__ long long chunk_row_base(const int32_t *cu_seqlens, int n, int T,
                                                    int chunk) {
  if (cu_seqlens == nullptr) return (long long)n * ((T + chunk - 1) / chunk);
  long long rows = 0;
  for (int m = (int)(threadIdx.x & 31); m < n; m += 32) {
    const long long len = (long long)cu_seqlens[m + 1] - cu_seqlens[m];
    rows += len > 0 ? (len + chunk - 1) / chunk : 0;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) rows += __shfl_xor_sync(0xffffffffu, rows, o);
  return rows;
}

}  // namespace dr
