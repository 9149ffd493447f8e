// layer.cuh -- the steps either side of the rule: short causal convolution + SiLU before
// it, per-head normalisation + SiLU output gate after it.
//
// "DeltaNet" (study notes, the layer diagram): the projected q/k and v each pass a
// depthwise convolution ("Conv*") and a SiLU before the rule, and the rule's output an
// RMSNorm.  "DeltaNet Attention" (class docstring, attributes norm and g_proj): the
// readout is normalised (LayerNorm) and then modulated by a SiLU-gated projection.
//
// Both steps are elementwise along the channels and bound by HBM: every input element is
// read once from HBM and every output written once.
//   conv:  y_p[c] = silu(sum_j w[c][j] x_{p-K+1+j}[c]); one thread per channel, adjacent
//          threads on adjacent channels (coalesced); the K-1 neighbouring tokens a thread
//          re-reads were just read by the same warp and come from L1.
//   norm:  one warp per (token, head) row of dv <= 128 values held in registers, two
//          (RMSNorm) or three (LayerNorm) warp reductions, the gate applied on the way out.
#pragma once

#include "dr_common.cuh"

namespace dr {

constexpr int CONV_MAX_K = 8;
constexpr int CONV_TOK = 32;  // tokens per CTA row of the convolution grid

// Sequence of flat token p (p = b*T + t; with cu_seqlens B = 1 and p = t): its index n
// and bounds [bos, eos) in flat positions.  False (and DR_ERR_SHAPE) if cu_seqlens does
// not contain p consistently.
__device__ __forceinline__ bool token_seq(const int32_t *cu, int n_seqs, int T, long long p,
                                          int &n, long long &bos, long long &eos) {
  if (cu == nullptr) {
    n = (int)(p / T);
    bos = (long long)n * T;
    eos = bos + T;
    return true;
  }
  int lo = 0, hi = n_seqs - 1;  // largest n with cu[n] <= p
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (cu[mid] <= p) lo = mid; else hi = mid - 1;
  }
  n = lo;
  bos = cu[n];
  eos = cu[n + 1];
  if (bos < 0 || bos > p || p >= eos || eos > T) {
    raise_status(DR_ERR_SHAPE);
    return false;
  }
  return true;
}

// Input of channel c at flat position s of the sequence starting at bos (s >= bos - K + 1):
// the token itself, or the carried history (oldest first), or zero.
template <typename Tin>
__device__ __forceinline__ float conv_in(const Tin *x, const float *hist, long long s,
                                         long long bos, int C, int c, int K) {
  if (s >= bos) return io<Tin>::ld(x + s * C + c);
  return hist ? hist[(int)(s - bos) + K - 1] : 0.f;
}

__device__ __forceinline__ float silu_f(float x) { return x / (1.f + expf(-x)); }

template <typename Tin, typename Tout>
__global__ void __launch_bounds__(128) conv_silu_kernel(const Tin *__restrict__ x,
                                                        const float *__restrict__ w, int K,
                                                        const float *__restrict__ state_in,
                                                        const int32_t *__restrict__ cu,
                                                        int n_seqs, int T, long long P, int C,
                                                        Tout *__restrict__ y) {
  const int c = blockIdx.y * 128 + threadIdx.x;  // grid: x = token tiles, y = channel blocks
  if (c >= C || n_seqs <= 0) return;
  float wr[CONV_MAX_K];
#pragma unroll
  for (int j = 0; j < CONV_MAX_K; ++j) wr[j] = j < K ? w[(size_t)c * K + j] : 0.f;
  const long long p0 = (long long)blockIdx.x * CONV_TOK;
  const long long p1 = p0 + CONV_TOK < P ? p0 + CONV_TOK : P;
  for (long long p = p0; p < p1; ++p) {
    int n;
    long long bos, eos;
    if (!token_seq(cu, n_seqs, T, p, n, bos, eos)) continue;
    const float *hist = state_in ? state_in + ((size_t)n * C + c) * (K - 1) : nullptr;
    float acc = 0.f;
#pragma unroll
    for (int j = 0; j < CONV_MAX_K; ++j)
      if (j < K) acc += wr[j] * conv_in(x, hist, p - K + 1 + j, bos, C, c, K);
    io<Tout>::st(y + p * C + c, silu_f(acc));
  }
}

// The last K-1 inputs of every sequence (history included for short ones), oldest first.
// All are read before any is written, so state_out may be state_in itself.
template <typename Tin>
__global__ void __launch_bounds__(128) conv_state_kernel(const Tin *__restrict__ x, int K,
                                                         const float *state_in,
                                                         const int32_t *__restrict__ cu,
                                                         int n_seqs, int N, int T, int C,
                                                         float *state_out) {
  const long long idx = (long long)blockIdx.x * 128 + threadIdx.x;
  if (idx >= (long long)N * C) return;
  const int n = (int)(idx / C), c = (int)(idx % C);
  int batch, bos_t, eos_t;
  if (!seq_bounds(cu, n, n_seqs, T, batch, bos_t, eos_t)) return;
  const long long bos = (long long)batch * T + bos_t, eos = (long long)batch * T + eos_t;
  const float *hist = state_in ? state_in + ((size_t)n * C + c) * (K - 1) : nullptr;
  float v[CONV_MAX_K - 1];
#pragma unroll
  for (int m = 0; m < CONV_MAX_K - 1; ++m)
    v[m] = m < K - 1 ? conv_in(x, hist, eos - K + 1 + m, bos, C, c, K) : 0.f;
#pragma unroll
  for (int m = 0; m < CONV_MAX_K - 1; ++m)
    if (m < K - 1) state_out[((size_t)n * C + c) * (K - 1) + m] = v[m];
}

template <typename Tin, typename Tz, typename Tout>
__global__ void __launch_bounds__(256) norm_gate_kernel(const Tin *o, const float *__restrict__ wt,
                                                        const float *__restrict__ bias,
                                                        const Tz *__restrict__ z, long long rows,
                                                        int dv, int layer, float eps, Tout *y) {
  const long long row = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const Tin *src = o + row * dv;
  float xv[4];
  float s1 = 0.f;
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int i = lane + 32 * u;
    xv[u] = i < dv ? io<Tin>::ld(src + i) : 0.f;
    s1 += xv[u];
  }
  float r, mu = 0.f;
  if (layer) {
    mu = warp_sum(s1) / (float)dv;
    float s2 = 0.f;
#pragma unroll
    for (int u = 0; u < 4; ++u)
      if (lane + 32 * u < dv) s2 += (xv[u] - mu) * (xv[u] - mu);
    r = rsqrtf(warp_sum(s2) / (float)dv + eps);
  } else {
    float s2 = 0.f;
#pragma unroll
    for (int u = 0; u < 4; ++u) s2 += xv[u] * xv[u];
    r = rsqrtf(warp_sum(s2) / (float)dv + eps);
  }
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int i = lane + 32 * u;
    if (i >= dv) continue;
    float out = (xv[u] - mu) * r * wt[i];
    if (layer && bias) out += bias[i];
    if (z) out *= silu_f(io<Tz>::ld(z + row * dv + i));
    io<Tout>::st(y + row * dv + i, out);
  }
}

}  // namespace dr
