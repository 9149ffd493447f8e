// decode.cuh -- fused decode step (one token per sequence), state updated in place.
//
// Operation ("linear_attention" page: token-by-token rule on a decode step,
// cached state overwritten in place; "DeltaNet" page, "The Delta Rule":
// retrieve-and-replace form):
//     H' = alpha H;  v_old = H'^T k;  delta = beta (v - v_old)
//     H  = H' + k delta^T;            o = H^T q = alpha H^T q + (q.k) delta
// with H = S^T stored [dk, dv] fp32 (dv contiguous) per (batch, v-head).
// Per-key-channel gates (CG, g [B, Hv, dk]): H' = diag(alpha) H, so alpha_i folds
// into k_i and q_i for the two reductions and scales row i of the update.
//
// The step is bound by HBM: each (b, h) state is read once and written once
// (2 * dk * dv * 4 bytes) against ~4 dk dv flops.  One CTA owns one (b, h)
// state.  A warp covers one full 512-byte state row with 16-byte vector
// accesses (perfectly coalesced), the CTA's 8 warps cover 8 rows per pass, and
// each thread keeps its 16 x 4 state values in registers between the read and
// the write: the state touches HBM exactly twice and never goes through shared
// memory.  The two column reductions over dk (H^T k and H^T q) are per-thread
// partial sums followed by one cross-warp pass through shared memory.
#pragma once

#include "dr_common.cuh"

namespace dr {

template <int DK, int DV>
struct DecodeShape {
  static constexpr int C4 = DV / 4;                            // float4 per state row
  static constexpr int RP = (256 / C4 < DK) ? 256 / C4 : DK;   // rows covered per pass
  static constexpr int NT = C4 * RP;                           // threads per CTA
  static constexpr int RPT = DK / RP;                          // rows per thread
  static_assert(DV % 4 == 0 && DK % RP == 0, "unsupported decode shape");
};

// CG: per-key-channel gates, a compile-time switch so that the scalar-gate kernel carries
// none of its code.
template <int DK, int DV, typename Tin, typename Tout, bool CG>
__global__ void __launch_bounds__(DecodeShape<DK, DV>::NT)
    decode_step_kernel(const Tin *__restrict__ q, const Tin *__restrict__ k,
                       const Tin *__restrict__ v, const float *__restrict__ g,
                       const float *__restrict__ beta, float *__restrict__ state, int Hqk,
                       int Hv, float scale, Tout *__restrict__ o, int l2n) {
  using S = DecodeShape<DK, DV>;
  constexpr int C4 = S::C4, RP = S::RP, NT = S::NT, RPT = S::RPT;
  __shared__ float ks[DK], qs[DK], alc[CG ? DK : 1];  // alc: per-channel decay
  __shared__ float4 red_k[RP][C4], red_q[RP][C4];
  __shared__ float qk_shared, nrm[2];

  const int unit = blockIdx.x;  // b * Hv + h
  const int b = unit / Hv, h = unit - (unit / Hv) * Hv;
  const int hq = h / (Hv / Hqk);
  const int t = threadIdx.x, c4 = t % C4, r0 = t / C4;

  float4 *H = reinterpret_cast<float4 *>(state + (size_t)unit * DK * DV);
  // Issue every state load first: RPT independent 16-byte loads per thread.
  float4 hr[RPT];
#pragma unroll
  for (int i = 0; i < RPT; ++i) hr[i] = __ldcs(&H[(size_t)(r0 + i * RP) * C4 + c4]);

  const size_t qk_off = ((size_t)b * Hqk + hq) * DK;
  for (int i = t; i < DK; i += NT) {
    ks[i] = io<Tin>::ld(k + qk_off + i);
    qs[i] = scale * io<Tin>::ld(q + qk_off + i);
    if constexpr (CG) alc[i] = expf(g[(size_t)unit * DK + i]);
  }
  __syncthreads();
  if (l2n) {  // k and q (= scale q) rows divided by their norms; zero rows stay zero
    if (t < 64) {
      const float *x = (t < 32) ? ks : qs;
      float acc = 0.f;
      for (int i = t & 31; i < DK; i += 32) acc += x[i] * x[i];
      acc = warp_sum(acc);
      if ((t & 31) == 0)
        nrm[t >> 5] = acc > 0.f ? ((t < 32) ? rsqrtf(acc) : fabsf(scale) * rsqrtf(acc)) : 0.f;
    }
    __syncthreads();
    const float ik = nrm[0], iq = nrm[1];
    for (int i = t; i < DK; i += NT) {
      ks[i] *= ik;
      qs[i] *= iq;
    }
    __syncthreads();
  }
  if (t < 32) {
    float acc = 0.f;
    for (int i = t; i < DK; i += 32) acc += ks[i] * qs[i];
    acc = warp_sum(acc);
    if (t == 0) qk_shared = acc;
  }
  float4 pk = make_float4(0.f, 0.f, 0.f, 0.f), pq = pk;
#pragma unroll
  for (int i = 0; i < RPT; ++i) {
    float kr = ks[r0 + i * RP], qr = qs[r0 + i * RP];
    if constexpr (CG) {
      kr *= alc[r0 + i * RP];
      qr *= alc[r0 + i * RP];
    }
    pk.x += kr * hr[i].x; pk.y += kr * hr[i].y; pk.z += kr * hr[i].z; pk.w += kr * hr[i].w;
    pq.x += qr * hr[i].x; pq.y += qr * hr[i].y; pq.z += qr * hr[i].z; pq.w += qr * hr[i].w;
  }
  red_k[r0][c4] = pk;
  red_q[r0][c4] = pq;
  __syncthreads();
  float4 sk = make_float4(0.f, 0.f, 0.f, 0.f), sq = sk;
#pragma unroll 8
  for (int r = 0; r < RP; ++r) {
    const float4 a = red_k[r][c4], c = red_q[r][c4];
    sk.x += a.x; sk.y += a.y; sk.z += a.z; sk.w += a.w;
    sq.x += c.x; sq.y += c.y; sq.z += c.z; sq.w += c.w;
  }
  const float alpha = (g && !CG) ? expf(g[unit]) : 1.f;
  const float bt = beta[unit];
  const size_t vo = (size_t)unit * DV + 4 * c4;
  float4 d;
  d.x = bt * (io<Tin>::ld(v + vo + 0) - alpha * sk.x);
  d.y = bt * (io<Tin>::ld(v + vo + 1) - alpha * sk.y);
  d.z = bt * (io<Tin>::ld(v + vo + 2) - alpha * sk.z);
  d.w = bt * (io<Tin>::ld(v + vo + 3) - alpha * sk.w);
#pragma unroll
  for (int i = 0; i < RPT; ++i) {
    const float kr = ks[r0 + i * RP];
    float ar = alpha;
    if constexpr (CG) ar = alc[r0 + i * RP];
    float4 nh;
    nh.x = ar * hr[i].x + kr * d.x;
    nh.y = ar * hr[i].y + kr * d.y;
    nh.z = ar * hr[i].z + kr * d.z;
    nh.w = ar * hr[i].w + kr * d.w;
    __stcs(&H[(size_t)(r0 + i * RP) * C4 + c4], nh);
  }
  if (r0 == 0) {
    const float qk = qk_shared;
    io<Tout>::st(o + vo + 0, alpha * sq.x + qk * d.x);
    io<Tout>::st(o + vo + 1, alpha * sq.y + qk * d.y);
    io<Tout>::st(o + vo + 2, alpha * sq.z + qk * d.z);
    io<Tout>::st(o + vo + 3, alpha * sq.w + qk * d.w);
  }
}

template <int DK, int DV, typename Tin, typename Tout>
cudaError_t launch_decode(const void *q, const void *k, const void *v, const float *g,
                          const float *beta, float *state, int B, int Hqk, int Hv, float scale,
                          void *o, int l2n, int cg, cudaStream_t stream) {
  const unsigned units = (unsigned)B * (unsigned)Hv;
  auto kern = cg ? decode_step_kernel<DK, DV, Tin, Tout, true>
                 : decode_step_kernel<DK, DV, Tin, Tout, false>;
  kern<<<units, DecodeShape<DK, DV>::NT, 0, stream>>>(
      (const Tin *)q, (const Tin *)k, (const Tin *)v, g, beta, state, Hqk, Hv, scale, (Tout *)o,
      l2n);
  return cudaGetLastError();
}

}  // namespace dr
