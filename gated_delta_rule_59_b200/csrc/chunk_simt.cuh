// chunk_simt.cuh -- chunked prefill on CUDA cores, fp32 arithmetic throughout.
//
// This is the prefill kernel for fp32 inputs (its results must stay within
// 1e-4 of the fp64 oracle, which rules out TF32/bf16 tensor-core operands) and
// the path for head dimensions the tensor-core kernel does not cover.
//
// Chunk form ("Parallelizing Linear Transformers with the Delta Rule over
// Sequence Length", the chunkwise algorithm both DeltaNet pages cite, with the
// per-token decay of the "linear_attention" page folded in).  For a chunk of C
// tokens with start state H0 (= S^T, dk x dv):
//     b_r = sum_{i<=r} g_i, gamma_r = e^{b_r}, Gamma_rs = e^{b_r - b_s} (s <= r)
//     L = strict_lower(diag(beta) (Gamma * K K^T)),  T = (I + L)^-1
//     W = T diag(beta gamma) K,  U = T diag(beta) V,  Delta = U - W H0
//     O = diag(gamma) Q H0 + (Gamma * Q K^T * incl_lower) Delta
//     H = gamma_last H0 + sum_s e^{b_last - b_s} k_s Delta_s^T
// Rows past the end of a sequence are padded with q = k = v = 0, beta = 0,
// g = 0, which leaves Delta = 0 for them and changes nothing else.
//
// Per-key-channel gates (the "linear_attention" page's ChannelGates, g [.., dk]):
// b_r is a vector and the decay between tokens s <= r, diag(e^{b_r - b_s}), no
// longer factors out of the key products, so it goes inside them:
//     A_rs = sum_i k_r[i] k_s[i] e^{b_r[i] - b_s[i]},  P_rs likewise with q_r;
//     W = T diag(beta) (K o e^b),  O = (Q o e^b) H0 + P Delta,
//     H = diag(e^{b_last}) H0 + (K o e^{b_last - b})^T Delta.
// Every exponent is <= 0 for non-positive gates.
//
// One CTA owns one (sequence, v-head, dv-slice of DVS columns): the state
// columns evolve independently given k, beta and g, so slices need no
// communication; K K^T, Q K^T and T are recomputed per slice.
#pragma once

#include "dr_common.cuh"

namespace dr {

struct PrefillArgs {
  const void *q, *k, *v;
  const float *g, *beta, *state_in;
  const int32_t *cu_seqlens;
  int n_seqs, B, T, Hqk, Hv;
  float scale;
  void *o;
  float *state_out;
  int qk_l2norm;  // 1: divide q and k rows by their L2 norms first (zero rows stay zero)
  float *chunk_states;  // [rows, Hv, dk, dv] state after every 64 tokens, or null
  int channel_gates;    // 1: g is [B, T, Hv, dk], one log decay per key channel
};

// Token count between two stored chunk states (the tensor-core kernel's chunk length).
constexpr int STATE_CHUNK = DR_CHUNK;

template <int DK, int DVS, int C>
struct SimtSmem {
  static constexpr int KP = DK + 1;   // padded row pitch of K, Q, W
  static constexpr int VP = DVS + 1;  // padded row pitch of V, U, Delta, H
  static constexpr int CP = C + 1;    // padded row pitch of the C x C tiles
  static constexpr int floats =
      3 * C * KP + DK * VP + 3 * C * VP + 2 * C * CP + 4 * C;
  static constexpr size_t bytes = sizeof(float) * floats;
  // per-key-channel gates add the cumulative decays b[r][i] and K o e^b
  static constexpr size_t bytes_cg = bytes + sizeof(float) * 2 * C * KP;
};

template <int DK, int DVS, int C, typename Tin, typename Tout>
__global__ void __launch_bounds__(256) chunk_simt_kernel(PrefillArgs a, int dv) {
  using SM = SimtSmem<DK, DVS, C>;
  constexpr int KP = SM::KP, VP = SM::VP, CP = SM::CP, NT = 256;
  extern __shared__ float smem[];
  float *Ks = smem;             // [C][KP]
  float *Qs = Ks + C * KP;      // [C][KP] (scaled by `scale`)
  float *Ws = Qs + C * KP;      // [C][KP]
  float *Hs = Ws + C * KP;      // [DK][VP] running state slice
  float *Vs = Hs + DK * VP;     // [C][VP]
  float *Us = Vs + C * VP;      // [C][VP]
  float *Ds = Us + C * VP;      // [C][VP] Delta
  float *Ls = Ds + C * VP;      // [C][CP] L, then T
  float *Ps = Ls + C * CP;      // [C][CP] Gamma * Q K^T, lower incl.
  float *bs = Ps + C * CP;      // [C] cumulative log decay
  float *betas = bs + C;        // [C]
  float *bgs = betas + C;       // [C] beta * gamma
  float *ktil = bgs + C;        // [C] e^{b_last - b_s}
  float *Gb = ktil + C;         // [C][KP] channel gates: cumulative log decay b[r][i]
  float *Kb = Gb + C * KP;      // [C][KP] channel gates: K o e^{b}
  const bool cg = a.channel_gates != 0;

  const int tid = threadIdx.x;
  const int unit = blockIdx.x, n = unit / a.Hv, h = unit % a.Hv;
  const int hq = h / (a.Hv / a.Hqk);
  const int j0 = blockIdx.y * DVS;
  int batch, bos, eos;
  if (!seq_bounds(a.cu_seqlens, n, a.n_seqs, a.T, batch, bos, eos)) return;

  const Tin *q = (const Tin *)a.q, *k = (const Tin *)a.k, *v = (const Tin *)a.v;
  Tout *o = (Tout *)a.o;
  const size_t st_off = ((size_t)n * a.Hv + h) * DK * dv;

  for (int idx = tid; idx < DK * DVS; idx += NT) {
    const int i = idx / DVS, j = idx % DVS;
    Hs[i * VP + j] = a.state_in ? a.state_in[st_off + (size_t)i * dv + j0 + j] : 0.f;
  }

  const long long cbase =
      a.chunk_states ? chunk_row_base(a.cu_seqlens, n, a.T, STATE_CHUNK) : 0;

  for (int c0 = bos; c0 < eos; c0 += C) {
    const int L = min(C, eos - c0);
    __syncthreads();  // previous chunk finished with every buffer
    // ---- load the chunk (zero padded) ----
    for (int idx = tid; idx < C * DK; idx += NT) {
      const int r = idx / DK, i = idx % DK;
      float kv = 0.f, qv = 0.f;
      if (r < L) {
        const size_t off = (((size_t)batch * a.T + c0 + r) * a.Hqk + hq) * DK + i;
        kv = io<Tin>::ld(k + off);
        qv = a.scale * io<Tin>::ld(q + off);
      }
      Ks[r * KP + i] = kv;
      Qs[r * KP + i] = qv;
    }
    for (int idx = tid; idx < C * DVS; idx += NT) {
      const int r = idx / DVS, j = idx % DVS;
      Vs[r * VP + j] = r < L ? io<Tin>::ld(v + (((size_t)batch * a.T + c0 + r) * a.Hv + h) * dv + j0 + j) : 0.f;
    }
    if (a.qk_l2norm) {  // rows of K and of Q (= scale q) divided by their norms
      __syncthreads();
      const int w = tid >> 5, ln = tid & 31;
      for (int r = w; r < C; r += NT / 32) {
        float sk = 0.f, sq = 0.f;
        for (int i = ln; i < DK; i += 32) {
          sk += Ks[r * KP + i] * Ks[r * KP + i];
          sq += Qs[r * KP + i] * Qs[r * KP + i];
        }
        sk = warp_sum(sk);
        sq = warp_sum(sq);
        const float ik = sk > 0.f ? rsqrtf(sk) : 0.f;
        const float iq = sq > 0.f ? fabsf(a.scale) * rsqrtf(sq) : 0.f;  // |scale| / |scale q|
        for (int i = ln; i < DK; i += 32) {
          Ks[r * KP + i] *= ik;
          Qs[r * KP + i] *= iq;
        }
      }
    }
    if (cg) {
      // per-key-channel gates: b[r][i] = sum of g over the chunk's rows <= r, per channel
      for (int idx = tid; idx < C * DK; idx += NT) {
        const int r = idx / DK, i = idx % DK;
        Gb[r * KP + i] =
            r < L ? a.g[(((size_t)batch * a.T + c0 + r) * a.Hv + h) * DK + i] : 0.f;
      }
      __syncthreads();
      for (int i = tid; i < DK; i += NT) {
        float acc = 0.f;
        for (int r = 0; r < C; ++r) {
          acc += Gb[r * KP + i];
          Gb[r * KP + i] = acc;
        }
      }
    }
    if (tid < 32) {
      // inclusive prefix sum of g over the chunk (C <= 32 handled per lane); with channel
      // gates the scalar decay is 1 and b lives in Gb
      for (int base = 0; base < C; base += 32) {
        const int r = base + tid;
        float gv = 0.f, bv = 0.f;
        if (r < L) {
          const size_t go = ((size_t)batch * a.T + c0 + r) * a.Hv + h;
          gv = (a.g && !cg) ? a.g[go] : 0.f;
          bv = a.beta[go];
        }
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
          const float y = __shfl_up_sync(0xffffffffu, gv, off);
          if (tid >= off) gv += y;
        }
        const float carry = base > 0 ? bs[base - 1] : 0.f;
        if (r < C) {
          bs[r] = gv + carry;
          betas[r] = bv;
        }
        __syncwarp();
      }
    }
    __syncthreads();
    const float blast = bs[C - 1];
    if (tid < C) {
      bgs[tid] = betas[tid] * expf(bs[tid]);
      ktil[tid] = expf(blast - bs[tid]);
    }
    // ---- L = strict_lower(beta Gamma K K^T), P = lower(Gamma Q K^T) ----
    for (int idx = tid; idx < C * C; idx += NT) {
      const int r = idx / C, s = idx % C;
      float lv = 0.f, pv = 0.f;
      if (s <= r) {
        float akk = 0.f, aqk = 0.f;
        if (cg) {  // the decay between s and r differs per channel: inside the sums
          for (int i = 0; i < DK; ++i) {
            const float ks_ = Ks[s * KP + i] * expf(Gb[r * KP + i] - Gb[s * KP + i]);
            akk += Ks[r * KP + i] * ks_;
            aqk += Qs[r * KP + i] * ks_;
          }
        } else {
          for (int i = 0; i < DK; ++i) {
            const float ks_ = Ks[s * KP + i];
            akk += Ks[r * KP + i] * ks_;
            aqk += Qs[r * KP + i] * ks_;
          }
        }
        const float gam = expf(bs[r] - bs[s]);
        pv = gam * aqk;
        if (s < r) lv = betas[r] * gam * akk;
      }
      Ls[r * CP + s] = lv;
      Ps[r * CP + s] = pv;
    }
    __syncthreads();
    // ---- T = (I + L)^-1 by forward substitution, one column per thread ----
    if (tid < C) {
      const int c = tid;
      float col[C];
#pragma unroll
      for (int r = 0; r < C; ++r) col[r] = (r == c) ? 1.f : 0.f;
#pragma unroll
      for (int r = 1; r < C; ++r) {
        float acc = 0.f;
#pragma unroll
        for (int s = 0; s < r; ++s) acc += Ls[r * CP + s] * col[s];
        if (r > c) col[r] = -acc;
      }
      __syncwarp();
      // every lane has read all of L: overwrite it with T column by column
#pragma unroll
      for (int r = 0; r < C; ++r) Ls[r * CP + c] = col[r];
    }
    __syncthreads();
    if (cg) {
      // K -> K o e^{b} (into Kb, for W), K -> K o e^{b_last - b} (in place, for the state),
      // Q -> Q o e^{b} (in place, for the read of H0)
      for (int idx = tid; idx < C * DK; idx += NT) {
        const int r = idx / DK, i = idx % DK;
        const float b = Gb[r * KP + i], kv = Ks[r * KP + i];
        Kb[r * KP + i] = kv * expf(b);
        Ks[r * KP + i] = kv * expf(Gb[(C - 1) * KP + i] - b);
        Qs[r * KP + i] *= expf(b);
      }
      __syncthreads();
    }
    float *Ts = Ls;
    const float *Kw = cg ? Kb : Ks;
    // ---- W = T diag(beta gamma) K, U = T diag(beta) V ----
    for (int idx = tid; idx < C * DK; idx += NT) {
      const int r = idx / DK, i = idx % DK;
      float acc = 0.f;
      for (int s = 0; s <= r; ++s) acc += Ts[r * CP + s] * bgs[s] * Kw[s * KP + i];
      Ws[r * KP + i] = acc;
    }
    for (int idx = tid; idx < C * DVS; idx += NT) {
      const int r = idx / DVS, j = idx % DVS;
      float acc = 0.f;
      for (int s = 0; s <= r; ++s) acc += Ts[r * CP + s] * betas[s] * Vs[s * VP + j];
      Us[r * VP + j] = acc;
    }
    __syncthreads();
    // ---- Delta = U - W H0 ----
    for (int idx = tid; idx < C * DVS; idx += NT) {
      const int r = idx / DVS, j = idx % DVS;
      float acc = 0.f;
      for (int i = 0; i < DK; ++i) acc += Ws[r * KP + i] * Hs[i * VP + j];
      Ds[r * VP + j] = Us[r * VP + j] - acc;
    }
    __syncthreads();
    // ---- O = diag(gamma) Q H0 + P Delta  (reads H0: before the state update) ----
    for (int idx = tid; idx < C * DVS; idx += NT) {
      const int r = idx / DVS, j = idx % DVS;
      if (r >= L) continue;
      float acc = 0.f;
      for (int i = 0; i < DK; ++i) acc += Qs[r * KP + i] * Hs[i * VP + j];
      float acc2 = 0.f;
      for (int s = 0; s <= r; ++s) acc2 += Ps[r * CP + s] * Ds[s * VP + j];
      const float out = expf(bs[r]) * acc + acc2;
      io<Tout>::st(o + (((size_t)batch * a.T + c0 + r) * a.Hv + h) * dv + j0 + j, out);
    }
    __syncthreads();
    // ---- H = gamma_last H0 + Ktil^T Delta; stored too at a 64-token boundary ----
    const float glast = expf(blast);
    const bool keep = a.chunk_states && ((c0 + L - bos) % STATE_CHUNK == 0 || c0 + L == eos);
    float *hc = keep ? a.chunk_states +
                           ((size_t)(cbase + (c0 - bos) / STATE_CHUNK) * a.Hv + h) * DK * dv + j0
                     : nullptr;
    for (int idx = tid; idx < DK * DVS; idx += NT) {
      const int i = idx / DVS, j = idx % DVS;
      float acc = 0.f;
      for (int s = 0; s < C; ++s) acc += ktil[s] * Ks[s * KP + i] * Ds[s * VP + j];
      const float gl = cg ? expf(Gb[(C - 1) * KP + i]) : glast;
      const float hn = gl * Hs[i * VP + j] + acc;
      Hs[i * VP + j] = hn;
      if (keep) hc[(size_t)i * dv + j] = hn;
    }
  }
  __syncthreads();
  if (a.state_out) {
    for (int idx = tid; idx < DK * DVS; idx += NT) {
      const int i = idx / DVS, j = idx % DVS;
      a.state_out[st_off + (size_t)i * dv + j0 + j] = Hs[i * VP + j];
    }
  }
}

template <int DK, int DV, typename Tin, typename Tout>
cudaError_t launch_chunk_simt(const PrefillArgs &a, int N, cudaStream_t stream) {
  constexpr int DVS = DV < 32 ? DV : 32;
  constexpr int C = 32;
  static_assert(STATE_CHUNK % C == 0, "chunk states are taken at chunk ends");
  using SM = SimtSmem<DK, DVS, C>;
  auto kern = chunk_simt_kernel<DK, DVS, C, Tin, Tout>;
  const size_t smem = a.channel_gates ? SM::bytes_cg : SM::bytes;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid((unsigned)N * (unsigned)a.Hv, DV / DVS);
  kern<<<grid, 256, smem, stream>>>(a, DV);
  return cudaGetLastError();
}

}  // namespace dr
