// chunk_pair.cuh -- the tensor-core chunked prefill on a CTA pair (a thread-block cluster
// of two CTAs on two SMs) for bf16 inputs, dk = dv = 128.
//
// The chunk algebra is the one of chunk_tc.cuh (UT/WY form of the delta rule with the
// per-token decay folded in; every product a tcgen05.mma with M = 128 in the transposed
// orientation).  What changes is the split of the work.  Per chunk it has two parts:
//   state-independent ("prep"): G = [K;Q] K^T, L, T = (I + L)^-1, T diag(beta),
//       T diag(beta gamma), W^T = K^T (T diag(beta gamma))^T, P = Gamma * Q K^T (masked);
//   state-dependent ("state"): U^T = V^T (T diag(beta))^T, Delta^T = U^T + H0^T (-W^T),
//       O^T = diag(gamma) H0^T Q^T + Delta^T P^T, H = gamma_C H0 + Delta~^T K.
// Only the state part is sequential over chunks; on one SM the prep part, being mostly
// CUDA-core work (the triangular inverse), was the longer of the two.  Here:
//   CTA rank 0 (prep): two prep instances (warpgroups 1 and 2) work on alternate chunks
//       at the same time, fed by one TMA producer warp (a ring of 3 K/Q stages) and one
//       MMA issuer warp.  In an instance two warps build L and then T = (I + L)^-1 one
//       column per thread by forward substitution in registers (no barriers, broadcast
//       shared loads), writing T diag(beta) and T diag(beta gamma) straight into their
//       operand tiles, while the other two build P.  (The second instance's Gram MMA is
//       [Q;K] K^T, so the two instances' serial warps sit on different SM sub-partitions.)
//       A shipper warp sends T diag(beta) | P (32 KB) and -W^T (16 KB) per chunk into the
//       partner's shared memory with bulk copies over the cluster's distributed shared
//       memory, completing on the partner's mbarriers.
//   CTA rank 1 (state): TMA producer (K/Q and V, two stages), MMA issuer, gates warp,
//       a courier warp that acknowledges landed copies to the prep CTA;
//       warpgroups 1-2 hold the fp32 master state in registers and run the chain
//       Delta epilogue -> state update; warpgroup 3 writes the outputs off the chain.
//       Delta^T and Delta~^T (bf16 hi/lo pairs) go to tensor memory and are the A operand
//       of their two MMAs, so shared memory holds two stages of every input.
// Cross-CTA signals: the copies' complete_tx on the state CTA's barriers; relaxed remote
// mbarrier arrives back to the prep CTA when a copy has landed (its source may be reused)
// and when the state CTA has finished with an incoming slot.
#pragma once

#include "chunk_tc.cuh"

namespace dr {
namespace tcp {

using tck::C;
using tck::DK;
using tck::DV;
using tck::LOG2E;
constexpr int NT = 512;

// ---- shared memory (bytes from a 1024-aligned base) ----
constexpr uint32_t KQ_BYTES = 32768;  // K0 Q0 K1 Q1 boxes of 8 KB ([K;Q] for k < 64, then k >= 64)
constexpr uint32_t KQ_K0 = 0, KQ_Q0 = 8192;
// prep CTA
constexpr uint32_t P_NKQ = 3;                   // K/Q ring stages
constexpr uint32_t P_OFF_WA = P_NKQ * KQ_BYTES; // two instance work areas
constexpr uint32_t WA_BYTES = 49152;
constexpr uint32_t WA_LT = 0;      // L^T fp32 [64][64]       -> T diag(beta) hi | lo (shipped)
constexpr uint32_t WA_T = 16384;   // P hi | lo (shipped)
constexpr uint32_t WA_X = 32768;   // merge scratch -> T diag(beta gamma) hi | lo -> -W^T (shipped)
constexpr uint32_t P_OFF_TF = P_OFF_WA + 2 * WA_BYTES;  // per instance: T fp32 [64][64]
constexpr uint32_t TF_BYTES = 64 * 64 * 4;
constexpr uint32_t P_OFF_GATES = P_OFF_TF + 2 * TF_BYTES;  // 2 slots x {bs2, beta, gam}[64]
// state CTA
constexpr uint32_t S_OFF_QK = 0;                      // two K/Q stages (outputs staged over them)
constexpr uint32_t V_BYTES = 16384;
constexpr uint32_t S_OFF_V = 2 * KQ_BYTES;            // two V stages
constexpr uint32_t S_OFF_IN = S_OFF_V + 2 * V_BYTES;  // two incoming slots
constexpr uint32_t IN_BYTES = 49152, IN_A_BYTES = 32768, IN_W = 32768, IN_W_BYTES = 16384;
constexpr uint32_t S_OFF_GATES = S_OFF_IN + 2 * IN_BYTES;  // 2 slots x {bs2, beta, gam, dtil}[64]
// both: the barrier block sits at the same offset in the two CTAs (remote arrives address it)
constexpr uint32_t OFF_BARS = P_OFF_GATES + 2 * 768;
constexpr uint32_t SMEM_BYTES = OFF_BARS + 512 + 1024;  // + alignment slack
static_assert(S_OFF_GATES + 2 * 1024 <= OFF_BARS, "state shared memory");
static_assert(SMEM_BYTES <= 232448, "shared memory budget");

// ---- TMEM columns ----
constexpr uint32_t P_TMEM_COLS = 256;  // prep: instance i: G at 128 i, W^T at 128 i + 64
constexpr uint32_t COL_DU = 0, COL_OA = 64, COL_OB = 128, COL_HU = 192, COL_H0 = 320;
constexpr uint32_t COL_DH = 384, COL_DL = 416, COL_DTH = 448, COL_DTL = 480;
constexpr uint32_t S_TMEM_COLS = 512;

// ---- mbarriers (one array at the same offset in both CTAs; each CTA initialises its range) ----
enum Bar {
  // prep CTA
  P_KQ_FULL = 0,      // [3] TMA -> issuer
  P_KQ_EMPTY = 3,     // [3] issuer (after W) -> TMA
  P_GATE_FULL = 6,    // [2] gates warp -> instance
  P_GATE_EMPTY = 8,   // [2] instance (4 warps) -> gates warp
  P_G_FULL = 10,      // [2] issuer -> instance
  P_G_EMPTY = 12,     // [2] instance -> issuer
  P_TBG_FULL = 14,    // [2] instance (4 warps) -> issuer (T diag(beta gamma) ready)
  P_W_FULL = 16,      // [2] issuer -> instance
  P_W_EMPTY = 18,     // [2] instance -> issuer
  P_IN_EMPTY = 20,    // [2] state CTA (remote) -> instance: the incoming slot is free
  P_INA_READ = 22,    // [2] state CTA (remote): T diag(beta) | P has landed
  P_INW_READ = 24,    // [2] state CTA (remote): -W^T has landed
  P_SHIP_A = 26,      // [2] instance (4 warps) -> shipper: T diag(beta) | P written
  P_SHIP_W = 28,      // [2] instance (4 warps) -> shipper: -W^T written
  // state CTA
  S_QK_FULL = 32,     // [2]
  S_QK_EMPTY = 34,    // [2] output warps (after the staged store left) -> TMA
  S_V_FULL = 36,      // [2]
  S_V_EMPTY = 38,     // [2] issuer (after U) -> TMA
  S_GATE_FULL = 40,   // [2]
  S_GATE_EMPTY = 42,  // [2] state (8 warps) + output (4 warps)
  S_INA_FULL = 44,    // [2] prep CTA copies (complete_tx) -> issuer
  S_INW_FULL = 46,    // [2]
  S_H0_FULL = 48,     // state (8) -> issuer
  S_DMMA_FULL = 49,   // issuer -> state
  S_D_FULL = 50,      // state (8) -> issuer
  S_H_FULL = 51,      // issuer -> state
  S_OB_FULL = 52,     // issuer -> output
  S_OA_EMPTY = 53,    // output (4) -> issuer
  NUM_BARS = 54
};

// Per-chunk gate terms of one (sequence, head): with b = cumsum(g) over the chunk,
// bs2 = b log2(e), beta, gam = e^b, dtil = e^{b_C - b}.  Tokens past the end of the
// sequence get g = beta = 0 (so they change nothing).  One warp.
__device__ __forceinline__ void chunk_gates(const PrefillArgs &a, float *gs, int zbase, int t0,
                                            int L, int h, int lane, bool with_dtil) {
  float g0 = 0.f, g1 = 0.f, b0 = 0.f, b1 = 0.f;
  const size_t i0 = ((size_t)zbase + t0 + lane) * a.Hv + h;
  if (lane < L) {
    g0 = a.g ? a.g[i0] : 0.f;
    b0 = a.beta[i0];
  }
  if (lane + 32 < L) {
    g1 = a.g ? a.g[i0 + (size_t)32 * a.Hv] : 0.f;
    b1 = a.beta[i0 + (size_t)32 * a.Hv];
  }
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const float y0 = __shfl_up_sync(0xffffffffu, g0, off);
    const float y1 = __shfl_up_sync(0xffffffffu, g1, off);
    if (lane >= off) {
      g0 += y0;
      g1 += y1;
    }
  }
  g1 += __shfl_sync(0xffffffffu, g0, 31);
  const float blast = __shfl_sync(0xffffffffu, g1, 31);
  gs[lane] = g0 * LOG2E;
  gs[lane + 32] = g1 * LOG2E;
  gs[64 + lane] = b0;
  gs[96 + lane] = b1;
  gs[128 + lane] = tc::ex2(g0 * LOG2E);
  gs[160 + lane] = tc::ex2(g1 * LOG2E);
  if (with_dtil) {
    gs[192 + lane] = tc::ex2((blast - g0) * LOG2E);
    gs[224 + lane] = tc::ex2((blast - g1) * LOG2E);
  }
}

// Sum of squares of row r of a 64 x 128 bf16 operand held as two 128-byte-swizzled boxes of
// 64 columns (box0, box0 + 16384), e.g. one K or Q tile of a chunk.
__device__ __forceinline__ float row_sumsq(uint32_t box0, int r) {
  float acc = 0.f;
#pragma unroll
  for (int b = 0; b < 2; ++b) {
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const uint4 w = tc::ld_shared_v4(box0 + 16384u * b + tc::sw128_off(r, j));
      const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const float lo = __uint_as_float(ws[t] << 16), hi = __uint_as_float(ws[t] & 0xffff0000u);
        acc = fmaf(lo, lo, acc);
        acc = fmaf(hi, hi, acc);
      }
    }
  }
  return acc;
}
__device__ __forceinline__ float inv_norm(float sumsq) { return sumsq > 0.f ? rsqrtf(sumsq) : 0.f; }

__device__ __forceinline__ void split2(float x0, float x1, uint32_t &hi, uint32_t &lo) {
  const float h0 = __bfloat162float(__float2bfloat16_rn(x0));
  const float h1 = __bfloat162float(__float2bfloat16_rn(x1));
  hi = tc::pack_bf16(h0, h1);
  lo = tc::pack_bf16(x0 - h0, x1 - h1);
}

static_assert(C == STATE_CHUNK, "one stored state per chunk");

// L2N: q and k rows are L2-normalised first; CS: the state after every chunk is stored to
// a.chunk_states.  Both are compile-time switches, so that the plain path carries none of
// their code.
template <bool OUT_F32, bool L2N, bool CS>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(NT, 1)
    chunk_pair_kernel(const __grid_constant__ CUtensorMap tm_q,
                      const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v,
                      const __grid_constant__ CUtensorMap tm_o, PrefillArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // Align by offsetting the shared array itself (not through an integer cast), so that every
  // pointer derived from it stays in the shared address space: plain LDS/STS, not generic
  // loads and stores.
  uint8_t *smem = smem_raw + ((1024u - (tc::smem_u32(smem_raw) & 1023u)) & 1023u);
  const uint32_t sb = tc::smem_u32(smem);
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + OFF_BARS);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + NUM_BARS);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
  auto bar = [&](int i) { return tc::smem_u32(&bars[i]); };

  const uint32_t rank = tc::cluster_rank();  // 0: prep, 1: state
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int wg = warp >> 2, q4 = warp & 3;
  const int row = 32 * q4 + lane;  // TMEM lane this thread reads
  const uint32_t lane_off = (uint32_t)(32 * q4) << 16;

  const int unit = blockIdx.x >> 1, n = unit / a.Hv, h = unit % a.Hv;
  const int hq = h / (a.Hv / a.Hqk);
  int batch, bos, eos;
  // same decision in both CTAs of the pair, taken before any cluster barrier
  if (!seq_bounds(a.cu_seqlens, n, a.n_seqs, a.T, batch, bos, eos)) return;
  const int nchunks = (eos - bos + C - 1) / C;
  const int zbase = batch * a.T;
  const size_t st_off = ((size_t)n * a.Hv + h) * DK * DV;
  const uint32_t tmem_cols = rank == 0 ? P_TMEM_COLS : S_TMEM_COLS;

  if (tid == 0) {
    // arrival counts: 1 = one thread (TMA expect_tx, tcgen05.commit, copy expect_tx or a
    // remote arrive), else one elected lane per warp of the signalling group
    static constexpr uint8_t pc[30] = {1, 1, 1, 1, 1, 1, 1, 1, 4, 4, 1, 1, 4, 4, 4,
                                       4, 1, 1, 4, 4, 1, 1, 1, 1, 1, 1, 4, 4, 4, 4};
    static constexpr uint8_t sc[22] = {1, 1, 1, 1, 1, 1, 1, 1, 1, 1, 12,
                                       12, 1, 1, 1, 1, 8, 1, 8, 1, 1, 4};
    if (rank == 0)
      for (int i = 0; i < 30; ++i) tc::mbar_init(bar(i), pc[i]);
    else
      for (int i = 0; i < 22; ++i) tc::mbar_init(bar(32 + i), sc[i]);
    *abort_flag = 0;
    tc::fence_barrier_init();
  }
  if (warp == 0) {
    tc::tmem_alloc(tc::smem_u32(tmem_slot), tmem_cols);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncwarp();
  __syncthreads();
  tc::tc_fence_after();
  tc::cluster_sync();  // both CTAs' barriers exist before any remote arrive or copy
  const uint32_t tmem = *tmem_slot;

  auto wait = [&](int i, uint32_t parity) { tc::mbar_wait(bar(i), parity, abort_flag); };
  // Producers and gates poll too: a thread suspended in try_wait was measured to resume up to
  // ~1 us after the phase completed, and the gates of a chunk are on its instance's path.
  auto wait_sleep = [&](int i, uint32_t parity) { tc::mbar_wait(bar(i), parity, abort_flag); };
  // Phases completed from the partner CTA are polled at CTA scope too: incoming operands are
  // made visible by the copies' complete_tx (as for any bulk or TMA copy), and the partner's
  // acknowledgements publish no data.  (Cluster-scope acquire polls measured slower.)
  auto wait_cl = [&](int i, uint32_t parity) { tc::mbar_wait(bar(i), parity, abort_flag); };
  // Loops of several threads never leave on the abort flag (threads could read it at
  // different times and part at a named barrier); after an abort every wait returns at once.
  auto role_wait = [&](int i, uint32_t parity, bool leader, uint32_t bar_id, uint32_t nthreads) {
    if (leader) tc::mbar_wait(bar(i), parity, abort_flag);
    tc::named_bar(bar_id, nthreads);
  };
  auto adv = [](uint64_t d, uint32_t bytes) { return d + (uint64_t)(bytes >> 4); };

  // Warpgroup 3 of the prep CTA has no role.
  if (rank == 0) {
    // ================================================================ prep CTA
    if (warp == 0) {
      // ------------------------------------------------ TMA producer: K/Q ring of 3
      if (lane == 0 && nchunks > 0) {
        tc::prefetch_tmap(&tm_q);
        tc::prefetch_tmap(&tm_k);
        for (int c = 0; c < nchunks; ++c) {
          const uint32_t r = (uint32_t)c % P_NKQ, u = (uint32_t)c / P_NKQ;
          const int z = zbase + bos + c * C;
          if (c >= (int)P_NKQ) wait_sleep(P_KQ_EMPTY + r, (u - 1) & 1u);
          if (*abort_flag) break;
          // even chunks: K0 Q0 K1 Q1 (G = [K;Q] K^T), odd chunks: Q0 K0 Q1 K1 (G = [Q;K] K^T)
          const uint32_t dst = sb + r * KQ_BYTES, ko = (c & 1) ? 8192u : 0u, qo = 8192u - ko;
          tc::mbar_arrive_expect_tx(bar(P_KQ_FULL + r), KQ_BYTES);
          tc::tma_load_3d(dst + ko, &tm_k, bar(P_KQ_FULL + r), 0, hq, z);
          tc::tma_load_3d(dst + ko + 16384, &tm_k, bar(P_KQ_FULL + r), 64, hq, z);
          tc::tma_load_3d(dst + qo, &tm_q, bar(P_KQ_FULL + r), 0, hq, z);
          tc::tma_load_3d(dst + qo + 16384, &tm_q, bar(P_KQ_FULL + r), 64, hq, z);
        }
      }
    } else if (warp == 1) {
      // ------------------------------------------------ MMA issuer: G and W^T per chunk
      if (lane == 0 && nchunks > 0) {
        const uint64_t dKQ = tc::sdesc_sw128(sb, 16, 1024);      // [K;Q] / [Q;K], K (K-major)
        const uint64_t dKmn = tc::sdesc_sw128(sb, 16384, 1024);  // K as K^T (MN-major A)
        const uint64_t dTBG0 = tc::sdesc_sw128(sb + P_OFF_WA + WA_X, 16, 1024);
        auto issue_G = [&](int c) {
          const uint32_t r = (uint32_t)c % P_NKQ, u = (uint32_t)c / P_NKQ;
          const int pi = c & 1, it = c >> 1;
          wait(P_KQ_FULL + r, u & 1u);
          if (it > 0) wait(P_G_EMPTY + pi, (uint32_t)(it - 1) & 1u);
          if (*abort_flag) return;
          tc::tc_fence_after();
          const uint64_t d0 = adv(dKQ, r * KQ_BYTES);
          const uint32_t ko = pi ? 8192u : 0u;  // K box of this chunk's stage
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t o = (kk >> 2) * 16384u + (kk & 3) * 32u;
            tc::mma_bf16(tmem + 128 * pi, adv(d0, o), adv(d0, ko + o), tck::ID_G, kk > 0);
          }
          tc::mma_commit(bar(P_G_FULL + pi));
        };
        auto issue_W = [&](int c) {
          const uint32_t r = (uint32_t)c % P_NKQ;
          const int pi = c & 1, it = c >> 1;
          wait(P_TBG_FULL + pi, (uint32_t)it & 1u);
          if (it > 0) wait(P_W_EMPTY + pi, (uint32_t)(it - 1) & 1u);
          if (*abort_flag) return;
          tc::tc_fence_after();
          const uint64_t dk = adv(dKmn, r * KQ_BYTES + (pi ? 8192u : 0u));
          const uint64_t dt = adv(dTBG0, (uint32_t)pi * WA_BYTES);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t ak = adv(dk, kk * 2048u);
            tc::mma_bf16(tmem + 128 * pi + 64, ak, adv(dt, kk * 32u), tck::ID_MNK, kk > 0);
            tc::mma_bf16(tmem + 128 * pi + 64, ak, adv(dt, 8192u + kk * 32u), tck::ID_MNK, 1);
          }
          tc::mma_commit(bar(P_W_FULL + pi));
          tc::mma_commit(bar(P_KQ_EMPTY + r));
        };
        issue_G(0);
        if (nchunks > 1) issue_G(1);
        for (int c = 0; c < nchunks && !*abort_flag; ++c) {
          issue_W(c);
          if (c + 2 < nchunks) issue_G(c + 2);
        }
      }
    } else if (warp == 2) {
      // ------------------------------------------------ gates
      for (int c = 0; c < nchunks; ++c) {
        const int s = c & 1, t0 = bos + c * C;
        if (c >= 2) {
          if (lane == 0) wait_sleep(P_GATE_EMPTY + s, ((uint32_t)(c - 2) >> 1) & 1u);
          __syncwarp();
        }
        chunk_gates(a, reinterpret_cast<float *>(smem + P_OFF_GATES) + 192 * s, zbase, t0,
                    min(C, eos - t0), h, lane, false);
        tck::warp_arrive(bar(P_GATE_FULL + s), lane);
      }
    } else if (warp == 3) {
      // ------------------------------------------------ shipper: operand copies, in chunk order
      if (lane == 0 && nchunks > 0) {
        for (int c = 0; c < nchunks; ++c) {
          const int pi = c & 1, it = c >> 1;
          const uint32_t wa = sb + P_OFF_WA + (uint32_t)pi * WA_BYTES;
          const uint32_t rIN = tc::mapa(sb + S_OFF_IN + (uint32_t)pi * IN_BYTES, 1);
          wait(P_SHIP_A + pi, (uint32_t)it & 1u);
          if (it > 0) wait_cl(P_IN_EMPTY + pi, (uint32_t)(it - 1) & 1u);  // the slot is free
          if (*abort_flag) break;
          const uint32_t rINA = tc::mapa(bar(S_INA_FULL + pi), 1);
          tc::mbar_expect_tx_remote_relaxed(rINA, IN_A_BYTES);
          tc::bulk_copy_to_cluster(rIN, wa + WA_LT, IN_A_BYTES, rINA);
          wait(P_SHIP_W + pi, (uint32_t)it & 1u);
          if (*abort_flag) break;
          const uint32_t rINW = tc::mapa(bar(S_INW_FULL + pi), 1);
          tc::mbar_expect_tx_remote_relaxed(rINW, IN_W_BYTES);
          tc::bulk_copy_to_cluster(rIN + IN_W, wa + WA_X, IN_W_BYTES, rINW);
        }
      }
    } else if (wg == 1 || wg == 2) {
      // ------------------------------------------------ prep instance pi: chunks c = pi mod 2
      const int pi = wg - 1, pt = tid - 128 * wg;  // pt: 0..127
      const uint32_t nb = 1 + (uint32_t)pi;        // named barrier of the instance (128)
      const uint32_t nbL = 3 + (uint32_t)pi;       // named barrier of its two L warps (64)
      const uint32_t nbP = 5 + (uint32_t)pi;       // named barrier of its two P warps (64)
      const uint32_t wa = sb + P_OFF_WA + (uint32_t)pi * WA_BYTES;
      float *LT = reinterpret_cast<float *>(smem + P_OFF_WA + pi * WA_BYTES + WA_LT);
      float *Tf = reinterpret_cast<float *>(smem + P_OFF_TF + pi * TF_BYTES);  // T, row-major
      float *Xs = reinterpret_cast<float *>(smem + P_OFF_WA + pi * WA_BYTES + WA_X);  // scratch
      float *TDT = Xs + 512;  // diagonal blocks of T transposed [4][16 m][16 r]
      float *gsm = reinterpret_cast<float *>(smem + P_OFF_GATES) + 192 * pi;
      const float *gs = gsm;
      const uint32_t colG = 128u * (uint32_t)pi, colW = colG + 64;
      // G rows 0-63 are K K^T for instance 0 and Q K^T for instance 1: the warps on the
      // TMEM lanes of the K K^T rows build L and T, the other two build P.
      const bool lrole = (q4 >> 1) == pi;
      const int rr = row & 63;  // the chunk row (token) of this thread: an L/P row, a T column
      int it = 0;
      for (int c = pi; c < nchunks; c += 2, ++it) {
        const uint32_t ph = (uint32_t)it & 1u, pph = (uint32_t)(it - 1) & 1u;
        if (pt == 0) {
          if (it > 0) wait_cl(P_INA_READ + pi, pph);  // L^T and P regions: last copy has landed
          wait(P_GATE_FULL + pi, ph);
        }
        role_wait(P_G_FULL + pi, ph, pt == 0, nb, 128);
        tc::tc_fence_after();
        // this thread's row of G: a row of K K^T (L warps) or of Q K^T (P warps)
        uint32_t u0[32], u1[32];
        tc::tmem_ld32_nw(tmem + lane_off + colG, u0);
        tc::tmem_ld32_nw(tmem + lane_off + colG + 32, u1);
        tc::tmem_wait_ld();
        tc::reg_fence(u0);
        tc::reg_fence(u1);
        // q/k L2 normalisation as exact fp32 scalings: L and P take 1/|k_s| per column and
        // 1/|k_r| or 1/|q_r| per row; T diag(beta gamma) takes 1/|k_s| per column (W = T
        // diag(beta gamma) K^).  |k_r|^2 is the diagonal of K K^T; the column factors are
        // exchanged through the diagonal of L^T, which is never read as L.
        float rinv = 1.f;
        if constexpr (L2N) {
          if (lrole) {
            float d = 0.f;
#pragma unroll
            for (int t = 0; t < 32; ++t) {
              if (t == rr) d = __uint_as_float(u0[t]);
              if (t + 32 == rr) d = __uint_as_float(u1[t]);
            }
            rinv = inv_norm(d);
            LT[rr * 65] = rinv;
            gsm[128 + rr] *= rinv;
          } else {
            if (rr == 0) wait(P_KQ_FULL + (c % (int)P_NKQ), ((uint32_t)c / P_NKQ) & 1u);
            tc::named_bar(nbP, 64);  // the Q tile of this chunk is visible to every P thread
            const uint32_t qbox = sb + ((uint32_t)c % P_NKQ) * KQ_BYTES + ((c & 1) ? 0u : 8192u);
            rinv = inv_norm(row_sumsq(qbox, rr));
          }
          tc::named_bar(nb, 128);  // every 1/|k_s| is on the diagonal of L^T
        }
        if (lrole) {
          // ---- L^T[s][r] = L_rs = beta_r Gamma_rs (k_r . k_s), s < r; r = this thread ----
          {
            const float br = gs[rr], bt = gs[64 + rr] * rinv;
#pragma unroll
            for (int q = 0; q < 16; ++q) {
              const float4 b4 = reinterpret_cast<const float4 *>(gs)[q];
              const float bs[4] = {b4.x, b4.y, b4.z, b4.w};
#pragma unroll
              for (int t = 0; t < 4; ++t) {
                const int s_ = 4 * q + t;
                const float kk = __uint_as_float(s_ < 32 ? u0[s_ & 31] : u1[s_ & 31]);
                const float cs = L2N ? LT[s_ * 65] : 1.f;
                LT[s_ * 64 + rr] = (s_ < rr) ? bt * tc::ex2(br - bs[t]) * kk * cs
                                             : ((s_ == rr && L2N) ? rinv : 0.f);
              }
            }
          }
          if (rr == 0 && it > 0) wait_cl(P_INW_READ + pi, pph);  // X region: -W^T copy landed
          tc::named_bar(nbL, 64);  // L^T complete
          // ---- T = (I + L)^-1: the 16x16 diagonal blocks by forward substitution, one
          //      column per thread (written to T and, transposed, to TDT) ----
          {
            const int b = rr >> 4, cI = rr & 15, R = 16 * b;
            float x[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) x[i] = (i == cI) ? 1.f : 0.f;
#pragma unroll
            for (int q = 0; q < 15; ++q) {
              const float xq = x[q];
#pragma unroll
              for (int i = q + 1; i < 16; ++i) x[i] = fmaf(-LT[(R + q) * 64 + R + i], xq, x[i]);
            }
#pragma unroll
            for (int i = 0; i < 16; ++i) Tf[(R + i) * 64 + R + cI] = x[i];
            float4 *trow = reinterpret_cast<float4 *>(TDT + b * 256 + cI * 16);
#pragma unroll
            for (int g = 0; g < 4; ++g)
              trow[g] = make_float4(x[4 * g], x[4 * g + 1], x[4 * g + 2], x[4 * g + 3]);
          }
        } else {
          // ---- P rows: scale Gamma_rs (q_r . k_s), s <= r -> bf16 hi/lo tiles ----
          const float br = gs[rr], sr = a.scale * rinv;
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            const float4 b4a = reinterpret_cast<const float4 *>(gs)[2 * q];
            const float4 b4b = reinterpret_cast<const float4 *>(gs)[2 * q + 1];
            const float bs[8] = {b4a.x, b4a.y, b4a.z, b4a.w, b4b.x, b4b.y, b4b.z, b4b.w};
            float v[8];
#pragma unroll
            for (int t = 0; t < 8; ++t) {
              const int s_ = 8 * q + t;
              const float qk = __uint_as_float(s_ < 32 ? u0[s_ & 31] : u1[s_ & 31]);
              const float cs = L2N ? LT[s_ * 65] : 1.f;
              v[t] = (s_ <= rr) ? sr * tc::ex2(br - bs[t]) * qk * cs : 0.f;
            }
            tck::st_row_chunk_split(wa + WA_T, wa + WA_T + 8192, rr, q, v);
          }
        }
        tc::tc_fence_before();
        tck::warp_arrive(bar(P_G_EMPTY + pi), lane);  // G has been read
        tc::named_bar(nb, 128);  // L^T and the diagonal blocks of T are complete
        // ---- the off-diagonal blocks of T: two rounds of block merges (all four warps) ----
        tck::merges_2round(pt, LT, Tf, Xs, Xs + 2048, TDT, Xs + 3072, nb);
        // ---- T diag(beta) -> L^T's region, T diag(beta gamma) -> X region: 16-byte chunks
        //      of 8 columns, bf16 hi/lo, by all four warps ----
#pragma unroll 1
        for (int e = pt; e < 64 * 8; e += 128) {
          const int r = e >> 3, q = e & 7;
          const float *trow = Tf + r * 64;
          const float4 ta = *reinterpret_cast<const float4 *>(trow + 8 * q);
          const float4 tb4 = *reinterpret_cast<const float4 *>(trow + 8 * q + 4);
          const float4 ba = reinterpret_cast<const float4 *>(gs + 64)[2 * q];
          const float4 bb = reinterpret_cast<const float4 *>(gs + 64)[2 * q + 1];
          const float4 ga = reinterpret_cast<const float4 *>(gs + 128)[2 * q];
          const float4 gb = reinterpret_cast<const float4 *>(gs + 128)[2 * q + 1];
          const float tv[8] = {ta.x, ta.y, ta.z, ta.w, tb4.x, tb4.y, tb4.z, tb4.w};
          const float bv[8] = {ba.x, ba.y, ba.z, ba.w, bb.x, bb.y, bb.z, bb.w};
          const float gv[8] = {ga.x, ga.y, ga.z, ga.w, gb.x, gb.y, gb.z, gb.w};
          float tb[8], tbg[8];
#pragma unroll
          for (int m = 0; m < 8; ++m) {
            tb[m] = (8 * q + m <= r) ? tv[m] * bv[m] : 0.f;
            tbg[m] = tb[m] * gv[m];
          }
          tck::st_row_chunk_split(wa + WA_LT, wa + WA_LT + 8192, r, q, tb);
          tck::st_row_chunk_split(wa + WA_X, wa + WA_X + 8192, r, q, tbg);
        }
        tc::fence_async_smem();
        tck::warp_arrive(bar(P_TBG_FULL + pi), lane);
        tck::warp_arrive(bar(P_SHIP_A + pi), lane);
        // ---- -W^T (TMEM lane = key row k, 64 values of r) -> MN-major B tile over X ----
        role_wait(P_W_FULL + pi, ph, pt == 0, nb, 128);
        tc::tc_fence_after();
        {
          uint32_t u0[32], u1[32];
          tc::tmem_ld32_nw(tmem + lane_off + colW, u0);
          tc::tmem_ld32_nw(tmem + lane_off + colW + 32, u1);
          tc::tmem_wait_ld();
          tc::reg_fence(u0);
          tc::reg_fence(u1);
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            float v[8];
#pragma unroll
            for (int t = 0; t < 8; ++t)
              v[t] = -__uint_as_float(q < 4 ? u0[(8 * q + t) & 31] : u1[(8 * q + t) & 31]);
            tck::st_row_chunk(wa + WA_X, row, q, v);
          }
        }
        tc::fence_async_smem();
        tc::tc_fence_before();
        tck::warp_arrive(bar(P_W_EMPTY + pi), lane);
        tck::warp_arrive(bar(P_GATE_EMPTY + pi), lane);
        tck::warp_arrive(bar(P_SHIP_W + pi), lane);
      }
      // the last copies have landed before this CTA may finish
      if (pt == 0 && it > 0) {
        wait_cl(P_INA_READ + pi, (uint32_t)(it - 1) & 1u);
        wait_cl(P_INW_READ + pi, (uint32_t)(it - 1) & 1u);
      }
    }
  } else {
    // ================================================================ state CTA
    if (warp == 0) {
      // ------------------------------------------------ TMA producer: V, K/Q (two stages)
      if (lane == 0 && nchunks > 0) {
        tc::prefetch_tmap(&tm_q);
        tc::prefetch_tmap(&tm_k);
        tc::prefetch_tmap(&tm_v);
        for (int c = 0; c < nchunks; ++c) {
          const int s = c & 1, z = zbase + bos + c * C;
          const uint32_t pph = (((uint32_t)c >> 1) - 1) & 1u;
          if (c >= 2) wait_sleep(S_V_EMPTY + s, pph);
          if (*abort_flag) break;
          const uint32_t vd = sb + S_OFF_V + (uint32_t)s * V_BYTES;
          tc::mbar_arrive_expect_tx(bar(S_V_FULL + s), V_BYTES);
          tc::tma_load_3d(vd, &tm_v, bar(S_V_FULL + s), 0, h, z);
          tc::tma_load_3d(vd + 8192, &tm_v, bar(S_V_FULL + s), 64, h, z);
          if (c >= 2) wait_sleep(S_QK_EMPTY + s, pph);
          if (*abort_flag) break;
          const uint32_t dst = sb + S_OFF_QK + (uint32_t)s * KQ_BYTES;
          tc::mbar_arrive_expect_tx(bar(S_QK_FULL + s), KQ_BYTES);
          tc::tma_load_3d(dst + 0, &tm_k, bar(S_QK_FULL + s), 0, hq, z);
          tc::tma_load_3d(dst + 16384, &tm_k, bar(S_QK_FULL + s), 64, hq, z);
          tc::tma_load_3d(dst + 8192, &tm_q, bar(S_QK_FULL + s), 0, hq, z);
          tc::tma_load_3d(dst + 24576, &tm_q, bar(S_QK_FULL + s), 64, hq, z);
        }
      }
    } else if (warp == 1) {
      // ------------------------------------------------ MMA issuer
      if (lane == 0 && nchunks > 0) {
        const uint64_t dQ = tc::sdesc_sw128(sb + S_OFF_QK + KQ_Q0, 16, 1024);     // Q (K-major B)
        const uint64_t dKmn = tc::sdesc_sw128(sb + S_OFF_QK + KQ_K0, 16384, 1024); // K (MN-major B)
        const uint64_t dV = tc::sdesc_sw128(sb + S_OFF_V, 8192, 1024);            // V^T (MN-major A)
        const uint64_t dTB = tc::sdesc_sw128(sb + S_OFF_IN, 16, 1024);            // T diag(beta)
        const uint64_t dP = tc::sdesc_sw128(sb + S_OFF_IN + 16384, 16, 1024);     // P
        const uint64_t dW = tc::sdesc_sw128(sb + S_OFF_IN + IN_W, 8192, 1024);    // -W^T (MN-major B)
        auto issue_U = [&](int c) {  // U^T = V^T (T diag(beta))^T into the Delta accumulator
          const int s = c & 1;
          const uint32_t ph = ((uint32_t)c >> 1) & 1u;
          wait_cl(S_INA_FULL + s, ph);
          wait(S_V_FULL + s, ph);
          if (*abort_flag) return;
          tc::tc_fence_after();
          const uint64_t tb = adv(dTB, (uint32_t)s * IN_BYTES);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t av = adv(dV, (uint32_t)s * V_BYTES + kk * 2048u);
            tc::mma_bf16(tmem + COL_DU, av, adv(tb, kk * 32u), tck::ID_MNK, kk > 0);
            tc::mma_bf16(tmem + COL_DU, av, adv(tb, 8192u + kk * 32u), tck::ID_MNK, 1);
          }
          tc::mma_commit(bar(S_V_EMPTY + s));
        };
        auto issue_D = [&](int c) {  // Delta^T += H0^T (-W^T)
          const int s = c & 1;
          wait_cl(S_INW_FULL + s, ((uint32_t)c >> 1) & 1u);
          wait(S_H0_FULL, (uint32_t)c & 1u);
          if (*abort_flag) return;
          tc::tc_fence_after();
          const uint64_t w = adv(dW, (uint32_t)s * IN_BYTES);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            tc::mma_bf16_ta(tmem + COL_DU, tmem + COL_H0 + 8 * kk, adv(w, kk * 2048u),
                            tck::ID_KMN64, 1);
          tc::mma_commit(bar(S_DMMA_FULL));
        };
        auto issue_Oa = [&](int c) {  // Oa = H0^T Q^T
          const int s = c & 1;
          if (c > 0) wait(S_OA_EMPTY, (uint32_t)(c - 1) & 1u);
          wait(S_QK_FULL + s, ((uint32_t)c >> 1) & 1u);
          if (*abort_flag) return;
          tc::tc_fence_after();
          const uint64_t q = adv(dQ, (uint32_t)s * KQ_BYTES);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            tc::mma_bf16_ta(tmem + COL_OA, tmem + COL_H0 + 8 * kk,
                            adv(q, (kk >> 2) * 16384u + (kk & 3) * 32u), tck::ID_KK64, kk > 0);
        };
        auto issue_Hupd = [&](int c) {  // Hupd = Delta~^T K
          wait(S_D_FULL, (uint32_t)c & 1u);
          if (*abort_flag) return;
          tc::tc_fence_after();
          const uint64_t k = adv(dKmn, (uint32_t)(c & 1) * KQ_BYTES);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t bk = adv(k, kk * 2048u);
            tc::mma_bf16_ta(tmem + COL_HU, tmem + COL_DTH + 8 * kk, bk, tck::ID_KMN128, kk > 0);
            tc::mma_bf16_ta(tmem + COL_HU, tmem + COL_DTL + 8 * kk, bk, tck::ID_KMN128, 1);
          }
          tc::mma_commit(bar(S_H_FULL));
        };
        auto issue_Ob = [&](int c) {  // Ob = Delta^T P^T
          const uint64_t p = adv(dP, (uint32_t)(c & 1) * IN_BYTES);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t bph = adv(p, kk * 32u), bpl = adv(p, 8192u + kk * 32u);
            tc::mma_bf16_ta(tmem + COL_OB, tmem + COL_DH + 8 * kk, bph, tck::ID_KK64, kk > 0);
            tc::mma_bf16_ta(tmem + COL_OB, tmem + COL_DL + 8 * kk, bph, tck::ID_KK64, 1);
            tc::mma_bf16_ta(tmem + COL_OB, tmem + COL_DH + 8 * kk, bpl, tck::ID_KK64, 1);
          }
          tc::mma_commit(bar(S_OB_FULL));
        };
        issue_U(0);
        for (int c = 0; c < nchunks && !*abort_flag; ++c) {
          issue_D(c);
          issue_Oa(c);  // reads H0 (c): issued before the commit that lets H0 be rewritten
          issue_Hupd(c);
          if (*abort_flag) break;
          issue_Ob(c);
          if (c + 1 < nchunks) issue_U(c + 1);
        }
      }
    } else if (warp == 2) {
      // ------------------------------------------------ gates
      for (int c = 0; c < nchunks; ++c) {
        const int s = c & 1, t0 = bos + c * C;
        if (c >= 2) {
          if (lane == 0) wait_sleep(S_GATE_EMPTY + s, ((uint32_t)(c - 2) >> 1) & 1u);
          __syncwarp();
        }
        float *gsl = reinterpret_cast<float *>(smem + S_OFF_GATES) + 256 * s;
        chunk_gates(a, gsl, zbase, t0, min(C, eos - t0), h, lane, true);
        // the output scaling gam_r (/ |q_r|) goes to the first array (bs2 is not used here);
        // the state update's e^{b_C - b_s} takes 1/|k_s|
        if constexpr (L2N) {
          if (lane == 0) wait(S_QK_FULL + s, ((uint32_t)c >> 1) & 1u);
          __syncwarp();
          const uint32_t stg = sb + S_OFF_QK + (uint32_t)s * KQ_BYTES;
#pragma unroll 1
          for (int hh = 0; hh < 2; ++hh) {
            const int r = lane + 32 * hh;
            gsl[192 + r] *= inv_norm(row_sumsq(stg + KQ_K0, r));
            gsl[r] = gsl[128 + r] * inv_norm(row_sumsq(stg + KQ_Q0, r));
          }
        } else {
          gsl[lane] = gsl[128 + lane];
          gsl[lane + 32] = gsl[160 + lane];
        }
        tck::warp_arrive(bar(S_GATE_FULL + s), lane);
      }
    } else if (warp == 3) {
      // ------------------------------------------------ courier: tell the prep CTA which
      // copies have landed (their sources may be overwritten)
      if (lane == 0 && nchunks > 0) {
        for (int c = 0; c < nchunks; ++c) {
          const int s = c & 1;
          const uint32_t ph = ((uint32_t)c >> 1) & 1u;
          wait_cl(S_INA_FULL + s, ph);
          if (*abort_flag) break;
          tc::mbar_arrive_remote_relaxed(tc::mapa(bar(P_INA_READ + s), 0));
          wait_cl(S_INW_FULL + s, ph);
          if (*abort_flag) break;
          tc::mbar_arrive_remote_relaxed(tc::mapa(bar(P_INW_READ + s), 0));
        }
      }
    } else if (wg == 1 || wg == 2) {
      // ------------------------------------------------ state chain (fp32 state in registers)
      const int swg = wg - 1, st = tid - 128;  // swg: key rows [64 swg, +64), r columns [32 swg, +32)
      long long cbase = 0;  // first chunk-state row of this sequence
      if constexpr (CS) cbase = chunk_row_base(a.cu_seqlens, n, a.T, C);
      float Hr[64];
#pragma unroll
      for (int m = 0; m < 64; ++m)
        Hr[m] = a.state_in ? a.state_in[st_off + (size_t)(64 * swg + m) * DV + row] : 0.f;
      auto store_h0 = [&]() {
        uint32_t pk[32];
#pragma unroll
        for (int t = 0; t < 32; ++t) pk[t] = tc::pack_bf16(Hr[2 * t], Hr[2 * t + 1]);
        tc::tmem_st32(tmem + lane_off + COL_H0 + 32 * swg, pk);
        tc::tc_fence_before();
      };
      if (nchunks > 0) {
        store_h0();
        tck::warp_arrive(bar(S_H0_FULL), lane);
      }
      for (int c = 0; c < nchunks; ++c) {
        const int s = c & 1;
        const float *gs = reinterpret_cast<const float *>(smem + S_OFF_GATES) + 256 * s;
        if (st == 0) wait(S_GATE_FULL + s, ((uint32_t)c >> 1) & 1u);
        role_wait(S_DMMA_FULL, (uint32_t)c & 1u, st == 0, 3, 256);
        tc::tc_fence_after();
        // ---- Delta^T, Delta~^T (row j = this lane, columns r of this half) -> bf16 hi/lo
        //      pairs in TMEM, the A operands of Ob and Hupd ----
#pragma unroll
        for (int part = 0; part < 2; ++part) {
          const int r0 = 32 * swg + 16 * part;
          float v[16], dt[16];
          tc::tmem_ld16(tmem + lane_off + COL_DU + r0, v);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const float4 d4 = reinterpret_cast<const float4 *>(gs + 192 + r0)[q];
            dt[4 * q] = d4.x; dt[4 * q + 1] = d4.y; dt[4 * q + 2] = d4.z; dt[4 * q + 3] = d4.w;
          }
          uint32_t hi[8], lo[8];
#pragma unroll
          for (int t = 0; t < 8; ++t) split2(v[2 * t], v[2 * t + 1], hi[t], lo[t]);
          tc::tmem_st8(tmem + lane_off + COL_DH + (r0 >> 1), hi);
          tc::tmem_st8(tmem + lane_off + COL_DL + (r0 >> 1), lo);
#pragma unroll
          for (int t = 0; t < 8; ++t)
            split2(v[2 * t] * dt[2 * t], v[2 * t + 1] * dt[2 * t + 1], hi[t], lo[t]);
          tc::tmem_st8(tmem + lane_off + COL_DTH + (r0 >> 1), hi);
          tc::tmem_st8(tmem + lane_off + COL_DTL + (r0 >> 1), lo);
        }
        tc::tmem_wait_st();
        tc::tc_fence_before();
        tck::warp_arrive(bar(S_D_FULL), lane);
        role_wait(S_H_FULL, (uint32_t)c & 1u, st == 0, 3, 256);
        tc::tc_fence_after();
        // ---- state: H = gamma_C H + Hupd; new H0^T operand ----
        {
          const float gC = gs[128 + 63];
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            float u[32];
            tc::tmem_ld32(tmem + lane_off + COL_HU + 64 * swg + 32 * half, u);
#pragma unroll
            for (int m = 0; m < 32; ++m) Hr[32 * half + m] = gC * Hr[32 * half + m] + u[m];
          }
          store_h0();
        }
        tck::warp_arrive(bar(S_H0_FULL), lane);
        tck::warp_arrive(bar(S_GATE_EMPTY + s), lane);
        if constexpr (CS) {
          // after the arrivals: the stores leave the chain's critical path
          float *hc = a.chunk_states + ((size_t)(cbase + c) * a.Hv + h) * DK * DV;
#pragma unroll
          for (int m = 0; m < 64; ++m) hc[(size_t)(64 * swg + m) * DV + row] = Hr[m];
        }
      }
      if (a.state_out) {
#pragma unroll
        for (int m = 0; m < 64; ++m)
          a.state_out[st_off + (size_t)(64 * swg + m) * DV + row] = Hr[m];
      }
    } else if (wg == 3) {
      // ------------------------------------------------ outputs (warpgroup 3)
      // O[r][j] = scale gamma_r Oa[j][r] + Ob[j][r].  A full chunk is staged over its own
      // K/Q stage (free once Ob has completed) and written by one TMA store; a partial
      // last chunk is stored row by row so that no token past the sequence is touched.
      using OutT = typename std::conditional<OUT_F32, float, __nv_bfloat16>::type;
      const int ot = tid - 384;
      for (int c = 0; c < nchunks; ++c) {
        const int s = c & 1, t0 = bos + c * C, L = min(C, eos - t0);
        const float *gs = reinterpret_cast<const float *>(smem + S_OFF_GATES) + 256 * s;
        if (ot == 0) wait(S_GATE_FULL + s, ((uint32_t)c >> 1) & 1u);
        role_wait(S_OB_FULL, (uint32_t)c & 1u, ot == 0, 4, 128);
        tc::tc_fence_after();
        OutT *stage_o = reinterpret_cast<OutT *>(smem + S_OFF_QK + s * KQ_BYTES);  // [64][DV]
        const bool full = (L == C);
        const size_t obase = ((size_t)zbase + t0) * a.Hv + h;
        // Oa / Ob in two halves of 32 columns; one TMEM round trip per half.  The chunk is
        // always staged in shared memory (thread = value column j, so the stores of a warp
        // are contiguous); a full chunk leaves by one TMA store, a partial one by a short
        // copy of its valid rows.
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          uint32_t ua[32], ub[32];
          tc::tmem_ld32_nw(tmem + lane_off + COL_OA + 32 * half, ua);
          tc::tmem_ld32_nw(tmem + lane_off + COL_OB + 32 * half, ub);
          tc::tmem_wait_ld();
          tc::reg_fence(ua);
          tc::reg_fence(ub);
          if (half == 1) {
            tc::tc_fence_before();
            tck::warp_arrive(bar(S_OA_EMPTY), lane);  // Oa / Ob read: the next Oa MMA may start
          }
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            const float4 g4 = reinterpret_cast<const float4 *>(gs + 32 * half)[q];
            const float gg[4] = {g4.x, g4.y, g4.z, g4.w};
#pragma unroll
            for (int t = 0; t < 4; ++t)
              io<OutT>::st(stage_o + (32 * half + 4 * q + t) * DV + row,
                           a.scale * gg[t] * __uint_as_float(ua[4 * q + t]) +
                               __uint_as_float(ub[4 * q + t]));
          }
        }
        if (!full) {
#pragma unroll 1
          for (int r = 0; r < L; ++r)
            static_cast<OutT *>(a.o)[(obase + (size_t)r * a.Hv) * DV + row] = stage_o[r * DV + row];
        }
        if (ot == 0)  // Ob (c) has completed: the incoming slot is free
          tc::mbar_arrive_remote_relaxed(tc::mapa(bar(P_IN_EMPTY + s), 0));
        if (full) {
          tc::fence_async_smem();
          tc::named_bar(4, 128);
          if (ot == 0) {
            tc::tma_store_3d(&tm_o, sb + S_OFF_QK + (uint32_t)s * KQ_BYTES, 0, h, zbase + t0);
            tc::bulk_commit();
            tc::bulk_wait_read();
          }
        }
        if (ot == 0) tc::mbar_arrive(bar(S_QK_EMPTY + s));
        tck::warp_arrive(bar(S_GATE_EMPTY + s), lane);
      }
      if (ot == 0) tc::bulk_wait_all();
    }
  }

  tc::tc_fence_before();
  __syncwarp();  // single-lane roles rejoin their warp before the CTA barrier
  __syncthreads();
  if (warp == 0) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, tmem_cols);
  }
  tc::cluster_sync();  // no CTA leaves while its partner may still signal or copy into it
}

}  // namespace tcp

inline cudaError_t pair_dispatch(bool out_f32, const PrefillArgs &a, int N, cudaStream_t stream) {
  CUtensorMap mq, mk, mv, mo;
  const long long rows = (long long)a.B * a.T;
  if (!tck::make_map(&mq, a.q, 128, a.Hqk, rows) || !tck::make_map(&mk, a.k, 128, a.Hqk, rows) ||
      !tck::make_map(&mv, a.v, 128, a.Hv, rows) ||
      !tck::make_map_out(&mo, a.o, 128, a.Hv, rows, out_f32))
    return cudaErrorInvalidValue;
  using Kern = void (*)(const CUtensorMap, const CUtensorMap, const CUtensorMap,
                       const CUtensorMap, PrefillArgs);
  static constexpr Kern kerns[8] = {
      tcp::chunk_pair_kernel<false, false, false>, tcp::chunk_pair_kernel<false, false, true>,
      tcp::chunk_pair_kernel<false, true, false>,  tcp::chunk_pair_kernel<false, true, true>,
      tcp::chunk_pair_kernel<true, false, false>,  tcp::chunk_pair_kernel<true, false, true>,
      tcp::chunk_pair_kernel<true, true, false>,   tcp::chunk_pair_kernel<true, true, true>};
  const Kern kern = kerns[(out_f32 ? 4 : 0) + (a.qk_l2norm ? 2 : 0) + (a.chunk_states ? 1 : 0)];
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)tcp::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  kern<<<2u * (unsigned)N * (unsigned)a.Hv, tcp::NT, tcp::SMEM_BYTES, stream>>>(mq, mk, mv, mo, a);
  return cudaGetLastError();
}

// The tensor-core prefill: the CTA-pair kernel; no tokens at all (only the state copy)
// goes to the CUDA-core kernel.
inline cudaError_t prefill_tc_dispatch(int dk, int dv, bool out_f32, const PrefillArgs &a, int N,
                                       cudaStream_t stream) {
  if (!tc_supported(dk, dv)) return cudaErrorNotSupported;
  if ((long long)a.B * a.T == 0)
    return out_f32 ? launch_chunk_simt<128, 128, __nv_bfloat16, float>(a, N, stream)
                   : launch_chunk_simt<128, 128, __nv_bfloat16, __nv_bfloat16>(a, N, stream);
  return pair_dispatch(out_f32, a, N, stream);
}

}  // namespace dr
