// chunk_tc.cuh -- tcgen05 tensor-core chunked prefill for bf16 inputs (dk = dv = 128).
//
// Method: the chunkwise UT/WY form of the delta rule ("Parallelizing Linear
// Transformers with the Delta Rule over Sequence Length", cited by both
// DeltaNet pages) with the per-token decay of the "linear_attention" page
// folded in.  Per 64-token chunk with start state H0 = S^T (dk x dv):
//   b = cumsum(g), gamma = e^b, Gamma_rs = e^{b_r - b_s} (s <= r)
//   L = strict_lower(diag(beta) (Gamma * K K^T)),   T = (I + L)^-1
//   W = T diag(beta gamma) K,   U = T diag(beta) V,   Delta = U - W H0
//   O = diag(gamma) Q H0 + (Gamma * Q K^T * incl_lower) Delta
//   H = gamma_C H0 + Ktil^T Delta,  Ktil_s = e^{b_C - b_s} k_s
//
// B200 mapping.  One CTA of 512 threads per (sequence, v-head); the chunk chain
// is sequential inside the CTA, and the CTA is warp-specialised so that the
// state-independent work of chunk c+1 runs under the state-dependent chain of
// chunk c:
//   warpgroup 0  warp 0: TMA producer (Q, K double-buffered; V single)
//                warp 1: tcgen05.mma issuer (one thread)
//                warp 2: gates: prefix sums of g, e^b, e^{b_C - b} per chunk
//   warpgroup 1  "prep" (chunk c+1): L and P from the Gram MMA, the fp32
//                triangular inverse T, the T diag(beta[gamma]) operands, -W^T
//   warpgroups 2-3 "state" (chunk c): Delta epilogue, outputs, state update;
//                the fp32 master state lives in their registers (thread = one
//                TMEM lane = one value column j; 64 of the key rows each)
// Every product is a tcgen05.mma with M = 128 (bf16 operands, fp32 TMEM
// accumulators):
//        G       = [K; Q] K^T                (rows 0-63: K K^T, 64-127: Q K^T)
//        W^T     = K^T (T diag(beta gamma))^T,   U^T = V^T (T diag(beta))^T
//        Delta^T = U^T + H0^T (-W^T)         (accumulates onto U^T in TMEM)
//        Oa      = H0^T Q^T,   Ob = Delta^T P^T     (O^T = diag(gamma) Oa + Ob)
//        Hupd    = Delta~^T K  with Delta~_s = e^{b_C - b_s} Delta_s
// H0^T (bf16) is the A operand of two of them and is read from TMEM, written
// there by the state warps each chunk.
// Precision: operands computed in fp32 inside the kernel (T diag(beta),
// T diag(beta gamma), P, Delta, Delta~) go to the tensor core as a bf16 pair
// x = hi + lo (hi = bf16(x), lo = bf16(x - hi)): two MMAs into one accumulator
// (three for P Delta, dropping lo x lo).  A single bf16 rounding of these
// (2^-8 relative) alone exceeds the 2e-2 max/RMS error budget on short
// sequences; the pair keeps ~2^-16.  q, k, v are exact in bf16.
// Decays are always formed from differences of cumulative log decays, never as
// ratios of separate exponentials (no overflow for strongly negative g).
#pragma once

#include <cuda.h>

#include <mutex>
#include <type_traits>

#include "chunk_simt.cuh"
#include "tc_ptx.cuh"

namespace dr {
namespace tck {

constexpr int C = 64, DK = 128, DV = 128, NT = 512;
constexpr float LOG2E = 1.4426950408889634f;

// ---- shared memory (bytes from a 1024-aligned base) ----
constexpr uint32_t QK_BYTES = 32768;                        // K0 Q0 K1 Q1, 8 KB boxes
constexpr uint32_t QK_K0 = 0, QK_Q0 = 8192, QK_K1 = 16384, QK_Q1 = 24576;
constexpr uint32_t OFF_QK = 0;                              // 2 stages
constexpr uint32_t OFF_V = 2 * QK_BYTES;                    // V0, V1 (single stage)
constexpr uint32_t V_BYTES = 16384;
constexpr uint32_t OFF_RL = OFF_V + V_BYTES;                // L fp32 [64][65] | T diag(beta) hi, lo
constexpr uint32_t OFF_RT = OFF_RL + 17408;                 // T fp32 [64][64] | -W^T bf16
constexpr uint32_t OFF_RX = OFF_RT + 16384;                 // merge scratch | T diag(beta gamma) hi, lo
constexpr uint32_t OFF_P = OFF_RX + 16384;                  // P hi, P lo
constexpr uint32_t OFF_DH = OFF_P + 16384;                  // Delta^T hi
constexpr uint32_t OFF_DL = OFF_DH + 16384;                 // Delta^T lo
constexpr uint32_t OFF_DTH = OFF_DL + 16384;                // Delta~^T hi
constexpr uint32_t OFF_DTL = OFF_DTH + 16384;               // Delta~^T lo
constexpr uint32_t OFF_GATES = OFF_DTL + 16384;             // 2 slots x {bs2, beta, gam, dtil}[64]
constexpr uint32_t OFF_BARS = OFF_GATES + 2 * 4 * 64 * 4;
constexpr uint32_t SMEM_BYTES = OFF_BARS + 256 + 1024;      // + alignment slack
static_assert(SMEM_BYTES <= 232448, "shared memory budget");
static_assert(OFF_RL % 1024 == 0 && OFF_RT % 1024 == 0 && OFF_RX % 1024 == 0 &&
                  OFF_P % 1024 == 0 && OFF_DH % 1024 == 0 && OFF_DTL % 1024 == 0,
              "operand tiles must be 1024-byte aligned");

// ---- TMEM columns ----
constexpr uint32_t COL_G = 0, COL_W = 64, COL_DU = 128, COL_OA = 192, COL_OB = 256;
constexpr uint32_t COL_HU = 320, COL_H0 = 448, TMEM_COLS = 512;

constexpr uint32_t ID_G = tc::idesc_bf16(128, 64, 0, 0);        // [K;Q] K^T
constexpr uint32_t ID_MNK = tc::idesc_bf16(128, 64, 1, 0);      // K^T / V^T x T^T
constexpr uint32_t ID_KMN64 = tc::idesc_bf16(128, 64, 0, 1);    // H0^T x (-W^T)
constexpr uint32_t ID_KK64 = tc::idesc_bf16(128, 64, 0, 0);     // H0^T Q^T, Delta^T P^T
constexpr uint32_t ID_KMN128 = tc::idesc_bf16(128, 128, 0, 1);  // Delta~^T K

// ---- mbarriers ----
enum Bar {
  B_QK_FULL = 0,   // [2] TMA -> MMA
  B_QK_EMPTY = 2,  // [2] MMA (after Hupd) -> TMA
  B_V_FULL = 4,
  B_V_EMPTY = 5,
  B_GATE_FULL = 6,   // [2] gates warp (32) -> prep, state
  B_GATE_EMPTY = 8,  // [2] prep (128) + state (256) -> gates warp
  B_G_FULL = 10,     // MMA -> prep
  B_G_EMPTY = 11,    // prep (128) -> MMA
  B_TB_FULL = 12,    // prep (128) -> MMA
  B_P_FULL = 13,     // prep (128) -> MMA
  B_W_FULL = 14,     // MMA -> prep
  B_MW_FULL = 15,    // prep (128) -> MMA
  B_H0_FULL = 16,    // state (256) -> MMA
  B_DMMA_FULL = 17,  // MMA -> state
  B_D_FULL = 18,     // state (256) -> MMA
  B_DU_EMPTY = 19,   // state (256) -> MMA
  B_H_FULL = 20,     // MMA -> state, prep
  B_OA_EMPTY = 21,   // state (256) -> MMA: Oa/Ob accumulators have been read
  NUM_BARS = 22
};

__device__ __forceinline__ void st_row_chunk(uint32_t tile, int row, int chunk, const float *v) {
  tc::st_shared_v4(tile + tc::sw128_off(row, chunk), tc::pack_bf16(v[0], v[1]),
                   tc::pack_bf16(v[2], v[3]), tc::pack_bf16(v[4], v[5]),
                   tc::pack_bf16(v[6], v[7]));
}
// Same, as the bf16 pair hi = bf16(x), lo = bf16(x - hi) into two tiles.
__device__ __forceinline__ void st_row_chunk_split(uint32_t tile_hi, uint32_t tile_lo, int row,
                                                   int chunk, const float *v) {
  float hi[8], lo[8];
#pragma unroll
  for (int t = 0; t < 8; ++t) {
    hi[t] = __bfloat162float(__float2bfloat16_rn(v[t]));
    lo[t] = v[t] - hi[t];
  }
  st_row_chunk(tile_hi, row, chunk, hi);
  st_row_chunk(tile_lo, row, chunk, lo);
}

// Block merges of T = (I + L)^-1 (64 x 64; blocks of 16), 128 threads, two rounds:
//   A: T_10 = -T_11 (L_10 T_00), T_32 = -T_33 (L_32 T_22)        (16 -> 32, 2x2 tiles)
//   B: T_BA = -T_BB (L_BA T_AA) for the 32x32 halves A, B        (32 -> 64, 2x4 tiles)
// Register tiles with float2/float4 shared operands; no K splits, so no shuffles.
// In: LT = L^T [64][64]; Tf [64][64] with the four 16x16 diagonal blocks of T; TDT [4][16][16] =
// the diagonal blocks transposed.  Scratch: XA [2][16][16], XB [32][32], TBBT [32][32].
// Out: Tf lower blocks complete.
__device__ __forceinline__ void merges_2round(int pt, const float *LT, float *Tf, float *XA,
                                              float *XB, const float *TDT, float *TBBT,
                                              uint32_t nb = 1) {
  // ---- round A: T_10 = -T_11 (L_10 T_00), T_32 = -T_33 (L_32 T_22); 2x2 tiles ----
  {
    const int b = pt >> 6, lt = pt & 63, tr = lt >> 3, tcl = lt & 7;  // b: 0 -> (1,0), 1 -> (3,2)
    const int i = 2 * b + 1, j = 2 * b;
    const int r0 = 16 * i + 2 * tr, c0 = 16 * j + 2 * tcl;
    float a00 = 0.f, a01 = 0.f, a10 = 0.f, a11 = 0.f;
#pragma unroll
    for (int m = 0; m < 16; ++m) {
      const float2 l = *reinterpret_cast<const float2 *>(&LT[(16 * j + m) * 64 + r0]);
      const float2 t = *reinterpret_cast<const float2 *>(&Tf[(16 * j + m) * 64 + c0]);
      a00 = fmaf(l.x, t.x, a00); a01 = fmaf(l.x, t.y, a01);
      a10 = fmaf(l.y, t.x, a10); a11 = fmaf(l.y, t.y, a11);
    }
    float *X = XA + b * 256;
    *reinterpret_cast<float2 *>(&X[(2 * tr) * 16 + 2 * tcl]) = make_float2(a00, a01);
    *reinterpret_cast<float2 *>(&X[(2 * tr + 1) * 16 + 2 * tcl]) = make_float2(a10, a11);
    tc::named_bar(nb, 128);
    a00 = a01 = a10 = a11 = 0.f;
#pragma unroll
    for (int m = 0; m < 16; ++m) {  // T_ii^T[m][r] (zero for m > r)
      const float2 l = *reinterpret_cast<const float2 *>(&TDT[i * 256 + m * 16 + 2 * tr]);
      const float2 x = *reinterpret_cast<const float2 *>(&X[m * 16 + 2 * tcl]);
      a00 = fmaf(l.x, x.x, a00); a01 = fmaf(l.x, x.y, a01);
      a10 = fmaf(l.y, x.x, a10); a11 = fmaf(l.y, x.y, a11);
    }
    *reinterpret_cast<float2 *>(&Tf[(r0) * 64 + c0]) = make_float2(-a00, -a01);
    *reinterpret_cast<float2 *>(&Tf[(r0 + 1) * 64 + c0]) = make_float2(-a10, -a11);
    if (b == 1) {  // T_BB^T [m][r] (local indices): T_32^T block at m in 0..15, r in 16..31
      TBBT[(2 * tcl) * 32 + 16 + 2 * tr] = -a00;     TBBT[(2 * tcl) * 32 + 17 + 2 * tr] = -a10;
      TBBT[(2 * tcl + 1) * 32 + 16 + 2 * tr] = -a01; TBBT[(2 * tcl + 1) * 32 + 17 + 2 * tr] = -a11;
    }
  }
  {  // the rest of T_BB^T: diagonal blocks T_22^T, T_33^T and the zero block (m in 16..31, r in 0..15)
    for (int e = pt; e < 768; e += 128) {
      const int q = e >> 8, w = e & 255, m = w >> 4, r = w & 15;
      if (q == 0) TBBT[m * 32 + r] = TDT[2 * 256 + m * 16 + r];
      else if (q == 1) TBBT[(16 + m) * 32 + 16 + r] = TDT[3 * 256 + m * 16 + r];
      else TBBT[(16 + m) * 32 + r] = 0.f;
    }
  }
  tc::named_bar(nb, 128);
  // ---- round B: X = L_BA T_AA (rows 32..63, cols 0..31), 2x4 tiles; column block uniform per warp ----
  {
    const int cb = pt >> 6, lt = pt & 63, tr = lt >> 2, tcl = lt & 3;
    const int r0 = 32 + 2 * tr, c0 = 16 * cb + 4 * tcl;
    float acc[8];
#pragma unroll
    for (int t = 0; t < 8; ++t) acc[t] = 0.f;
    const int kbeg = 16 * cb;  // T_AA[k][c] = 0 for k < 16 when c >= 16
#pragma unroll 4
    for (int k = kbeg; k < 32; ++k) {
      const float2 l = *reinterpret_cast<const float2 *>(&LT[k * 64 + r0]);
      const float4 t = *reinterpret_cast<const float4 *>(&Tf[k * 64 + c0]);
      acc[0] = fmaf(l.x, t.x, acc[0]); acc[1] = fmaf(l.x, t.y, acc[1]);
      acc[2] = fmaf(l.x, t.z, acc[2]); acc[3] = fmaf(l.x, t.w, acc[3]);
      acc[4] = fmaf(l.y, t.x, acc[4]); acc[5] = fmaf(l.y, t.y, acc[5]);
      acc[6] = fmaf(l.y, t.z, acc[6]); acc[7] = fmaf(l.y, t.w, acc[7]);
    }
    *reinterpret_cast<float4 *>(&XB[(2 * tr) * 32 + c0]) = make_float4(acc[0], acc[1], acc[2], acc[3]);
    *reinterpret_cast<float4 *>(&XB[(2 * tr + 1) * 32 + c0]) = make_float4(acc[4], acc[5], acc[6], acc[7]);
    tc::named_bar(nb, 128);
#pragma unroll
    for (int t = 0; t < 8; ++t) acc[t] = 0.f;
#pragma unroll 4
    for (int m = 0; m < 32; ++m) {  // T_BB^T[m][r] (zero for m > r)
      const float2 l = *reinterpret_cast<const float2 *>(&TBBT[m * 32 + 2 * tr]);
      const float4 x = *reinterpret_cast<const float4 *>(&XB[m * 32 + c0]);
      acc[0] = fmaf(l.x, x.x, acc[0]); acc[1] = fmaf(l.x, x.y, acc[1]);
      acc[2] = fmaf(l.x, x.z, acc[2]); acc[3] = fmaf(l.x, x.w, acc[3]);
      acc[4] = fmaf(l.y, x.x, acc[4]); acc[5] = fmaf(l.y, x.y, acc[5]);
      acc[6] = fmaf(l.y, x.z, acc[6]); acc[7] = fmaf(l.y, x.w, acc[7]);
    }
    *reinterpret_cast<float4 *>(&Tf[r0 * 64 + c0]) = make_float4(-acc[0], -acc[1], -acc[2], -acc[3]);
    *reinterpret_cast<float4 *>(&Tf[(r0 + 1) * 64 + c0]) = make_float4(-acc[4], -acc[5], -acc[6], -acc[7]);
  }
  tc::named_bar(nb, 128);
}

// Every lane has finished its shared/tensor-memory work for this hand-off (and fenced it);
// one elected lane per warp then arrives.
__device__ __forceinline__ void warp_arrive(uint32_t bar, int lane) {
  __syncwarp();
  if (lane == 0) tc::mbar_arrive(bar);
}

template <bool OUT_F32>
__global__ void __launch_bounds__(NT, 1)
    chunk_tc_kernel(const __grid_constant__ CUtensorMap tm_q,
                    const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v,
                    const __grid_constant__ CUtensorMap tm_o, PrefillArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // Align by offsetting the shared array itself (not through an integer cast), so that every
  // pointer derived from it stays in the shared address space: plain LDS/STS, not generic
  // loads and stores.
  uint8_t *smem = smem_raw + ((1024u - (tc::smem_u32(smem_raw) & 1023u)) & 1023u);
  const uint32_t sb = tc::smem_u32(smem);
  float *gates = reinterpret_cast<float *>(smem + OFF_GATES);  // slot s: gates + 256 s
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + OFF_BARS);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + NUM_BARS);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
  auto bar = [&](int i) { return tc::smem_u32(&bars[i]); };

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int wg = warp >> 2, q4 = warp & 3;
  const int row = 32 * q4 + lane;                        // TMEM lane this thread reads
  const uint32_t lane_off = (uint32_t)(32 * q4) << 16;

  const int unit = blockIdx.x, n = unit / a.Hv, h = unit % a.Hv;
  const int hq = h / (a.Hv / a.Hqk);
  int batch, bos, eos;
  if (!seq_bounds(a.cu_seqlens, n, a.n_seqs, a.T, batch, bos, eos)) return;  // CTA-uniform
  const int nchunks = (eos - bos + C - 1) / C;
  const int zbase = batch * a.T;
  const size_t st_off = ((size_t)n * a.Hv + h) * DK * DV;

  if (tid == 0) {
    // arrival counts: 1 = one thread (TMA expect_tx or tcgen05.commit), else one elected
    // lane per warp of the signalling group (gates 1, prep 4, state 8, prep + state 12)
    static constexpr uint16_t counts[NUM_BARS] = {1, 1, 1, 1, 1, 1, 1, 1, 12, 12, 1,
                                                  4, 4, 4, 1, 4, 8, 1, 8, 8, 1, 8};
    for (int i = 0; i < NUM_BARS; ++i) tc::mbar_init(bar(i), counts[i]);
    *abort_flag = 0;
    tc::fence_barrier_init();
  }
  if (warp == 0) {
    tc::tmem_alloc(tc::smem_u32(tmem_slot), TMEM_COLS);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncwarp();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // Hand-off waits.  Critical-path waits poll (mbarrier.test_wait); in the prep and state
  // roles only one leader thread polls while the rest of the role blocks in a hardware
  // named barrier, which costs no issue slots and releases as soon as the leader arrives.
  auto wait = [&](int i, uint32_t parity) { tc::mbar_wait(bar(i), parity, abort_flag); };
  auto wait_sleep = [&](int i, uint32_t parity) {
    tc::mbar_wait_sleep(bar(i), parity, abort_flag);
  };
  auto role_wait = [&](int i, uint32_t parity, bool leader, uint32_t bar_id, uint32_t nthreads) {
    if (leader) tc::mbar_wait(bar(i), parity, abort_flag);
    tc::named_bar(bar_id, nthreads);
  };

  if (wg == 0) {
    // =========================================================== producer roles
    if (warp == 0 && lane == 0 && nchunks > 0) {
      tc::prefetch_tmap(&tm_q);
      tc::prefetch_tmap(&tm_k);
      tc::prefetch_tmap(&tm_v);
      for (int c = 0; c < nchunks; ++c) {
        const int s = c & 1, z = zbase + bos + c * C;
        const uint32_t dst = sb + OFF_QK + (uint32_t)s * QK_BYTES;
        if (c >= 2) wait_sleep(B_QK_EMPTY + s, (((uint32_t)c >> 1) & 1u) ^ 1u);
        if (*abort_flag) break;
        tc::mbar_arrive_expect_tx(bar(B_QK_FULL + s), QK_BYTES);
        tc::tma_load_3d(dst + QK_K0, &tm_k, bar(B_QK_FULL + s), 0, hq, z);
        tc::tma_load_3d(dst + QK_K1, &tm_k, bar(B_QK_FULL + s), 64, hq, z);
        tc::tma_load_3d(dst + QK_Q0, &tm_q, bar(B_QK_FULL + s), 0, hq, z);
        tc::tma_load_3d(dst + QK_Q1, &tm_q, bar(B_QK_FULL + s), 64, hq, z);
        if (c >= 1) wait_sleep(B_V_EMPTY, (uint32_t)(c - 1) & 1u);
        if (*abort_flag) break;
        tc::mbar_arrive_expect_tx(bar(B_V_FULL), V_BYTES);
        tc::tma_load_3d(sb + OFF_V, &tm_v, bar(B_V_FULL), 0, h, z);
        tc::tma_load_3d(sb + OFF_V + 8192, &tm_v, bar(B_V_FULL), 64, h, z);
      }
    } else if (warp == 1 && lane == 0 && nchunks > 0) {
      // ------------------------------------------------------- MMA issuer
      // Shared-memory descriptors are built once; per chunk only the stage base changes.
      const uint64_t dKQ = tc::sdesc_sw128(sb + OFF_QK, 16, 1024);              // [K;Q], K (K-major)
      const uint64_t dKmn = tc::sdesc_sw128(sb + OFF_QK + QK_K0, 16384, 1024);  // K (MN-major)
      const uint64_t dQ = tc::sdesc_sw128(sb + OFF_QK + QK_Q0, 16, 1024);       // Q (K-major)
      const uint64_t dV = tc::sdesc_sw128(sb + OFF_V, 8192, 1024);              // V (MN-major)
      const uint64_t dTB = tc::sdesc_sw128(sb + OFF_RL, 16, 1024);              // T diag(beta) hi
      const uint64_t dTBG = tc::sdesc_sw128(sb + OFF_RX, 16, 1024);             // T diag(beta gamma) hi
      const uint64_t dW = tc::sdesc_sw128(sb + OFF_RT, 8192, 1024);             // -W^T (MN-major)
      const uint64_t dDH = tc::sdesc_sw128(sb + OFF_DH, 16, 1024);
      const uint64_t dDL = tc::sdesc_sw128(sb + OFF_DL, 16, 1024);
      const uint64_t dDTH = tc::sdesc_sw128(sb + OFF_DTH, 16, 1024);
      const uint64_t dDTL = tc::sdesc_sw128(sb + OFF_DTL, 16, 1024);
      const uint64_t dPH = tc::sdesc_sw128(sb + OFF_P, 16, 1024);
      const uint64_t dPL = tc::sdesc_sw128(sb + OFF_P + 8192, 16, 1024);
      // descriptor address field is in 16-byte units
      auto adv = [](uint64_t d, uint32_t bytes) { return d + (uint64_t)(bytes >> 4); };
      auto issue_G = [&](int c) {
        const int s = c & 1;
        wait(B_QK_FULL + s, ((uint32_t)c >> 1) & 1u);
        if (c > 0) wait(B_G_EMPTY, (uint32_t)(c - 1) & 1u);
        if (*abort_flag) return;
        tc::tc_fence_after();
        const uint64_t d0 = adv(dKQ, (uint32_t)s * QK_BYTES);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t d = adv(d0, (kk >> 2) * 16384u + (kk & 3) * 32u);
          tc::mma_bf16(tmem + COL_G, d, d, ID_G, kk > 0);
        }
        tc::mma_commit(bar(B_G_FULL));
      };
      auto issue_WU = [&](int c) {
        wait(B_TB_FULL, (uint32_t)c & 1u);
        if (*abort_flag) return;
        tc::tc_fence_after();
        const uint64_t dk = adv(dKmn, (uint32_t)(c & 1) * QK_BYTES);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {  // W^T first: the prep role waits for it
          const uint64_t ak = adv(dk, kk * 2048u);
          tc::mma_bf16(tmem + COL_W, ak, adv(dTBG, kk * 32u), ID_MNK, kk > 0);
          tc::mma_bf16(tmem + COL_W, ak, adv(dTBG, 8192u + kk * 32u), ID_MNK, 1);
        }
        tc::mma_commit(bar(B_W_FULL));
        wait(B_V_FULL, (uint32_t)c & 1u);
        if (c > 0) wait(B_DU_EMPTY, (uint32_t)(c - 1) & 1u);
        if (*abort_flag) return;
        tc::tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint64_t av = adv(dV, kk * 2048u);
          tc::mma_bf16(tmem + COL_DU, av, adv(dTB, kk * 32u), ID_MNK, kk > 0);
          tc::mma_bf16(tmem + COL_DU, av, adv(dTB, 8192u + kk * 32u), ID_MNK, 1);
        }
        tc::mma_commit(bar(B_V_EMPTY));
      };
      auto issue_DO = [&](int c) {
        wait(B_MW_FULL, (uint32_t)c & 1u);
        wait(B_H0_FULL, (uint32_t)c & 1u);
        if (*abort_flag) return;
        tc::tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          tc::mma_bf16_ta(tmem + COL_DU, tmem + COL_H0 + 8 * kk, adv(dW, kk * 2048u), ID_KMN64, 1);
        tc::mma_commit(bar(B_DMMA_FULL));
        if (c > 0) wait(B_OA_EMPTY, (uint32_t)(c - 1) & 1u);  // outputs of c-1 read out
        tc::tc_fence_after();
        const uint64_t dq = adv(dQ, (uint32_t)(c & 1) * QK_BYTES);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          tc::mma_bf16_ta(tmem + COL_OA, tmem + COL_H0 + 8 * kk,
                          adv(dq, (kk >> 2) * 16384u + (kk & 3) * 32u), ID_KK64, kk > 0);
      };
      auto issue_HO = [&](int c) {
        wait(B_D_FULL, (uint32_t)c & 1u);
        if (*abort_flag) return;
        tc::tc_fence_after();
        const uint64_t dk = adv(dKmn, (uint32_t)(c & 1) * QK_BYTES);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {  // the state update first: it is on the critical path
          const uint64_t bk = adv(dk, kk * 2048u);
          tc::mma_bf16(tmem + COL_HU, adv(dDTH, kk * 32u), bk, ID_KMN128, kk > 0);
          tc::mma_bf16(tmem + COL_HU, adv(dDTL, kk * 32u), bk, ID_KMN128, 1);
        }
        wait(B_P_FULL, (uint32_t)c & 1u);
        if (*abort_flag) return;
        tc::tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint64_t adh = adv(dDH, kk * 32u), adl = adv(dDL, kk * 32u);
          const uint64_t bph = adv(dPH, kk * 32u), bpl = adv(dPL, kk * 32u);
          tc::mma_bf16(tmem + COL_OB, adh, bph, ID_KK64, kk > 0);
          tc::mma_bf16(tmem + COL_OB, adl, bph, ID_KK64, 1);
          tc::mma_bf16(tmem + COL_OB, adh, bpl, ID_KK64, 1);
        }
        tc::mma_commit(bar(B_H_FULL));
        tc::mma_commit(bar(B_QK_EMPTY + (c & 1)));
      };
      issue_G(0);
      issue_WU(0);
      for (int c = 0; c < nchunks; ++c) {
        issue_DO(c);
        if (c + 1 < nchunks) issue_G(c + 1);
        issue_HO(c);
        if (c + 1 < nchunks) issue_WU(c + 1);
      }
    } else if (warp == 2) {
      // ------------------------------------------------------- gates
      for (int c = 0; c < nchunks; ++c) {
        const int s = c & 1, t0 = bos + c * C, L = min(C, eos - t0);
        if (c >= 2) {
          if (lane == 0) wait_sleep(B_GATE_EMPTY + s, ((uint32_t)(c - 2) >> 1) & 1u);
          __syncwarp();
        }
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
        float *gs = gates + 256 * s;  // bs2[64], beta[64], gam[64], dtil[64]
        gs[lane] = g0 * LOG2E;
        gs[lane + 32] = g1 * LOG2E;
        gs[64 + lane] = b0;
        gs[96 + lane] = b1;
        gs[128 + lane] = tc::ex2(g0 * LOG2E);
        gs[160 + lane] = tc::ex2(g1 * LOG2E);
        gs[192 + lane] = tc::ex2((blast - g0) * LOG2E);
        gs[224 + lane] = tc::ex2((blast - g1) * LOG2E);
        warp_arrive(bar(B_GATE_FULL + s), lane);
      }
    }
  } else if (wg == 1) {
    // =========================================================== prep (chunk c+1 ahead)
    const int pt = tid - 128;  // 0..127
    float *LT = reinterpret_cast<float *>(smem + OFF_RL);  // L^T fp32 [64 s][64 r]
    float *Tf = reinterpret_cast<float *>(smem + OFF_RT);  // T fp32 [64][64], row-major
    float *Xs = reinterpret_cast<float *>(smem + OFF_RX);  // merge scratch [2][16][16] | TDT | XB | TBBT
    float *TDT = Xs + 512;                                 // diagonal blocks transposed [4][16 m][16 r]
    for (int c = 0; c < nchunks; ++c) {
      const int s = c & 1;
      const float *gs = gates + 256 * s;
      if (pt == 0) wait(B_GATE_FULL + s, ((uint32_t)c >> 1) & 1u);
      role_wait(B_G_FULL, (uint32_t)c & 1u, pt == 0, 1, 128);
      tc::tc_fence_after();
      // ---- L^T (TMEM lanes 0-63 hold rows r of K K^T): L_rs = beta_r Gamma_rs (k_r . k_s), s < r ----
      if (q4 < 2) {
        const int r = row;
        const float br = gs[r], bt = gs[64 + r];
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          float v[32], bs[32];
          tc::tmem_ld32(tmem + lane_off + COL_G + 32 * half, v);
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            const float4 b4 = reinterpret_cast<const float4 *>(gs)[8 * half + q];
            bs[4 * q] = b4.x; bs[4 * q + 1] = b4.y; bs[4 * q + 2] = b4.z; bs[4 * q + 3] = b4.w;
          }
#pragma unroll
          for (int cc = 0; cc < 32; ++cc) {
            const int s_ = 32 * half + cc;
            LT[s_ * 64 + r] = (s_ < r) ? bt * tc::ex2(br - bs[cc]) * v[cc] : 0.f;
          }
        }
      }
      tc::named_bar(1, 128);
      // ---- T = (I + L)^-1, diagonal 16x16 blocks by forward substitution (one column each) ----
      if (pt < 64) {
        const int blk = pt >> 4, cI = pt & 15, R = 16 * blk;
        float x[16];
#pragma unroll
        for (int r = 0; r < 16; ++r) x[r] = (r == cI) ? 1.f : 0.f;
#pragma unroll
        for (int r = 1; r < 16; ++r) {
          float acc = 0.f;
#pragma unroll
          for (int q = 0; q < r; ++q) acc += LT[(R + q) * 64 + R + r] * x[q];
          if (r > cI) x[r] = -acc;
        }
#pragma unroll
        for (int r = 0; r < 16; ++r) {
          Tf[(R + r) * 64 + R + cI] = x[r];
          TDT[blk * 256 + cI * 16 + r] = x[r];  // (T_bb)^T[m = cI][r]
        }
      }
      tc::named_bar(1, 128);
      // ---- block merges (two rounds, see merges_2round) ----
      merges_2round(pt, LT, Tf, Xs, Xs + 2048, TDT, Xs + 3072);
      // ---- T diag(beta) (over L's region) and T diag(beta gamma) (over the scratch) ----
      for (int e = pt; e < 64 * 8; e += 128) {
        const int r = e >> 3, q = e & 7;
        float tb[8], tbg[8];
        const float4 ta = *reinterpret_cast<const float4 *>(&Tf[r * 64 + 8 * q]);
        const float4 tb4 = *reinterpret_cast<const float4 *>(&Tf[r * 64 + 8 * q + 4]);
        const float tv[8] = {ta.x, ta.y, ta.z, ta.w, tb4.x, tb4.y, tb4.z, tb4.w};
#pragma unroll
        for (int m = 0; m < 8; ++m) {
          const int s_ = 8 * q + m;
          tb[m] = (s_ <= r) ? tv[m] * gs[64 + s_] : 0.f;
          tbg[m] = tb[m] * gs[128 + s_];
        }
        st_row_chunk_split(sb + OFF_RL, sb + OFF_RL + 8192, r, q, tb);
        st_row_chunk_split(sb + OFF_RX, sb + OFF_RX + 8192, r, q, tbg);
      }
      tc::fence_async_smem();
      warp_arrive(bar(B_TB_FULL), lane);
      // ---- P rows (TMEM lanes 64-127): scale Gamma_rs (q_r . k_s), s <= r ----
      if (c > 0) role_wait(B_H_FULL, (uint32_t)(c - 1) & 1u, pt == 0, 1, 128);  // Ob(c-1) read P
      if (q4 >= 2) {
        const int r = row - 64;
        const float br = gs[r];
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          float v[32];
          tc::tmem_ld32(tmem + lane_off + COL_G + 32 * half, v);
#pragma unroll
          for (int cc = 0; cc < 32; ++cc) {
            const int s_ = 32 * half + cc;
            v[cc] = (s_ <= r) ? a.scale * tc::ex2(br - gs[s_]) * v[cc] : 0.f;
          }
#pragma unroll
          for (int q = 0; q < 4; ++q)
            st_row_chunk_split(sb + OFF_P, sb + OFF_P + 8192, r, 4 * half + q, &v[8 * q]);
        }
      }
      tc::fence_async_smem();
      tc::tc_fence_before();
      warp_arrive(bar(B_P_FULL), lane);
      warp_arrive(bar(B_G_EMPTY), lane);
      // ---- -W^T (TMEM lane i, 64 values of r) -> MN-major B tile over T's region ----
      role_wait(B_W_FULL, (uint32_t)c & 1u, pt == 0, 1, 128);
      tc::tc_fence_after();
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        float v[32];
        tc::tmem_ld32(tmem + lane_off + COL_W + 32 * half, v);
#pragma unroll
        for (int cc = 0; cc < 32; ++cc) v[cc] = -v[cc];
#pragma unroll
        for (int q = 0; q < 4; ++q) st_row_chunk(sb + OFF_RT, row, 4 * half + q, &v[8 * q]);
      }
      tc::fence_async_smem();
      tc::tc_fence_before();
      warp_arrive(bar(B_MW_FULL), lane);
      warp_arrive(bar(B_GATE_EMPTY + s), lane);
    }
  } else {
    // =========================================================== state chain
    const int swg = wg - 2;  // 0 or 1: key rows [64 swg, 64 swg + 64), value-column halves
    float Hr[64];
#pragma unroll
    for (int m = 0; m < 64; ++m)
      Hr[m] = a.state_in ? a.state_in[st_off + (size_t)(64 * swg + m) * DV + row] : 0.f;
    auto store_h0 = [&]() {  // H0^T row j (this lane), k = key rows of this half, bf16 pairs
      uint32_t pk[32];
#pragma unroll
      for (int t = 0; t < 32; ++t) pk[t] = tc::pack_bf16(Hr[2 * t], Hr[2 * t + 1]);
      tc::tmem_st32(tmem + lane_off + COL_H0 + 32 * swg, pk);
      tc::tc_fence_before();
    };
    if (nchunks > 0) {
      store_h0();
      warp_arrive(bar(B_H0_FULL), lane);
    }
    for (int c = 0; c < nchunks; ++c) {
      const int s = c & 1, t0 = bos + c * C, L = min(C, eos - t0);
      const float *gs = gates + 256 * s;
      const int st = tid - 256;
      if (st == 0) {
        tc::bulk_wait_read();  // the previous chunk's output store has left shared memory
        wait(B_GATE_FULL + s, ((uint32_t)c >> 1) & 1u);
      }
      role_wait(B_DMMA_FULL, (uint32_t)c & 1u, st == 0, 2, 256);
      tc::tc_fence_after();
      // ---- Delta^T, Delta~^T -> bf16 hi/lo K-major A tiles (row j, columns r of this half) ----
#pragma unroll
      for (int part = 0; part < 2; ++part) {
        float v[16], w[16], dt[16];  // dt: e^{b_C - b_r} for these 16 columns
        const int r0 = 32 * swg + 16 * part;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float4 d4 = reinterpret_cast<const float4 *>(gs + 192 + r0)[q];
          dt[4 * q] = d4.x; dt[4 * q + 1] = d4.y; dt[4 * q + 2] = d4.z; dt[4 * q + 3] = d4.w;
        }
        tc::tmem_ld16(tmem + lane_off + COL_DU + r0, v);
#pragma unroll
        for (int cc = 0; cc < 16; ++cc) w[cc] = v[cc] * dt[cc];
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          const int ch = (r0 >> 3) + q;
          st_row_chunk_split(sb + OFF_DH, sb + OFF_DL, row, ch, &v[8 * q]);
          st_row_chunk_split(sb + OFF_DTH, sb + OFF_DTL, row, ch, &w[8 * q]);
        }
      }
      tc::fence_async_smem();
      tc::tc_fence_before();
      warp_arrive(bar(B_D_FULL), lane);
      warp_arrive(bar(B_DU_EMPTY), lane);
      role_wait(B_H_FULL, (uint32_t)c & 1u, st == 0, 2, 256);
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
      warp_arrive(bar(B_H0_FULL), lane);  // the next chunk's Delta MMA may start
      // ---- outputs: O[r][j] = scale gamma_r Oa[j][r] + Ob[j][r].  A full chunk is staged in
      //      shared memory (over the Delta^T tiles, free until the next Delta epilogue) and
      //      written by one TMA store; a partial last chunk is stored row by row so that no
      //      token past the end of the sequence is touched. ----
      {
        using OutT = typename std::conditional<OUT_F32, float, __nv_bfloat16>::type;
        OutT *stage_o = reinterpret_cast<OutT *>(smem + OFF_DH);  // [64][DV]
        const bool full = (L == C);
        const size_t obase = ((size_t)zbase + t0) * a.Hv + h;
#pragma unroll
        for (int part = 0; part < 2; ++part) {
          float oa[16], ob[16], gsc[16];  // gsc: scale * gamma_r for these 16 rows
          const int r0 = 32 * swg + 16 * part;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const float4 g4 = reinterpret_cast<const float4 *>(gs + 128 + r0)[q];
            gsc[4 * q] = a.scale * g4.x; gsc[4 * q + 1] = a.scale * g4.y;
            gsc[4 * q + 2] = a.scale * g4.z; gsc[4 * q + 3] = a.scale * g4.w;
          }
          tc::tmem_ld16(tmem + lane_off + COL_OA + r0, oa);
          tc::tmem_ld16(tmem + lane_off + COL_OB + r0, ob);
#pragma unroll
          for (int cc = 0; cc < 16; ++cc) {
            const int r = r0 + cc;
            const float val = gsc[cc] * oa[cc] + ob[cc];
            if (full) {
              io<OutT>::st(stage_o + r * DV + row, val);
            } else if (r < L) {
              io<OutT>::st(static_cast<OutT *>(a.o) + (obase + (size_t)r * a.Hv) * DV + row, val);
            }
          }
        }
        tc::tc_fence_before();
        warp_arrive(bar(B_OA_EMPTY), lane);  // Oa / Ob read: the next Oa MMA may overwrite
        if (full) {
          tc::fence_async_smem();
          tc::named_bar(2, 256);
          if (st == 0) {
            tc::tma_store_3d(&tm_o, sb + OFF_DH, 0, h, zbase + t0);
            tc::bulk_commit();
          }
        }
      }
      warp_arrive(bar(B_GATE_EMPTY + s), lane);
    }
    if (a.state_out) {
#pragma unroll
      for (int m = 0; m < 64; ++m) a.state_out[st_off + (size_t)(64 * swg + m) * DV + row] = Hr[m];
    }
    if (tid == 256) tc::bulk_wait_all();
  }

  tc::tc_fence_before();
  __syncwarp();  // single-lane roles rejoin their warp before the CTA barrier
  __syncthreads();
  if (warp == 0) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, TMEM_COLS);
  }
}

// ------------------------------------------------------------------ host side

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// [rows = B*T][heads][d] bf16 viewed as a 3-D tensor (d, heads, rows); box 64 x 1 x 64.
inline bool make_map(CUtensorMap *m, const void *base, int d, int heads, long long rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)heads, (cuuint64_t)rows};
  const cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)heads * d * 2};
  const cuuint32_t box[3] = {64, 1, 64};
  const cuuint32_t es[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box,
             es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Output o [rows = B*T][heads][d] (fp32 or bf16), box d x 1 x 64, no swizzle (row-major tile).
inline bool make_map_out(CUtensorMap *m, void *base, int d, int heads, long long rows, bool f32) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const int es_bytes = f32 ? 4 : 2;
  const cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)heads, (cuuint64_t)rows};
  const cuuint64_t strides[2] = {(cuuint64_t)d * es_bytes, (cuuint64_t)heads * d * es_bytes};
  const cuuint32_t box[3] = {(cuuint32_t)d, 1, 64};
  const cuuint32_t es[3] = {1, 1, 1};
  return enc(m, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, base,
             dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
             CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace tck

inline bool tc_supported(int dk, int dv) { return dk == 128 && dv == 128; }

inline cudaError_t tc_dispatch(int dk, int dv, bool out_f32, const PrefillArgs &a, int N,
                               cudaStream_t stream) {
  if (!tc_supported(dk, dv)) return cudaErrorNotSupported;
  if ((long long)a.B * a.T == 0) {  // no tokens: only the state copy, done by the CUDA-core kernel
    return out_f32 ? launch_chunk_simt<128, 128, __nv_bfloat16, float>(a, N, stream)
                   : launch_chunk_simt<128, 128, __nv_bfloat16, __nv_bfloat16>(a, N, stream);
  }
  CUtensorMap mq, mk, mv, mo;
  const long long rows = (long long)a.B * a.T;
  if (!tck::make_map(&mq, a.q, dk, a.Hqk, rows) || !tck::make_map(&mk, a.k, dk, a.Hqk, rows) ||
      !tck::make_map(&mv, a.v, dv, a.Hv, rows) ||
      !tck::make_map_out(&mo, a.o, dv, a.Hv, rows, out_f32))
    return cudaErrorInvalidValue;
  auto kern = out_f32 ? tck::chunk_tc_kernel<true> : tck::chunk_tc_kernel<false>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)tck::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  kern<<<(unsigned)N * (unsigned)a.Hv, tck::NT, tck::SMEM_BYTES, stream>>>(mq, mk, mv, mo, a);
  return cudaGetLastError();
}

}  // namespace dr
