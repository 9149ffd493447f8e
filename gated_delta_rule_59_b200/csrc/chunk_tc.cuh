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
// B200 mapping (one CTA of 256 threads per (sequence, v-head); the recurrence
// over chunks is sequential inside the CTA):
//  * Every matrix product is a tcgen05.mma (bf16 operands from shared memory,
//    fp32 accumulators in TMEM), issued by one thread.  All products are
//    arranged with M = 128 so the tensor core runs its full-width shape:
//        G     = [K; Q] K^T                 (rows 0-63: K K^T, 64-127: Q K^T)
//        W^T   = K^T (T diag(beta gamma))^T,  U^T = V^T (T diag(beta))^T
//        Delta^T = U^T + H0^T (-W^T)        (accumulates onto U^T in TMEM)
//        Oa    = H0^T Q^T,   Ob = Delta^T P^T   (O^T = diag(gamma) Oa + Ob)
//        Hupd  = Delta~^T K   with Delta~_s = e^{b_C - b_s} Delta_s
//  * The fp32 master state lives in registers (thread = one TMEM lane = one
//    value column j, 64 of the dk rows per warpgroup); a bf16 copy of H0^T in
//    shared memory is the MMA operand.  Each chunk the state update
//    H = gamma_C H + Hupd is done in registers from the TMEM accumulator.
//  * Q, K, V chunks arrive by TMA (128-byte swizzle, no multicast) one chunk
//    ahead into a second buffer.  Sequence starts need no alignment: rows past
//    the end of a sequence are neutralised by beta = g = 0.
//  * T = (I + L)^-1 is inverted in fp32 in shared memory by blocked forward
//    substitution (16x16 diagonal blocks, then three block-merge rounds).
//  * Precision: operands computed in fp32 inside the kernel (T diag(beta),
//    T diag(beta gamma), P, Delta, Delta~) are fed to the tensor core as a
//    bf16 pair x = hi + lo (hi = bf16(x), lo = bf16(x - hi)), two MMAs into the
//    same accumulator (three for P Delta, dropping lo x lo).  A single bf16
//    rounding of these (2^-8 relative) alone exceeds the 2e-2 max/RMS error
//    budget on short sequences; the pair keeps ~2^-16.  Inputs (q, k, v) are
//    exact in bf16; the H0 operand stays a single bf16 copy.
#pragma once

#include <cuda.h>

#include <mutex>

#include "chunk_simt.cuh"
#include "tc_ptx.cuh"

namespace dr {
namespace tck {

constexpr int C = 64, DK = 128, DV = 128, NT = 256;
constexpr float LOG2E = 1.4426950408889634f;

// shared-memory map (bytes from a 1024-aligned base).  Regions R1-R3 are reused
// by operands whose lifetimes within a chunk do not overlap.
constexpr uint32_t STAGE_BYTES = 49152;  // K0 Q0 K1 Q1 V0 V1, 8 KB each
constexpr uint32_t OFF_K0 = 0, OFF_Q0 = 8192, OFF_K1 = 16384, OFF_Q1 = 24576;
constexpr uint32_t OFF_V0 = 32768, OFF_V1 = 40960;
constexpr uint32_t OFF_H = 2 * STAGE_BYTES;  // H0^T bf16, 2 x 16 KB (K-major, k = dk)
constexpr uint32_t OFF_R1 = OFF_H + 32768;   // L fp32 [64][65]          | Delta^T lo
constexpr uint32_t OFF_R2 = OFF_R1 + 17408;  // T fp32 [64][64] | -W^T   | Delta~^T lo
constexpr uint32_t OFF_R3 = OFF_R2 + 16384;  // merge scratch | T diag(beta), T diag(beta gamma)
                                             //   (hi, lo: 4 x 8 KB) | Delta^T hi, Delta~^T hi
constexpr uint32_t OFF_R4 = OFF_R3 + 32768;  // P hi, P lo (8 KB each)
constexpr uint32_t OFF_TB_H = OFF_R3, OFF_TB_L = OFF_R3 + 8192;
constexpr uint32_t OFF_TBG_H = OFF_R3 + 16384, OFF_TBG_L = OFF_R3 + 24576;
constexpr uint32_t OFF_W = OFF_R2;
constexpr uint32_t OFF_D_H = OFF_R3, OFF_DT_H = OFF_R3 + 16384;
constexpr uint32_t OFF_D_L = OFF_R1, OFF_DT_L = OFF_R2;
constexpr uint32_t OFF_P_H = OFF_R4, OFF_P_L = OFF_R4 + 8192;
constexpr uint32_t OFF_L = OFF_R1, OFF_T = OFF_R2, OFF_X = OFF_R3;
constexpr uint32_t OFF_SMALL = OFF_R4 + 16384;
constexpr uint32_t SMALL_BYTES = 4 * 64 * 4 + 64;
constexpr uint32_t SMEM_BYTES = OFF_SMALL + SMALL_BYTES + 1024;  // + alignment slack
static_assert(SMEM_BYTES <= 232448, "shared memory budget");
static_assert(OFF_R2 % 1024 == 0 && OFF_R3 % 1024 == 0 && OFF_R4 % 1024 == 0, "tile alignment");

// TMEM columns (fp32 accumulators, 128 lanes each)
constexpr uint32_t COL_G = 0, COL_W = 64, COL_DU = 128, COL_OA = 192, COL_OB = 256, COL_HU = 320;
constexpr uint32_t TMEM_COLS = 512;

constexpr uint32_t ID_G = tc::idesc_bf16(128, 64, 0, 0);    // [K;Q] K^T
constexpr uint32_t ID_MNK = tc::idesc_bf16(128, 64, 1, 0);  // K^T / V^T (MN-major A) x K-major B
constexpr uint32_t ID_KMN64 = tc::idesc_bf16(128, 64, 0, 1);    // H0^T x (-W^T), MN-major B
constexpr uint32_t ID_KK64 = tc::idesc_bf16(128, 64, 0, 0);     // H0^T Q^T, Delta^T P^T
constexpr uint32_t ID_KMN128 = tc::idesc_bf16(128, 128, 0, 1);  // Delta~^T K

// Write 8 fp32 values as one 16-byte bf16 chunk of a swizzled 128-byte row.
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

template <bool OUT_F32>
__global__ void __launch_bounds__(NT, 1)
    chunk_tc_kernel(const __grid_constant__ CUtensorMap tm_q,
                    const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, PrefillArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = tc::smem_u32(smem);
  float *bs2 = reinterpret_cast<float *>(smem + OFF_SMALL);  // b * log2(e)
  float *betas = bs2 + 64;
  float *gam = betas + 64;   // e^{b_r}
  float *dtil = gam + 64;    // e^{b_C - b_r}
  uint64_t *bars = reinterpret_cast<uint64_t *>(dtil + 64);  // full0, full1, mma
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 3);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
  float *Lf = reinterpret_cast<float *>(smem + OFF_L);  // [64][65]
  float *Tf = reinterpret_cast<float *>(smem + OFF_T);  // [64][64]
  float *Xf = reinterpret_cast<float *>(smem + OFF_X);  // merge scratch
  const uint32_t bar_full[2] = {tc::smem_u32(&bars[0]), tc::smem_u32(&bars[1])};
  const uint32_t bar_mma = tc::smem_u32(&bars[2]);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int wg = warp >> 2, q4 = warp & 3;
  const int row = 32 * q4 + lane;  // the TMEM lane (accumulator row) this thread reads
  const uint32_t lane_off = (uint32_t)(32 * q4) << 16;

  const int unit = blockIdx.x, n = unit / a.Hv, h = unit % a.Hv;
  const int hq = h / (a.Hv / a.Hqk);
  int batch, bos, eos;
  if (!seq_bounds(a.cu_seqlens, n, a.n_seqs, a.T, batch, bos, eos)) return;  // CTA-uniform
  const float scale = a.scale;
  const size_t st_off = ((size_t)n * a.Hv + h) * DK * DV;

  if (tid == 0) {
    tc::mbar_init(bar_full[0], 1);
    tc::mbar_init(bar_full[1], 1);
    tc::mbar_init(bar_mma, 1);
    *abort_flag = 0;
    tc::fence_barrier_init();
    tc::prefetch_tmap(&tm_q);
    tc::prefetch_tmap(&tm_k);
    tc::prefetch_tmap(&tm_v);
  }
  if (warp == 0) {
    tc::tmem_alloc(tc::smem_u32(tmem_slot), TMEM_COLS);
    tc::tmem_relinquish();
  }

  // Master state: this thread owns H[i][row] for i in [64 wg, 64 wg + 64).
  float Hr[64];
#pragma unroll
  for (int m = 0; m < 64; ++m)
    Hr[m] = a.state_in ? a.state_in[st_off + (size_t)(64 * wg + m) * DV + row] : 0.f;
  auto write_shadow = [&]() {
    const uint32_t tile = sb + OFF_H + (uint32_t)wg * 16384u;
#pragma unroll
    for (int cc = 0; cc < 8; ++cc) st_row_chunk(tile, row, cc, &Hr[8 * cc]);
  };
  write_shadow();
  tc::fence_async_smem();
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  const int nchunks = (eos - bos + C - 1) / C;
  const int zbase = batch * a.T;  // token row of (batch, t = 0) in the [B*T] axis
  auto issue_tma = [&](int stage, int t0) {
    const uint32_t dst = sb + (uint32_t)stage * STAGE_BYTES;
    const int z = zbase + t0;
    tc::mbar_arrive_expect_tx(bar_full[stage], STAGE_BYTES);
    tc::tma_load_3d(dst + OFF_K0, &tm_k, bar_full[stage], 0, hq, z);
    tc::tma_load_3d(dst + OFF_K1, &tm_k, bar_full[stage], 64, hq, z);
    tc::tma_load_3d(dst + OFF_Q0, &tm_q, bar_full[stage], 0, hq, z);
    tc::tma_load_3d(dst + OFF_Q1, &tm_q, bar_full[stage], 64, hq, z);
    tc::tma_load_3d(dst + OFF_V0, &tm_v, bar_full[stage], 0, h, z);
    tc::tma_load_3d(dst + OFF_V1, &tm_v, bar_full[stage], 64, h, z);
  };
  int tma_issued = 0;  // chunks whose loads have been issued (thread 0 only)
  if (tid == 0 && nchunks > 0) {
    issue_tma(0, bos);
    tma_issued = 1;
  }
  uint32_t mma_phase = 0;
  auto mma_wait = [&]() {
    tc::mbar_wait(bar_mma, mma_phase, abort_flag);
    mma_phase ^= 1u;
    tc::tc_fence_after();
  };
  auto sync_for_mma = [&]() {  // smem writes + TMEM reads done -> next MMA may run
    tc::fence_async_smem();
    tc::tc_fence_before();
    __syncthreads();
  };

  // gates / write strengths of the next chunk are loaded one chunk ahead (warp 0)
  float gn0 = 0.f, gn1 = 0.f, bn0 = 0.f, bn1 = 0.f;
  auto load_gb = [&](int t0) {
    const int L = min(C, eos - t0);
    const size_t i0 = ((size_t)zbase + t0 + lane) * a.Hv + h;
    gn0 = gn1 = bn0 = bn1 = 0.f;
    if (lane < L) {
      gn0 = a.g ? a.g[i0] : 0.f;
      bn0 = a.beta[i0];
    }
    if (lane + 32 < L) {
      gn1 = a.g ? a.g[i0 + (size_t)32 * a.Hv] : 0.f;
      bn1 = a.beta[i0 + (size_t)32 * a.Hv];
    }
  };
  if (warp == 0 && nchunks > 0) load_gb(bos);

  for (int c = 0; c < nchunks; ++c) {
    const int t0 = bos + c * C;
    const int L = min(C, eos - t0);
    const int s = c & 1;
    const uint32_t stg = sb + (uint32_t)s * STAGE_BYTES;

    // ---- cumulative log decay of this chunk (rows past the end have g = beta = 0) ----
    if (warp == 0) {
      float g0 = gn0, g1 = gn1;
      const float b0 = bn0, b1 = bn1;
      if (c + 1 < nchunks) load_gb(t0 + C);
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
      bs2[lane] = g0 * LOG2E;
      bs2[lane + 32] = g1 * LOG2E;
      betas[lane] = b0;
      betas[lane + 32] = b1;
      gam[lane] = exp2f(g0 * LOG2E);
      gam[lane + 32] = exp2f(g1 * LOG2E);
      dtil[lane] = exp2f((blast - g0) * LOG2E);
      dtil[lane + 32] = exp2f((blast - g1) * LOG2E);
    }
    if (tid == 0 && c + 1 < nchunks) {
      issue_tma(s ^ 1, t0 + C);
      ++tma_issued;
    }
    tc::mbar_wait(bar_full[s], (uint32_t)(c >> 1) & 1u, abort_flag);
    __syncthreads();

    // ---- G = [K; Q] K^T  (M=128, N=64, K=128) ----
    if (tid == 0 && !*abort_flag) {
      tc::tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const uint32_t at = stg + (kk >> 2) * 16384u + (kk & 3) * 32u;
        const uint64_t d = tc::sdesc_sw128(at, 16, 1024);
        tc::mma_bf16(tmem + COL_G, d, d, ID_G, kk > 0);
      }
      tc::mma_commit(bar_mma);
    }
    mma_wait();
    {
      float v[32];
      tc::tmem_ld32(tmem + lane_off + COL_G + 32 * wg, v);
      if (row < 64) {  // L row r: beta_r Gamma_rs (k_r . k_s), s < r
        const int r = row;
        const float br = bs2[r], bt = betas[r];
#pragma unroll
        for (int cc = 0; cc < 32; ++cc) {
          const int s_ = 32 * wg + cc;
          Lf[r * 65 + s_] = (s_ < r) ? bt * exp2f(br - bs2[s_]) * v[cc] : 0.f;
        }
      } else {  // P row r: scale Gamma_rs (q_r . k_s), s <= r  -> bf16, K-major B tile
        const int r = row - 64;
        const float br = bs2[r];
#pragma unroll
        for (int cc = 0; cc < 32; ++cc) {
          const int s_ = 32 * wg + cc;
          v[cc] = (s_ <= r) ? scale * exp2f(br - bs2[s_]) * v[cc] : 0.f;
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) st_row_chunk_split(sb + OFF_P_H, sb + OFF_P_L, r, 4 * wg + q, &v[8 * q]);
      }
    }
    tc::tc_fence_before();
    __syncthreads();

    // ---- T = (I + L)^-1: 16x16 diagonal blocks by forward substitution ----
    if (tid < 64) {
      const int blk = tid >> 4, cI = tid & 15, R = 16 * blk;
      float x[16];
#pragma unroll
      for (int r = 0; r < 16; ++r) x[r] = (r == cI) ? 1.f : 0.f;
#pragma unroll
      for (int r = 1; r < 16; ++r) {
        float acc = 0.f;
#pragma unroll
        for (int q = 0; q < r; ++q) acc += Lf[(R + r) * 65 + R + q] * x[q];
        if (r > cI) x[r] = -acc;
      }
#pragma unroll
      for (int r = 0; r < 16; ++r) Tf[(R + r) * 64 + R + cI] = x[r];
    }
    __syncthreads();
    // ---- block merges: T_ij = -T_ii sum_{k=j}^{i-1} L_ik T_kj, by distance d = i - j ----
#pragma unroll 1
    for (int d = 1; d < 4; ++d) {
      const int nblk = 4 - d;
      for (int e = tid; e < nblk * 256; e += NT) {  // X = sum_k L_ik T_kj
        const int bi = e >> 8, rc = e & 255, r = rc >> 4, cI = rc & 15;
        const int i = bi + d, j = bi;
        float acc = 0.f;
        for (int k = j; k < i; ++k) {
#pragma unroll
          for (int m = 0; m < 16; ++m)
            acc += Lf[(16 * i + r) * 65 + 16 * k + m] * Tf[(16 * k + m) * 64 + 16 * j + cI];
        }
        Xf[e] = acc;
      }
      __syncthreads();
      for (int e = tid; e < nblk * 256; e += NT) {  // T_ij = -T_ii X
        const int bi = e >> 8, rc = e & 255, r = rc >> 4, cI = rc & 15;
        const int i = bi + d, j = bi;
        float acc = 0.f;
#pragma unroll
        for (int m = 0; m < 16; ++m)
          acc += Tf[(16 * i + r) * 64 + 16 * i + m] * Xf[(bi << 8) + m * 16 + cI];
        Tf[(16 * i + r) * 64 + 16 * j + cI] = -acc;
      }
      __syncthreads();
    }
    // ---- T diag(beta) and T diag(beta gamma) as bf16 hi/lo K-major B tiles ----
    for (int e = tid; e < 64 * 8; e += NT) {
      const int r = e >> 3, q = e & 7;
      float tb[8], tbg[8];
#pragma unroll
      for (int m = 0; m < 8; ++m) {
        const int s_ = 8 * q + m;
        const float t = (s_ <= r) ? Tf[r * 64 + s_] : 0.f;
        tb[m] = t * betas[s_];
        tbg[m] = tb[m] * gam[s_];
      }
      st_row_chunk_split(sb + OFF_TB_H, sb + OFF_TB_L, r, q, tb);
      st_row_chunk_split(sb + OFF_TBG_H, sb + OFF_TBG_L, r, q, tbg);
    }
    sync_for_mma();

    // ---- W^T = K^T (T diag(beta gamma))^T,  U^T = V^T (T diag(beta))^T  (M=128, N=64, K=64) ----
    if (tid == 0 && !*abort_flag) {
      tc::tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const uint64_t ak = tc::sdesc_sw128(stg + OFF_K0 + kk * 2048u, 16384, 1024);
        const uint64_t av = tc::sdesc_sw128(stg + OFF_V0 + kk * 2048u, 8192, 1024);
        tc::mma_bf16(tmem + COL_W, ak, tc::sdesc_sw128(sb + OFF_TBG_H + kk * 32u, 16, 1024), ID_MNK, kk > 0);
        tc::mma_bf16(tmem + COL_W, ak, tc::sdesc_sw128(sb + OFF_TBG_L + kk * 32u, 16, 1024), ID_MNK, 1);
        tc::mma_bf16(tmem + COL_DU, av, tc::sdesc_sw128(sb + OFF_TB_H + kk * 32u, 16, 1024), ID_MNK, kk > 0);
        tc::mma_bf16(tmem + COL_DU, av, tc::sdesc_sw128(sb + OFF_TB_L + kk * 32u, 16, 1024), ID_MNK, 1);
      }
      tc::mma_commit(bar_mma);
    }
    mma_wait();
    {  // -W^T -> bf16 (row i = TMEM lane, 64 values of r: MN-major B for the Delta product)
      float v[32];
      tc::tmem_ld32(tmem + lane_off + COL_W + 32 * wg, v);
#pragma unroll
      for (int cc = 0; cc < 32; ++cc) v[cc] = -v[cc];
#pragma unroll
      for (int q = 0; q < 4; ++q) st_row_chunk(sb + OFF_W, row, 4 * wg + q, &v[8 * q]);
    }
    sync_for_mma();

    // ---- Delta^T = U^T + H0^T (-W^T) (K=128, onto U^T);  Oa = H0^T Q^T ----
    if (tid == 0 && !*abort_flag) {
      tc::tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const uint64_t ah = tc::sdesc_sw128(sb + OFF_H + (kk >> 2) * 16384u + (kk & 3) * 32u, 16, 1024);
        const uint64_t bw = tc::sdesc_sw128(sb + OFF_W + kk * 2048u, 8192, 1024);
        const uint64_t bq = tc::sdesc_sw128(stg + OFF_Q0 + (kk >> 2) * 16384u + (kk & 3) * 32u, 16, 1024);
        tc::mma_bf16(tmem + COL_DU, ah, bw, ID_KMN64, 1);
        tc::mma_bf16(tmem + COL_OA, ah, bq, ID_KK64, kk > 0);
      }
      tc::mma_commit(bar_mma);
    }
    mma_wait();
    {  // Delta^T and Delta~^T (scaled by e^{b_C - b_s}) -> bf16 hi/lo K-major A tiles
      float v[32], w[32];
      tc::tmem_ld32(tmem + lane_off + COL_DU + 32 * wg, v);
#pragma unroll
      for (int cc = 0; cc < 32; ++cc) w[cc] = v[cc] * dtil[32 * wg + cc];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        st_row_chunk_split(sb + OFF_D_H, sb + OFF_D_L, row, 4 * wg + q, &v[8 * q]);
        st_row_chunk_split(sb + OFF_DT_H, sb + OFF_DT_L, row, 4 * wg + q, &w[8 * q]);
      }
    }
    sync_for_mma();

    // ---- Ob = Delta^T P^T (N=64, K=64);  Hupd = Delta~^T K (N=128, K=64); hi/lo pairs ----
    if (tid == 0 && !*abort_flag) {
      tc::tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const uint64_t adh = tc::sdesc_sw128(sb + OFF_D_H + kk * 32u, 16, 1024);
        const uint64_t adl = tc::sdesc_sw128(sb + OFF_D_L + kk * 32u, 16, 1024);
        const uint64_t bph = tc::sdesc_sw128(sb + OFF_P_H + kk * 32u, 16, 1024);
        const uint64_t bpl = tc::sdesc_sw128(sb + OFF_P_L + kk * 32u, 16, 1024);
        const uint64_t bk = tc::sdesc_sw128(stg + OFF_K0 + kk * 2048u, 16384, 1024);
        tc::mma_bf16(tmem + COL_OB, adh, bph, ID_KK64, kk > 0);
        tc::mma_bf16(tmem + COL_OB, adl, bph, ID_KK64, 1);
        tc::mma_bf16(tmem + COL_OB, adh, bpl, ID_KK64, 1);
        tc::mma_bf16(tmem + COL_HU, tc::sdesc_sw128(sb + OFF_DT_H + kk * 32u, 16, 1024), bk, ID_KMN128, kk > 0);
        tc::mma_bf16(tmem + COL_HU, tc::sdesc_sw128(sb + OFF_DT_L + kk * 32u, 16, 1024), bk, ID_KMN128, 1);
      }
      tc::mma_commit(bar_mma);
    }
    mma_wait();
    {  // outputs: O[r][j] = scale gamma_r Oa[j][r] + Ob[j][r]
      float oa[32], ob[32];
      tc::tmem_ld32(tmem + lane_off + COL_OA + 32 * wg, oa);
      tc::tmem_ld32(tmem + lane_off + COL_OB + 32 * wg, ob);
      const size_t obase = ((size_t)zbase + t0) * a.Hv + h;
#pragma unroll
      for (int cc = 0; cc < 32; ++cc) {
        const int r = 32 * wg + cc;
        if (r < L) {
          const float val = scale * gam[r] * oa[cc] + ob[cc];
          const size_t off = (obase + (size_t)r * a.Hv) * DV + row;
          if constexpr (OUT_F32)
            static_cast<float *>(a.o)[off] = val;
          else
            static_cast<__nv_bfloat16 *>(a.o)[off] = __float2bfloat16_rn(val);
        }
      }
    }
    {  // state: H = gamma_C H + Hupd; refresh the bf16 shadow
      const float gC = gam[63];
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        float u[32];
        tc::tmem_ld32(tmem + lane_off + COL_HU + 64 * wg + 32 * half, u);
#pragma unroll
        for (int m = 0; m < 32; ++m) Hr[32 * half + m] = gC * Hr[32 * half + m] + u[m];
      }
      write_shadow();
    }
    sync_for_mma();
    tc::tc_fence_after();
  }

  if (a.state_out) {
#pragma unroll
    for (int m = 0; m < 64; ++m) a.state_out[st_off + (size_t)(64 * wg + m) * DV + row] = Hr[m];
  }
  // Wind down: make sure no TMA write into this CTA's shared memory is still in flight.
  if (tid == 0 && *abort_flag) {
    for (int c = 0; c < tma_issued; ++c) tc::mbar_wait(bar_full[c & 1], (uint32_t)(c >> 1) & 1u, abort_flag, 1u << 20);
  }
  tc::tc_fence_before();
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

}  // namespace tck

inline bool tc_supported(int dk, int dv) { return dk == 128 && dv == 128; }

inline cudaError_t tc_dispatch(int dk, int dv, bool out_f32, const PrefillArgs &a, int N,
                               cudaStream_t stream) {
  if (!tc_supported(dk, dv)) return cudaErrorNotSupported;
  if ((long long)a.B * a.T == 0) {  // no tokens: only the state copy, done by the CUDA-core kernel
    return out_f32 ? launch_chunk_simt<128, 128, __nv_bfloat16, float>(a, N, stream)
                   : launch_chunk_simt<128, 128, __nv_bfloat16, __nv_bfloat16>(a, N, stream);
  }
  CUtensorMap mq, mk, mv;
  const long long rows = (long long)a.B * a.T;
  if (!tck::make_map(&mq, a.q, dk, a.Hqk, rows) || !tck::make_map(&mk, a.k, dk, a.Hqk, rows) ||
      !tck::make_map(&mv, a.v, dv, a.Hv, rows))
    return cudaErrorInvalidValue;
  auto kern = out_f32 ? tck::chunk_tc_kernel<true> : tck::chunk_tc_kernel<false>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)tck::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  kern<<<(unsigned)N * (unsigned)a.Hv, tck::NT, tck::SMEM_BYTES, stream>>>(mq, mk, mv, a);
  return cudaGetLastError();
}

}  // namespace dr
