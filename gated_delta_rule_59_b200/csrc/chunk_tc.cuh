// chunk_tc.cuh -- shared pieces of the tcgen05 tensor-core chunked prefill (bf16, dk = dv = 128).
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
// This file holds the pieces of that algebra shared by the tensor-core prefill kernel
// (chunk_pair.cuh): the MMA instruction descriptors, the swizzled operand-tile stores, the
// block merges of the triangular inverse and the TMA tensor maps.
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

constexpr int C = 64, DK = 128, DV = 128;
constexpr float LOG2E = 1.4426950408889634f;

constexpr uint32_t ID_G = tc::idesc_bf16(128, 64, 0, 0);        // [K;Q] K^T
constexpr uint32_t ID_MNK = tc::idesc_bf16(128, 64, 1, 0);      // K^T / V^T x T^T
constexpr uint32_t ID_KMN64 = tc::idesc_bf16(128, 64, 0, 1);    // H0^T x (-W^T)
constexpr uint32_t ID_KK64 = tc::idesc_bf16(128, 64, 0, 0);     // H0^T Q^T, Delta^T P^T
constexpr uint32_t ID_KMN128 = tc::idesc_bf16(128, 128, 0, 1);  // Delta~^T K

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

}  // namespace dr
