// dr_lib.cu -- the C ABI of libdr.so (declared in include/dr.h).
//
// Host side only: argument validation (before anything is launched), dtype and
// head-dimension dispatch, launch on the caller's stream, status mapping.  All
// kernels are compiled into this one translation unit so that they share the
// device status word without relocatable device code.
#include <cmath>
#include <cstdint>

#include "dr.h"
#include "dr_common.cuh"
#include "decode.cuh"
#include "chunk_simt.cuh"
#include "chunk_tc.cuh"
#include "chunk_pair.cuh"
#include "layer.cuh"

#define DR_VERSION_NUMBER 100  // 0.1.0

namespace {

bool dim_ok(int d) { return d == 16 || d == 32 || d == 64 || d == 128; }
bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }
bool dtype_ok(dr_dtype t) { return t == DR_F32 || t == DR_BF16; }

template <typename Tin, typename Tout>
cudaError_t decode_dispatch(int dk, int dv, const void *q, const void *k, const void *v,
                            const float *g, const float *beta, float *state, int B, int Hqk,
                            int Hv, float scale, void *o, int l2n, int cg, cudaStream_t s) {
#define DR_DEC(DK, DV)                                                                  \
  if (dk == DK && dv == DV)                                                             \
    return dr::launch_decode<DK, DV, Tin, Tout>(q, k, v, g, beta, state, B, Hqk, Hv, scale, o, \
                                                l2n, cg, s);
#define DR_DEC_ROW(DK) DR_DEC(DK, 16) DR_DEC(DK, 32) DR_DEC(DK, 64) DR_DEC(DK, 128)
  DR_DEC_ROW(16) DR_DEC_ROW(32) DR_DEC_ROW(64) DR_DEC_ROW(128)
#undef DR_DEC_ROW
#undef DR_DEC
  return cudaErrorInvalidValue;
}

template <typename Tin, typename Tout>
cudaError_t simt_dispatch(int dk, int dv, const dr::PrefillArgs &a, int N, cudaStream_t s) {
#define DR_SIMT(DK, DV) \
  if (dk == DK && dv == DV) return dr::launch_chunk_simt<DK, DV, Tin, Tout>(a, N, s);
#define DR_SIMT_ROW(DK) DR_SIMT(DK, 16) DR_SIMT(DK, 32) DR_SIMT(DK, 64) DR_SIMT(DK, 128)
  DR_SIMT_ROW(16) DR_SIMT_ROW(32) DR_SIMT_ROW(64) DR_SIMT_ROW(128)
#undef DR_SIMT_ROW
#undef DR_SIMT
  return cudaErrorInvalidValue;
}

template <typename Tin>
cudaError_t simt_dispatch_out(dr_dtype od, int dk, int dv, const dr::PrefillArgs &a, int N,
                              cudaStream_t s) {
  return od == DR_F32 ? simt_dispatch<Tin, float>(dk, dv, a, N, s)
                      : simt_dispatch<Tin, __nv_bfloat16>(dk, dv, a, N, s);
}

template <typename Tin, typename Tout>
cudaError_t launch_conv(const void *x, const float *w, int K, const float *state_in,
                        const int32_t *cu, int n_seqs, int T, long long P, int C, void *y,
                        cudaStream_t s) {
  if (P == 0) return cudaSuccess;
  const dim3 grid((unsigned)((P + dr::CONV_TOK - 1) / dr::CONV_TOK), (unsigned)((C + 127) / 128));
  dr::conv_silu_kernel<Tin, Tout><<<grid, 128, 0, s>>>((const Tin *)x, w, K, state_in, cu,
                                                       cu ? n_seqs : 1, T, P, C, (Tout *)y);
  return cudaGetLastError();
}

template <typename Tin>
cudaError_t conv_dispatch_out(dr_dtype yd, const void *x, const float *w, int K,
                              const float *state_in, const int32_t *cu, int n_seqs, int T,
                              long long P, int C, void *y, cudaStream_t s) {
  return yd == DR_F32 ? launch_conv<Tin, float>(x, w, K, state_in, cu, n_seqs, T, P, C, y, s)
                      : launch_conv<Tin, __nv_bfloat16>(x, w, K, state_in, cu, n_seqs, T, P, C, y, s);
}

template <typename Tin>
cudaError_t launch_conv_state(const void *x, int K, const float *state_in, const int32_t *cu,
                              int n_seqs, int N, int T, int C, float *state_out, cudaStream_t s) {
  const long long threads = (long long)N * C;
  if (threads == 0 || K == 1) return cudaSuccess;
  dr::conv_state_kernel<Tin><<<(unsigned)((threads + 127) / 128), 128, 0, s>>>(
      (const Tin *)x, K, state_in, cu, n_seqs, N, T, C, state_out);
  return cudaGetLastError();
}

template <typename Tin, typename Tz>
cudaError_t norm_dispatch_out(dr_dtype yd, const void *o, const float *wt, const float *bias,
                              const void *z, long long rows, int dv, int layer, float eps, void *y,
                              cudaStream_t s) {
  const unsigned blocks = (unsigned)((rows + 7) / 8);
  if (yd == DR_F32)
    dr::norm_gate_kernel<Tin, Tz, float><<<blocks, 256, 0, s>>>(
        (const Tin *)o, wt, bias, (const Tz *)z, rows, dv, layer, eps, (float *)y);
  else
    dr::norm_gate_kernel<Tin, Tz, __nv_bfloat16><<<blocks, 256, 0, s>>>(
        (const Tin *)o, wt, bias, (const Tz *)z, rows, dv, layer, eps, (__nv_bfloat16 *)y);
  return cudaGetLastError();
}

size_t dsize(dr_dtype t) { return t == DR_F32 ? 4 : 2; }

}  // namespace

extern "C" {

dr_status dr_short_conv_silu(const void *x, dr_dtype x_dtype, const float *w, int32_t K,
                             const float *conv_state_in, float *conv_state_out,
                             const int32_t *cu_seqlens, int32_t n_seqs, int32_t B, int32_t T,
                             int32_t C, void *y, dr_dtype y_dtype, dr_stream stream) {
  if (!dtype_ok(x_dtype) || !dtype_ok(y_dtype)) return DR_ERR_DTYPE;
  if (B < 0 || T < 0 || C <= 0 || K < 1) return DR_ERR_SHAPE;
  if (K > dr::CONV_MAX_K) return DR_ERR_UNSUPPORTED;
  if (cu_seqlens && (B != 1 || n_seqs < 0)) return DR_ERR_SHAPE;
  const long long P = (long long)B * T;
  if (cu_seqlens && n_seqs == 0 && P > 0) return DR_ERR_SHAPE;
  const int64_t N = cu_seqlens ? n_seqs : B;
  if (P > 0 && (!x || !w || !y)) return DR_ERR_NULL;
  if (!aligned(x, dsize(x_dtype)) || !aligned(y, dsize(y_dtype)) || !aligned(w, 4) ||
      !aligned(conv_state_in, 4) || !aligned(conv_state_out, 4) || !aligned(cu_seqlens, 4))
    return DR_ERR_ALIGN;
  if ((P + dr::CONV_TOK - 1) / dr::CONV_TOK > 0x7fffffffLL || (C + 127) / 128 > 65535 ||
      N * (int64_t)C > 0x3fffffffffLL)
    return DR_ERR_UNSUPPORTED;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e;
  if (x_dtype == DR_F32)
    e = conv_dispatch_out<float>(y_dtype, x, w, K, conv_state_in, cu_seqlens, n_seqs, T, P, C, y, s);
  else
    e = conv_dispatch_out<__nv_bfloat16>(y_dtype, x, w, K, conv_state_in, cu_seqlens, n_seqs, T, P,
                                         C, y, s);
  if (e == cudaSuccess && conv_state_out)
    e = x_dtype == DR_F32
            ? launch_conv_state<float>(x, K, conv_state_in, cu_seqlens, n_seqs, (int)N, T, C,
                                       conv_state_out, s)
            : launch_conv_state<__nv_bfloat16>(x, K, conv_state_in, cu_seqlens, n_seqs, (int)N, T,
                                               C, conv_state_out, s);
  return e == cudaSuccess ? DR_OK : DR_ERR_CUDA;
}

dr_status dr_norm_gate(const void *o, dr_dtype o_dtype, const float *weight, const float *bias,
                       const void *z, dr_dtype z_dtype, int64_t rows, int32_t dv, int32_t kind,
                       float eps, void *y, dr_dtype y_dtype, dr_stream stream) {
  if (!dtype_ok(o_dtype) || !dtype_ok(y_dtype) || (z && !dtype_ok(z_dtype))) return DR_ERR_DTYPE;
  if (rows < 0 || dv <= 0) return DR_ERR_SHAPE;
  if (dv > 128 || (kind != DR_NORM_RMS && kind != DR_NORM_LAYER) || !(eps >= 0.f) ||
      !std::isfinite(eps))
    return DR_ERR_UNSUPPORTED;
  if (rows == 0) return DR_OK;
  if (!o || !weight || !y) return DR_ERR_NULL;
  if (!aligned(o, dsize(o_dtype)) || !aligned(y, dsize(y_dtype)) || !aligned(weight, 4) ||
      !aligned(bias, 4) || (z && !aligned(z, dsize(z_dtype))))
    return DR_ERR_ALIGN;
  if ((rows + 7) / 8 > 0x7fffffffLL) return DR_ERR_UNSUPPORTED;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int layer = kind == DR_NORM_LAYER ? 1 : 0;
  const bool zf = z == nullptr || z_dtype == DR_F32;
  cudaError_t e;
  if (o_dtype == DR_F32)
    e = zf ? norm_dispatch_out<float, float>(y_dtype, o, weight, bias, z, rows, dv, layer, eps, y, s)
           : norm_dispatch_out<float, __nv_bfloat16>(y_dtype, o, weight, bias, z, rows, dv, layer,
                                                     eps, y, s);
  else
    e = zf ? norm_dispatch_out<__nv_bfloat16, float>(y_dtype, o, weight, bias, z, rows, dv, layer,
                                                     eps, y, s)
           : norm_dispatch_out<__nv_bfloat16, __nv_bfloat16>(y_dtype, o, weight, bias, z, rows, dv,
                                                             layer, eps, y, s);
  return e == cudaSuccess ? DR_OK : DR_ERR_CUDA;
}


dr_status dr_chunk_fwd(const void *q, const void *k, const void *v, const float *g,
                       const float *beta, const float *state_in, const int32_t *cu_seqlens,
                       int32_t n_seqs, int32_t B, int32_t T, int32_t Hqk, int32_t Hv,
                       int32_t dk, int32_t dv, dr_dtype in_dtype, float scale, void *o,
                       dr_dtype o_dtype, float *state_out, float *chunk_states,
                       uint32_t flags, dr_stream stream) {
  if (!dtype_ok(in_dtype) || !dtype_ok(o_dtype)) return DR_ERR_DTYPE;
  if (flags & ~(DR_QK_L2NORM | DR_GATE_PER_CHANNEL)) return DR_ERR_UNSUPPORTED;
  if (B < 0 || T < 0 || Hqk <= 0 || Hv <= 0 || dk <= 0 || dv <= 0) return DR_ERR_SHAPE;
  if (Hv % Hqk != 0) return DR_ERR_SHAPE;
  if (cu_seqlens && (B != 1 || n_seqs < 0)) return DR_ERR_SHAPE;
  if (!dim_ok(dk) || !dim_ok(dv)) return DR_ERR_UNSUPPORTED;
  if (!std::isfinite(scale)) return DR_ERR_UNSUPPORTED;
  const int64_t N = cu_seqlens ? n_seqs : B;
  const bool tokens = (int64_t)B * T > 0;
  const bool cg = (flags & DR_GATE_PER_CHANNEL) != 0;
  if (tokens && (!q || !k || !v || !beta || !o || (cg && !g))) return DR_ERR_NULL;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) ||
      !aligned(state_in, 16) || !aligned(state_out, 16) || !aligned(chunk_states, 16) ||
      !aligned(g, 4) ||
      !aligned(beta, 4) || !aligned(cu_seqlens, 4))
    return DR_ERR_ALIGN;
  if (N == 0) return DR_OK;
  if (N * Hv > 0x3fffffff) return DR_ERR_UNSUPPORTED;  // grid x of the CTA-pair launch: 2 N Hv

  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  dr::PrefillArgs a{q, k, v, g, beta, state_in, cu_seqlens, (int)N, B, T, Hqk, Hv,
                    scale, o, state_out, (flags & DR_QK_L2NORM) ? 1 : 0, chunk_states,
                    cg ? 1 : 0};
  cudaError_t e;
  if (in_dtype == DR_BF16 && dr::tc_supported(dk, dv) && !cg) {
    e = dr::prefill_tc_dispatch(dk, dv, o_dtype == DR_F32, a, (int)N, s);
  } else if (in_dtype == DR_F32) {
    e = simt_dispatch_out<float>(o_dtype, dk, dv, a, (int)N, s);
  } else {
    e = simt_dispatch_out<__nv_bfloat16>(o_dtype, dk, dv, a, (int)N, s);
  }
  return e == cudaSuccess ? DR_OK : DR_ERR_CUDA;
}

dr_status dr_recurrent_step(const void *q, const void *k, const void *v, const float *g,
                            const float *beta, float *state, int32_t B, int32_t Hqk,
                            int32_t Hv, int32_t dk, int32_t dv, dr_dtype in_dtype,
                            float scale, void *o, dr_dtype o_dtype, uint32_t flags,
                            dr_stream stream) {
  if (!dtype_ok(in_dtype) || !dtype_ok(o_dtype)) return DR_ERR_DTYPE;
  if (flags & ~(DR_QK_L2NORM | DR_GATE_PER_CHANNEL)) return DR_ERR_UNSUPPORTED;
  if (B < 0 || Hqk <= 0 || Hv <= 0 || dk <= 0 || dv <= 0) return DR_ERR_SHAPE;
  if (Hv % Hqk != 0) return DR_ERR_SHAPE;
  if (!dim_ok(dk) || !dim_ok(dv)) return DR_ERR_UNSUPPORTED;
  if (!std::isfinite(scale)) return DR_ERR_UNSUPPORTED;
  if (B == 0) return DR_OK;
  const int cg = (flags & DR_GATE_PER_CHANNEL) ? 1 : 0;
  if (!q || !k || !v || !beta || !state || !o || (cg && !g)) return DR_ERR_NULL;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) ||
      !aligned(state, 16) || !aligned(g, 4) || !aligned(beta, 4))
    return DR_ERR_ALIGN;
  if ((int64_t)B * Hv > 0x7fffffff) return DR_ERR_UNSUPPORTED;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int l2n = (flags & DR_QK_L2NORM) ? 1 : 0;
  cudaError_t e;
  if (in_dtype == DR_BF16)
    e = o_dtype == DR_F32
            ? decode_dispatch<__nv_bfloat16, float>(dk, dv, q, k, v, g, beta, state, B, Hqk, Hv, scale, o, l2n, cg, s)
            : decode_dispatch<__nv_bfloat16, __nv_bfloat16>(dk, dv, q, k, v, g, beta, state, B, Hqk, Hv, scale, o, l2n, cg, s);
  else
    e = o_dtype == DR_F32
            ? decode_dispatch<float, float>(dk, dv, q, k, v, g, beta, state, B, Hqk, Hv, scale, o, l2n, cg, s)
            : decode_dispatch<float, __nv_bfloat16>(dk, dv, q, k, v, g, beta, state, B, Hqk, Hv, scale, o, l2n, cg, s);
  return e == cudaSuccess ? DR_OK : DR_ERR_CUDA;
}

dr_kernel dr_chunk_fwd_kernel(dr_dtype in_dtype, int32_t dk, int32_t dv) {
  if (!dtype_ok(in_dtype) || !dim_ok(dk) || !dim_ok(dv)) return DR_KERNEL_NONE;
  if (in_dtype == DR_BF16 && dr::tc_supported(dk, dv)) return DR_KERNEL_TC_BF16;
  return DR_KERNEL_SIMT_F32;
}

const char *dr_status_string(dr_status status) {
  switch (status) {
    case DR_OK: return "ok";
    case DR_ERR_NULL: return "a required pointer is NULL";
    case DR_ERR_SHAPE: return "inconsistent or invalid sizes";
    case DR_ERR_DTYPE: return "unknown dtype";
    case DR_ERR_ALIGN: return "pointer not aligned (16 bytes for tensors, 4 for g/beta/cu_seqlens)";
    case DR_ERR_UNSUPPORTED: return "unsupported head dimension or argument";
    case DR_ERR_CUDA: return "CUDA runtime error";
    case DR_ERR_TIMEOUT: return "a bounded device-side wait gave up";
  }
  return "unknown status";
}

dr_status dr_get_device_status(dr_stream stream) {
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return DR_ERR_CUDA;
  int word = 0;
  if (cudaMemcpyFromSymbol(&word, dr::g_device_status, sizeof(int)) != cudaSuccess)
    return DR_ERR_CUDA;
  if (word != 0) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(dr::g_device_status, &zero, sizeof(int)) != cudaSuccess)
      return DR_ERR_CUDA;
  }
  if (word & (1 << DR_ERR_TIMEOUT)) return DR_ERR_TIMEOUT;
  if (word & (1 << DR_ERR_SHAPE)) return DR_ERR_SHAPE;
  return DR_OK;
}

int32_t dr_version(void) { return DR_VERSION_NUMBER; }

}  // extern "C"
