/*
 * dr.h -- C ABI of the B200 gated delta-rule library (libdr.so).
 *
 * The operation (per sequence n and value head h, query/key head
 * hq = h / (Hv / Hqk)):
 *
 *     S_t = alpha_t S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,
 *     o_t = S_t (scale * q_t),          alpha_t = exp(g_t)
 *
 * - update of the "DeltaNet Attention" page (class docstring); its error-correction
 *   and retrieve-and-replace forms are on the "DeltaNet" page ("The Delta Rule");
 * - gate (decays), write strength (betas), head layout and state_input semantics
 *   of the "linear_attention" page (LinearAttention): decays are float32 log
 *   kept-fractions, betas are in (0, 1) or (0, 2), the query reads the updated
 *   state, and the state is one key_dim x value_dim matrix per head.
 *
 * State is stored as H = S^T:  [.., dk, dv] float32, row-major (dv contiguous).
 *
 * Conventions for every call
 * - All tensor pointers are DEVICE memory owned by the caller.  The library
 *   never allocates device memory and never frees.  Tensors are dense, row-major
 *   and contiguous in the layouts below.
 * - q, k, v, o, state_in, state_out and state must be 16-byte aligned; g and beta
 *   4-byte aligned; cu_seqlens 4-byte aligned.
 * - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy default).
 *   Argument errors are detected on the host before anything is launched and
 *   leave every output untouched.  A failed launch returns DR_ERR_CUDA.
 * - Errors the host cannot see (malformed cu_seqlens contents, a bounded
 *   device-side wait that ran out) set a device status word instead: the kernel
 *   skips the affected work unit, and dr_get_device_status() reports it.
 * - Supported: dk, dv in {16, 32, 64, 128}; Hv % Hqk == 0 (GQA: value head h uses
 *   query/key head h / (Hv / Hqk)); scale is any finite float (1.0 = o = S q).
 * - No call throws, exits or keeps mutable host state; calls are thread-safe.
 */
#ifndef DR_H
#define DR_H

#include <stdint.h>

#if defined(__GNUC__)
#define DR_API __attribute__((visibility("default")))
#else
#define DR_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  DR_OK = 0,
  DR_ERR_NULL = 1,        /* a required pointer is NULL                          */
  DR_ERR_SHAPE = 2,       /* inconsistent or negative sizes (incl. Hv % Hqk != 0) */
  DR_ERR_DTYPE = 3,       /* unknown dtype code                                  */
  DR_ERR_ALIGN = 4,       /* a pointer violates the alignment rule above          */
  DR_ERR_UNSUPPORTED = 5, /* valid but unsupported (e.g. dk = 96)                 */
  DR_ERR_CUDA = 6,        /* a CUDA runtime call or launch failed                 */
  DR_ERR_TIMEOUT = 7      /* a bounded device-side wait gave up                   */
} dr_status;

typedef enum { DR_F32 = 0, DR_BF16 = 1 } dr_dtype;

/* Same type as cudaStream_t. */
typedef struct CUstream_st *dr_stream;

/* Tokens per chunk of dr_chunk_fwd: the spacing of the states it returns in chunk_states. */
#define DR_CHUNK 64

/* Option bits of dr_chunk_fwd / dr_recurrent_step (any other bit => DR_ERR_UNSUPPORTED). */
#define DR_QK_L2NORM 1u /* divide every q and k row (per token and q/k head) by its L2 norm
                           first (an all-zero row stays zero): the pages' qk_l2norm step
                           ("DeltaNet Attention": queries and keys are L2-normalised before
                           the rule), folded into the kernels as fp32 row and column scalings */
#define DR_GATE_PER_CHANNEL 2u /* g holds one log decay per key channel, [.., Hv, dk] f32: the
                                  "linear_attention" page's ChannelGates (its KDA subclass).
                                  Row i of the stored state decays by exp(g[i]) before the
                                  write.  g must not be NULL.  dr_chunk_fwd then always runs
                                  the CUDA-core kernel (fp32 arithmetic) */

/*
 * dr_chunk_fwd -- prompt (prefill) pass: the "chunked rule on a prompt" of the
 * "linear_attention" page, computed chunkwise in the UT/WY form of
 * "Parallelizing Linear Transformers with the Delta Rule over Sequence Length"
 * (the reference both DeltaNet pages cite), 64-token chunks, decays folded in.
 *
 *   q, k       [B, T, Hqk, dk]   in_dtype (DR_BF16 or DR_F32); L2-normalised by the caller,
 *                                or by the kernel with DR_QK_L2NORM in flags
 *   v          [B, T, Hv, dv]    in_dtype
 *   g          [B, T, Hv] f32    log decay (<= 0 expected); NULL => no decay (plain DeltaNet);
 *                                [B, T, Hv, dk] with DR_GATE_PER_CHANNEL
 *   beta       [B, T, Hv] f32    write strength
 *   state_in   [N, Hv, dk, dv] f32 or NULL (=> zero state: a fresh prompt).  Read only.
 *   cu_seqlens device int32 [n_seqs + 1] or NULL.  If given, B must be 1, N = n_seqs,
 *              sequence n is tokens [cu_seqlens[n], cu_seqlens[n+1]) with
 *              cu_seqlens[0] = 0, non-decreasing, cu_seqlens[n_seqs] = T (checked on
 *              the device: a violation skips that sequence and sets DR_ERR_SHAPE
 *              in the device status).  If NULL, N = B sequences of T tokens.
 *   o          [B, T, Hv, dv]    o_dtype (DR_F32 or DR_BF16); every token's output is written
 *   state_out  [N, Hv, dk, dv] f32 or NULL (=> final state not returned).  It may be
 *              state_in itself (in-place update); a partial overlap is undefined.
 *   chunk_states [R, Hv, dk, dv] f32 or NULL (=> not returned): the intermediate states
 *              the "linear_attention" page's recurrent route exposes, sampled at chunk ends: the
 *              state after every DR_CHUNK tokens of each sequence and after its last
 *              token.  Sequence n owns ceil(max(len_n, 0) / DR_CHUNK) rows, in sequence
 *              order, so R = sum_n of that count (N * ceil(T / DR_CHUNK) without
 *              cu_seqlens); row j of a sequence holds the state after
 *              min((j + 1) DR_CHUNK, len_n) tokens, and its last row equals its
 *              state_out.  Caller-owned, 16-byte aligned, overlapping no other
 *              argument; rows of a sequence that a bad cu_seqlens skips are not written.
 *   flags      0 or an OR of DR_QK_L2NORM and DR_GATE_PER_CHANNEL
 *   T = 0 or N = 0 is valid: nothing is read from q/k/v; state_out (if given) receives
 *   state_in (or zeros).
 */
DR_API dr_status dr_chunk_fwd(const void *q, const void *k, const void *v, const float *g,
                              const float *beta, const float *state_in,
                              const int32_t *cu_seqlens, int32_t n_seqs, int32_t B, int32_t T,
                              int32_t Hqk, int32_t Hv, int32_t dk, int32_t dv,
                              dr_dtype in_dtype, float scale, void *o, dr_dtype o_dtype,
                              float *state_out, float *chunk_states, uint32_t flags,
                              dr_stream stream);

/* Which prefill kernel dr_chunk_fwd launches for these inputs without DR_GATE_PER_CHANNEL
   (host only, no device call); with it the kernel is always DR_KERNEL_SIMT_F32. */
typedef enum {
  DR_KERNEL_NONE = 0,     /* unsupported dtype / head dimensions                  */
  DR_KERNEL_SIMT_F32 = 1, /* CUDA-core kernel, fp32 arithmetic                    */
  DR_KERNEL_TC_BF16 = 2   /* tcgen05 tensor-core kernel, bf16 operands, fp32 state */
} dr_kernel;
DR_API dr_kernel dr_chunk_fwd_kernel(dr_dtype in_dtype, int32_t dk, int32_t dv);

/*
 * dr_recurrent_step -- one decode token per sequence: the "token-by-token rule on
 * a decode step" of the "linear_attention" page, with the cache overwritten in
 * place (state_input semantics there).  Computed as
 *     H' = alpha H;  v_old = H'^T k;  delta = beta (v - v_old);
 *     H  = H' + k delta^T (in place);  o = H^T (scale q)
 * which is the retrieve-and-replace form of the "DeltaNet" page ("The Delta Rule").
 *
 *   q, k   [B, Hqk, dk] in_dtype;   v [B, Hv, dv] in_dtype
 *   g      [B, Hv] f32 or NULL ([B, Hv, dk] with DR_GATE_PER_CHANNEL: H' = diag(alpha) H);
 *   beta   [B, Hv] f32
 *   state  [B, Hv, dk, dv] f32, read and overwritten in place
 *   o      [B, Hv, dv] o_dtype
 */
DR_API dr_status dr_recurrent_step(const void *q, const void *k, const void *v,
                                   const float *g, const float *beta, float *state, int32_t B,
                                   int32_t Hqk, int32_t Hv, int32_t dk, int32_t dv,
                                   dr_dtype in_dtype, float scale, void *o, dr_dtype o_dtype,
                                   uint32_t flags, dr_stream stream);
/* flags of dr_recurrent_step: 0 or an OR of DR_QK_L2NORM and DR_GATE_PER_CHANNEL. */

/*
 * dr_short_conv_silu -- the step before the rule in the "DeltaNet" layer diagram: a
 * causal depthwise convolution ("Conv*") of the projected q, k or v, then SiLU:
 *     y_t[c] = silu(sum_{j<K} w[c][j] x_{t-K+1+j}[c]),   silu(u) = u / (1 + e^-u)
 * Tap K-1 weighs the current token.  Before a sequence's first token the inputs are the
 * sequence's conv_state_in (its last K-1 inputs of a previous call, oldest first) or zero;
 * sequences never see one another.
 *
 *   x          [B, T, C] x_dtype (C channels, e.g. heads * head_dim, contiguous)
 *   w          [C, K] f32, 1 <= K <= 8
 *   conv_state_in  [N, C, K-1] f32 or NULL (zero history)
 *   conv_state_out [N, C, K-1] f32 or NULL: the last K-1 inputs of every sequence (history
 *              included when a sequence is shorter); may be conv_state_in itself
 *   cu_seqlens as for dr_chunk_fwd (B = 1, N = n_seqs); else N = B sequences of T tokens
 *   y          [B, T, C] y_dtype; must not overlap x
 */
DR_API dr_status dr_short_conv_silu(const void *x, dr_dtype x_dtype, const float *w, int32_t K,
                                    const float *conv_state_in, float *conv_state_out,
                                    const int32_t *cu_seqlens, int32_t n_seqs, int32_t B,
                                    int32_t T, int32_t C, void *y, dr_dtype y_dtype,
                                    dr_stream stream);

typedef enum { DR_NORM_RMS = 0, DR_NORM_LAYER = 1 } dr_norm_kind;

/*
 * dr_norm_gate -- the step after the rule: per-(token, head) normalisation of the
 * readout over its dv values ("DeltaNet": RMSNorm; "DeltaNet Attention": LayerNorm
 * `norm`), then the SiLU output gate of "DeltaNet Attention" (`g_proj`):
 *     RMS:    u = o / sqrt(mean(o^2) + eps) * weight
 *     LAYER:  u = (o - mean(o)) / sqrt(var(o) + eps) * weight + bias   (biased variance)
 *     y = z ? u * silu(z) : u
 *
 *   o       [rows, dv] o_dtype (rows = B * T * Hv), dv <= 128
 *   weight  [dv] f32;  bias [dv] f32 or NULL (LayerNorm only)
 *   z       [rows, dv] z_dtype or NULL (no gate)
 *   y       [rows, dv] y_dtype; may be o itself when the dtypes match
 *   eps     >= 0 (1e-6 for RMSNorm and 1e-5 for LayerNorm are the usual values)
 */
DR_API dr_status dr_norm_gate(const void *o, dr_dtype o_dtype, const float *weight,
                              const float *bias, const void *z, dr_dtype z_dtype, int64_t rows,
                              int32_t dv, int32_t kind, float eps, void *y, dr_dtype y_dtype,
                              dr_stream stream);

/* Static English description of a status code (never NULL). */
DR_API const char *dr_status_string(dr_status status);

/*
 * Synchronises `stream`, then reports and clears the device status word of the
 * current device: DR_OK, DR_ERR_SHAPE (bad cu_seqlens contents) or
 * DR_ERR_TIMEOUT (a bounded device wait gave up).  DR_ERR_CUDA if the
 * synchronisation itself failed.
 */
DR_API dr_status dr_get_device_status(dr_stream stream);

/* Library version: major * 10000 + minor * 100 + patch. */
DR_API int32_t dr_version(void);

#ifdef __cplusplus
}
#endif

#endif /* DR_H */
