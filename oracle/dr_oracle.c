/*
 * dr_oracle.c -- fp64 CPU oracle for the (gated) delta-rule recurrence.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the
 * cpu_baseline / reference legs of bench.py may load this library.  It shares
 * no code, header, table or helper with the CUDA path.
 *
 * What it computes (token by token, plain loops, double precision):
 *
 *   math state S (d_v x d_k) per (sequence, v-head), starting from
 *   state_in^T (or zero).  For every token t of the sequence:
 *       alpha_t = exp(g_t)                      (g absent => alpha_t = 1)
 *       S'      = alpha_t * S
 *       S       = S' - beta_t (S' k_t - v_t) k_t^T
 *       o_t     = S (scale * q_t)
 *   and at the end state_out = S^T (stored d_k x d_v, "key_dim by value_dim").
 *
 * Sources (page title, section):
 *   - "DeltaNet Attention" (frankenstein-transformer docs), class docstring:
 *     the update S_t = S_{t-1}(I - beta_t k_t k_t^T) + beta_t v_t k_t^T, beta
 *     per head, L2-normalised keys; forward(): token-by-token processing.
 *   - "DeltaNet" (study notes), section "The Delta Rule": the error-correcting
 *     form, its reading as one SGD step on 1/2||S k - v||^2, and the
 *     retrieve-and-replace form with v_old / v_new.
 *   - "linear_attention" (nnterp docs), LinearAttention: per-token decay gate
 *     given as the log of the kept fraction (float32, non-positive) applied
 *     before the key/value write; the query reads the updated state; state
 *     stored as one key_dim x value_dim matrix per head; state_input None on a
 *     prompt, the cached state on a decode step.
 *
 * Three independent inner updates are implemented (selected by `form`) so that
 * tests can pin each against the others:
 *   form 1  projection form: S = alpha S (I - beta k k^T) + beta v k^T, with the
 *           d_k x d_k matrix (I - beta k k^T) built explicitly;
 *   form 2  error-correction / SGD form on S' = alpha S (the default);
 *   form 3  retrieve-and-replace: v_old = S' k, v_new = beta v + (1-beta) v_old,
 *           S = S' - v_old k^T + v_new k^T.
 *
 * Per-key-channel gates (channel_gates = 1): the "linear_attention" page's
 * ChannelGates, [batch, seq, heads, key_dim], the gate of the KDA subclass.
 * Read as one log kept-fraction per key channel: S' = S diag(alpha_t), i.e.
 * column i of S (row i of the stored state) decays by exp(g_t[i]); the delta
 * write that follows is unchanged.  A scalar gate is the case of equal entries.
 *
 * Readings where the pages are silent: the decay multiplies the state before
 * the delta write; the query reads after the write; `scale` multiplies q
 * (1.0 reproduces o = S q); query/key head h_qk = h_v / (Hv / Hqk).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* Error codes of oracle_run. */
#define ORACLE_OK 0
#define ORACLE_EARG 1
#define ORACLE_ENOMEM 2

static void update_form1(double *S, double *A, const double *k, const double *v,
                         double alpha, double beta, int dk, int dv) {
  /* A = alpha (I - beta k k^T), d_k x d_k */
  for (int a = 0; a < dk; ++a)
    for (int b = 0; b < dk; ++b)
      A[a * dk + b] = alpha * ((a == b ? 1.0 : 0.0) - beta * k[a] * k[b]);
  /* S <- S A + beta v k^T, row by row of S (d_v rows of length d_k) */
  double *row = (double *)malloc(sizeof(double) * (size_t)dk);
  for (int j = 0; j < dv; ++j) {
    for (int b = 0; b < dk; ++b) {
      double acc = 0.0;
      for (int a = 0; a < dk; ++a) acc += S[j * dk + a] * A[a * dk + b];
      row[b] = acc;
    }
    for (int b = 0; b < dk; ++b) S[j * dk + b] = row[b] + beta * v[j] * k[b];
  }
  free(row);
}

static void update_form2(double *S, const double *k, const double *v, double alpha,
                         double beta, int dk, int dv) {
  for (int j = 0; j < dv; ++j) {
    double *Sj = S + (size_t)j * dk;
    for (int i = 0; i < dk; ++i) Sj[i] *= alpha;
    double pred = 0.0; /* (S' k)_j */
    for (int i = 0; i < dk; ++i) pred += Sj[i] * k[i];
    double err = pred - v[j]; /* gradient of 1/2 ||S k - v||^2 is (S k - v) k^T */
    for (int i = 0; i < dk; ++i) Sj[i] -= beta * err * k[i];
  }
}

static void update_form3(double *S, const double *k, const double *v, double alpha,
                         double beta, int dk, int dv) {
  for (int j = 0; j < dv; ++j) {
    double *Sj = S + (size_t)j * dk;
    for (int i = 0; i < dk; ++i) Sj[i] *= alpha;
    double v_old = 0.0;
    for (int i = 0; i < dk; ++i) v_old += Sj[i] * k[i];
    double v_new = beta * v[j] + (1.0 - beta) * v_old;
    for (int i = 0; i < dk; ++i) Sj[i] = Sj[i] - v_old * k[i] + v_new * k[i];
  }
}

/*
 * oracle_run: run the recurrence for every (sequence, v-head) unit.
 *
 * Layouts (all host, contiguous, row-major, double):
 *   q, k        [B, T, Hqk, dk]
 *   v, o        [B, T, Hv, dv]
 *   g, beta     [B, T, Hv]        (g may be NULL: no decay); with channel_gates
 *               g is [B, T, Hv, dk], one log decay per key channel
 *   state_in    [N, Hv, dk, dv]   (may be NULL: zero state)
 *   state_out   [N, Hv, dk, dv]   (may be NULL)
 *   chunk_states [NC, Hv, dk, dv] (may be NULL): the stored state S^T after
 *                every chunk_len tokens of each sequence and after its last
 *                token.  Sequence n owns ceil(len_n / chunk_len) rows starting
 *                at the sum of that count over the sequences before it; row j
 *                holds the state after min((j+1) chunk_len, len_n) tokens, so a
 *                sequence's last row equals its state_out.
 * With cu_seqlens (host int32 [N+1], N = n_seqs) B must be 1 and sequence n
 * covers tokens [cu_seqlens[n], cu_seqlens[n+1]); without it N = B and every
 * sequence has T tokens.
 * n_threads <= 0 uses the OpenMP default.
 */
int oracle_run(const double *q, const double *k, const double *v, const double *g,
               const double *beta, const double *state_in, const int32_t *cu_seqlens,
               int n_seqs, int B, int T, int Hqk, int Hv, int dk, int dv, double scale,
               int form, int n_threads, double *o, double *state_out, int chunk_len,
               double *chunk_states, int channel_gates) {
  if (!q || !k || !v || !beta || !o) return ORACLE_EARG;
  if (B < 0 || T < 0 || Hqk <= 0 || Hv <= 0 || dk <= 0 || dv <= 0) return ORACLE_EARG;
  if (Hv % Hqk != 0) return ORACLE_EARG;
  if (form < 1 || form > 3) return ORACLE_EARG;
  if (chunk_states && chunk_len <= 0) return ORACLE_EARG;
  int N = cu_seqlens ? n_seqs : B;
  if (cu_seqlens) {
    if (B != 1 || n_seqs < 0) return ORACLE_EARG;
    if (cu_seqlens[0] != 0 || cu_seqlens[n_seqs] != T) return ORACLE_EARG;
    for (int n = 0; n < n_seqs; ++n)
      if (cu_seqlens[n + 1] < cu_seqlens[n]) return ORACLE_EARG;
  }
  const int group = Hv / Hqk;
  const long units = (long)N * Hv;
  int fail = 0;

#ifdef _OPENMP
  if (n_threads > 0) omp_set_num_threads(n_threads);
#pragma omp parallel for schedule(dynamic, 1) reduction(| : fail)
#endif
  for (long u = 0; u < units; ++u) {
    const int n = (int)(u / Hv), h = (int)(u % Hv), hq = h / group;
    long b, t0, t1;
    if (cu_seqlens) {
      b = 0;
      t0 = cu_seqlens[n];
      t1 = cu_seqlens[n + 1];
    } else {
      b = n;
      t0 = 0;
      t1 = T;
    }
    long cbase = 0; /* first chunk_states row of sequence n */
    if (chunk_states) {
      for (int m = 0; m < n; ++m) {
        const long len = cu_seqlens ? (long)cu_seqlens[m + 1] - cu_seqlens[m] : (long)T;
        cbase += (len + chunk_len - 1) / chunk_len;
      }
    }
    double *S = (double *)calloc((size_t)dv * dk, sizeof(double));
    double *A = form == 1 ? (double *)malloc(sizeof(double) * (size_t)dk * dk) : NULL;
    double *qs = (double *)malloc(sizeof(double) * (size_t)dk);
    if (!S || !qs || (form == 1 && !A)) {
      fail |= 1;
      free(S);
      free(A);
      free(qs);
      continue;
    }
    if (state_in) {
      const double *H0 = state_in + ((size_t)n * Hv + h) * dk * dv;
      for (int i = 0; i < dk; ++i)
        for (int j = 0; j < dv; ++j) S[(size_t)j * dk + i] = H0[(size_t)i * dv + j];
    }
    for (long t = t0; t < t1; ++t) {
      const size_t tok = (size_t)b * T + t;
      const double *kt = k + (tok * Hqk + hq) * dk;
      const double *qt = q + (tok * Hqk + hq) * dk;
      const double *vt = v + (tok * Hv + h) * dv;
      const double bt = beta[tok * Hv + h];
      double alpha = 1.0;
      if (g && channel_gates) {
        /* S' = S diag(alpha_t): column i of S scales by exp(g_t[i]) */
        const double *gt = g + (tok * Hv + h) * dk;
        for (int j = 0; j < dv; ++j)
          for (int i = 0; i < dk; ++i) S[(size_t)j * dk + i] *= exp(gt[i]);
      } else if (g) {
        alpha = exp(g[tok * Hv + h]);
      }
      if (form == 1)
        update_form1(S, A, kt, vt, alpha, bt, dk, dv);
      else if (form == 2)
        update_form2(S, kt, vt, alpha, bt, dk, dv);
      else
        update_form3(S, kt, vt, alpha, bt, dk, dv);
      for (int i = 0; i < dk; ++i) qs[i] = scale * qt[i];
      double *ot = o + (tok * Hv + h) * dv;
      for (int j = 0; j < dv; ++j) {
        double acc = 0.0;
        for (int i = 0; i < dk; ++i) acc += S[(size_t)j * dk + i] * qs[i];
        ot[j] = acc;
      }
      if (chunk_states && ((t + 1 - t0) % chunk_len == 0 || t + 1 == t1)) {
        const long row = cbase + (t - t0) / chunk_len;
        double *Hc = chunk_states + ((size_t)row * Hv + h) * dk * dv;
        for (int i = 0; i < dk; ++i)
          for (int j = 0; j < dv; ++j) Hc[(size_t)i * dv + j] = S[(size_t)j * dk + i];
      }
    }
    if (state_out) {
      double *H1 = state_out + ((size_t)n * Hv + h) * dk * dv;
      for (int i = 0; i < dk; ++i)
        for (int j = 0; j < dv; ++j) H1[(size_t)i * dv + j] = S[(size_t)j * dk + i];
    }
    free(S);
    free(A);
    free(qs);
  }
  return fail ? ORACLE_ENOMEM : ORACLE_OK;
}

/* Number of threads an OpenMP parallel region would use (1 without OpenMP). */
int oracle_max_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}
