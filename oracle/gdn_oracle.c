/*
 * gdn_oracle.c -- plain, slow, fp64 CPU oracle for the Gated DeltaNet (GDN) token mixer.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call, link or load this
 * file: only the test suite, the smoke check and the benchmark's CPU-baseline leg use
 * it.  It shares no code, header, table or constant with the CUDA library.
 *
 * What it computes, and where each step is defined:
 *   - width-4 depthwise causal convolution of the q, k and v streams, followed by SiLU
 *     ("Qwen3.8-Flash-Next" technical report, Fig. 2: short causal convolutions on the
 *     projected query, key and value streams; "Qwen3-Next 80B-A3B" field guide, §02
 *     "Gated DeltaNet state update": width-4 depthwise causal convolution);
 *   - L2 normalisation of q and k (technical report, Fig. 2);
 *   - decay gate g = -exp(A_log) * softplus(a + dt_bias)  ("Qwen3.8-Flash-Next" model
 *     notes, the GatedDeltaNet decay-gate note), alpha = exp(g); write gate
 *     beta = sigmoid(b) (technical report, Fig. 2 names the write gate beta_t);
 *   - the gated delta rule on one d_v x d_k state per value head, in the six steps of
 *     the field guide, §02 (column-vector convention: S maps a key to a value):
 *         S' = alpha S;  vhat = S' k;  e = v - vhat;  (beta e);  S'' = S' + (beta e) k^T;
 *         y = S'' q;
 *   - output RMS normalisation gated by SiLU(z) (field guide, §02, last line).
 *
 * The chunked form (oracle_recurrence_chunked) is an exact algebraic rewrite of the
 * per-token rule, kept here only so the test suite can prove that rewrite on tiny
 * inputs; its inter-chunk state carry is the update in the model notes' chunk-loop
 * note (state = state * chunk decay + key^T @ new values), written in the
 * column-vector convention.
 *
 * Readings where the pages are silent (each is also listed in the design notes):
 *   - no query scale (q_scale = 1 reproduces y = S'' q exactly);
 *   - conv taps: w[c][3] multiplies the current token, w[c][0] the token three back;
 *     history before a sequence's first token is zero; no conv bias;
 *   - L2 norm x / sqrt(sum x^2 + eps); RMSNorm per value head over d_v, then * norm_w,
 *     then * silu(z);
 *   - value head h reads QK head h / (h_v / h_qk).
 *
 * Everything is fp64.  Inputs are fp32 or bf16 element encodings, widened exactly.
 * No blocking, fusion or reordering beyond what the definitions state.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define OR_ENC_F32 0  /* element encoding: IEEE fp32 */
#define OR_ENC_BF16 1 /* element encoding: bf16 (the upper 16 bits of an fp32) */

/* Exact widening of one stored element to double. */
static double or_load(const void* p, size_t i, int enc) {
  if (enc == OR_ENC_BF16) {
    uint32_t u = ((uint32_t)((const uint16_t*)p)[i]) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
  }
  return (double)((const float*)p)[i];
}

/* ---- scalar functions ------------------------------------------------------------ */

/* softplus(x) = log(1 + e^x), written in the overflow-free form max(x,0) + log1p(e^-|x|). */
double oracle_softplus(double x) { return (x > 0 ? x : 0.0) + log1p(exp(-fabs(x))); }

/* sigmoid(x) = 1 / (1 + e^-x). */
double oracle_sigmoid(double x) { return 1.0 / (1.0 + exp(-x)); }

/* SiLU(x) = x * sigmoid(x). */
double oracle_silu(double x) { return x / (1.0 + exp(-x)); }

/* Decay gate g (model notes, decay-gate note): g = -exp(A_log) * softplus(a + dt_bias). */
double oracle_decay_gate(double a, double A_log, double dt_bias) {
  return -exp(A_log) * oracle_softplus(a + dt_bias);
}

/* ---- stage functions (one sequence, one channel or one head) ------------------------ */

/*
 * Causal depthwise convolution of width 4, then SiLU, over one channel of one sequence.
 *   out[t] = silu( sum_{i=0..3} w[i] * x[t-3+i] ),  x[tau] = hist[tau+3] for tau < 0.
 * hist holds x[-3], x[-2], x[-1] (zeros at a sequence start); NULL means zeros.
 * x and out are strided: element t sits at x[t * stride].
 */
void oracle_conv_silu_channel(const double* x, long stride, long T, const double w[4],
                              const double hist[3], double* out) {
  for (long t = 0; t < T; ++t) {
    double acc = 0.0;
    for (int i = 0; i < 4; ++i) {
      long tau = t - 3 + i;
      double xv = tau >= 0 ? x[tau * stride] : (hist ? hist[tau + 3] : 0.0);
      acc += w[i] * xv;
    }
    out[t * stride] = oracle_silu(acc);
  }
}

/* L2 normalisation of one vector of length n: x / sqrt(sum x^2 + eps), in place. */
void oracle_l2norm(double* x, int n, double eps) {
  double ss = 0.0;
  for (int i = 0; i < n; ++i) ss += x[i] * x[i];
  double r = 1.0 / sqrt(ss + eps);
  for (int i = 0; i < n; ++i) x[i] *= r;
}

/*
 * Output gate of one (token, value head) (field guide, §02, last line):
 *   y = y_raw / sqrt(mean(y_raw^2) + eps) * norm_w * silu(z).
 */
void oracle_gated_rmsnorm(const double* y_raw, const double* z, const double* norm_w, int dv,
                          double eps, double* y) {
  double ss = 0.0;
  for (int i = 0; i < dv; ++i) ss += y_raw[i] * y_raw[i];
  double r = 1.0 / sqrt(ss / dv + eps);
  for (int i = 0; i < dv; ++i) y[i] = y_raw[i] * r * norm_w[i] * oracle_silu(z[i]);
}

/*
 * One token of the gated delta rule, the six steps of the field guide, §02, in order.
 * S is d_v x d_k row-major (S[i*dk + j] maps key component j to value component i) and
 * is updated in place from S to S''.  y_raw receives S'' (q_scale * q).
 */
void oracle_delta_step(double* S, int dv, int dk, const double* k, const double* q,
                       const double* v, double g, double beta, double q_scale, double* y_raw,
                       double* scratch /* 2*dv doubles */) {
  double* vhat = scratch;
  double* e = scratch + dv;
  const double alpha = exp(g);
  /* 1. decay old state: S' = alpha S */
  for (int i = 0; i < dv; ++i)
    for (int j = 0; j < dk; ++j) S[(size_t)i * dk + j] *= alpha;
  /* 2. read current association: vhat = S' k */
  for (int i = 0; i < dv; ++i) {
    double acc = 0.0;
    for (int j = 0; j < dk; ++j) acc += S[(size_t)i * dk + j] * k[j];
    vhat[i] = acc;
  }
  /* 3. measure value error: e = v - vhat;  4. gate the correction: beta e */
  for (int i = 0; i < dv; ++i) e[i] = beta * (v[i] - vhat[i]);
  /* 5. write error (x) key: S'' = S' + (beta e) k^T */
  for (int i = 0; i < dv; ++i)
    for (int j = 0; j < dk; ++j) S[(size_t)i * dk + j] += e[i] * k[j];
  /* 6. read with query: y = S'' q */
  for (int i = 0; i < dv; ++i) {
    double acc = 0.0;
    for (int j = 0; j < dk; ++j) acc += S[(size_t)i * dk + j] * (q_scale * q[j]);
    y_raw[i] = acc;
  }
}

/*
 * Per-token recurrence over one sequence of one value head, on the already convolved,
 * normalised streams.  qh, kh: [T][dk]; v: [T][dv]; g, beta: [T]; S: [dv][dk] in/out.
 * y_raw: [T][dv].
 */
void oracle_recurrence_token(long T, int dk, int dv, const double* qh, const double* kh,
                             const double* v, const double* g, const double* beta,
                             double q_scale, double* S, double* y_raw) {
  double* scratch = (double*)malloc(sizeof(double) * 2 * dv);
  for (long t = 0; t < T; ++t)
    oracle_delta_step(S, dv, dk, kh + t * dk, qh + t * dk, v + t * dv, g[t], beta[t], q_scale,
                      y_raw + t * dv, scratch);
  free(scratch);
}

/* Forward substitution: solve (I + A) X = B for unit-lower-triangular I + A (A strictly lower),
 * A: [C][C], B and X: [C][n] row-major.  X may alias B. */
static void or_unit_lower_solve(int C, int n, const double* A, double* X) {
  for (int t = 0; t < C; ++t)
    for (int s = 0; s < t; ++s) {
      double a = A[(size_t)t * C + s];
      if (a != 0.0)
        for (int c = 0; c < n; ++c) X[(size_t)t * n + c] -= a * X[(size_t)s * n + c];
    }
}

/*
 * Chunked form of the same recurrence, chunk length C (last chunk partial).  An exact
 * rewrite of oracle_recurrence_token, used only to prove the chunk algebra the GPU uses.
 * With S_0 the state at the chunk start (rows t, s index the chunk's tokens):
 *   gamma_t = sum_{r<=t} g_r
 *   A[t][s] = beta_t exp(gamma_t - gamma_s) (k_t . k_s)   for s < t, else 0
 *   (I + A) U = diag(beta) (V - diag(exp(gamma)) K S_0^T)          [solve for U]
 *   Y = diag(exp(gamma)) Q S_0^T + (M o Q K^T) U,  M[t][s] = exp(gamma_t - gamma_s), s <= t
 *   S_C = exp(gamma_C) S_0 + U^T diag(exp(gamma_C - gamma)) K
 * The last line is the chunk-loop state update of the model notes in column-vector form.
 */
void oracle_recurrence_chunked(long T, int dk, int dv, int C, const double* qh,
                               const double* kh, const double* v, const double* g,
                               const double* beta, double q_scale, double* S, double* y_raw) {
  double* gam = (double*)malloc(sizeof(double) * C);
  double* A = (double*)malloc(sizeof(double) * C * C);
  double* U = (double*)malloc(sizeof(double) * C * dv);
  double* Snew = (double*)malloc(sizeof(double) * dv * dk);
  for (long c0 = 0; c0 < T; c0 += C) {
    int L = (int)((T - c0) < C ? (T - c0) : C);
    const double* Kc = kh + c0 * dk;
    const double* Qc = qh + c0 * dk;
    const double* Vc = v + c0 * dv;
    double run = 0.0;
    for (int t = 0; t < L; ++t) {
      run += g[c0 + t];
      gam[t] = run;
    }
    /* A (strictly lower triangular) */
    for (int t = 0; t < L; ++t)
      for (int s = 0; s < L; ++s) {
        double a = 0.0;
        if (s < t) {
          double kk = 0.0;
          for (int j = 0; j < dk; ++j) kk += Kc[(size_t)t * dk + j] * Kc[(size_t)s * dk + j];
          a = beta[c0 + t] * exp(gam[t] - gam[s]) * kk;
        }
        A[(size_t)t * L + s] = a;
      }
    /* right-hand side diag(beta)(V - diag(exp(gamma)) K S_0^T), then solve */
    for (int t = 0; t < L; ++t)
      for (int i = 0; i < dv; ++i) {
        double ks = 0.0;
        for (int j = 0; j < dk; ++j) ks += Kc[(size_t)t * dk + j] * S[(size_t)i * dk + j];
        U[(size_t)t * dv + i] = beta[c0 + t] * (Vc[(size_t)t * dv + i] - exp(gam[t]) * ks);
      }
    or_unit_lower_solve(L, dv, A, U);
    /* outputs */
    for (int t = 0; t < L; ++t)
      for (int i = 0; i < dv; ++i) {
        double qs = 0.0;
        for (int j = 0; j < dk; ++j) qs += Qc[(size_t)t * dk + j] * S[(size_t)i * dk + j];
        double acc = exp(gam[t]) * qs;
        for (int s = 0; s <= t; ++s) {
          double qk = 0.0;
          for (int j = 0; j < dk; ++j) qk += Qc[(size_t)t * dk + j] * Kc[(size_t)s * dk + j];
          acc += exp(gam[t] - gam[s]) * qk * U[(size_t)s * dv + i];
        }
        y_raw[(c0 + t) * dv + i] = q_scale * acc;
      }
    /* state carry */
    for (int i = 0; i < dv; ++i)
      for (int j = 0; j < dk; ++j) {
        double acc = exp(gam[L - 1]) * S[(size_t)i * dk + j];
        for (int s = 0; s < L; ++s)
          acc += U[(size_t)s * dv + i] * exp(gam[L - 1] - gam[s]) * Kc[(size_t)s * dk + j];
        Snew[(size_t)i * dk + j] = acc;
      }
    memcpy(S, Snew, sizeof(double) * dv * dk);
  }
  free(gam);
  free(A);
  free(U);
  free(Snew);
}

/* ---- whole-mixer entry points --------------------------------------------------------- */

typedef struct {
  int32_t n_seqs, total_tokens, h_qk, h_v, d_k, d_v;
  int32_t in_enc;       /* OR_ENC_F32 or OR_ENC_BF16: q, k, v, z (and decode conv_state) */
  double q_scale, l2_eps, rms_eps;
  int32_t chunk;        /* 0 = per-token recurrence; > 0 = chunked form with this length */
  int32_t n_threads;    /* <= 0: library default */
} oracle_dims;

/*
 * Prepare the convolved, normalised streams and the gates of one (sequence, value head):
 * qh, kh [T][dk]; vv [T][dv]; g, beta [T].  hist3 (optional) gives the raw history
 * x[-3..-1] of every conv channel as [3][C_conv] in the input encoding; NULL = zeros.
 */
static void or_prepare_head(const oracle_dims* d, long t0, long T, int h, const void* q,
                            const void* k, const void* v, const float* a, const float* b,
                            const float* A_log, const float* dt_bias, const float* conv_w,
                            const void* hist3, double* qh, double* kh, double* vv, double* g,
                            double* beta, double* colbuf, double* colout) {
  const int dk = d->d_k, dv = d->d_v, hq = d->h_qk, hv = d->h_v;
  const int j = h / (hv / hq);
  const long cconv = 2L * hq * dk + (long)hv * dv;
  /* channel blocks: q head j, k head j, v head h */
  const long ch_base[3] = {(long)j * dk, (long)hq * dk + (long)j * dk,
                           2L * hq * dk + (long)h * dv};
  const void* src[3] = {q, k, v};
  const long src_row[3] = {(long)hq * dk, (long)hq * dk, (long)hv * dv};
  const long src_off[3] = {(long)j * dk, (long)j * dk, (long)h * dv};
  double* dst[3] = {qh, kh, vv};
  const int width[3] = {dk, dk, dv};
  for (int m = 0; m < 3; ++m)
    for (int c = 0; c < width[m]; ++c) {
      double w[4], hist[3];
      for (int i = 0; i < 4; ++i) w[i] = conv_w[(ch_base[m] + c) * 4 + i];
      for (int i = 0; i < 3; ++i)
        hist[i] = hist3 ? or_load(hist3, (size_t)i * cconv + ch_base[m] + c, d->in_enc) : 0.0;
      for (long t = 0; t < T; ++t)
        colbuf[t] = or_load(src[m], (size_t)(t0 + t) * src_row[m] + src_off[m] + c, d->in_enc);
      oracle_conv_silu_channel(colbuf, 1, T, w, hist, colout);
      for (long t = 0; t < T; ++t) dst[m][t * width[m] + c] = colout[t];
    }
  for (long t = 0; t < T; ++t) {
    oracle_l2norm(qh + t * dk, dk, d->l2_eps);
    oracle_l2norm(kh + t * dk, dk, d->l2_eps);
    g[t] = oracle_decay_gate((double)a[(t0 + t) * hv + h], (double)A_log[h], (double)dt_bias[h]);
    beta[t] = oracle_sigmoid((double)b[(t0 + t) * hv + h]);
  }
}

/*
 * Whole prefill over packed sequences.  Tensors in the library's layouts:
 *   q, k [T_tot][h_qk][d_k]; v, z [T_tot][h_v][d_v] (encoding d->in_enc);
 *   a, b [T_tot][h_v] fp32; A_log, dt_bias [h_v]; conv_w [C_conv][4] channel order q|k|v;
 *   norm_w [d_v]; init_state [N][h_v][d_v][d_k] fp32 or NULL (zeros);
 *   cu_seqlens [N+1] host int32 (NULL = one sequence of T_tot tokens).
 * Only value heads hv0 <= h < hv1 are computed; their y and final-state entries are written,
 * the rest are left untouched.  y, y_raw: [T_tot][h_v][d_v] fp64 (y_raw may be NULL);
 * final_state [N][h_v][d_v][d_k] fp64 (may be NULL).  Returns 0, or -1 on bad arguments.
 */
int oracle_prefill(const oracle_dims* d, const void* q, const void* k, const void* v,
                   const void* z, const float* a, const float* b, const float* A_log,
                   const float* dt_bias, const float* conv_w, const float* norm_w,
                   const float* init_state, const int32_t* cu_seqlens, int hv0, int hv1,
                   double* y, double* y_raw_out, double* final_state) {
  const int dk = d->d_k, dv = d->d_v, hv = d->h_v;
  if (d->n_seqs < 1 || d->h_qk < 1 || hv % d->h_qk || hv0 < 0 || hv1 > hv || hv0 > hv1)
    return -1;
  const int nseq = d->n_seqs;
  const long npair = (long)nseq * (hv1 - hv0);
#ifdef _OPENMP
  int nt = d->n_threads > 0 ? d->n_threads : omp_get_max_threads();
#pragma omp parallel for schedule(dynamic, 1) num_threads(nt)
#endif
  for (long p = 0; p < npair; ++p) {
    const int n = (int)(p / (hv1 - hv0));
    const int h = hv0 + (int)(p % (hv1 - hv0));
    const long t0 = cu_seqlens ? cu_seqlens[n] : 0;
    const long t1 = cu_seqlens ? cu_seqlens[n + 1] : d->total_tokens;
    const long T = t1 - t0;
    double* S = (double*)malloc(sizeof(double) * dv * dk);
    for (long i = 0; i < (long)dv * dk; ++i)
      S[i] = init_state ? init_state[((size_t)n * hv + h) * dv * dk + i] : 0.0;
    if (T > 0) {
      double* qh = (double*)malloc(sizeof(double) * T * dk);
      double* kh = (double*)malloc(sizeof(double) * T * dk);
      double* vv = (double*)malloc(sizeof(double) * T * dv);
      double* g = (double*)malloc(sizeof(double) * T);
      double* beta = (double*)malloc(sizeof(double) * T);
      double* colbuf = (double*)malloc(sizeof(double) * T);
      double* colout = (double*)malloc(sizeof(double) * T);
      double* yr = (double*)malloc(sizeof(double) * T * dv);
      double* zz = (double*)malloc(sizeof(double) * dv);
      double* nw = (double*)malloc(sizeof(double) * dv);
      double* yo = (double*)malloc(sizeof(double) * dv);
      or_prepare_head(d, t0, T, h, q, k, v, a, b, A_log, dt_bias, conv_w, NULL, qh, kh, vv, g,
                      beta, colbuf, colout);
      if (d->chunk > 0)
        oracle_recurrence_chunked(T, dk, dv, d->chunk, qh, kh, vv, g, beta, d->q_scale, S, yr);
      else
        oracle_recurrence_token(T, dk, dv, qh, kh, vv, g, beta, d->q_scale, S, yr);
      for (int i = 0; i < dv; ++i) nw[i] = norm_w[i];
      for (long t = 0; t < T; ++t) {
        const size_t row = ((size_t)(t0 + t) * hv + h) * dv;
        for (int i = 0; i < dv; ++i) zz[i] = or_load(z, row + i, d->in_enc);
        oracle_gated_rmsnorm(yr + t * dv, zz, nw, dv, d->rms_eps, yo);
        for (int i = 0; i < dv; ++i) {
          y[row + i] = yo[i];
          if (y_raw_out) y_raw_out[row + i] = yr[t * dv + i];
        }
      }
      free(qh); free(kh); free(vv); free(g); free(beta); free(colbuf); free(colout);
      free(yr); free(zz); free(nw); free(yo);
    }
    if (final_state)
      memcpy(final_state + ((size_t)n * hv + h) * dv * dk, S, sizeof(double) * dv * dk);
    free(S);
  }
  return 0;
}

/*
 * One decode step: one new token per sequence, on resident state and conv history.
 *   q, k [N][h_qk][d_k]; v, z [N][h_v][d_v]; a, b [N][h_v];
 *   conv_state [N][3][C_conv] (raw x_{t-3}, x_{t-2}, x_{t-1}, input encoding);
 *   state [N][h_v][d_v][d_k] fp32 (read only here).
 * Outputs: y [N][h_v][d_v], state_out [N][h_v][d_v][d_k] fp64 (S after the token) and
 * conv_state_out [N][3][C_conv] fp64 = raw [x_{t-2}, x_{t-1}, x_t].
 */
int oracle_decode(const oracle_dims* d, const void* q, const void* k, const void* v,
                  const void* z, const float* a, const float* b, const float* A_log,
                  const float* dt_bias, const float* conv_w, const float* norm_w,
                  const void* conv_state, const float* state, double* y, double* y_raw_out,
                  double* state_out, double* conv_state_out) {
  const int dk = d->d_k, dv = d->d_v, hq = d->h_qk, hv = d->h_v;
  if (d->n_seqs < 1 || hq < 1 || hv % hq) return -1;
  const int nseq = d->n_seqs;
  const long cconv = 2L * hq * dk + (long)hv * dv;
  const long npair = (long)nseq * hv;
#ifdef _OPENMP
  int nt = d->n_threads > 0 ? d->n_threads : omp_get_max_threads();
#pragma omp parallel for schedule(dynamic, 16) num_threads(nt)
#endif
  for (long p = 0; p < npair; ++p) {
    const int n = (int)(p / hv), h = (int)(p % hv);
    double qh[512], kh[512], vv[512], g, beta, colbuf[1], colout[1];
    double* S = (double*)malloc(sizeof(double) * dv * dk);
    double yr[512], zz[512], nw[512], yo[512];
    /* The token is row n of the [N][..] inputs: present it as a one-token sequence at
     * position t0 = n of a packed layout with the same per-token row strides. */
    or_prepare_head(d, n, 1, h, q, k, v, a, b, A_log, dt_bias, conv_w,
                    (const uint8_t*)conv_state +
                        (size_t)n * 3 * cconv * (d->in_enc == OR_ENC_BF16 ? 2 : 4),
                    qh, kh, vv, &g, &beta, colbuf, colout);
    for (long i = 0; i < (long)dv * dk; ++i) S[i] = state[((size_t)n * hv + h) * dv * dk + i];
    oracle_recurrence_token(1, dk, dv, qh, kh, vv, &g, &beta, d->q_scale, S, yr);
    for (int i = 0; i < dv; ++i) {
      zz[i] = or_load(z, ((size_t)n * hv + h) * dv + i, d->in_enc);
      nw[i] = norm_w[i];
    }
    oracle_gated_rmsnorm(yr, zz, nw, dv, d->rms_eps, yo);
    for (int i = 0; i < dv; ++i) {
      y[((size_t)n * hv + h) * dv + i] = yo[i];
      if (y_raw_out) y_raw_out[((size_t)n * hv + h) * dv + i] = yr[i];
    }
    if (state_out) memcpy(state_out + ((size_t)n * hv + h) * dv * dk, S, sizeof(double) * dv * dk);
    free(S);
  }
  /* conv history shift: raw [x_{t-2}, x_{t-1}, x_t] per channel */
  if (conv_state_out)
    for (int n = 0; n < nseq; ++n)
      for (long c = 0; c < cconv; ++c) {
        double xt;
        if (c < (long)hq * dk)
          xt = or_load(q, (size_t)n * hq * dk + c, d->in_enc);
        else if (c < 2L * hq * dk)
          xt = or_load(k, (size_t)n * hq * dk + (c - (long)hq * dk), d->in_enc);
        else
          xt = or_load(v, (size_t)n * hv * dv + (c - 2L * hq * dk), d->in_enc);
        double* o = conv_state_out + (size_t)n * 3 * cconv;
        o[0 * cconv + c] = or_load(conv_state, ((size_t)n * 3 + 1) * cconv + c, d->in_enc);
        o[1 * cconv + c] = or_load(conv_state, ((size_t)n * 3 + 2) * cconv + c, d->in_enc);
        o[2 * cconv + c] = xt;
      }
  return 0;
}
