/*
 * gdla_oracle.c -- fp64 CPU oracle for the forward pass of Grouped Differential
 * Latent Attention (GDLA).
 *
 * TEST INFRASTRUCTURE. Only the test suite, the smoke check and the CPU-baseline
 * leg of the benchmark load this file. The product path (the CUDA library) never
 * does, and this file shares no code, header or table with it.
 *
 * It follows the statement of the layer in "Motif 3: Technical Report"
 * (montaan.com/papers/2608.09119), section "Architecture" (the GDLA paragraphs
 * and the model-configuration paragraph), step by step, in plain loops:
 *
 *   1. the whole compressed KV latent is RMS-normalised once;
 *   2. one up-projection W_UKV expands it into n_kv content-key (nope) and
 *      value heads that both query paths share;
 *   3. RoPE is applied only to the rotary query part and to the decoupled
 *      rotary key (one per token, shared by all heads);
 *   4. scores s = tau * (q_nope . k_nope + q_rope . k_rope) under a full causal
 *      or sliding-window mask;
 *   5. softmax over the visible keys;
 *   6. H = sum_j p_j v_j, separately for every signal and noise head;
 *   7. D = H_S - lambda * Repeat_g(H_N), lambda = sigmoid(lambda logit);
 *   8. Y = sigmoid(G) * D, the element-wise output gate.
 *
 * The definitions it borrows from "Open-Source Frontier Models: Architecture
 * and Benchmarks of Rnj-1 and Motif-2" (akillness.github.io):
 *   - scaled dot-product softmax with scale 1/sqrt(d_k) (section 1, the
 *     attention equation);
 *   - sliding-window attention: a token sees the W most recent tokens
 *     (section 1);
 *   - RoPE block rotation with theta_i = b^(-2(i-1)/d) (section 2, the RoPE
 *     equation), with the rotate-half pairing (k, k + d/2) of the
 *     implementation section.
 *
 * Readings where the pages are silent (each is also listed with the design
 * notes): RMSNorm with a learnable gain gamma and epsilon (the report says only
 * "normalized"); signal head i uses KV head and noise head floor(i/g)
 * (Repeat_g read as repeat-interleave); one lambda per (token, signal head),
 * broadcast over d_v; key j is visible to query i under a window W iff
 * i - W < j <= i; token t of a prefill sequence sits at position t; the decode
 * cache holds the normalised latent and the already-rotated rotary key.
 *
 * Everything is double precision. No blocking, fusion or reordering is done
 * beyond computing one KV group at a time.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_MASK_CAUSAL 0
#define ORACLE_MASK_SLIDING 1

int gdla_oracle_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

/* ---- step 1: RMS normalisation of the compressed KV latent --------------------
 * c_hat[t,k] = gamma[k] * c[t,k] / sqrt(mean_k c[t,k]^2 + eps)
 */
void gdla_oracle_latent_norm(const double* c, const double* gamma, long T, int d_c,
                             double eps, double* c_hat) {
  for (long t = 0; t < T; ++t) {
    const double* ct = c + t * d_c;
    double ss = 0.0;
    for (int k = 0; k < d_c; ++k) ss += ct[k] * ct[k];
    double r = 1.0 / sqrt(ss / d_c + eps);
    for (int k = 0; k < d_c; ++k) c_hat[t * d_c + k] = gamma[k] * ct[k] * r;
  }
}

/* The inputs of the differential epilogue from the layer's activations ("Motif 3:
 * Technical Report", section "Architecture": lambda_t = sigmoid(x_t W_lambda), and
 * an element-wise sigmoid gate computed from the normalised query latent, i.e.
 * G_t = c_hat_Q,t W_G): a plain row-by-matrix product
 *   out[t, n] = sum_{k=0}^{K-1} a[t, k] * w[k, n],
 * summed in increasing k. The query latent is normalised with
 * gdla_oracle_latent_norm before it is projected. */
void gdla_oracle_project(const double* a, long T, int K, const double* w, int N, double* out) {
  for (long t = 0; t < T; ++t)
    for (int n = 0; n < N; ++n) {
      double acc = 0.0;
      for (int k = 0; k < K; ++k) acc += a[t * K + k] * w[(long)k * N + n];
      out[t * N + n] = acc;
    }
}

/* One token of step 2: out[n] = sum_{k=0}^{d_c-1} c_hat[k] * W[k, col0+n], summed in
 * increasing k for every n (the loop over n is innermost only for memory order). */
static void expand_token(const double* c_hat_t, const double* w_ukv, int d_c, long ncol, long col0,
                         int d_n, int d_v, double* k_n_t, double* v_t) {
  double acc[1024];
  const int nn = d_n + d_v;
  for (int n = 0; n < nn; ++n) acc[n] = 0.0;
  for (int k = 0; k < d_c; ++k) {
    const double a = c_hat_t[k];
    const double* wr = w_ukv + k * ncol + col0;
    for (int n = 0; n < nn; ++n) acc[n] += a * wr[n];
  }
  for (int n = 0; n < d_n; ++n) k_n_t[n] = acc[n];
  for (int n = 0; n < d_v; ++n) v_t[n] = acc[d_n + n];
}

/* ---- step 2: one up-projection into n_kv key (nope) and value heads ------------
 * W_UKV is [d_c, n_kv*(d_n+d_v)] row-major; the columns of KV head h are
 * h*(d_n+d_v) .. h*(d_n+d_v)+d_n-1 for the key and the next d_v for the value.
 * Only head `h` is produced: k_n [T, d_n], v [T, d_v].
 */
void gdla_oracle_expand_head(const double* c_hat, const double* w_ukv, long T, int d_c,
                             int n_kv, int d_n, int d_v, int h, double* k_n, double* v) {
  const long ncol = (long)n_kv * (d_n + d_v);
  const long col0 = (long)h * (d_n + d_v);
#pragma omp parallel for schedule(static)
  for (long t = 0; t < T; ++t) expand_token(c_hat + t * d_c, w_ukv, d_c, ncol, col0, d_n, d_v,
                                            k_n + t * d_n, v + t * d_v);
}

/* ---- step 3: RoPE, rotate-half pairing -----------------------------------------
 * theta_k = base^(-2k/d_R), k = 0 .. d_R/2-1; the pair (x[k], x[k+d_R/2]) is
 * rotated by the angle pos*theta_k.
 */
static void rope_apply(const double* x, long pos, int d_R, double base, const double* inv_freq, double* y) {
  const int half = d_R / 2;
  for (int k = 0; k < half; ++k) {
    /* the frequencies come from the base, or are given (a rescaled RoPE such as YaRN) */
    double theta = inv_freq ? inv_freq[k] : pow(base, -2.0 * k / (double)d_R);
    double a = (double)pos * theta;
    double c = cos(a), s = sin(a);
    double x1 = x[k], x2 = x[k + half];
    y[k] = x1 * c - x2 * s;
    y[k + half] = x2 * c + x1 * s;
  }
}

void gdla_oracle_rope(const double* x, long pos, int d_R, double base, double* y) {
  rope_apply(x, pos, d_R, base, 0, y);
}

/* ---- YaRN frequency scaling ("Open-Source Frontier Models: Architecture and Benchmarks of Rnj-1 and Motif-2", section 2) ----
 * Extending the context by a factor s = L_new / L_native: with the wavelength of
 * frequency k, lambda_k = 2 pi / theta_k, frequencies whose wavelength is below
 * orig/beta_fast are kept (scale 1), those above orig/beta_slow are interpolated
 * (scale 1/s), and in between the scale moves linearly with the wavelength:
 *   alpha_k = clamp((lambda_k - orig/beta_fast) / (orig/beta_slow - orig/beta_fast), 0, 1)
 *   theta'_k = theta_k * ((1 - alpha_k) + alpha_k / s).
 * The logit temperature is a separate factor (see the Python wrapper). */
void gdla_oracle_yarn_inv_freq(int d_R, double base, double factor, double orig_max_pos, double beta_fast,
                               double beta_slow, double* inv_freq) {
  const int half = d_R / 2;
  const double lam_fast = orig_max_pos / beta_fast, lam_slow = orig_max_pos / beta_slow;
  for (int k = 0; k < half; ++k) {
    const double theta = pow(base, -2.0 * k / (double)d_R);
    const double lam = 2.0 * acos(-1.0) / theta;  /* 2 pi / theta */
    double alpha;
    if (lam_slow > lam_fast) {
      alpha = (lam - lam_fast) / (lam_slow - lam_fast);
      alpha = alpha < 0.0 ? 0.0 : (alpha > 1.0 ? 1.0 : alpha);
    } else {
      alpha = lam > lam_fast ? 1.0 : 0.0;
    }
    inv_freq[k] = theta * ((1.0 - alpha) + alpha / factor);
  }
}

/* The cos/sin table the oracle itself would use: tab[pos*half + k]. */
void gdla_oracle_rope_table(long max_pos, int d_R, double base, double* cos_tab,
                            double* sin_tab) {
  const int half = d_R / 2;
  for (long p = 0; p < max_pos; ++p)
    for (int k = 0; k < half; ++k) {
      double a = (double)p * pow(base, -2.0 * k / (double)d_R);
      cos_tab[p * half + k] = cos(a);
      sin_tab[p * half + k] = sin(a);
    }
}

/* Is key j visible to query i? */
static int visible(long i, long j, int mask, long window) {
  if (j > i || j < 0) return 0;
  if (mask == ORACLE_MASK_SLIDING) return j > i - window;
  return 1;
}

/* ---- steps 4-6: one query row of one head ---------------------------------------
 * q_n [d_n], q_r [d_R] (already rotated), keys/values indexed by absolute token
 * j with row strides; returns H = sum_j softmax_j(s) v_j in h_out [d_v]. If
 * p_out is not NULL it receives the probabilities for j = 0..i (zero where
 * masked).
 */
void gdla_oracle_attend_row(const double* q_n, const double* q_r, const double* k_n,
                            long k_n_stride, const double* k_r, long k_r_stride,
                            const double* v, long v_stride, int d_n, int d_R, int d_v, long i,
                            int mask, long window, double scale, double* h_out,
                            double* p_out) {
  double* s = (double*)malloc(sizeof(double) * (size_t)(i + 1));
  double smax = -INFINITY;
  for (long j = 0; j <= i; ++j) {
    if (!visible(i, j, mask, window)) {
      s[j] = -INFINITY;
      continue;
    }
    double dot = 0.0;
    for (int k = 0; k < d_n; ++k) dot += q_n[k] * k_n[j * k_n_stride + k];
    for (int k = 0; k < d_R; ++k) dot += q_r[k] * k_r[j * k_r_stride + k];
    s[j] = scale * dot;
    if (s[j] > smax) smax = s[j];
  }
  double denom = 0.0;
  for (long j = 0; j <= i; ++j) {
    s[j] = (s[j] == -INFINITY) ? 0.0 : exp(s[j] - smax);
    denom += s[j];
  }
  for (int n = 0; n < d_v; ++n) h_out[n] = 0.0;
  for (long j = 0; j <= i; ++j) {
    double p = s[j] / denom;
    if (p_out) p_out[j] = p;
    if (p == 0.0) continue;
    for (int n = 0; n < d_v; ++n) h_out[n] += p * v[j * v_stride + n];
  }
  free(s);
}

static double sigmoid(double x) { return 1.0 / (1.0 + exp(-x)); }

/* ---- steps 7-8: grouped differential and output gate ----------------------------
 * For one token: signal heads h_s [n_S, d_v], noise heads h_nz [n_N, d_v],
 * lambda logits lam [n_S], gate logits gate [n_S, d_v] -> y [n_S, d_v].
 *   D_i = H_S,i - sigmoid(lam_i) * H_N,floor(i/g);  Y = sigmoid(G) * D
 */
void gdla_oracle_differential_gate(const double* h_s, const double* h_nz, const double* lam,
                                   const double* gate, int n_S, int g, int d_v, double* y) {
  for (int i = 0; i < n_S; ++i) {
    double l = sigmoid(lam[i]);
    const double* hn = h_nz + (long)(i / g) * d_v;
    for (int n = 0; n < d_v; ++n) {
      double d = h_s[(long)i * d_v + n] - l * hn[n];
      y[(long)i * d_v + n] = sigmoid(gate[(long)i * d_v + n]) * d;
    }
  }
}

/* ---- prefill: selected output rows ----------------------------------------------
 * Inputs (all double, row-major):
 *   c_kv   [B, L, d_c]   pre-norm latent         gamma [d_c]
 *   k_rope [B, L, d_R]   pre-RoPE rotary key     w_ukv [d_c, n_kv*(d_n+d_v)]
 *   rows   nrows pairs (row_b[r], row_i[r]): which query tokens to compute
 *   q_rows [nrows, n_S+n_N, d_n+d_R]  heads 0..n_S-1 signal, then the n_N noise
 *          heads; per head the nope part first, then the pre-RoPE rotary part
 *   lam_rows [nrows, n_S]; gate_rows [nrows, n_S, d_v]
 * kv_sel [n_kv] (optional) restricts the work to the KV groups whose flag is
 * non-zero (their noise head and g signal heads); the other groups' outputs are
 * zero.
 * Outputs: y_rows [nrows, n_S, d_v]; heads_out (optional) [nrows, n_S+n_N, d_v]
 * holds every head's H before the differential step.
 * n_N must equal n_kv. Returns 0, or -1 on bad arguments.
 */
int gdla_oracle_prefill_rows(int B, long L, int d_c, int d_R, int n_kv, int d_n, int d_v,
                             int g, int mask, long window, double scale, double eps,
                             double rope_base, const double* inv_freq, const double* c_kv, const double* gamma,
                             const double* k_rope, const double* w_ukv, long nrows,
                             const long* row_b, const long* row_i, const double* q_rows,
                             const double* lam_rows, const double* gate_rows, const int* kv_sel,
                             double* y_rows, double* heads_out) {
  if (B < 1 || L < 1 || g < 1 || n_kv < 1 || d_R % 2 || d_R > 512 || d_n + d_v > 1024 ||
      (mask == ORACLE_MASK_SLIDING && window < 1))
    return -1;
  const int n_N = n_kv, n_S = g * n_N, H_q = n_S + n_N, d_qk = d_n + d_R;
  for (long r = 0; r < nrows; ++r)
    if (row_b[r] < 0 || row_b[r] >= B || row_i[r] < 0 || row_i[r] >= L) return -1;

  double* heads = (double*)calloc((size_t)nrows * H_q * d_v, sizeof(double));
  double* c_hat = (double*)malloc(sizeof(double) * (size_t)L * d_c);
  double* k_r_rot = (double*)malloc(sizeof(double) * (size_t)L * d_R);
  double* k_n = (double*)malloc(sizeof(double) * (size_t)L * d_n);
  double* v = (double*)malloc(sizeof(double) * (size_t)L * d_v);
  char* need = (char*)malloc((size_t)L);

  for (int b = 0; b < B; ++b) {
    /* which tokens of sequence b any selected row can see */
    memset(need, 0, (size_t)L);
    long maxtok = -1;
    for (long r = 0; r < nrows; ++r) {
      if (row_b[r] != b) continue;
      long i = row_i[r];
      long lo = (mask == ORACLE_MASK_SLIDING && i - window + 1 > 0) ? i - window + 1 : 0;
      for (long j = lo; j <= i; ++j) need[j] = 1;
      if (i > maxtok) maxtok = i;
    }
    if (maxtok < 0) continue;
    const long T = maxtok + 1;

    /* step 1 (the whole latent) and step 3 for the shared rotary key */
    gdla_oracle_latent_norm(c_kv + (long)b * L * d_c, gamma, T, d_c, eps, c_hat);
    for (long j = 0; j < T; ++j)
      rope_apply(k_rope + ((long)b * L + j) * d_R, j, d_R, rope_base, inv_freq, k_r_rot + j * d_R);

    for (int h = 0; h < n_kv; ++h) {
      if (kv_sel && !kv_sel[h]) continue;
      /* step 2 for KV head h, only at the tokens that are needed */
      const long ncol = (long)n_kv * (d_n + d_v);
      const long col0 = (long)h * (d_n + d_v);
#pragma omp parallel for schedule(static)
      for (long t = 0; t < T; ++t)
        if (need[t])
          expand_token(c_hat + t * d_c, w_ukv, d_c, ncol, col0, d_n, d_v, k_n + t * d_n, v + t * d_v);
      /* steps 3-6 for the heads that read KV head h: noise head h and signal
       * heads h*g .. h*g+g-1 */
#pragma omp parallel for schedule(dynamic)
      for (long rr = 0; rr < nrows * (g + 1); ++rr) {
        long r = rr / (g + 1);
        int which = (int)(rr % (g + 1));
        if (row_b[r] != b) continue;
        int head = (which < g) ? h * g + which : n_S + h;
        long i = row_i[r];
        const double* qh = q_rows + ((long)r * H_q + head) * d_qk;
        double q_r[512];
        rope_apply(qh + d_n, i, d_R, rope_base, inv_freq, q_r);
        gdla_oracle_attend_row(qh, q_r, k_n, d_n, k_r_rot, d_R, v, d_v, d_n, d_R, d_v, i, mask,
                               window, scale, heads + ((long)r * H_q + head) * d_v, NULL);
      }
    }
  }

  /* steps 7-8 */
  for (long r = 0; r < nrows; ++r)
    gdla_oracle_differential_gate(heads + (long)r * H_q * d_v,
                                  heads + ((long)r * H_q + n_S) * d_v, lam_rows + r * n_S,
                                  gate_rows + r * n_S * d_v, n_S, g, d_v,
                                  y_rows + r * n_S * d_v);
  if (heads_out) memcpy(heads_out, heads, sizeof(double) * (size_t)nrows * H_q * d_v);
  free(heads);
  free(c_hat);
  free(k_r_rot);
  free(k_n);
  free(v);
  free(need);
  return 0;
}

/* ---- decode: one new token of one sequence over its latent cache ---------------
 * The cache holds, for tokens 0..T-1, the normalised latent c_hat [T, d_c] and
 * the rotated rotary key [T, d_R]. The query q [n_S+n_N, d_n+d_R] (rotary part
 * pre-RoPE) sits at position T-1. Keys and values are expanded from the cache
 * with W_UKV exactly as in prefill (no absorption). kv_sel [n_kv] (optional)
 * restricts the work to the KV groups whose flag is non-zero; rows of y for
 * the other groups are left untouched.
 */
int gdla_oracle_decode_seq(long T, int d_c, int d_R, int n_kv, int d_n, int d_v, int g,
                           int mask, long window, double scale, double rope_base, const double* inv_freq,
                           const double* c_hat, const double* k_r_rot, const double* q,
                           const double* w_ukv, const double* lam, const double* gate,
                           const int* kv_sel, double* y, double* heads_out) {
  if (T < 1 || g < 1 || n_kv < 1 || d_R % 2 || d_R > 512 || d_n + d_v > 1024 ||
      (mask == ORACLE_MASK_SLIDING && window < 1))
    return -1;
  const int n_N = n_kv, n_S = g * n_N, H_q = n_S + n_N, d_qk = d_n + d_R;
  const long i = T - 1;
  double* heads = (double*)calloc((size_t)H_q * d_v, sizeof(double));
  double* k_n = (double*)malloc(sizeof(double) * (size_t)T * d_n);
  double* v = (double*)malloc(sizeof(double) * (size_t)T * d_v);
  for (int h = 0; h < n_kv; ++h) {
    if (kv_sel && !kv_sel[h]) continue;
    gdla_oracle_expand_head(c_hat, w_ukv, T, d_c, n_kv, d_n, d_v, h, k_n, v);
#pragma omp parallel for schedule(dynamic)
    for (int which = 0; which <= g; ++which) {
      int head = (which < g) ? h * g + which : n_S + h;
      const double* qh = q + (long)head * d_qk;
      double q_r[512];
      rope_apply(qh + d_n, i, d_R, rope_base, inv_freq, q_r);
      gdla_oracle_attend_row(qh, q_r, k_n, d_n, k_r_rot, d_R, v, d_v, d_n, d_R, d_v, i, mask,
                             window, scale, heads + (long)head * d_v, NULL);
    }
    /* steps 7-8 for this group's signal heads */
    double* tmp = (double*)malloc(sizeof(double) * (size_t)g * d_v);
    gdla_oracle_differential_gate(heads + (long)h * g * d_v, heads + (long)(n_S + h) * d_v,
                                  lam + (long)h * g, gate + (long)h * g * d_v, g, g, d_v, tmp);
    memcpy(y + (long)h * g * d_v, tmp, sizeof(double) * (size_t)g * d_v);
    free(tmp);
  }
  if (heads_out) memcpy(heads_out, heads, sizeof(double) * (size_t)H_q * d_v);
  free(heads);
  free(k_n);
  free(v);
  return 0;
}
