/*
 * Float64 CPU oracle for the GDLA (Grouped Differential Latent Attention)
 * forward pass.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may link, load or
 * call this file: it exists so that tests, the smoke check and the benchmark's
 * CPU-baseline leg can compare the CUDA kernels against a plain, slow,
 * obviously correct restatement of the method.  It shares no code, header or
 * constant with the CUDA library.
 *
 * Sources (web pages; "step 2" is the page's own numbering):
 *   [R]  "Motif 3: Technical Report" digest at paper.rainbus.top, step 2
 *        ("GDLA forward"): x_t -> query latent c^Q_t (1024) and KV latent
 *        c_KV,t (512) -> RMSNorm -> W^KV_b expands 16 KV heads -> signal and
 *        noise query paths each attend over the shared KV heads -> noise output
 *        repeated g times per group -> D_t = H_S,t - lambda_t (.) Repeat_g(H_N,t)
 *        -> sigmoid gate G_t from the query latent multiplies D_t elementwise
 *        -> W^O.  Same page, "technical novelty" paragraph: both query paths
 *        share one up-projected KV; lambda is per token and sigmoid-bounded.
 *   [P]  "Вышла новая модель Motif 3" (pikabu.ru): 16 shared KV heads for
 *        64 signal / 16 noise query heads; window 128 with full attention in
 *        every 4th layer.
 *
 * Readings taken where the pages are silent:
 *   - signal head h uses KV head floor(h/g) and noise head floor(h/g)
 *     (interleaved repeat: "repeat per group" in [R]);
 *   - noise head n uses KV head n (Hn == Hkv);
 *   - lambda is one scalar per (token, signal head); lambda and the gate arrive
 *     already passed through their sigmoids;
 *   - sliding window W keeps keys j with i-W < j <= i; W = 0 means full causal;
 *   - RMSNorm is c / sqrt(mean(c^2) + eps) * w;
 *   - the W^KV_b columns of KV head h are [K_h (dk) | V_h (dv)];
 *   - decoupled rotary term ([R] "technical novelty" paragraph: both query
 *     paths share the up-projected KV and one broadcast decoupled rotary
 *     key): every head of both paths has its own rotary query q_r (d_rope
 *     wide), every token one rotary key k_r shared by all heads, and the
 *     score is scale * (q . k + q_r . k_r).  The rotation itself is applied
 *     before the attention (q_r and k_r arrive rotated), as lambda and the
 *     gate arrive after their sigmoids.  d_rope = 0 is the score without it.
 *
 * Every function computes in double, in the order the definition is written:
 * no tiling, no online softmax, no reassociation.  Inputs may be given as
 * bfloat16 bit patterns, float32 or float64 (dtype codes below); bfloat16 and
 * float32 widen to double exactly.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_BF16 0
#define ORACLE_F64 1
#define ORACLE_F32 2

static double load_elem(const void *p, int dtype, int64_t i) {
  if (dtype == ORACLE_F64) return ((const double *)p)[i];
  if (dtype == ORACLE_F32) return (double)((const float *)p)[i];
  /* bfloat16: the upper 16 bits of an IEEE binary32 */
  uint32_t bits = ((uint32_t)((const uint16_t *)p)[i]) << 16;
  float f;
  memcpy(&f, &bits, sizeof f);
  return (double)f;
}

int gdla_oracle_version(void) { return 1; }

/*
 * RMSNorm of the KV latent ([R] step 2: "c_KV,t ... -> RMSNorm").
 *   out[t, k] = c[t, k] / sqrt(mean_k c[t, k]^2 + eps) * w[k]
 * w == NULL means a weight of ones.
 */
void gdla_oracle_rmsnorm(const void *c, int c_dt, const void *w, int w_dt,
                         double eps, int64_t n_tokens, int d_latent,
                         double *out) {
  int64_t t;
#pragma omp parallel for schedule(static)
  for (t = 0; t < n_tokens; ++t) {
    double ss = 0.0;
    for (int k = 0; k < d_latent; ++k) {
      double x = load_elem(c, c_dt, t * d_latent + k);
      ss += x * x;
    }
    double r = sqrt(ss / (double)d_latent + eps);
    for (int k = 0; k < d_latent; ++k) {
      double wk = w ? load_elem(w, w_dt, k) : 1.0;
      out[t * d_latent + k] = load_elem(c, c_dt, t * d_latent + k) / r * wk;
    }
  }
}

/*
 * Up-projection W^KV_b ([R] step 2: "W^KV_b expands 16 KV heads").
 *   KV[t, col] = sum_k c_hat[t, k] * W[k, col],  W is [d_latent, Hkv*(dk+dv)]
 *   K[t, h, x] = KV[t, h*(dk+dv) + x]          for x <  dk
 *   V[t, h, x] = KV[t, h*(dk+dv) + dk + x]     for x <  dv
 */
void gdla_oracle_kv_expand(const double *c_hat, const void *w, int w_dt,
                           int64_t n_tokens, int d_latent, int n_kv_heads,
                           int dk, int dv, double *k_out, double *v_out) {
  const int64_t ncol = (int64_t)n_kv_heads * (dk + dv);
  int64_t t;
#pragma omp parallel for schedule(static)
  for (t = 0; t < n_tokens; ++t) {
    for (int64_t col = 0; col < ncol; ++col) {
      double acc = 0.0;
      for (int k = 0; k < d_latent; ++k)
        acc += c_hat[t * d_latent + k] * load_elem(w, w_dt, (int64_t)k * ncol + col);
      int64_t h = col / (dk + dv), x = col % (dk + dv);
      if (x < dk)
        k_out[(t * n_kv_heads + h) * dk + x] = acc;
      else
        v_out[(t * n_kv_heads + h) * dv + (x - dk)] = acc;
    }
  }
}

/* Key range kept by the mask for query i ([P]: window 128, full attention
 * every 4th layer).  causal == 0: all keys.  causal, window == 0: j <= i.
 * causal, window W > 0: i - W < j <= i. */
static void key_range(int64_t i, int64_t T, int64_t window, int causal,
                      int64_t *lo, int64_t *hi) {
  if (!causal) {
    *lo = 0;
    *hi = T - 1;
    return;
  }
  *hi = i;
  *lo = 0;
  if (window > 0 && i - window + 1 > 0) *lo = i - window + 1;
}

/*
 * One attention path (signal or noise), [R] step 2: each query path attends
 * over the shared KV heads.  For every requested row r = b*T + i and head h:
 *   s_j = scale * sum_c Q[b,i,h,c] K[b,j,kv(h),c]         j in J(i)
 *   p_j = exp(s_j - max_j s_j)
 *   H[row, h, :] = sum_j p_j V[b,j,kv(h),:] / sum_j p_j
 * kv(h) = h / (H / Hkv).  Q is [B,T,H,d], K and V are [B,T,Hkv,d].
 * With the decoupled rotary term (dr > 0) the score of key j adds
 *   sum_c Qr[b,i,h,c] Kr[b,j,c]                            c < dr
 * inside the scale: Qr is [B,T,H,dr] (laid out like Q), Kr is [B,T,dr], one
 * rotary key per token for every head.  dr == 0 leaves the score as above.
 * rows == NULL means every row (n_rows must then be B*T).
 */
static void attention_path_impl(const void *q, int q_dt, int q_compact,
                                const void *qr, int qr_dt, const void *k,
                                int k_dt, const void *kr, int kr_dt, int dr,
                                const void *v, int v_dt, int64_t T, int H,
                                int Hkv, int d, int64_t window, int causal,
                                double scale, const int64_t *rows,
                                int64_t n_rows, double *out) {
  const int group = H / Hkv;
  int64_t task;
#pragma omp parallel
  {
    double *s = (double *)malloc(sizeof(double) * (size_t)(T > 0 ? T : 1));
    double *acc = (double *)malloc(sizeof(double) * (size_t)d);
#pragma omp for schedule(dynamic, 1)
    for (task = 0; task < n_rows * H; ++task) {
      int64_t ri = task / H;
      int h = (int)(task % H);
      int64_t row = rows ? rows[ri] : ri;
      int64_t b = row / T, i = row % T;
      int kvh = h / group;
      int64_t lo, hi;
      key_range(i, T, window, causal, &lo, &hi);
      const int64_t qoff = ((q_compact ? ri : row) * H + h) * d;
      const int64_t qroff = ((q_compact ? ri : row) * H + h) * (int64_t)dr;
      double m = -INFINITY;
      for (int64_t j = lo; j <= hi; ++j) {
        const int64_t koff = ((b * T + j) * Hkv + kvh) * d;
        double dot = 0.0;
        for (int c = 0; c < d; ++c)
          dot += load_elem(q, q_dt, qoff + c) * load_elem(k, k_dt, koff + c);
        /* the rotary key of token j: one vector for every head */
        for (int c = 0; c < dr; ++c)
          dot += load_elem(qr, qr_dt, qroff + c) *
                 load_elem(kr, kr_dt, (b * T + j) * (int64_t)dr + c);
        s[j - lo] = scale * dot;
        if (s[j - lo] > m) m = s[j - lo];
      }
      double denom = 0.0;
      for (int c = 0; c < d; ++c) acc[c] = 0.0;
      for (int64_t j = lo; j <= hi; ++j) {
        const double p = exp(s[j - lo] - m);
        const int64_t voff = ((b * T + j) * Hkv + kvh) * d;
        denom += p;
        for (int c = 0; c < d; ++c) acc[c] += p * load_elem(v, v_dt, voff + c);
      }
      double *o = out + (ri * H + h) * d;
      for (int c = 0; c < d; ++c) o[c] = acc[c] / denom;
    }
    free(s);
    free(acc);
  }
}

void gdla_oracle_attention_path(const void *q, int q_dt, const void *k,
                                int k_dt, const void *v, int v_dt, int B,
                                int64_t T, int H, int Hkv, int d,
                                int64_t window, int causal, double scale,
                                const int64_t *rows, int64_t n_rows,
                                double *out) {
  (void)B;
  attention_path_impl(q, q_dt, 0, NULL, ORACLE_F64, k, k_dt, NULL, ORACLE_F64, 0,
                      v, v_dt, T, H, Hkv, d, window, causal, scale, rows, n_rows,
                      out);
}

/*
 * Differential combine and output gate, [R] step 2:
 *   D[h]  = H_S[h] - lambda[h] * H_N[h / g]          (Repeat_g, interleaved)
 *   O[h]  = G[h*d : (h+1)*d] (.) D[h]
 * hs: [n_rows, Hs, d], hn: [n_rows, Hn, d] (already gathered per row).
 * lambda: [B*T, Hs], gate: [B*T, Hs*d], both addressed by the flat row index
 * rows[ri] (rows == NULL: ri itself).  out: [n_rows, Hs*d].
 */
static void differential_gate_impl(const double *hs, const double *hn,
                                   const void *lam, int lam_dt,
                                   const void *gate, int gate_dt,
                                   int lg_compact, int Hs, int Hn, int d,
                                   const int64_t *rows, int64_t n_rows,
                                   double *out) {
  const int g = Hs / Hn;
  int64_t ri;
#pragma omp parallel for schedule(static)
  for (ri = 0; ri < n_rows; ++ri) {
    const int64_t row = (rows && !lg_compact) ? rows[ri] : ri;
    for (int h = 0; h < Hs; ++h) {
      const double l = load_elem(lam, lam_dt, row * Hs + h);
      const int n = h / g;
      for (int c = 0; c < d; ++c) {
        const double diff = hs[(ri * Hs + h) * d + c] - l * hn[(ri * Hn + n) * d + c];
        const double gv = load_elem(gate, gate_dt, row * (int64_t)Hs * d + (int64_t)h * d + c);
        out[ri * (int64_t)Hs * d + (int64_t)h * d + c] = gv * diff;
      }
    }
  }
}

void gdla_oracle_differential_gate(const double *hs, const double *hn,
                                   const void *lam, int lam_dt,
                                   const void *gate, int gate_dt, int Hs,
                                   int Hn, int d, const int64_t *rows,
                                   int64_t n_rows, double *out) {
  differential_gate_impl(hs, hn, lam, lam_dt, gate, gate_dt, 0, Hs, Hn, d,
                         rows, n_rows, out);
}

/*
 * Whole GDLA attention forward for a subset of rows: the signal path over
 * Q_sig (Hs heads, KV head h/g), the noise path over Q_noise (Hn heads, KV
 * head n), then the differential combine and the gate.
 * compact == 0: q_sig, q_noise, lambda and gate are full [B,T,...] tensors.
 * compact == 1: they hold only the evaluated rows, in the order of rows[]
 * (K and V stay full).  Returns 0, or -1 when the head counts do not divide
 * (Hs % Hn, Hn != Hkv).
 */
static int attn_impl(const void *q_sig, int qs_dt, const void *q_noise,
                     int qn_dt, const void *qr_sig, int qrs_dt,
                     const void *qr_noise, int qrn_dt, const void *k, int k_dt,
                     const void *kr, int kr_dt, int dr, const void *v,
                     int v_dt, const void *lam, int lam_dt, const void *gate,
                     int gate_dt, int compact, int64_t T, int Hs, int Hn,
                     int Hkv, int d, int64_t window, int causal, double scale,
                     const int64_t *rows, int64_t n_rows, double *out) {
  if (Hn <= 0 || Hkv <= 0 || Hs % Hn != 0 || Hn != Hkv) return -1;
  double *hs = (double *)malloc(sizeof(double) * (size_t)(n_rows * Hs * d));
  double *hn = (double *)malloc(sizeof(double) * (size_t)(n_rows * Hn * d));
  if (!hs || !hn) {
    free(hs);
    free(hn);
    return -2;
  }
  attention_path_impl(q_sig, qs_dt, compact, qr_sig, qrs_dt, k, k_dt, kr, kr_dt,
                      dr, v, v_dt, T, Hs, Hkv, d, window, causal, scale, rows,
                      n_rows, hs);
  attention_path_impl(q_noise, qn_dt, compact, qr_noise, qrn_dt, k, k_dt, kr,
                      kr_dt, dr, v, v_dt, T, Hn, Hkv, d, window, causal, scale,
                      rows, n_rows, hn);
  differential_gate_impl(hs, hn, lam, lam_dt, gate, gate_dt, compact, Hs, Hn,
                         d, rows, n_rows, out);
  free(hs);
  free(hn);
  return 0;
}

int gdla_oracle_attn(const void *q_sig, int qs_dt, const void *q_noise,
                     int qn_dt, const void *k, int k_dt, const void *v,
                     int v_dt, const void *lam, int lam_dt, const void *gate,
                     int gate_dt, int B, int64_t T, int Hs, int Hn, int Hkv,
                     int d, int64_t window, int causal, double scale,
                     const int64_t *rows, int64_t n_rows, double *out) {
  (void)B;
  return attn_impl(q_sig, qs_dt, q_noise, qn_dt, NULL, ORACLE_F64, NULL,
                   ORACLE_F64, k, k_dt, NULL, ORACLE_F64, 0, v, v_dt, lam,
                   lam_dt, gate, gate_dt, 0, T, Hs, Hn, Hkv, d, window, causal,
                   scale, rows, n_rows, out);
}

int gdla_oracle_attn_compact(const void *q_sig, int qs_dt, const void *q_noise,
                             int qn_dt, const void *k, int k_dt, const void *v,
                             int v_dt, const void *lam, int lam_dt,
                             const void *gate, int gate_dt, int64_t T, int Hs,
                             int Hn, int Hkv, int d, int64_t window,
                             int causal, double scale, const int64_t *rows,
                             int64_t n_rows, double *out) {
  return attn_impl(q_sig, qs_dt, q_noise, qn_dt, NULL, ORACLE_F64, NULL,
                   ORACLE_F64, k, k_dt, NULL, ORACLE_F64, 0, v, v_dt, lam,
                   lam_dt, gate, gate_dt, 1, T, Hs, Hn, Hkv, d, window, causal,
                   scale, rows, n_rows, out);
}

/*
 * gdla_oracle_attn with the decoupled rotary term ([R] "technical novelty"
 * paragraph): qr_sig [.., Hs, dr] and qr_noise [.., Hn, dr] are laid out like
 * q_sig and q_noise (full, or one entry per evaluated row when compact), kr
 * is [B, T, dr], one rotary key per token shared by every head of both
 * paths.  Returns as gdla_oracle_attn.
 */
int gdla_oracle_attn_rope(const void *q_sig, int qs_dt, const void *q_noise,
                          int qn_dt, const void *qr_sig, int qrs_dt,
                          const void *qr_noise, int qrn_dt, const void *k,
                          int k_dt, const void *kr, int kr_dt, int dr,
                          const void *v, int v_dt, const void *lam, int lam_dt,
                          const void *gate, int gate_dt, int compact,
                          int64_t T, int Hs, int Hn, int Hkv, int d,
                          int64_t window, int causal, double scale,
                          const int64_t *rows, int64_t n_rows, double *out) {
  if (dr < 0 || (dr > 0 && (!qr_sig || !qr_noise || !kr))) return -1;
  return attn_impl(q_sig, qs_dt, q_noise, qn_dt, qr_sig, qrs_dt, qr_noise,
                   qrn_dt, k, k_dt, kr, kr_dt, dr, v, v_dt, lam, lam_dt, gate,
                   gate_dt, compact, T, Hs, Hn, Hkv, d, window, causal, scale,
                   rows, n_rows, out);
}

/*
 * Decode over the latent cache ([R] "technical novelty" paragraph: the two
 * query paths share one up-projected KV, so the inference cache is the KV
 * latent alone, the same size as MLA's).  Sequence b has cache_len[b] tokens
 * whose KV latents c_KV are cached; its newest token, i = cache_len[b] - 1,
 * is the query.  The result is the forward pass of [R] step 2 for that one
 * row, written out as the definition:
 *   c_hat = RMSNorm(c_KV[b, 0..i])                 (gdla_oracle_rmsnorm)
 *   K, V  = c_hat W^KV_b                           (gdla_oracle_kv_expand)
 *   O[b]  = G (.) (H_S - lambda Repeat_g(H_N))     for row i (attn_impl)
 * q_sig [B, Hs, d], q_noise [B, Hn, d], lambda [B, Hs], gate [B, Hs*d] hold
 * the query token of each sequence; c_kv is [B, L_max, d_latent].  Only the
 * keys J(i) of the window enter (window 0 = full causal).  out: [B, Hs*d].
 * With the decoupled rotary term (dr > 0) the cache also holds each token's
 * rotary key, kr [B, L_max, dr] (cached beside the latent, as in MLA), and
 * qr_sig [B, Hs, dr], qr_noise [B, Hn, dr] are the query token's rotary
 * queries; dr == 0 ignores all three.
 * Returns 0, -1 for bad head counts or lengths, -2 when out of memory.
 */
int gdla_oracle_decode(const void *q_sig, int qs_dt, const void *q_noise,
                       int qn_dt, const void *qr_sig, int qrs_dt,
                       const void *qr_noise, int qrn_dt, const void *c_kv,
                       int c_dt, const void *kr, int kr_dt, int dr,
                       const int64_t *cache_len, const void *rms_w, int w_dt,
                       double eps, const void *w_kvb, int wk_dt,
                       const void *lam, int lam_dt, const void *gate,
                       int gate_dt, int B, int64_t L_max, int d_latent,
                       int Hs, int Hn, int Hkv, int d, int64_t window,
                       double scale, double *out) {
  if (Hn <= 0 || Hkv <= 0 || Hs % Hn != 0 || Hn != Hkv) return -1;
  if (dr < 0 || (dr > 0 && (!qr_sig || !qr_noise || !kr))) return -1;
  for (int b = 0; b < B; ++b) {
    const int64_t Lb = cache_len[b];
    if (Lb < 1 || Lb > L_max) return -1;
    /* only the cached tokens the query's mask keeps are normalised and
     * expanded: [first, Lb) with first = Lb - window under a window */
    const int64_t first = (window > 0 && Lb > window) ? Lb - window : 0;
    const int64_t L = Lb - first;
    double *chat = (double *)malloc(sizeof(double) * (size_t)(L * d_latent));
    double *k = (double *)malloc(sizeof(double) * (size_t)(L * Hkv * d));
    double *v = (double *)malloc(sizeof(double) * (size_t)(L * Hkv * d));
    if (!chat || !k || !v) {
      free(chat);
      free(k);
      free(v);
      return -2;
    }
    /* the kept cache rows of sequence b */
    const int64_t c_off = ((int64_t)b * L_max + first) * d_latent;
    const void *cb;
    if (c_dt == ORACLE_F64) cb = (const double *)c_kv + c_off;
    else if (c_dt == ORACLE_F32) cb = (const float *)c_kv + c_off;
    else cb = (const uint16_t *)c_kv + c_off;
    gdla_oracle_rmsnorm(cb, c_dt, rms_w, w_dt, eps, L, d_latent, chat);
    gdla_oracle_kv_expand(chat, w_kvb, wk_dt, L, d_latent, Hkv, d, d, k, v);
    /* the query token's inputs, addressed as the one evaluated row; it is
     * the last of the L kept tokens */
    const int64_t row = L - 1;
    const void *qs_b, *qn_b, *lam_b, *gate_b;
#define ORACLE_AT(ptr, dt, off) \
    ((dt) == ORACLE_F64 ? (const void *)((const double *)(ptr) + (off)) : \
     (dt) == ORACLE_F32 ? (const void *)((const float *)(ptr) + (off)) : \
                          (const void *)((const uint16_t *)(ptr) + (off)))
    qs_b = ORACLE_AT(q_sig, qs_dt, (int64_t)b * Hs * d);
    qn_b = ORACLE_AT(q_noise, qn_dt, (int64_t)b * Hn * d);
    lam_b = ORACLE_AT(lam, lam_dt, (int64_t)b * Hs);
    gate_b = ORACLE_AT(gate, gate_dt, (int64_t)b * Hs * d);
    /* rotary queries of the query token, rotary keys of the kept tokens */
    const void *qrs_b = NULL, *qrn_b = NULL, *kr_b = NULL;
    if (dr > 0) {
      qrs_b = ORACLE_AT(qr_sig, qrs_dt, (int64_t)b * Hs * dr);
      qrn_b = ORACLE_AT(qr_noise, qrn_dt, (int64_t)b * Hn * dr);
      kr_b = ORACLE_AT(kr, kr_dt, ((int64_t)b * L_max + first) * dr);
    }
#undef ORACLE_AT
    const int rc = attn_impl(qs_b, qs_dt, qn_b, qn_dt, qrs_b, qrs_dt, qrn_b, qrn_dt,
                             k, ORACLE_F64, kr_b, kr_dt, dr, v, ORACLE_F64, lam_b,
                             lam_dt, gate_b, gate_dt, 1, L, Hs, Hn, Hkv, d, window,
                             1, scale, &row, 1, out + (int64_t)b * Hs * d);
    free(chat);
    free(k);
    free(v);
    if (rc != 0) return rc;
  }
  return 0;
}

/*
 * Backward of the GDLA attention forward ([R] step 2; the model is trained
 * with GDLA, "Вышла новая модель Motif 3", pikabu.ru).  The pages give the
 * forward only; this is its gradient by the chain rule, written out in the
 * forward's order, for the loss sum(dO (.) O) with dO given.  For each token:
 *   dG[h]      = dO[h] (.) D[h],            D[h] = H_S[h] - lambda[h] H_N[h/g]
 *   dD[h]      = dO[h] (.) G[h]
 *   dlambda[h] = - sum_c dD[h][c] H_N[h/g][c]
 *   dH_S[h]    = dD[h]
 *   dH_N[n]    = - sum_{h : h/g = n} lambda[h] dD[h]
 * and for every head x of either path (output H_x, upstream gradient dH_x),
 * with s_ij = scale q_i . k_j and p_ij = softmax_j(s_ij) over J(i):
 *   dp_ij      = dH_x[i] . V[j]
 *   ds_ij      = p_ij (dp_ij - sum_{j' in J(i)} p_ij' dp_ij')   (softmax Jacobian)
 *   dQ_x[i]    = scale sum_j ds_ij K[j]
 *   dK[j]     += scale sum_i ds_ij Q_x[i]   (every head reading KV head kv(x))
 *   dV[j]     += sum_i p_ij dH_x[i]
 * Inputs as gdla_oracle_attn (full tensors, every row); d_out [B,T,Hs*d].
 * Outputs (float64): dq_sig [B,T,Hs,d], dq_noise [B,T,Hn,d], dk, dv
 * [B,T,Hkv,d], dlam [B,T,Hs], dgate [B,T,Hs*d].  Returns 0, -1 for bad head
 * counts, -2 when out of memory.
 */
int gdla_oracle_attn_bwd(const void *q_sig, int qs_dt, const void *q_noise,
                         int qn_dt, const void *k, int k_dt, const void *v,
                         int v_dt, const void *lam, int lam_dt,
                         const void *gate, int gate_dt, const void *d_out,
                         int do_dt, int B, int64_t T, int Hs, int Hn, int Hkv,
                         int d, int64_t window, int causal, double scale,
                         double *dq_sig, double *dq_noise, double *dk,
                         double *dv, double *dlam, double *dgate) {
  if (Hn <= 0 || Hkv <= 0 || Hs % Hn != 0 || Hn != Hkv) return -1;
  const int g = Hs / Hn;
  const int64_t N = (int64_t)B * T;
  double *hs = (double *)malloc(sizeof(double) * (size_t)(N * Hs * d));
  double *hn = (double *)malloc(sizeof(double) * (size_t)(N * Hn * d));
  double *dhs = (double *)malloc(sizeof(double) * (size_t)(N * Hs * d));
  double *dhn = (double *)malloc(sizeof(double) * (size_t)(N * Hn * d));
  if (!hs || !hn || !dhs || !dhn) {
    free(hs);
    free(hn);
    free(dhs);
    free(dhn);
    return -2;
  }
  /* the forward's two attention paths, every row */
  attention_path_impl(q_sig, qs_dt, 0, NULL, ORACLE_F64, k, k_dt, NULL,
                      ORACLE_F64, 0, v, v_dt, T, Hs, Hkv, d, window, causal,
                      scale, NULL, N, hs);
  attention_path_impl(q_noise, qn_dt, 0, NULL, ORACLE_F64, k, k_dt, NULL,
                      ORACLE_F64, 0, v, v_dt, T, Hn, Hkv, d, window, causal,
                      scale, NULL, N, hn);
  /* the gate and the differential, token by token */
  int64_t row;
#pragma omp parallel for schedule(static)
  for (row = 0; row < N; ++row) {
    for (int n = 0; n < Hn; ++n)
      for (int c = 0; c < d; ++c) dhn[(row * Hn + n) * d + c] = 0.0;
    for (int h = 0; h < Hs; ++h) {
      const double l = load_elem(lam, lam_dt, row * Hs + h);
      const int n = h / g;
      double dl = 0.0;
      for (int c = 0; c < d; ++c) {
        const int64_t oc = row * (int64_t)Hs * d + (int64_t)h * d + c;
        const double hnv = hn[(row * Hn + n) * d + c];
        const double dd = hs[(row * Hs + h) * d + c] - l * hnv;
        const double go = load_elem(d_out, do_dt, oc);
        dgate[oc] = go * dd;
        const double ddd = go * load_elem(gate, gate_dt, oc);
        dhs[(row * Hs + h) * d + c] = ddd;
        dl -= ddd * hnv;
        dhn[(row * Hn + n) * d + c] -= l * ddd;
      }
      dlam[row * Hs + h] = dl;
    }
  }
  for (int64_t i = 0; i < N * Hkv * d; ++i) {
    dk[i] = 0.0;
    dv[i] = 0.0;
  }
  /* the attention backward of every head; one task per (batch, KV group)
   * so that the group's dK and dV are accumulated by one thread */
  int64_t task;
#pragma omp parallel
  {
    double *p = (double *)malloc(sizeof(double) * (size_t)(T > 0 ? T : 1));
    double *dp = (double *)malloc(sizeof(double) * (size_t)(T > 0 ? T : 1));
#pragma omp for schedule(dynamic, 1)
    for (task = 0; task < (int64_t)B * Hkv; ++task) {
      const int64_t b = task / Hkv;
      const int kvh = (int)(task % Hkv);
      for (int x = 0; x <= g; ++x) {
        /* x < g: signal head g*kvh + x; x == g: noise head kvh */
        const int noise = x == g;
        const int H = noise ? Hn : Hs;
        const int hh = noise ? kvh : g * kvh + x;
        const void *q = noise ? q_noise : q_sig;
        const int q_dt = noise ? qn_dt : qs_dt;
        const double *dh = noise ? dhn : dhs;
        double *dq = noise ? dq_noise : dq_sig;
        for (int64_t i = 0; i < T; ++i) {
          const int64_t r = b * T + i;
          const int64_t qoff = (r * H + hh) * d;
          int64_t lo, hi;
          key_range(i, T, window, causal, &lo, &hi);
          double m = -INFINITY;
          for (int64_t j = lo; j <= hi; ++j) {
            const int64_t koff = ((b * T + j) * Hkv + kvh) * d;
            double dot = 0.0;
            for (int c = 0; c < d; ++c)
              dot += load_elem(q, q_dt, qoff + c) * load_elem(k, k_dt, koff + c);
            p[j - lo] = scale * dot;
            if (p[j - lo] > m) m = p[j - lo];
          }
          double denom = 0.0;
          for (int64_t j = lo; j <= hi; ++j) {
            p[j - lo] = exp(p[j - lo] - m);
            denom += p[j - lo];
          }
          double delta = 0.0;
          for (int64_t j = lo; j <= hi; ++j) {
            const int64_t voff = ((b * T + j) * Hkv + kvh) * d;
            p[j - lo] /= denom;
            double dot = 0.0;
            for (int c = 0; c < d; ++c) dot += dh[qoff + c] * load_elem(v, v_dt, voff + c);
            dp[j - lo] = dot;
            delta += p[j - lo] * dot;
          }
          for (int c = 0; c < d; ++c) dq[qoff + c] = 0.0;
          for (int64_t j = lo; j <= hi; ++j) {
            const int64_t koff = ((b * T + j) * Hkv + kvh) * d;
            const double ds = p[j - lo] * (dp[j - lo] - delta);
            for (int c = 0; c < d; ++c) {
              dq[qoff + c] += scale * ds * load_elem(k, k_dt, koff + c);
              dk[koff + c] += scale * ds * load_elem(q, q_dt, qoff + c);
              dv[koff + c] += p[j - lo] * dh[qoff + c];
            }
          }
        }
      }
    }
    free(p);
    free(dp);
  }
  free(hs);
  free(hn);
  free(dhs);
  free(dhn);
  return 0;
}
