/*
 * CPU oracle for ETA block-sparse decode — TEST INFRASTRUCTURE ONLY.
 *
 * Only the tests, the smoke check and the benchmark's CPU-baseline leg may
 * load this library. The product path (the CUDA library) never calls it and
 * shares no code, header or table with it.
 *
 * Source: "Elastic Threshold Attention: Learned Contextual Sparsity for
 * Long-Context Decoding" (Haris, Li, Karimzadehgan), as summarised on the
 * picx.dev page (Methodology §1 "Threshold Prediction", Eq. 1; §2
 * "Differentiable Masking and Tail Suppression", Eq. 2-3; §4 "Inference-Time
 * Block Pruning", Eq. 5) and the thelatestinai.com page (Figure 1, Figure 6).
 *
 * Precision. The block metadata, the block scores and the threshold decide
 * which blocks are admitted, an integer outcome. They are computed in fp32
 * with one fixed, stated order of operations (explicit fmaf, IEEE sqrtf and
 * division, no contraction: build with -ffp-contract=off), so the CUDA path
 * can take the same decisions bit for bit. The attention itself (Eq. 2-3
 * over the admitted keys) is computed in double.
 *
 * Storage dtypes: 0 = fp32, 1 = bf16 (upper 16 bits of an fp32).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define OR_F32 0
#define OR_BF16 1
#define OR_FP8 2   /* e4m3, "fn" variant: bias 7, no infinities, S.1111.111 = NaN */

/* e4m3 byte -> value, from the format's definition: (-1)^s 2^(e-7) (1 + m/8)
 * for e > 0, (-1)^s 2^-6 (m/8) for e = 0. */
static float e4m3(uint8_t b) {
  const int s = b >> 7, e = (b >> 3) & 15, m = b & 7;
  if (e == 15 && m == 7) return NAN;
  const double v = e == 0 ? ldexp((double)m / 8.0, -6) : ldexp(1.0 + (double)m / 8.0, e - 7);
  return (float)(s ? -v : v);
}

static float elem(const void* base, int dtype, int64_t i) {
  if (dtype == OR_F32) return ((const float*)base)[i];
  if (dtype == OR_FP8) return e4m3(((const uint8_t*)base)[i]);
  uint32_t bits = (uint32_t)((const uint16_t*)base)[i] << 16;
  float f;
  memcpy(&f, &bits, 4);
  return f;
}

/* Widen n stored values to fp32 (exact for both dtypes). */
void oracle_to_f32(int dtype, const void* src, int64_t n, float* dst) {
  for (int64_t i = 0; i < n; ++i) dst[i] = elem(src, dtype, i);
}

/*
 * Block metadata — Methodology §4, "Dual Probabilistic-Geometric Block Index":
 * population centroid mu_B, coordinate-wise (population) variance sigma^2_B
 * and maximum key norm M_B of one block of `rows` keys.
 *   k    : the block's first key; keys are `d` apart
 *   mu   : [d]  mu_i = (sum_r k_ri) / rows, sum taken in increasing r
 *   var  : [d]  var_i = (sum_r e*e) / rows, e = k_ri - mu_i, accumulated by fmaf
 *   maxn : M_B = sqrt(max_r N_r), N_r = sum_i k_ri^2 accumulated by fmaf in increasing i
 */
void oracle_block_meta(int dtype, const void* k, int64_t first, int rows, int d,
                       float* mu, float* var, float* maxn) {
  for (int i = 0; i < d; ++i) {
    float t = 0.0f;
    for (int r = 0; r < rows; ++r) t = t + elem(k, dtype, first + (int64_t)r * d + i);
    mu[i] = t / (float)rows;
  }
  for (int i = 0; i < d; ++i) {
    float v = 0.0f;
    for (int r = 0; r < rows; ++r) {
      float e = elem(k, dtype, first + (int64_t)r * d + i) - mu[i];
      v = fmaf(e, e, v);
    }
    var[i] = v / (float)rows;
  }
  float best = 0.0f;
  for (int r = 0; r < rows; ++r) {
    float nr = 0.0f;
    for (int i = 0; i < d; ++i) {
      float x = elem(k, dtype, first + (int64_t)r * d + i);
      nr = fmaf(x, x, nr);
    }
    if (nr > best) best = nr;
  }
  *maxn = sqrtf(best);
}

/*
 * Metadata of full blocks [0, nblk) of one (batch, kv head) cache slice.
 *   k   : slice [cap][d] in `dtype`
 *   mu, var : [nblk][d];  maxn : [nblk]
 */
void oracle_slice_meta(int dtype, const void* k, int d, int bs, int64_t nblk,
                       float* mu, float* var, float* maxn) {
  for (int64_t j = 0; j < nblk; ++j)
    oracle_block_meta(dtype, k, j * bs * (int64_t)d, bs, d, mu + j * d, var + j * d, maxn + j);
}

/*
 * Threshold predictor — Methodology §1, Eq. 1: tau_h = qbar . W[:,h] + b_h,
 * qbar the concatenation of the H query heads (length H*d), W in R^{Hd x H}
 * (row-major, W[j][h] at j*H + h), b in R^H.
 * Summation order: 32 running partials, partial l folding the terms j with
 * j mod 32 == l in increasing j by fmaf; then pairwise sums of partials l and
 * l^o for o = 16, 8, 4, 2, 1 (after the last step all partials are equal);
 * finally tau_h = partial_0 + b_h.
 */
void oracle_predict_tau(const float* qbar, int Hd, int H, const float* W, const float* bias,
                        float* tau) {
  for (int h = 0; h < H; ++h) {
    float p[32], t[32];
    for (int l = 0; l < 32; ++l) p[l] = 0.0f;
    for (int j = 0; j < Hd; ++j) p[j % 32] = fmaf(qbar[j], W[(int64_t)j * H + h], p[j % 32]);
    for (int o = 16; o >= 1; o >>= 1) {
      for (int l = 0; l < 32; ++l) t[l] = p[l] + p[l ^ o];
      for (int l = 0; l < 32; ++l) p[l] = t[l];
    }
    tau[h] = p[0] + bias[h];
  }
}

/*
 * Dual screening score — Methodology §4, Eq. 5:
 *   Score = s * min(<q,mu_B> + z * sigma_S, ||q||_2 * M_B),
 *   sigma_S = sqrt(sum_i q_i^2 sigma^2_B,i),  s = 1/sqrt(d_h) rounded to fp32.
 * Order: for i = 0..d-1: D = fmaf(q_i, mu_i, D); V = fmaf(q_i*q_i, var_i, V);
 * Q = fmaf(q_i, q_i, Q). Then A = D + z*sqrt(V), C = sqrt(Q)*M_B, min, times s.
 */
float oracle_block_score(const float* q, int d, const float* mu, const float* var, float maxn,
                         float z, float s) {
  float D = 0.0f, V = 0.0f, Q = 0.0f;
  for (int i = 0; i < d; ++i) {
    float qq = q[i] * q[i];
    D = fmaf(q[i], mu[i], D);
    V = fmaf(qq, var[i], V);
    Q = fmaf(q[i], q[i], Q);
  }
  float A = D + z * sqrtf(V);
  float C = sqrtf(Q) * maxn;
  float m = (A < C) ? A : C;
  return m * s;
}

/* s = 1/sqrt(d) computed in double, rounded to fp32 */
float oracle_inv_sqrt_d(int d) { return (float)(1.0 / sqrt((double)d)); }

/*
 * Screen one query head — Methodology §4: a block is bypassed when its score
 * is below the adjusted threshold tau~ = tau - a, and admitted otherwise
 * (a tie is admitted). The last n_local blocks (the one holding the current
 * token among them) are admitted without screening.
 *   mu, var : [>=ns][d], maxn : [>=ns] metadata of the slice's full blocks
 *   list    : [nb] out, ascending admitted block indices; returns the count
 *   scores  : [ns] out (may be NULL), the score of each screened block
 */
int oracle_screen_head(const float* q, int d, const float* mu, const float* var,
                       const float* maxn, int64_t nb, int n_local, float z,
                       float tau, float offset_a, int32_t* list, float* scores) {
  const float s = oracle_inv_sqrt_d(d);
  const float tau_t = tau - offset_a;
  int64_t ns = nb - n_local;
  if (ns < 0) ns = 0;
  int cnt = 0;
  for (int64_t j = 0; j < ns; ++j) {
    float sc = oracle_block_score(q, d, mu + j * d, var + j * d, maxn[j], z, s);
    if (scores) scores[j] = sc;
    if (!(sc < tau_t)) list[cnt++] = (int32_t)j;
  }
  for (int64_t j = ns; j < nb; ++j) list[cnt++] = (int32_t)j;
  return cnt;
}

/*
 * Sub-block envelope (a labelled reading): the pages name a "sub-block
 * envelope" as the remedy for variance dilution under flat block variance
 * (Table 16 caption; Table 12's 1.45B header, b = 64) without defining it.
 * Reading taken here: each block of b tokens is split into r = b / b_s
 * sub-blocks of b_s consecutive tokens, each with its own metadata (mean,
 * population variance, largest key norm, as for a block of b_s tokens); the
 * block's score is the largest of its r sub-block scores (Eq. 5 on each
 * sub-block), i.e. the upper envelope, and the admission rule is unchanged.
 * r = 1 is Eq. 5 as printed.
 *   mu, var : [>= ns*r][d], maxn : [>= ns*r] sub-block metadata
 *   list    : [nb] out, ascending admitted block indices; returns the count
 *   scores  : [ns] out (may be NULL), the envelope score of each screened block
 */
int oracle_screen_head_env(const float* q, int d, const float* mu, const float* var,
                           const float* maxn, int64_t nb, int r, int n_local, float z,
                           float tau, float offset_a, int32_t* list, float* scores) {
  const float s = oracle_inv_sqrt_d(d);
  const float tau_t = tau - offset_a;
  int64_t ns = nb - n_local;
  if (ns < 0) ns = 0;
  int cnt = 0;
  for (int64_t j = 0; j < ns; ++j) {
    float env = -INFINITY;
    for (int u = 0; u < r; ++u) {
      const int64_t sb = j * r + u;
      const float sc = oracle_block_score(q, d, mu + sb * d, var + sb * d, maxn[sb], z, s);
      if (sc > env) env = sc;
    }
    if (scores) scores[j] = env;
    if (!(env < tau_t)) list[cnt++] = (int32_t)j;
  }
  for (int64_t j = ns; j < nb; ++j) list[cnt++] = (int32_t)j;
  return cnt;
}

static double sigmoid(double x) { return 1.0 / (1.0 + exp(-x)); }

/*
 * Gated attention of one query head over its admitted blocks (double) —
 * Methodology §2, Eq. 2-3, restricted to the loaded blocks (Figure 6):
 *   S_s = <q, k_s> / sqrt(d)
 *   g_s = S_s                                  if s = t (the current token, t = n-1)
 *   g_s = S_s * sigma(beta * (S_s - tau))      otherwise (gate 0: the multiplicative
 *                                              gate, the pages' "normal mode")
 *   g_s = S_s if S_s >= tau, else -infinity    otherwise (gate 1: "strict mode", hard
 *                                              additive masking, Tables 6-7)
 *   o   = sum_s exp(g_s - max g) v_s / sum_s exp(g_s - max g)
 * over every token s < n of every listed block.
 *   k, v : slice [cap][d] in kv_dtype;  q : [d] fp32 values;  out : [d]
 */
void oracle_attend_head(int kv_dtype, const void* k, const void* v, int d, int bs, int64_t n,
                        const float* q, const int32_t* list, int cnt, float tau, float beta, int gate,
                        double* out) {
  const double inv = 1.0 / sqrt((double)d);
  const int64_t t = n - 1;
  int64_t m = 0;
  double* g = (double*)malloc(sizeof(double) * (size_t)(cnt > 0 ? cnt : 1) * (size_t)bs);
  int64_t* pos = (int64_t*)malloc(sizeof(int64_t) * (size_t)(cnt > 0 ? cnt : 1) * (size_t)bs);
  double gmax = -INFINITY;
  for (int c = 0; c < cnt; ++c) {
    for (int r = 0; r < bs; ++r) {
      int64_t s = (int64_t)list[c] * bs + r;
      if (s >= n) break;
      double S = 0.0;
      for (int i = 0; i < d; ++i) S += (double)q[i] * (double)elem(k, kv_dtype, s * d + i);
      S *= inv;
      double gs;
      if (s == t) gs = S;                                   /* Eq. 3: the current token is exempt */
      else if (gate == 0) gs = S * sigmoid((double)beta * (S - (double)tau));   /* Eq. 2 */
      else gs = (S >= (double)tau) ? S : -INFINITY;         /* strict mode: hard mask */
      g[m] = gs;
      pos[m] = s;
      if (gs > gmax) gmax = gs;
      ++m;
    }
  }
  double den = 0.0;
  for (int i = 0; i < d; ++i) out[i] = 0.0;
  for (int64_t j = 0; j < m; ++j) {
    double w = exp(g[j] - gmax);
    den += w;
    for (int i = 0; i < d; ++i) out[i] += w * (double)elem(v, kv_dtype, pos[j] * d + i);
  }
  for (int i = 0; i < d; ++i) out[i] /= den;
  free(g);
  free(pos);
}

/*
 * Block statistics for the screen diagnostics of Table 16 (false negatives,
 * false positives, token recall, missed mass), for one query head over the
 * blocks [0, nb) of its cache slice, n tokens (t = n - 1 the current token):
 *   S_s       = fl(fl(sum_i q_i k_si) * s), the sum by fused multiply-adds in
 *               increasing i and s = fl(1/sqrt(d)) (fp32, so the comparisons
 *               with the threshold below are reproducible bit for bit)
 *   bmax[j]   = max over the block's tokens of S_s
 *   above[j]  = number of the block's tokens with S_s >= tau_screen
 *   blse[j]   = log sum over the block's tokens of exp(g_s), g_s the gated
 *               logit of Eq. 2-3 (gate 0) or of strict mode (gate 1) with
 *               threshold tau, the current token exempt (double)
 * "Missed mass" of Table 16 is then sum over rejected j of exp(blse[j] - LSE)
 * with LSE the log-sum-exp over all blocks: the fraction of the dense gated
 * softmax mass that the screen dropped.
 */
void oracle_block_stats(int kv_dtype, const void* k, int d, int bs, int64_t n, int nb, const float* q,
                        float tau_screen, float tau, float beta, int gate, float* bmax, int32_t* above,
                        double* blse) {
  const float s = (float)(1.0 / sqrt((double)d));
  const int64_t t = n - 1;
  for (int j = 0; j < nb; ++j) {
    float mx = -INFINITY;
    int cnt = 0;
    double m = -INFINITY;
    double gs_buf[1024];
    int m_rows = 0;
    for (int r = 0; r < bs; ++r) {
      const int64_t tok = (int64_t)j * bs + r;
      if (tok >= n) break;
      float acc = 0.0f;
      for (int i = 0; i < d; ++i) acc = fmaf(q[i], elem(k, kv_dtype, tok * d + i), acc);
      const float S = acc * s;
      if (S > mx) mx = S;
      if (S >= tau_screen) ++cnt;
      const double Sd = (double)S;
      double g;
      if (tok == t) g = Sd;
      else if (gate == 0) g = Sd * sigmoid((double)beta * (Sd - (double)tau));
      else g = (Sd >= (double)tau) ? Sd : -INFINITY;
      gs_buf[m_rows++] = g;
      if (g > m) m = g;
    }
    double z = 0.0;
    for (int r = 0; r < m_rows; ++r) z += exp(gs_buf[r] - m);
    bmax[j] = mx;
    above[j] = cnt;
    blse[j] = (m == -INFINITY) ? -INFINITY : m + log(z);
  }
}
