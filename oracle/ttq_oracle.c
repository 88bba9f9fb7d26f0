/*
 * ttq_oracle.c — plain, slow CPU definition of the TTQ hot path.
 *
 * TEST INFRASTRUCTURE ONLY. Only the tests, the smoke check and the CPU
 * baseline leg of the benchmark load this file. It shares no code, header,
 * table or constant with the CUDA library; it does not include ttq.h.
 *
 * Source: "TTQ: Activation-Aware Test-Time Quantization to Accelerate LLM
 * Inference On The Fly" as summarised by the nubint.ai review ("TTQ
 * review"), section "Proposed method" (제안 방법), bullets 1-5. The pages
 * print no formula; where they are silent the readings are:
 *   (a) the channel statistic is the p-th absolute moment over the prompt's
 *       tokens, m_j = (1/T) sum_t |x_tj|^p (p = 2: diagonal of E[x x^T]);
 *   (b) shrinkage toward the mean of the diagonal:
 *       c_j = (1 - lambda) m_j + lambda mean_k(m_k);
 *   (c) the AWQ scale is the statistic's root raised to alpha:
 *       s_j = c_j^(alpha/p), with s_j = 1 when alpha == 0 or c_j <= 0;
 *   (d) RTN is asymmetric min-max over the range widened to contain 0:
 *       D = (mx - mn)/(2^b - 1), z = rint(-mn/D), q = rint(w/D) + z, each
 *       quotient an IEEE fp32 division and rint round-half-to-even;
 *   (e) the all-zero group has D = 1, z = 0.
 *   (f) two valid fp32 evaluations of w/D (a division, or a product with a
 *       rounded reciprocal) can round to different codes only where the
 *       quotient lies within one fp32 step of a half-integer; such
 *       "near-ties" are found and counted here, per weight and, for the
 *       zero point, per group (a zero-point near-tie can move every code of
 *       its group).
 *
 * Precision: statistics, scales, GEMM and loss in fp64; the quantizer in
 * fp32 with IEEE operations only (compile with -ffp-contract=off, never
 * with -ffast-math), because its integer outputs must be reproducible.
 *
 * Parity pins (tests/test_oracle_pins.py): closed forms for constant and
 * one-hot inputs, alpha = 0 gives s = 1, lambda = 0 with alpha = p gives
 * s = m, a brute-force argmin over the 2^b grid on tiny inputs, a
 * hand-worked quantization example (tests/golden), pack/unpack round trip,
 * the GEMM against a dense fp64 matmul of the dequantized weight, the loss
 * against its trace form, the low-rank reconstruction.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ---- Step 1: per-channel statistic (Proposed method, bullets 2-3) ---- */

/* sum_out[j] = sum_t |X[t][j]|^p in fp64 (the mean is sum / T). */
void oracle_act_sums(const float* X, int64_t T, int64_t K, int64_t ldx,
                     double p, double* sum_out) {
  for (int64_t j = 0; j < K; ++j) sum_out[j] = 0.0;
  for (int64_t t = 0; t < T; ++t) {
    const float* row = X + t * ldx;
    for (int64_t j = 0; j < K; ++j) {
      double a = fabs((double)row[j]);
      double v;
      if (p == 2.0)
        v = a * a;
      else if (p == 1.0)
        v = a;
      else
        v = pow(a, p);
      sum_out[j] += v;
    }
  }
}

/* ---- Step 2: AWQ scales from the shrunk diagonal (bullets 2-4) ---- */

void oracle_awq_scales(const double* sum, int64_t T_total, int64_t K,
                       double alpha, double lambda, double p, double* s,
                       double* inv_s) {
  double* m = (double*)malloc(sizeof(double) * (size_t)K);
  double mbar = 0.0;
  for (int64_t j = 0; j < K; ++j) {
    m[j] = sum[j] / (double)T_total;
    mbar += m[j];
  }
  mbar /= (double)K;
  for (int64_t j = 0; j < K; ++j) {
    double c = (1.0 - lambda) * m[j] + lambda * mbar;
    double sj;
    if (alpha == 0.0 || !(c > 0.0) || !isfinite(c))
      sj = 1.0;
    else
      sj = pow(c, alpha / p);
    s[j] = sj;
    inv_s[j] = 1.0 / sj;
  }
  free(m);
}

/* Step 2 with the mean of the shrinkage given: for a layer whose input
 * channels are split into shards, mbar is the mean over ALL channels while
 * m_j and the scales are this shard's (the same formulas as above). */
void oracle_awq_scales_given_mean(const double* sum, int64_t T_total,
                                  int64_t K, double mbar, double alpha,
                                  double lambda, double p, double* s,
                                  double* inv_s) {
  for (int64_t j = 0; j < K; ++j) {
    double m = sum[j] / (double)T_total;
    double c = (1.0 - lambda) * m + lambda * mbar;
    double sj;
    if (alpha == 0.0 || !(c > 0.0) || !isfinite(c))
      sj = 1.0;
    else
      sj = pow(c, alpha / p);
    s[j] = sj;
    inv_s[j] = 1.0 / sj;
  }
}

/* ---- Packing (storage format of the codes; ours, the pages fix none) ----
 * Block k of a row holds channels 32k..32k+31 in `bits` words; channel
 * 32k + c sits at bits [c*bits, c*bits + bits) of the block. */

static void put_code(uint32_t* row_words, int64_t j, int bits, uint32_t q) {
  int64_t block = j / 32;
  int c = (int)(j % 32);
  int bit = c * bits;
  uint32_t* w = row_words + block * bits;
  int word = bit / 32, shift = bit % 32;
  w[word] |= q << shift;
  if (shift + bits > 32) w[word + 1] |= q >> (32 - shift);
}

static uint32_t get_code(const uint32_t* row_words, int64_t j, int bits) {
  int64_t block = j / 32;
  int c = (int)(j % 32);
  int bit = c * bits;
  const uint32_t* w = row_words + block * bits;
  int word = bit / 32, shift = bit % 32;
  uint64_t v = (uint64_t)w[word] >> shift;
  if (shift + bits > 32) v |= (uint64_t)w[word + 1] << (32 - shift);
  return (uint32_t)(v & ((1u << bits) - 1u));
}

void oracle_pack_codes(const uint8_t* q, int64_t N, int64_t K, int bits,
                       uint32_t* codes) {
  int64_t words = K * bits / 32;
  memset(codes, 0, sizeof(uint32_t) * (size_t)(N * words));
  for (int64_t n = 0; n < N; ++n)
    for (int64_t j = 0; j < K; ++j)
      put_code(codes + n * words, j, bits, q[n * K + j]);
}

void oracle_unpack_codes(const uint32_t* codes, int64_t N, int64_t K,
                         int bits, uint8_t* q) {
  int64_t words = K * bits / 32;
  for (int64_t n = 0; n < N; ++n)
    for (int64_t j = 0; j < K; ++j)
      q[n * K + j] = (uint8_t)get_code(codes + n * words, j, bits);
}

/* ---- Step 3: group-wise RTN with QDQ (bullet 1), fp32 IEEE ---- */

static float clampf(float v, float lo, float hi) {
  return v < lo ? lo : (v > hi ? hi : v);
}

/* Quantizes one group of `g` scaled weights; writes the codes to q. */
static void rtn_group(const float* w, int g, int bits, uint8_t* q,
                      float* delta, uint8_t* zero) {
  const float qmax = (float)((1 << bits) - 1);
  float mn = 0.0f, mx = 0.0f; /* the range always contains 0 */
  for (int i = 0; i < g; ++i) {
    if (w[i] < mn) mn = w[i];
    if (w[i] > mx) mx = w[i];
  }
  float d = (mx - mn) / qmax;
  if (d == 0.0f) d = 1.0f;
  float z = clampf(rintf(-mn / d), 0.0f, qmax);
  for (int i = 0; i < g; ++i) {
    float v = rintf(w[i] / d) + z;
    q[i] = (uint8_t)clampf(v, 0.0f, qmax);
  }
  *delta = d;
  *zero = (uint8_t)z;
}

void oracle_quantize(const float* W, int64_t N, int64_t K, int64_t ldw,
                     const float* s, int bits, int group, uint32_t* codes,
                     float* delta, uint8_t* zero) {
  int64_t G = K / group;
  int64_t words = K * bits / 32;
  float* w = (float*)malloc(sizeof(float) * (size_t)group);
  uint8_t* q = (uint8_t*)malloc((size_t)K);
  for (int64_t n = 0; n < N; ++n) {
    for (int64_t gi = 0; gi < G; ++gi) {
      for (int i = 0; i < group; ++i) {
        int64_t j = gi * group + i;
        float sj = s ? s[j] : 1.0f;
        w[i] = W[n * ldw + j] * sj;
      }
      rtn_group(w, group, bits, q + gi * group, &delta[n * G + gi],
                &zero[n * G + gi]);
    }
    memset(codes + n * words, 0, sizeof(uint32_t) * (size_t)words);
    for (int64_t j = 0; j < K; ++j) put_code(codes + n * words, j, bits, q[j]);
  }
  free(q);
  free(w);
}

/* 1 when the fp32 value v is a half-integer k + 1/2 or one of the two fp32
 * neighbours of the half-integer nearest to it. */
static int near_half(float v) {
  float h = floorf(v) + 0.5f; /* the nearest half-integer (exact, |v| < 2^22) */
  return v == h || nextafterf(v, INFINITY) == h ||
         nextafterf(v, -INFINITY) == h;
}

/* Marks the near-ties of oracle_quantize's rounding, with the same
 * arithmetic. Bit 0 of mask[n*K + j] is set where the pre-round quotient
 * w_j/D lies within one fp32 step of a half-integer; bit 1 where the zero
 * point's quotient -mn/D of j's group does (every code of that group may
 * move with it). Returns the number of weight near-ties; *group_ties
 * receives the number of groups with a zero-point near-tie. mask may be
 * NULL. */
int64_t oracle_near_tie_mask(const float* W, int64_t N, int64_t K,
                             int64_t ldw, const float* s, int bits, int group,
                             uint8_t* mask, int64_t* group_ties) {
  int64_t G = K / group, weights = 0, groups = 0;
  const float qmax = (float)((1 << bits) - 1);
  float* w = (float*)malloc(sizeof(float) * (size_t)group);
  for (int64_t n = 0; n < N; ++n)
    for (int64_t gi = 0; gi < G; ++gi) {
      float mn = 0.0f, mx = 0.0f;
      for (int i = 0; i < group; ++i) {
        int64_t j = gi * group + i;
        w[i] = W[n * ldw + j] * (s ? s[j] : 1.0f);
        if (w[i] < mn) mn = w[i];
        if (w[i] > mx) mx = w[i];
      }
      float d = (mx - mn) / qmax;
      if (d == 0.0f) d = 1.0f;
      int zero_tie = near_half(-mn / d);
      groups += zero_tie;
      for (int i = 0; i < group; ++i) {
        int weight_tie = near_half(w[i] / d);
        weights += weight_tie;
        if (mask)
          mask[n * K + gi * group + i] =
              (uint8_t)(weight_tie | (zero_tie << 1));
      }
    }
  free(w);
  if (group_ties) *group_ties = groups;
  return weights;
}

/* Number of weight near-ties (see oracle_near_tie_mask). */
int64_t oracle_count_near_ties(const float* W, int64_t N, int64_t K,
                               int64_t ldw, const float* s, int bits,
                               int group) {
  return oracle_near_tie_mask(W, N, K, ldw, s, bits, group, NULL, NULL);
}

/* Scaled-domain dequantized weight What_s[n][j] = (q - z) * D in fp64. */
void oracle_dequantize(const uint32_t* codes, const float* delta,
                       const uint8_t* zero, int64_t N, int64_t K, int bits,
                       int group, double* What_s) {
  int64_t G = K / group, words = K * bits / 32;
  for (int64_t n = 0; n < N; ++n)
    for (int64_t j = 0; j < K; ++j) {
      double q = (double)get_code(codes + n * words, j, bits);
      double z = (double)zero[n * G + j / group];
      What_s[n * K + j] = (q - z) * (double)delta[n * G + j / group];
    }
}

/* ---- Step 4: the projection (bullets 1, 5, 7), fp64 ----
 * Y[i][n] = sum_j (x_tj * inv_s_j) (q_nj - z) D + sum_rho (x_t . A_rho) B_n,rho
 * for the token rows t = rows[i] (all T rows when rows == NULL). */
void oracle_lowbit_gemm(const float* X, int64_t T, int64_t K, int64_t ldx,
                        const int64_t* rows, int64_t n_rows,
                        const float* inv_s, const uint32_t* codes,
                        const float* delta, const uint8_t* zero, int64_t N,
                        int bits, int group, const float* A, const float* B,
                        int r, double* Y) {
  int64_t G = K / group, words = K * bits / 32;
  int64_t nr = rows ? n_rows : T;
  double* xs = (double*)malloc(sizeof(double) * (size_t)K);
  double* u = (double*)malloc(sizeof(double) * (size_t)(r > 0 ? r : 1));
  for (int64_t i = 0; i < nr; ++i) {
    int64_t t = rows ? rows[i] : i;
    const float* x = X + t * ldx;
    for (int64_t j = 0; j < K; ++j) xs[j] = (double)x[j] * (double)inv_s[j];
    for (int rho = 0; rho < r; ++rho) {
      double acc = 0.0;
      for (int64_t j = 0; j < K; ++j)
        acc += (double)x[j] * (double)A[(int64_t)rho * K + j];
      u[rho] = acc;
    }
    for (int64_t n = 0; n < N; ++n) {
      const uint32_t* cw = codes + n * words;
      double acc = 0.0;
      for (int64_t j = 0; j < K; ++j) {
        double q = (double)get_code(cw, j, bits);
        double z = (double)zero[n * G + j / group];
        acc += xs[j] * ((q - z) * (double)delta[n * G + j / group]);
      }
      for (int rho = 0; rho < r; ++rho)
        acc += u[rho] * (double)B[n * r + rho];
      Y[i * N + n] = acc;
    }
  }
  free(u);
  free(xs);
}

/* ---- Objective (bullet 3): L = (1/T) || (W - W_eff) X^T ||_F^2 ----
 * W_eff is the effective weight the caller passes ((q - z) D / s_j). */
double oracle_loss(const float* W, int64_t N, int64_t K,
                   const double* W_eff, const float* X, int64_t T) {
  double total = 0.0;
  double* e = (double*)malloc(sizeof(double) * (size_t)K);
  for (int64_t n = 0; n < N; ++n) {
    for (int64_t j = 0; j < K; ++j)
      e[j] = (double)W[n * K + j] - W_eff[n * K + j];
    for (int64_t t = 0; t < T; ++t) {
      double d = 0.0;
      for (int64_t j = 0; j < K; ++j) d += e[j] * (double)X[t * K + j];
      total += d * d;
    }
  }
  free(e);
  return total / (double)T;
}
