/*
 * BitNest nested W4/W8 linear layer: plain CPU oracle.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or
 * call this file: only the tests, the smoke check and the benchmark's CPU
 * baseline leg use it.  It shares no code, header, table or constant with
 * the CUDA library.
 *
 * Every routine is the plainest reading of the "BitNest-Llama-3-8B" model
 * card (the only page that fixes the arithmetic):
 *   - section "Files", planes.safetensors entry: the plane layout (uint8
 *     [N, K/2], unsigned nibbles u = q + 8, byte j holds column 2j in its low
 *     nibble and column 2j+1 in its high nibble), the fp16 group scales
 *     [N, K/128] and the two dequantisation formulas
 *         draft  W4 = (hi - 8) * scale
 *         target W8 = (16 * (hi - 8) + (lo - 8)) * scale / 16 ;
 *   - the model table, row "Activations": symmetric int8 per token, per
 *     128-column group for o_proj;
 *   - the model table, row "Weights": group size 128.
 * Where the card is silent the reading taken is stated at the routine.
 *
 * Floating point: IEEE binary32 for the activation quantiser (the decision
 * that produces an integer code is taken in fp32 on both sides), binary64
 * for the layer output.  Build without -ffast-math and with
 * -ffp-contract=off so that every operation is one correctly rounded IEEE
 * operation.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_GROUP 128
#define ORACLE_DRAFT 0
#define ORACLE_TARGET 1

int oracle_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

/* ---- fp16 (IEEE binary16) decoding, from the format's definition ------- */
/* 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits.  Every binary16
 * value is exactly representable in binary32 and binary64.              */
double oracle_half_to_double(uint16_t h) {
  int sign = (h >> 15) & 1;
  int e = (h >> 10) & 0x1f;
  int f = h & 0x3ff;
  double v;
  if (e == 0)
    v = ldexp((double)f, -24); /* zero or subnormal: f * 2^-24 */
  else if (e == 31)
    v = f ? NAN : INFINITY;
  else
    v = ldexp((double)(1024 + f), e - 25); /* (1 + f/1024) * 2^(e-15) */
  return sign ? -v : v;
}

float oracle_half_to_float(uint16_t h) { return (float)oracle_half_to_double(h); }

/* ---- fp16 encoding: binary32 -> binary16, round to nearest, ties to even --
 * From the format's definition: the value is f = (-1)^s * m * 2^e with m an
 * integer mantissa; binary16 keeps 11 significant bits for normal values
 * (exponent -14 .. 15) and a fixed quantum of 2^-24 below 2^-14.  Rounding
 * is done on the exact integer multiple of the target quantum, ties to even;
 * magnitudes that round to 2^16 or more become infinity.                */
uint16_t oracle_float_to_half(float f) {
  uint32_t bits;
  memcpy(&bits, &f, 4);
  uint16_t sign = (uint16_t)((bits >> 16) & 0x8000u);
  if (isnan(f)) return (uint16_t)(sign | 0x7e00u);
  double a = fabs((double)f);
  if (isinf(f) || a >= 65520.0) return (uint16_t)(sign | 0x7c00u); /* 65520 = 65504 + half a quantum */
  if (a == 0.0) return sign;
  int e2;
  frexp(a, &e2);           /* a = fr * 2^e2 with fr in [0.5, 1) */
  int exp = e2 - 1;        /* a in [2^exp, 2^(exp+1)) */
  if (exp < -14) exp = -14; /* subnormal range: quantum 2^-24 */
  double quantum = ldexp(1.0, exp - 10);
  double mult = a / quantum; /* exact: a is a binary32 value */
  double r = nearbyint(mult); /* default rounding mode: to nearest, ties to even */
  uint32_t m = (uint32_t)r;
  if (m == 2048) { /* rounded up to the next power of two */
    m = 1024;
    exp += 1;
  }
  if (m < 1024) return (uint16_t)(sign | m); /* subnormal (exp == -14) */
  if (exp > 15) return (uint16_t)(sign | 0x7c00u);
  return (uint16_t)(sign | ((uint32_t)(exp + 15) << 10) | (m - 1024));
}

/* ---- plane packing (model card, "Files": byte j = col 2j | col 2j+1 << 4) */
void oracle_pack_plane(const uint8_t *u, int64_t N, int64_t K, uint8_t *plane) {
  for (int64_t n = 0; n < N; ++n)
    for (int64_t j = 0; j < K / 2; ++j) {
      uint8_t low = u[n * K + 2 * j] & 0xf;
      uint8_t high = u[n * K + 2 * j + 1] & 0xf;
      plane[n * (K / 2) + j] = (uint8_t)(low | (high << 4));
    }
}

void oracle_unpack_plane(const uint8_t *plane, int64_t N, int64_t K, uint8_t *u) {
  for (int64_t n = 0; n < N; ++n)
    for (int64_t k = 0; k < K; ++k) {
      uint8_t byte = plane[n * (K / 2) + k / 2];
      u[n * K + k] = (k % 2 == 0) ? (byte & 0xf) : (byte >> 4);
    }
}

/* nibble of column k in row n of a plane */
static int nibble(const uint8_t *plane, int64_t K, int64_t n, int64_t k) {
  uint8_t byte = plane[n * (K / 2) + k / 2];
  return (k % 2 == 0) ? (byte & 0xf) : (byte >> 4);
}

/* Integer weight code of the model card's formulas, before the scale:
 *   draft  : hi - 8                      in [-8, 7]
 *   target : 16 * (hi - 8) + (lo - 8)    in [-136, 119]
 * (the target code does not fit int8; it is taken literally).           */
static int weight_code(int mode, const uint8_t *hi, const uint8_t *lo, int64_t K,
                       int64_t n, int64_t k) {
  int h = nibble(hi, K, n, k);
  if (mode == ORACLE_DRAFT) return h - 8;
  int l = nibble(lo, K, n, k);
  return 16 * (h - 8) + (l - 8);
}

/* ---- dequantised weights (model card, "Files", the two formulas) ------- */
void oracle_dequant(int mode, const uint8_t *hi, const uint8_t *lo, const uint16_t *scale,
                    int64_t N, int64_t K, double *W) {
  int64_t G = K / ORACLE_GROUP;
  for (int64_t n = 0; n < N; ++n)
    for (int64_t k = 0; k < K; ++k) {
      double s = oracle_half_to_double(scale[n * G + k / ORACLE_GROUP]);
      int h = nibble(hi, K, n, k);
      if (mode == ORACLE_DRAFT) {
        W[n * K + k] = (double)(h - 8) * s;
      } else {
        int l = nibble(lo, K, n, k);
        W[n * K + k] = (double)(16 * (h - 8) + (l - 8)) * s / 16.0;
      }
    }
}

/* ---- packer from fp weights ----------------------------------------------
 * Model card, opening paragraph: the high nibble is a 4-bit model fitted
 * first, the low nibble the closed-form residual back to 8 bits; section
 * "Files": u = q + 8, one fp16 scale per row and 128-column group, draft
 * W4 = (hi - 8) * scale, target W8 = (16 (hi - 8) + (lo - 8)) * scale / 16.
 * Readings (the card is silent on them; its GPTQ fit of the high nibble is
 * not reproduced):
 *   scale   s = fp16(max|W| / 7)   (the fp32 quotient rounded to fp16);
 *   high    q4 = rne(t), t = W / s (one correctly rounded fp32 division);
 *           |t| <= 7 (1 + 2^-10) keeps q4 in [-7, 7]: symmetric, no clamp;
 *   low     ql = clamp(rne(16 (t - q4)), -8, 7)   (t - q4 is exact);
 *   an all-zero group gets s = 0 and q4 = ql = 0.
 * Outputs the unpacked nibbles uh = q4 + 8, ul = ql + 8 [N, K] and the fp16
 * scale bits [N, K/128].                                                */
void oracle_pack_weights(const uint16_t *w, int64_t N, int64_t K, uint8_t *uh, uint8_t *ul,
                         uint16_t *scale) {
  int64_t G = K / ORACLE_GROUP;
  for (int64_t n = 0; n < N; ++n)
    for (int64_t g = 0; g < G; ++g) {
      const uint16_t *wr = w + n * K + g * ORACLE_GROUP;
      float amax = 0.0f;
      for (int64_t k = 0; k < ORACLE_GROUP; ++k) {
        float a = fabsf(oracle_half_to_float(wr[k]));
        if (a > amax) amax = a;
      }
      uint16_t sbits = oracle_float_to_half(amax / 7.0f);
      float s = oracle_half_to_float(sbits);
      scale[n * G + g] = sbits;
      for (int64_t k = 0; k < ORACLE_GROUP; ++k) {
        int q4 = 0, ql = 0;
        if (s != 0.0f) {
          float t = oracle_half_to_float(wr[k]) / s;
          float r4 = nearbyintf(t);
          q4 = (int)r4;
          float rl = nearbyintf(16.0f * (t - r4));
          if (rl > 7.0f) rl = 7.0f;
          if (rl < -8.0f) rl = -8.0f;
          ql = (int)rl;
        }
        uh[n * K + g * ORACLE_GROUP + k] = (uint8_t)(q4 + 8);
        ul[n * K + g * ORACLE_GROUP + k] = (uint8_t)(ql + 8);
      }
    }
}

/* ---- nested KV cache: decode attention -----------------------------------
 * Model card, model table row "KV cache": nested at runtime, the draft reads
 * KV4, the target KV8.  The card gives no layout; the reading taken is the
 * weights' nesting applied to the cache: every K (and V) row of one token and
 * one KV head (head_dim = 128 values, one group) is packed at runtime with
 * oracle_pack_weights' rule (fp16 scale max|x| / 7, round-to-nearest high
 * nibble, closed-form residual low nibble); the draft dequantises
 * (hi - 8) s, the target (16 (hi - 8) + (lo - 8)) s / 16.
 * Decode attention of one new token, in fp64 from the definition:
 *   head h (of H) reads KV head h / (H / Hkv)  (grouped-query attention);
 *   score[t] = q_h . K[t] / sqrt(D), p = softmax(score) over t < T,
 *   out_h = sum_t p[t] V[t].
 * q: fp16 [H, D]; planes: uint8 [T * Hkv, D / 2] (row t * Hkv + j);
 * scales: fp16 [T * Hkv, D / 128]; out: fp64 [H, D].                    */
static double kv_value(int mode, const uint8_t *hi, const uint8_t *lo, const uint16_t *scale,
                       int64_t D, int64_t row, int64_t k) {
  double s = oracle_half_to_double(scale[row * (D / ORACLE_GROUP) + k / ORACLE_GROUP]);
  int h = nibble(hi, D, row, k);
  if (mode == ORACLE_DRAFT) return (double)(h - 8) * s;
  int l = nibble(lo, D, row, k);
  return (double)(16 * (h - 8) + (l - 8)) * s / 16.0;
}

void oracle_nested_attention(int mode, const uint16_t *q, int64_t H, int64_t Hkv, int64_t D,
                             int64_t T, const uint8_t *k_hi, const uint8_t *k_lo,
                             const uint16_t *k_scale, const uint8_t *v_hi,
                             const uint8_t *v_lo, const uint16_t *v_scale, double *out) {
  double *score = (double *)malloc(sizeof(double) * (size_t)(T > 0 ? T : 1));
  for (int64_t h = 0; h < H; ++h) {
    int64_t j = h / (H / Hkv);
    double mx = -INFINITY;
    for (int64_t t = 0; t < T; ++t) {
      double acc = 0.0;
      for (int64_t k = 0; k < D; ++k)
        acc += oracle_half_to_double(q[h * D + k]) *
               kv_value(mode, k_hi, k_lo, k_scale, D, t * Hkv + j, k);
      score[t] = acc / sqrt((double)D);
      if (score[t] > mx) mx = score[t];
    }
    double den = 0.0;
    for (int64_t t = 0; t < T; ++t) {
      score[t] = exp(score[t] - mx); /* shifted by the maximum: same softmax */
      den += score[t];
    }
    for (int64_t k = 0; k < D; ++k) {
      double acc = 0.0;
      for (int64_t t = 0; t < T; ++t)
        acc += score[t] * kv_value(mode, v_hi, v_lo, v_scale, D, t * Hkv + j, k);
      out[h * D + k] = acc / den;
    }
  }
  free(score);
}

/* ---- online Hadamard rotation of the down_proj input ---------------------
 * Model card, model table row "Rotation": an online Hadamard (R4) on the
 * down_proj inputs; the card ships the matrices, not their construction.
 * Reading: x_rot = x H / sqrt(K) with H a Hadamard matrix of order K:
 *   K = 2^b       : Sylvester's matrix, H[i][j] = (-1)^popcount(i & j);
 *   K = 28 * 2^b  : H = H28 (x) H_{2^b} (Kronecker product, the order-28
 *                   factor outer: index i = i28 * 2^b + i'), H28 = I + S from
 *                   Paley's construction I over GF(27): S = [[0, 1^T],
 *                   [-1, Q]], Q[a][b] = chi(a - b), chi the quadratic
 *                   character of GF(27) = GF(3)[x] / (x^3 - x - 1).
 * Computed from the definition, one output at a time in fp64.          */
static int gf27_add(int a, int b) {
  int r = 0, p = 1;
  for (int d = 0; d < 3; ++d, a /= 3, b /= 3, p *= 3) r += ((a % 3 + b % 3) % 3) * p;
  return r;
}
static int gf27_neg(int a) {
  int r = 0, p = 1;
  for (int d = 0; d < 3; ++d, a /= 3, p *= 3) r += ((3 - a % 3) % 3) * p;
  return r;
}
static int gf27_mul(int a, int b) {
  /* polynomial product of a0 + a1 x + a2 x^2 and b0 + b1 x + b2 x^2, reduced
   * with x^3 = x + 1 and x^4 = x^2 + x */
  int ac[3] = {a % 3, a / 3 % 3, a / 9}, bc[3] = {b % 3, b / 3 % 3, b / 9};
  int c[5] = {0, 0, 0, 0, 0};
  for (int i = 0; i < 3; ++i)
    for (int j = 0; j < 3; ++j) c[i + j] += ac[i] * bc[j];
  c[1] += c[3]; c[0] += c[3]; /* x^3 -> x + 1 */
  c[2] += c[4]; c[1] += c[4]; /* x^4 -> x^2 + x */
  return c[0] % 3 + 3 * (c[1] % 3) + 9 * (c[2] % 3);
}
/* H28[i][j] in {+1, -1} */
int oracle_h28(int i, int j) {
  static int chi[27];
  static int ready = 0;
  if (!ready) {
    for (int a = 0; a < 27; ++a) chi[a] = -1;
    chi[0] = 0;
    for (int a = 1; a < 27; ++a) chi[gf27_mul(a, a)] = 1;
    ready = 1;
  }
  int sij;
  if (i == j) return 1; /* H = I + S, S has a zero diagonal */
  if (i == 0) sij = 1;
  else if (j == 0) sij = -1;
  else sij = chi[gf27_add(i - 1, gf27_neg(j - 1))];
  return sij;
}
static int popcount64(uint64_t v) {
  int c = 0;
  for (; v; v &= v - 1) ++c;
  return c;
}
/* H[i][j] of order K (K a power of two, or 28 times one) */
int oracle_hadamard_entry(int64_t K, int64_t i, int64_t j) {
  int64_t p = (K % 28 == 0) ? K / 28 : K;
  int s = (popcount64((uint64_t)((i % p) & (j % p))) & 1) ? -1 : 1;
  if (K % 28 == 0) s *= oracle_h28((int)(i / p), (int)(j / p));
  return s;
}
/* x fp16 [M, K] -> xr fp64 [M, K] = x H / sqrt(K) */
void oracle_hadamard_rotate(const uint16_t *x, int64_t M, int64_t K, double *xr) {
  double norm = 1.0 / sqrt((double)K);
#pragma omp parallel for schedule(static)
  for (int64_t j = 0; j < K; ++j)
    for (int64_t m = 0; m < M; ++m) {
      double acc = 0.0;
      for (int64_t i = 0; i < K; ++i)
        acc += oracle_half_to_double(x[m * K + i]) * (double)oracle_hadamard_entry(K, i, j);
      xr[m * K + j] = acc * norm;
    }
}

/* The activation quantiser on fp32 inputs (the rotated activations rounded
 * to fp32): the same steps as oracle_quantize, per token.               */
void oracle_quantize_f32(const float *x, int64_t M, int64_t K, int8_t *q, float *xs) {
  for (int64_t m = 0; m < M; ++m) {
    const float *xr = x + m * K;
    float amax = 0.0f;
    for (int64_t k = 0; k < K; ++k)
      if (fabsf(xr[k]) > amax) amax = fabsf(xr[k]);
    float s = amax / 127.0f;
    xs[m] = s;
    for (int64_t k = 0; k < K; ++k) {
      if (s == 0.0f) {
        q[m * K + k] = 0;
        continue;
      }
      float r = nearbyintf(xr[k] / s);
      if (r > 127.0f) r = 127.0f;
      if (r < -127.0f) r = -127.0f;
      q[m * K + k] = (int8_t)r;
    }
  }
}

/* ---- symmetric int8 activation quantiser --------------------------------
 * Model card, model table row "Activations": symmetric int8 per token, and
 * per 128-column group for o_proj.  Readings where the card is silent:
 *   scale s = max|x| / 127 in fp32 (one correctly rounded division);
 *   q = round-half-even(x / s) (one correctly rounded fp32 division, then
 *   rounding to the nearest integer, ties to even), clamped to [-127, 127];
 *   a row (group) whose max|x| is 0 gets s = 0 and q = 0 (no division).
 * group == 0: one scale per token, xs is [M];
 * group == 128: one scale per (token, 128-column group), xs is [M, K/128]. */
void oracle_quantize(const uint16_t *x, int64_t M, int64_t K, int group, int8_t *q,
                     float *xs) {
  int64_t span = (group == 0) ? K : group;
  int64_t nspan = K / span;
  for (int64_t m = 0; m < M; ++m)
    for (int64_t t = 0; t < nspan; ++t) {
      const uint16_t *xr = x + m * K + t * span;
      int8_t *qr = q + m * K + t * span;
      float amax = 0.0f;
      for (int64_t k = 0; k < span; ++k) {
        float a = fabsf(oracle_half_to_float(xr[k]));
        if (a > amax) amax = a;
      }
      float s = amax / 127.0f;
      xs[m * nspan + t] = s;
      for (int64_t k = 0; k < span; ++k) {
        if (s == 0.0f) {
          qr[k] = 0;
          continue;
        }
        float ratio = oracle_half_to_float(xr[k]) / s;
        float r = nearbyintf(ratio); /* default rounding: to nearest, ties to even */
        if (r > 127.0f) r = 127.0f;
        if (r < -127.0f) r = -127.0f;
        qr[k] = (int8_t)r;
      }
    }
}

/* ---- per-group integer sums ----------------------------------------------
 * S[m, n, g] = sum over the 128 columns k of group g of q[m, k] * code[n, k],
 * with code the integer weight code above.  Summed in int64; returns the
 * number of sums that do not fit int32 (always 0 for valid inputs).     */
int64_t oracle_group_sums(int mode, const uint8_t *hi, const uint8_t *lo, const int8_t *q,
                          int64_t M, int64_t N, int64_t K, int32_t *S) {
  int64_t G = K / ORACLE_GROUP;
  int64_t overflow = 0;
#pragma omp parallel for reduction(+ : overflow) schedule(static)
  for (int64_t n = 0; n < N; ++n)
    for (int64_t m = 0; m < M; ++m)
      for (int64_t g = 0; g < G; ++g) {
        int64_t acc = 0;
        for (int64_t k = g * ORACLE_GROUP; k < (g + 1) * ORACLE_GROUP; ++k)
          acc += (int64_t)q[m * K + k] * weight_code(mode, hi, lo, K, n, k);
        if (acc > INT32_MAX || acc < INT32_MIN) ++overflow;
        S[(m * N + n) * G + g] = (int32_t)acc;
      }
  return overflow;
}

/* ---- the layer output -----------------------------------------------------
 * y[m, n] = sum_k xdeq[m, k] * W[n, k] + bias[n], in fp64, with
 *   xdeq[m, k] = q[m, k] * xs  (xs per token, or per (token, group))
 *   W[n, k]    = the model card's draft or target dequantised weight.
 * bias may be NULL.  The output rows n and tokens m computed are the lists
 * rows[0..nrows) and toks[0..ntoks); y is [ntoks, nrows] (row-major).    */
void oracle_linear_subset(int mode, const uint8_t *hi, const uint8_t *lo,
                          const uint16_t *scale, const int8_t *q, const float *xs,
                          int64_t M, int64_t N, int64_t K, int act_group,
                          const uint16_t *bias, const int64_t *toks, int64_t ntoks,
                          const int64_t *rows, int64_t nrows, double *y) {
  int64_t G = K / ORACLE_GROUP;
  (void)M;
  (void)N;
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t i = 0; i < nrows; ++i) {
    int64_t n = rows[i];
    for (int64_t j = 0; j < ntoks; ++j) {
      int64_t m = toks[j];
      double acc = 0.0;
      for (int64_t k = 0; k < K; ++k) {
        int64_t g = k / ORACLE_GROUP;
        double xsv = (act_group == 0) ? (double)xs[m] : (double)xs[m * G + g];
        double xdeq = (double)q[m * K + k] * xsv;
        double s = oracle_half_to_double(scale[n * G + g]);
        double w;
        if (mode == ORACLE_DRAFT)
          w = (double)(nibble(hi, K, n, k) - 8) * s;
        else
          w = (double)(16 * (nibble(hi, K, n, k) - 8) + (nibble(lo, K, n, k) - 8)) * s / 16.0;
        acc += xdeq * w;
      }
      if (bias) acc += oracle_half_to_double(bias[n]);
      y[j * nrows + i] = acc;
    }
  }
}

/* Full output y [M, N]. */
void oracle_linear(int mode, const uint8_t *hi, const uint8_t *lo, const uint16_t *scale,
                   const int8_t *q, const float *xs, int64_t M, int64_t N, int64_t K,
                   int act_group, const uint16_t *bias, double *y) {
  int64_t *toks = (int64_t *)malloc(sizeof(int64_t) * (size_t)(M > 0 ? M : 1));
  int64_t *rows = (int64_t *)malloc(sizeof(int64_t) * (size_t)(N > 0 ? N : 1));
  for (int64_t m = 0; m < M; ++m) toks[m] = m;
  for (int64_t n = 0; n < N; ++n) rows[n] = n;
  oracle_linear_subset(mode, hi, lo, scale, q, xs, M, N, K, act_group, bias, toks, M, rows,
                       N, y);
  free(toks);
  free(rows);
}
