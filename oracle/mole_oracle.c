/*
 * mole_oracle.c -- plain, slow fp64 CPU oracle for the Mixture-of-Lookup-Experts
 * (MoLE) lookup path.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path links, loads or calls
 * this file; only the test-suite, the smoke check and the CPU-baseline leg of the
 * benchmark do.  It shares no code, header, table or constant with the CUDA
 * library: every number it uses is derived here from the definitions below.
 *
 * Source page ("MoLE page"): "ICML 2025 Spotlight | 华为诺亚提出端侧大模型新架构MoLE，
 * 内存搬运代价降低1000倍" (zejuncao.github.io, 2025-05-07).  Sections cited by
 * their headings: 思考 (motivation), 训练阶段 (training stage), 推理阶段
 * (inference stage), 复杂度分析 (complexity analysis), 实验结果 (results).
 *
 * Readings taken where the page is silent (its formulas and figures did not
 * survive extraction):
 *   - routed expert j is f_j(x) = act(x . W1_j) . W2_j, no biases, no norm;
 *   - the router is a full softmax over all N routed experts (no top-k);
 *   - the kernel output is the routed mixture only: sum_j g_j LUT[id, j, :];
 *   - NF3 = NormalFloat 3-bit levels (QLoRA construction, k = 3), rounded to
 *     fp16, with one fp16 absmax scale per 64 consecutive elements of a row.
 *
 * Precision: everything is fp64 except (a) the optional bf16 rounding of the
 * expert hidden activation in the table build (the precision point a bf16
 * tensor-core build has, made explicit here) and (b) the NF3 quantiser, which
 * is specified in IEEE fp32 so that codes are reproducible bit for bit.
 * Compile with -ffp-contract=off and without -ffast-math.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { OR_F32 = 0, OR_BF16 = 1 };
enum {
  OR_ACT_GELU_ERF = 0,
  OR_ACT_GELU_TANH = 1,
  OR_ACT_RELU = 2,
  OR_ACT_SILU = 3,
  OR_ACT_IDENTITY = 4
};

/* ------------------------------------------------------------------------- */
/* scalar helpers                                                              */
/* ------------------------------------------------------------------------- */

/* Read element i of a buffer holding fp32 values or bf16 bit patterns, exactly. */
static double load_elem(const void* p, int dtype, int64_t i) {
  if (dtype == OR_F32) return (double)((const float*)p)[i];
  uint32_t bits = ((uint32_t)((const uint16_t*)p)[i]) << 16;
  float f;
  memcpy(&f, &bits, sizeof f);
  return (double)f;
}

/* Round a double to the nearest value with `sig` significant bits, ties to
 * even, never going below the quantum 2^min_exp (gradual underflow).  This is
 * the definition of round-to-nearest-even into a binary format whose normal
 * numbers carry `sig` significant bits and whose smallest subnormal is
 * 2^min_exp.  Overflow is not handled here (callers bound their inputs). */
static double round_to_format(double x, int sig, int min_exp) {
  if (x == 0.0 || !isfinite(x)) return x;
  int e;
  frexp(x, &e);               /* |x| = m * 2^e, m in [0.5, 1) */
  int q = e - sig;            /* exponent of one unit in the last place */
  if (q < min_exp) q = min_exp;
  double scaled = ldexp(x, -q);
  double r = nearbyint(scaled); /* default rounding mode: nearest, ties to even */
  return ldexp(r, q);
}

/* bf16: 8 significant bits, smallest subnormal 2^-133. */
static double round_bf16(double x) { return round_to_format(x, 8, -133); }
/* fp16: 11 significant bits, smallest subnormal 2^-24, largest finite 65504. */
static double round_f16(double x) {
  double r = round_to_format(x, 11, -24);
  if (fabs(r) > 65504.0) r = copysign(INFINITY, r);
  return r;
}

/* Encode an fp16-representable double into its IEEE binary16 bit pattern. */
static uint16_t f16_bits(double x) {
  uint16_t s = signbit(x) ? 0x8000u : 0u;
  double a = fabs(x);
  if (a == 0.0) return s;
  if (isinf(a)) return (uint16_t)(s | 0x7c00u);
  if (a >= 0x1p-14) {
    int e;
    double m = frexp(a, &e); /* a = m 2^e, m in [0.5,1) => a = (2m) 2^(e-1) */
    int biased = (e - 1) + 15;
    uint16_t frac = (uint16_t)llround((2.0 * m - 1.0) * 1024.0);
    return (uint16_t)(s | (biased << 10) | frac);
  }
  return (uint16_t)(s | (uint16_t)llround(a * 0x1p24));
}

/* Decode an IEEE binary16 bit pattern. */
static double f16_value(uint16_t b) {
  int s = (b >> 15) & 1, e = (b >> 10) & 31, f = b & 1023;
  double v;
  if (e == 0) v = ldexp((double)f, -24);
  else if (e == 31) v = f ? NAN : INFINITY;
  else v = ldexp(1.0 + f / 1024.0, e - 15);
  return s ? -v : v;
}

/* Activation of the expert FFN.  GELU is the exact form u * Phi(u), with the
 * normal CDF written through erfc so that it keeps full relative accuracy in
 * the negative tail. */
static double act_fn(int act, double u) {
  switch (act) {
    case OR_ACT_GELU_ERF: return u * (0.5 * erfc(-u / sqrt(2.0))); /* u Phi(u) */
    case OR_ACT_GELU_TANH: {
      const double c = sqrt(2.0 / 3.14159265358979323846);
      return 0.5 * u * (1.0 + tanh(c * (u + 0.044715 * u * u * u)));
    }
    case OR_ACT_RELU: return u > 0.0 ? u : 0.0;
    case OR_ACT_SILU: return u / (1.0 + exp(-u));
    case OR_ACT_IDENTITY: return u;
    default: return NAN;
  }
}

double oracle_act(int act, double u) { return act_fn(act, u); }
double oracle_round_bf16(double x) { return round_bf16(x); }
double oracle_round_f16(double x) { return round_f16(x); }

static void set_threads(int nthreads) {
#ifdef _OPENMP
  if (nthreads > 0) omp_set_num_threads(nthreads);
#else
  (void)nthreads;
#endif
}

int oracle_max_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

/* ------------------------------------------------------------------------- */
/* Reparameterisation: build the lookup table  (MoLE page, 推理阶段)            */
/* ------------------------------------------------------------------------- */
/*
 * The embedding weight matrix E[V, D] holds every embedding token, so feeding
 * it to each routed expert yields the whole token-id -> expert-output map:
 *     LUT[v, j, :] = f_j(E[v, :]) = act(E[v, :] . W1[j]) . W2[j]
 * with W1[N, D, Dr] and W2[N, Dr, D] row-major.  Rows listed in `rows`
 * (or all V rows when rows == NULL, n_rows == V) are written to
 * out[n_rows, N, D].  When round_h != 0 each hidden activation is rounded to
 * bf16 (ties to even) before the second product.
 * Returns 0, or -1 on a bad argument / row index.
 */
/* One unit in the last place of the bf16 value b (normal range; the larger of
 * the two ulps at a power of two). */
static double bf16_ulp_of(double b) {
  double a = fabs(b);
  if (a < 0x1p-126) return 0x1p-133;
  int e;
  frexp(a, &e); /* a = m 2^e, m in [0.5, 1): a lies in [2^(e-1), 2^e) */
  return ldexp(1.0, e - 1 - 7);
}

/*
 * As oracle_build_lut, plus (when allow != NULL, bf16 rounding only) an error
 * allowance per output element for hidden activations whose bf16 rounding is
 * ambiguous.  A device computes u = x . W1 in fp32 and the activation in
 * fp32, so its pre-rounding value may sit on the other side of a bf16
 * rounding boundary than the exact one when the exact value is closer to that
 * boundary than
 *     beta_k = 1.2 * 2^-19 * M_k + 2^-21 |a_k|,
 * with M_k the largest magnitude of the running sum of u_k taken in order of
 * d (1.2 bounds the activation's slope, 2^-19 M_k the fp32 accumulation error
 * over K/16 steps of 16 products with margin, 2^-21 |a_k| the activation's
 * own error).  For such k either rounding is legitimate, so
 *     allow[r, j, e] = sum_{ambiguous k} ulp(a_k) |W2[j, k, e]|.
 * n_ambiguous (nullable) receives the number of ambiguous hidden values.
 */
int oracle_build_lut_ex(const void* E, const void* W1, const void* W2, int64_t V,
                        int64_t D, int32_t N, int64_t Dr, int act, int dtype,
                        int round_h, const int64_t* rows, int64_t n_rows,
                        double* out, double* allow, int64_t* n_ambiguous, int nthreads);

int oracle_build_lut(const void* E, const void* W1, const void* W2, int64_t V,
                     int64_t D, int32_t N, int64_t Dr, int act, int dtype,
                     int round_h, const int64_t* rows, int64_t n_rows,
                     double* out, int nthreads) {
  return oracle_build_lut_ex(E, W1, W2, V, D, N, Dr, act, dtype, round_h, rows, n_rows, out, NULL,
                             NULL, nthreads);
}

int oracle_build_lut_ex(const void* E, const void* W1, const void* W2, int64_t V,
                        int64_t D, int32_t N, int64_t Dr, int act, int dtype,
                        int round_h, const int64_t* rows, int64_t n_rows,
                        double* out, double* allow, int64_t* n_ambiguous, int nthreads) {
  if (V <= 0 || D <= 0 || N <= 0 || Dr <= 0 || n_rows < 0) return -1;
  if (rows == NULL && n_rows != V) return -1;
  for (int64_t r = 0; r < n_rows; ++r) {
    int64_t v = rows ? rows[r] : r;
    if (v < 0 || v >= V) return -1;
  }
  set_threads(nthreads);
  int bad = 0;
  int64_t n_amb = 0;
#pragma omp parallel for schedule(dynamic) reduction(| : bad) reduction(+ : n_amb)
  for (int64_t r = 0; r < n_rows; ++r) {
    int64_t v = rows ? rows[r] : r;
    double* x = (double*)malloc(sizeof(double) * (size_t)D);
    double* u = (double*)malloc(sizeof(double) * (size_t)Dr);
    double* mag = (double*)malloc(sizeof(double) * (size_t)Dr);
    double* amb = (double*)malloc(sizeof(double) * (size_t)Dr);
    if (!x || !u || !mag || !amb) { bad = 1; free(x); free(u); free(mag); free(amb); continue; }
    for (int64_t d = 0; d < D; ++d) x[d] = load_elem(E, dtype, v * D + d);
    for (int32_t j = 0; j < N; ++j) {
      /* u = x . W1[j], tracking the largest running magnitude of each sum */
      for (int64_t k = 0; k < Dr; ++k) { u[k] = 0.0; mag[k] = 0.0; }
      for (int64_t d = 0; d < D; ++d) {
        const int64_t base = ((int64_t)j * D + d) * Dr;
        for (int64_t k = 0; k < Dr; ++k) {
          u[k] += x[d] * load_elem(W1, dtype, base + k);
          if (fabs(u[k]) > mag[k]) mag[k] = fabs(u[k]);
        }
      }
      /* a = act(u), optionally rounded to bf16; amb[k] = ulp if ambiguous */
      for (int64_t k = 0; k < Dr; ++k) {
        double a = act_fn(act, u[k]);
        amb[k] = 0.0;
        if (round_h) {
          double ar = round_bf16(a);
          if (allow) {
            double ulp = bf16_ulp_of(ar);
            double to_boundary = 0.5 * ulp - fabs(a - ar);
            double beta = 1.2 * 0x1p-19 * mag[k] + 0x1p-21 * fabs(a);
            if (to_boundary <= beta) { amb[k] = ulp; n_amb += 1; }
          }
          a = ar;
        }
        u[k] = a;
      }
      /* out = a . W2[j] */
      double* o = out + (r * N + j) * D;
      double* al = allow ? allow + (r * N + j) * D : NULL;
      for (int64_t e = 0; e < D; ++e) { o[e] = 0.0; if (al) al[e] = 0.0; }
      for (int64_t k = 0; k < Dr; ++k) {
        const int64_t base = ((int64_t)j * Dr + k) * D;
        for (int64_t e = 0; e < D; ++e) {
          double w = load_elem(W2, dtype, base + e);
          o[e] += u[k] * w;
          if (al && amb[k] != 0.0) al[e] += amb[k] * fabs(w);
        }
      }
    }
    free(x);
    free(u);
    free(mag);
    free(amb);
  }
  if (n_ambiguous) *n_ambiguous = n_amb;
  return bad ? -1 : 0;
}

/* Element-wise bf16 rounding (ties to even) of n doubles. */
void oracle_round_bf16_array(const double* x, double* y, int64_t n) {
  for (int64_t i = 0; i < n; ++i) y[i] = round_bf16(x[i]);
}

/* ------------------------------------------------------------------------- */
/* Router + direct-addressed lookup + gate-weighted sum                        */
/* (MoLE page, 训练阶段: router on the previous layer's output, all routed     */
/*  experts active; 推理阶段: rows fetched by token id)                        */
/* ------------------------------------------------------------------------- */

/* Softmax of z[0..N) into g, subtracting the maximum first. */
static void softmax(const double* z, int32_t N, double* g) {
  double m = z[0];
  for (int32_t j = 1; j < N; ++j) if (z[j] > m) m = z[j];
  double s = 0.0;
  for (int32_t j = 0; j < N; ++j) { g[j] = exp(z[j] - m); s += g[j]; }
  for (int32_t j = 0; j < N; ++j) g[j] /= s;
}

/*
 * For each token t:
 *   z_j = sum_d h[t, d] Wr[d, j]            (router on the hidden state)
 *   g   = softmax(z)                         (all N routed experts active)
 *   out[t, :] = sum_j g_j LUT[ids[t], j, :]  (direct addressing by token id)
 * h is [T, D], Wr is [D, N], lut is [V, N, D]; each in fp32 or bf16.
 * A token whose id lies outside [0, V) gets a NaN output row (and NaN gates).
 * gates (nullable) receives g as [T, N].  Returns the number of such tokens,
 * or -1 on a bad argument.
 */
int64_t oracle_combine(const int32_t* ids, int64_t T, const void* h, int h_dtype,
                       const void* Wr, int w_dtype, const void* lut, int lut_dtype,
                       int64_t V, int32_t N, int64_t D, double* out, double* gates,
                       int nthreads) {
  if (T < 0 || V <= 0 || N <= 0 || D <= 0) return -1;
  set_threads(nthreads);
  int64_t n_bad = 0;
#pragma omp parallel for schedule(static) reduction(+ : n_bad)
  for (int64_t t = 0; t < T; ++t) {
    double z[256], g[256];
    double* o = out + t * D;
    int32_t id = ids[t];
    if (N > 256 || id < 0 || (int64_t)id >= V) {
      for (int64_t e = 0; e < D; ++e) o[e] = NAN;
      if (gates) for (int32_t j = 0; j < N; ++j) gates[t * N + j] = NAN;
      n_bad += 1;
      continue;
    }
    for (int32_t j = 0; j < N; ++j) {
      double acc = 0.0;
      for (int64_t d = 0; d < D; ++d)
        acc += load_elem(h, h_dtype, t * D + d) * load_elem(Wr, w_dtype, d * N + j);
      z[j] = acc;
    }
    softmax(z, N, g);
    if (gates) for (int32_t j = 0; j < N; ++j) gates[t * N + j] = g[j];
    for (int64_t e = 0; e < D; ++e) o[e] = 0.0;
    for (int32_t j = 0; j < N; ++j) {
      const int64_t base = ((int64_t)id * N + j) * D;
      for (int64_t e = 0; e < D; ++e) o[e] += g[j] * load_elem(lut, lut_dtype, base + e);
    }
  }
  return n_bad;
}

/* ------------------------------------------------------------------------- */
/* Gather plan: the distinct token ids of a batch, sorted, and each token's     */
/* slot among them (the set of rows a batch has to fetch; MoLE page, 复杂度分析) */
/* ------------------------------------------------------------------------- */

static int cmp_i32(const void* a, const void* b) {
  int32_t x = *(const int32_t*)a, y = *(const int32_t*)b;
  return (x > y) - (x < y);
}

/* uniq receives the ascending distinct ids (capacity T), *n_uniq their count,
 * slot[t] the index of ids[t] in uniq.  Returns 0, or -1 if an id is outside
 * [0, V). */
int oracle_gather_plan(const int32_t* ids, int64_t T, int64_t V, int32_t* uniq,
                       int32_t* n_uniq, int32_t* slot) {
  for (int64_t t = 0; t < T; ++t)
    if (ids[t] < 0 || (int64_t)ids[t] >= V) return -1;
  int32_t* s = (int32_t*)malloc(sizeof(int32_t) * (size_t)(T > 0 ? T : 1));
  if (!s) return -1;
  memcpy(s, ids, sizeof(int32_t) * (size_t)T);
  qsort(s, (size_t)T, sizeof(int32_t), cmp_i32);
  int32_t n = 0;
  for (int64_t t = 0; t < T; ++t)
    if (n == 0 || s[t] != uniq[n - 1]) uniq[n++] = s[t];
  *n_uniq = n;
  for (int64_t t = 0; t < T; ++t) {
    /* binary search of ids[t] in uniq[0..n) */
    int32_t lo = 0, hi = n - 1;
    while (lo < hi) {
      int32_t mid = lo + (hi - lo) / 2;
      if (uniq[mid] < ids[t]) lo = mid + 1; else hi = mid;
    }
    slot[t] = lo;
  }
  free(s);
  return 0;
}

/* ------------------------------------------------------------------------- */
/* NF3 compression of the table (MoLE page, 实验结果: the table tolerates       */
/* 3-bit storage such as NF3)                                                  */
/* ------------------------------------------------------------------------- */

/* Standard normal CDF and its inverse by bisection (plain, slow, exact to the
 * last bit of a double within 200 halvings). */
static double normal_cdf(double x) { return 0.5 * erfc(-x / sqrt(2.0)); }
static double normal_quantile(double p) {
  double lo = -40.0, hi = 40.0;
  for (int it = 0; it < 200; ++it) {
    double mid = 0.5 * (lo + hi);
    if (normal_cdf(mid) < p) lo = mid; else hi = mid;
  }
  return 0.5 * (lo + hi);
}

/*
 * NormalFloat levels for k = 3 bits (QLoRA, Dettmers et al. 2023, the
 * asymmetric NormalFloat data type with an exact zero): with
 *   delta = (1/(2(2^k - 1)) + 1/(2 * 2^k)) / 2,  p_hi = 1 - delta,
 * the positive levels are the normal quantiles of 2^(k-1) probabilities evenly
 * spaced from p_hi towards 1/2 (2^(k-1)+1 points, 1/2 itself dropped), the
 * negative levels the negated quantiles of 2^(k-1)-1 probabilities spaced the
 * same way (2^(k-1) points, 1/2 dropped), plus 0; all divided by the largest
 * so the set spans [-1, 1].  Written ascending into lv[8].
 */
void oracle_nf3_levels(double lv[8]) {
  const int k = 3, half = 1 << (k - 1);
  const double delta = 0.5 * (1.0 / (2.0 * ((1 << k) - 1)) + 1.0 / (2.0 * (1 << k)));
  const double p_hi = 1.0 - delta;
  double v[8];
  int n = 0;
  for (int i = 0; i < half; ++i) { /* half+1 evenly spaced points, last (=1/2) dropped */
    double p = p_hi + (0.5 - p_hi) * (double)i / (double)half;
    v[n++] = normal_quantile(p);
  }
  for (int i = 0; i < half - 1; ++i) { /* half points, last dropped */
    double p = p_hi + (0.5 - p_hi) * (double)i / (double)(half - 1);
    v[n++] = -normal_quantile(p);
  }
  v[n++] = 0.0;
  double mx = 0.0;
  for (int i = 0; i < 8; ++i) if (fabs(v[i]) > mx) mx = fabs(v[i]);
  for (int i = 0; i < 8; ++i) v[i] /= mx;
  /* sort ascending (insertion sort) */
  for (int i = 1; i < 8; ++i) {
    double x = v[i];
    int j = i - 1;
    while (j >= 0 && v[j] > x) { v[j + 1] = v[j]; --j; }
    v[j + 1] = x;
  }
  memcpy(lv, v, sizeof v);
}

/* The NF3 levels as stored: each rounded to fp16 (ties to even). */
void oracle_nf3_levels_f16(uint16_t bits[8]) {
  double lv[8];
  oracle_nf3_levels(lv);
  for (int i = 0; i < 8; ++i) bits[i] = f16_bits(round_f16(lv[i]));
}

/* Decision thresholds: fp32 midpoints of adjacent stored levels. */
void oracle_nf3_midpoints(float mid[7]) {
  uint16_t b[8];
  oracle_nf3_levels_f16(b);
  for (int i = 0; i < 7; ++i) {
    double a = f16_value(b[i]), c = f16_value(b[i + 1]);
    mid[i] = (float)((a + c) / 2.0); /* a + c is exact in double; one rounding */
  }
}

/* Index of the level 0 among the stored levels. */
static int nf3_zero_code(const uint16_t b[8]) {
  for (int i = 0; i < 8; ++i) if (f16_value(b[i]) == 0.0) return i;
  return -1;
}

/*
 * Quantise a bf16 table [V, N, D] (D a multiple of 64) block by block.  A block
 * is 64 consecutive elements x_0..x_63 of one (v, j) row.  In IEEE fp32:
 *   amax = max |x_e|;  s = fp16(min(amax, 65504)) (ties to even)
 *   s == 0:  every code is the index of level 0
 *   else:    y_e = x_e / s (correctly rounded);  c_e = #{k : y_e > mid_k}
 * (so a value exactly on a midpoint takes the lower level).  Code e occupies
 * bits [3e, 3e+3) of the block's 24-byte little-endian bit string.
 * codes: [V, N, D/64, 24] bytes; scales: [V, N, D/64] fp16 bit patterns.
 * Returns 0, or -1 on a bad argument.
 */
int oracle_quantize_nf3(const uint16_t* lut_bf16, int64_t V, int32_t N, int64_t D,
                        uint8_t* codes, uint16_t* scales) {
  if (V <= 0 || N <= 0 || D <= 0 || D % 64 != 0) return -1;
  uint16_t lvb[8];
  float mid[7];
  oracle_nf3_levels_f16(lvb);
  oracle_nf3_midpoints(mid);
  const int zero_code = nf3_zero_code(lvb);
  const int64_t nb = D / 64;
  for (int64_t blk = 0; blk < V * N * nb; ++blk) {
    const uint16_t* xb = lut_bf16 + blk * 64;
    float x[64];
    float amax = 0.0f;
    for (int e = 0; e < 64; ++e) {
      x[e] = (float)load_elem(xb, OR_BF16, e);
      float a = fabsf(x[e]);
      if (a > amax) amax = a;
    }
    if (amax > 65504.0f) amax = 65504.0f;
    double s_d = round_f16((double)amax);
    scales[blk] = f16_bits(s_d);
    float s = (float)s_d;
    uint8_t* cb = codes + blk * 24;
    memset(cb, 0, 24);
    for (int e = 0; e < 64; ++e) {
      int c;
      if (s == 0.0f) {
        c = zero_code;
      } else {
        float y = x[e] / s;
        c = 0;
        for (int k = 0; k < 7; ++k) if (y > mid[k]) c += 1;
      }
      for (int b = 0; b < 3; ++b) {
        int pos = 3 * e + b;
        cb[pos / 8] |= (uint8_t)(((c >> b) & 1) << (pos % 8));
      }
    }
  }
  return 0;
}

/* Read code e of a 24-byte block. */
int oracle_nf3_code(const uint8_t* block, int e) {
  int c = 0;
  for (int b = 0; b < 3; ++b) {
    int pos = 3 * e + b;
    c |= ((block[pos / 8] >> (pos % 8)) & 1) << b;
  }
  return c;
}

/* Dequantise a whole NF3 table into doubles: value = level[c] * s. */
int oracle_dequantize_nf3(const uint8_t* codes, const uint16_t* scales, int64_t V,
                          int32_t N, int64_t D, double* out) {
  if (V <= 0 || N <= 0 || D <= 0 || D % 64 != 0) return -1;
  uint16_t lvb[8];
  oracle_nf3_levels_f16(lvb);
  const int64_t nb = D / 64;
  for (int64_t blk = 0; blk < V * N * nb; ++blk) {
    double s = f16_value(scales[blk]);
    for (int e = 0; e < 64; ++e)
      out[blk * 64 + e] = f16_value(lvb[oracle_nf3_code(codes + blk * 24, e)]) * s;
  }
  return 0;
}

/*
 * The combine of oracle_combine over an NF3 table: the row element used for
 * (id, j, d) is level[c] * s of its block, formed exactly (an fp16 level times
 * an fp16 scale is exact in fp32 and in fp64).  Returns the number of tokens
 * with an out-of-range id (NaN rows), or -1 on a bad argument.
 */
int64_t oracle_combine_nf3(const int32_t* ids, int64_t T, const void* h, int h_dtype,
                           const void* Wr, int w_dtype, const uint8_t* codes,
                           const uint16_t* scales, int64_t V, int32_t N, int64_t D,
                           double* out, int nthreads) {
  if (T < 0 || V <= 0 || N <= 0 || D <= 0 || D % 64 != 0) return -1;
  uint16_t lvb[8];
  double lv[8];
  oracle_nf3_levels_f16(lvb);
  for (int i = 0; i < 8; ++i) lv[i] = f16_value(lvb[i]);
  const int64_t nb = D / 64;
  set_threads(nthreads);
  int64_t n_bad = 0;
#pragma omp parallel for schedule(static) reduction(+ : n_bad)
  for (int64_t t = 0; t < T; ++t) {
    double z[256], g[256];
    double* o = out + t * D;
    int32_t id = ids[t];
    if (N > 256 || id < 0 || (int64_t)id >= V) {
      for (int64_t e = 0; e < D; ++e) o[e] = NAN;
      n_bad += 1;
      continue;
    }
    for (int32_t j = 0; j < N; ++j) {
      double acc = 0.0;
      for (int64_t d = 0; d < D; ++d)
        acc += load_elem(h, h_dtype, t * D + d) * load_elem(Wr, w_dtype, d * N + j);
      z[j] = acc;
    }
    softmax(z, N, g);
    for (int64_t e = 0; e < D; ++e) o[e] = 0.0;
    for (int32_t j = 0; j < N; ++j) {
      for (int64_t b = 0; b < nb; ++b) {
        const int64_t blk = ((int64_t)id * N + j) * nb + b;
        double s = f16_value(scales[blk]);
        for (int e = 0; e < 64; ++e)
          o[b * 64 + e] += g[j] * (lv[oracle_nf3_code(codes + blk * 24, e)] * s);
      }
    }
  }
  return n_bad;
}
