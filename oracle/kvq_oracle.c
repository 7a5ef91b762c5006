/*
 * CPU oracle for pattern-aligned residual KV quantization and decode attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call, link or
 * load this file: only tests/, the package smoke check and the benchmark's CPU
 * baseline use it.  It shares no code, header, table or constant with the CUDA
 * library; it restates the method from the pages, plainly and slowly.
 *
 * Sources (page title, section / equation):
 *   [PKV]   "PatternKV: Flattening KV Representation Expands Quantization Headroom"
 *   [KVarN] "KVarN: Variance-Normalized KV-Cache Quantization Mitigates Error
 *            Accumulation in Reasoning Tasks" (abstract)
 *
 * Precision contract: everything is float64 except the quantization step, which
 * is written as single IEEE fp32 operations in a fixed order (pre-transform
 * apply, residual, min-max distance, group min/max, scale and zero, the
 * (R - z) / s division, round-half-even, clamp), so that a GPU can reproduce
 * indices and codes bit for bit.  Build with -ffp-contract=off (no fused
 * multiply-add) and without fast-math.
 *
 * Head dimension is fixed at D = 128 everywhere in this file.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define D 128

/* ------------------------------------------------------------------------- */
/* Pattern mining: Lloyd k-means under the Euclidean metric.                 */
/* [PKV] Section 3.1 "Pattern Mining", Eq. 4: minimise the within-pattern    */
/* sum of squared distances; centroids are the patterns.                     */
/*                                                                           */
/* Readings where the page is silent: deterministic strided initialisation   */
/* M_j = x[floor(j*n/P)]; squared distances in float64 summed over channels  */
/* 0..127 in order; ties go to the lowest index; centroid = fp32 rounding of */
/* the float64 mean (sum in token order); an empty cluster keeps its pattern.*/
/* ------------------------------------------------------------------------- */

/* Squared Euclidean distance, float64, channels in ascending order, no FMA. */
double kvqo_sqdist(const float* x, const float* m) {
  double acc = 0.0;
  for (int d = 0; d < D; ++d) {
    double t = (double)x[d] - (double)m[d];
    double sq = t * t;
    acc = acc + sq;
  }
  return acc;
}

/* Index of the nearest pattern under kvqo_sqdist; the lowest index wins ties. */
int32_t kvqo_nearest_euclid(const float* x, const float* M, int32_t P) {
  int32_t best = 0;
  double bd = kvqo_sqdist(x, M);
  for (int32_t j = 1; j < P; ++j) {
    double dj = kvqo_sqdist(x, M + (size_t)j * D);
    if (dj < bd) { bd = dj; best = j; }
  }
  return best;
}

/*
 * x: n rows of 128 floats.  M (out): P x 128 patterns.  assign (out, may be
 * NULL): the assignment of the last iteration (made against the patterns
 * that iteration started from).  Returns 0, or -1 if n < P or P < 1.
 */
int kvqo_mine(const float* x, int64_t n, int32_t P, int32_t iters, float* M, int32_t* assign) {
  if (P < 1 || n < P || iters < 0) return -1;
  for (int32_t j = 0; j < P; ++j) {
    int64_t src = (int64_t)((j * n) / P);
    memcpy(M + (size_t)j * D, x + (size_t)src * D, D * sizeof(float));
  }
  int32_t* a = (int32_t*)malloc((size_t)n * sizeof(int32_t));
  double* sum = (double*)malloc((size_t)P * D * sizeof(double));
  int64_t* cnt = (int64_t*)malloc((size_t)P * sizeof(int64_t));
  if (!a || !sum || !cnt) { free(a); free(sum); free(cnt); return -2; }
  for (int32_t it = 0; it < iters; ++it) {
    /* assignment step */
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) a[i] = kvqo_nearest_euclid(x + (size_t)i * D, M, P);
    /* update step: float64 sums in token order, then the mean rounded to fp32 */
    memset(sum, 0, (size_t)P * D * sizeof(double));
    memset(cnt, 0, (size_t)P * sizeof(int64_t));
    for (int64_t i = 0; i < n; ++i) {
      double* s = sum + (size_t)a[i] * D;
      const float* xi = x + (size_t)i * D;
      for (int d = 0; d < D; ++d) s[d] = s[d] + (double)xi[d];
      cnt[a[i]] += 1;
    }
    for (int32_t j = 0; j < P; ++j) {
      if (cnt[j] == 0) continue;
      for (int d = 0; d < D; ++d) M[(size_t)j * D + d] = (float)(sum[(size_t)j * D + d] / (double)cnt[j]);
    }
  }
  if (assign) memcpy(assign, a, (size_t)n * sizeof(int32_t));
  free(a); free(sum); free(cnt);
  return 0;
}

/* Within-pattern objective of Eq. 4 for given patterns and assignment (float64). */
double kvqo_objective(const float* x, int64_t n, const float* M, const int32_t* a) {
  double tot = 0.0;
  for (int64_t i = 0; i < n; ++i) tot += kvqo_sqdist(x + (size_t)i * D, M + (size_t)a[i] * D);
  return tot;
}

/* ------------------------------------------------------------------------- */
/* Pre-transform: Hadamard rotation + dual-axis variance normalisation.      */
/* [KVarN] abstract: a Hadamard rotation followed by a dual-scaling variance */
/* normalisation over both axes (tokens and channels) of K and of V.         */
/*                                                                           */
/* Readings: Sylvester-ordered Walsh-Hadamard transform of size 128, as the  */
/* in-place butterfly with strides 1, 2, 4, ..., 64, each step (a+b, a-b) in */
/* fp32; left unnormalised (a global factor cancels in the per-token         */
/* normalisation below and is undone exactly by 1/128 on the way back).      */
/* Column factors c are fitted once on the prefill block in float64 by 3     */
/* alternating passes (divide every row by its population std, then every    */
/* column by its population std; c = product of the column divisors, rounded */
/* to fp32).  Every token then gets its own row factor r = population std of */
/* u = x'/c over the 128 channels, computed in fp32 with halving sums; the   */
/* quantized vector is y = u / r.  A zero std counts as 1.                   */
/* ------------------------------------------------------------------------- */

/* In-place fp32 butterfly: for h = 1, 2, ..., 64 pair i and i+h inside each block of 2h. */
void kvqo_fwht(float* v) {
  for (int h = 1; h < D; h *= 2)
    for (int i0 = 0; i0 < D; i0 += 2 * h)
      for (int i = i0; i < i0 + h; ++i) {
        float a = v[i], b = v[i + h];
        v[i] = a + b;
        v[i + h] = a - b;
      }
}

/* Same butterfly in float64. */
void kvqo_fwht64(double* v) {
  for (int h = 1; h < D; h *= 2)
    for (int i0 = 0; i0 < D; i0 += 2 * h)
      for (int i = i0; i < i0 + h; ++i) {
        double a = v[i], b = v[i + h];
        v[i] = a + b;
        v[i + h] = a - b;
      }
}

/* fp32 sum of 128 values by halving: add the upper half onto the lower half until one is left. */
float kvqo_halving_sum(const float* v) {
  float w[D];
  memcpy(w, v, sizeof(w));
  for (int h = D / 2; h >= 1; h /= 2)
    for (int i = 0; i < h; ++i) w[i] = w[i] + w[i + h];
  return w[0];
}

/* Population std of the n values v[0], v[stride], ... in float64 (two passes). */
static double std64(const double* v, int64_t n, int64_t stride) {
  double mean = 0.0, var = 0.0;
  for (int64_t i = 0; i < n; ++i) mean += v[i * stride];
  mean /= (double)n;
  for (int64_t i = 0; i < n; ++i) {
    double t = v[i * stride] - mean;
    var += t * t;
  }
  return sqrt(var / (double)n);
}

/* xp: n rows already passed through kvqo_fwht.  c (out): 128 column factors. */
int kvqo_fit_colscale(const float* xp, int64_t n, int32_t passes, float* c) {
  if (n < 1) return -1;
  double* v = (double*)malloc((size_t)n * D * sizeof(double));
  if (!v) return -2;
  double C[D];
  for (int d = 0; d < D; ++d) C[d] = 1.0;
  for (int64_t i = 0; i < n * D; ++i) v[i] = (double)xp[i];
  for (int p = 0; p < passes; ++p) {
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < n; ++t) {
      double r = std64(v + (size_t)t * D, D, 1);
      if (r == 0.0) r = 1.0;
      for (int d = 0; d < D; ++d) v[(size_t)t * D + d] /= r;
    }
    for (int d = 0; d < D; ++d) {
      double s = std64(v + d, n, D);
      if (s == 0.0) s = 1.0;
      for (int64_t t = 0; t < n; ++t) v[(size_t)t * D + d] /= s;
      C[d] *= s;
    }
  }
  for (int d = 0; d < D; ++d) c[d] = (float)C[d];
  free(v);
  return 0;
}

/* One token: x (raw row) -> y (normalised, fp32) and its row factor r. */
void kvqo_apply_row(const float* x, const float* c, float* y, float* r_out) {
  float u[D], dev2[D];
  memcpy(u, x, sizeof(u));
  kvqo_fwht(u);
  for (int d = 0; d < D; ++d) u[d] = u[d] / c[d];
  float mean = kvqo_halving_sum(u) / 128.0f;
  for (int d = 0; d < D; ++d) {
    float t = u[d] - mean;
    dev2[d] = t * t;
  }
  float var = kvqo_halving_sum(dev2) / 128.0f;
  float r = sqrtf(var);
  if (r == 0.0f) r = 1.0f;
  for (int d = 0; d < D; ++d) y[d] = u[d] / r;
  *r_out = r;
}

/* ------------------------------------------------------------------------- */
/* Pattern alignment: [PKV] Section 3.2, min-max distance and Eq. 6.         */
/*   d_mm(x, m) = max_i (x_i - m_i) - min_j (x_j - m_j)                      */
/*   M* = argmin over the pattern set of d_mm(X, M),  R = X - M*             */
/* Evaluated in fp32: r_d = fl32(x_d - m_d), d = fl32(max r - min r); the    */
/* lowest index wins ties.                                                   */
/* ------------------------------------------------------------------------- */

float kvqo_dmm(const float* x, const float* m) {
  float mx = x[0] - m[0], mn = mx;
  for (int d = 1; d < D; ++d) {
    float r = x[d] - m[d];
    if (r > mx) mx = r;
    if (r < mn) mn = r;
  }
  return mx - mn;
}

int32_t kvqo_assign(const float* x, const float* M, int32_t P) {
  int32_t best = 0;
  float bd = kvqo_dmm(x, M);
  for (int32_t j = 1; j < P; ++j) {
    float dj = kvqo_dmm(x, M + (size_t)j * D);
    if (dj < bd) { bd = dj; best = j; }
  }
  return best;
}

/* ------------------------------------------------------------------------- */
/* Flattening-sensitive adaptive threshold for V: [PKV] Section 3.3, Eq. 7-10.*/
/* A one-sided z-test at level alpha accepts flattening (use of the pattern) */
/* only when the contraction ratio rho = R_flat / R_raw satisfies            */
/*   1 - rho^2 >= 2 z_{1-alpha} / sqrt(5 d) * sqrt(1 + rho^4),               */
/* i.e. rho <= rho*(d, alpha), the root of the equality (Eq. 10).            */
/* Readings: R_raw = max v - min v of the V vector, R_flat = d_mm(v, M*)     */
/* (the range of its residual); the test is made in fp32 as                  */
/*   use the pattern  iff  R_flat <= fl32(rho*_fp32 * R_raw);                */
/* a rejected vector stores index 255 and is quantized raw (pattern 0).      */
/* ------------------------------------------------------------------------- */

/* Standard normal upper quantile z with P(Z > z) = a, by bisection on erfc. */
double kvqo_normal_upper_quantile(double a) {
  double lo = -40.0, hi = 40.0;
  for (int it = 0; it < 200; ++it) {
    double mid = 0.5 * (lo + hi);
    double tail = 0.5 * erfc(mid / sqrt(2.0)); /* P(Z > mid), decreasing in mid */
    if (tail > a) lo = mid; else hi = mid;
  }
  return 0.5 * (lo + hi);
}

/* rho*(d, alpha): the root in (0, 1) of (1 - rho^2) - 2 z / sqrt(5 d) sqrt(1 + rho^4), by bisection. */
double kvqo_rho_star(int32_t d, double alpha) {
  const double z = kvqo_normal_upper_quantile(alpha);
  const double k = 2.0 * z / sqrt(5.0 * (double)d);
  double lo = 0.0, hi = 1.0; /* f(0) = 1 - k > 0 for the d, alpha of interest; f(1) < 0 */
  for (int it = 0; it < 200; ++it) {
    double mid = 0.5 * (lo + hi);
    double f = (1.0 - mid * mid) - k * sqrt(1.0 + mid * mid * mid * mid);
    if (f > 0.0) lo = mid; else hi = mid;
  }
  return 0.5 * (lo + hi);
}

/* fp32 range max - min of a 128-vector. */
float kvqo_range(const float* x) {
  float mx = x[0], mn = x[0];
  for (int d = 1; d < D; ++d) {
    if (x[d] > mx) mx = x[d];
    if (x[d] < mn) mn = x[d];
  }
  return mx - mn;
}

/* ------------------------------------------------------------------------- */
/* Asymmetric n-bit group quantizer: [PKV] Section 2.1, Eq. 1.               */
/*   Q = round((X - z) / s),  s = (max X - min X) / (2^n - 1),  z = min X    */
/* fp32, in this order: mn, mx exact; s = fl32(fl32(mx - mn) / (2^n - 1));   */
/* z = mn; q = s == 0 ? 0 : clamp(rne(fl32(fl32(R - z) / s)), 0, 2^n - 1).   */
/* ------------------------------------------------------------------------- */

void kvqo_quant_group(const float* R, int64_t n, int64_t stride, int32_t bits, float* s_out, float* z_out,
                      int32_t* q, int64_t qstride) {
  float mn = R[0], mx = R[0];
  for (int64_t i = 1; i < n; ++i) {
    float v = R[i * stride];
    if (v < mn) mn = v;
    if (v > mx) mx = v;
  }
  const float levels = (float)((1 << bits) - 1);
  float span = mx - mn;
  float s = span / levels;
  float z = mn;
  for (int64_t i = 0; i < n; ++i) {
    int32_t code = 0;
    if (s != 0.0f) {
      float t = R[i * stride] - z;
      float u = t / s;
      float rq = rintf(u); /* round-half-even under the default rounding mode */
      code = (int32_t)rq;
      if (code < 0) code = 0;
      if (code > (1 << bits) - 1) code = (1 << bits) - 1;
    }
    q[i * qstride] = code;
  }
  *s_out = s;
  *z_out = z;
}

/* ------------------------------------------------------------------------- */
/* Encoding of one (sequence, KV head) token stream of N tokens.             */
/* Granularity ([PKV] Section 4.1, matching KIVI): K per channel, V per      */
/* token, group 32.  V is quantized per token over 4 groups of 32 channels.  */
/* K is quantized per channel over each complete group of 32 tokens; the    */
/* N % 32 most recent K tokens are not quantized (they stay full precision). */
/* Patterns are aligned after RoPE, i.e. on the inputs as given ([PKV] 4.1). */
/*                                                                           */
/* Outputs (natural order, one byte per code):                               */
/*   kcode[G][32][128], ks/kz[G][128], kidx[G][32], krow[G][32]              */
/*   vcode[N][128], vs/vz[N][4], vidx[N], vrow[N]                            */
/* with G = N / 32.  cK/cV NULL means no pre-transform (rows are then 1).    */
/* v_rho > 0 enables the V adaptive threshold (Section 3.3) with that fp32   */
/* rho*; v_rho <= 0 always uses the nearest pattern.                         */
/* ------------------------------------------------------------------------- */

static void prep_row(const float* x, const float* c, float* y, float* r) {
  if (c) {
    kvqo_apply_row(x, c, y, r);
  } else {
    memcpy(y, x, D * sizeof(float));
    *r = 1.0f;
  }
}

int kvqo_encode(const float* K, const float* V, int64_t N, int32_t bits, int32_t P, const float* MK,
                const float* MV, const float* cK, const float* cV, float v_rho, uint8_t* kcode, float* ks,
                float* kz, uint8_t* kidx, float* krow, uint8_t* vcode, float* vs, float* vz, uint8_t* vidx,
                float* vrow) {
  if (bits != 2 && bits != 4) return -1;
  if (P < 1 || P > 255) return -1;
  /* V: every token */
#pragma omp parallel for schedule(static)
  for (int64_t t = 0; t < N; ++t) {
    float y[D], R[D];
    prep_row(V + (size_t)t * D, cV, y, &vrow[t]);
    int32_t j = kvqo_assign(y, MV, P);
    int use = 1;
    if (v_rho > 0.0f) {
      float r_flat = kvqo_dmm(y, MV + (size_t)j * D);
      float r_raw = kvqo_range(y);
      float limit = v_rho * r_raw;
      use = r_flat <= limit;
    }
    vidx[t] = use ? (uint8_t)j : (uint8_t)255;
    for (int d = 0; d < D; ++d) R[d] = use ? y[d] - MV[(size_t)j * D + d] : y[d];
    int32_t q[D];
    for (int g = 0; g < 4; ++g) kvqo_quant_group(R + 32 * g, 32, 1, bits, &vs[t * 4 + g], &vz[t * 4 + g], q + 32 * g, 1);
    for (int d = 0; d < D; ++d) vcode[(size_t)t * D + d] = (uint8_t)q[d];
  }
  /* K: complete groups of 32 tokens */
  int64_t G = N / 32;
#pragma omp parallel for schedule(static)
  for (int64_t g = 0; g < G; ++g) {
    float R[32][D];
    for (int t = 0; t < 32; ++t) {
      float y[D];
      int64_t tok = g * 32 + t;
      prep_row(K + (size_t)tok * D, cK, y, &krow[g * 32 + t]);
      int32_t j = kvqo_assign(y, MK, P);
      kidx[g * 32 + t] = (uint8_t)j;
      for (int d = 0; d < D; ++d) R[t][d] = y[d] - MK[(size_t)j * D + d];
    }
    int32_t q[32][D];
    for (int d = 0; d < D; ++d) kvqo_quant_group(&R[0][d], 32, D, bits, &ks[g * D + d], &kz[g * D + d], &q[0][d], D);
    for (int t = 0; t < 32; ++t)
      for (int d = 0; d < D; ++d) kcode[((size_t)g * 32 + t) * D + d] = (uint8_t)q[t][d];
  }
  return 0;
}

/* ------------------------------------------------------------------------- */
/* Decode-time pattern insertion: [PKV] Section 3.1 "Decoding Stage", Eq. 5. */
/* The Chebyshev center of a window of KV vectors, per dimension the mean of */
/* its minimum and maximum, becomes a new pattern:                           */
/*   M_new_d = fl32(fl32(min_i X_id + max_i X_id) * 0.5).                    */
/* Readings: windows of G_pattern tokens aligned to multiples of G_pattern   */
/* (the prefill length is one); the vectors are the (pre-transformed) K and  */
/* V vectors appended after the prefill; the new K and V patterns join their */
/* sets as index P (the sets grow together, up to a capacity, then stop) and */
/* are used from the next token on.                                          */
/* ------------------------------------------------------------------------- */

void kvqo_chebyshev_center(const float* X, int64_t n, float* M) {
  for (int d = 0; d < D; ++d) {
    float mn = X[d], mx = X[d];
    for (int64_t i = 1; i < n; ++i) {
      float v = X[(size_t)i * D + d];
      if (v < mn) mn = v;
      if (v > mx) mx = v;
    }
    float s = mn + mx;
    M[d] = s * 0.5f;
  }
}

/* One V token: assign (d_mm), optional adaptive threshold, residual, 4 groups of Eq. 1. */
static void encode_v_token(const float* x, const float* cV, const float* MV, int32_t P, int32_t bits, float v_rho,
                           uint8_t* vcode, float* vs, float* vz, uint8_t* vidx, float* vrow, float* y_out) {
  float y[D], R[D];
  prep_row(x, cV, y, vrow);
  int32_t j = kvqo_assign(y, MV, P);
  int use = 1;
  if (v_rho > 0.0f) {
    float r_flat = kvqo_dmm(y, MV + (size_t)j * D);
    float limit = v_rho * kvqo_range(y);
    use = r_flat <= limit;
  }
  *vidx = use ? (uint8_t)j : (uint8_t)255;
  for (int d = 0; d < D; ++d) R[d] = use ? y[d] - MV[(size_t)j * D + d] : y[d];
  int32_t q[D];
  for (int g = 0; g < 4; ++g) kvqo_quant_group(R + 32 * g, 32, 1, bits, &vs[g], &vz[g], q + 32 * g, 1);
  for (int d = 0; d < D; ++d) vcode[d] = (uint8_t)q[d];
  if (y_out) memcpy(y_out, y, sizeof(y));
}

/* One complete K group of 32 tokens: assign each vector, quantize per channel. */
static void encode_k_group(const float* K32, const float* cK, const float* MK, int32_t P, int32_t bits,
                           uint8_t* kcode, float* ks, float* kz, uint8_t* kidx, float* krow) {
  float R[32][D];
  for (int t = 0; t < 32; ++t) {
    float y[D];
    prep_row(K32 + (size_t)t * D, cK, y, &krow[t]);
    int32_t j = kvqo_assign(y, MK, P);
    kidx[t] = (uint8_t)j;
    for (int d = 0; d < D; ++d) R[t][d] = y[d] - MK[(size_t)j * D + d];
  }
  int32_t q[32][D];
  for (int d = 0; d < D; ++d) kvqo_quant_group(&R[0][d], 32, D, bits, &ks[d], &kz[d], &q[0][d], D);
  for (int t = 0; t < 32; ++t)
    for (int d = 0; d < D; ++d) kcode[(size_t)t * D + d] = (uint8_t)q[t][d];
}

/*
 * Streaming encoding of one (sequence, KV head): tokens [0, L0) are the prefill (encoded with
 * the first P0 patterns, as kvqo_encode does); tokens L0 .. N-1 arrive one at a time.  Token p:
 * its V vector is encoded with the patterns present; if it completes a K group, that group's 32
 * keys are encoded with the patterns present; then, with G > 0, it joins the window of positions
 * [G floor(p / G), G floor(p / G) + G), and when p + 1 is a multiple of G the Chebyshev centers
 * of the window's K and V vectors become patterns P and P + 0 of the K and V sets (if P < Pmax).
 * MK, MV: [Pmax][128], first P0 rows given, grown in place; *P_out: patterns at the end.
 * L0 must be a multiple of G when G > 0.  Outputs as kvqo_encode.
 */
int kvqo_encode_stream(const float* K, const float* V, int64_t N, int64_t L0, int32_t G, int32_t bits, int32_t P0,
                       int32_t Pmax, float* MK, float* MV, const float* cK, const float* cV, float v_rho,
                       int32_t* P_out, uint8_t* kcode, float* ks, float* kz, uint8_t* kidx, float* krow,
                       uint8_t* vcode, float* vs, float* vz, uint8_t* vidx, float* vrow) {
  if (bits != 2 && bits != 4) return -1;
  if (P0 < 1 || Pmax < P0 || Pmax > 255 || L0 < 0 || L0 > N) return -1;
  if (G < 0 || (G > 0 && L0 % G != 0)) return -1;
  int32_t P = P0;
  /* prefill: V tokens and complete K groups with the initial patterns */
  if (kvqo_encode(K, V, L0, bits, P0, MK, MV, cK, cV, v_rho, kcode, ks, kz, kidx, krow, vcode, vs, vz, vidx,
                  vrow) != 0)
    return -1;
  float* wk = (float*)malloc((size_t)(G > 0 ? G : 1) * D * sizeof(float));
  float* wv = (float*)malloc((size_t)(G > 0 ? G : 1) * D * sizeof(float));
  if (!wk || !wv) { free(wk); free(wv); return -2; }
  int32_t nw = 0; /* vectors in the current window */
  for (int64_t p = L0; p < N; ++p) {
    float yv[D];
    encode_v_token(V + (size_t)p * D, cV, MV, P, bits, v_rho, vcode + (size_t)p * D, vs + p * 4, vz + p * 4,
                   vidx + p, vrow + p, yv);
    if ((p + 1) % 32 == 0) {
      int64_t g = p / 32;
      encode_k_group(K + (size_t)g * 32 * D, cK, MK, P, bits, kcode + (size_t)g * 32 * D, ks + g * D, kz + g * D,
                     kidx + g * 32, krow + g * 32);
    }
    if (G > 0) {
      float r;
      prep_row(K + (size_t)p * D, cK, wk + (size_t)nw * D, &r);
      memcpy(wv + (size_t)nw * D, yv, sizeof(yv));
      nw += 1;
      if ((p + 1) % G == 0) {
        if (P < Pmax) {
          kvqo_chebyshev_center(wk, nw, MK + (size_t)P * D);
          kvqo_chebyshev_center(wv, nw, MV + (size_t)P * D);
          P += 1;
        }
        nw = 0;
      }
    }
  }
  free(wk);
  free(wv);
  *P_out = P;
  return 0;
}

/* ------------------------------------------------------------------------- */
/* Dequantization / reconstruction ([PKV] Section 3.2: fetch the pattern by  */
/* its stored index and undo the residualisation; Eq. 1: s*Q + z), float64.  */
/* With the pre-transform the result is mapped back: x = r * (y (.) c) H / 128.*/
/* ------------------------------------------------------------------------- */

static void unrotate(double* v, const float* c, float r) {
  for (int d = 0; d < D; ++d) v[d] = (double)r * (v[d] * (double)c[d]);
  kvqo_fwht64(v);
  for (int d = 0; d < D; ++d) v[d] /= 128.0;
}

/* Khat[G*32][128] from the K groups, Vhat[N][128] from the V tokens (original space). */
void kvqo_dequant(int64_t N, const float* MK, const float* MV, const float* cK, const float* cV,
                  const uint8_t* kcode, const float* ks, const float* kz, const uint8_t* kidx, const float* krow,
                  const uint8_t* vcode, const float* vs, const float* vz, const uint8_t* vidx, const float* vrow,
                  double* Khat, double* Vhat) {
  int64_t G = N / 32;
#pragma omp parallel for schedule(static)
  for (int64_t t = 0; t < G * 32; ++t) {
    int64_t g = t / 32;
    double* o = Khat + (size_t)t * D;
    const float* m = MK + (size_t)kidx[t] * D;
    for (int d = 0; d < D; ++d)
      o[d] = (double)ks[g * D + d] * (double)kcode[(size_t)t * D + d] + (double)kz[g * D + d] + (double)m[d];
    if (cK) unrotate(o, cK, krow[t]);
  }
#pragma omp parallel for schedule(static)
  for (int64_t t = 0; t < N; ++t) {
    double* o = Vhat + (size_t)t * D;
    const float* m = vidx[t] == 255 ? NULL : MV + (size_t)vidx[t] * D; /* 255: quantized raw */
    for (int d = 0; d < D; ++d)
      o[d] = (double)vs[t * 4 + d / 32] * (double)vcode[(size_t)t * D + d] + (double)vz[t * 4 + d / 32] +
             (m ? (double)m[d] : 0.0);
    if (cV) unrotate(o, cV, vrow[t]);
  }
}

/* ------------------------------------------------------------------------- */
/* Decode attention for the query heads sharing one KV head (GQA), float64:  */
/*   o_h = softmax(scale * q_h . Khat^T) Vhat, max-subtracted softmax.       */
/* Khat / Vhat hold N rows (quantized tokens reconstructed, the K tail exact).*/
/* ------------------------------------------------------------------------- */

void kvqo_attention(const double* q, int32_t Gq, const double* Khat, const double* Vhat, int64_t N, double scale,
                    double* out) {
  double* sc = (double*)malloc((size_t)(N > 0 ? N : 1) * sizeof(double));
  for (int32_t h = 0; h < Gq; ++h) {
    const double* qh = q + (size_t)h * D;
    double mx = -INFINITY;
    for (int64_t t = 0; t < N; ++t) {
      double s = 0.0;
      for (int d = 0; d < D; ++d) s += qh[d] * Khat[(size_t)t * D + d];
      sc[t] = scale * s;
      if (sc[t] > mx) mx = sc[t];
    }
    double l = 0.0;
    for (int64_t t = 0; t < N; ++t) {
      sc[t] = exp(sc[t] - mx);
      l += sc[t];
    }
    double* o = out + (size_t)h * D;
    for (int d = 0; d < D; ++d) o[d] = 0.0;
    for (int64_t t = 0; t < N; ++t)
      for (int d = 0; d < D; ++d) o[d] += sc[t] * Vhat[(size_t)t * D + d];
    for (int d = 0; d < D; ++d) o[d] = (N > 0) ? o[d] / l : 0.0;
  }
  free(sc);
}
