/*
 * Seeded synthetic K/V/q generator.
 *
 * This module only draws random inputs.  It holds none of the quantization,
 * pattern or attention arithmetic; both the CUDA path and the CPU oracle take
 * their inputs from here.
 *
 * Random numbers come from a counter-based generator: every value is a pure
 * function of (seed, stream, counter), so any slice of a workload can be
 * regenerated on its own (random access by sequence, position and head).
 *
 *   key(seed, stream)   = mix64(seed * G + mix64(stream + 1))
 *   bits(seed, s, ctr)  = mix64(key + (ctr + 1) * G)
 *   uniform             = ((bits >> 11) + 1) * 2^-53            in (0, 1]
 *   normal(i)           = Box-Muller on the uniforms at counters 2*(i/2) and
 *                         2*(i/2)+1: cos branch for even i, sin branch for odd i
 *
 * mix64 is the SplitMix64 finaliser, G = 0x9E3779B97F4A7C15.
 *
 * Workload recipe (per KV head h, sequence b, position p, channel d):
 *   centers      cen[h][c][d] ~ N(0,1), one mixture for K and one for V
 *   per-sample   cen_b = cen + sample_sigma * N(0,1)          (breadth workload)
 *   drift        for p >= drift_start: cen + drift_step*floor((p-drift_start)/drift_block)*u[h][c]
 *   choice       c ~ uniform over the centers, iid per (b, p, h), separately for K and V
 *   value        center + sigma * N(0,1)
 *   outliers     K only: n_outlier channels (first entries of a seeded permutation
 *                per head) scaled by U[out_lo, out_hi]
 *   RoPE         K only, optional: pairs (i, i+64), angle p * base^(-i/64)
 *   rounding     to fp16 or bf16, round-to-nearest-even (via fp32)
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define SYN_G 0x9E3779B97F4A7C15ULL

enum {
  ST_CENTER_K = 1, ST_CENTER_V, ST_CHOICE_K, ST_CHOICE_V, ST_NOISE_K, ST_NOISE_V,
  ST_OUTPERM, ST_OUTSCALE, ST_SAMPLE_K, ST_SAMPLE_V, ST_DRIFT_K, ST_DRIFT_V, ST_Q
};

typedef struct {
  uint64_t seed;
  int32_t B, S, Hkv, D;
  int32_t nck, ncv;
  double sigma_k, sigma_v;
  int32_t n_outlier;
  double out_lo, out_hi;
  int32_t rope;
  double rope_base;
  double sample_sigma;
  int32_t drift_start;   /* < 0: no drift */
  int32_t drift_block;
  double drift_step;
  int32_t dtype;         /* 0 = fp16, 1 = bf16 */
} synth_params;

static inline uint64_t mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xbf58476d1ce4e5b9ULL;
  z = (z ^ (z >> 27)) * 0x94d049bb133111ebULL;
  return z ^ (z >> 31);
}

static inline uint64_t syn_key(uint64_t seed, uint64_t stream) {
  return mix64(seed * SYN_G + mix64(stream + 1));
}

static inline double syn_uniform(uint64_t key, uint64_t ctr) {
  uint64_t b = mix64(key + (ctr + 1) * SYN_G);
  return ((double)(b >> 11) + 1.0) * (1.0 / 9007199254740992.0);
}

static inline double syn_normal(uint64_t key, uint64_t i) {
  uint64_t j = i >> 1;
  double u1 = syn_uniform(key, 2 * j), u2 = syn_uniform(key, 2 * j + 1);
  double r = sqrt(-2.0 * log(u1));
  double t = 6.283185307179586476925 * u2;
  return (i & 1) ? r * sin(t) : r * cos(t);
}

static inline uint16_t to_bf16(double v) {
  float f = (float)v;
  uint32_t u;
  memcpy(&u, &f, 4);
  u += 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

static inline uint16_t to_fp16(double v) {
  _Float16 h = (_Float16)(float)v;
  uint16_t u;
  memcpy(&u, &h, 2);
  return u;
}

static inline uint16_t to_dtype(double v, int dtype) { return dtype ? to_bf16(v) : to_fp16(v); }

/* Outlier channels of head h: first n entries of a Fisher-Yates shuffle of 0..D-1. */
static void outlier_channels(const synth_params* P, int h, int32_t* ch, double* scale) {
  int32_t perm[1024];
  uint64_t kp = syn_key(P->seed, ST_OUTPERM), ks = syn_key(P->seed, ST_OUTSCALE);
  for (int i = 0; i < P->D; ++i) perm[i] = i;
  for (int i = P->D - 1; i > 0; --i) {
    int j = (int)(syn_uniform(kp, (uint64_t)h * P->D + i) * (i + 1));
    if (j > i) j = i;
    int32_t t = perm[i]; perm[i] = perm[j]; perm[j] = t;
  }
  for (int k = 0; k < P->n_outlier; ++k) {
    ch[k] = perm[k];
    scale[k] = P->out_lo + (P->out_hi - P->out_lo) * syn_uniform(ks, (uint64_t)h * 64 + k);
  }
}

static inline uint64_t tok_ctr(int b, int p, int h) {
  return (((uint64_t)b << 32) + (uint64_t)(uint32_t)p) * 256u + (uint64_t)h;
}

/* Center table tab[h][c][d] for one sequence b (base mixture plus the per-sample offset). */
static void center_table(const synth_params* P, int kv, int b, double* tab) {
  int nc = kv ? P->ncv : P->nck;
  uint64_t kc = syn_key(P->seed, kv ? ST_CENTER_V : ST_CENTER_K);
  uint64_t ks = syn_key(P->seed, kv ? ST_SAMPLE_V : ST_SAMPLE_K);
  for (int h = 0; h < P->Hkv; ++h)
    for (int c = 0; c < nc; ++c)
      for (int d = 0; d < P->D; ++d) {
        uint64_t idx = ((uint64_t)h * nc + c) * P->D + d;
        double v = syn_normal(kc, idx);
        if (P->sample_sigma != 0.0) {
          uint64_t sidx = (((uint64_t)b * P->Hkv + h) * nc + c) * P->D + d;
          v += P->sample_sigma * syn_normal(ks, sidx);
        }
        tab[idx] = v;
      }
}

/* Drift directions u[h][c][d] ~ N(0, I). */
static void drift_table(const synth_params* P, int kv, double* tab) {
  int nc = kv ? P->ncv : P->nck;
  uint64_t kd = syn_key(P->seed, kv ? ST_DRIFT_V : ST_DRIFT_K);
  for (uint64_t i = 0; i < (uint64_t)P->Hkv * nc * P->D; ++i) tab[i] = syn_normal(kd, i);
}

/*
 * Generate K and V for sequences [b0, b1) and positions [p0, p1) into
 * out_k / out_v laid out [b1-b0][p1-p0][Hkv][D] as fp16/bf16 bit patterns.
 * Either output may be NULL.  Returns 0, or -1 on a size the generator does
 * not support (D > 1024, Hkv > 64, more than 64 outliers).
 */
int synth_kv(const synth_params* P, int32_t b0, int32_t b1, int32_t p0, int32_t p1,
             uint16_t* out_k, uint16_t* out_v) {
  const int D = P->D, H = P->Hkv;
  if (D > 1024 || D % 2 || H > 64 || P->n_outlier > 64 || P->n_outlier > D) return -1;
  const int64_t np = p1 - p0;
  int32_t och[64][64];
  double osc[64][64];
  for (int h = 0; h < H; ++h) outlier_channels(P, h, och[h], osc[h]);
  uint64_t kck = syn_key(P->seed, ST_CHOICE_K), kcv = syn_key(P->seed, ST_CHOICE_V);
  uint64_t knk = syn_key(P->seed, ST_NOISE_K), knv = syn_key(P->seed, ST_NOISE_V);
  size_t tk = (size_t)H * P->nck * D, tv = (size_t)H * P->ncv * D;
  double* cen_k = (double*)malloc(tk * sizeof(double));
  double* cen_v = (double*)malloc(tv * sizeof(double));
  double* dr_k = (double*)calloc(tk, sizeof(double));
  double* dr_v = (double*)calloc(tv, sizeof(double));
  if (!cen_k || !cen_v || !dr_k || !dr_v) { free(cen_k); free(cen_v); free(dr_k); free(dr_v); return -2; }
  if (P->drift_start >= 0) { drift_table(P, 0, dr_k); drift_table(P, 1, dr_v); }

  for (int b = b0; b < b1; ++b) {
    if (b == b0 || P->sample_sigma != 0.0) { center_table(P, 0, b, cen_k); center_table(P, 1, b, cen_v); }
#pragma omp parallel for schedule(static)
    for (int64_t pi = 0; pi < np; ++pi) {
      int p = (int)(p0 + pi);
      double row[1024], cs[512], sn[512];
      double blk = 0.0;
      if (P->drift_start >= 0 && p >= P->drift_start)
        blk = P->drift_step * (double)((p - P->drift_start) / P->drift_block);
      if (P->rope) {
        for (int i = 0; i < D / 2; ++i) {
          double th = (double)p * pow(P->rope_base, -(double)i / (double)(D / 2));
          cs[i] = cos(th);
          sn[i] = sin(th);
        }
      }
      for (int h = 0; h < H; ++h) {
        uint64_t tc = tok_ctr(b, p, h);
        size_t off = ((((size_t)(b - b0) * np) + pi) * H + h) * D;
        if (out_k) {
          int c = (int)(syn_uniform(kck, tc) * P->nck);
          if (c >= P->nck) c = P->nck - 1;
          const double* cen = cen_k + ((size_t)h * P->nck + c) * D;
          const double* dr = dr_k + ((size_t)h * P->nck + c) * D;
          for (int d = 0; d < D; ++d)
            row[d] = cen[d] + blk * dr[d] + P->sigma_k * syn_normal(knk, tc * D + d);
          for (int k = 0; k < P->n_outlier; ++k) row[och[h][k]] *= osc[h][k];
          if (P->rope) {
            for (int i = 0; i < D / 2; ++i) {
              double a = row[i], bb = row[i + D / 2];
              row[i] = a * cs[i] - bb * sn[i];
              row[i + D / 2] = a * sn[i] + bb * cs[i];
            }
          }
          for (int d = 0; d < D; ++d) out_k[off + d] = to_dtype(row[d], P->dtype);
        }
        if (out_v) {
          int c = (int)(syn_uniform(kcv, tc) * P->ncv);
          if (c >= P->ncv) c = P->ncv - 1;
          const double* cen = cen_v + ((size_t)h * P->ncv + c) * D;
          const double* dr = dr_v + ((size_t)h * P->ncv + c) * D;
          for (int d = 0; d < D; ++d)
            row[d] = cen[d] + blk * dr[d] + P->sigma_v * syn_normal(knv, tc * D + d);
          for (int d = 0; d < D; ++d) out_v[off + d] = to_dtype(row[d], P->dtype);
        }
      }
    }
  }
  free(cen_k); free(cen_v); free(dr_k); free(dr_v);
  return 0;
}

/* Decode queries q[b][hq][d] ~ N(0,1) for one step, as fp16/bf16 bits, sequences [b0, b1). */
void synth_q(uint64_t seed, int32_t step, int32_t B, int32_t b0, int32_t b1, int32_t Hq, int32_t D,
             int32_t dtype, uint16_t* out) {
  uint64_t kq = syn_key(seed, ST_Q);
  for (int b = b0; b < b1; ++b)
    for (int h = 0; h < Hq; ++h)
      for (int d = 0; d < D; ++d) {
        uint64_t i = (((uint64_t)step * B + b) * Hq + h) * D + d;
        out[((size_t)(b - b0) * Hq + h) * D + d] = to_dtype(syn_normal(kq, i), dtype);
      }
}

/* Raw access for tests of the generator itself. */
double synth_uniform(uint64_t seed, uint64_t stream, uint64_t ctr) {
  return syn_uniform(syn_key(seed, stream), ctr);
}
double synth_normal(uint64_t seed, uint64_t stream, uint64_t i) {
  return syn_normal(syn_key(seed, stream), i);
}
void synth_outliers(const synth_params* P, int32_t h, int32_t* ch, double* scale) {
  outlier_channels(P, h, ch, scale);
}
