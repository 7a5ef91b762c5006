// Prefill pattern mining: Lloyd k-means under the Euclidean metric, one
// independent problem per (pattern set, KV head) ("PatternKV", Section 3.1,
// Eq. 4, and the GPU-parallel KMeans of Section 3.4), optionally after fitting
// the KVarN pre-transform (Hadamard rotation + 3 alternating row / column std
// normalisation passes).
//
// Numerics: squared distances in float64 accumulated over channels 0..127 in
// order (ties to the lowest index), centroid sums in float64, centroid =
// fp32 rounding of the float64 mean, empty clusters keep their pattern.
#include <algorithm>

#include <cuda.h>
#include <cudaTypedefs.h>

#include "kvq_common.cuh"
#include "kvq_internal.h"

namespace kvq {

namespace {

constexpr int kFitPasses = 3;
constexpr int kFitChunk = 1024;  // tokens per block of a fit pass: the fixed order of the column sums
constexpr int kFitWarps = 8;

struct MineWs {
  int32_t* status;  // device status word (KVQ_DEV_* bits), at offset 0 of the workspace
  double* sums;     // [NP][P][128]
  uint32_t* cnt;    // [NP][P]
  int32_t* assign;  // [NP][n]
  float* xsq;       // [NP][n] |x|^2 of every token (the tcgen05 assignment's cache)
  int32_t* amb;     // [NP][n] tokens the tcgen05 assignment left undecided
  uint32_t* ambc;   // [NP][n][2] their candidate patterns (8 bytes: up to 8 indices)
  uint8_t* ambn;    // [NP][n] candidates listed (255: more than 8, every pattern is checked)
  int32_t* amb_cnt; // [NP]
  float* y;         // [NP][n][128] (transform only)
  double* rrow;     // [2][NP][n] reciprocal of each row's running divisor product, one buffer per pass parity
  double* colpart;  // [NP][fit chunks][2][128] per-chunk shifted column sums and sums of squares
  double* colscale; // [NP][128]  running product of column divisors
  double* cinv;     // [NP][128]  its reciprocal
  double* accpart;  // [NP][sum chunks][P][128] per-CTA cluster sums of the fp32 rows (transform only)
};

__host__ __device__ inline size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

// Cluster-sum CTAs per problem for the fp32 (pre-transformed) rows, whose float64 sums depend on
// the order of the additions: each CTA writes its own partials, which the update adds in CTA
// order, so the result is the same on every run.  A fixed CTA budget (two per SM of a 148-SM
// part) keeps the workspace independent of the device.
constexpr int kAccF32Ctas = 296;
inline int64_t fit_chunks(int64_t n) { return (n + kFitChunk - 1) / kFitChunk; }
inline int accum_f32_chunks(int64_t n, int NP, int P) {
  const int slices = P <= 64 ? 1 : (P <= 128 ? 2 : 4);
  const int64_t ntiles = (n + 127) / 128;
  return (int)std::max<int64_t>(1, std::min<int64_t>(ntiles, std::max(1, kAccF32Ctas / (slices * NP))));
}

inline MineWs carve(void* ws, int64_t n, int NP, int P, int transform, int32_t* assign_out) {
  uint8_t* p = (uint8_t*)ws;
  MineWs w{};
  w.status = (int32_t*)p; p += 256;
  w.sums = (double*)p; p += align256((size_t)NP * P * kD * sizeof(double));
  w.cnt = (uint32_t*)p; p += align256((size_t)NP * P * sizeof(uint32_t));
  if (assign_out) w.assign = assign_out;
  else { w.assign = (int32_t*)p; p += align256((size_t)NP * n * sizeof(int32_t)); }
  w.xsq = (float*)p; p += align256((size_t)NP * n * sizeof(float));
  w.amb = (int32_t*)p; p += align256((size_t)NP * n * sizeof(int32_t));
  w.ambc = (uint32_t*)p; p += align256((size_t)NP * n * 2 * sizeof(uint32_t));
  w.ambn = (uint8_t*)p; p += align256((size_t)NP * n);
  w.amb_cnt = (int32_t*)p; p += align256((size_t)NP * sizeof(int32_t));
  if (transform) {
    w.y = (float*)p; p += align256((size_t)NP * n * kD * sizeof(float));
    w.rrow = (double*)p; p += align256((size_t)2 * NP * n * sizeof(double));
    w.colpart = (double*)p; p += align256((size_t)NP * fit_chunks(n) * 2 * kD * sizeof(double));
    w.colscale = (double*)p; p += align256((size_t)NP * kD * sizeof(double));
    w.cinv = (double*)p; p += align256((size_t)NP * kD * sizeof(double));
    w.accpart = (double*)p; p += align256((size_t)NP * accum_f32_chunks(n, NP, P) * P * kD * sizeof(double));
  }
  return w;
}

struct Src {
  const uint16_t* x;
  int dtype;
  int64_t n, ts, hs, ss;
  int heads;
  const float* y;  // transformed rows, or null
  __device__ __forceinline__ float at(int prob, int64_t i, int d) const {
    if (y) return y[((size_t)prob * n + i) * kD + d];
    int set = prob / heads, h = prob % heads;
    return load_elem(x + set * ss + i * ts + h * hs + d, dtype);
  }
};

// ---- pre-transform fit ------------------------------------------------------
//
// Three passes of (row normalisation, column std) over v = fwht(x) (KVarN's dual-axis fit), with
// the rotated rows never stored: pass p recomputes each row as v_p = fwht(x) * (1 / C_p) *
// (1 / R_{p-1}) (C_p: product of the earlier passes' column divisors, R_{p-1}: of the row's own
// earlier divisors, kept as its reciprocal), takes its population std r_p (mean first, then
// squared deviations), and
// adds w = v_p / r_p, shifted by row 0's w, into per-column sums and sums of squares; the
// column std is sqrt(S2 / n - (S1 / n)^2) of those shifted values.  float64 throughout; the
// products and reciprocals stand for the sequential divisions of the definition, a few ulps
// apart.  Each block takes a fixed chunk of tokens and writes its partial sums, which the
// finish kernel adds in chunk order, so the fit is the same on every run.

// warp: R rows' normalised values w (this lane's channels lane + 32 k) and the reciprocals of
// their std, the rows' steps interleaved (each row's operations as for one row alone).  rin:
// the rows' running reciprocal divisors of the earlier passes, or null.
template <int R>
__device__ __forceinline__ void fit_rows_eval(const Src& s, int prob, const int64_t (&i)[R], const double (&ci)[4],
                                              const double* rin, int lane, double (&w)[R][4], double (&ri)[R]) {
  float v[R][4];
#pragma unroll
  for (int q = 0; q < R; ++q)
#pragma unroll
    for (int k = 0; k < 4; ++k) v[q][k] = s.at(prob, i[q], lane + 32 * k);
  // the butterfly of fwht_warp, row by row within each stage
#pragma unroll
  for (int h = 1; h < 32; h <<= 1)
#pragma unroll
    for (int q = 0; q < R; ++q)
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float o = __shfl_xor_sync(kFull, v[q][k], h);
        v[q][k] = (lane & h) ? __fsub_rn(o, v[q][k]) : __fadd_rn(v[q][k], o);
      }
  double u[R][4], m[R], sq[R];
#pragma unroll
  for (int q = 0; q < R; ++q) {
    const float a0 = v[q][0], b0 = v[q][1], a1 = v[q][2], b1 = v[q][3];
    const float t0 = __fadd_rn(a0, b0), t1 = __fsub_rn(a0, b0), t2 = __fadd_rn(a1, b1), t3 = __fsub_rn(a1, b1);
    const float f[4] = {__fadd_rn(t0, t2), __fadd_rn(t1, t3), __fsub_rn(t0, t2), __fsub_rn(t1, t3)};
    const double rr = rin ? rin[i[q]] : 1.0;
#pragma unroll
    for (int k = 0; k < 4; ++k) u[q][k] = (double)f[k] * ci[k] * rr;
    m[q] = (u[q][0] + u[q][1]) + (u[q][2] + u[q][3]);
  }
#pragma unroll
  for (int o = 16; o; o >>= 1)
#pragma unroll
    for (int q = 0; q < R; ++q) m[q] += __shfl_xor_sync(kFull, m[q], o);
#pragma unroll
  for (int q = 0; q < R; ++q) {
    const double mean = m[q] / 128.0;
    sq[q] = 0.0;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const double t = u[q][k] - mean;
      sq[q] += t * t;
    }
  }
#pragma unroll
  for (int o = 16; o; o >>= 1)
#pragma unroll
    for (int q = 0; q < R; ++q) sq[q] += __shfl_xor_sync(kFull, sq[q], o);
#pragma unroll
  for (int q = 0; q < R; ++q) {
    double r = sqrt(sq[q] / 128.0);
    if (r == 0.0) r = 1.0;
    ri[q] = 1.0 / r;
#pragma unroll
    for (int k = 0; k < 4; ++k) w[q][k] = u[q][k] * ri[q];
  }
}

// One fit pass over the tokens of chunk blockIdx.x of problem blockIdx.y; warp w takes rows
// i0 + w, i0 + w + kFitWarps, ... (one at a time: interleaving four rows per warp measured
// slower, its registers halving the warps per SM).  rin: the previous pass's reciprocal row
// products (null in pass 0); cinv: 1 / C_p (null in pass 0).
constexpr int kFitRows = 1;
__global__ void __launch_bounds__(kFitWarps * 32, 4) fit_pass_kernel(Src s, const double* __restrict__ cinv,
                                                                  const double* __restrict__ rin,
                                                                  double* __restrict__ rout,
                                                                  double* __restrict__ colpart) {
  __shared__ double shift[kD];
  __shared__ double red[kFitWarps][2][kD];
  const int prob = blockIdx.y, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t i0 = (int64_t)blockIdx.x * kFitChunk, i1 = min(s.n, i0 + kFitChunk);
  double ci[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) ci[k] = cinv ? cinv[prob * kD + lane + 32 * k] : 1.0;
  const double* rp = rin ? rin + (size_t)prob * s.n : nullptr;
  double* ro = rout + (size_t)prob * s.n;
  if (warp == 0) {
    const int64_t z[1] = {0};
    double w0[1][4], r0[1];
    fit_rows_eval<1>(s, prob, z, ci, rp, lane, w0, r0);
#pragma unroll
    for (int k = 0; k < 4; ++k) shift[lane + 32 * k] = w0[0][k];
  }
  __syncthreads();
  double sh[4], s1[4] = {0.0, 0.0, 0.0, 0.0}, s2[4] = {0.0, 0.0, 0.0, 0.0};
#pragma unroll
  for (int k = 0; k < 4; ++k) sh[k] = shift[lane + 32 * k];
  for (int64_t b = i0 + warp; b < i1; b += kFitRows * kFitWarps) {
    int64_t ii[kFitRows];
#pragma unroll
    for (int q = 0; q < kFitRows; ++q) ii[q] = min(b + (int64_t)q * kFitWarps, i1 - 1);  // past the end: a repeat, unused
    double w[kFitRows][4], ri[kFitRows];
    fit_rows_eval<kFitRows>(s, prob, ii, ci, rp, lane, w, ri);
#pragma unroll
    for (int q = 0; q < kFitRows; ++q) {
      if (b + (int64_t)q * kFitWarps >= i1) break;
      if (lane == 0) ro[ii[q]] = rp ? rp[ii[q]] * ri[q] : ri[q];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const double t = w[q][k] - sh[k];
        s1[k] += t;
        s2[k] += t * t;
      }
    }
  }
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    red[warp][0][lane + 32 * k] = s1[k];
    red[warp][1][lane + 32 * k] = s2[k];
  }
  __syncthreads();
  if (threadIdx.x < kD) {
    const int d = threadIdx.x;
    double a = 0.0, c = 0.0;
    for (int q = 0; q < kFitWarps; ++q) {
      a += red[q][0][d];
      c += red[q][1][d];
    }
    double* out = colpart + ((size_t)prob * gridDim.x + blockIdx.x) * 2 * kD;
    out[d] = a;
    out[kD + d] = c;
  }
}

// Column std of the pass from the chunk partials (added in chunk order); C_{p+1} = C_p * std
// (1 where the std is 0) and its reciprocal.  One block of 128 threads per problem.
__global__ void fit_finish_kernel(int64_t n, int chunks, const double* __restrict__ colpart,
                                  double* __restrict__ colscale, double* __restrict__ cinv, int first) {
  const int prob = blockIdx.x, d = threadIdx.x;
  double a = 0.0, b = 0.0;
  const double* q = colpart + (size_t)prob * chunks * 2 * kD + d;
  int c = 0;
  for (; c + 8 <= chunks; c += 8) {  // eight chunks' loads in flight, added in order
    double qa[8], qb[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      qa[e] = q[(size_t)(c + e) * 2 * kD];
      qb[e] = q[(size_t)(c + e) * 2 * kD + kD];
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      a += qa[e];
      b += qb[e];
    }
  }
  for (; c < chunks; ++c) {
    a += q[(size_t)c * 2 * kD];
    b += q[(size_t)c * 2 * kD + kD];
  }
  const double m = a / (double)n;
  double var = b / (double)n - m * m;
  if (var < 0.0) var = 0.0;
  double sd = sqrt(var);
  if (sd == 0.0) sd = 1.0;
  const double C = (first ? 1.0 : colscale[prob * kD + d]) * sd;
  colscale[prob * kD + d] = C;
  cinv[prob * kD + d] = 1.0 / C;
}

__global__ void fit_output_kernel(const double* colscale, float* colscale_out) {
  const int prob = blockIdx.x, d = threadIdx.x;
  colscale_out[prob * kD + d] = (float)colscale[prob * kD + d];
}

// y = transform(x) with the fitted factors; warp per token.
__global__ void apply_kernel(Src s, const float* colscale_out, float* y) {
  const int prob = blockIdx.y, lane = threadIdx.x & 31;
  const int64_t i = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (i >= s.n) return;
  float v[4], r;
#pragma unroll
  for (int k = 0; k < 4; ++k) v[k] = s.at(prob, i, lane + 32 * k);
  transform_row_warp(v, colscale_out + prob * kD, r, lane);
  float* row = y + ((size_t)prob * s.n + i) * kD;
#pragma unroll
  for (int k = 0; k < 4; ++k) row[lane + 32 * k] = v[k];
}

// ---- Lloyd -------------------------------------------------------------------

__global__ void mine_init_kernel(Src s, int P, float* M) {
  const int prob = blockIdx.y, j = blockIdx.x, d = threadIdx.x;
  int64_t src = ((int64_t)j * s.n) / P;
  M[((size_t)prob * P + j) * kD + d] = s.at(prob, src, d);
}

// One thread per token: nearest pattern by float64 squared distance (channels in order).
__global__ void __launch_bounds__(128) mine_assign_kernel(Src s, int P, const float* __restrict__ M,
                                                          int32_t* __restrict__ assign) {
  extern __shared__ __align__(16) uint8_t smraw[];
  float* Ms = reinterpret_cast<float*>(smraw);
  const int prob = blockIdx.y;
  const float* Mp = M + (size_t)prob * P * kD;
  for (int i = threadIdx.x; i < P * kD; i += blockDim.x) Ms[i] = Mp[i];
  __syncthreads();
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= s.n) return;
  float xr[kD];
#pragma unroll
  for (int d = 0; d < kD; ++d) xr[d] = s.at(prob, i, d);
  double best = 0.0;
  int bj = 0;
  for (int j = 0; j < P; ++j) {
    const float* m = Ms + j * kD;
    double acc = 0.0;
#pragma unroll
    for (int d = 0; d < kD; ++d) {
      double t = __dsub_rn((double)xr[d], (double)m[d]);
      acc = __dadd_rn(acc, __dmul_rn(t, t));
    }
    if (j == 0 || acc < best) { best = acc; bj = j; }
  }
  assign[(size_t)prob * s.n + i] = bj;
}

// ---- tensor-core assignment with exact certification ------------------------------
//
// Scores e_j = |m_j|^2 - 2 x.m_j come from bf16 m16n8k16 MMAs.  Every pattern value is
// split into bf16 terms hi + mid (the remainder below them is at most 2^-16 |m|); inputs
// are exact in one bf16 term (bf16 input) or split into hi + lo (fp16 input exactly,
// fp32 pre-transformed rows to 2^-16).  Each product of terms (x_a, m_b) runs in its own
// fp32 accumulator chain of 8 MMAs (x_lo . m_mid, below 2^-16 |x| |m|, is left out), and
// the chains are added at the end.  If a tensor core truncated each MMA's sum to 22 bits
// of its largest term, a chain would be off by at most 8 * 17 * 2^-22 |x_a| |m_b|; with
// the terms left out and the final adds, |e_hat_j - e_j| stays below 2^-12.6 |x| |m_j|
// plus the fp32 rounding of |m_j|^2 and of the final combination, which
// E_j = 2^-12 |x| |m_j| + 2^-20 (|x|^2 + |m_j|^2) covers.
//
// With U = min_j (e_hat_j + E_j), the float64 argmin can only be a pattern with
// e_hat_j - E_j <= U + delta.  A token whose best two scores are more than 2 max_j E_j +
// delta apart is decided at once; the others (well under 1 %) are decided by
// recomputing float64 distances of the candidates exactly as the sequential reference
// does.
//
// The MMA k index runs over channels in the order pi(kp, tig, e) = 8 (4 kp + tig) + e for
// k-step 2 kp + (e >> 2) ... so that every lane's A operands of a pair of k-steps are 8
// consecutive channels (one 16-byte load) and its B operands 8 consecutive bf16 values of
// a pattern row (one 16-byte shared load).  A dot product does not depend on the order of k.
constexpr int kMmaMaxP = 128;
constexpr int kMmaWarps = 4;
constexpr int kBLd = kD + 32;  // bf16 row of a pattern split: 320 B = 64 mod 128, conflict-free 16-byte loads

__device__ __forceinline__ void mma_bf16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// bf16 hi / lo parts of two fp32 values by truncation (hi + lo keeps 16 significant bits).
__device__ __forceinline__ void split_trunc(float x0, float x1, uint32_t& hi, uint32_t& lo) {
  const uint32_t u0 = __float_as_uint(x0), u1 = __float_as_uint(x1);
  hi = __byte_perm(u0, u1, 0x7632);
  const float r0 = x0 - __uint_as_float(u0 & 0xFFFF0000u), r1 = x1 - __uint_as_float(u1 & 0xFFFF0000u);
  lo = __byte_perm(__float_as_uint(r0), __float_as_uint(r1), 0x7632);
}

// Smallest score, its pattern and the second smallest score.  A thread sees its patterns
// in increasing order, so a strict comparison keeps the lowest index among equal scores.
struct Top2 {
  float m1, m2;
  int j1;
};
__device__ __forceinline__ void top2_add(Top2& t, float e, int j) {
  const bool lt = e < t.m1;
  t.m2 = lt ? t.m1 : fminf(t.m2, e);
  t.j1 = lt ? j : t.j1;
  t.m1 = lt ? e : t.m1;
}
__device__ __forceinline__ void top2_merge_xor(Top2& t, int mask) {
  const float om1 = __shfl_xor_sync(kFull, t.m1, mask), om2 = __shfl_xor_sync(kFull, t.m2, mask);
  const int oj = __shfl_xor_sync(kFull, t.j1, mask);
  const float lo2 = fminf(t.m2, om2);
  if (om1 < t.m1 || (om1 == t.m1 && oj < t.j1)) { t.m2 = fminf(t.m1, lo2); t.m1 = om1; t.j1 = oj; }
  else t.m2 = fminf(om1, lo2);
}

// Input kinds: 0 = bf16 rows (one exact bf16 term), 1 = fp16 rows, 2 = fp32 pre-transformed rows.
// A warp tile's raw row data (8 consecutive channels per load) is fetched one tile ahead.
template <int KIND>
struct RawRows {
  static constexpr int kMt = KIND == 0 ? 2 : 1;
  static constexpr int kW = KIND == 2 ? 2 : 1;  // 16-byte words per 8 channels
  uint4 u[kMt][2][4][kW];
};

template <int KIND>
__device__ __forceinline__ void load_raw(const Src& s, int prob, int64_t t0, int gq, int tig, RawRows<KIND>& R) {
  constexpr int kMt = RawRows<KIND>::kMt;
  const int set = prob / s.heads, h = prob % s.heads;
#pragma unroll
  for (int mt = 0; mt < kMt; ++mt)
#pragma unroll
    for (int rh = 0; rh < 2; ++rh) {
      const int64_t i = t0 + 16 * mt + 8 * rh + gq;
#pragma unroll
      for (int kp = 0; kp < 4; ++kp) {
        const int c = 8 * (4 * kp + tig);
        if (i < s.n) {
          if constexpr (KIND == 2) {
            const uint4* p = reinterpret_cast<const uint4*>(s.y + ((size_t)prob * s.n + i) * kD + c);
            R.u[mt][rh][kp][0] = p[0];
            R.u[mt][rh][kp][1] = p[1];
          } else {
            R.u[mt][rh][kp][0] = __ldg(reinterpret_cast<const uint4*>(s.x + set * s.ss + i * s.ts + h * s.hs + c));
          }
        } else {
#pragma unroll
          for (int k = 0; k < RawRows<KIND>::kW; ++k) R.u[mt][rh][kp][k] = make_uint4(0u, 0u, 0u, 0u);
        }
      }
    }
}

// MMA operand words (bf16 pairs, lower channel in the low half) of 8 raw values, and the
// sum of their squares.
template <int KIND>
__device__ __forceinline__ void to_operands(const uint4 (&raw)[RawRows<KIND>::kW], uint32_t (&hi)[4],
                                            uint32_t (&lo)[4], float& nrm) {
  if constexpr (KIND == 2) {
    const float v[8] = {__uint_as_float(raw[0].x), __uint_as_float(raw[0].y), __uint_as_float(raw[0].z),
                        __uint_as_float(raw[0].w), __uint_as_float(raw[1].x), __uint_as_float(raw[1].y),
                        __uint_as_float(raw[1].z), __uint_as_float(raw[1].w)};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      split_trunc(v[2 * q], v[2 * q + 1], hi[q], lo[q]);
      nrm = fmaf(v[2 * q], v[2 * q], nrm);
      nrm = fmaf(v[2 * q + 1], v[2 * q + 1], nrm);
    }
  } else {
    const uint32_t w[4] = {raw[0].x, raw[0].y, raw[0].z, raw[0].w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      float v0, v1;
      if constexpr (KIND == 0) {
        hi[q] = w[q];
        v0 = __uint_as_float(w[q] << 16);
        v1 = __uint_as_float(w[q] & 0xFFFF0000u);
      } else {
        v0 = __half2float(__ushort_as_half((uint16_t)(w[q] & 0xffff)));
        v1 = __half2float(__ushort_as_half((uint16_t)(w[q] >> 16)));
        split_trunc(v0, v1, hi[q], lo[q]);
      }
      nrm = fmaf(v0, v0, nrm);
      nrm = fmaf(v1, v1, nrm);
    }
  }
}

template <int KIND>
__global__ void __launch_bounds__(kMmaWarps * 32, 2) mine_assign_mma_kernel(Src s, int P, const float* __restrict__ M,
                                                                             int32_t* __restrict__ assign) {
  constexpr int NA = KIND == 0 ? 1 : 2;  // bf16 terms of an input value
  constexpr int NC = NA + 1;             // accumulator chains: (hi,hi), (hi,mid), (lo,hi)
  constexpr int kMt = NA == 1 ? 2 : 1;   // 16-token m-tiles per warp tile
  constexpr int kTok = 16 * kMt;         // tokens per warp tile
  extern __shared__ __align__(16) uint8_t smraw[];
  uint8_t* sm = smraw;
  const int prob = blockIdx.y;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int gq = lane >> 2, tig = lane & 3;
  const int Pp = (P + 7) & ~7;  // padded to whole n-tiles
  __nv_bfloat16* Bs = reinterpret_cast<__nv_bfloat16*>(sm);                       // [2][Pp][kBLd]
  float* mnorm = reinterpret_cast<float*>(sm + (size_t)2 * Pp * kBLd * 2);           // [Pp] |m_j|
  float* msq = mnorm + Pp;                                                            // [Pp] |m_j|^2
  const int eld = Pp + 2;                                                             // even: aligned float2 rows
  float* escr = msq + Pp;                                                             // [warps][kTok][eld]
  float* xn = escr + kMmaWarps * kTok * eld;                                          // [warps][kTok] |x|^2
  float* gmax = xn + kMmaWarps * kTok;                                                // [2] max |m|, max |m|^2
  const float* Mp = M + (size_t)prob * P * kD;

  // pattern splits (natural channel order) and norms
  for (int i = threadIdx.x; i < Pp * kD; i += blockDim.x) {
    const int j = i / kD, d = i % kD;
    const float m = j < P ? Mp[(size_t)j * kD + d] : 0.f;
    const __nv_bfloat16 h = __float2bfloat16_rn(m);
    Bs[(0 * Pp + j) * kBLd + d] = h;
    Bs[(1 * Pp + j) * kBLd + d] = __float2bfloat16_rn(m - __bfloat162float(h));
  }
  if (threadIdx.x == 0) { gmax[0] = 0.f; gmax[1] = 0.f; }
  __syncthreads();
  for (int j = threadIdx.x; j < Pp; j += blockDim.x) {
    double acc = 0.0;
    if (j < P)
      for (int d = 0; d < kD; ++d) { const double m = Mp[(size_t)j * kD + d]; acc += m * m; }
    msq[j] = (float)acc;
    mnorm[j] = (float)(sqrt(acc) * (1.0 + 1e-6));
    atomicMax(reinterpret_cast<int*>(&gmax[0]), __float_as_int(mnorm[j]));
    atomicMax(reinterpret_cast<int*>(&gmax[1]), __float_as_int(msq[j] * (1.0f + 1e-6f)));
  }
  __syncthreads();
  const float nm_max = gmax[0], msq_max = gmax[1];

  float* esc = escr + warp * kTok * eld;
  float* xnw = xn + warp * kTok;
  const int64_t ntiles = (s.n + kTok - 1) / kTok;
  const int64_t tstep = (int64_t)gridDim.x * kMmaWarps;
  int64_t tile = (int64_t)blockIdx.x * kMmaWarps + warp;
  RawRows<KIND> raw;
  if (tile < ntiles) load_raw<KIND>(s, prob, tile * kTok, gq, tig, raw);
  for (; tile < ntiles; tile += tstep) {
    const int64_t t0 = tile * kTok;
    // A operands: rows gq (+8) of each m-tile, channels 8(4kp + tig) .. +7 for k-step pair kp
    uint32_t A[NA][kMt][2][4][4];  // [term][mt][row half][kp][reg]
    float nrm[kMt][2];
#pragma unroll
    for (int mt = 0; mt < kMt; ++mt)
#pragma unroll
      for (int rh = 0; rh < 2; ++rh) {
        nrm[mt][rh] = 0.f;
#pragma unroll
        for (int kp = 0; kp < 4; ++kp)
          to_operands<KIND>(raw.u[mt][rh][kp], A[0][mt][rh][kp], A[NA - 1][mt][rh][kp], nrm[mt][rh]);
      }
    // the next tile's rows are in flight while this one is scored
    if (tile + tstep < ntiles) load_raw<KIND>(s, prob, (tile + tstep) * kTok, gq, tig, raw);
#pragma unroll
    for (int mt = 0; mt < kMt; ++mt)
#pragma unroll
      for (int rh = 0; rh < 2; ++rh) {
        float v = nrm[mt][rh];
        v += __shfl_xor_sync(kFull, v, 1);
        v += __shfl_xor_sync(kFull, v, 2);
        nrm[mt][rh] = v;
        if (tig == 0) xnw[16 * mt + 8 * rh + gq] = v * (1.0f + 1e-6f);
      }
    Top2 top[kMt][2];
#pragma unroll
    for (int mt = 0; mt < kMt; ++mt)
#pragma unroll
      for (int rh = 0; rh < 2; ++rh) top[mt][rh] = Top2{INFINITY, INFINITY, 0};
    // scores, one n-tile (8 patterns) at a time
    for (int nt = 0; nt < Pp / 8; ++nt) {
      float acc[NC][kMt][4];
#pragma unroll
      for (int ch = 0; ch < NC; ++ch)
#pragma unroll
        for (int mt = 0; mt < kMt; ++mt) acc[ch][mt][0] = acc[ch][mt][1] = acc[ch][mt][2] = acc[ch][mt][3] = 0.f;
#pragma unroll
      for (int sp = 0; sp < 2; ++sp) {
        const __nv_bfloat16* brow = Bs + ((size_t)sp * Pp + 8 * nt + gq) * kBLd + 8 * tig;
#pragma unroll
        for (int kp = 0; kp < 4; ++kp) {
          const uint4 bv = *reinterpret_cast<const uint4*>(brow + 32 * kp);  // channels 8(4kp+tig)..+7
#pragma unroll
          for (int a = 0; a < NA; ++a) {
            if (a == 1 && sp == 1) continue;  // x_lo . m_mid: left out
            const int ch = a == 0 ? sp : 2;
#pragma unroll
            for (int mt = 0; mt < kMt; ++mt) {
              // k-step 2kp: channels +0..+3 -> (a0a1, a4a5) / (b0, b1); rows gq and gq+8 -> a0a1 / a2a3
              mma_bf16(acc[ch][mt], A[a][mt][0][kp][0], A[a][mt][1][kp][0], A[a][mt][0][kp][1], A[a][mt][1][kp][1],
                       bv.x, bv.y);
              mma_bf16(acc[ch][mt], A[a][mt][0][kp][2], A[a][mt][1][kp][2], A[a][mt][0][kp][3], A[a][mt][1][kp][3],
                       bv.z, bv.w);
            }
          }
        }
      }
#pragma unroll
      for (int mt = 0; mt < kMt; ++mt) {
        float dot[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          float v = acc[0][mt][q] + acc[1][mt][q];
          if constexpr (NC == 3) v += acc[2][mt][q];
          dot[q] = v;
        }
        const int j0 = 8 * nt + 2 * tig;
        const float e0 = msq[j0] - 2.0f * dot[0], e1 = msq[j0 + 1] - 2.0f * dot[1];
        const float e2 = msq[j0] - 2.0f * dot[2], e3 = msq[j0 + 1] - 2.0f * dot[3];
        *reinterpret_cast<float2*>(&esc[(16 * mt + gq) * eld + j0]) = make_float2(e0, e1);
        *reinterpret_cast<float2*>(&esc[(16 * mt + gq + 8) * eld + j0]) = make_float2(e2, e3);
        if (j0 < P) { top2_add(top[mt][0], e0, j0); top2_add(top[mt][1], e2, j0); }
        if (j0 + 1 < P) { top2_add(top[mt][0], e1, j0 + 1); top2_add(top[mt][1], e3, j0 + 1); }
      }
    }
    // gap test per row, then the exact path for the rows that fail it
    uint32_t need = 0;
#pragma unroll
    for (int mt = 0; mt < kMt; ++mt)
#pragma unroll
      for (int rh = 0; rh < 2; ++rh) {
        top2_merge_xor(top[mt][rh], 1);
        top2_merge_xor(top[mt][rh], 2);
        const float xsq = nrm[mt][rh] * (1.0f + 1e-6f), nx = sqrtf(xsq) * (1.0f + 1e-6f);
        const float Eb = 0x1p-12f * nx * nm_max + 0x1p-20f * (xsq + msq_max);
        const int64_t i = t0 + 16 * mt + 8 * rh + gq;
        const bool unique = top[mt][rh].m2 - top[mt][rh].m1 > 2.0f * Eb + 1e-9f * (xsq + msq_max);
        if (unique && tig == 0 && i < s.n) assign[(size_t)prob * s.n + i] = top[mt][rh].j1;
        if (!unique) need |= 1u << (16 * mt + 8 * rh + gq);
      }
    need = __reduce_or_sync(kFull, need);
    if (need) {
      __syncwarp();
      if (lane < kTok && ((need >> lane) & 1)) {
        const int64_t i = t0 + lane;
        if (i < s.n) {
          const float* e = esc + lane * eld;
          const float xsq = xnw[lane];
          const uint16_t* xrow = s.x ? s.x + (prob / s.heads) * s.ss + i * s.ts + (prob % s.heads) * s.hs : nullptr;
          const float nx = sqrtf(xsq) * (1.0f + 1e-6f);
          float U = INFINITY;
          for (int j = 0; j < P; ++j) U = fminf(U, e[j] + 0x1p-12f * nx * mnorm[j] + 0x1p-20f * (xsq + msq[j]));
          double bd = 0.0;
          int bj = 0;
          bool have = false;
          for (int j = 0; j < P; ++j) {
            const float E = 0x1p-12f * nx * mnorm[j] + 0x1p-20f * (xsq + msq[j]);
            if (!(e[j] - E <= U + 1e-9f * (xsq + msq[j]))) continue;
            // exact float64 distance, channels in order, as the sequential reference computes it;
            // the loads do not depend on the running sum, so they are issued well ahead of it
            const float* m = Mp + (size_t)j * kD;
            double acc = 0.0;
#pragma unroll 8
            for (int d = 0; d < kD; d += 4) {
              float xv[4];
              if constexpr (KIND == 2) {
                const float4 t4 = *reinterpret_cast<const float4*>(s.y + ((size_t)prob * s.n + i) * kD + d);
                xv[0] = t4.x; xv[1] = t4.y; xv[2] = t4.z; xv[3] = t4.w;
              } else {
                const uint2 u = __ldg(reinterpret_cast<const uint2*>(xrow + d));
                xv[0] = bits_to_float((uint16_t)(u.x & 0xffff), s.dtype);
                xv[1] = bits_to_float((uint16_t)(u.x >> 16), s.dtype);
                xv[2] = bits_to_float((uint16_t)(u.y & 0xffff), s.dtype);
                xv[3] = bits_to_float((uint16_t)(u.y >> 16), s.dtype);
              }
              const float4 m4 = __ldg(reinterpret_cast<const float4*>(m + d));
              const float mv[4] = {m4.x, m4.y, m4.z, m4.w};
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                const double t = __dsub_rn((double)xv[q], (double)mv[q]);
                acc = __dadd_rn(acc, __dmul_rn(t, t));
              }
            }
            if (!have || acc < bd) { bd = acc; bj = j; have = true; }
          }
          assign[(size_t)prob * s.n + i] = bj;
        }
      }
    }
    __syncwarp();
  }
}

size_t mine_mma_smem(int P, int KIND) {
  const int Pp = (P + 7) & ~7, kTok = KIND == 0 ? 32 : 16;
  return (size_t)2 * Pp * kBLd * 2 + 2 * Pp * 4 + (size_t)kMmaWarps * kTok * (Pp + 2) * 4 + kMmaWarps * kTok * 4 + 16;
}

// Per-cluster float64 sums and sizes in one streaming pass.  A CTA walks a contiguous run
// of 128-token tiles of one problem (and one channel slice).  One producer warp copies each
// tile with one TMA box (128 tokens x the slice's channels, row-major; completion counted in
// bytes on the stage's "full" mbarrier) into a ring of shared-memory stages, and before that
// groups the tile's rows by cluster (a counting sort through shared-memory counters and a
// warp scan: per stage an offset per cluster and the list of rows).  16 consumer warps each
// take every tile: warp w owns clusters w, w + 16, w + 32, ..., walks exactly their rows and
// adds them into float64 accumulators held in registers (lane l: channels E*l .. E*l + E - 1
// of the slice), then arrives on the stage's "empty" mbarrier.  A stage is refilled once all
// 16 warps are done with it, so fast warps run ahead instead of waiting at a block barrier.
// float64 sums of fp16 / bf16 values are exact, so the order of the additions does not change
// them and each CTA adds its totals to global memory with atomics.  float64 sums of fp32 rows
// (the pre-transformed input) round, so for them every step has a fixed order: the rows of a
// cluster are listed in token order (ranks from __match_any_sync, not from atomics), and each
// CTA writes its totals to its own slot of `part`, which the update adds in CTA order.  Every
// wait is bounded; on expiry KVQ_DEV_TIMEOUT goes to `status`, and the producer waits
// (bounded) for the copies it issued before the CTA exits.
constexpr int kAccWarps = 16;
constexpr int kAccT = 128;  // tokens per tile
constexpr uint32_t kAccSpinLimit = 1u << 24;

__device__ __forceinline__ uint32_t sa32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }
__device__ __forceinline__ void mb_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(sa32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void mb_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(sa32(bar)), "r"(bytes) : "memory");
}
__device__ __forceinline__ void mb_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(sa32(bar)) : "memory");
}
__device__ __forceinline__ bool mb_wait(uint64_t* bar, uint32_t parity) {
  for (uint32_t it = 0; it < kAccSpinLimit; ++it) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(sa32(bar)), "r"(parity)
        : "memory");
    if (ok) return true;
  }
  return false;
}
__device__ __forceinline__ void tma_load_4d(void* dst, const CUtensorMap* map, int c0, int c1, int c2, int c3,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4, %5}], "
      "[%6];" ::"r"(sa32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(sa32(bar))
      : "memory");
}
__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, int c0, int c1, int c2, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], "
      "[%5];" ::"r"(sa32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(sa32(bar))
      : "memory");
}

// x * 2^-896 as a float64 built from the bits of the bf16 value x in the low / high half of
// w: the bf16 sign, exponent and mantissa fields become the float64 sign, the low 8 bits of
// its exponent and the top of its mantissa, so every finite bf16 value (subnormals included,
// as float64 subnormals) maps exactly; float64 sums of these stay exact and the factor is
// undone once at the end.  Integer operations instead of a float conversion, whose unit runs
// at a fraction of the integer pipe's rate.  The fp16 forms give x * 2^-1008 (5-bit exponent
// field), the fp32 form x * 2^-896 (both words of the float64).
__device__ __forceinline__ double bf16lo_scaled(uint32_t w) {
  return __hiloint2double((int)(((w << 16) & 0x80000000u) | ((w << 13) & 0x0FFFE000u)), 0);
}
__device__ __forceinline__ double bf16hi_scaled(uint32_t w) {
  return __hiloint2double((int)((w & 0x80000000u) | ((w >> 3) & 0x0FFFE000u)), 0);
}
__device__ __forceinline__ double f16lo_scaled(uint32_t w) {
  return __hiloint2double((int)(((w << 16) & 0x80000000u) | ((w << 10) & 0x01FFFC00u)), 0);
}
__device__ __forceinline__ double f16hi_scaled(uint32_t w) {
  return __hiloint2double((int)((w & 0x80000000u) | ((w >> 6) & 0x01FFFC00u)), 0);
}
__device__ __forceinline__ double f32_scaled(uint32_t f) {
  return __hiloint2double((int)((f & 0x80000000u) | ((f & 0x7FFFFFFFu) >> 3)), (int)(f << 29));
}

// 16-bit rows and up to 4 clusters per warp: two CTAs per SM, each with a ring in half the
// shared memory (and registers for two); otherwise one
template <int CPW, int ES>
constexpr int accum_ctas_per_sm() { return ES == 2 && CPW <= 4 ? 2 : 1; }
template <int CPW, int RB, int ES>
constexpr int accum_stages() {
  return (200 * 1024 / accum_ctas_per_sm<CPW, ES>()) / (kAccT * RB) < 4
             ? (200 * 1024 / accum_ctas_per_sm<CPW, ES>()) / (kAccT * RB)
             : 4;
}

// CPW clusters per warp, E channels per lane (slice = 32 E channels), ES bytes per element
// (2: the fp16 / bf16 input, 4: the fp32 pre-transformed rows)
template <int CPW, int E, int ES>
__global__ void __launch_bounds__((kAccWarps + 1) * 32, accum_ctas_per_sm<CPW, ES>()) mine_accum_kernel(const __grid_constant__ CUtensorMap amap,
                                                                            Src s, int P,
                                                                            const int32_t* __restrict__ assign,
                                                                            double* __restrict__ sums,
                                                                            uint32_t* __restrict__ cnt,
                                                                            double* __restrict__ part,
                                                                            int32_t* __restrict__ status) {
  constexpr int CW = 32 * E, RB = CW * ES;  // channels and bytes of a staged row
  constexpr int kStages = accum_stages<CPW, RB, ES>();
  constexpr int kStageBytes = kAccT * RB;
  constexpr int kOff = kAccWarps * CPW + 1;  // cluster offsets of a stage's member list
  extern __shared__ __align__(16) uint8_t smraw[];
  uint64_t* full = reinterpret_cast<uint64_t*>(smraw + (size_t)kStages * kStageBytes);
  uint64_t* empty = full + kStages;
  int32_t* offs = reinterpret_cast<int32_t*>(empty + kStages);  // [kStages][kOff]
  int32_t* lists = offs + kStages * kOff;                        // [kStages][kAccT] rows by cluster
  int32_t* counts = lists + kStages * kAccT;                     // [kOff] producer scratch
  const int slice = blockIdx.y, prob = blockIdx.z;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t ntiles = (s.n + kAccT - 1) / kAccT;
  const int64_t per = (ntiles + gridDim.x - 1) / gridDim.x;
  const int64_t k0 = (int64_t)blockIdx.x * per, k1 = min(ntiles, k0 + per);
  if (k0 >= k1) {
    if constexpr (ES == 4) {  // no tiles: this CTA's partial slot is zero
      double* gp = part + ((size_t)prob * gridDim.x + blockIdx.x) * P * kD;
      for (int i = threadIdx.x; i < P * CW; i += blockDim.x) gp[(size_t)(i / CW) * kD + slice * CW + i % CW] = 0.0;
    }
    return;
  }
  const int nt = (int)(k1 - k0);
  const int set = prob / s.heads, h = prob % s.heads;
  const int32_t* a = assign + (size_t)prob * s.n;
  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mb_init(&full[i], 1);
      mb_init(&empty[i], kAccWarps);
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();

  if (warp == kAccWarps) {
    // ---- producer: rows of tile k into stage k % kStages once every consumer left it.  The
    // tile's assignments are loaded one tile ahead (their latency overlaps the previous tile).
    int last = -1;  // newest tile whose copy was issued
    int aj_next[kAccT / 32];
#pragma unroll
    for (int q = 0; q < kAccT / 32; ++q) {
      const int64_t i = (int64_t)(k0 * kAccT) + 32 * q + lane;
      aj_next[q] = i < s.n ? __ldg(a + i) : -1;
    }
    for (int k = 0; k < nt; ++k) {
      const int st = k % kStages;
      bool ok = true;
      if (k >= kStages) ok = mb_wait(&empty[st], (uint32_t)(((k / kStages) - 1) & 1));
      if (!__all_sync(kFull, ok)) {  // consumers time out on the full barrier in turn
        if (lane == 0) set_status(status, KVQ_DEV_TIMEOUT);
        break;
      }
      const int tb = (int)((k0 + k) * kAccT);
      // the tile's rows grouped by cluster (counting sort): offs[st][j] .. offs[st][j + 1] of
      // lists[st] are the rows of cluster j
      int aj[kAccT / 32], pos[kAccT / 32];
#pragma unroll
      for (int q = 0; q < kAccT / 32; ++q) {
        aj[q] = aj_next[q];
        const int64_t i = (int64_t)tb + kAccT + 32 * q + lane;  // the next tile's rows
        aj_next[q] = (k + 1 < nt && i < s.n) ? __ldg(a + i) : -1;
      }
      for (int i = lane; i < P; i += 32) counts[i] = 0;
      __syncwarp();
      if constexpr (ES == 4) {
        // fixed order: a cluster's rows in token order (rank among equal lanes, then later q)
#pragma unroll
        for (int q = 0; q < kAccT / 32; ++q) {
          const unsigned peers = __match_any_sync(kFull, aj[q]);
          const int leader = __ffs(peers) - 1;
          int base = 0;
          if (aj[q] >= 0 && lane == leader) base = atomicAdd(&counts[aj[q]], __popc(peers));
          base = __shfl_sync(kFull, base, leader);
          pos[q] = aj[q] >= 0 ? base + __popc(peers & ((1u << lane) - 1u)) : -1;
        }
      } else {
#pragma unroll
        for (int q = 0; q < kAccT / 32; ++q) pos[q] = aj[q] >= 0 ? atomicAdd(&counts[aj[q]], 1) : -1;
      }
      __syncwarp();
      {
        // exclusive scan: lane l owns clusters [l * per, (l + 1) * per)
        const int per = (P + 31) / 32, c0 = lane * per;
        int run = 0;
        for (int c = c0; c < min(P, c0 + per); ++c) run += counts[c];
        int incl = run;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
          const int v = __shfl_up_sync(kFull, incl, off);
          if (lane >= off) incl += v;
        }
        int base = incl - run;
        int32_t* o = offs + st * kOff;
        for (int c = c0; c < min(P, c0 + per); ++c) { o[c] = base; base += counts[c]; }
        if (lane == 31) o[P] = incl;
      }
      __syncwarp();
#pragma unroll
      for (int q = 0; q < kAccT / 32; ++q)
        if (aj[q] >= 0) lists[st * kAccT + offs[st * kOff + aj[q]] + pos[q]] = 32 * q + lane;
      __syncwarp();
      if (lane == 0) {
        // one box of 128 tokens x CW channels lands row-major; rows past the end read as zeros
        uint8_t* dst = smraw + (size_t)st * kStageBytes;
        mb_expect_tx(&full[st], (uint32_t)kStageBytes);
        if constexpr (ES == 2) tma_load_4d(dst, &amap, slice * CW, h, tb, set, &full[st]);
        else tma_load_3d(dst, &amap, slice * CW, tb, prob, &full[st]);
      }
      last = k;
      __syncwarp();
    }
    // drain: a stage is refilled only after every consumer left it, so at most the newest copy of
    // each stage can still be in flight; wait (bounded) for those before the CTA may exit
    if (lane == 0) {
      for (int st = 0; st < kStages && st <= last; ++st) {
        const int k = st + ((last - st) / kStages) * kStages;
        if (!mb_wait(&full[st], (uint32_t)((k / kStages) & 1))) set_status(status, KVQ_DEV_TIMEOUT);
      }
    }
    return;
  }

  // ---- consumers: float64 sums of the rows scaled by 2^-896 (bf16, fp32) or 2^-1008 (fp16)
  const bool f16 = ES == 2 && s.dtype == KVQ_F16;
  double acc[CPW][E];
  uint32_t members[CPW];
#pragma unroll
  for (int c = 0; c < CPW; ++c) {
    members[c] = 0;
#pragma unroll
    for (int e = 0; e < E; ++e) acc[c][e] = 0.0;
  }
  for (int k = 0; k < nt; ++k) {
    const int st = k % kStages;
    const bool ok = mb_wait(&full[st], (uint32_t)((k / kStages) & 1));
    if (!__all_sync(kFull, ok)) {
      if (lane == 0) set_status(status, KVQ_DEV_TIMEOUT);
      break;
    }
    const uint8_t* stg = smraw + (size_t)st * kStageBytes;
    const int32_t* o = offs + st * kOff;
    const int32_t* lst = lists + st * kAccT;
#pragma unroll
    for (int c = 0; c < CPW; ++c) {
      const int j = warp + kAccWarps * c;
      if (j >= P) break;
      const int x0 = o[j], x1 = o[j + 1];
      members[c] += (uint32_t)(x1 - x0);
      for (int x = x0; x < x1; ++x) {
        const int t = lst[x];
        const uint8_t* row = stg + t * RB + lane * (E * ES);
        double v[E];
        if constexpr (ES == 4) {
          if constexpr (E == 4) {
            const uint4 f = *reinterpret_cast<const uint4*>(row);
            v[0] = f32_scaled(f.x); v[1] = f32_scaled(f.y); v[2] = f32_scaled(f.z); v[3] = f32_scaled(f.w);
          } else if constexpr (E == 2) {
            const uint2 f = *reinterpret_cast<const uint2*>(row);
            v[0] = f32_scaled(f.x); v[1] = f32_scaled(f.y);
          } else {
            v[0] = f32_scaled(*reinterpret_cast<const uint32_t*>(row));
          }
        } else {
          uint32_t b[(E + 1) / 2];
          if constexpr (E == 4) { const uint2 u = *reinterpret_cast<const uint2*>(row); b[0] = u.x; b[1] = u.y; }
          else if constexpr (E == 2) b[0] = *reinterpret_cast<const uint32_t*>(row);
          else b[0] = *reinterpret_cast<const uint16_t*>(row);
#pragma unroll
          for (int e = 0; e < E; ++e)
            v[e] = f16 ? ((e & 1) ? f16hi_scaled(b[e >> 1]) : f16lo_scaled(b[e >> 1]))
                       : ((e & 1) ? bf16hi_scaled(b[e >> 1]) : bf16lo_scaled(b[e >> 1]));
        }
#pragma unroll
        for (int e = 0; e < E; ++e) acc[c][e] += v[e];
      }
    }
    __syncwarp();
    if (lane == 0) mb_arrive(&empty[st]);
  }

  const double unscale = f16 ? 0x1p1008 : 0x1p896;
  double* gs = (ES == 4 ? part + ((size_t)prob * gridDim.x + blockIdx.x) * P * kD : sums + (size_t)prob * P * kD) +
               slice * CW + lane * E;
#pragma unroll
  for (int c = 0; c < CPW; ++c) {
    const int j = warp + kAccWarps * c;
    if (j >= P) break;
#pragma unroll
    for (int e = 0; e < E; ++e) {
      if constexpr (ES == 4) gs[(size_t)j * kD + e] = acc[c][e] * unscale;  // this CTA's slot, zeros included
      else if (acc[c][e] != 0.0) atomicAdd(gs + (size_t)j * kD + e, acc[c][e] * unscale);
    }
    if (slice == 0 && lane == 0 && members[c]) atomicAdd(cnt + (size_t)prob * P + j, members[c]);
  }
}

template <int CPW, int E, int ES>
constexpr size_t accum_smem() {
  constexpr int st = accum_stages<CPW, 32 * E * ES, ES>();
  return (size_t)st * (kAccT * 32 * E * ES) + 2 * st * sizeof(uint64_t) +
         ((size_t)st * (kAccWarps * CPW + 1) + (size_t)st * kAccT + kAccWarps * CPW + 1) * sizeof(int32_t);
}

template <int CPW, int E, int ES>
cudaError_t launch_accum_t(const CUtensorMap& amap, const Src& s, int P, int NP, int sms, const int32_t* assign,
                           double* sums, uint32_t* cnt, double* part, int32_t* status, cudaStream_t st) {
  constexpr size_t smem = accum_smem<CPW, E, ES>();
  cudaError_t e = cudaFuncSetAttribute(mine_accum_kernel<CPW, E, ES>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  const int slices = 4 / E;
  const int64_t ntiles = (s.n + kAccT - 1) / kAccT;
  const int64_t want = std::max<int64_t>(1, accum_ctas_per_sm<CPW, ES>() * sms / std::max(1, slices * NP));
  // fp32 rows: the CTA count fixes the partial slots of the workspace
  const unsigned chunks = ES == 4 ? (unsigned)accum_f32_chunks(s.n, NP, P)
                                  : (unsigned)std::max<int64_t>(1, std::min<int64_t>(ntiles, want));
  mine_accum_kernel<CPW, E, ES><<<dim3(chunks, slices, NP), (kAccWarps + 1) * 32, smem, st>>>(amap, s, P, assign,
                                                                                              sums, cnt, part, status);
  return cudaGetLastError();
}

// P <= 64: one 128-channel slice, 4 clusters per warp; P <= 128: two 64-channel slices, 8
// clusters per warp; P <= 256: four 32-channel slices, 16 clusters per warp
int accum_slice_channels(int P) { return P <= 4 * kAccWarps ? 128 : (P <= 8 * kAccWarps ? 64 : 32); }

cudaError_t launch_accum(const CUtensorMap& amap, const Src& s, int P, int NP, int sms, const int32_t* assign,
                         double* sums, uint32_t* cnt, double* part, int32_t* status, cudaStream_t st) {
  const bool f32 = s.y != nullptr;
  if (P <= 4 * kAccWarps)
    return f32 ? launch_accum_t<4, 4, 4>(amap, s, P, NP, sms, assign, sums, cnt, part, status, st)
               : launch_accum_t<4, 4, 2>(amap, s, P, NP, sms, assign, sums, cnt, part, status, st);
  if (P <= 8 * kAccWarps)
    return f32 ? launch_accum_t<8, 2, 4>(amap, s, P, NP, sms, assign, sums, cnt, part, status, st)
               : launch_accum_t<8, 2, 2>(amap, s, P, NP, sms, assign, sums, cnt, part, status, st);
  return f32 ? launch_accum_t<16, 1, 4>(amap, s, P, NP, sms, assign, sums, cnt, part, status, st)
             : launch_accum_t<16, 1, 2>(amap, s, P, NP, sms, assign, sums, cnt, part, status, st);
}

// ---- tcgen05 assignment (bf16 input, P <= 128) ------------------------------------------
//
// The same certified argmin as mine_assign_mma_kernel, with the distance contraction on
// the 5th-generation tensor cores, as a warp-specialised pipeline with no block barrier in
// its loop (two CTAs per SM for P <= 64, one above; roles hand stages and accumulators over
// through mbarriers):
//   * producer warp: per 128-token tile, two TMA loads (a box of 64 channels x 128 tokens
//     each, 4-D tensor map over channels x heads x tokens x sets, 128-byte swizzle; rows past
//     the end read as zeros) into a ring of shared-memory stages: the canonical K-major
//     layout with 128-byte swizzle, 8-row x 128-byte atoms (SBO = 1024 B), channels 0-63
//     and 64-127 in two 16 KB halves;
//   * MMA warp (one thread): 16 tcgen05.mma of M = 128 (tokens) x N = Pn (padded patterns) x
//     K = 16, the 8 K steps against the bf16 hi parts of the patterns and then the 8 against
//     their mid parts, into one fp32 accumulator in one of four TMEM buffers (Pn columns each);
//     commits to the buffer's "full" and the stage's "free" barriers.  One chain of 16 MMAs:
//     under the truncation model above it is off by at most 16 * 17 * 2^-22 |x| |m_j| (times
//     1.008 for the partial sums' bound), which with the 2^-16 |m| below hi + mid gives
//     |e_hat_j - e_j| <= 2^-12.59 |x| |m_j| plus the fp32 roundings, within E_j;
//   * 8 epilogue warps, two warpgroups: warpgroup g takes every other tile, in TMEM buffers g
//     and g + 2 in turn, so the MMAs of its next tile run while it scores this one; token t's
//     scores are TMEM lane t, so each warp handles its 32 tokens alone, with no barrier
//     between warps: u_j = |m_j|^2 / 2 - x.m_j (e_j = 2 u_j) with the pattern index
//     written into the 7 low mantissa bits (a move of at most 2^-16 |u_j|), one running pair
//     of smallest tagged values per chain, so one min chain yields the candidate, its index
//     and the gap; the gap test widened by twice the largest move.  A token that fails it
//     (well under 1 %) is listed for mine_fixup_kernel, which decides it with float64
//     distances before the cluster sums.  |x|^2 comes from the staged tile in the first
//     iteration and from a per-token cache after that.
// Every mbarrier wait is bounded.
constexpr int kTcM = 128;
// ring depth: two stages for P <= 64 (two CTAs per SM share the SM's shared memory and TMEM),
// up to five above (one CTA per SM)
constexpr int kTcMaxStages = 5;
constexpr int kTcTileBytes = kTcM * kD * 2;
constexpr uint32_t kTcSpinLimit = 1u << 22;
constexpr int kTcEpiWarps = 8;
constexpr int kTcThreads = (2 + kTcEpiWarps) * 32;

__device__ __forceinline__ uint32_t su32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

// shared-memory matrix descriptor, K-major with 128-byte swizzle: start (bytes >> 4), LBO unused
// (1), SBO = 1024 B between 8-row atoms, descriptor version 1, layout type 2 (128-byte swizzle).
// The start may move by 32 B per K = 16 step inside an atom; atoms are 1024-byte aligned.
__device__ __forceinline__ uint64_t umma_desc_sw128(uint32_t saddr) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | (1ull << 16) | ((uint64_t)(1024u >> 4) << 32) | (1ull << 46) |
         (2ull << 61);
}
// byte offset of (row, 16-byte chunk c of the 128-byte atom row) in a 128-byte-swizzled block
__host__ __device__ constexpr uint32_t sw128_off(int row, int c) {
  return (uint32_t)(row >> 3) * 1024u + (uint32_t)(row & 7) * 128u + (uint32_t)((c ^ (row & 7)) * 16);
}
// instruction descriptor, kind::f16: D fp32, A and B bf16, both K-major, N >> 3, M >> 4
__host__ __device__ constexpr uint32_t umma_idesc(int M, int N) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc, int accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(su32(bar))
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_proxy_async() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// 8 consecutive fp32 columns of this thread's TMEM lane, without waiting (tmem_ld_wait() before use)
__device__ __forceinline__ void tmem_ld8_issue(uint32_t taddr, float (&v)[8]) {
  uint32_t r[8];
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
               : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 8; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ bool tc_wait(uint64_t* bar, uint32_t parity) {
  for (uint32_t it = 0; it < kTcSpinLimit; ++it) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(su32(bar)), "r"(parity)
        : "memory");
    if (ok) return true;
  }
  return false;
}


constexpr float kTcPad = 1.0e38f;  // |m_j|^2 / 2 of the padding patterns past P: never the minimum

// u with its 7 low mantissa bits replaced by j (j < 128)
__device__ __forceinline__ float tag_score(float u, int j) {
  return __uint_as_float((__float_as_uint(u) & 0xFFFFFF80u) | (uint32_t)j);
}
// running two smallest values
__device__ __forceinline__ void low2_add(float& m1, float& m2, float v) {
  m2 = fminf(m2, fmaxf(m1, v));
  m1 = fminf(m1, v);
}
__global__ void __launch_bounds__(kTcThreads, 2) mine_assign_tc_kernel(const __grid_constant__ CUtensorMap xmap, Src s,
                                                                      int P, const float* __restrict__ M,
                                                                      int32_t* __restrict__ assign,
                                                                      float* __restrict__ xsq_cache, int first,
                                                                      int32_t* __restrict__ amb,
                                                                      uint32_t* __restrict__ ambc,
                                                                      uint8_t* __restrict__ ambn,
                                                                      int32_t* __restrict__ amb_cnt, int nst,
                                                                      int32_t* __restrict__ status) {
  const int prob = blockIdx.y;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int Pn = (P + 15) & ~15, N = 2 * Pn;
  // four accumulator buffers of Pn columns (hi and mid parts of a pattern in one chain), each
  // starting at a power-of-two column (16 .. 128)
  const uint32_t buf_cols = Pn <= 16 ? 16u : Pn <= 32 ? 32u : Pn <= 64 ? 64u : 128u;
  const uint32_t tcols = 4 * buf_cols;
  const uint32_t half_b = (uint32_t)N * 128u;      // B: channels 64-127 start N x 128 B in
  extern __shared__ __align__(16) uint8_t smraw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smraw) + 1023) & ~uintptr_t(1023));
  uint8_t* Bt = base;                                                   // [2 halves][N rows][128 B], swizzled
  uint8_t* At = base + (size_t)N * kD * 2;                              // [nst][2 halves][128 rows][128 B]
  float* hm = reinterpret_cast<float*>(At + (size_t)nst * kTcTileBytes);   // [Pn] |m_j|^2 / 2, padding past P
  float* gmax = hm + Pn;                                                // [4]
  uint64_t* bars = reinterpret_cast<uint64_t*>(gmax + 4);               // full[nst], sfree[nst], tfull[4], tempty[4]
  uint64_t* full = bars;
  uint64_t* sfree = bars + nst;
  uint64_t* tfull = bars + 2 * nst;
  uint64_t* tempty = tfull + 4;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(tempty + 4);
  const float* Mp = M + (size_t)prob * P * kD;
  const int set = prob / s.heads, h = prob % s.heads;

  // ---- B: bf16 hi parts (rows 0..Pn-1) and mid parts (rows Pn..2Pn-1) of the patterns
  for (int i = tid; i < N * 16; i += blockDim.x) {
    const int n = i >> 4, c = i & 15;
    const int j = n < Pn ? n : n - Pn;
    uint32_t wv[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      uint16_t hv[2];
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const float m = j < P ? Mp[(size_t)j * kD + 8 * c + 2 * q + e] : 0.f;
        const __nv_bfloat16 hi = __float2bfloat16_rn(m);
        const __nv_bfloat16 v = n < Pn ? hi : __float2bfloat16_rn(m - __bfloat162float(hi));
        hv[e] = __bfloat16_as_ushort(v);
      }
      wv[q] = (uint32_t)hv[0] | ((uint32_t)hv[1] << 16);
    }
    *reinterpret_cast<uint4*>(Bt + (size_t)(c >> 3) * half_b + sw128_off(n, c & 7)) =
        make_uint4(wv[0], wv[1], wv[2], wv[3]);
  }
  if (tid == 0) {
    gmax[0] = 0.f;
    gmax[1] = 0.f;
    for (int i = 0; i < nst; ++i) {
      mb_init(&full[i], 1);
      // the MMA commit, and in the first iteration the 4 warps of the tile's warpgroup (they read
      // the staged rows for |x|^2)
      mb_init(&sfree[i], first ? 1 + kTcEpiWarps / 2 : 1);
    }
    for (int i = 0; i < 4; ++i) {
      mb_init(&tfull[i], 1);
      mb_init(&tempty[i], kTcEpiWarps / 2);  // buffer i belongs to warpgroup i % 2
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(su32(tslot)), "r"(tcols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  __syncthreads();
  for (int j = tid; j < Pn; j += blockDim.x) {
    double acc = 0.0;
    if (j < P)
      for (int d = 0; d < kD; ++d) { const double m = Mp[(size_t)j * kD + d]; acc += m * m; }
    const float msq = (float)acc;
    hm[j] = j < P ? 0.5f * msq : kTcPad;
    atomicMax(reinterpret_cast<int*>(&gmax[0]), __float_as_int((float)(sqrt(acc) * (1.0 + 1e-6))));
    atomicMax(reinterpret_cast<int*>(&gmax[1]), __float_as_int(msq * (1.0f + 1e-6f)));
  }
  fence_proxy_async();  // B (generic stores) before the tensor cores read it
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tslot;

  const int64_t ntiles = (s.n + kTcM - 1) / kTcM;
  const int nt = ntiles > blockIdx.x ? (int)((ntiles - blockIdx.x + gridDim.x - 1) / gridDim.x) : 0;
  auto tile_t0 = [&](int k) { return ((int64_t)blockIdx.x + (int64_t)k * gridDim.x) * kTcM; };

  if (warp == 0) {
    // ---- producer
    if (lane == 0) {
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&xmap)) : "memory");
      int last = -1;  // newest tile whose copies were issued
      for (int k = 0; k < nt; ++k) {
        const int st = k % nst;
        if (k >= nst && !tc_wait(&sfree[st], (uint32_t)(((k / nst) - 1) & 1))) {
          set_status(status, KVQ_DEV_TIMEOUT);
          break;
        }
        uint8_t* dst = At + (size_t)st * kTcTileBytes;
        mb_expect_tx(&full[st], (uint32_t)kTcTileBytes);
        const int t0 = (int)tile_t0(k);
        tma_load_4d(dst, &xmap, 0, h, t0, set, &full[st]);
        tma_load_4d(dst + kTcTileBytes / 2, &xmap, 64, h, t0, set, &full[st]);
        last = k;
      }
      // drain: a stage is reloaded only after the MMAs of its previous tile committed, so at most
      // the newest copy of each stage can still be in flight; wait (bounded) for those
      for (int st = 0; st < nst && st <= last; ++st) {
        const int k = st + ((last - st) / nst) * nst;
        if (!tc_wait(&full[st], (uint32_t)((k / nst) & 1))) set_status(status, KVQ_DEV_TIMEOUT);
      }
    }
  } else if (warp == 1) {
    // ---- MMA issuer
    if (lane == 0) {
      const uint32_t idesc = umma_idesc(kTcM, Pn);
      const uint32_t b0 = su32(Bt);
      int last = -1;  // newest tile whose MMAs were committed
      for (int k = 0; k < nt; ++k) {
        const int st = k % nst, buf = k & 3;
        if (!tc_wait(&full[st], (uint32_t)((k / nst) & 1)) ||
            (k >= 4 && !tc_wait(&tempty[buf], (uint32_t)(((k >> 2) - 1) & 1)))) {
          set_status(status, KVQ_DEV_TIMEOUT);
          break;
        }
        tc_fence_after();
        const uint32_t a0 = su32(At + (size_t)st * kTcTileBytes);
        const uint32_t d = tbase + (uint32_t)buf * buf_cols;
        // x.hi_j then x.mid_j into the same accumulator: 16 MMAs of N = Pn; the mid rows start
        // Pn rows (Pn x 128 B, whole 8-row atoms) into each half of B
#pragma unroll
        for (int ks = 0; ks < 2 * (kD / 16); ++ks) {  // K step ks & 7: half (ks & 7) / 4, 32 B per step
          const int kk = ks & 7;
          const uint32_t bpart = ks < kD / 16 ? 0u : (uint32_t)Pn * 128u;
          umma_bf16(d, umma_desc_sw128(a0 + (kk >> 2) * (kTcTileBytes / 2) + (kk & 3) * 32),
                    umma_desc_sw128(b0 + bpart + (kk >> 2) * half_b + (kk & 3) * 32), idesc, ks > 0);
        }
        umma_commit(&tfull[buf]);
        umma_commit(&sfree[st]);
        last = k;
      }
      // drain: a commit tracks every tcgen05 operation this thread issued before it, so the
      // newest tile's commit landing means no MMA still writes TMEM or reads shared memory
      if (last >= 0 && !tc_wait(&tfull[last & 3], (uint32_t)((last >> 2) & 1))) set_status(status, KVQ_DEV_TIMEOUT);
    }
  } else {
    // ---- epilogue warps: warpgroup g takes tiles k with k % 2 == g, in TMEM buffers g and g + 2
    // in turn (the next tile's MMAs run while this one is scored), each warp its 32 rows, with no
    // barrier between warps
    const int ew = warp - 2, wg = ew >> 2, q4 = warp & 3;  // TMEM lane quarter of this warp
    const int row = q4 * 32 + lane;
    const float nm_max = gmax[0], msq_max = gmax[1];
    const uint32_t tlane = tbase + ((uint32_t)(q4 * 32) << 16);
    for (int k = wg; k < nt; k += 2) {
      const int st = k % nst;
      const int64_t i = tile_t0(k) + row;
      const bool valid = i < s.n;
      float xsq = 0.f;
      if (!first && valid) xsq = xsq_cache[(size_t)prob * s.n + i];
      const int buf = k & 3;
      const uint32_t taddr = tlane + (uint32_t)buf * buf_cols;
      if (!__all_sync(kFull, tc_wait(&tfull[buf], (uint32_t)((k >> 2) & 1)))) {
        if (lane == 0) set_status(status, KVQ_DEV_TIMEOUT);
        break;
      }
      tc_fence_after();
      float hv[8], hn[8];
      tmem_ld8_issue(taddr, hv);
      if (first) {
        // |x|^2 of the row from the staged tile (two swizzled halves of 64 channels)
        const uint8_t* stg = At + (size_t)st * kTcTileBytes;
        float a0 = 0.f, a1 = 0.f, b0 = 0.f, b1 = 0.f;
#pragma unroll 2
        for (int hc = 0; hc < 16; ++hc) {
          const uint4 u = *reinterpret_cast<const uint4*>(stg + (hc >> 3) * (kTcTileBytes / 2) + sw128_off(row, hc & 7));
          const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const float v0 = __uint_as_float(w[q] << 16), v1 = __uint_as_float(w[q] & 0xFFFF0000u);
            if (q & 1) fma2f(v0, v1, v0, v1, b0, b1, b0, b1);
            else fma2f(v0, v1, v0, v1, a0, a1, a0, a1);
          }
        }
        xsq = (a0 + a1) + (b0 + b1);
        if (valid) xsq_cache[(size_t)prob * s.n + i] = xsq;
      }
      if (first) {
        __syncwarp();
        if (lane == 0) mb_arrive(&sfree[st]);
      }
      tmem_ld_wait();
      // the two smallest tagged scores in two chains (even / odd patterns); blocks of 8
      // columns, the next block's loads in flight while one is scored
      float m1a = INFINITY, m2a = INFINITY, m1b = INFINITY, m2b = INFINITY;
      for (int c0 = 0; c0 < Pn; c0 += 8) {
        const bool more = c0 + 8 < Pn;
        if (more) tmem_ld8_issue(taddr + c0 + 8, hn);
#pragma unroll
        for (int q = 0; q < 8; q += 4) {
          const float4 hq = *reinterpret_cast<const float4*>(hm + c0 + q);
          float u0, u1, u2, u3;
          sub2(hq.x, hq.y, hv[q], hv[q + 1], u0, u1);
          sub2(hq.z, hq.w, hv[q + 2], hv[q + 3], u2, u3);
          low2_add(m1a, m2a, tag_score(u0, c0 + q));
          low2_add(m1b, m2b, tag_score(u1, c0 + q + 1));
          low2_add(m1a, m2a, tag_score(u2, c0 + q + 2));
          low2_add(m1b, m2b, tag_score(u3, c0 + q + 3));
        }
        if (more) {
          tmem_ld_wait();
#pragma unroll
          for (int q = 0; q < 8; ++q) hv[q] = hn[q];
        }
      }
      const float m1 = fminf(m1a, m1b);
      const float m2 = fminf(fmaxf(m1a, m1b), fminf(m2a, m2b));
      const float xs = xsq * (1.0f + 1e-6f);
      const float nx = sqrtf(xs) * (1.0f + 1e-6f);
      const float Eb = 0x1p-12f * nx * nm_max + 0x1p-20f * (xs + msq_max);
      const float Pe = 0x1p-16f * (msq_max + 2.0f * nx * nm_max);  // largest tag move of e = 2 u
      const float dl = 1e-9f * (xs + msq_max);
      const bool und = valid && !(2.0f * (m2 - m1) > 2.0f * Eb + 2.0f * Pe + dl);
      if (valid && !und) assign[(size_t)prob * s.n + i] = (int32_t)(__float_as_uint(m1) & 127u);
      if (__any_sync(kFull, und)) {
        // undecided: list the patterns that can still be the float64 argmin, those whose tagged
        // score is within m1 + Eb + Pe + dl (the score error, the tag move and the float64
        // rounding allowance, each counted on both sides), from a second pass over the columns
        float thr = m1 + Eb + Pe + dl;
        thr += fabsf(thr) * 0x1p-20f;  // the roundings of the sum above
        uint32_t c0w = 0u, c1w = 0u;
        int cnt = 0;
        for (int c0 = 0; c0 < Pn; c0 += 8) {
          tmem_ld8_issue(taddr + c0, hv);
          tmem_ld_wait();
#pragma unroll
          for (int q = 0; q < 8; q += 4) {
            const float4 hq = *reinterpret_cast<const float4*>(hm + c0 + q);
            float u[4];
            sub2(hq.x, hq.y, hv[q], hv[q + 1], u[0], u[1]);
            sub2(hq.z, hq.w, hv[q + 2], hv[q + 3], u[2], u[3]);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int j = c0 + q + e;
              if (und && j < P && tag_score(u[e], j) <= thr) {
                if (cnt < 4) c0w |= (uint32_t)j << (8 * cnt);
                else if (cnt < 8) c1w |= (uint32_t)j << (8 * (cnt - 4));
                ++cnt;
              }
            }
          }
        }
        if (und) {
          const size_t r = (size_t)prob * s.n + atomicAdd(amb_cnt + prob, 1);
          amb[r] = (int32_t)i;
          ambc[2 * r] = c0w;
          ambc[2 * r + 1] = c1w;
          ambn[r] = (uint8_t)(cnt > 8 ? 255 : cnt);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mb_arrive(&tempty[buf]);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tbase), "r"(tcols) : "memory");
}

// Tokens the tcgen05 assignment left undecided, with the candidate patterns its epilogue
// listed (P <= 128): a lane per (token, candidate) computes the float64 squared distance exactly
// as the sequential definition (channels 0..127 in order, no fused multiply-add), and the eight
// lanes of a token keep the smallest (lowest index among equal distances).  A warp takes four
// tokens at a time; a token with more than eight candidates has its eight lanes check every
// pattern instead.  The float64 row of the input is built from its bits (f32_scaled) and one exact
// multiply, as in the cluster sums.
constexpr int kFixWarps = 8;
__global__ void __launch_bounds__(kFixWarps * 32) mine_fixup_kernel(Src s, int P, const float* __restrict__ M,
                                                                    const int32_t* __restrict__ amb,
                                                                    const uint32_t* __restrict__ ambc,
                                                                    const uint8_t* __restrict__ ambn,
                                                                    const int32_t* __restrict__ amb_cnt,
                                                                    int32_t* __restrict__ assign) {
  const int prob = blockIdx.y, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tok = lane >> 3, slot = lane & 7;  // token tok of the warp's four, candidate `slot`
  const int count = amb_cnt[prob];
  const float* Mp = M + (size_t)prob * P * kD;
  const int set = prob / s.heads, h = prob % s.heads;
  for (int r0 = (blockIdx.x * kFixWarps + warp) * 4; r0 < count; r0 += gridDim.x * kFixWarps * 4) {
    const int r = r0 + tok;
    const bool act = r < count;
    const size_t ra = (size_t)prob * s.n + (act ? r : 0);
    const int64_t i = act ? amb[ra] : 0;
    const int nc = act ? (int)ambn[ra] : 0;
    const uint32_t cw = act ? ambc[2 * ra + (slot >> 2)] : 0u;
    const uint16_t* xrow = s.x + set * s.ss + i * s.ts + h * s.hs;
    double bd = INFINITY;
    int bj = 1 << 30;
    // the candidates of this lane: its slot, or (more than eight) every eighth pattern
    const int njobs = nc == 255 ? (P - slot + 7) / 8 : (slot < nc ? 1 : 0);
    for (int q = 0; q < njobs; ++q) {
      const int j = nc == 255 ? slot + 8 * q : (int)((cw >> (8 * (slot & 3))) & 0xffu);
      const float* m = Mp + (size_t)j * kD;
      double acc = 0.0;
#pragma unroll 8
      for (int d = 0; d < kD; d += 8) {
        const uint4 u = __ldg(reinterpret_cast<const uint4*>(xrow + d));
        const float4 ma = __ldg(reinterpret_cast<const float4*>(m + d));
        const float4 mb = __ldg(reinterpret_cast<const float4*>(m + d + 4));
        const uint32_t xw[4] = {u.x, u.y, u.z, u.w};
        const float mv[8] = {ma.x, ma.y, ma.z, ma.w, mb.x, mb.y, mb.z, mb.w};
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float xv = bits_to_float((uint16_t)((e & 1) ? (xw[e >> 1] >> 16) : (xw[e >> 1] & 0xffffu)), s.dtype);
          const double t = __dsub_rn((double)xv, (double)mv[e]);
          acc = __dadd_rn(acc, __dmul_rn(t, t));
        }
      }
      if (acc < bd || (acc == bd && j < bj)) { bd = acc; bj = j; }
    }
#pragma unroll
    for (int off = 4; off > 0; off >>= 1) {
      const double od = __shfl_xor_sync(kFull, bd, off);
      const int oj = __shfl_xor_sync(kFull, bj, off);
      if (od < bd || (od == bd && oj < bj)) { bd = od; bj = oj; }
    }
    if (act && slot == 0) assign[(size_t)prob * s.n + i] = bj;
  }
}

// ring depth that fits next to the patterns in 227 KB, and the dynamic shared memory it needs
int mine_tc_stages(int P) {
  const int Pn = (P + 15) & ~15;
  if (Pn <= 64) return 2;
  const int fixed = 2 * Pn * kD * 2 + Pn * 4 + 16 + (2 * kTcMaxStages + 8) * 8 + 16 + 1024;
  return std::max(2, std::min(kTcMaxStages, (227 * 1024 - fixed) / kTcTileBytes));
}
size_t mine_tc_smem(int P) {
  const int Pn = (P + 15) & ~15, nst = mine_tc_stages(P);
  return (size_t)2 * Pn * kD * 2 + (size_t)nst * kTcTileBytes + Pn * 4 + 16 + (2 * nst + 8) * 8 + 16 + 1024;
}

// Centroid = fl32(float64 sum / count); an empty cluster keeps its pattern.  With `part` (fp32
// rows) the sum is the CTAs' partials added in CTA order.
__global__ void mine_update_kernel(int P, float* M, double* sums, uint32_t* cnt, int32_t* amb_cnt,
                                   const double* part, int chunks) {
  const int prob = blockIdx.y, j = blockIdx.x, d = threadIdx.x;
  if (amb_cnt && j == 0 && d == 0) amb_cnt[prob] = 0;  // the next iteration's list starts empty
  const size_t pj = (size_t)prob * P + j;
  uint32_t c = cnt[pj];
  double sum;
  if (part) {
    sum = 0.0;
    for (int q = 0; q < chunks; ++q) sum += part[(((size_t)prob * chunks + q) * P + j) * kD + d];
  } else {
    sum = sums[pj * kD + d];
  }
  if (c > 0) M[pj * kD + d] = (float)(sum / (double)c);
  sums[pj * kD + d] = 0.0;
  __syncthreads();
  if (d == 0) cnt[pj] = 0;
}

}  // namespace

size_t mine_workspace(int64_t n, int sets, int heads, int P, int transform) {
  const int NP = sets * heads;
  size_t b = 256 + align256((size_t)NP * P * kD * sizeof(double)) + align256((size_t)NP * P * sizeof(uint32_t)) +
             align256((size_t)NP * (size_t)n * sizeof(int32_t)) + align256((size_t)NP * (size_t)n * sizeof(float)) +
             align256((size_t)NP * (size_t)n * sizeof(int32_t)) + align256((size_t)NP * (size_t)n * 8) +
             align256((size_t)NP * (size_t)n) + align256((size_t)NP * sizeof(int32_t));
  if (transform)
    b += align256((size_t)NP * n * kD * sizeof(float)) + align256((size_t)2 * NP * n * sizeof(double)) +
         align256((size_t)NP * fit_chunks(n) * 2 * kD * sizeof(double)) + 2 * align256((size_t)NP * kD * sizeof(double)) +
         align256((size_t)NP * accum_f32_chunks(n, NP, P) * P * kD * sizeof(double));
  return b + 256;
}

// Tiled TMA tensor maps (no swizzle; loads past the end read as zeros).  cuTensorMapEncodeTiled
// comes from the driver through the runtime's entry-point query.
cudaError_t encode_tiled_map(CUtensorMap* map, CUtensorMapDataType dt, int rank, const void* base,
                             const cuuint64_t* dims, const cuuint64_t* strides, const cuuint32_t* box,
                             CUtensorMapSwizzle swz) {
  static PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
  if (!encode) {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
    if (e != cudaSuccess) return e;
    if (q != cudaDriverEntryPointSuccess || !fn) return cudaErrorNotSupported;
    encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  }
  const cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  const CUresult r = encode(map, dt, (cuuint32_t)rank, const_cast<void*>(base), dims, strides, box, estr,
                            CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// The 16-bit input as (128 channels, heads, tokens, sets) with a box of `box_ch` channels x 1
// head x 128 tokens x 1 set.
static cudaError_t make_x_map(const MineArgs& a, CUtensorMap* map, int box_ch,
                              CUtensorMapSwizzle swz = CU_TENSOR_MAP_SWIZZLE_NONE) {
  const cuuint64_t dims[4] = {(cuuint64_t)kD, (cuuint64_t)a.heads, (cuuint64_t)a.n, (cuuint64_t)a.sets};
  const cuuint64_t strides[3] = {(cuuint64_t)a.head_stride * 2, (cuuint64_t)a.tok_stride * 2,
                                 (cuuint64_t)std::max<int64_t>(a.set_stride, 8) * 2};
  const cuuint32_t box[4] = {(cuuint32_t)box_ch, 1, 128, 1};
  return encode_tiled_map(map, a.dtype == KVQ_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 4,
                    a.x, dims, strides, box, swz);
}

// The fp32 pre-transformed rows y [problems][n][128] as (128 channels, tokens, problems) with a
// box of `box_ch` channels x 128 tokens x 1 problem.
static cudaError_t make_y_map(const float* y, int64_t n, int NP, CUtensorMap* map, int box_ch) {
  const cuuint64_t dims[3] = {(cuuint64_t)kD, (cuuint64_t)n, (cuuint64_t)NP};
  const cuuint64_t strides[2] = {(cuuint64_t)kD * 4, (cuuint64_t)n * kD * 4};
  const cuuint32_t box[3] = {(cuuint32_t)box_ch, 128, 1};
  return encode_tiled_map(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, y, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_NONE);
}

cudaError_t launch_mine(const MineArgs& a, void* ws, size_t ws_bytes, cudaStream_t st) {
  const int NP = a.sets * a.heads;
  if (NP == 0) return cudaSuccess;
  MineWs w = carve(ws, a.n, NP, a.P, a.transform, a.assign);
  Src s{(const uint16_t*)a.x, a.dtype, a.n, a.tok_stride, a.head_stride, a.set_stride, a.heads, nullptr};
  cudaError_t e;
  const dim3 rows_grid((unsigned)((a.n + 7) / 8), NP);
  const unsigned chunks = (unsigned)fit_chunks(a.n);
  if ((e = cudaMemsetAsync(w.status, 0, sizeof(int32_t), st)) != cudaSuccess) return e;

  if (a.transform) {
    for (int p = 0; p < kFitPasses; ++p) {
      double* rin = p == 0 ? nullptr : w.rrow + (size_t)((p + 1) & 1) * NP * a.n;
      double* rout = w.rrow + (size_t)(p & 1) * NP * a.n;
      fit_pass_kernel<<<dim3(chunks, NP), kFitWarps * 32, 0, st>>>(s, p == 0 ? nullptr : w.cinv, rin, rout, w.colpart);
      fit_finish_kernel<<<NP, kD, 0, st>>>(a.n, (int)chunks, w.colpart, w.colscale, w.cinv, p == 0);
    }
    fit_output_kernel<<<NP, kD, 0, st>>>(w.colscale, a.colscale);
    apply_kernel<<<rows_grid, 256, 0, st>>>(s, a.colscale, w.y);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    s.y = w.y;
  }

  mine_init_kernel<<<dim3(a.P, NP), kD, 0, st>>>(s, a.P, a.patterns);
  if ((e = cudaMemsetAsync(w.amb_cnt, 0, (size_t)NP * sizeof(int32_t), st)) != cudaSuccess ||
      (e = cudaMemsetAsync(w.sums, 0, (size_t)NP * a.P * kD * sizeof(double), st)) != cudaSuccess ||
      (e = cudaMemsetAsync(w.cnt, 0, (size_t)NP * a.P * sizeof(uint32_t), st)) != cudaSuccess)
    return e;
  size_t smem_assign = (size_t)a.P * kD * sizeof(float);
  if ((e = cudaFuncSetAttribute(mine_assign_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)smem_assign)) != cudaSuccess)
    return e;
  const int KIND = a.transform ? 2 : (a.dtype == KVQ_F16 ? 1 : 0);
  const bool use_mma = a.P <= kMmaMaxP;
  const size_t smem_mma = mine_mma_smem(a.P, KIND);
  if (use_mma) {
    if (KIND == 0) e = cudaFuncSetAttribute(mine_assign_mma_kernel<0>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_mma);
    else if (KIND == 1) e = cudaFuncSetAttribute(mine_assign_mma_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_mma);
    else e = cudaFuncSetAttribute(mine_assign_mma_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_mma);
    if (e != cudaSuccess) return e;
  }
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int tok_per_cta = kMmaWarps * (KIND == 0 ? 32 : 16);
  const unsigned mma_ctas = (unsigned)std::max<int64_t>(
      1, std::min<int64_t>((a.n + tok_per_cta - 1) / tok_per_cta, (int64_t)(2 * sms + NP - 1) / NP));
  // the cluster-sum kernel reads tiles of 128 rows through a tensor map (x, or the pre-transformed y)
  CUtensorMap amap;
  if ((e = a.transform ? make_y_map(w.y, a.n, NP, &amap, accum_slice_channels(a.P))
                       : make_x_map(a, &amap, accum_slice_channels(a.P))) != cudaSuccess)
    return e;
  // bf16 input and P <= 128: the tcgen05 kernel, one CTA (copy ring, 256 or 512 TMEM columns) per SM,
  // reading x through a 4-D tensor map (channels, heads, tokens, sets)
  const bool use_tc = KIND == 0 && a.P <= kMmaMaxP;
  const size_t smem_tc = mine_tc_smem(a.P);
  CUtensorMap xmap;
  if (use_tc) {
    if ((e = cudaFuncSetAttribute(mine_assign_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)smem_tc)) != cudaSuccess)
      return e;
    if ((e = make_x_map(a, &xmap, 64, CU_TENSOR_MAP_SWIZZLE_128B)) != cudaSuccess) return e;
  }
  const unsigned tc_ctas = (unsigned)std::max<int64_t>(
      1, std::min<int64_t>((a.n + kTcM - 1) / kTcM, (int64_t)std::max(1, (a.P <= 64 ? 2 : 1) * sms / NP)));
  for (int it = 0; it < a.iters; ++it) {
    const dim3 ag(mma_ctas, NP);
    if (use_tc) {
      mine_assign_tc_kernel<<<dim3(tc_ctas, NP), kTcThreads, smem_tc, st>>>(
          xmap, s, a.P, a.patterns, w.assign, w.xsq, it == 0, w.amb, w.ambc, w.ambn, w.amb_cnt, mine_tc_stages(a.P),
          w.status);
      mine_fixup_kernel<<<dim3((unsigned)std::max(1, 4 * sms / NP), NP), kFixWarps * 32, 0, st>>>(
          s, a.P, a.patterns, w.amb, w.ambc, w.ambn, w.amb_cnt, w.assign);
    } else if (use_mma && KIND == 0)
      mine_assign_mma_kernel<0><<<ag, kMmaWarps * 32, smem_mma, st>>>(s, a.P, a.patterns, w.assign);
    else if (use_mma && KIND == 1)
      mine_assign_mma_kernel<1><<<ag, kMmaWarps * 32, smem_mma, st>>>(s, a.P, a.patterns, w.assign);
    else if (use_mma)
      mine_assign_mma_kernel<2><<<ag, kMmaWarps * 32, smem_mma, st>>>(s, a.P, a.patterns, w.assign);
    else
      mine_assign_kernel<<<dim3((unsigned)((a.n + 127) / 128), NP), 128, smem_assign, st>>>(s, a.P, a.patterns,
                                                                                           w.assign);
    if ((e = launch_accum(amap, s, a.P, NP, sms, w.assign, w.sums, w.cnt, w.accpart, w.status, st)) != cudaSuccess)
      return e;
    mine_update_kernel<<<dim3(a.P, NP), kD, 0, st>>>(a.P, a.patterns, w.sums, w.cnt, use_tc ? w.amb_cnt : nullptr,
                                                     a.transform ? w.accpart : nullptr,
                                                     a.transform ? accum_f32_chunks(a.n, NP, a.P) : 0);
  }
  return cudaGetLastError();
}

}  // namespace kvq
