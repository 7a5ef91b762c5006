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

#include "kvq_common.cuh"
#include "kvq_internal.h"

namespace kvq {

namespace {

constexpr int kFitPasses = 3;
constexpr int kReduceChunk = 4096;

struct MineWs {
  double* sums;     // [NP][P][128]
  uint32_t* cnt;    // [NP][P]
  int32_t* assign;  // [NP][n]
  float* y;         // [NP][n][128] (transform only)
  double* v64;      // [NP][n][128] (transform only)
  double* colsum;   // [NP][128]
  double* colsq;    // [NP][128]
  double* colscale; // [NP][128]  running product of column divisors
  double* coldiv;   // [NP][128]  this pass's divisor
};

__host__ __device__ inline size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

inline MineWs carve(void* ws, int64_t n, int NP, int P, int transform, int32_t* assign_out) {
  uint8_t* p = (uint8_t*)ws;
  MineWs w{};
  w.sums = (double*)p; p += align256((size_t)NP * P * kD * sizeof(double));
  w.cnt = (uint32_t*)p; p += align256((size_t)NP * P * sizeof(uint32_t));
  if (assign_out) w.assign = assign_out;
  else { w.assign = (int32_t*)p; p += align256((size_t)NP * n * sizeof(int32_t)); }
  if (transform) {
    w.y = (float*)p; p += align256((size_t)NP * n * kD * sizeof(float));
    w.v64 = (double*)p; p += align256((size_t)NP * n * kD * sizeof(double));
    w.colsum = (double*)p; p += align256((size_t)NP * kD * sizeof(double));
    w.colsq = (double*)p; p += align256((size_t)NP * kD * sizeof(double));
    w.colscale = (double*)p; p += align256((size_t)NP * kD * sizeof(double));
    w.coldiv = (double*)p; p += align256((size_t)NP * kD * sizeof(double));
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

// v64 = fwht(x) (fp32 butterfly) per token; warp per token.
__global__ void fit_prep_kernel(Src s, double* v64, double* colscale) {
  const int prob = blockIdx.y, lane = threadIdx.x & 31;
  const int64_t i = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (blockIdx.x == 0 && threadIdx.x < kD) colscale[prob * kD + threadIdx.x] = 1.0;
  if (i >= s.n) return;
  float v[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) v[k] = s.at(prob, i, lane + 32 * k);
  fwht_warp(v, lane);
  double* row = v64 + ((size_t)prob * s.n + i) * kD;
#pragma unroll
  for (int k = 0; k < 4; ++k) row[lane + 32 * k] = (double)v[k];
}

// Row pass: divide every row by its population std (1 if zero); warp per row.  Also applies
// the previous column pass's divisors first when `coldiv` is given.
__global__ void fit_row_kernel(int64_t n, double* v64, const double* coldiv) {
  const int prob = blockIdx.y, lane = threadIdx.x & 31;
  const int64_t i = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (i >= n) return;
  double* row = v64 + ((size_t)prob * n + i) * kD;
  double v[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    v[k] = row[lane + 32 * k];
    if (coldiv) v[k] = v[k] / coldiv[prob * kD + lane + 32 * k];
  }
  double mean = warp_sum_d(v[0] + v[1] + v[2] + v[3]) / 128.0;
  double sq = 0.0;
#pragma unroll
  for (int k = 0; k < 4; ++k) { double t = v[k] - mean; sq += t * t; }
  double r = sqrt(warp_sum_d(sq) / 128.0);
  if (r == 0.0) r = 1.0;
#pragma unroll
  for (int k = 0; k < 4; ++k) row[lane + 32 * k] = v[k] / r;
}

// Column statistics: pass 0 sums, pass 1 squared deviations from the mean; 128 threads = channels.
__global__ void fit_col_kernel(int64_t n, const double* v64, double* colsum, double* colsq, int which) {
  const int prob = blockIdx.y, d = threadIdx.x;
  const int64_t i0 = (int64_t)blockIdx.x * kReduceChunk, i1 = min(n, i0 + kReduceChunk);
  const double* base = v64 + (size_t)prob * n * kD;
  double acc = 0.0;
  if (which == 0) {
    for (int64_t i = i0; i < i1; ++i) acc += base[i * kD + d];
    atomicAdd(colsum + prob * kD + d, acc);
  } else {
    double mean = colsum[prob * kD + d] / (double)n;
    for (int64_t i = i0; i < i1; ++i) { double t = base[i * kD + d] - mean; acc += t * t; }
    atomicAdd(colsq + prob * kD + d, acc);
  }
}

__global__ void fit_colfinish_kernel(int64_t n, double* colsum, double* colsq, double* colscale, double* coldiv) {
  const int prob = blockIdx.x, d = threadIdx.x;
  double s = sqrt(colsq[prob * kD + d] / (double)n);
  if (s == 0.0) s = 1.0;
  colscale[prob * kD + d] *= s;
  coldiv[prob * kD + d] = s;
  colsum[prob * kD + d] = 0.0;
  colsq[prob * kD + d] = 0.0;
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
// Scores e_j = |m_j|^2 - 2 x.m_j come from bf16 m16n8k16 MMAs: every pattern is split
// exactly into three bf16 terms (8+8+8 bits), inputs are exact in bf16 (bf16 input) or
// split into two bf16 terms (fp16 input exactly; fp32 pre-transformed rows to 2^-17).
// With E_j a bound on |e_hat_j - e_j| and U = min_j (e_hat_j + E_j), the float64
// argmin can only be a pattern with e_hat_j - E_j <= U + delta.  One such pattern is
// the answer; several are decided by recomputing their float64 distances exactly as
// the sequential reference does.  E_j = 2^-10 |x| |m_j| + 2^-20 (|x|^2 + |m_j|^2)
// covers fp32 accumulation in the tensor cores with a wide margin (the exact bound
// for 400 fp32 additions of exact products is below 2^-13.6 |x| |m_j|).
constexpr int kMmaMaxP = 128;
constexpr int kMmaWarps = 4;
constexpr int kBLd = kD + 8;  // padded bf16 row of a pattern split in shared memory

__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// hi and lo bf16 parts of two fp32 values (hi = rn(x), lo = rn(x - hi)).
__device__ __forceinline__ void split2(float x0, float x1, uint32_t& hi, uint32_t& lo) {
  __nv_bfloat162 h = __floats2bfloat162_rn(x0, x1);
  float2 hf = __bfloat1622float2(h);
  hi = *reinterpret_cast<uint32_t*>(&h);
  lo = pack_bf16(x0 - hf.x, x1 - hf.y);
}

// NA = number of bf16 terms of the input (1: exact bf16 input; 2: fp16 or fp32 input).
template <int NA>
__global__ void __launch_bounds__(kMmaWarps * 32) mine_assign_mma_kernel(Src s, int P, const float* __restrict__ M,
                                                                          int32_t* __restrict__ assign) {
  constexpr int kMt = NA == 1 ? 2 : 1;  // 16-token m-tiles per warp
  constexpr int kTok = 16 * kMt;        // tokens per warp tile
  extern __shared__ __align__(16) uint8_t smraw[];
  uint8_t* sm = smraw;
  const int prob = blockIdx.y;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int gq = lane >> 2, tig = lane & 3;
  const int Pp = (P + 7) & ~7;  // padded to whole n-tiles
  __nv_bfloat16* Bs = reinterpret_cast<__nv_bfloat16*>(sm);                       // [3][Pp][kBLd]
  float* mnorm = reinterpret_cast<float*>(sm + (size_t)3 * Pp * kBLd * 2);           // [Pp] |m_j|
  float* msq = mnorm + Pp;                                                            // [Pp] |m_j|^2
  float* escr = msq + Pp;                                                             // [warps][kTok][Pp+1]
  float* xn = escr + kMmaWarps * kTok * (Pp + 1);                                     // [warps][kTok] |x|^2
  const float* Mp = M + (size_t)prob * P * kD;

  // pattern splits and norms
  for (int i = threadIdx.x; i < Pp * kD; i += blockDim.x) {
    const int j = i / kD, d = i % kD;
    const float m = j < P ? Mp[(size_t)j * kD + d] : 0.f;
    const __nv_bfloat16 h = __float2bfloat16_rn(m);
    const float r1 = m - __bfloat162float(h);
    const __nv_bfloat16 mid = __float2bfloat16_rn(r1);
    const __nv_bfloat16 lo = __float2bfloat16_rn(r1 - __bfloat162float(mid));
    Bs[(0 * Pp + j) * kBLd + d] = h;
    Bs[(1 * Pp + j) * kBLd + d] = mid;
    Bs[(2 * Pp + j) * kBLd + d] = lo;
  }
  for (int j = threadIdx.x; j < Pp; j += blockDim.x) {
    double acc = 0.0;
    if (j < P)
      for (int d = 0; d < kD; ++d) { const double m = Mp[(size_t)j * kD + d]; acc += m * m; }
    msq[j] = (float)acc;
    mnorm[j] = (float)(sqrt(acc) * (1.0 + 1e-6));
  }
  __syncthreads();

  float* esc = escr + warp * kTok * (Pp + 1);
  float* xnw = xn + warp * kTok;
  const int64_t ntiles = (s.n + kTok - 1) / kTok;
  for (int64_t tile = (int64_t)blockIdx.x * kMmaWarps + warp; tile < ntiles; tile += (int64_t)gridDim.x * kMmaWarps) {
    const int64_t t0 = tile * kTok;
    // A fragments (NA bf16 terms) and the squared norms of the rows
    uint32_t A[NA][kMt][8][4];
    float nrm[kMt][2];
#pragma unroll
    for (int mt = 0; mt < kMt; ++mt) {
      nrm[mt][0] = nrm[mt][1] = 0.f;
#pragma unroll
      for (int rh = 0; rh < 2; ++rh) {
        const int64_t i = t0 + 16 * mt + 8 * rh + gq;
        const bool ok = i < s.n;
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
#pragma unroll
          for (int ch = 0; ch < 2; ++ch) {
            const int d = 16 * ks + 8 * ch + 2 * tig;
            const float x0 = ok ? s.at(prob, i, d) : 0.f, x1 = ok ? s.at(prob, i, d + 1) : 0.f;
            nrm[mt][rh] = fmaf(x0, x0, fmaf(x1, x1, nrm[mt][rh]));
            const int r = rh + 2 * ch;
            if constexpr (NA == 1) {
              A[0][mt][ks][r] = pack_bf16(x0, x1);
            } else {
              split2(x0, x1, A[0][mt][ks][r], A[NA - 1][mt][ks][r]);
            }
          }
      }
    }
#pragma unroll
    for (int mt = 0; mt < kMt; ++mt)
#pragma unroll
      for (int rh = 0; rh < 2; ++rh) {
        float v = nrm[mt][rh];
        v += __shfl_xor_sync(kFull, v, 1);
        v += __shfl_xor_sync(kFull, v, 2);
        if (tig == 0) xnw[16 * mt + 8 * rh + gq] = v * (1.0f + 1e-6f);
      }
    // scores, one n-tile (8 patterns) at a time
    for (int nt = 0; nt < Pp / 8; ++nt) {
      float acc[kMt][4];
#pragma unroll
      for (int mt = 0; mt < kMt; ++mt) acc[mt][0] = acc[mt][1] = acc[mt][2] = acc[mt][3] = 0.f;
#pragma unroll
      for (int sp = 0; sp < 3; ++sp) {
        const __nv_bfloat16* brow = Bs + ((size_t)sp * Pp + 8 * nt + gq) * kBLd + 2 * tig;
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          const uint32_t b0 = *reinterpret_cast<const uint32_t*>(brow + 16 * ks);
          const uint32_t b1 = *reinterpret_cast<const uint32_t*>(brow + 16 * ks + 8);
#pragma unroll
          for (int a = 0; a < NA; ++a)
#pragma unroll
            for (int mt = 0; mt < kMt; ++mt) mma_bf16(acc[mt], A[a][mt][ks], b0, b1);
        }
      }
#pragma unroll
      for (int mt = 0; mt < kMt; ++mt) {
        const int j0 = 8 * nt + 2 * tig;
        esc[(16 * mt + gq) * (Pp + 1) + j0] = msq[j0] - 2.0f * acc[mt][0];
        esc[(16 * mt + gq) * (Pp + 1) + j0 + 1] = msq[j0 + 1] - 2.0f * acc[mt][1];
        esc[(16 * mt + gq + 8) * (Pp + 1) + j0] = msq[j0] - 2.0f * acc[mt][2];
        esc[(16 * mt + gq + 8) * (Pp + 1) + j0 + 1] = msq[j0 + 1] - 2.0f * acc[mt][3];
      }
    }
    __syncwarp();
    // certify per token (lane = token of the tile)
    if (lane < kTok) {
      const int64_t i = t0 + lane;
      if (i < s.n) {
        const float* e = esc + lane * (Pp + 1);
        const float xsq = xnw[lane];
        const float nx = sqrtf(xsq) * (1.0f + 1e-6f);
        float U = INFINITY, best = INFINITY;
        int bj = 0;
        for (int j = 0; j < P; ++j) {
          const float E = 0x1p-10f * nx * mnorm[j] + 0x1p-20f * (xsq + msq[j]);
          U = fminf(U, e[j] + E);
          if (e[j] < best) { best = e[j]; bj = j; }
        }
        int cnt = 0;
        float emax = 0.f;
        for (int j = 0; j < P; ++j) {
          const float E = 0x1p-10f * nx * mnorm[j] + 0x1p-20f * (xsq + msq[j]);
          emax = fmaxf(emax, msq[j]);
          if (e[j] - E <= U + 1e-9f * (xsq + msq[j])) ++cnt;
        }
        if (cnt > 1) {
          // exact float64 distances of the candidates, channel order, lowest index on ties
          double bd = 0.0;
          bool have = false;
          for (int j = 0; j < P; ++j) {
            const float E = 0x1p-10f * nx * mnorm[j] + 0x1p-20f * (xsq + msq[j]);
            if (!(e[j] - E <= U + 1e-9f * (xsq + msq[j]))) continue;
            const float* m = Mp + (size_t)j * kD;
            double acc = 0.0;
            for (int d = 0; d < kD; ++d) {
              const double t = __dsub_rn((double)s.at(prob, i, d), (double)__ldg(m + d));
              acc = __dadd_rn(acc, __dmul_rn(t, t));
            }
            if (!have || acc < bd) { bd = acc; bj = j; have = true; }
          }
        }
        assign[(size_t)prob * s.n + i] = bj;
      }
    }
    __syncwarp();
  }
}

size_t mine_mma_smem(int P, int NA) {
  const int Pp = (P + 7) & ~7, kTok = NA == 1 ? 32 : 16;
  return (size_t)3 * Pp * kBLd * 2 + 2 * Pp * 4 + (size_t)kMmaWarps * kTok * (Pp + 1) * 4 + kMmaWarps * kTok * 4;
}

// Per-cluster float64 sums over a chunk of tokens for one quarter of the channels;
// one warp per CTA, lane = channel; flushed with global atomics.
__global__ void __launch_bounds__(32) mine_reduce_kernel(Src s, int P, const int32_t* __restrict__ assign,
                                                         double* __restrict__ sums, uint32_t* __restrict__ cnt) {
  extern __shared__ __align__(16) uint8_t smraw[];
  double* sm = reinterpret_cast<double*>(smraw);  // [P][32] sums, then [P] counts (as uint32 in the tail)
  uint32_t* scnt = reinterpret_cast<uint32_t*>(sm + (size_t)P * 32);
  const int prob = blockIdx.z, quarter = blockIdx.y, lane = threadIdx.x;
  const int d = quarter * 32 + lane;
  for (int j = 0; j < P; ++j) sm[j * 32 + lane] = 0.0;
  for (int j = lane; j < P; j += 32) scnt[j] = 0;
  __syncwarp();
  const int64_t i0 = (int64_t)blockIdx.x * kReduceChunk, i1 = min(s.n, i0 + kReduceChunk);
  const int32_t* a = assign + (size_t)prob * s.n;
  int64_t i = i0;
  for (; i + 8 <= i1; i += 8) {  // 8 independent loads in flight, then the dependent adds
    int j[8];
    float x[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) { j[u] = a[i + u]; x[u] = s.at(prob, i + u, d); }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      sm[j[u] * 32 + lane] += (double)x[u];
      if (quarter == 0 && lane == 0) scnt[j[u]] += 1;
    }
  }
  for (; i < i1; ++i) {
    const int j = a[i];
    sm[j * 32 + lane] += (double)s.at(prob, i, d);
    if (quarter == 0 && lane == 0) scnt[j] += 1;
  }
  __syncwarp();
  double* gs = sums + (size_t)prob * P * kD;
  for (int j = 0; j < P; ++j) {
    double v = sm[j * 32 + lane];
    if (v != 0.0) atomicAdd(gs + j * kD + d, v);
  }
  if (quarter == 0)
    for (int j = lane; j < P; j += 32)
      if (scnt[j]) atomicAdd(cnt + (size_t)prob * P + j, scnt[j]);
}

__global__ void mine_update_kernel(int P, float* M, double* sums, uint32_t* cnt) {
  const int prob = blockIdx.y, j = blockIdx.x, d = threadIdx.x;
  const size_t pj = (size_t)prob * P + j;
  uint32_t c = cnt[pj];
  if (c > 0) M[pj * kD + d] = (float)(sums[pj * kD + d] / (double)c);
  sums[pj * kD + d] = 0.0;
  __syncthreads();
  if (d == 0) cnt[pj] = 0;
}

}  // namespace

size_t mine_workspace(int64_t n, int sets, int heads, int P, int transform) {
  size_t NP = (size_t)sets * heads;
  size_t b = align256(NP * P * kD * sizeof(double)) + align256(NP * P * sizeof(uint32_t)) +
             align256(NP * (size_t)n * sizeof(int32_t));
  if (transform)
    b += align256(NP * n * kD * sizeof(float)) + align256(NP * n * kD * sizeof(double)) +
         4 * align256(NP * kD * sizeof(double));
  return b + 256;
}

cudaError_t launch_mine(const MineArgs& a, void* ws, size_t ws_bytes, cudaStream_t st) {
  const int NP = a.sets * a.heads;
  if (NP == 0) return cudaSuccess;
  MineWs w = carve(ws, a.n, NP, a.P, a.transform, a.assign);
  Src s{(const uint16_t*)a.x, a.dtype, a.n, a.tok_stride, a.head_stride, a.set_stride, a.heads, nullptr};
  cudaError_t e;
  const dim3 rows_grid((unsigned)((a.n + 7) / 8), NP);
  const unsigned chunks = (unsigned)((a.n + kReduceChunk - 1) / kReduceChunk);

  if (a.transform) {
    fit_prep_kernel<<<rows_grid, 256, 0, st>>>(s, w.v64, w.colscale);
    cudaMemsetAsync(w.colsum, 0, (size_t)NP * kD * sizeof(double), st);
    cudaMemsetAsync(w.colsq, 0, (size_t)NP * kD * sizeof(double), st);
    for (int p = 0; p < kFitPasses; ++p) {
      fit_row_kernel<<<rows_grid, 256, 0, st>>>(a.n, w.v64, p == 0 ? nullptr : w.coldiv);
      fit_col_kernel<<<dim3(chunks, NP), kD, 0, st>>>(a.n, w.v64, w.colsum, w.colsq, 0);
      fit_col_kernel<<<dim3(chunks, NP), kD, 0, st>>>(a.n, w.v64, w.colsum, w.colsq, 1);
      fit_colfinish_kernel<<<NP, kD, 0, st>>>(a.n, w.colsum, w.colsq, w.colscale, w.coldiv);
    }
    fit_output_kernel<<<NP, kD, 0, st>>>(w.colscale, a.colscale);
    apply_kernel<<<rows_grid, 256, 0, st>>>(s, a.colscale, w.y);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    s.y = w.y;
  }

  mine_init_kernel<<<dim3(a.P, NP), kD, 0, st>>>(s, a.P, a.patterns);
  cudaMemsetAsync(w.sums, 0, (size_t)NP * a.P * kD * sizeof(double), st);
  cudaMemsetAsync(w.cnt, 0, (size_t)NP * a.P * sizeof(uint32_t), st);
  size_t smem_assign = (size_t)a.P * kD * sizeof(float);
  size_t smem_reduce = (size_t)a.P * 32 * sizeof(double) + (size_t)a.P * sizeof(uint32_t);
  if ((e = cudaFuncSetAttribute(mine_assign_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)smem_assign)) != cudaSuccess)
    return e;
  if ((e = cudaFuncSetAttribute(mine_reduce_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)smem_reduce)) != cudaSuccess)
    return e;
  const int NA = (a.transform || a.dtype == KVQ_F16) ? 2 : 1;
  const bool use_mma = a.P <= kMmaMaxP;
  const size_t smem_mma = mine_mma_smem(a.P, NA);
  if (use_mma) {
    if (NA == 1) e = cudaFuncSetAttribute(mine_assign_mma_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_mma);
    else e = cudaFuncSetAttribute(mine_assign_mma_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_mma);
    if (e != cudaSuccess) return e;
  }
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int tok_per_cta = kMmaWarps * (NA == 1 ? 32 : 16);
  const unsigned mma_ctas = (unsigned)std::max<int64_t>(
      1, std::min<int64_t>((a.n + tok_per_cta - 1) / tok_per_cta, (int64_t)(2 * sms + NP - 1) / NP));
  for (int it = 0; it < a.iters; ++it) {
    if (use_mma && NA == 1)
      mine_assign_mma_kernel<1><<<dim3(mma_ctas, NP), kMmaWarps * 32, smem_mma, st>>>(s, a.P, a.patterns, w.assign);
    else if (use_mma)
      mine_assign_mma_kernel<2><<<dim3(mma_ctas, NP), kMmaWarps * 32, smem_mma, st>>>(s, a.P, a.patterns, w.assign);
    else
      mine_assign_kernel<<<dim3((unsigned)((a.n + 127) / 128), NP), 128, smem_assign, st>>>(s, a.P, a.patterns,
                                                                                           w.assign);
    mine_reduce_kernel<<<dim3(chunks, 4, NP), 32, smem_reduce, st>>>(s, a.P, w.assign, w.sums, w.cnt);
    mine_update_kernel<<<dim3(a.P, NP), kD, 0, st>>>(a.P, a.patterns, w.sums, w.cnt);
  }
  return cudaGetLastError();
}

}  // namespace kvq
