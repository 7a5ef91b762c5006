// Prefill pattern mining: Lloyd k-means under the Euclidean metric, one
// independent problem per (pattern set, KV head) ("PatternKV", Section 3.1,
// Eq. 4, and the GPU-parallel KMeans of Section 3.4), optionally after fitting
// the KVarN pre-transform (Hadamard rotation + 3 alternating row / column std
// normalisation passes).
//
// Numerics: squared distances in float64 accumulated over channels 0..127 in
// order (ties to the lowest index), centroid sums in float64, centroid =
// fp32 rounding of the float64 mean, empty clusters keep their pattern.
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
  extern __shared__ float Ms[];
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

// Per-cluster float64 sums over a chunk of tokens for one quarter of the channels;
// one warp per CTA, lane = channel; flushed with global atomics.
__global__ void __launch_bounds__(32) mine_reduce_kernel(Src s, int P, const int32_t* __restrict__ assign,
                                                         double* __restrict__ sums, uint32_t* __restrict__ cnt) {
  extern __shared__ double sm[];  // [P][32] sums, then [P] counts (as uint32 in the tail)
  uint32_t* scnt = reinterpret_cast<uint32_t*>(sm + (size_t)P * 32);
  const int prob = blockIdx.z, quarter = blockIdx.y, lane = threadIdx.x;
  const int d = quarter * 32 + lane;
  for (int j = 0; j < P; ++j) sm[j * 32 + lane] = 0.0;
  for (int j = lane; j < P; j += 32) scnt[j] = 0;
  __syncwarp();
  const int64_t i0 = (int64_t)blockIdx.x * kReduceChunk, i1 = min(s.n, i0 + kReduceChunk);
  const int32_t* a = assign + (size_t)prob * s.n;
  for (int64_t i = i0; i < i1; ++i) {
    int j = a[i];
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
  for (int it = 0; it < a.iters; ++it) {
    mine_assign_kernel<<<dim3((unsigned)((a.n + 127) / 128), NP), 128, smem_assign, st>>>(s, a.P, a.patterns,
                                                                                         w.assign);
    mine_reduce_kernel<<<dim3(chunks, 4, NP), 32, smem_reduce, st>>>(s, a.P, w.assign, w.sums, w.cnt);
    mine_update_kernel<<<dim3(a.P, NP), kD, 0, st>>>(a.P, a.patterns, w.sums, w.cnt);
  }
  return cudaGetLastError();
}

}  // namespace kvq
