// Quantize-append: align each new K/V vector to its nearest pattern under the
// min-max distance, quantize the residual per group and store it in the paged
// cache ("PatternKV", Section 3.2 and Eq. 6; Eq. 1; granularity of Section 4.1).
//
// Launch 1 (page tasks): one CTA per (touched page, KV head, sequence).  It
//   quantizes the V vectors of the page's new tokens (per token, 4 groups of 32
//   channels) and, when the page's 32nd token arrives, seals the K group: the 32
//   keys (older ones from the K tail, new ones from the input) are aligned and
//   quantized per channel.
// Launch 2 (tail + commit): one CTA per sequence writes the keys of the newest,
//   incomplete group into the K tail and advances seq_len.  Splitting the two
//   keeps every tail read of launch 1 ahead of every tail write.
#include "kvq_common.cuh"
#include "kvq_internal.h"

namespace kvq {

namespace {

constexpr int kAppendThreads = 128;

struct PageCtx {
  int L, n, pg, a, e, set;
  bool fresh, seal;
  uint8_t* sub;
  const float* MK;
  const float* MV;
  const float* cK;
  const float* cV;
};

// Returns false if the CTA has nothing to do (or an error was flagged).
__device__ bool page_context(const Geom& g, int n_new, PageCtx& c) {
  const int b = blockIdx.z, h = blockIdx.y;
  c.L = g.seq_len[b];
  c.n = n_new;
  if (c.L < 0 || (int64_t)c.L + n_new > (int64_t)g.maxp * kG) {
    if (blockIdx.x == 0 && h == 0 && threadIdx.x == 0) set_status(g.status, KVQ_DEV_OVERFLOW);
    return false;
  }
  c.pg = c.L / kG + blockIdx.x;
  c.a = max(c.L, c.pg * kG);
  c.e = min(c.L + n_new, c.pg * kG + kG);
  if (c.a >= c.e) return false;
  int phys = g.page_table[(size_t)b * g.maxp + c.pg];
  if (phys < 0 || phys >= g.npages) {
    if (threadIdx.x == 0) set_status(g.status, KVQ_DEV_BAD_PAGE);
    return false;
  }
  c.set = g.seq_to_set ? g.seq_to_set[b] : 0;
  if (c.set < 0 || c.set >= g.S) {
    if (threadIdx.x == 0) set_status(g.status, KVQ_DEV_BAD_SET);
    return false;
  }
  c.fresh = (c.a == c.pg * kG);
  c.seal = (c.e == c.pg * kG + kG);
  c.sub = g.pool + (size_t)phys * g.page_bytes + (size_t)h * g.sub_bytes;
  size_t pat = ((size_t)c.set * g.H + h) * g.P * kD;
  c.MK = g.kpat + pat;
  c.MV = g.vpat + pat;
  c.cK = g.tx ? g.kcol + ((size_t)c.set * g.H + h) * kD : nullptr;
  c.cV = g.tx ? g.vcol + ((size_t)c.set * g.H + h) * kD : nullptr;
  return true;
}

// Write the 32-bit code words of a block from a smem code matrix X (row-major, ld = cols).
// keep(row, col) selects elements whose old bits are preserved (read-modify-write).
template <typename KeepFn>
__device__ void write_code_block(uint32_t* dst, const uint8_t* X, int ld, int bits, int KS, bool rmw, KeepFn keep) {
  const int nwords = kG * kD * bits / 32;
  const int slots = 16 / bits;  // codes per 16-bit half
  for (int w = threadIdx.x; w < nwords; w += blockDim.x) {
    uint32_t word = 0, keepmask = 0;
    for (int odd = 0; odd < 2; ++odd)
      for (int s = 0; s < slots; ++s) {
        int row, col;
        frag_elem(bits, KS, w, s, odd, row, col);
        int bit = bits * s + 16 * odd;
        uint32_t mask = ((1u << bits) - 1u) << bit;
        if (rmw && keep(row, col)) keepmask |= mask;
        else word |= ((uint32_t)X[row * ld + col] << bit) & mask;
      }
    if (rmw && keepmask) word |= dst[w] & keepmask;
    dst[w] = word;
  }
}

__global__ void __launch_bounds__(kAppendThreads) append_pages_kernel(Geom g, const uint16_t* __restrict__ k_new,
                                                                      const uint16_t* __restrict__ v_new,
                                                                      int n_new) {
  PageCtx c;
  if (!page_context(g, n_new, c)) return;
  const int b = blockIdx.z, h = blockIdx.y;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;

  __shared__ uint8_t vq[kD][kG];          // V codes, [channel][token]
  __shared__ uint8_t kq[kG][kD];          // K codes, [token][channel]
  __shared__ float kres[kG][kD];          // K residuals
  __shared__ float vs_s[kG][4], vz_s[kG][4], vrow_s[kG], krow_s[kG];
  __shared__ uint8_t vidx_s[kG], kidx_s[kG];

  for (int i = threadIdx.x; i < kD * kG; i += blockDim.x) (&vq[0][0])[i] = 0;
  if (threadIdx.x < kG) {
    for (int q = 0; q < 4; ++q) { vs_s[threadIdx.x][q] = 0.f; vz_s[threadIdx.x][q] = 0.f; }
    vrow_s[threadIdx.x] = 0.f;
    vidx_s[threadIdx.x] = 0;
  }
  __syncthreads();

  // ---- V: every new token of the page
  for (int t = c.a + warp; t < c.e; t += nwarps) {
    const int slot = t - c.pg * kG;
    const uint16_t* src = v_new + (((size_t)b * n_new + (t - c.L)) * g.H + h) * kD;
    float y[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) y[k] = load_elem(src + lane + 32 * k, g.dtype);
    float r = 1.0f;
    if (g.tx) transform_row_warp(y, c.cV, r, lane);
    int j = assign_warp(y, c.MV, g.P, lane);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      float R = __fsub_rn(y[k], c.MV[(size_t)j * kD + lane + 32 * k]);
      float s, z;
      int code = quant_warp(R, g.bits, s, z);
      vq[lane + 32 * k][slot] = (uint8_t)code;
      if (lane == 0) { vs_s[slot][k] = s; vz_s[slot][k] = z; }
    }
    if (lane == 0) { vidx_s[slot] = (uint8_t)j; vrow_s[slot] = r; }
  }

  // ---- K: seal the group when its last token arrives
  if (c.seal) {
    for (int slot = warp; slot < kG; slot += nwarps) {
      const int t = c.pg * kG + slot;
      const uint16_t* src = (t < c.L) ? g.k_tail + (((size_t)b * g.H + h) * kG + slot) * kD
                                      : k_new + (((size_t)b * n_new + (t - c.L)) * g.H + h) * kD;
      float y[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) y[k] = load_elem(src + lane + 32 * k, g.dtype);
      float r = 1.0f;
      if (g.tx) transform_row_warp(y, c.cK, r, lane);
      int j = assign_warp(y, c.MK, g.P, lane);
#pragma unroll
      for (int k = 0; k < 4; ++k) kres[slot][lane + 32 * k] = __fsub_rn(y[k], c.MK[(size_t)j * kD + lane + 32 * k]);
      if (lane == 0) { kidx_s[slot] = (uint8_t)j; krow_s[slot] = r; }
    }
  }
  __syncthreads();

  float* ks_g = reinterpret_cast<float*>(c.sub + g.off_ks);
  float* kz_g = reinterpret_cast<float*>(c.sub + g.off_kz);
  if (c.seal) {
    // per channel over the 32 tokens
    for (int d = threadIdx.x; d < kD; d += blockDim.x) {
      float mn = kres[0][d], mx = mn;
      for (int t = 1; t < kG; ++t) { mn = fminf(mn, kres[t][d]); mx = fmaxf(mx, kres[t][d]); }
      float s = __fdiv_rn(__fsub_rn(mx, mn), (float)((1 << g.bits) - 1));
      for (int t = 0; t < kG; ++t) {
        int code = 0;
        if (s != 0.0f) {
          code = __float2int_rn(__fdiv_rn(__fsub_rn(kres[t][d], mn), s));
          code = min(max(code, 0), (1 << g.bits) - 1);
        }
        kq[t][d] = (uint8_t)code;
      }
      ks_g[ksc_pos(d)] = s;
      kz_g[ksc_pos(d)] = mn;
    }
  }
  __syncthreads();

  // ---- stores
  const int lo = c.a - c.pg * kG, hi = c.e - c.pg * kG;  // new slots [lo, hi)
  write_code_block(reinterpret_cast<uint32_t*>(c.sub + g.off_vc), &vq[0][0], kG, g.bits, 2, !c.fresh,
                   [&](int row, int col) { return col < lo; });
  float* vs_g = reinterpret_cast<float*>(c.sub + g.off_vs);
  float* vz_g = reinterpret_cast<float*>(c.sub + g.off_vz);
  uint8_t* vidx_g = c.sub + g.off_vidx;
  float* vrow_g = reinterpret_cast<float*>(c.sub + g.off_vrow);
  for (int i = threadIdx.x; i < kG * 4; i += blockDim.x) {
    int slot = i >> 2, q = i & 3;
    if (c.fresh || (slot >= lo && slot < hi)) {
      vs_g[vsc_pos(slot, q)] = vs_s[slot][q];
      vz_g[vzc_pos(slot, q)] = vz_s[slot][q];
    }
  }
  for (int slot = threadIdx.x; slot < kG; slot += blockDim.x) {
    if (c.fresh || (slot >= lo && slot < hi)) {
      vidx_g[tok_pos(slot)] = vidx_s[slot];
      if (g.tx) vrow_g[tok_pos(slot)] = vrow_s[slot];
    }
  }
  if (c.seal) {
    write_code_block(reinterpret_cast<uint32_t*>(c.sub), &kq[0][0], kD, g.bits, 8, false,
                     [](int, int) { return false; });
    uint8_t* kidx_g = c.sub + g.off_kidx;
    float* krow_g = reinterpret_cast<float*>(c.sub + g.off_krow);
    for (int slot = threadIdx.x; slot < kG; slot += blockDim.x) {
      kidx_g[tok_pos(slot)] = kidx_s[slot];
      if (g.tx) krow_g[tok_pos(slot)] = krow_s[slot];
    }
  }
}

__global__ void append_tail_kernel(Geom g, const uint16_t* __restrict__ k_new, int n_new) {
  const int b = blockIdx.x;
  const int L = g.seq_len[b];
  if (L < 0 || (int64_t)L + n_new > (int64_t)g.maxp * kG) return;  // flagged by the page kernel
  const int newL = L + n_new;
  const int t0 = max(L, (newL / kG) * kG);
  const int per_tok = g.H * kD;
  for (int i = threadIdx.x; i < (newL - t0) * per_tok; i += blockDim.x) {
    int t = t0 + i / per_tok, rem = i % per_tok;
    int h = rem / kD, d = rem % kD;
    g.k_tail[(((size_t)b * g.H + h) * kG + (t % kG)) * kD + d] =
        k_new[(((size_t)b * n_new + (t - L)) * g.H + h) * kD + d];
  }
  __syncthreads();
  if (threadIdx.x == 0) g.seq_len[b] = newL;
}

}  // namespace

cudaError_t launch_append(const Geom& g, const void* k_new, const void* v_new, int n_new, cudaStream_t st) {
  if (n_new <= 0 || g.B == 0) return cudaSuccess;
  dim3 grid(n_new / kG + 2, g.H, g.B);
  append_pages_kernel<<<grid, kAppendThreads, 0, st>>>(g, (const uint16_t*)k_new, (const uint16_t*)v_new, n_new);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  append_tail_kernel<<<g.B, 256, 0, st>>>(g, (const uint16_t*)k_new, n_new);
  return cudaGetLastError();
}

}  // namespace kvq
