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

  // vectors of this page: the new V tokens (slots lo..hi-1), then all 32 K tokens if the group seals
  constexpr int kLd = kD + 4;                       // padded row (floats)
  __shared__ __align__(16) float vec[2 * kG][kLd];  // pre-transformed rows y
  __shared__ uint8_t vq[kD][kG];                    // V codes, [channel][token]
  __shared__ uint8_t kq[kG][kD];                    // K codes, [token][channel]
  __shared__ float vs_s[kG][4], vz_s[kG][4], vrow_s[kG], krow_s[kG];
  __shared__ uint8_t vidx_s[kG], kidx_s[kG];
  const int lo = c.a - c.pg * kG, hi = c.e - c.pg * kG;  // new slots [lo, hi)
  const int nv = hi - lo, nk = c.seal ? kG : 0, nvec = nv + nk;

  for (int i = threadIdx.x; i < kD * kG; i += blockDim.x) (&vq[0][0])[i] = 0;
  if (threadIdx.x < kG) {
    for (int q = 0; q < 4; ++q) { vs_s[threadIdx.x][q] = 0.f; vz_s[threadIdx.x][q] = 0.f; }
    vrow_s[threadIdx.x] = 0.f;
    vidx_s[threadIdx.x] = 0;
  }

  // ---- load (and pre-transform) every vector: warp per vector
  for (int v = warp; v < nvec; v += nwarps) {
    const uint16_t* src;
    const float* col;
    if (v < nv) {
      const int t = c.a + v;
      src = v_new + (((size_t)b * n_new + (t - c.L)) * g.H + h) * kD;
      col = c.cV;
    } else {
      const int slot = v - nv, t = c.pg * kG + slot;
      src = (t < c.L) ? g.k_tail + (((size_t)b * g.H + h) * kG + slot) * kD
                      : k_new + (((size_t)b * n_new + (t - c.L)) * g.H + h) * kD;
      col = c.cK;
    }
    float y[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) y[k] = load_elem(src + lane + 32 * k, g.dtype);
    float r = 1.0f;
    if (g.tx) transform_row_warp(y, col, r, lane);
#pragma unroll
    for (int k = 0; k < 4; ++k) vec[v][lane + 32 * k] = y[k];
    if (lane == 0) {
      if (v < nv) vrow_s[lo + v] = r;
      else krow_s[v - nv] = r;
    }
  }
  __syncthreads();

  // ---- nearest pattern: two threads per vector, each over half of the patterns
  {
    const int v = threadIdx.x >> 1, half = threadIdx.x & 1;
    float best = INFINITY;
    int bj = 0x7fffffff;
    if (v < nvec) {
      float y[kD];
#pragma unroll
      for (int d4 = 0; d4 < kD / 4; ++d4) {
        const float4 t = *reinterpret_cast<const float4*>(&vec[v][4 * d4]);
        y[4 * d4] = t.x; y[4 * d4 + 1] = t.y; y[4 * d4 + 2] = t.z; y[4 * d4 + 3] = t.w;
      }
      const float* M = (v < nv) ? c.MV : c.MK;
      for (int j = half; j < g.P; j += 2) {
        const float d = dmm_reg(y, M + (size_t)j * kD);
        if (d < best) { best = d; bj = j; }
      }
    }
    const float ob = __shfl_xor_sync(kFull, best, 1);
    const int oj = __shfl_xor_sync(kFull, bj, 1);
    if (ob < best || (ob == best && oj < bj)) { best = ob; bj = oj; }
    if (v < nvec && half == 0) {
      if (v < nv) vidx_s[lo + v] = (uint8_t)bj;
      else kidx_s[v - nv] = (uint8_t)bj;
    }
  }
  __syncthreads();

  // ---- V: residual and per-token group quantization, warp per token
  for (int v = warp; v < nv; v += nwarps) {
    const int slot = lo + v;
    const int j = vidx_s[slot];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float R = __fsub_rn(vec[v][lane + 32 * k], c.MV[(size_t)j * kD + lane + 32 * k]);
      float s, z;
      const int code = quant_warp(R, g.bits, s, z);
      vq[lane + 32 * k][slot] = (uint8_t)code;
      if (lane == 0) { vs_s[slot][k] = s; vz_s[slot][k] = z; }
    }
  }

  // ---- K: per-channel quantization over the 32 tokens of the sealed group
  float* ks_g = reinterpret_cast<float*>(c.sub + g.off_ks);
  float* kz_g = reinterpret_cast<float*>(c.sub + g.off_kz);
  if (c.seal) {
    for (int d = threadIdx.x; d < kD; d += blockDim.x) {
      float R[kG];
      float mn = INFINITY, mx = -INFINITY;
#pragma unroll
      for (int t = 0; t < kG; ++t) {
        R[t] = __fsub_rn(vec[nv + t][d], c.MK[(size_t)kidx_s[t] * kD + d]);
        mn = fminf(mn, R[t]);
        mx = fmaxf(mx, R[t]);
      }
      const float s = __fdiv_rn(__fsub_rn(mx, mn), (float)((1 << g.bits) - 1));
#pragma unroll
      for (int t = 0; t < kG; ++t) {
        int code = 0;
        if (s != 0.0f) {
          code = __float2int_rn(__fdiv_rn(__fsub_rn(R[t], mn), s));
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
  write_code_block(reinterpret_cast<uint32_t*>(c.sub + g.off_vc), &vq[0][0], kG, g.bits, 2, !c.fresh,
                   [&](int row, int col) { return col < lo; });
  float* vs_g = reinterpret_cast<float*>(c.sub + g.off_vs);
  float* vz_g = reinterpret_cast<float*>(c.sub + g.off_vz);
  uint8_t* vidx_g = c.sub + g.off_vidx;
  float* vrow_g = reinterpret_cast<float*>(c.sub + g.off_vrow);
  for (int i = threadIdx.x; i < kG * 4; i += blockDim.x) {
    const int slot = i >> 2, q = i & 3;
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
