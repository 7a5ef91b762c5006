// Quantize-append: align each new K/V vector to its nearest pattern under the
// min-max distance, quantize the residual per group and store it in the paged
// cache ("PatternKV", Section 3.2 and Eq. 6; Eq. 1; granularity of Section 4.1).
//
// Launch 0 (prep, per call): for every (set, KV head) and K / V pattern set, bf16
//   copies of the patterns and their squared norms (for a tensor-core Euclidean
//   guess), and the table T[j][k] = d_mm(m_j, m_k) of min-max distances between
//   patterns.
// Launch 1 (page tasks): one CTA per (touched page, KV head, sequence).
//   * the new V vectors of the page and, when the page's 32nd token arrives, its 32
//     K vectors (older ones from the K tail) are staged in shared memory (after the
//     pre-transform, if enabled);
//   * a seed pattern per vector from bf16 MMAs (Euclidean nearest, approximate);
//   * the exact fp32 d_mm of the seed, then exact pruning: d_mm is a seminorm, so
//     d_mm(x, m_j) >= T[j][s] - d_mm(x, m_s); every j with T[j][s] > 2 d_mm(x, m_s) plus
//     a rounding margin is strictly farther than the seed and skipped;
//   * a second exact bound for the survivors: the residual range over 16 channels (those
//     whose values differ most across the patterns) never exceeds the full range, so a
//     pattern whose partial range already exceeds the seed's distance is farther too;
//   * the remaining (vector, pattern) pairs go through a shared work queue; their
//     exact d_mm values meet in a 64-bit (distance, index) atomic minimum, so the
//     lowest index wins ties exactly as in the definition;
//   * residuals, group quantization (fp32; the correctly rounded division decides
//     wherever it could change a code), packing and stores.
// Launch 2 (tail + commit): one CTA per sequence writes the keys of the newest,
//   incomplete group into the K tail and advances seq_len.  Splitting launches 1 and
//   2 keeps every tail read ahead of every tail write.
#include "kvq_common.cuh"
#include "kvq_internal.h"

namespace kvq {

namespace {

constexpr int kAppendThreads = 128;
constexpr int kPLd = kD + 32;  // bf16 pattern row in the prep workspace (16-byte aligned rows)
constexpr int kQueueCap = 1024;

constexpr int kProbe = 16;  // channels of the partial-range bound

struct AppendWs {
  __nv_bfloat16* pb;  // [S][H][2][Pp][kPLd] bf16 patterns (0 = K, 1 = V)
  float* msq;         // [S][H][2][Pp] squared norms
  float* tab;         // [S][H][2][P][P] d_mm between patterns
  float* minf;        // [S][H][2] max |m|_inf
  int32_t* probe;     // [S][H][2][kProbe] channels with the widest spread across patterns
};

__host__ __device__ inline size_t al256(size_t v) { return (v + 255) & ~size_t(255); }

inline AppendWs carve_append(void* ws, int S, int H, int P) {
  const int Pp = (P + 7) & ~7;
  uint8_t* p = (uint8_t*)ws;
  AppendWs w;
  w.pb = (__nv_bfloat16*)p; p += al256((size_t)S * H * 2 * Pp * kPLd * 2);
  w.msq = (float*)p; p += al256((size_t)S * H * 2 * Pp * 4);
  w.tab = (float*)p; p += al256((size_t)S * H * 2 * P * P * 4);
  w.minf = (float*)p; p += al256((size_t)S * H * 2 * 4);
  w.probe = (int32_t*)p;
  return w;
}

// ---- launch 0: per (set, head, K|V) pattern tables --------------------------------------
__global__ void append_prep_kernel(Geom g, AppendWs w) {
  const int sh = blockIdx.x, kv = blockIdx.y;  // sh = set * H + head
  const int P = g.P, Pp = (P + 7) & ~7;
  const float* M = (kv ? g.vpat : g.kpat) + (size_t)sh * P * kD;
  const size_t o = (size_t)sh * 2 + kv;
  __nv_bfloat16* pb = w.pb + o * Pp * kPLd;
  for (int i = threadIdx.x; i < Pp * kD; i += blockDim.x) {
    const int j = i / kD, d = i % kD;
    pb[j * kPLd + d] = __float2bfloat16_rn(j < P ? M[(size_t)j * kD + d] : 0.f);
  }
  float mx = 0.f;
  for (int j = threadIdx.x; j < Pp; j += blockDim.x) {
    float acc = 0.f;
    if (j < P)
      for (int d = 0; d < kD; ++d) {
        const float m = M[(size_t)j * kD + d];
        acc = fmaf(m, m, acc);
        mx = fmaxf(mx, fabsf(m));
      }
    w.msq[o * Pp + j] = acc;
  }
  mx = warp_max(mx);
  __shared__ float wm[32];
  if ((threadIdx.x & 31) == 0) wm[threadIdx.x >> 5] = mx;
  __syncthreads();
  if (threadIdx.x == 0) {
    float m = 0.f;
    for (int i = 0; i < (int)(blockDim.x >> 5); ++i) m = fmaxf(m, wm[i]);
    w.minf[o] = m;
  }
  // d_mm(m_j, m_k) for all pairs, from a shared copy of the patterns
  extern __shared__ __align__(16) float Ms[];  // [P][kD + 4]
  constexpr int ld = kD + 4;
  for (int i = threadIdx.x; i < P * kD; i += blockDim.x) Ms[(i / kD) * ld + i % kD] = M[i];
  __syncthreads();
  float* tab = w.tab + o * P * P;
  for (int i = threadIdx.x; i < P * P; i += blockDim.x) {
    const int j = i / P, k = i % P;
    const float4* a4 = reinterpret_cast<const float4*>(Ms + j * ld);
    const float4* b4 = reinterpret_cast<const float4*>(Ms + k * ld);
    float hi = -INFINITY, lo = INFINITY;
#pragma unroll 8
    for (int d = 0; d < kD / 4; ++d) {
      const float4 x = a4[d], y = b4[d];
      float r0, r1, r2, r3;
      sub2(x.x, x.y, y.x, y.y, r0, r1);
      sub2(x.z, x.w, y.z, y.w, r2, r3);
      hi = max3(hi, r0, r1);
      lo = min3(lo, r0, r1);
      hi = max3(hi, r2, r3);
      lo = min3(lo, r2, r3);
    }
    tab[i] = __fsub_rn(hi, lo);
  }
  // probe channels: the kProbe widest spreads (max_j m_jd - min_j m_jd), by rank selection
  __shared__ float spread[kD];
  for (int d = threadIdx.x; d < kD; d += blockDim.x) {
    float hi = -INFINITY, lo = INFINITY;
    for (int j = 0; j < P; ++j) { hi = fmaxf(hi, Ms[j * ld + d]); lo = fminf(lo, Ms[j * ld + d]); }
    spread[d] = hi - lo;
  }
  __syncthreads();
  for (int d = threadIdx.x; d < kD; d += blockDim.x) {
    int rank = 0;
    for (int e = 0; e < kD; ++e) rank += (spread[e] > spread[d]) || (spread[e] == spread[d] && e < d);
    if (rank < kProbe) w.probe[o * kProbe + rank] = d;
  }
}

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
  const int phys = g.page_table[(size_t)b * g.maxp + c.pg];
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
  const size_t pat = ((size_t)c.set * g.H + h) * g.P * kD;
  c.MK = g.kpat + pat;
  c.MV = g.vpat + pat;
  c.cK = g.tx ? g.kcol + ((size_t)c.set * g.H + h) * kD : nullptr;
  c.cV = g.tx ? g.vcol + ((size_t)c.set * g.H + h) * kD : nullptr;
  return true;
}

__device__ __forceinline__ void mma_bf16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Exact partial max / min of y - m over channels [c0, c0 + 64) (y staged, m global).
__device__ __forceinline__ void dmm_half(const float* __restrict__ y, const float* __restrict__ m, int c0, float& mx,
                                         float& mn) {
  const float4* y4 = reinterpret_cast<const float4*>(y + c0);
  const float4* m4 = reinterpret_cast<const float4*>(m + c0);
  mx = -INFINITY;
  mn = INFINITY;
#pragma unroll 4
  for (int c = 0; c < 16; ++c) {
    const float4 a = y4[c], bq = __ldg(m4 + c);
    float r0, r1, r2, r3;
    sub2(a.x, a.y, bq.x, bq.y, r0, r1);
    sub2(a.z, a.w, bq.z, bq.w, r2, r3);
    mx = max3(mx, r0, r1);
    mn = min3(mn, r0, r1);
    mx = max3(mx, r2, r3);
    mn = min3(mn, r2, r3);
  }
}

__device__ __forceinline__ float dmm_full(const float* __restrict__ y, const float* __restrict__ m) {
  float mx0, mn0, mx1, mn1;
  dmm_half(y, m, 0, mx0, mn0);
  dmm_half(y, m, 64, mx1, mn1);
  return __fsub_rn(fmaxf(mx0, mx1), fminf(mn0, mn1));
}

// Code of one value: q = rne(fl32((R - z) / s)) clamped to [0, maxc].  The quotient comes
// from a multiply by the correctly rounded reciprocal (error < 3e-6 for quotients below 16)
// unless it lies within 1e-5 of a rounding boundary, where the correctly rounded division
// decides.
__device__ __forceinline__ int quant_code(float R, float z, float s, float rinv, int maxc) {
  if (s == 0.0f) return 0;
  const float t = __fsub_rn(R, z);
  const float u = __fmul_rn(t, rinv);
  const float f = __fsub_rn(u, floorf(u));
  float q = rintf(u);
  if (fabsf(f - 0.5f) < 1e-5f) q = rintf(__fdiv_rn(t, s));
  return min(max((int)q, 0), maxc);
}

// Write the 32-bit code words of one block from a shared code matrix X (row-major, ld = cols).
// Elements whose token index is below keep_lo keep their old bits.
__device__ void write_code_block(uint32_t* dst, const uint8_t* X, int ld, int bits, int KS, int keep_lo,
                                 bool cols_are_tokens) {
  const int nwords = kG * kD * bits / 32;
  const int slots = 16 / bits;
  const uint32_t cmask = (1u << bits) - 1u;
  for (int wd = threadIdx.x; wd < nwords; wd += blockDim.x) {
    uint32_t word = 0, keep = 0;
    for (int odd = 0; odd < 2; ++odd)
      for (int sl = 0; sl < slots; ++sl) {
        int row, col;
        frag_elem(bits, KS, wd, sl, odd, row, col);
        const int bit = bits * sl + 16 * odd;
        const int tok = cols_are_tokens ? col : row;
        if (tok < keep_lo) keep |= cmask << bit;
        else word |= ((uint32_t)X[row * ld + col] & cmask) << bit;
      }
    if (keep) word |= dst[wd] & keep;
    dst[wd] = word;
  }
}

__global__ void __launch_bounds__(kAppendThreads) append_pages_kernel(Geom g, AppendWs wsp,
                                                                      const uint16_t* __restrict__ k_new,
                                                                      const uint16_t* __restrict__ v_new,
                                                                      int n_new) {
  PageCtx c;
  if (!page_context(g, n_new, c)) return;
  const int b = blockIdx.z, h = blockIdx.y;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  const int gq = lane >> 2, tig = lane & 3;
  const int P = g.P, Pp = (P + 7) & ~7;

  // staged vectors: rows 0..31 = V page slots, rows 32..63 = K page slots
  constexpr int kLd = kD + 4;
  __shared__ __align__(16) float vec[2 * kG][kLd];
  __shared__ uint8_t vq[kD][kG];  // V codes, [channel][token]
  __shared__ uint8_t kq[kG][kD];  // K codes, [token][channel]
  __shared__ float vs_s[kG][4], vz_s[kG][4], vrow_s[kG], krow_s[kG];
  __shared__ unsigned long long best[2 * kG];  // (d_mm bits << 32) | pattern, per row
  __shared__ float dseed[2 * kG], xinf[2 * kG];
  __shared__ int seed[2 * kG];
  __shared__ uint32_t queue[kQueueCap];
  __shared__ int qn;
  const int lo = c.a - c.pg * kG, hi = c.e - c.pg * kG;  // new slots [lo, hi)
  const size_t shk = ((size_t)c.set * g.H + h) * 2;       // tables: K at shk, V at shk + 1
  auto row_on = [&](int r) { return r < kG ? (r >= lo && r < hi) : c.seal; };

  for (int i = threadIdx.x; i < kD * kG; i += blockDim.x) (&vq[0][0])[i] = 0;
  if (threadIdx.x < kG) {
    for (int q = 0; q < 4; ++q) { vs_s[threadIdx.x][q] = 0.f; vz_s[threadIdx.x][q] = 0.f; }
    vrow_s[threadIdx.x] = 0.f;
  }
  if (threadIdx.x == 0) qn = 0;

  // ---- stage (and pre-transform) every vector: warp per row
  for (int r = warp; r < 2 * kG; r += nwarps) {
    if (!row_on(r)) continue;
    const bool isv = r < kG;
    const int slot = isv ? r : r - kG;
    const int t = c.pg * kG + slot;
    const uint16_t* src;
    if (isv) src = v_new + (((size_t)b * n_new + (t - c.L)) * g.H + h) * kD;
    else src = (t < c.L) ? g.k_tail + (((size_t)b * g.H + h) * kG + slot) * kD
                         : k_new + (((size_t)b * n_new + (t - c.L)) * g.H + h) * kD;
    float y[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) y[k] = load_elem(src + lane + 32 * k, g.dtype);
    float rr = 1.0f;
    if (g.tx) transform_row_warp(y, isv ? c.cV : c.cK, rr, lane);
    float am = 0.f;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      vec[r][lane + 32 * k] = y[k];
      am = fmaxf(am, fabsf(y[k]));
    }
    am = warp_max(am);
    if (lane == 0) {
      xinf[r] = am;
      if (isv) vrow_s[slot] = rr;
      else krow_s[slot] = rr;
    }
  }
  __syncthreads();

  // ---- seed: Euclidean nearest pattern from bf16 MMAs; warp w owns rows 16w .. 16w+15.
  // The MMA k index runs over channels 8(4kp + tig) + e so every lane's operands of a
  // pair of k-steps are 8 consecutive channels (a dot product does not depend on k order).
  {
    const int r0 = 16 * warp;
    bool active = false;
    for (int r = r0; r < r0 + 16; ++r) active |= row_on(r);
    if (active) {
      const size_t o = shk + (r0 < kG ? 1 : 0);
      const __nv_bfloat16* pb = wsp.pb + o * Pp * kPLd;
      const float* msq = wsp.msq + o * Pp;
      uint32_t A[2][4][4];
#pragma unroll
      for (int rh = 0; rh < 2; ++rh)
#pragma unroll
        for (int kp = 0; kp < 4; ++kp) {
          const float4* p = reinterpret_cast<const float4*>(&vec[r0 + 8 * rh + gq][8 * (4 * kp + tig)]);
          const float4 u = p[0], v = p[1];
          A[rh][kp][0] = __byte_perm(__float_as_uint(u.x), __float_as_uint(u.y), 0x7632);
          A[rh][kp][1] = __byte_perm(__float_as_uint(u.z), __float_as_uint(u.w), 0x7632);
          A[rh][kp][2] = __byte_perm(__float_as_uint(v.x), __float_as_uint(v.y), 0x7632);
          A[rh][kp][3] = __byte_perm(__float_as_uint(v.z), __float_as_uint(v.w), 0x7632);
        }
      float bmin[2] = {INFINITY, INFINITY};
      int bj[2] = {0, 0};
      for (int nt = 0; nt < Pp / 8; ++nt) {
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
        const __nv_bfloat16* brow = pb + (size_t)(8 * nt + gq) * kPLd + 8 * tig;
#pragma unroll
        for (int kp = 0; kp < 4; ++kp) {
          const uint4 bv = __ldg(reinterpret_cast<const uint4*>(brow + 32 * kp));
          mma_bf16(acc, A[0][kp][0], A[1][kp][0], A[0][kp][1], A[1][kp][1], bv.x, bv.y);
          mma_bf16(acc, A[0][kp][2], A[1][kp][2], A[0][kp][3], A[1][kp][3], bv.z, bv.w);
        }
        const int j0 = 8 * nt + 2 * tig;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int j = j0 + (q & 1), rh = q >> 1;
          const float e = msq[j] - 2.0f * acc[q];
          if (j < P && e < bmin[rh]) { bmin[rh] = e; bj[rh] = j; }
        }
      }
#pragma unroll
      for (int rh = 0; rh < 2; ++rh) {
#pragma unroll
        for (int m = 1; m <= 2; m <<= 1) {
          const float ob = __shfl_xor_sync(kFull, bmin[rh], m);
          const int oj = __shfl_xor_sync(kFull, bj[rh], m);
          if (ob < bmin[rh] || (ob == bmin[rh] && oj < bj[rh])) { bmin[rh] = ob; bj[rh] = oj; }
        }
        if (tig == 0) seed[r0 + 8 * rh + gq] = bj[rh];
      }
    }
  }
  __syncthreads();

  // ---- exact d_mm of the seed: two threads per row (channel halves)
  {
    const int r = threadIdx.x >> 1, half = threadIdx.x & 1;
    const bool on = row_on(r);
    float mx = -INFINITY, mn = INFINITY;
    if (on) dmm_half(vec[r], (r < kG ? c.MV : c.MK) + (size_t)seed[r] * kD, 64 * half, mx, mn);
    mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 1));
    mn = fminf(mn, __shfl_xor_sync(kFull, mn, 1));
    if (on && half == 0) {
      const float d = __fsub_rn(mx, mn);
      dseed[r] = d;
      best[r] = ((unsigned long long)__float_as_uint(d) << 32) | (uint32_t)seed[r];
    }
  }
  __syncthreads();

  // ---- exact pruning: queue every pattern neither bound can exclude
  {
    const int r = threadIdx.x >> 1, half = threadIdx.x & 1;
    if (row_on(r)) {
      const size_t o = shk + (r < kG ? 1 : 0);
      const int s = seed[r];
      const float ds = dseed[r];
      const float* trow = wsp.tab + o * P * P + (size_t)s * P;
      const float thr = 2.0f * ds + 0x1p-19f * (xinf[r] + wsp.minf[o]);
      const float* M = r < kG ? c.MV : c.MK;
      int pc[kProbe];
      float py[kProbe];
#pragma unroll
      for (int u = 0; u < kProbe; ++u) {
        pc[u] = __ldg(wsp.probe + o * kProbe + u);
        py[u] = vec[r][pc[u]];
      }
      for (int j = half; j < P; j += 2) {
        if (j == s || __ldg(trow + j) > thr) continue;
        // residual range over the probe channels: a lower bound of d_mm(x, m_j), exactly
        const float* m = M + (size_t)j * kD;
        float hi = -INFINITY, lo = INFINITY;
#pragma unroll
        for (int u = 0; u < kProbe; ++u) {
          const float rr = __fsub_rn(py[u], __ldg(m + pc[u]));
          hi = fmaxf(hi, rr);
          lo = fminf(lo, rr);
        }
        const float lb = __fsub_rn(hi, lo);
        if (lb > ds || (lb == ds && j > s)) continue;
        const int pos = atomicAdd(&qn, 1);
        if (pos < kQueueCap) queue[pos] = ((uint32_t)r << 16) | (uint32_t)j;
      }
    }
  }
  __syncthreads();

  // ---- exact d_mm of the candidates; (distance, index) minimum per row
  if (qn <= kQueueCap) {
    for (int i = threadIdx.x; i < qn; i += blockDim.x) {
      const uint32_t e = queue[i];
      const int r = e >> 16, j = e & 0xffff;
      const float d = dmm_full(vec[r], (r < kG ? c.MV : c.MK) + (size_t)j * kD);
      atomicMin(&best[r], ((unsigned long long)__float_as_uint(d) << 32) | (uint32_t)j);
    }
  } else {
    // the bound excluded too little: every pattern for every row, two threads per row
    const int r = threadIdx.x >> 1, half = threadIdx.x & 1;
    if (row_on(r)) {
      const float* M = r < kG ? c.MV : c.MK;
      for (int j = half; j < P; j += 2) {
        const float d = dmm_full(vec[r], M + (size_t)j * kD);
        atomicMin(&best[r], ((unsigned long long)__float_as_uint(d) << 32) | (uint32_t)j);
      }
    }
  }
  __syncthreads();

  // ---- residuals in place: R = y - M[k*], warp per row
  for (int r = warp; r < 2 * kG; r += nwarps) {
    if (!row_on(r)) continue;
    const float* m = (r < kG ? c.MV : c.MK) + (size_t)(best[r] & 0xffffffffu) * kD;
#pragma unroll
    for (int k = 0; k < 4; ++k) vec[r][lane + 32 * k] = __fsub_rn(vec[r][lane + 32 * k], __ldg(m + lane + 32 * k));
  }
  __syncthreads();

  // ---- V: per-token group quantization, warp per token
  for (int slot = lo + warp; slot < hi; slot += nwarps) {
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float R = vec[slot][lane + 32 * k];
      const float mn = warp_min(R), mx = warp_max(R);
      const float s = __fdiv_rn(__fsub_rn(mx, mn), (float)((1 << g.bits) - 1));
      const float rinv = s != 0.0f ? __frcp_rn(s) : 0.0f;
      vq[lane + 32 * k][slot] = (uint8_t)quant_code(R, mn, s, rinv, (1 << g.bits) - 1);
      if (lane == 0) { vs_s[slot][k] = s; vz_s[slot][k] = mn; }
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
        R[t] = vec[kG + t][d];
        mn = fminf(mn, R[t]);
        mx = fmaxf(mx, R[t]);
      }
      const float s = __fdiv_rn(__fsub_rn(mx, mn), (float)((1 << g.bits) - 1));
      const float rinv = s != 0.0f ? __frcp_rn(s) : 0.0f;
#pragma unroll
      for (int t = 0; t < kG; ++t) kq[t][d] = (uint8_t)quant_code(R[t], mn, s, rinv, (1 << g.bits) - 1);
      ks_g[ksc_pos(d)] = s;
      kz_g[ksc_pos(d)] = mn;
    }
  }
  __syncthreads();

  // ---- stores
  write_code_block(reinterpret_cast<uint32_t*>(c.sub + g.off_vc), &vq[0][0], kG, g.bits, 2, c.fresh ? 0 : lo, true);
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
    const bool present = slot >= lo && slot < hi;
    if (c.fresh || present) {
      vidx_g[tok_pos(slot)] = present ? (uint8_t)(best[slot] & 0xff) : (uint8_t)0;
      if (g.tx) vrow_g[tok_pos(slot)] = vrow_s[slot];
    }
  }
  if (c.seal) {
    write_code_block(reinterpret_cast<uint32_t*>(c.sub), &kq[0][0], kD, g.bits, 8, 0, false);
    uint8_t* kidx_g = c.sub + g.off_kidx;
    float* krow_g = reinterpret_cast<float*>(c.sub + g.off_krow);
    for (int slot = threadIdx.x; slot < kG; slot += blockDim.x) {
      kidx_g[tok_pos(slot)] = (uint8_t)(best[kG + slot] & 0xff);
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
    const int t = t0 + i / per_tok, rem = i % per_tok;
    const int h = rem / kD, d = rem % kD;
    g.k_tail[(((size_t)b * g.H + h) * kG + (t % kG)) * kD + d] =
        k_new[(((size_t)b * n_new + (t - L)) * g.H + h) * kD + d];
  }
  __syncthreads();
  if (threadIdx.x == 0) g.seq_len[b] = newL;
}

}  // namespace

size_t append_workspace(const Geom& g) {
  const int Pp = (g.P + 7) & ~7;
  return al256((size_t)g.S * g.H * 2 * Pp * kPLd * 2) + al256((size_t)g.S * g.H * 2 * Pp * 4) +
         al256((size_t)g.S * g.H * 2 * g.P * g.P * 4) + al256((size_t)g.S * g.H * 2 * 4) +
         al256((size_t)g.S * g.H * 2 * kProbe * 4) + 256;
}

cudaError_t launch_append(const Geom& g, const void* k_new, const void* v_new, int n_new, void* ws, cudaStream_t st) {
  if (n_new <= 0 || g.B == 0) return cudaSuccess;
  AppendWs w = carve_append(ws, g.S, g.H, g.P);
  const size_t prep_smem = (size_t)g.P * (kD + 4) * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(append_prep_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)prep_smem);
  if (e != cudaSuccess) return e;
  append_prep_kernel<<<dim3(g.S * g.H, 2), 256, prep_smem, st>>>(g, w);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  dim3 grid(n_new / kG + 2, g.H, g.B);
  append_pages_kernel<<<grid, kAppendThreads, 0, st>>>(g, w, (const uint16_t*)k_new, (const uint16_t*)v_new, n_new);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  append_tail_kernel<<<g.B, 256, 0, st>>>(g, (const uint16_t*)k_new, n_new);
  return cudaGetLastError();
}

}  // namespace kvq
