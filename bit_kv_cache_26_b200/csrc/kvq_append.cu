// Quantize-append: align each new K/V vector to its nearest pattern under the
// min-max distance, quantize the residual per group and store it in the paged
// cache ("PatternKV", Section 3.2 and Eq. 6; Eq. 1; granularity of Section 4.1).
//
// Launch 0 (prep, per call): for every (set, KV head) and K / V pattern set, the 32
//   probe channels (those whose values differ most across the patterns, in that order) and
//   every pattern's values there.
// Launch 1 (page tasks): one CTA per (touched page, KV head, sequence).
//   * the new V vectors of the page and, when the page's 32nd token arrives, its 32
//     K vectors (older ones from the K tail) are staged in shared memory (after the
//     pre-transform, if enabled);
//   * an exact lower bound of d_mm(y, m_j) for every pattern: max and min only grow
//     with the channel set, so the residual range over the probe channels (the first 16
//     for K, all 32 for V) never exceeds the range over all channels (same fp32
//     subtractions, no rounding of its own); one lane per vector, every pattern;
//   * the pattern with the smallest bound is the seed; its exact d_mm is an upper bound
//     of the minimum, and every pattern whose bound already exceeds it (or equals it
//     with a higher index) is excluded exactly;
//   * the few remaining (vector, pattern) pairs go through a shared work queue and are
//     evaluated exactly, channel block by channel block, stopping as soon as the partial
//     range rules the pattern out; the exact distances meet in a 64-bit (distance,
//     index) atomic minimum, so the lowest index wins ties as in the definition;
//   * residuals, fp32 scale / zero per group, then every 32-bit code word of the page
//     computed by one thread straight from the residuals (the correctly rounded
//     division decides wherever the fast quotient could change a code), and stores.
// Launch 2 (tail + commit): one CTA per sequence writes the keys of the newest,
//   incomplete group into the K tail and advances seq_len.  Splitting launches 1 and
//   2 keeps every tail read ahead of every tail write.
#include <algorithm>

#include <cuda_fp16.h>

#include "kvq_common.cuh"
#include "kvq_internal.h"

namespace kvq {

namespace {

constexpr int kAppendThreads = 128;
constexpr int kQueueCap = 2048;  // candidate (row, pattern) entries of a page; more: every pattern for every row
constexpr int kProbe = 32;   // probe channels stored per pattern set (by decreasing spread)
constexpr int kProbeK = 16;  // used for K rows (outlier channels make 16 enough) ...
constexpr int kProbeKtx = 32;  // ... but not after the Hadamard rotation, which spreads them
constexpr int kProbeV = 32;  // used for V rows (a tighter bound picks a better seed)
constexpr int kLd = kD + 4;  // staged row stride (floats): 16-byte aligned, conflict-free columns

struct AppendWs {
  int32_t* probe;  // [S][H][2][kProbe] probe channels (0 = K, 1 = V)
  float* pv;       // [S][H][2][P][kProbe] pattern values at the probe channels
};

__host__ __device__ inline size_t al256(size_t v) { return (v + 255) & ~size_t(255); }

inline AppendWs carve_append(void* ws, int S, int H, int P) {
  uint8_t* p = (uint8_t*)ws;
  AppendWs w;
  w.probe = (int32_t*)p; p += al256((size_t)S * H * 2 * kProbe * 4);
  w.pv = (float*)p;
  return w;
}

// ---- launch 0: probe channels and pattern values there, per (set, head, K|V) ----------
__global__ void __launch_bounds__(kD) append_prep_kernel(Geom g, AppendWs w) {
  const int sh = blockIdx.x, kv = blockIdx.y;  // sh = set * H + head
  const int P = g.P, Pe = p_eff(g, sh);  // table strides use the capacity P, contents the Pe patterns in use
  const float* M = (kv ? g.vpat : g.kpat) + (size_t)sh * P * kD;
  const size_t o = (size_t)sh * 2 + kv;
  __shared__ float spread[kD];
  __shared__ int pcs[kProbe];
  const int d = threadIdx.x;
  float hi = -INFINITY, lo = INFINITY;
  for (int j = 0; j < Pe; ++j) {
    const float m = M[(size_t)j * kD + d];
    hi = fmaxf(hi, m);
    lo = fminf(lo, m);
  }
  spread[d] = hi - lo;
  __syncthreads();
  // rank of channel d by decreasing spread (ties: lower channel first)
  int rank = 0;
  for (int e = 0; e < kD; ++e) rank += (spread[e] > spread[d]) || (spread[e] == spread[d] && e < d);
  if (rank < kProbe) {
    w.probe[o * kProbe + rank] = d;
    pcs[rank] = d;
  }
  __syncthreads();
  float* pv = w.pv + o * P * kProbe;
  for (int i = threadIdx.x; i < Pe * kProbe; i += blockDim.x) pv[i] = M[(size_t)(i / kProbe) * kD + pcs[i % kProbe]];
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

// Returns false if the CTA has nothing to do (or an error was flagged).  CTA x takes the x-th
// page the call touches.
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

// Exact partial max / min of y - m over channels [c0, c0 + 32) (y staged, m global).
__device__ __forceinline__ void range32(const float* __restrict__ y, const float* __restrict__ m, int c0, float& mx,
                                        float& mn) {
  const float4* y4 = reinterpret_cast<const float4*>(y + c0);
  const float4* m4 = reinterpret_cast<const float4*>(m + c0);
#pragma unroll
  for (int c = 0; c < 8; ++c) {
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

// Exact partial max / min of y - m over the 64 channels [c0, c0 + 64), its 16-byte chunks
// taken from chunk `rot` on (wrapping), so that two threads reading the two halves of one
// staged row (rot 0 and 1) hit different shared-memory banks.
__device__ __forceinline__ void range64(const float* __restrict__ y, const float* __restrict__ m, int c0, int rot,
                                        float& mx, float& mn) {
  const float4* y4 = reinterpret_cast<const float4*>(y + c0);
  const float4* m4 = reinterpret_cast<const float4*>(m + c0);
#pragma unroll
  for (int k = 0; k < 16; ++k) {
    const int c = (k + rot) & 15;
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

__device__ __forceinline__ unsigned long long dkey(float d, int j) {
  return ((unsigned long long)__float_as_uint(d) << 32) | (uint32_t)j;
}

// Two codes q = rne(fl32((R - z) / s)), returned as (q0 | q1 << 16).  The quotients come
// from a multiply by the correctly rounded reciprocal (error below 2^-19 for quotients below
// 16), rounded to an integer by adding 1.5 * 2^23 (the integer is then the low mantissa
// bits); a quotient within 1e-5 of a rounding boundary is recomputed with the correctly
// rounded division.  R >= z and, for a normal scale, the quotient stays below maxc + 2^-19;
// the division's result is clamped to maxc (a subnormal scale carries less precision); s == 0
// gives rinv == 0 and code 0.
template <int BITS>
__device__ __forceinline__ uint32_t code_pair(float R0, float R1, float z0, float z1, float ri0, float ri1,
                                              const float* s2) {
  constexpr float kMaxc = (float)((1 << BITS) - 1);
  constexpr float kShift = 12582912.0f;  // 1.5 * 2^23
  float t0, t1, u0, u1, v0, v1, b0, b1, e0, e1;
  sub2(R0, R1, z0, z1, t0, t1);
  mul2f(t0, t1, ri0, ri1, u0, u1);
  add2f(u0, u1, kShift, kShift, v0, v1);
  sub2(v0, v1, kShift, kShift, b0, b1);
  sub2(u0, u1, b0, b1, e0, e1);  // u - rne(u), exact
  // near a rounding boundary, or not finite (a scale so small that 1/s overflows): the
  // correctly rounded division; the comparisons are written so that NaN selects it
  const bool f0 = !(fabsf(e0) <= 0.5f - 1e-5f), f1 = !(fabsf(e1) <= 0.5f - 1e-5f);
  if (f0 || f1) {
    if (f0) v0 = __fadd_rn(fminf(rintf(__fdiv_rn(t0, s2[0])), kMaxc), kShift);
    if (f1) v1 = __fadd_rn(fminf(rintf(__fdiv_rn(t1, s2[1])), kMaxc), kShift);
  }
  return __byte_perm(__float_as_uint(v0), __float_as_uint(v1), 0x5410) & 0x00FF00FFu;
}

// One 32-bit code word of the V block (rows = channels, 2 column tiles of 16 tokens) from
// the staged residuals Rv[token][channel] and per-(group, token) s / z / 1/s.  Tokens below
// keep_lo keep their bits from `old`; tokens at or above tok_hi get code 0.
template <int BITS, bool MASK>
__device__ __forceinline__ uint32_t v_word(int wd, const float (*Rv)[kLd], const float* vs, const float* vz,
                                           const float* vr, int keep_lo, int tok_hi, uint32_t old) {
  constexpr int SPW = 16 / BITS, maxc = (1 << BITS) - 1;
  const int ln = (wd & 127) >> 2, gq = ln >> 2, tig = ln & 3;
  const int w = (wd >> 7) * 4 + (wd & 3);
  uint32_t word = 0;
#pragma unroll
  for (int slot = 0; slot < SPW; ++slot) {
    const int tile = (SPW * w + slot) >> 2, r = slot & 3;
    const int ch = 16 * (tile >> 1) + 8 * (r & 1) + gq;
    const int tok = 16 * (tile & 1) + 8 * (r >> 1) + 2 * tig;
    const int gi = (ch >> 5) * kG + tok;
    const float2 z = *reinterpret_cast<const float2*>(vz + gi);
    const float2 ri = *reinterpret_cast<const float2*>(vr + gi);
    const uint32_t c01 = code_pair<BITS>(Rv[tok][ch], Rv[tok + 1][ch], z.x, z.y, ri.x, ri.y, vs + gi);
    const int b0 = BITS * slot, b1 = b0 + 16;
    if constexpr (MASK) {
      const uint32_t c0 = c01 & 0xffu, c1 = c01 >> 16;
      word |= (tok < keep_lo ? (old >> b0) & maxc : tok < tok_hi ? c0 : 0u) << b0;
      word |= (tok + 1 < keep_lo ? (old >> b1) & maxc : tok + 1 < tok_hi ? c1 : 0u) << b1;
    } else {
      word |= c01 << b0;
    }
  }
  return word;
}

// Halves per row of the fp16 lower-bound table [64 rows][.]: an odd number of 32-bit words, so
// that 32 consecutive rows (the bound pass, a lane a row) and 16 rows x 2 pattern halves (the
// candidate scan) fall in different banks.
__host__ __device__ inline int lb_ld(int P) { return 2 * (((P + 1) >> 1) | 1); }

// ---- codes of whole pages: one FMA per code, 16-bit codes staged row-major, words by ldmatrix
// A code is rne(fl32(fl32(R - z) / s)).  v = t (1/s) + (1.5 * 2^7 + 1/2) with t = R - z in
// [0, maxc s] stays in [128, 256): its bits 16-22 hold 64 + the code and bits 0-15 the fraction.
// v differs from the exact t / s + 1/2 by less than 2^-17 (its own rounding) + 15 * 2^-24 (the
// reciprocal's), under one fraction step; so the code can be wrong, or the quotient a tie that
// rounds to even, only when the fraction is 0x0000 or 0xFFFF (about 2 codes in 65536).  Those
// units, and every unit with a scale below 2^-125 (whose reciprocal is not within 2^-24 of
// 1 / s, or overflows), are recomputed with the correctly rounded division.
constexpr float kCodeMagic = 192.5f;    // 1.5 * 2^7 + 1/2: 16 fraction bits, +1/2 folded in
constexpr float kMinScale = 0x1p-125f;  // below this (and nonzero) 1 / s is not within 2^-24 of exact

__device__ __forceinline__ uint32_t vmin_u16x2(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("min.u16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}
__device__ __forceinline__ bool tiny_scale(float s) { return s != 0.0f && s < kMinScale; }
// Codes of N residuals as N / 2 words of two 16-bit halves (the code in bits 8-11 of each half:
// byte 2 of the FMA result, 0x40 | code); zr(i, z0, z1, r0, r1) gives the zeros and reciprocal
// scales of values 2i, 2i + 1.  Returns true if no fraction is 0x0000 or 0xFFFF.
template <int N, class ZR>
__device__ __forceinline__ bool codes_fma(const float (&x)[N], uint32_t (&p)[N / 2], ZR zr) {
  uint32_t acc = 0xFFFFFFFFu;  // per half: min over the pairs of (fraction + 1) mod 2^16
#pragma unroll
  for (int i = 0; i < N / 2; ++i) {
    float z0, z1, r0, r1, t0, t1, v0, v1;
    zr(i, z0, z1, r0, r1);
    sub2(x[2 * i], x[2 * i + 1], z0, z1, t0, t1);
    fma2f(t0, t1, r0, r1, kCodeMagic, kCodeMagic, v0, v1);
    const uint32_t u0 = __float_as_uint(v0), u1 = __float_as_uint(v1);
    p[i] = __byte_perm(u0, u1, 0x6420);
    // a carry out of the low half only happens when that half is flagged anyway
    acc = vmin_u16x2(acc, __byte_perm(u0, u1, 0x5410) + 0x00010001u);
  }
  return (acc & 0x0000FFFEu) != 0u && (acc & 0xFFFE0000u) != 0u;
}
// Byte offset of channel ch (0..127) of row `row` in a 16-bit code buffer of two 64-channel
// halves of 32 rows x 128 B, 16-byte chunks XOR-swizzled by (row & 7) (conflict-free ldmatrix).
__device__ __forceinline__ uint32_t cb_off(int row, int ch) {
  return (uint32_t)((ch >> 6) * 4096 + row * 128 + ((((ch & 63) >> 3) ^ (row & 7)) << 4) + (ch & 7) * 2);
}
// The rare paths (a fraction of 0x0000 / 0xFFFF somewhere, or a scale below 2^-125): the
// unit's codes by the definition (the correctly rounded quotient, round half to even, clamp),
// written as 16-bit codes; out of line, reading the residuals from shared memory.
// V: the 32 residuals y of row `row`, channels c0 .., zero z, scale s.
__device__ __noinline__ void v_codes_exact(const float* y, float z, float s, int maxc, uint8_t* cb, int row, int c0) {
  for (int i = 0; i < 32; ++i) {
    uint32_t c = 0u;
    if (s != 0.0f) c = (uint32_t)min(max(__float2int_rn(__fdiv_rn(__fsub_rn(y[i], z), s)), 0), maxc);
    *reinterpret_cast<uint16_t*>(cb + cb_off(row, c0 + i)) = (uint16_t)(c << 8);
  }
}
// K: channels 4 cbk + 32 k .. + 3 (k = 0..3) of residual row y, zero kz[c], scale ks[c].
__device__ __noinline__ void k_codes_exact(const float* y, const float* kz, const float* ks, int cbk, int maxc,
                                           uint8_t* cb, int row) {
  for (int i = 0; i < 16; ++i) {
    const int c = 4 * cbk + 32 * (i >> 2) + (i & 3);
    const float s = ks[c];
    uint32_t code = 0u;
    if (s != 0.0f) code = (uint32_t)min(max(__float2int_rn(__fdiv_rn(__fsub_rn(y[c], kz[c]), s)), 0), maxc);
    *reinterpret_cast<uint16_t*>(cb + cb_off(row, c)) = (uint16_t)(code << 8);
  }
}
__device__ __forceinline__ uint32_t su32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }
__device__ __forceinline__ void ldsm4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm4t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
// Words 4 wq .. 4 wq + 3 of every lane of a page's code block from a 16-bit code buffer
// ([32 tokens][128 channels], cb_off layout): the MMA fragment order of include/kvq.h, the
// V block (isV) with rows = channels (a transposed ldmatrix), the K block with rows = tokens.
__device__ __forceinline__ uint4 pack_chunk(const uint8_t* cb, bool isV, int bits, int wq, int lane) {
  const int mi = lane >> 3, ri8 = lane & 7;
  uint32_t wd[4] = {0u, 0u, 0u, 0u};
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int w = 4 * wq + u;
#pragma unroll
    for (int tt = 0; tt < 2; ++tt) {
      if (bits == 4 && tt == 1) continue;
      const int tile = bits == 2 ? 2 * w + tt : w;
      int rt, ct;  // row tile (16 rows of the code matrix) and column tile
      if (isV) { rt = tile >> 1; ct = tile & 1; }  // V: rows = channels, 2 column tiles of tokens
      else { rt = tile >> 3; ct = tile & 7; }      // K: rows = tokens, 8 column tiles of channels
      uint32_t a0, a1, a2, a3;
      if (isV) {
        const int tok = 16 * ct + 8 * (mi >> 1) + ri8, ch = 16 * rt + 8 * (mi & 1);
        ldsm4t(su32(cb) + cb_off(tok, ch), a0, a1, a2, a3);
      } else {
        const int tok = 16 * rt + 8 * (mi & 1) + ri8, ch = 16 * ct + 8 * (mi >> 1);
        ldsm4(su32(cb) + cb_off(tok, ch), a0, a1, a2, a3);
      }
      const uint32_t av[4] = {a0, a1, a2, a3};
#pragma unroll
      for (int rg = 0; rg < 4; ++rg) {
        if (bits == 2) {
          const int sl = 4 * tt + rg;  // 2-bit slot: codes at bits 2 sl and 16 + 2 sl
          const uint32_t v = av[rg] & 0x03000300u;
          wd[u] |= sl < 4 ? v >> (8 - 2 * sl) : v << (2 * sl - 8);
        } else {
          const int sl = rg;  // 4-bit slot: codes at bits 4 sl and 16 + 4 sl
          const uint32_t v = av[rg] & 0x0F000F00u;
          wd[u] |= sl < 2 ? v >> (8 - 4 * sl) : v << (4 * sl - 8);
        }
      }
    }
  }
  return make_uint4(wd[0], wd[1], wd[2], wd[3]);
}

// Lower bounds over the NPROBE probe channels pc (shared memory) for patterns [j0, j1) of one
// staged vector y (one lane), from the patterns' values there (shared memory, [P][NPROBE]);
// written to lbuf[row][j] rounded toward zero to fp16 (still a lower bound); running argmin
// of the fp32 bounds (ties: lowest j) to (blb, bj).
template <int NPROBE>
__device__ __forceinline__ void lb_pass(const float* y, const int32_t* pc, const float* pvt, int j0, int j1,
                                        __half* lbuf, int ldh, int row, float& blb_out, int& bj_out) {
  float py[NPROBE];
#pragma unroll
  for (int u = 0; u < NPROBE; ++u) py[u] = y[pc[u]];
  float blb = INFINITY;
  int bj = j0;
#pragma unroll 2
  for (int j = j0; j < j1; ++j) {
    const float4* m4 = reinterpret_cast<const float4*>(pvt + (size_t)j * NPROBE);
    float mx = -INFINITY, mn = INFINITY;
#pragma unroll
    for (int q = 0; q < NPROBE / 4; ++q) {
      const float4 m = m4[q];
      float r0, r1, r2, r3;
      sub2(py[4 * q], py[4 * q + 1], m.x, m.y, r0, r1);
      sub2(py[4 * q + 2], py[4 * q + 3], m.z, m.w, r2, r3);
      mx = max3(mx, r0, r1);
      mn = min3(mn, r0, r1);
      mx = max3(mx, r2, r3);
      mn = min3(mn, r2, r3);
    }
    const float lb = __fsub_rn(mx, mn);
    lbuf[row * ldh + j] = __float2half_rz(lb);
    if (lb < blb) { blb = lb; bj = j; }
  }
  blb_out = blb;
  bj_out = bj;
}

// fp32 scale / zero / reciprocal of a group from its min and max
__device__ __forceinline__ void group_sz(float mn, float mx, int bits, float& s, float& z, float& rinv) {
  s = __fdiv_rn(__fsub_rn(mx, mn), (float)((1 << bits) - 1));
  z = mn;
  rinv = s != 0.0f ? __frcp_rn(s) : 0.0f;
}

__global__ void __launch_bounds__(kAppendThreads, 4) append_pages_kernel(Geom g, AppendWs wsp,
                                                                         const uint16_t* __restrict__ k_new,
                                                                         const uint16_t* __restrict__ v_new,
                                                                         int n_new) {
  PageCtx c;
  if (!page_context(g, n_new, c)) return;
  const int b = blockIdx.z, h = blockIdx.y;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nwarps = blockDim.x >> 5;
  const int P = g.P;                          // capacity: the layout of the tables
  const int Pe = p_eff(g, c.set * g.H + h);   // patterns in use

  // staged vectors: rows 0..31 = V page slots, rows 32..63 = K page slots
  __shared__ __align__(16) float vec[2 * kG][kLd];
  __shared__ float vrow_s[kG], krow_s[kG];
  __shared__ unsigned long long best[2 * kG];  // (d_mm bits << 32) | pattern, per row
  __shared__ float dseed[2 * kG], hlb[2][2 * kG];
  __shared__ float rraw[kG];      // V rows: range max - min of the vector (adaptive threshold)
  __shared__ bool vkeep[kG];      // V rows: the pattern is kept (else quantized raw, index 255)
  __shared__ int seed[2 * kG], hj[2][2 * kG];
  __shared__ int qn;
  // dynamic: fp16 lower bounds lb[row][j], then the probe tables (V: [P][32], K: [P][16]) and
  // probe channels (32 + 16), whose region holds the work queue once the bounds are done;
  // after the assignment the s / z / 1/s tables and the 16-bit code buffers reuse the region
  extern __shared__ __align__(16) float dsm[];
  const int ldh = lb_ld(P);
  __half* lbuf = reinterpret_cast<__half*>(dsm);  // [64 rows][ldh]
  float* tabV = dsm + 32 * ldh;
  const int nprk = g.tx ? kProbeKtx : kProbeK;  // K probe channels
  float* tabK = tabV + kProbeV * P;
  int32_t* pcV = reinterpret_cast<int32_t*>(tabK + nprk * P);
  int32_t* pcK = pcV + kProbeV;
  uint32_t* queue = reinterpret_cast<uint32_t*>(tabV);  // [kQueueCap]
  float* vsz = dsm;            // [3][4][kG]: s, z, 1/s per (group, V slot)
  float* ksz = dsm + 12 * kG;  // [3][kD]:   s, z, 1/s per K channel
  uint8_t* cbV = reinterpret_cast<uint8_t*>(dsm + 1024);  // 16-bit V codes [32 tokens][128], cb_off layout
  uint8_t* cbK = cbV + 8192;                              // 16-bit K codes
  __shared__ int ktiny;  // some K scale of the page is below 2^-125

  const int lo = c.a - c.pg * kG, hi = c.e - c.pg * kG;  // new slots [lo, hi)
  const size_t shk = ((size_t)c.set * g.H + h) * 2;       // tables: K at shk, V at shk + 1
  auto row_on = [&](int r) { return r < kG ? (r >= lo && r < hi) : c.seal; };
  auto row_src = [&](int r) -> const uint16_t* {
    const int slot = r < kG ? r : r - kG;
    const int t = c.pg * kG + slot;
    if (r < kG) return v_new + (((size_t)b * n_new + (t - c.L)) * g.H + h) * kD;
    return (t < c.L) ? g.k_tail + (((size_t)b * g.H + h) * kG + slot) * kD
                     : k_new + (((size_t)b * n_new + (t - c.L)) * g.H + h) * kD;
  };
  if (tid == 0) qn = 0;
  {
    // probe tables of this (set, head): V's 32 probe channels, K's first nprk
    const float4* gV = reinterpret_cast<const float4*>(wsp.pv + (shk + 1) * P * kProbe);
    const float* gK = wsp.pv + shk * P * kProbe;
    const int nk4 = nprk / 4;
#pragma unroll 4
    for (int i = tid; i < Pe * (kProbeV / 4); i += kAppendThreads) reinterpret_cast<float4*>(tabV)[i] = __ldg(gV + i);
#pragma unroll 2
    for (int i = tid; i < Pe * nk4; i += kAppendThreads)
      reinterpret_cast<float4*>(tabK)[i] =
          __ldg(reinterpret_cast<const float4*>(gK + (size_t)(i / nk4) * kProbe) + i % nk4);
    if (tid < kProbeV) pcV[tid] = __ldg(wsp.probe + (shk + 1) * kProbe + tid);
    if (tid < nprk) pcK[tid] = __ldg(wsp.probe + shk * kProbe + tid);
  }

  // ---- stage (and pre-transform) every vector: 16 threads per row, 8 channels (one 16-byte
  // load) each, all loads issued first
  {
    uint4 raw[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int r = (tid >> 4) + 8 * u;
      if (row_on(r)) raw[u] = __ldg(reinterpret_cast<const uint4*>(row_src(r) + 8 * (tid & 15)));
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int r = (tid >> 4) + 8 * u;
      if (!row_on(r)) continue;
      const uint32_t wv[4] = {raw[u].x, raw[u].y, raw[u].z, raw[u].w};
      float f[8];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        f[2 * k] = bits_to_float((uint16_t)(wv[k] & 0xffffu), g.dtype);
        f[2 * k + 1] = bits_to_float((uint16_t)(wv[k] >> 16), g.dtype);
      }
      float4* dst = reinterpret_cast<float4*>(&vec[r][8 * (tid & 15)]);
      dst[0] = make_float4(f[0], f[1], f[2], f[3]);
      dst[1] = make_float4(f[4], f[5], f[6], f[7]);
    }
  }
  if (g.tx) {
    // in place, two staged rows per warp at a time: Hadamard rotation and the fitted column / row
    // normalisation (rows the call does not touch are transformed too and not kept)
    __syncthreads();
    for (int r0 = warp; r0 < 2 * kG; r0 += 2 * nwarps) {
      const int rs[2] = {r0, r0 + nwarps};
      float y[2][4], rr[2];
      const float* cq[2] = {rs[0] < kG ? c.cV : c.cK, rs[1] < kG ? c.cV : c.cK};
#pragma unroll
      for (int q = 0; q < 2; ++q)
#pragma unroll
        for (int k = 0; k < 4; ++k) y[q][k] = row_on(rs[q]) ? vec[rs[q]][lane + 32 * k] : 0.f;
      transform_rows_warp<2>(y, cq, rr, lane);
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        if (!row_on(rs[q])) continue;
#pragma unroll
        for (int k = 0; k < 4; ++k) vec[rs[q]][lane + 32 * k] = y[q][k];
        if (lane == 0) {
          if (rs[q] < kG) vrow_s[rs[q]] = rr[q];
          else krow_s[rs[q] - kG] = rr[q];
        }
      }
    }
  }
  __syncthreads();

  // ---- probe-channel lower bounds: warp (kind = warp & 1: 0 V, 1 K; half = warp >> 1),
  // lane = row; patterns split in two halves.  Running argmin per half (ties: lowest j).
  const int P0 = (Pe + 1) >> 1;
  {
    const int kind = warp & 1, half = warp >> 1;
    const int r = kind * kG + lane;
    if (kind == 0)
      lb_pass<kProbeV>(vec[r], pcV, tabV, half ? P0 : 0, half ? Pe : P0, lbuf, ldh, r, hlb[half][r], hj[half][r]);
    else if (c.seal)
      g.tx ? lb_pass<kProbeKtx>(vec[r], pcK, tabK, half ? P0 : 0, half ? Pe : P0, lbuf, ldh, r, hlb[half][r], hj[half][r])
           : lb_pass<kProbeK>(vec[r], pcK, tabK, half ? P0 : 0, half ? Pe : P0, lbuf, ldh, r, hlb[half][r], hj[half][r]);
    if (kind == 0 || c.seal) {
      // the half's best pattern is the likely seed: its row into L1 ahead of the exact range
      const float* mrow = (kind ? c.MK : c.MV) + (size_t)min(max(hj[half][r], 0), Pe - 1) * kD;
#pragma unroll
      for (int u = 0; u < 4; ++u) asm volatile("prefetch.global.L1 [%0];" ::"l"(mrow + 32 * u));
    }
  }
  __syncthreads();

  // ---- seed = smallest bound; its exact d_mm, two threads per row (channel halves); then the
  // warp's 16 rows queue the patterns whose bound does not exclude them (lane: row 16 w + (lane &
  // 15), pattern half lane >> 4, the row's seed and distance by shuffle)
  {
    const int r = tid >> 1, hh = tid & 1;
    const bool on = row_on(r);
    int s = 0;
    float mx = -INFINITY, mn = INFINITY, ymx = -INFINITY, ymn = INFINITY;
    if (on) {
      s = hlb[1][r] < hlb[0][r] ? hj[1][r] : hj[0][r];
      s = min(max(s, 0), Pe - 1);
      const float* m = (r < kG ? c.MV : c.MK) + (size_t)s * kD;
      range64(vec[r], m, 64 * hh, hh, mx, mn);
      if (r < kG && g.vrho > 0.0f) {  // the V vector's own range, for the adaptive threshold
        const float4* y4 = reinterpret_cast<const float4*>(vec[r] + 64 * hh);
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          const float4 a = y4[k];
          ymx = max3(ymx, a.x, a.y);
          ymn = min3(ymn, a.x, a.y);
          ymx = max3(ymx, a.z, a.w);
          ymn = min3(ymn, a.z, a.w);
        }
      }
    }
    mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 1));
    mn = fminf(mn, __shfl_xor_sync(kFull, mn, 1));
    ymx = fmaxf(ymx, __shfl_xor_sync(kFull, ymx, 1));
    ymn = fminf(ymn, __shfl_xor_sync(kFull, ymn, 1));
    if (on && hh == 0 && r < kG) rraw[r] = __fsub_rn(ymx, ymn);
    const float ds = __fsub_rn(mx, mn);
    if (on && hh == 0) {
      dseed[r] = ds;
      seed[r] = s;
      best[r] = dkey(ds, s);
    }
    const int src = 2 * (lane & 15);
    const int r2 = 16 * warp + (lane & 15), hh2 = lane >> 4;
    const float ds2 = __shfl_sync(kFull, ds, src);
    const int s2 = __shfl_sync(kFull, s, src);
    if (row_on(r2)) {
      // a pattern is left out only when its bound (fp16, rounded toward zero) exceeds the seed's
      // distance rounded up to fp16, so its d_mm is above the seed's; ties and near-ties go to
      // the exact comparison.  Two bounds (one 4-byte word: the row stride is even) per compare.
      const __half dsh = __float2half_ru(ds2);
      const __half2 dsh2 = __half2half2(dsh);
      const __half* lrow = lbuf + r2 * ldh;
      auto push = [&](int jj) {
        if (jj == s2) return;
        const int pos = atomicAdd(&qn, 1);
        if (pos < kQueueCap) queue[pos] = ((uint32_t)r2 << 16) | (uint32_t)jj;
      };
      int j = hh2 ? P0 : 0;
      const int j1 = hh2 ? Pe : P0;
      if ((j & 1) && j < j1) {
        if (!__hgt(lrow[j], dsh)) push(j);
        ++j;
      }
#pragma unroll 4
      for (; j + 2 <= j1; j += 2) {
        const unsigned gt = __hgt2_mask(*reinterpret_cast<const __half2*>(lrow + j), dsh2);
        if (!(gt & 0xFFFFu)) push(j);
        if (!(gt >> 16)) push(j + 1);
      }
      if (j < j1 && !__hgt(lrow[j], dsh)) push(j);
    }
  }
  __syncthreads();

  // ---- exact d_mm of the survivors, 32-channel blocks, stopping once a block's partial
  // range excludes the pattern; (distance, index) minimum per row
  if (qn <= kQueueCap) {
    for (int i = tid; i < qn; i += blockDim.x) {
      const uint32_t e = queue[i];
      const int r = e >> 16, j = e & 0xffff;
      const float* m = (r < kG ? c.MV : c.MK) + (size_t)j * kD;
      const float ds = dseed[r];
      const int s = seed[r];
      float mx = -INFINITY, mn = INFINITY, d = 0.f;
      bool out = false;
      range32(vec[r], m, 0, mx, mn);  // both 32-channel blocks' loads in flight together
      range32(vec[r], m, 32, mx, mn);
      d = __fsub_rn(mx, mn);
      out = d > ds || (d == ds && j > s);
      if (!out) {
        range32(vec[r], m, 64, mx, mn);
        range32(vec[r], m, 96, mx, mn);
        d = __fsub_rn(mx, mn);
        out = d > ds || (d == ds && j > s);
      }
      if (!out) atomicMin(&best[r], dkey(d, j));
    }
  } else {
    // the bound excluded too little: every pattern for every row, two threads per row
    const int r = tid >> 1, hh = tid & 1;
    if (row_on(r)) {
      const float* M = r < kG ? c.MV : c.MK;
      for (int j = hh; j < Pe; j += 2) {
        float mx = -INFINITY, mn = INFINITY;
        for (int cb = 0; cb < kD; cb += 32) range32(vec[r], M + (size_t)j * kD, cb, mx, mn);
        atomicMin(&best[r], dkey(__fsub_rn(mx, mn), j));
      }
    }
  }
  __syncthreads();

  // ---- residuals in place, R = y - M[k*], one thread per (row, 32-channel group): rows
  // lane and lane + 32 (V slot, K slot) of group `warp`; the V groups' scale / zero on the way,
  // and, on a page the call writes whole, the V codes
  const int maxc = (1 << g.bits) - 1;
  const bool whole = c.fresh && lo == 0 && hi == kG;  // every token of the page is new
  if (tid == 0) ktiny = 0;
  {
    const int q = warp;
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int r = lane + kG * u;
      float s = 0.f, z = 0.f, ri = 0.f;
      if (row_on(r)) {
        // V: the adaptive threshold may drop the pattern (residual = the vector itself)
        const bool keep = u || v_keep_pattern(g.vrho, __uint_as_float((uint32_t)(best[r] >> 32)), rraw[r]);
        if (u == 0 && q == 0) vkeep[r] = keep;
        const float4* m4 = reinterpret_cast<const float4*>((u ? c.MK : c.MV) + (size_t)(best[r] & 0xffffffffu) * kD +
                                                           32 * q);
        float4* y4 = reinterpret_cast<float4*>(&vec[r][32 * q]);
        float4 mv[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) mv[k] = keep ? __ldg(m4 + k) : make_float4(0.f, 0.f, 0.f, 0.f);
        float mx = -INFINITY, mn = INFINITY;
        float x[32];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const float4 a = y4[k];
          float4 o;
          sub2(a.x, a.y, mv[k].x, mv[k].y, o.x, o.y);
          sub2(a.z, a.w, mv[k].z, mv[k].w, o.z, o.w);
          y4[k] = o;
          x[4 * k] = o.x; x[4 * k + 1] = o.y; x[4 * k + 2] = o.z; x[4 * k + 3] = o.w;
          mx = max3(mx, o.x, o.y);
          mn = min3(mn, o.x, o.y);
          mx = max3(mx, o.z, o.w);
          mn = min3(mn, o.z, o.w);
        }
        if (u == 0) {
          group_sz(mn, mx, g.bits, s, z, ri);
          if (whole) {
            uint32_t pc[16];
            const float zz = z, rr = ri;
            const bool clean = codes_fma<32>(x, pc, [&](int, float& z0, float& z1, float& r0, float& r1) {
              z0 = z1 = zz;
              r0 = r1 = rr;
            });
            if (clean && !tiny_scale(s)) {
#pragma unroll
              for (int cc = 0; cc < 4; ++cc)
                *reinterpret_cast<uint4*>(cbV + cb_off(r, 32 * q + 8 * cc)) =
                    make_uint4(pc[4 * cc], pc[4 * cc + 1], pc[4 * cc + 2], pc[4 * cc + 3]);
            } else {
              v_codes_exact(&vec[r][32 * q], z, s, maxc, cbV, r, 32 * q);
            }
          }
        }
      }
      if (u == 0) {  // V: every slot, zeros for tokens not in this call
        vsz[(0 * 4 + q) * kG + lane] = s;
        vsz[(1 * 4 + q) * kG + lane] = z;
        vsz[(2 * 4 + q) * kG + lane] = ri;
      }
    }
  }
  __syncthreads();

  // ---- K scale / zero per channel over the page
  float* ks_g = reinterpret_cast<float*>(c.sub + g.off_ks);
  float* kz_g = reinterpret_cast<float*>(c.sub + g.off_kz);
  if (c.seal) {
    for (int d = tid; d < kD; d += blockDim.x) {
      float mx = -INFINITY, mn = INFINITY;
#pragma unroll
      for (int t = 0; t < kG; t += 2) {
        mx = max3(mx, vec[kG + t][d], vec[kG + t + 1][d]);
        mn = min3(mn, vec[kG + t][d], vec[kG + t + 1][d]);
      }
      float s, z, ri;
      group_sz(mn, mx, g.bits, s, z, ri);
      if (tiny_scale(s)) ktiny = 1;
      ksz[0 * kD + d] = s;
      ksz[1 * kD + d] = z;
      ksz[2 * kD + d] = ri;
      ks_g[ksc_pos(d)] = s;
      kz_g[ksc_pos(d)] = z;
    }
  }
  __syncthreads();

  // ---- K codes of a sealed page (a unit: row and 16 channels, 4 x 4 channels 32 apart)
  if (c.seal) {
    for (int u = tid; u < kG * 8; u += blockDim.x) {
      const int r = u >> 3, cbk = u & 7;
      float x[16], zs[16], rs[16];
#pragma unroll
      for (int k4 = 0; k4 < 4; ++k4) {
        const int ch = 4 * cbk + 32 * k4;
        const float4 a = *reinterpret_cast<const float4*>(&vec[kG + r][ch]);
        const float4 z4 = *reinterpret_cast<const float4*>(ksz + kD + ch);
        const float4 r4 = *reinterpret_cast<const float4*>(ksz + 2 * kD + ch);
        x[4 * k4] = a.x; x[4 * k4 + 1] = a.y; x[4 * k4 + 2] = a.z; x[4 * k4 + 3] = a.w;
        zs[4 * k4] = z4.x; zs[4 * k4 + 1] = z4.y; zs[4 * k4 + 2] = z4.z; zs[4 * k4 + 3] = z4.w;
        rs[4 * k4] = r4.x; rs[4 * k4 + 1] = r4.y; rs[4 * k4 + 2] = r4.z; rs[4 * k4 + 3] = r4.w;
      }
      uint32_t pc[8];
      const bool clean = codes_fma<16>(x, pc, [&](int i2, float& z0, float& z1, float& r0, float& r1) {
        z0 = zs[2 * i2]; z1 = zs[2 * i2 + 1];
        r0 = rs[2 * i2]; r1 = rs[2 * i2 + 1];
      });
      if (clean && ktiny == 0) {
#pragma unroll
        for (int k4 = 0; k4 < 4; ++k4)
          *reinterpret_cast<uint2*>(cbK + cb_off(r, 4 * cbk + 32 * k4)) = make_uint2(pc[2 * k4], pc[2 * k4 + 1]);
      } else {
        k_codes_exact(vec[kG + r], ksz + kD, ksz, cbk, maxc, cbK, r);
      }
    }
  }
  __syncthreads();

  // ---- code words: the whole-page V block and a sealed K block from the 16-bit codes (16-byte
  // chunks of four words per lane, spread over the warps); a partly written V block one word per
  // thread, keeping the codes of the tokens already in the page; then scales, zeros, indices
  {
    uint32_t* vdst = reinterpret_cast<uint32_t*>(c.sub + g.off_vc);
    const int nc = g.bits == 2 ? 2 : 4;  // chunks per block
    const int nch = (whole ? nc : 0) + (c.seal ? nc : 0);
    for (int ch = warp; ch < nch; ch += nwarps) {
      const bool isV = whole && ch < nc;
      const int wq = isV ? ch : ch - (whole ? nc : 0);
      uint32_t* blk = isV ? vdst : reinterpret_cast<uint32_t*>(c.sub);
      *reinterpret_cast<uint4*>(blk + wq * 128 + lane * 4) = pack_chunk(isV ? cbV : cbK, isV, g.bits, wq, lane);
    }
    if (!whole) {
      const int nwords = kG * kD * g.bits / 32;
      const int keep_lo = c.fresh ? 0 : lo;
      const float(*Rv)[kLd] = vec;
      for (int wd = tid; wd < nwords; wd += blockDim.x) {
        const uint32_t old = keep_lo > 0 ? vdst[wd] : 0u;  // tokens already in the page keep their codes
        vdst[wd] = g.bits == 2 ? v_word<2, true>(wd, Rv, vsz, vsz + 4 * kG, vsz + 8 * kG, keep_lo, hi, old)
                               : v_word<4, true>(wd, Rv, vsz, vsz + 4 * kG, vsz + 8 * kG, keep_lo, hi, old);
      }
    }
  }
  float* vs_g = reinterpret_cast<float*>(c.sub + g.off_vs);
  float* vz_g = reinterpret_cast<float*>(c.sub + g.off_vz);
  uint8_t* vidx_g = c.sub + g.off_vidx;
  float* vrow_g = reinterpret_cast<float*>(c.sub + g.off_vrow);
  {
    const int slot = tid >> 2, q = tid & 3;
    if (c.fresh || (slot >= lo && slot < hi)) {
      vs_g[vsc_pos(slot, q)] = vsz[(0 * 4 + q) * kG + slot];
      vz_g[vzc_pos(slot, q)] = vsz[(1 * 4 + q) * kG + slot];
    }
  }
  if (tid < kG) {
    const int slot = tid;
    const bool present = slot >= lo && slot < hi;
    if (c.fresh || present) {
      vidx_g[tok_pos(slot)] = !present ? (uint8_t)0 : vkeep[slot] ? (uint8_t)(best[slot] & 0xff) : (uint8_t)kRawIndex;
      if (g.tx) vrow_g[tok_pos(slot)] = present ? vrow_s[slot] : 0.f;
    }
  }
  if (c.seal && tid < kG) {
    uint8_t* kidx_g = c.sub + g.off_kidx;
    float* krow_g = reinterpret_cast<float*>(c.sub + g.off_krow);
    kidx_g[tok_pos(tid)] = (uint8_t)(best[kG + tid] & 0xff);
    if (g.tx) krow_g[tok_pos(tid)] = krow_s[tid];
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
  return al256((size_t)g.S * g.H * 2 * kProbe * 4) + al256((size_t)g.S * g.H * 2 * g.P * kProbe * 4) + 256;
}

cudaError_t launch_append(const Geom& g, const void* k_new, const void* v_new, int n_new, void* ws, cudaStream_t st) {
  if (n_new <= 0 || g.B == 0) return cudaSuccess;
  AppendWs w = carve_append(ws, g.S, g.H, g.P);
  append_prep_kernel<<<dim3(g.S * g.H, 2), kD, 0, st>>>(g, w);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  // fp16 lower bounds [P][64 rows], probe tables and channels (later the work queue); later the
  // s / z tables (12 kG + 3 kD floats) from the start
  const int nprk = g.tx ? kProbeKtx : kProbeK;
  const size_t tabs = std::max<size_t>((size_t)(kProbeV + nprk) * g.P + kProbeV + nprk, kQueueCap);
  // (after the assignment: the s / z tables, then two 8 KB code buffers from float 1024 on)
  const size_t dyn = std::max<size_t>((size_t)32 * lb_ld(g.P) + tabs, 1024 + 4096) * sizeof(float);
  if ((e = cudaFuncSetAttribute(append_pages_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)dyn)) !=
      cudaSuccess)
    return e;
  // one CTA per (page the call touches, KV head, sequence)
  dim3 grid(n_new / kG + 2, g.H, g.B);
  append_pages_kernel<<<grid, kAppendThreads, dyn, st>>>(g, w, (const uint16_t*)k_new, (const uint16_t*)v_new,
                                                         n_new);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  append_tail_kernel<<<g.B, 256, 0, st>>>(g, (const uint16_t*)k_new, n_new);
  return cudaGetLastError();
}

}  // namespace kvq
