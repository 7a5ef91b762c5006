// Shared device-side definitions of libkvq: cache geometry, the page layout,
// exact fp32 building blocks and warp utilities.
//
// Every bit-exact step (pre-transform, residual, min-max distance, group
// quantization) is written with explicit round-to-nearest intrinsics so the
// compiler cannot fuse a multiply into an add.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/kvq.h"

namespace kvq {

constexpr int kD = 128;       // head_dim
constexpr int kG = 32;        // tokens per page / K group; channels per V group
constexpr unsigned kFull = 0xffffffffu;

// ---------------------------------------------------------------------------
// Geometry of one cache, copied by value into every kernel.
// ---------------------------------------------------------------------------
struct Geom {
  int32_t B, H, bits, P, S, maxp, npages, dtype, tx;
  int64_t sub_bytes, page_bytes;
  int32_t cb;          // code bytes per K or V block
  int32_t off_ks, off_kz, off_vc, off_vs, off_vz, off_kidx, off_vidx, off_krow, off_vrow;
  uint8_t* pool;
  const int32_t* page_table;
  int32_t* seq_len;
  uint16_t* k_tail;
  const float* kpat;
  const float* vpat;
  const int32_t* seq_to_set;
  const float* kcol;
  const float* vcol;
  int32_t* status;
  uint32_t wait_limit;  // iterations of a bounded page-copy wait (decode)
  float vrho;           // V adaptive threshold rho* (0 = off)
  int32_t* counts;      // [S][H] patterns in use, or null (all P)
  float* window;        // [B][H][4][128] running min / max of the insertion window, or null
  int32_t gwin;         // insertion window length (0 = off)
};

// Patterns in use by (set, KV head): the set's count (clamped to 1..P) or P.
__device__ __forceinline__ int p_eff(const Geom& g, int sh) {
  return g.counts ? min(max(g.counts[sh], 1), g.P) : g.P;
}

__host__ __device__ inline int64_t subblock_bytes_of(int bits, int tx) {
  return 2 * (kG * kD * bits / 8) + 2112 + (tx ? 256 : 0);
}

inline Geom make_geom(const kvq_cache& c) {
  Geom g;
  g.B = c.num_seqs; g.H = c.num_kv_heads; g.bits = c.bits; g.P = c.num_patterns; g.S = c.num_sets;
  g.maxp = c.max_pages_per_seq; g.npages = c.num_pages; g.dtype = c.dtype; g.tx = c.transform;
  g.cb = kG * kD * c.bits / 8;
  g.sub_bytes = subblock_bytes_of(c.bits, c.transform);
  g.page_bytes = g.sub_bytes * c.num_kv_heads;
  g.off_ks = g.cb;
  g.off_kz = g.cb + 512;
  g.off_vc = g.cb + 1024;
  g.off_vs = 2 * g.cb + 1024;
  g.off_vz = 2 * g.cb + 1536;
  g.off_kidx = 2 * g.cb + 2048;
  g.off_vidx = 2 * g.cb + 2080;
  g.off_krow = 2 * g.cb + 2112;
  g.off_vrow = 2 * g.cb + 2240;
  g.pool = (uint8_t*)c.page_pool;
  g.page_table = c.page_table;
  g.seq_len = c.seq_len;
  g.k_tail = (uint16_t*)c.k_tail;
  g.kpat = c.k_patterns;
  g.vpat = c.v_patterns;
  g.seq_to_set = c.seq_to_set;
  g.kcol = c.k_colscale;
  g.vcol = c.v_colscale;
  g.status = c.status;
  g.wait_limit = 1u << 22;
  g.vrho = c.v_rho;
  g.counts = c.pattern_counts;
  g.window = c.pattern_window;
  g.gwin = c.pattern_window_len;
  return g;
}

// ---------------------------------------------------------------------------
// Page layout (see include/kvq.h): fragment order of the code matrices and the
// orders of the per-channel / per-token fields.
// ---------------------------------------------------------------------------

// Position of element (row, col) of a (16*MT)x(16*KS) code matrix: 32-bit word of the block and bit.
// The lane's word w sits at block word (w/4)*128 + lane*4 + w%4 (lane-interleaved 16-byte chunks).
__host__ __device__ __forceinline__ void frag_pos(int bits, int KS, int row, int col, int& word, int& bit) {
  const int rr = row & 15, cc = col & 15;
  const int lane = (rr & 7) * 4 + ((cc & 7) >> 1);
  const int reg = ((row >> 4) * KS + (col >> 4)) * 4 + (rr >> 3) + 2 * (cc >> 3);
  const int odd = col & 1;
  int w;
  if (bits == 2) { w = reg >> 3; bit = 2 * (reg & 7) + 16 * odd; }
  else           { w = reg >> 2; bit = 4 * (reg & 3) + 16 * odd; }
  word = (w >> 2) * 128 + lane * 4 + (w & 3);
}

// Inverse: the element held by block word `word` at slot `slot` of half `odd`.
__host__ __device__ __forceinline__ void frag_elem(int bits, int KS, int word, int slot, int odd, int& row, int& col) {
  const int lane = (word & 127) >> 2;
  const int w = (word >> 7) * 4 + (word & 3);
  const int reg = bits == 2 ? w * 8 + slot : w * 4 + slot;
  const int g = lane >> 2, tig = lane & 3;
  const int r = reg & 3, tile = reg >> 2;
  row = 16 * (tile / KS) + 8 * (r & 1) + g;
  col = 16 * (tile % KS) + 8 * (r >> 1) + 2 * tig + odd;
}

// Field orders (include/kvq.h): position of a channel (KSC), of (token, group) (VSC, VZC),
// of a token (TOK).  A channel / token inside its 16-block is 2*tig + (e&1) + 8*(e>>1).
__host__ __device__ __forceinline__ int ksc_pos(int ch) {
  const int ks = ch >> 4, c = ch & 15;
  const int tig = (c & 7) >> 1, e = (c & 1) + 2 * (c >> 3);
  return ks * 16 + tig * 4 + e;
}
__host__ __device__ __forceinline__ int vsc_pos(int tok, int grp) {
  const int ks = tok >> 4, c = tok & 15;
  const int tig = (c & 7) >> 1, e = (c & 1) + 2 * (c >> 3);
  return ((ks * 4 + e) * 4 + tig) * 4 + grp;
}
__host__ __device__ __forceinline__ int vzc_pos(int tok, int grp) { return ((tok >> 3) * 8 + (tok & 7)) * 4 + grp; }
__host__ __device__ __forceinline__ int tok_pos(int tok) { return (tok & 7) * 4 + (tok >> 3); }

// ---------------------------------------------------------------------------
// Element access
// ---------------------------------------------------------------------------
__device__ __forceinline__ float load_elem(const uint16_t* p, int dtype) {
  uint16_t u = __ldg(p);
  if (dtype == KVQ_BF16) return __uint_as_float(((uint32_t)u) << 16);
  return __half2float(__ushort_as_half(u));
}

__device__ __forceinline__ float bits_to_float(uint16_t u, int dtype) {
  if (dtype == KVQ_BF16) return __uint_as_float(((uint32_t)u) << 16);
  return __half2float(__ushort_as_half(u));
}

__device__ __forceinline__ void set_status(int32_t* st, int bit) {
  if (st) atomicOr(st, bit);
}

// ---------------------------------------------------------------------------
// Warp helpers.  A 128-vector is held by a warp as v[k] = element lane + 32*k.
// ---------------------------------------------------------------------------
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v = fmaxf(v, __shfl_xor_sync(kFull, v, o));
  return v;
}
__device__ __forceinline__ float warp_min(float v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v = fminf(v, __shfl_xor_sync(kFull, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(kFull, v, o);
  return v;
}
__device__ __forceinline__ double warp_sum_d(double v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(kFull, v, o);
  return v;
}

// Walsh-Hadamard butterfly, strides 1, 2, ..., 64 in that order, (a+b, a-b) with a the lower
// index; unnormalised.  Matches the reference definition operation for operation.
__device__ __forceinline__ void fwht_warp(float v[4], int lane) {
#pragma unroll
  for (int h = 1; h < 32; h <<= 1) {
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      float p = __shfl_xor_sync(kFull, v[k], h);
      v[k] = (lane & h) ? __fsub_rn(p, v[k]) : __fadd_rn(v[k], p);
    }
  }
  // stride 32: pairs (k=0,k=1), (k=2,k=3)
  float a0 = v[0], b0 = v[1], a1 = v[2], b1 = v[3];
  v[0] = __fadd_rn(a0, b0); v[1] = __fsub_rn(a0, b0);
  v[2] = __fadd_rn(a1, b1); v[3] = __fsub_rn(a1, b1);
  // stride 64: pairs (k=0,k=2), (k=1,k=3)
  a0 = v[0]; b0 = v[2]; a1 = v[1]; b1 = v[3];
  v[0] = __fadd_rn(a0, b0); v[2] = __fsub_rn(a0, b0);
  v[1] = __fadd_rn(a1, b1); v[3] = __fsub_rn(a1, b1);
}

// fp32 sum of 128 values by halving (upper half added onto the lower half, stride 64 first).
// Every lane returns the total.
__device__ __forceinline__ float halving_sum_warp(const float v[4]) {
  float s0 = __fadd_rn(v[0], v[2]);  // i and i+64 for i = lane
  float s1 = __fadd_rn(v[1], v[3]);  // i = lane + 32
  float s = __fadd_rn(s0, s1);       // stride 32
#pragma unroll
  for (int o = 16; o; o >>= 1) s = __fadd_rn(s, __shfl_xor_sync(kFull, s, o));
  return s;
}

// Pre-transform of one token held by a warp: x -> y = fl32(fl32(x'/c) / r), r = population std.
__device__ __forceinline__ void transform_row_warp(float v[4], const float* c, float& r_out, int lane) {
  fwht_warp(v, lane);
#pragma unroll
  for (int k = 0; k < 4; ++k) v[k] = __fdiv_rn(v[k], __ldg(c + lane + 32 * k));
  float mean = __fmul_rn(halving_sum_warp(v), 0.0078125f);  // exact: divide by 128
  float dev[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    float t = __fsub_rn(v[k], mean);
    dev[k] = __fmul_rn(t, t);
  }
  float var = __fmul_rn(halving_sum_warp(dev), 0.0078125f);
  float r = __fsqrt_rn(var);
  if (r == 0.0f) r = 1.0f;
#pragma unroll
  for (int k = 0; k < 4; ++k) v[k] = __fdiv_rn(v[k], r);
  r_out = r;
}

// transform_row_warp for R tokens held by a warp at once, their steps interleaved (each token's
// operations exactly those of transform_row_warp).  c[q]: token q's column factors.
template <int R>
__device__ __forceinline__ void transform_rows_warp(float (&v)[R][4], const float* const (&c)[R], float (&r_out)[R],
                                                    int lane) {
#pragma unroll
  for (int h = 1; h < 32; h <<= 1)
#pragma unroll
    for (int q = 0; q < R; ++q)
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float p = __shfl_xor_sync(kFull, v[q][k], h);
        v[q][k] = (lane & h) ? __fsub_rn(p, v[q][k]) : __fadd_rn(v[q][k], p);
      }
  float sm[R];
#pragma unroll
  for (int q = 0; q < R; ++q) {
    const float a0 = v[q][0], b0 = v[q][1], a1 = v[q][2], b1 = v[q][3];
    const float t0 = __fadd_rn(a0, b0), t1 = __fsub_rn(a0, b0), t2 = __fadd_rn(a1, b1), t3 = __fsub_rn(a1, b1);
    v[q][0] = __fadd_rn(t0, t2);
    v[q][1] = __fadd_rn(t1, t3);
    v[q][2] = __fsub_rn(t0, t2);
    v[q][3] = __fsub_rn(t1, t3);
#pragma unroll
    for (int k = 0; k < 4; ++k) v[q][k] = __fdiv_rn(v[q][k], __ldg(c[q] + lane + 32 * k));
    sm[q] = __fadd_rn(__fadd_rn(v[q][0], v[q][2]), __fadd_rn(v[q][1], v[q][3]));
  }
#pragma unroll
  for (int o = 16; o; o >>= 1)
#pragma unroll
    for (int q = 0; q < R; ++q) sm[q] = __fadd_rn(sm[q], __shfl_xor_sync(kFull, sm[q], o));
  float sv[R];
#pragma unroll
  for (int q = 0; q < R; ++q) {
    const float mean = __fmul_rn(sm[q], 0.0078125f);
    float dev[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float t = __fsub_rn(v[q][k], mean);
      dev[k] = __fmul_rn(t, t);
    }
    sv[q] = __fadd_rn(__fadd_rn(dev[0], dev[2]), __fadd_rn(dev[1], dev[3]));
  }
#pragma unroll
  for (int o = 16; o; o >>= 1)
#pragma unroll
    for (int q = 0; q < R; ++q) sv[q] = __fadd_rn(sv[q], __shfl_xor_sync(kFull, sv[q], o));
#pragma unroll
  for (int q = 0; q < R; ++q) {
    float r = __fsqrt_rn(__fmul_rn(sv[q], 0.0078125f));
    if (r == 0.0f) r = 1.0f;
#pragma unroll
    for (int k = 0; k < 4; ++k) v[q][k] = __fdiv_rn(v[q][k], r);
    r_out[q] = r;
  }
}

// Nearest pattern under the min-max distance, warp-cooperative, lowest index on ties.
// y: this lane's 4 channels (lane + 32k).  M: P x 128 fp32 patterns (global or shared).
__device__ __forceinline__ int assign_warp(const float y[4], const float* M, int P, int lane) {
  float best = 0.0f;
  int bj = 0;
  for (int j = 0; j < P; ++j) {
    const float* m = M + (size_t)j * kD;
    float mx = -INFINITY, mn = INFINITY;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      float r = __fsub_rn(y[k], m[lane + 32 * k]);
      mx = fmaxf(mx, r);
      mn = fminf(mn, r);
    }
    mx = warp_max(mx);
    mn = warp_min(mn);
    float d = __fsub_rn(mx, mn);
    if (j == 0 || d < best) { best = d; bj = j; }
  }
  return bj;
}

// fp32 range of x - m over 128 channels, exact (no rounding beyond the per-element
// subtraction): packed f32x2 subtractions and three-input max / min.
__device__ __forceinline__ void sub2(float a0, float a1, float b0, float b1, float& r0, float& r1) {
  unsigned long long a, b, r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(a) : "f"(a0), "f"(a1));
  asm("mov.b64 %0, {%1, %2};" : "=l"(b) : "f"(b0), "f"(b1));
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  asm("mov.b64 {%0, %1}, %2;" : "=f"(r0), "=f"(r1) : "l"(r));
}
__device__ __forceinline__ void mul2f(float a0, float a1, float b0, float b1, float& r0, float& r1) {
  unsigned long long a, b, r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(a) : "f"(a0), "f"(a1));
  asm("mov.b64 %0, {%1, %2};" : "=l"(b) : "f"(b0), "f"(b1));
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  asm("mov.b64 {%0, %1}, %2;" : "=f"(r0), "=f"(r1) : "l"(r));
}
__device__ __forceinline__ void add2f(float a0, float a1, float b0, float b1, float& r0, float& r1) {
  unsigned long long a, b, r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(a) : "f"(a0), "f"(a1));
  asm("mov.b64 %0, {%1, %2};" : "=l"(b) : "f"(b0), "f"(b1));
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  asm("mov.b64 {%0, %1}, %2;" : "=f"(r0), "=f"(r1) : "l"(r));
}
__device__ __forceinline__ void fma2f(float a0, float a1, float b0, float b1, float c0, float c1, float& r0,
                                      float& r1) {
  unsigned long long a, b, c, r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(a) : "f"(a0), "f"(a1));
  asm("mov.b64 %0, {%1, %2};" : "=l"(b) : "f"(b0), "f"(b1));
  asm("mov.b64 %0, {%1, %2};" : "=l"(c) : "f"(c0), "f"(c1));
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  asm("mov.b64 {%0, %1}, %2;" : "=f"(r0), "=f"(r1) : "l"(r));
}
__device__ __forceinline__ float max3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}
__device__ __forceinline__ float min3(float a, float b, float c) {
  float d;
  asm("min.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}
// d_mm(y, m) for a vector held in registers (natural channel order) and a pattern in memory.
__device__ __forceinline__ float dmm_reg(const float (&y)[kD], const float* __restrict__ m) {
  const float4* m4 = reinterpret_cast<const float4*>(m);
  float mx = -INFINITY, mn = INFINITY;
#pragma unroll
  for (int c = 0; c < kD / 4; ++c) {
    const float4 v = __ldg(m4 + c);
    float r0, r1, r2, r3;
    sub2(y[4 * c], y[4 * c + 1], v.x, v.y, r0, r1);
    sub2(y[4 * c + 2], y[4 * c + 3], v.z, v.w, r2, r3);
    mx = max3(mx, r0, r1);
    mn = min3(mn, r0, r1);
    mx = max3(mx, r2, r3);
    mn = min3(mn, r2, r3);
  }
  return __fsub_rn(mx, mn);
}

// V adaptive threshold: keep the pattern iff R_flat <= fl32(rho* x R_raw) (rho* > 0), else quantize raw.
__device__ __forceinline__ bool v_keep_pattern(float vrho, float r_flat, float r_raw) {
  return !(vrho > 0.0f) || r_flat <= __fmul_rn(vrho, r_raw);
}
constexpr int kRawIndex = 255;  // stored V index of a vector quantized without its pattern

// Group quantizer on the 32 lanes of a warp (one value per lane): s, z and this lane's code.
__device__ __forceinline__ int quant_warp(float R, int bits, float& s_out, float& z_out) {
  float mn = warp_min(R), mx = warp_max(R);
  float levels = (float)((1 << bits) - 1);
  float s = __fdiv_rn(__fsub_rn(mx, mn), levels);
  int code = 0;
  if (s != 0.0f) {
    float u = __fdiv_rn(__fsub_rn(R, mn), s);
    code = __float2int_rn(u);
    code = min(max(code, 0), (1 << bits) - 1);
  }
  s_out = s;
  z_out = mn;
  return code;
}

}  // namespace kvq
