// Quantize-append of full pages ("PatternKV", Section 3.2: nearest pattern under the min-max
// distance, Eq. 6, residual quantized with Eq. 1; Section 3.3: V adaptive threshold; Section
// 4.1 granularity): every page whose 32 tokens all arrive in this call, which is nearly all of
// them in a prefill.  Pages only partly written by the call go through append_pages_kernel.
//
// Persistent CTAs of 8 warps, each walking a contiguous run of (KV head, sequence, page) tasks.
// A task's 32 V rows and 32 K rows arrive by TMA (two 64-channel boxes each, 128-byte swizzle)
// into one of two stage buffers; the copy of the task after next is issued as soon as a stage is
// free.  Every phase of a task spreads its work evenly over the 256 threads, with a block barrier
// between phases:
//   A  V seeds: the Euclidean nearest pattern on the tensor cores (m16n8k16 scores |m|^2/2 - x.m
//      against the patterns' 16-bit parts; only a guess), warps 0-1; the other warps gather each
//      row's values at the probe channels (the channels where the patterns differ most).
//   B  U = exact min-max distance of each V row to its seed, and the row's own range (adaptive
//      threshold), 4 threads a row; K lower bounds over 16 probe channels for every pattern
//      (lane = K row, warp w takes the w-th eighth of the patterns), kept in registers; the
//      smallest bound names the K seed.
//   C  U of each K row (4 threads a row); V lower bounds over 8 probe channels for every pattern
//      (lane = V row, the same split): a pattern whose bound could still beat the seed, or tie
//      it with a lower index, goes on the warp's own refinement list (a warp prefix sum of the
//      lanes' candidate counts places them), whose bounds over 32 probe channels the warp then
//      computes a lane an entry; the survivors go on the warp's exact list.
//   D  the K patterns of the warp's eighth whose bound does not exceed U join the exact list;
//      the warp computes the min-max distance of every entry over all 128 channels (4 lanes an
//      entry) and keeps the minimum (distance, index) per row.  A row whose candidates did not
//      fit a list is compared with every pattern instead.
//   F  V rows: residual, scale and zero per 32-channel group, codes (a thread a row and group);
//      K rows: residuals staged as fp32.
//   G  K scale and zero per channel over the page's 32 tokens (a thread a channel).
//   H  K codes (a thread a row and 16 channels).
//   I  the 16-bit codes, written over the consumed input rows, come back in the page's fragment
//      order through ldmatrix(.trans); a few shifts pack them into words.
// The bounds are exact lower bounds: the residual range over a channel subset never exceeds the
// range over all channels, and a subset's residuals are the same fp32 subtractions.  Ties keep
// the lowest pattern index (the minimum of (distance bits, index) keys).
//
// A code is rne(fl32(fl32(R - z) / s)), produced by one FMA, v = t (1/s) + (1.5 * 2^7 + 1/2)
// with t = R - z in [0, maxc s]: v stays in [128, 256), so the integer part of (t / s + 1/2) is
// 192 + code (bits 16-22) and its fraction fills bits 0-15.  v differs from the exact
// t / s + 1/2 by less than 2^-17 (its own rounding) + 15 * 2^-24 (the reciprocal's), under one
// fraction step (2^-16); so the integer part can be wrong, or the quotient a tie that rounds to
// even, only when the fraction is 0x0000 or 0xFFFF.  Those codes (about 2 in 65536), and every
// code of a scale below 2^-125 whose reciprocal is inexact, are recomputed with the correctly
// rounded division.
#include <algorithm>
#include <cstdint>

#include "kvq_common.cuh"
#include "kvq_internal.h"

namespace kvq {

namespace {

constexpr int kProbeAll = 32;  // probe channels per pattern set in the prep tables
constexpr int kV1 = 8;         // V: first-level bound channels
constexpr int kV2 = 32;        // V: refined bound channels
constexpr int kK1 = 16;        // K: bound channels
constexpr int kTabLd = 36;     // fp32 row stride of the V probe table and of the rows' probe values
constexpr int kPhiLd = 136;    // 16-bit row stride of the pattern table for ldmatrix (272 B: conflict-free)
constexpr int kRkLd = 144;     // fp32 row stride of the staged K residuals (16 mod 32 words)
constexpr int kStageBytes = 16384;  // V rows (2 x 4 KB halves) then K rows (2 x 4 KB halves)
constexpr int kMaxSlice = 16;       // patterns per warp in the bound passes (up to 128 patterns)
constexpr int kFullGroups = 2;      // 4-warp task groups per CTA (two CTAs per SM) for up to 64 patterns
constexpr int kW2Cap = 256;         // entries of a warp's refinement list
constexpr int kWECap = 128;         // entries of a warp's exact list
constexpr uint32_t kFSpin = 1u << 22;
constexpr float kCodeMagic = 192.5f;  // 1.5 * 2^7 + 1/2: 16 fractional bits, +1/2 folded in
constexpr float kMinScale = 0x1p-125f;  // below this (and nonzero) 1 / s is not within 2^-24 of exact

__device__ __forceinline__ uint32_t s32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ void fb_init(uint64_t* bar, uint32_t n) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(s32(bar)), "r"(n) : "memory");
}
__device__ __forceinline__ void fb_expect(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(s32(bar)), "r"(bytes) : "memory");
}
__device__ __forceinline__ bool fb_wait(uint64_t* bar, uint32_t parity) {
  for (uint32_t it = 0; it < kFSpin; ++it) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(s32(bar)), "r"(parity)
        : "memory");
    if (ok) return true;
  }
  return false;
}
__device__ __forceinline__ void tma3(void* dst, const CUtensorMap* map, int c0, int c1, int c2, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], "
      "[%5];" ::"r"(s32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(s32(bar))
      : "memory");
}
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
template <int DT>
__device__ __forceinline__ void mma_seed(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  if constexpr (DT == KVQ_BF16)
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
  else
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}


template <int DT>
__device__ __forceinline__ float cvt_lo(uint32_t w) {
  if constexpr (DT == KVQ_BF16) return __uint_as_float(w << 16);
  else return __half2float(__ushort_as_half((uint16_t)(w & 0xffffu)));
}
template <int DT>
__device__ __forceinline__ float cvt_hi(uint32_t w) {
  if constexpr (DT == KVQ_BF16) return __uint_as_float(w & 0xffff0000u);
  else return __half2float(__ushort_as_half((uint16_t)(w >> 16)));
}

// Byte offset of 16-byte chunk c (0..7) of row `row` in a 128-byte-swizzled 32 x 128 B half-box.
__device__ __forceinline__ uint32_t swz(int row, int c) { return (uint32_t)(row * 128 + ((c ^ (row & 7)) << 4)); }
// Byte offset of channel ch (0..127) of row `row` in a stage region of two swizzled half-boxes.
__device__ __forceinline__ uint32_t elem_off(int row, int ch) {
  return (uint32_t)((ch >> 6) * 4096) + swz(row, (ch & 63) >> 3) + (uint32_t)((ch & 7) * 2);
}

// Channels 32 q .. 32 q + 31 of staged row `row` (16-bit, swizzled) as fp32.
template <int DT>
__device__ __forceinline__ void load_x32(const uint8_t* rows, int row, int q, float (&x)[32]) {
  const uint8_t* hb = rows + (q >> 1) * 4096;
#pragma unroll
  for (int cc = 0; cc < 4; ++cc) {
    const uint4 u = *reinterpret_cast<const uint4*>(hb + swz(row, 4 * (q & 1) + cc));
    const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      x[8 * cc + 2 * e] = cvt_lo<DT>(w4[e]);
      x[8 * cc + 2 * e + 1] = cvt_hi<DT>(w4[e]);
    }
  }
}

// Range of x - m over 32 channels (m: 32 fp32 pattern values in global memory).
__device__ __forceinline__ void range32(const float (&x)[32], const float* __restrict__ m, float& mx, float& mn) {
  const float4* m4 = reinterpret_cast<const float4*>(m);
  float4 mv[8];
#pragma unroll
  for (int c = 0; c < 8; ++c) mv[c] = __ldg(m4 + c);
  mx = -INFINITY;
  mn = INFINITY;
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    float r0, r1, r2, r3;
    sub2(x[4 * c], x[4 * c + 1], mv[c].x, mv[c].y, r0, r1);
    sub2(x[4 * c + 2], x[4 * c + 3], mv[c].z, mv[c].w, r2, r3);
    mx = max3(mx, r0, r1);
    mn = min3(mn, r0, r1);
    mx = max3(mx, r2, r3);
    mn = min3(mn, r2, r3);
  }
}

// Range of y - t over N probe channels (both in shared memory, 16-byte aligned).
template <int N>
__device__ __forceinline__ float probe_range(const float* y, const float* t) {
  float mx = -INFINITY, mn = INFINITY;
#pragma unroll
  for (int q = 0; q < N / 4; ++q) {
    const float4 a = reinterpret_cast<const float4*>(y)[q];
    const float4 m = reinterpret_cast<const float4*>(t)[q];
    float r0, r1, r2, r3;
    sub2(a.x, a.y, m.x, m.y, r0, r1);
    sub2(a.z, a.w, m.z, m.w, r2, r3);
    mx = max3(mx, r0, r1);
    mn = min3(mn, r0, r1);
    mx = max3(mx, r2, r3);
    mn = min3(mn, r2, r3);
  }
  return __fsub_rn(mx, mn);
}

__device__ __forceinline__ unsigned long long dkey(float d, int j) {
  return ((unsigned long long)__float_as_uint(d) << 32) | (uint32_t)j;
}

// Range of y - t over N probe channels (y in registers, t in shared memory, 16-byte aligned).
template <int N>
__device__ __forceinline__ float probe_range_reg(const float (&y)[N], const float* t) {
  float mx = -INFINITY, mn = INFINITY;
#pragma unroll
  for (int q = 0; q < N / 4; ++q) {
    const float4 m = reinterpret_cast<const float4*>(t)[q];
    float r0, r1, r2, r3;
    sub2(y[4 * q], y[4 * q + 1], m.x, m.y, r0, r1);
    sub2(y[4 * q + 2], y[4 * q + 3], m.z, m.w, r2, r3);
    mx = max3(mx, r0, r1);
    mn = min3(mn, r0, r1);
    mx = max3(mx, r2, r3);
    mn = min3(mn, r2, r3);
  }
  return __fsub_rn(mx, mn);
}

// A warp's lanes each list the patterns j0 + i (bit i of `mask`) of their row `row`: the
// entries (row << 8 | pattern) go to list[base ..], placed by a warp prefix sum of the counts.
// Returns the new (uniform) size, at most cap; an entry past cap flags its row instead.
__device__ __forceinline__ int warp_compact(uint32_t mask, int lane, int row, int j0, uint16_t* list, int base,
                                            int cap, int* ovf_row, int* any_ovf) {
  const int n = __popc(mask);
  int incl = n;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(kFull, incl, o);
    if (lane >= o) incl += v;
  }
  const int total = __shfl_sync(kFull, incl, 31);
  int pos = base + incl - n;
  while (mask) {
    const int i = __ffs(mask) - 1;
    mask &= mask - 1u;
    if (pos < cap) list[pos] = (uint16_t)((row << 8) | (j0 + i));
    else { *ovf_row = 1; *any_ovf = 1; }
    ++pos;
  }
  return min(base + total, cap);
}
// Append of one entry per live lane (every lane of the warp calls it); returns the new size.
__device__ __forceinline__ int warp_append(bool live, uint32_t entry, uint16_t* list, int n, int cap, int* ovf_row,
                                           int* any_ovf, int lane) {
  const unsigned m = __ballot_sync(kFull, live);
  if (live) {
    const int pos = n + __popc(m & ((1u << lane) - 1u));
    if (pos < cap) list[pos] = (uint16_t)entry;
    else { *ovf_row = 1; *any_ovf = 1; }
  }
  return min(n + __popc(m), cap);
}

__device__ __forceinline__ uint32_t vmin_u16x2(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("min.u16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

// Codes of N residuals as N / 2 words of two 16-bit halves (the code in bits 8-11 of each
// half: byte 2 of the FMA result, 0x40 | code); zr(i, z0, z1, r0, r1) gives the zeros and
// reciprocal scales of values 2i, 2i + 1.  Returns true if no fraction is 0x0000 or 0xFFFF.
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

// 1 / s for the FMA codes: 0 for s == 0 (every code 0, as the definition gives)
__device__ __forceinline__ float code_rcp(float s) { return s != 0.0f ? __frcp_rn(s) : 0.0f; }
__device__ __forceinline__ bool tiny_scale(float s) { return s != 0.0f && s < kMinScale; }
// The definition's code: the correctly rounded quotient, rounded half to even, clamped.
__device__ __forceinline__ uint32_t exact_code(float t, float s, int maxc) {
  return s != 0.0f ? (uint32_t)min(max(__float2int_rn(__fdiv_rn(t, s)), 0), maxc) : 0u;
}
// fp32 index of (row, channel) in the staged K residuals: 4 floats between the 32-channel
// quarters and 144 floats between rows, so that the quarters and neighbouring rows fall in
// different banks
__device__ __forceinline__ int rk_at(int row, int ch) { return row * kRkLd + ch + 4 * (ch >> 5); }

// The rare paths of codes_fma (a fraction of 0x0000 / 0xFFFF somewhere, or a scale below
// 2^-125), out of line and reading their inputs from memory, so that no register array of the
// caller needs an address: every code of the unit recomputed with exact_code.
// V: channels 32 q .. 32 q + 31 of staged row r (16-bit input, minus the pattern's values m
// unless null), zero z, scale s; the 16-bit code words replace the input there.
template <int DT>
__device__ __noinline__ void v_codes_exact(uint8_t* rows, int r, int q, const float* m, float z, float s, int maxc) {
  uint8_t* hb = rows + (q >> 1) * 4096;
  for (int cc = 0; cc < 4; ++cc) {
    uint4* p = reinterpret_cast<uint4*>(hb + swz(r, 4 * (q & 1) + cc));
    const uint4 u = *p;
    uint32_t w4[4] = {u.x, u.y, u.z, u.w};
    for (int e = 0; e < 4; ++e) {
      const int c = 8 * cc + 2 * e;
      float x0 = cvt_lo<DT>(w4[e]), x1 = cvt_hi<DT>(w4[e]);
      if (m) {
        x0 = __fsub_rn(x0, __ldg(m + c));
        x1 = __fsub_rn(x1, __ldg(m + c + 1));
      }
      w4[e] = (exact_code(__fsub_rn(x0, z), s, maxc) << 8) | (exact_code(__fsub_rn(x1, z), s, maxc) << 24);
    }
    *p = make_uint4(w4[0], w4[1], w4[2], w4[3]);
  }
}
// K: channels 4 cb + 32 k .. + 3 (k = 0..3) of row r, residuals from Rk, zero / scale per channel.
__device__ __noinline__ void k_codes_exact(uint8_t* rowsK, const float* Rk, const float2* kzr, const float* kss, int r,
                                           int cb, int maxc) {
  for (int k4 = 0; k4 < 4; ++k4) {
    const int c = 4 * cb + 32 * k4;
    uint32_t w[2];
    for (int pr = 0; pr < 2; ++pr) {
      const int c0 = c + 2 * pr;
      const uint32_t a = exact_code(__fsub_rn(Rk[rk_at(r, c0)], kzr[c0].x), kss[c0], maxc);
      const uint32_t b = exact_code(__fsub_rn(Rk[rk_at(r, c0 + 1)], kzr[c0 + 1].x), kss[c0 + 1], maxc);
      w[pr] = (a << 8) | (b << 24);
    }
    *reinterpret_cast<uint2*>(rowsK + elem_off(r, c)) = make_uint2(w[0], w[1]);
  }
}

// Shared memory: the pattern tables of the current (set, head), shared by the CTA's groups, then
// one block per group (its stage(s), the union of the probe values and candidate lists with the
// K residuals, per-row state).
template <int NG, int GW>
struct FullCfg {
  static constexpr int kGT = GW * 32;          // threads of a group
  static constexpr int kNS = NG == 1 ? 2 : 1;  // stages per group
  static constexpr int kXpBytes = 64 * kTabLd * 4;
  static constexpr int kListBytes = GW * (kW2Cap + kWECap) * 2;
  static constexpr int kRkBytes = 32 * kRkLd * 4;
  static constexpr int kUnion = kRkBytes > kXpBytes + kListBytes ? kRkBytes : kXpBytes + kListBytes;
  static constexpr int kStage = 0;
  static constexpr int kU = kNS * kStageBytes;
  static constexpr int kRowu = kU + kUnion;
  static constexpr int kSeed = kRowu + 64 * 4;
  static constexpr int kBest = kSeed + 64 * 4;
  static constexpr int kKkey = kBest + 64 * 8;
  static constexpr int kRraw = kKkey + 32 * 4;
  static constexpr int kOvf = kRraw + 32 * 4;
  static constexpr int kCtr = kOvf + 64 * 4;
  static constexpr int kKzr = kCtr + 16;
  static constexpr int kKs = kKzr + kD * 8;
  static constexpr int kBars = kKs + kD * 4;
  static constexpr int kGroupBytes = (kBars + 16 + 1023) & ~1023;  // keeps the stages 1024-byte aligned
};
struct TabSmem {
  int phi, hnorm, tabv, tabk, pcv, pck, total;
};
__host__ __device__ inline TabSmem tab_smem(int P) {
  const int Pp = (P + 7) & ~7;
  TabSmem s;
  int o = 0;
  auto take = [&](int bytes) { const int r = o; o = (o + bytes + 15) & ~15; return r; };
  s.phi = take(Pp * kPhiLd * 2);
  s.hnorm = take(Pp * 4);
  s.tabv = take(P * kTabLd * 4);
  s.tabk = take(P * kK1 * 4);
  s.pcv = take(kProbeAll * 4);
  s.pck = take(kK1 * 4);
  s.total = (o + 1023) & ~1023;
  return s;
}
template <int NG, int GW>
inline int full_smem_bytes(int P) {
  return tab_smem(P).total + NG * FullCfg<NG, GW>::kGroupBytes + 1024;  // + room to align the base
}

struct Task {
  int h, b, pg, L, set, phys;  // pg < 0: not a page this call fills completely
};
// The length and pattern set of the last sequence seen: a CTA's run of tasks covers few sequences.
struct SeqCache {
  int b, L, set;
};

// Task t of this call: (KV head, sequence, f-th page that the call fills completely).  The
// page-table entry is loaded here and checked by task_check, later, so that the load's latency
// can overlap other work.
__device__ __forceinline__ Task task_load(const Geom& g, int n_new, int F, int64_t t, SeqCache& sc) {
  Task k;
  k.h = (int)(t / ((int64_t)g.B * F));
  k.b = (int)((t / F) % g.B);
  const int f = (int)(t % F);
  if (k.b != sc.b) {
    sc.b = k.b;
    sc.L = g.seq_len[k.b];
    sc.set = g.seq_to_set ? g.seq_to_set[k.b] : 0;
  }
  k.L = sc.L;
  k.set = sc.set;
  k.phys = -1;
  k.pg = -1;
  // a length out of range is flagged by the partial-page kernel
  if (k.L < 0 || (int64_t)k.L + n_new > (int64_t)g.maxp * kG) return k;
  const int pg = (k.L + kG - 1) / kG + f;
  if ((pg + 1) * kG > k.L + n_new) return k;
  k.pg = pg;
  k.phys = g.page_table[(size_t)k.b * g.maxp + pg];
  return k;
}
__device__ __forceinline__ bool task_check(const Geom& g, const Task& k, bool flag) {
  if (k.pg < 0) return false;
  if (k.phys < 0 || k.phys >= g.npages) {
    if (flag) set_status(g.status, KVQ_DEV_BAD_PAGE);
    return false;
  }
  if (k.set < 0 || k.set >= g.S) {
    if (flag) set_status(g.status, KVQ_DEV_BAD_SET);
    return false;
  }
  return true;
}


// The (set, head) whose pattern tables task t uses (the set clamped into range: a task with a bad
// set index is skipped by task_check, whatever tables are staged).
__device__ __forceinline__ int task_key(const Geom& g, int F, int64_t t, SeqCache& sc) {
  const int h = (int)(t / ((int64_t)g.B * F));
  const int b = (int)((t / F) % g.B);
  if (b != sc.b) {
    sc.b = b;
    sc.L = g.seq_len[b];
    sc.set = g.seq_to_set ? g.seq_to_set[b] : 0;
  }
  return min(max(sc.set, 0), g.S - 1) * g.H + h;
}

// NG groups of GW warps per CTA.  The CTA walks its run of tasks in segments of one (set, head):
// all threads stage the segment's tables, then group gi takes the segment's tasks s0 + gi,
// s0 + gi + NG, ... on its own (named barrier gi + 1, GW * 32 threads), so the groups' phases
// interleave on the SM; a group's stage refills with its next task when the current one is done
// (two stages, the copy two tasks ahead, when NG = 1).
template <int DT, int NG, int GW>
__global__ void __launch_bounds__(NG * GW * 32, NG <= 2 ? 2 : 1) append_full_kernel(const __grid_constant__ CUtensorMap kmap,
                                                                      const __grid_constant__ CUtensorMap vmap,
                                                                      Geom g, const int32_t* __restrict__ probe,
                                                                      const float* __restrict__ pvals, int n_new,
                                                                      int F, int64_t per_cta) {
  using C = FullCfg<NG, GW>;
  constexpr int GT = C::kGT, CT = NG * GT, NS = C::kNS;
  extern __shared__ uint8_t smraw[];
  const int P = g.P, Pp = (P + 7) & ~7;
  const TabSmem ts = tab_smem(P);
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smraw) + 1023) & ~uintptr_t(1023));
  uint16_t* phi = reinterpret_cast<uint16_t*>(base + ts.phi);
  float* hnorm = reinterpret_cast<float*>(base + ts.hnorm);
  float* tabv = reinterpret_cast<float*>(base + ts.tabv);  // [P][kTabLd]: V patterns at the 32 probe channels
  float* tabk = reinterpret_cast<float*>(base + ts.tabk);  // [P][16]: K patterns at the 16 probe channels
  int32_t* pcv = reinterpret_cast<int32_t*>(base + ts.pcv);
  int32_t* pck = reinterpret_cast<int32_t*>(base + ts.pck);

  const int tid = threadIdx.x, lane = tid & 31;
  const int gi = tid / GT, gtid = tid % GT, gw = gtid >> 5;  // group; thread and warp in the group
  uint8_t* gb = base + ts.total + gi * C::kGroupBytes;
  uint8_t* stage = gb + C::kStage;
  float* Rk = reinterpret_cast<float*>(gb + C::kU);  // K residuals, rk_at(row, channel): phases F-H
  float* xp = reinterpret_cast<float*>(gb + C::kU);  // [64 rows][kTabLd] probe values: phases A-D
  uint16_t* wl2 = reinterpret_cast<uint16_t*>(gb + C::kU + C::kXpBytes) + gw * kW2Cap;  // warp's refinement list
  uint16_t* wle = reinterpret_cast<uint16_t*>(gb + C::kU + C::kXpBytes + GW * kW2Cap * 2) + gw * kWECap;
  float* rowu = reinterpret_cast<float*>(gb + C::kRowu);  // per row: exact distance to the seed
  int32_t* rseed = reinterpret_cast<int32_t*>(gb + C::kSeed);
  unsigned long long* best = reinterpret_cast<unsigned long long*>(gb + C::kBest);  // (distance, index) keys
  uint32_t* kkey = reinterpret_cast<uint32_t*>(gb + C::kKkey);  // K rows: smallest (bound, index), 7-bit tag
  float* rraw = reinterpret_cast<float*>(gb + C::kRraw);      // V rows: the vector's own range
  int32_t* ovf = reinterpret_cast<int32_t*>(gb + C::kOvf);    // per row: candidates dropped by a full list
  int32_t* ctr = reinterpret_cast<int32_t*>(gb + C::kCtr);    // [0] a tiny K scale, [1] a row overflowed
  float2* kzr = reinterpret_cast<float2*>(gb + C::kKzr);      // per K channel: z, 1/s
  float* kss = reinterpret_cast<float*>(gb + C::kKs);         // per K channel: s
  uint64_t* full = reinterpret_cast<uint64_t*>(gb + C::kBars);
  const int maxc = (1 << g.bits) - 1;
  // group barriers: named barrier gi + 1 over the group's threads (literal ids, so that the
  // kernel reserves only the barriers it uses)
  auto gsync = [&]() {
    switch (gi) {
      case 0: asm volatile("bar.sync 1, %0;" ::"n"(GT) : "memory"); break;
      case 1: asm volatile("bar.sync 2, %0;" ::"n"(GT) : "memory"); break;
      case 2: asm volatile("bar.sync 3, %0;" ::"n"(GT) : "memory"); break;
      default: asm volatile("bar.sync 4, %0;" ::"n"(GT) : "memory"); break;
    }
  };
  auto gsync_or = [&](bool v) -> bool {
    uint32_t r;
#define KVQ_BAR_OR(ID)                                                                                   \
  asm volatile("{\n .reg .pred p, q;\n setp.ne.u32 p, %1, 0;\n bar.red.or.pred q, " #ID                   \
               ", %2, p;\n selp.u32 %0, 1, 0, q;\n}\n"                                                      \
               : "=r"(r)                                                                                 \
               : "r"((uint32_t)v), "n"(GT)                                                                \
               : "memory")
    switch (gi) {
      case 0: KVQ_BAR_OR(1); break;
      case 1: KVQ_BAR_OR(2); break;
      case 2: KVQ_BAR_OR(3); break;
      default: KVQ_BAR_OR(4); break;
    }
#undef KVQ_BAR_OR
    return r != 0u;
  };

  const int64_t T = (int64_t)g.H * g.B * F;
  const int64_t t0 = (int64_t)blockIdx.x * per_cta, t1 = min(T, t0 + per_cta);

  if (gtid == 0) {
    for (int s2 = 0; s2 < NS; ++s2) fb_init(&full[s2], 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();

  SeqCache sc{-1, 0, 0};   // sequence facts for the task walk
  SeqCache ksc{-1, 0, 0};  // and for the segment keys
  // next valid task of this group at or after t (stride NG) before e, into `out`; each task of
  // the group is checked once, so the group's thread 0 flags bad page / set indices here
  auto next_valid = [&](int64_t t, int64_t e, Task& out) -> int64_t {
    for (; t < e; t += NG) {
      out = task_load(g, n_new, F, t, sc);
      if (task_check(g, out, gtid == 0)) return t;
    }
    return e;
  };
  uint32_t n_issued[2] = {0u, 0u};  // group thread 0: copies issued into each stage
  auto issue = [&](const Task& k, int buf) {
    ++n_issued[buf];
    uint8_t* dst = stage + buf * kStageBytes;
    const int tok = k.b * n_new + (k.pg * kG - k.L);
    fb_expect(&full[buf], kStageBytes);
    tma3(dst, &vmap, 0, k.h, tok, &full[buf]);
    tma3(dst + 4096, &vmap, 64, k.h, tok, &full[buf]);
    tma3(dst + 8192, &kmap, 0, k.h, tok, &full[buf]);
    tma3(dst + 12288, &kmap, 64, k.h, tok, &full[buf]);
  };
  if (gtid == 0) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&kmap)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&vmap)) : "memory");
  }

  bool dead = false;             // a stage wait of this group expired: it only joins the segment barriers
  uint32_t waits[2] = {0u, 0u};  // completed waits per stage: the parity of the next one
  int q_ = 0;                    // this group's tasks so far: the stage of the next one is q_ % NS
  for (int64_t s0 = t0; s0 < t1;) {
    // ---- the segment [s0, s1) of one (set, head); every thread computes the same bounds
    const int sh = task_key(g, F, s0, ksc);
    int64_t s1 = s0 + 1;
    while (s1 < t1 && task_key(g, F, s1, ksc) == sh) ++s1;
    const float* MK = g.kpat + (size_t)sh * P * kD;
    const float* MV = g.vpat + (size_t)sh * P * kD;
    const int Pe = p_eff(g, sh), Pep = (Pe + 7) & ~7;  // patterns in use (P is the capacity)
    const int Sw = (Pe + GW - 1) / GW;                   // patterns per warp in the bound passes
    const int j0w = min(Pe, gw * Sw), nsl = min(Pe, j0w + Sw) - j0w;

    // this group's first tasks of the segment: their copies go out before the tables are staged
    Task kc, kn;
    int64_t cur = dead ? s1 : next_valid(s0 + gi, s1, kc);
    if (gtid == 0 && cur < s1) issue(kc, q_ % NS);
    int64_t nxt = s1;
    if (NS == 2 && cur < s1) {
      nxt = next_valid(cur + NG, s1, kn);
      if (gtid == 0 && nxt < s1) issue(kn, (q_ + 1) % NS);
    }

    // ---- pattern tables of this (set, head), by every thread (the previous segment is done)
    __syncthreads();
    for (int i4 = tid; i4 < Pp * (kD / 4); i4 += CT) {
      const int n = i4 / (kD / 4), c4 = i4 % (kD / 4);
      float4 m = n < Pe ? __ldg(reinterpret_cast<const float4*>(MV + (size_t)n * kD) + c4) : make_float4(0, 0, 0, 0);
      uint16_t h4[4];
      const float mv[4] = {m.x, m.y, m.z, m.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float v = -fminf(fmaxf(mv[e], -60000.f), 60000.f);
        h4[e] = DT == KVQ_BF16 ? __bfloat16_as_ushort(__float2bfloat16_rn(v)) : __half_as_ushort(__float2half_rn(v));
      }
      *reinterpret_cast<uint2*>(phi + (size_t)n * kPhiLd + 4 * c4) =
          make_uint2(h4[0] | ((uint32_t)h4[1] << 16), h4[2] | ((uint32_t)h4[3] << 16));
    }
    for (int n = tid; n < Pp; n += CT) {
      float acc = 0.f;
      if (n < Pe) {
        const float4* m4 = reinterpret_cast<const float4*>(MV + (size_t)n * kD);
        for (int c = 0; c < kD / 4; ++c) {
          const float4 m = __ldg(m4 + c);
          acc = fmaf(m.x, m.x, acc);
          acc = fmaf(m.y, m.y, acc);
          acc = fmaf(m.z, m.z, acc);
          acc = fmaf(m.w, m.w, acc);
        }
      }
      hnorm[n] = n < Pe ? 0.5f * acc : 1e30f;
    }
    {
      const size_t o = (size_t)sh * 2;
      for (int q = tid; q < Pe * kProbeAll; q += CT)
        tabv[(q / kProbeAll) * kTabLd + q % kProbeAll] = __ldg(pvals + (o + 1) * P * kProbeAll + q);
      for (int q = tid; q < Pe * kK1; q += CT)
        tabk[q] = __ldg(pvals + o * P * kProbeAll + (size_t)(q / kK1) * kProbeAll + q % kK1);
      if (tid < kProbeAll) pcv[tid] = __ldg(probe + (o + 1) * kProbeAll + tid);
      if (tid < kK1) pck[tid] = __ldg(probe + o * kProbeAll + tid);
    }
    __syncthreads();

    // ---- this group's tasks of the segment
    while (cur < s1) {
      const int buf = q_ % NS;
      const Task k = kc;
      // the group's task after the ones in flight: its loads now, its check at the end
      const int64_t ca = (NS == 2 ? nxt : cur) + NG;
      Task kca = kc;
      if (ca < s1 && (NS == 1 || nxt < s1)) kca = task_load(g, n_new, F, ca, sc);
      uint8_t* sub = g.pool + (size_t)k.phys * g.page_bytes + (size_t)k.h * g.sub_bytes;

      if (__all_sync(kFull, fb_wait(&full[buf], waits[buf] & 1u))) {
        ++waits[buf];
      } else {
        if (lane == 0) set_status(g.status, KVQ_DEV_TIMEOUT);
        dead = true;
      }
      if (gsync_or(dead)) {
        dead = true;
        break;
      }
      uint8_t* stV = stage + buf * kStageBytes;  // V rows; K rows at + 8192
      uint8_t* stK = stV + 8192;

      // ---- A: V seeds on the tensor cores (warps 0-1); probe values of every row; resets
      if (gw < 2) {
        const uint32_t rows_s = s32(stV);
        const int r = lane & 15;
        const int rb = 16 * (gw & 1);
        uint32_t A[8][4];
  #pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          const int arow = rb + (lane & 7) + 8 * ((lane >> 3) & 1);
          const int ach = 16 * ks + 8 * (lane >> 4);
          ldsm4(rows_s + elem_off(arow, ach), A[ks][0], A[ks][1], A[ks][2], A[ks][3]);
        }
        const int tig = lane & 3;
        float b0 = INFINITY, b8 = INFINITY;  // tagged scores of rows gq and gq + 8
        for (int nt = 0; nt < Pep / 8; ++nt) {
          float acc[4];
          acc[0] = acc[2] = hnorm[8 * nt + 2 * tig];
          acc[1] = acc[3] = hnorm[8 * nt + 2 * tig + 1];
          const uint32_t bbase = s32(phi + (size_t)(8 * nt + (lane & 7)) * kPhiLd + 8 * (lane >> 3));
  #pragma unroll
          for (int kp = 0; kp < 4; ++kp) {
            uint32_t q0, q1, q2, q3;
            ldsm4(bbase + kp * 64, q0, q1, q2, q3);  // k-steps 2kp (q0, q1) and 2kp + 1 (q2, q3)
            mma_seed<DT>(acc, A[2 * kp][0], A[2 * kp][1], A[2 * kp][2], A[2 * kp][3], q0, q1);
            mma_seed<DT>(acc, A[2 * kp + 1][0], A[2 * kp + 1][1], A[2 * kp + 1][2], A[2 * kp + 1][3], q2, q3);
          }
          const int j0 = 8 * nt + 2 * tig;
          b0 = fminf(b0, fminf(__uint_as_float((__float_as_uint(acc[0]) & ~127u) | (uint32_t)j0),
                               __uint_as_float((__float_as_uint(acc[1]) & ~127u) | (uint32_t)(j0 + 1))));
          b8 = fminf(b8, fminf(__uint_as_float((__float_as_uint(acc[2]) & ~127u) | (uint32_t)j0),
                               __uint_as_float((__float_as_uint(acc[3]) & ~127u) | (uint32_t)(j0 + 1))));
        }
        b0 = fminf(b0, __shfl_xor_sync(kFull, b0, 1));
        b0 = fminf(b0, __shfl_xor_sync(kFull, b0, 2));
        b8 = fminf(b8, __shfl_xor_sync(kFull, b8, 1));
        b8 = fminf(b8, __shfl_xor_sync(kFull, b8, 2));
        const float s_lo = __shfl_sync(kFull, b0, 4 * (r & 7)), s_hi = __shfl_sync(kFull, b8, 4 * (r & 7));
        int seed = (int)(__float_as_uint(r < 8 ? s_lo : s_hi) & 127u);
        seed = min(seed, Pe - 1);

        if (lane < 16) rseed[16 * gw + r] = seed;
      } else {
        // V rows: 32 probe values, K rows 16; units of 8 values
        for (int u = gtid - 64; u < 192; u += GT - 64) {
          if (u < 128) {
            const int row = u >> 2, k0 = 8 * (u & 3);
#pragma unroll
            for (int e = 0; e < 8; ++e)
              xp[row * kTabLd + k0 + e] =
                  cvt_lo<DT>(*reinterpret_cast<const uint16_t*>(stV + elem_off(row, pcv[k0 + e])));
          } else {
            const int row = (u - 128) >> 1, k0 = 8 * (u & 1);
#pragma unroll
            for (int e = 0; e < 8; ++e)
              xp[(32 + row) * kTabLd + k0 + e] =
                  cvt_lo<DT>(*reinterpret_cast<const uint16_t*>(stK + elem_off(row, pck[k0 + e])));
          }
        }
        for (int u = gtid - 64; u < 97; u += GT - 64) {
          if (u < 64) ovf[u] = 0;
          else if (u < 96) kkey[u - 64] = 0xFFFFFFFFu;
          else ctr[0] = ctr[1] = 0;
        }
      }
      gsync();

      // ---- B: V rows: exact distance to the seed and own range (4 threads a row)
      for (int u = gtid; u < 128; u += GT) {
        const int r = u >> 2, q = u & 3;
        float x[32];
        load_x32<DT>(stV, r, q, x);
        const int s = rseed[r];
        float mx, mn, ymx = -INFINITY, ymn = INFINITY;
        range32(x, MV + (size_t)s * kD + 32 * q, mx, mn);
#pragma unroll
        for (int c = 0; c < 32; c += 2) {
          ymx = max3(ymx, x[c], x[c + 1]);
          ymn = min3(ymn, x[c], x[c + 1]);
        }
#pragma unroll
        for (int o = 1; o <= 2; o <<= 1) {
          mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, o));
          mn = fminf(mn, __shfl_xor_sync(kFull, mn, o));
          ymx = fmaxf(ymx, __shfl_xor_sync(kFull, ymx, o));
          ymn = fminf(ymn, __shfl_xor_sync(kFull, ymn, o));
        }
        if (q == 0) {
          const float U = __fsub_rn(mx, mn);
          rowu[r] = U;
          best[r] = dkey(U, s);
          rraw[r] = __fsub_rn(ymx, ymn);
        }
      }
      // K rows: bounds over 16 probe channels for this warp's patterns (lane = K row), kept in
      // registers until the K candidates are listed; the smallest (tagged with its index in the 7
      // low bits) names the seed
      float klb[kMaxSlice];
      {
        float y[kK1];
#pragma unroll
        for (int q = 0; q < kK1 / 4; ++q) {
          const float4 a = reinterpret_cast<const float4*>(xp + (32 + lane) * kTabLd)[q];
          y[4 * q] = a.x; y[4 * q + 1] = a.y; y[4 * q + 2] = a.z; y[4 * q + 3] = a.w;
        }
        uint32_t kb = 0xFFFFFFFFu;
#pragma unroll
        for (int jj = 0; jj < kMaxSlice; ++jj) {
          klb[jj] = INFINITY;
          if (jj < nsl) {
            const int j = j0w + jj;
            klb[jj] = probe_range_reg<kK1>(y, tabk + (size_t)j * kK1);
            kb = min(kb, (__float_as_uint(klb[jj]) & ~127u) | (uint32_t)j);
          }
        }
        if (nsl > 0) atomicMin(&kkey[lane], kb);
      }
      gsync();

      // ---- C: K rows: exact distance to the seed (4 threads a row)
      for (int u = gtid; u < 128; u += GT) {
        const int r = u >> 2, q = u & 3;
        const int s = min((int)(kkey[r] & 127u), Pe - 1);
        float x[32];
        load_x32<DT>(stK, r, q, x);
        float mx, mn;
        range32(x, MK + (size_t)s * kD + 32 * q, mx, mn);
#pragma unroll
        for (int o = 1; o <= 2; o <<= 1) {
          mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, o));
          mn = fminf(mn, __shfl_xor_sync(kFull, mn, o));
        }
        if (q == 0) {
          const float U = __fsub_rn(mx, mn);
          rowu[32 + r] = U;
          rseed[32 + r] = s;
          best[32 + r] = dkey(U, s);
        }
      }
      // V rows: bounds over 8 probe channels for this warp's patterns (lane = V row); a pattern
      // that could still beat the seed, or tie it with a lower index, goes on the warp's
      // refinement list, whose bounds over 32 probe channels pass the survivors to its exact list
      int nE = 0;  // entries in this warp's exact list (the same in every lane)
      {
        float y[kV1];
#pragma unroll
        for (int q = 0; q < kV1 / 4; ++q) {
          const float4 a = reinterpret_cast<const float4*>(xp + lane * kTabLd)[q];
          y[4 * q] = a.x; y[4 * q + 1] = a.y; y[4 * q + 2] = a.z; y[4 * q + 3] = a.w;
        }
        const float U = rowu[lane];
        const int s = rseed[lane];
        uint32_t mask = 0u;
#pragma unroll
        for (int jj = 0; jj < kMaxSlice; ++jj) {
          if (jj < nsl) {
            const int j = j0w + jj;
            const float lb = probe_range_reg<kV1>(y, tabv + (size_t)j * kTabLd);
            if (j != s && (lb < U || (lb == U && j < s))) mask |= 1u << jj;
          }
        }
        const int n2 = warp_compact(mask, lane, lane, j0w, wl2, 0, kW2Cap, &ovf[lane], &ctr[1]);
        __syncwarp();
        for (int b0 = 0; b0 < n2; b0 += 32) {
          const int e = b0 + lane;
          bool live = false;
          uint32_t ent = 0u;
          int r = 0;
          if (e < n2) {
            ent = wl2[e];
            r = (int)(ent >> 8);
            const int j = (int)(ent & 255u);
            const float lb = probe_range<kV2>(xp + r * kTabLd, tabv + (size_t)j * kTabLd);
            const float Ur = rowu[r];
            live = lb < Ur || (lb == Ur && j < rseed[r]);
          }
          nE = warp_append(live, ent, wle, nE, kWECap, &ovf[r], &ctr[1], lane);
        }
      }
      gsync();

      // ---- D: the K candidates of this warp's patterns join its exact list; exact distances of
      // the list (4 lanes an entry), minimum (distance, index) per row
      const int q4 = lane & 3;
      auto exact = [&](bool on, int row, int j) {
        float mx = -INFINITY, mn = INFINITY;
        if (on) {
          float x[32];
          load_x32<DT>(row < 32 ? stV : stK, row & 31, q4, x);
          range32(x, (row < 32 ? MV : MK) + (size_t)j * kD + 32 * q4, mx, mn);
        }
#pragma unroll
        for (int o = 1; o <= 2; o <<= 1) {
          mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, o));
          mn = fminf(mn, __shfl_xor_sync(kFull, mn, o));
        }
        if (on && q4 == 0) atomicMin(&best[row], dkey(__fsub_rn(mx, mn), j));
      };
      {
        const float U = rowu[32 + lane];
        const int s = rseed[32 + lane];
        uint32_t mask = 0u;
#pragma unroll
        for (int jj = 0; jj < kMaxSlice; ++jj)
          if (jj < nsl && j0w + jj != s && klb[jj] <= U) mask |= 1u << jj;
        nE = warp_compact(mask, lane, 32 + lane, j0w, wle, nE, kWECap, &ovf[32 + lane], &ctr[1]);
        __syncwarp();
        for (int b0 = 0; b0 < nE; b0 += 8) {
          const int e = b0 + (lane >> 2);
          const uint32_t ent = e < nE ? wle[e] : 0u;
          exact(e < nE, (int)(ent >> 8), (int)(ent & 255u));
        }
      }
      gsync();
      if (ctr[1]) {
        // some row's candidates did not all fit a list: that row against every pattern (warp 0)
        if (gw == 0)
          for (int row = 0; row < 64; ++row) {
            if (!ovf[row]) continue;
            for (int jb = 0; jb < Pe; jb += 8) exact(jb + (lane >> 2) < Pe, row, jb + (lane >> 2));
          }
        gsync();
      }

      // ---- F: V rows quantized (a unit: row and 32-channel group); K residuals staged
      for (int u = gtid; u < 256; u += GT) {
        if (u < 128) {
          const int r = u >> 2, q = u & 3;
          const unsigned long long bk = best[r];
          const int j = (int)(bk & 0xffffffffu);
          const bool keep = v_keep_pattern(g.vrho, __uint_as_float((uint32_t)(bk >> 32)), rraw[r]);
          float x[32];
          load_x32<DT>(stV, r, q, x);
          const float* mrow = MV + (size_t)j * kD + 32 * q;
          if (keep) {
            const float4* m4 = reinterpret_cast<const float4*>(mrow);
            float4 mv[8];
#pragma unroll
            for (int c = 0; c < 8; ++c) mv[c] = __ldg(m4 + c);
#pragma unroll
            for (int c = 0; c < 8; ++c) {
              sub2(x[4 * c], x[4 * c + 1], mv[c].x, mv[c].y, x[4 * c], x[4 * c + 1]);
              sub2(x[4 * c + 2], x[4 * c + 3], mv[c].z, mv[c].w, x[4 * c + 2], x[4 * c + 3]);
            }
          }
          float gmx = -INFINITY, gmn = INFINITY;
#pragma unroll
          for (int c = 0; c < 32; c += 2) {
            gmx = max3(gmx, x[c], x[c + 1]);
            gmn = min3(gmn, x[c], x[c + 1]);
          }
          const float s = __fdiv_rn(__fsub_rn(gmx, gmn), (float)maxc);
          const float ri = code_rcp(s);
          reinterpret_cast<float*>(sub + g.off_vs)[vsc_pos(r, q)] = s;
          reinterpret_cast<float*>(sub + g.off_vz)[vzc_pos(r, q)] = gmn;
          if (q == 0) sub[g.off_vidx + tok_pos(r)] = keep ? (uint8_t)j : (uint8_t)kRawIndex;
          uint32_t pc[16];
          const bool clean = codes_fma<32>(x, pc, [&](int, float& z0, float& z1, float& r0, float& r1) {
            z0 = z1 = gmn;
            r0 = r1 = ri;
          });
          if (clean && !tiny_scale(s)) {
            uint8_t* hb = stV + (q >> 1) * 4096;
#pragma unroll
            for (int cc = 0; cc < 4; ++cc)
              *reinterpret_cast<uint4*>(hb + swz(r, 4 * (q & 1) + cc)) =
                  make_uint4(pc[4 * cc], pc[4 * cc + 1], pc[4 * cc + 2], pc[4 * cc + 3]);
          } else {
            v_codes_exact<DT>(stV, r, q, keep ? mrow : nullptr, gmn, s, maxc);
          }
        } else {
          const int r = (u - 128) >> 2, q = u & 3;
          const int j = (int)(best[32 + r] & 0xffffffffu);
          float x[32];
          load_x32<DT>(stK, r, q, x);
          const float4* m4 = reinterpret_cast<const float4*>(MK + (size_t)j * kD + 32 * q);
          float4 mv[8];
#pragma unroll
          for (int c = 0; c < 8; ++c) mv[c] = __ldg(m4 + c);
          float4* dst = reinterpret_cast<float4*>(Rk + rk_at(r, 32 * q));
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            float4 o;
            sub2(x[4 * c], x[4 * c + 1], mv[c].x, mv[c].y, o.x, o.y);
            sub2(x[4 * c + 2], x[4 * c + 3], mv[c].z, mv[c].w, o.z, o.w);
            dst[c] = o;
          }
          if (q == 0) sub[g.off_kidx + tok_pos(r)] = (uint8_t)j;
        }
      }
      gsync();

      // ---- G: K scale and zero per channel over the page (a thread a channel)
      for (int c = gtid; c < kD; c += GT) {
        const float* col = Rk + rk_at(0, c);
        float mx = -INFINITY, mn = INFINITY;
#pragma unroll
        for (int t = 0; t < kG; t += 2) {
          const float a = col[t * kRkLd], b2 = col[(t + 1) * kRkLd];
          mx = max3(mx, a, b2);
          mn = min3(mn, a, b2);
        }
        const float s = __fdiv_rn(__fsub_rn(mx, mn), (float)maxc);
        kzr[c] = make_float2(mn, code_rcp(s));
        kss[c] = s;
        reinterpret_cast<float*>(sub + g.off_ks)[ksc_pos(c)] = s;
        reinterpret_cast<float*>(sub + g.off_kz)[ksc_pos(c)] = mn;
        if (tiny_scale(s)) ctr[0] = 1;
      }
      gsync();

      // ---- H: K codes (a unit: row and 16 channels, 4 x 4 channels 32 apart)
      for (int u = gtid; u < 256; u += GT) {
        const int r = u >> 3, cb = u & 7;
        float x[16], zs[16], rs[16];
#pragma unroll
        for (int k4 = 0; k4 < 4; ++k4) {
          const int c = 4 * cb + 32 * k4;
          const float4 a = *reinterpret_cast<const float4*>(Rk + rk_at(r, c));
          x[4 * k4] = a.x; x[4 * k4 + 1] = a.y; x[4 * k4 + 2] = a.z; x[4 * k4 + 3] = a.w;
          const float4 p0 = *reinterpret_cast<const float4*>(kzr + c);
          const float4 p1 = *reinterpret_cast<const float4*>(kzr + c + 2);
          zs[4 * k4] = p0.x; rs[4 * k4] = p0.y; zs[4 * k4 + 1] = p0.z; rs[4 * k4 + 1] = p0.w;
          zs[4 * k4 + 2] = p1.x; rs[4 * k4 + 2] = p1.y; zs[4 * k4 + 3] = p1.z; rs[4 * k4 + 3] = p1.w;
        }
        uint32_t pc[8];
        const bool clean = codes_fma<16>(x, pc, [&](int i2, float& z0, float& z1, float& r0, float& r1) {
          z0 = zs[2 * i2]; z1 = zs[2 * i2 + 1];
          r0 = rs[2 * i2]; r1 = rs[2 * i2 + 1];
        });
        if (clean && ctr[0] == 0) {
#pragma unroll
          for (int k4 = 0; k4 < 4; ++k4)
            *reinterpret_cast<uint2*>(stK + elem_off(r, 4 * cb + 32 * k4)) = make_uint2(pc[2 * k4], pc[2 * k4 + 1]);
        } else {
          k_codes_exact(stK, Rk, kzr, kss, r, cb, maxc);
        }
      }
      gsync();

      // ---- I: code words in the page's fragment order: 16-byte chunks of four words per lane,
      // the V block's chunks then the K block's, spread over the group's warps
      {
        const int nc = g.bits == 2 ? 2 : 4;  // chunks per block
        const int mi = lane >> 3, ri8 = lane & 7;
        for (int ch = gw; ch < 2 * nc; ch += GW) {
          const bool isV = ch < nc;
          const int wq = isV ? ch : ch - nc;  // chunk: words 4 wq .. 4 wq + 3 of every lane
          uint32_t* blk = reinterpret_cast<uint32_t*>(sub + (isV ? g.off_vc : 0));
          uint32_t wd[4] = {0u, 0u, 0u, 0u};
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int w = 4 * wq + u;
            // the (up to) two 16 x 16 tiles of word w and their slot offsets
#pragma unroll
            for (int tt = 0; tt < 2; ++tt) {
              if (g.bits == 4 && tt == 1) continue;
              const int tile = g.bits == 2 ? 2 * w + tt : w;
              int rt, ct;  // row tile (16 rows of the code matrix) and column tile
              if (isV) { rt = tile >> 1; ct = tile & 1; }   // V: rows = channels, 2 column tiles of tokens
              else { rt = tile >> 3; ct = tile & 7; }       // K: rows = tokens, 8 column tiles of channels
              uint32_t a0, a1, a2, a3;
              if (isV) {
                // stored [token][channel]: the transposed load gives rows = channels, columns = tokens
                const int tok = 16 * ct + 8 * (mi >> 1) + ri8, chn = 16 * rt + 8 * (mi & 1);
                ldsm4t(s32(stV) + elem_off(tok, chn), a0, a1, a2, a3);
              } else {
                const int tok = 16 * rt + 8 * (mi & 1) + ri8, chn = 16 * ct + 8 * (mi >> 1);
                ldsm4(s32(stK) + elem_off(tok, chn), a0, a1, a2, a3);
              }
              const uint32_t av[4] = {a0, a1, a2, a3};
#pragma unroll
              for (int rg = 0; rg < 4; ++rg) {
                if (g.bits == 2) {
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
          *reinterpret_cast<uint4*>(blk + wq * 128 + lane * 4) = make_uint4(wd[0], wd[1], wd[2], wd[3]);
        }
      }

      // ---- end of the task: this stage refills with the group's task NS ahead (the generic
      // accesses of this task to the stage ordered before the tensor copy that overwrites it)
      int64_t after = s1;
      if (ca < s1 && (NS == 1 || nxt < s1)) after = task_check(g, kca, gtid == 0) ? ca : next_valid(ca + NG, s1, kca);
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      gsync();
      ++q_;
      if (gtid == 0 && after < s1) issue(kca, (q_ + NS - 1) % NS);
      if (NS == 2) {
        cur = nxt;
        kc = kn;
        nxt = after;
        kn = kca;
      } else {
        cur = after;
        kc = kca;
      }
    }
    s0 = s1;
  }
  // drain: every copy this group issued lands before the CTA exits (phases complete in order,
  // so the newest of each stage covers the older ones; only a group whose wait expired has
  // copies that were never awaited)
  if (gtid == 0 && dead) {
    for (int b2 = 0; b2 < NS; ++b2)
      if (n_issued[b2] > waits[b2] && !fb_wait(&full[b2], (n_issued[b2] - 1u) & 1u)) set_status(g.status, KVQ_DEV_TIMEOUT);
  }
}

}  // namespace

bool append_full_eligible(const Geom& g, int n_new) {
  return !g.tx && g.P <= 128 && n_new >= kG && g.B > 0 && (g.dtype == KVQ_BF16 || g.dtype == KVQ_F16);
}

namespace {
template <int NG, int GW>
cudaError_t launch_full_cfg(const Geom& g, const CUtensorMap& kmap, const CUtensorMap& vmap, int n_new, int F,
                            const void* probe, const void* pv, cudaStream_t st) {
  const int64_t T = (int64_t)g.H * g.B * F;
  const int smem = full_smem_bytes<NG, GW>(g.P);
  int dev = 0, sms = 148, occ = 1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  auto kern = g.dtype == KVQ_BF16 ? append_full_kernel<KVQ_BF16, NG, GW> : append_full_kernel<KVQ_F16, NG, GW>;
  if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem)) != cudaSuccess) return e;
  if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, NG * GW * 32, smem)) != cudaSuccess) return e;
  const int64_t ctas = std::max<int64_t>(1, std::min<int64_t>(T, (int64_t)std::max(occ, 1) * sms));
  const int64_t per = (T + ctas - 1) / ctas;
  kern<<<(unsigned)((T + per - 1) / per), NG * GW * 32, smem, st>>>(kmap, vmap, g, (const int32_t*)probe,
                                                                  (const float*)pv, n_new, F, per);
  return cudaGetLastError();
}
}  // namespace

cudaError_t launch_append_full(const Geom& g, const void* k_new, const void* v_new, int n_new, const void* probe,
                               const void* pv, cudaStream_t st) {
  const int F = n_new / kG + 1;  // most pages a sequence can fill completely in this call
  // K / V input as (128 channels, KV heads, tokens of all sequences), boxes of 64 channels x 32 tokens
  CUtensorMap kmap, vmap;
  const CUtensorMapDataType dt = g.dtype == KVQ_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  const cuuint64_t dims[3] = {(cuuint64_t)kD, (cuuint64_t)g.H, (cuuint64_t)g.B * n_new};
  const cuuint64_t strides[2] = {(cuuint64_t)kD * 2, (cuuint64_t)g.H * kD * 2};
  const cuuint32_t box[3] = {64, 1, 32};
  cudaError_t e;
  if ((e = encode_tiled_map(&kmap, dt, 3, k_new, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B)) != cudaSuccess ||
      (e = encode_tiled_map(&vmap, dt, 3, v_new, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B)) != cudaSuccess)
    return e;
  // up to 64 patterns: groups of 4 warps (a group a task), all of a CTA on one (set, head); more:
  // one group of 8
  if (g.P <= 4 * kMaxSlice) return launch_full_cfg<kFullGroups, 4>(g, kmap, vmap, n_new, F, probe, pv, st);
  return launch_full_cfg<1, 8>(g, kmap, vmap, n_new, F, probe, pv, st);
}

}  // namespace kvq
