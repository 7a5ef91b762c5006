// Quantize-append of full pages ("PatternKV", Section 3.2: nearest pattern under the min-max
// distance, Eq. 6, residual quantized with Eq. 1; Section 3.3: V adaptive threshold; Section
// 4.1 granularity): every page whose 32 tokens all arrive in this call, which is nearly all of
// them in a prefill.  Pages only partly written by the call go through append_pages_kernel.
//
// Persistent CTAs of 4 warps, each walking a contiguous run of (KV head, sequence, page) tasks.
// A task's 32 V rows and 32 K rows arrive by TMA (two 64-channel boxes each, 128-byte swizzle)
// into one of two stage buffers; the copy of the task after next is issued as soon as a stage is
// free.  Warps 0-1 handle the V rows, warps 2-3 the K rows (16 rows each), with no block-wide
// barrier inside a task: two lanes per row, lane (r, h) holding channels [64 h, 64 h + 64) of
// its row in registers and half of the patterns for the bounds.
//
// Exact nearest pattern (same fp32 operations as the definition, lowest index on ties):
//   V rows: seed = the Euclidean nearest pattern (m16n8k16 tensor-core scores |m|^2/2 - x.m
//     against the patterns' bf16 / fp16 parts; only a guess), U = its exact d_mm; then a lower
//     bound for every other pattern from the 8 channels where the patterns differ most (the
//     residual range over a channel subset never exceeds the range over all channels; same fp32
//     subtractions), refined to 32 channels for the survivors, and the exact d_mm of the few that
//     still could beat (or tie below) the seed.
//   K rows: the 16-channel bound for every pattern first (K's outlier channels make it nearly
//     exact), seed = its argmin, then the exact d_mm of the patterns whose bound does not exceed it.
// Quantization: residuals in registers; V scale / zero per (token, 32-channel group) in the lane;
// K scale / zero per channel from the residuals staged in shared memory.  A code is
// rne(fl32(fl32(R - z) / s)), produced by one FMA, v = t (1/s) + (1.5 * 2^15 + 0.5): the
// integer part of (t / s + 1/2) lands in bits 8-15 and its fraction in bits 0-7.  The fraction
// byte is zero only when t / s lies within 2^-9 of a half-integer; only there could the
// reciprocal's error move the result across a rounding boundary, and those codes are recomputed
// with the correctly rounded division.  The 16-bit codes are written over the staged input rows
// and ldmatrix(.trans) brings them back in the page's fragment order, where a few shifts pack
// them into words.
#include <algorithm>
#include <cstdint>

#include "kvq_common.cuh"
#include "kvq_internal.h"

namespace kvq {

namespace {

constexpr int kFThreads = 128;
constexpr int kProbeAll = 32;  // probe channels per pattern set in the prep tables
constexpr int kV1 = 8;         // V: first-level bound channels
constexpr int kK1 = 16;        // K: bound channels
constexpr int kPhiLd = 136;    // 16-bit row stride of the pattern table for ldmatrix (272 B: conflict-free)
constexpr int kRkLd = 132;     // fp32 row stride of the staged K residuals
constexpr int kStageBytes = 16384;  // V rows (2 x 4 KB halves) then K rows (2 x 4 KB halves)
constexpr uint32_t kFSpin = 1u << 22;
constexpr float kCodeMagic = 49152.5f;  // 1.5 * 2^15 + 0.5: 8 fractional bits, +1/2 folded in

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

struct FullSmem {
  int stage, rk, phi, hnorm, tabv, tabk, pcv, pck, lbk, kzr, ks, bars, total;
};
__host__ __device__ inline FullSmem full_smem(int P) {
  const int Pp = (P + 7) & ~7;
  FullSmem s;
  int o = 0;
  s.stage = o; o += 2 * kStageBytes;
  s.rk = o; o += 32 * kRkLd * 4;
  s.phi = o; o += Pp * kPhiLd * 2;
  s.hnorm = o; o += Pp * 4;
  s.tabv = o; o += P * kProbeAll * 4;
  s.tabk = o; o += P * kK1 * 4;
  s.pcv = o; o += kProbeAll * 4;
  s.pck = o; o += kK1 * 4;
  s.lbk = o; o += 32 * ((P + 7) & ~7) * 2;
  o = (o + 15) & ~15;
  s.kzr = o; o += kD * 8;
  s.ks = o; o += kD * 4;
  s.bars = o; o += 2 * 8;
  s.total = o + 1024;  // room to align the stage buffers to 1024 B (128-byte swizzle atoms)
  return s;
}

struct Task {
  int h, b, pg, L, set;
  bool ok;
};

// Task t of this call: (KV head, sequence, f-th page that the call fills completely).
__device__ __forceinline__ Task task_of(const Geom& g, int n_new, int F, int64_t t, bool flag) {
  Task k;
  k.h = (int)(t / ((int64_t)g.B * F));
  k.b = (int)((t / F) % g.B);
  const int f = (int)(t % F);
  k.L = g.seq_len[k.b];
  k.ok = false;
  k.set = 0;
  k.pg = 0;
  if (k.L < 0 || (int64_t)k.L + n_new > (int64_t)g.maxp * kG) return k;  // flagged by the partial-page kernel
  k.pg = (k.L + kG - 1) / kG + f;
  if ((k.pg + 1) * kG > k.L + n_new) return k;
  const int phys = g.page_table[(size_t)k.b * g.maxp + k.pg];
  if (phys < 0 || phys >= g.npages) {
    if (flag) set_status(g.status, KVQ_DEV_BAD_PAGE);
    return k;
  }
  k.set = g.seq_to_set ? g.seq_to_set[k.b] : 0;
  if (k.set < 0 || k.set >= g.S) {
    if (flag) set_status(g.status, KVQ_DEV_BAD_SET);
    return k;
  }
  k.ok = true;
  return k;
}

// Range of x - m over this lane's 64 channels (x in registers, m the pattern half in global memory).
__device__ __forceinline__ void half_range(const float (&x)[64], const float* __restrict__ m, float& mx, float& mn) {
  const float4* m4 = reinterpret_cast<const float4*>(m);
  mx = -INFINITY;
  mn = INFINITY;
#pragma unroll
  for (int c = 0; c < 16; ++c) {
    const float4 v = __ldg(m4 + c);
    float r0, r1, r2, r3;
    sub2(x[4 * c], x[4 * c + 1], v.x, v.y, r0, r1);
    sub2(x[4 * c + 2], x[4 * c + 3], v.z, v.w, r2, r3);
    mx = max3(mx, r0, r1);
    mn = min3(mn, r0, r1);
    mx = max3(mx, r2, r3);
    mn = min3(mn, r2, r3);
  }
}

// Exact d_mm of the candidates of both lanes of a row (lane hh's candidates: bit i of its mask =
// pattern jb(hh) + i, jb(0) = 0, jb(1) = P2), in ascending pattern order; the best (distance,
// index) so far is (bd, bj).  Both lanes of a row run the same list.
__device__ __forceinline__ void exact_candidates(const float (&x)[64], const float* __restrict__ M, int hh, int P2,
                                                 unsigned long long mine, float& bd, int& bj) {
  const unsigned long long other = __shfl_xor_sync(kFull, mine, 16);
  unsigned long long ml = hh ? other : mine, mh = hh ? mine : other;
#pragma unroll 1
  for (int q = 0; q < 2; ++q) {
    unsigned long long mq = q ? mh : ml;
    while (__any_sync(kFull, mq != 0ull)) {
      const bool act = mq != 0ull;
      const int j = act ? q * P2 + __ffsll((long long)mq) - 1 : 0;
      if (act) mq &= mq - 1;
      float mx = -INFINITY, mn = INFINITY;
      if (act) half_range(x, M + (size_t)j * kD + 64 * hh, mx, mn);
      mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 16));
      mn = fminf(mn, __shfl_xor_sync(kFull, mn, 16));
      const float d = __fsub_rn(mx, mn);
      if (act && (d < bd || (d == bd && j < bj))) { bd = d; bj = j; }
    }
  }
}

// Codes of this lane's 64 residuals as 32 pairs of 16-bit (code << 8 | fraction) words; zr(i,
// z0, z1, r0, r1) gives the zero and reciprocal scale of values 2i, 2i + 1.  Returns true if
// every fraction byte is nonzero (no code within 2^-9 of a rounding boundary).
template <class ZR>
__device__ __forceinline__ bool codes64(const float (&x)[64], uint32_t (&p)[32], ZR zr) {
  uint32_t acc = 0x01000100u;
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    float z0, z1, r0, r1, t0, t1, v0, v1;
    zr(i, z0, z1, r0, r1);
    sub2(x[2 * i], x[2 * i + 1], z0, z1, t0, t1);
    fma2f(t0, t1, r0, r1, kCodeMagic, kCodeMagic, v0, v1);
    const uint32_t w = __byte_perm(__float_as_uint(v0), __float_as_uint(v1), 0x5410);
    p[i] = w;
    acc &= (w & 0x00FF00FFu) + 0x00FF00FFu;
  }
  return (acc & 0x01000100u) == 0x01000100u;
}

// Exact code (the definition: the correctly rounded quotient, round half to even, clamp).
__device__ __forceinline__ uint32_t exact_code(float R, float z, float s, int maxc) {
  if (s == 0.0f) return 0u;
  const float u = __fdiv_rn(__fsub_rn(R, z), s);
  return (uint32_t)min(max(__float2int_rn(u), 0), maxc);
}

template <int DT>
__global__ void __launch_bounds__(kFThreads, 1) append_full_kernel(const __grid_constant__ CUtensorMap kmap,
                                                                   const __grid_constant__ CUtensorMap vmap, Geom g,
                                                                   const int32_t* __restrict__ probe,
                                                                   const float* __restrict__ pvals, int n_new,
                                                                   int F, int64_t per_cta) {
  extern __shared__ uint8_t smraw[];
  const int P = g.P, Pp = (P + 7) & ~7;
  const FullSmem sp = full_smem(P);
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smraw) + 1023) & ~uintptr_t(1023));
  uint8_t* stage = base + sp.stage;
  float* Rk = reinterpret_cast<float*>(base + sp.rk);
  uint16_t* phi = reinterpret_cast<uint16_t*>(base + sp.phi);
  float* hnorm = reinterpret_cast<float*>(base + sp.hnorm);
  float* tabv = reinterpret_cast<float*>(base + sp.tabv);
  float* tabk = reinterpret_cast<float*>(base + sp.tabk);
  int32_t* pcv = reinterpret_cast<int32_t*>(base + sp.pcv);
  int32_t* pck = reinterpret_cast<int32_t*>(base + sp.pck);
  __half* lbk = reinterpret_cast<__half*>(base + sp.lbk);
  float2* kzr = reinterpret_cast<float2*>(base + sp.kzr);  // per K channel: z, 1/s
  float* kss = reinterpret_cast<float*>(base + sp.ks);       // per K channel: s
  uint64_t* full = reinterpret_cast<uint64_t*>(base + sp.bars);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const bool isV = warp < 2;
  const int r = lane & 15, hh = lane >> 4;
  const int row = 16 * (warp & 1) + r;
  const int LdP = (P + 7) & ~7;  // row stride of the K bound table (halves)
  const int maxc = (1 << g.bits) - 1;

  const int64_t T = (int64_t)g.H * g.B * F;
  const int64_t t0 = (int64_t)blockIdx.x * per_cta, t1 = min(T, t0 + per_cta);

  if (tid == 0) {
    fb_init(&full[0], 1);
    fb_init(&full[1], 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();

  // next valid task at or after t (t1 if none); the scan visits every task once, so thread 0
  // flags bad page / set indices here
  auto next_valid = [&](int64_t t) -> int64_t {
    for (; t < t1; ++t)
      if (task_of(g, n_new, F, t, tid == 0).ok) return t;
    return t1;
  };
  uint32_t n_issued[2] = {0u, 0u};  // thread 0: copies issued into each stage
  auto issue = [&](int64_t t, int buf) {
    ++n_issued[buf];
    const Task k = task_of(g, n_new, F, t, false);
    uint8_t* dst = stage + buf * kStageBytes;
    const int tok = k.b * n_new + (k.pg * kG - k.L);
    fb_expect(&full[buf], kStageBytes);
    tma3(dst, &vmap, 0, k.h, tok, &full[buf]);
    tma3(dst + 4096, &vmap, 64, k.h, tok, &full[buf]);
    tma3(dst + 8192, &kmap, 0, k.h, tok, &full[buf]);
    tma3(dst + 12288, &kmap, 64, k.h, tok, &full[buf]);
  };

  int64_t cur = next_valid(t0);
  if (tid == 0) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&kmap)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&vmap)) : "memory");
    if (cur < t1) issue(cur, 0);
  }
  int64_t nxt = cur < t1 ? next_valid(cur + 1) : t1;
  if (tid == 0 && nxt < t1) issue(nxt, 1);

  int cached_sh = -1;
  bool timed_out = false;
  for (int i = 0; cur < t1; ++i) {
    const int buf = i & 1;
    const Task k = task_of(g, n_new, F, cur, false);
    const int sh = k.set * g.H + k.h;
    const float* MK = g.kpat + (size_t)sh * P * kD;
    const float* MV = g.vpat + (size_t)sh * P * kD;
    const int Pe = p_eff(g, sh), Pep = (Pe + 7) & ~7;  // patterns in use (P is the capacity)
    const int P2 = (Pe + 1) >> 1;
    const int jb = hh * P2, je = min(Pe, jb + P2);  // this lane's pattern half
    uint8_t* sub = g.pool + (size_t)g.page_table[(size_t)k.b * g.maxp + k.pg] * g.page_bytes + (size_t)k.h * g.sub_bytes;

    // ---- pattern tables of this (set, head), staged when they change
    if (sh != cached_sh) {
      cached_sh = sh;
      for (int i4 = tid; i4 < Pp * (kD / 4); i4 += kFThreads) {
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
      for (int n = tid; n < Pp; n += kFThreads) {
        float acc = 0.f;
        if (n < Pe)
          for (int c = 0; c < kD; ++c) { const float m = __ldg(MV + (size_t)n * kD + c); acc = fmaf(m, m, acc); }
        hnorm[n] = n < Pe ? 0.5f * acc : 1e30f;
      }
      const size_t o = (size_t)sh * 2;
      for (int q = tid; q < Pe * kProbeAll; q += kFThreads) tabv[q] = __ldg(pvals + (o + 1) * P * kProbeAll + q);
      for (int q = tid; q < Pe * kK1; q += kFThreads)
        tabk[q] = __ldg(pvals + o * P * kProbeAll + (size_t)(q / kK1) * kProbeAll + q % kK1);
      if (tid < kProbeAll) pcv[tid] = __ldg(probe + (o + 1) * kProbeAll + tid);
      if (tid < kK1) pck[tid] = __ldg(probe + o * kProbeAll + tid);
      __syncthreads();
    }

    if (!__all_sync(kFull, fb_wait(&full[buf], (uint32_t)((i >> 1) & 1)))) {
      if (lane == 0) set_status(g.status, KVQ_DEV_TIMEOUT);
      timed_out = true;
    }
    if (__syncthreads_or(timed_out)) break;
    uint8_t* rows = stage + buf * kStageBytes + (isV ? 0 : 8192);
    const uint32_t rows_s = s32(rows);

    // ---- this lane's 64 channels of its row
    float x[64];
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const uint4 u = *reinterpret_cast<const uint4*>(rows + hh * 4096 + swz(row, c));
      const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        x[8 * c + 2 * e] = cvt_lo<DT>(w4[e]);
        x[8 * c + 2 * e + 1] = cvt_hi<DT>(w4[e]);
      }
    }
    auto row_val = [&](int ch) -> float {
      const uint16_t u = *reinterpret_cast<const uint16_t*>(rows + elem_off(row, ch));
      return cvt_lo<DT>((uint32_t)u);
    };

    float bd;
    int bj;
    float rraw = 0.f;
    unsigned long long mask = 0ull;  // this lane's candidates: bit j - jb
    if (isV) {
      // ---- seed: Euclidean scores on the tensor cores (rows 16 (warp & 1) .. +15, all patterns)
      const int rb = 16 * (warp & 1);
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

      // ---- U = exact d_mm of the seed; the vector's own range (adaptive threshold)
      float mx, mn;
      half_range(x, MV + (size_t)seed * kD + 64 * hh, mx, mn);
      float ymx = -INFINITY, ymn = INFINITY;
#pragma unroll
      for (int c = 0; c < 64; c += 2) {
        ymx = max3(ymx, x[c], x[c + 1]);
        ymn = min3(ymn, x[c], x[c + 1]);
      }
      mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 16));
      mn = fminf(mn, __shfl_xor_sync(kFull, mn, 16));
      ymx = fmaxf(ymx, __shfl_xor_sync(kFull, ymx, 16));
      ymn = fminf(ymn, __shfl_xor_sync(kFull, ymn, 16));
      const float U = __fsub_rn(mx, mn);
      rraw = __fsub_rn(ymx, ymn);
      bd = U;
      bj = seed;

      // ---- bounds: 8 channels for every pattern of this lane's half, 32 for the survivors
      float pv[kProbeAll];
#pragma unroll
      for (int u = 0; u < kProbeAll; ++u) pv[u] = row_val(pcv[u]);
      for (int j = jb; j < je; ++j) {
        const float4* t4 = reinterpret_cast<const float4*>(tabv + (size_t)j * kProbeAll);
        float lmx = -INFINITY, lmn = INFINITY;
#pragma unroll
        for (int q = 0; q < kV1 / 4; ++q) {
          const float4 m = t4[q];
          float r0, r1, r2, r3;
          sub2(pv[4 * q], pv[4 * q + 1], m.x, m.y, r0, r1);
          sub2(pv[4 * q + 2], pv[4 * q + 3], m.z, m.w, r2, r3);
          lmx = max3(lmx, r0, r1);
          lmn = min3(lmn, r0, r1);
          lmx = max3(lmx, r2, r3);
          lmn = min3(lmn, r2, r3);
        }
        float lb = __fsub_rn(lmx, lmn);
        bool live = j != seed && (lb < U || (lb == U && j < seed));
        if (live) {
#pragma unroll
          for (int q = kV1 / 4; q < kProbeAll / 4; ++q) {
            const float4 m = t4[q];
            float r0, r1, r2, r3;
            sub2(pv[4 * q], pv[4 * q + 1], m.x, m.y, r0, r1);
            sub2(pv[4 * q + 2], pv[4 * q + 3], m.z, m.w, r2, r3);
            lmx = max3(lmx, r0, r1);
            lmn = min3(lmn, r0, r1);
            lmx = max3(lmx, r2, r3);
            lmn = min3(lmn, r2, r3);
          }
          lb = __fsub_rn(lmx, lmn);
          live = lb < U || (lb == U && j < seed);
        }
        if (live) mask |= 1ull << (j - jb);
      }
      exact_candidates(x, MV, hh, P2, mask, bd, bj);
    } else {
      // ---- bounds over 16 channels for every pattern of this lane's half; seed = their argmin
      float pk[kK1];
#pragma unroll
      for (int u = 0; u < kK1; ++u) pk[u] = row_val(pck[u]);
      float lbest = INFINITY;
      int lj = jb;
      for (int j = jb; j < je; ++j) {
        const float4* t4 = reinterpret_cast<const float4*>(tabk + (size_t)j * kK1);
        float lmx = -INFINITY, lmn = INFINITY;
#pragma unroll
        for (int q = 0; q < kK1 / 4; ++q) {
          const float4 m = t4[q];
          float r0, r1, r2, r3;
          sub2(pk[4 * q], pk[4 * q + 1], m.x, m.y, r0, r1);
          sub2(pk[4 * q + 2], pk[4 * q + 3], m.z, m.w, r2, r3);
          lmx = max3(lmx, r0, r1);
          lmn = min3(lmn, r0, r1);
          lmx = max3(lmx, r2, r3);
          lmn = min3(lmn, r2, r3);
        }
        const float lb = __fsub_rn(lmx, lmn);
        lbk[row * LdP + j] = __float2half_rz(lb);  // rounded toward zero: still a lower bound
        if (lb < lbest) { lbest = lb; lj = j; }
      }
      const float olb = __shfl_xor_sync(kFull, lbest, 16);
      const int oj = __shfl_xor_sync(kFull, lj, 16);
      if (olb < lbest || (olb == lbest && oj < lj)) { lbest = olb; lj = oj; }
      const int seed = min(max(lj, 0), Pe - 1);
      float mx, mn;
      half_range(x, MK + (size_t)seed * kD + 64 * hh, mx, mn);
      mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 16));
      mn = fminf(mn, __shfl_xor_sync(kFull, mn, 16));
      const float U = __fsub_rn(mx, mn);
      bd = U;
      bj = seed;
      __syncwarp();
      for (int j = jb; j < je; ++j) {
        const float lb = __half2float(lbk[row * LdP + j]);
        if (j != seed && lb <= U) mask |= 1ull << (j - jb);
      }
      exact_candidates(x, MK, hh, P2, mask, bd, bj);
    }

    // ---- index, then residuals (the pattern, or nothing for a V vector the threshold rejects)
    const bool keep = !isV || v_keep_pattern(g.vrho, bd, rraw);
    if (hh == 0) sub[(isV ? g.off_vidx : g.off_kidx) + tok_pos(row)] = keep ? (uint8_t)bj : (uint8_t)kRawIndex;
    {
      const float4* m4 = reinterpret_cast<const float4*>((isV ? MV : MK) + (size_t)bj * kD + 64 * hh);
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        const float4 m = keep ? __ldg(m4 + c) : make_float4(0.f, 0.f, 0.f, 0.f);
        sub2(x[4 * c], x[4 * c + 1], m.x, m.y, x[4 * c], x[4 * c + 1]);
        sub2(x[4 * c + 2], x[4 * c + 3], m.z, m.w, x[4 * c + 2], x[4 * c + 3]);
      }
    }

    uint32_t pcode[32];
    if (isV) {
      // ---- V: scale / zero of this lane's two groups (channels 32 (2 hh + q) ..), codes
      float gz[2], gr[2], ss[2];
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        float gmx = -INFINITY, gmn = INFINITY;
#pragma unroll
        for (int c = 0; c < 32; c += 2) {
          gmx = max3(gmx, x[32 * q + c], x[32 * q + c + 1]);
          gmn = min3(gmn, x[32 * q + c], x[32 * q + c + 1]);
        }
        const float s = __fdiv_rn(__fsub_rn(gmx, gmn), (float)maxc);
        const float ri = s != 0.0f ? __frcp_rn(s) : 0.0f;
        ss[q] = s;
        gz[q] = gmn;
        gr[q] = ri;
        const int grp = 2 * hh + q;
        reinterpret_cast<float*>(sub + g.off_vs)[vsc_pos(row, grp)] = s;
        reinterpret_cast<float*>(sub + g.off_vz)[vzc_pos(row, grp)] = gmn;
      }
      const bool clean = codes64(x, pcode, [&](int i2, float& z0, float& z1, float& r0, float& r1) {
        z0 = z1 = gz[i2 >> 4];
        r0 = r1 = gr[i2 >> 4];
      });
      if (!clean) {
#pragma unroll
        for (int i2 = 0; i2 < 32; ++i2) {
          const uint32_t c0 = exact_code(x[2 * i2], gz[i2 >> 4], ss[i2 >> 4], maxc);
          const uint32_t c1 = exact_code(x[2 * i2 + 1], gz[i2 >> 4], ss[i2 >> 4], maxc);
          pcode[i2] = (c0 << 8) | 0x80u | (c1 << 24) | 0x800000u;
        }
      }
    } else {
      // ---- K: residuals to shared memory; scale / zero per channel over the page's 32 tokens
      float4* dst = reinterpret_cast<float4*>(Rk + row * kRkLd + 64 * hh);
#pragma unroll
      for (int c = 0; c < 16; ++c) dst[c] = make_float4(x[4 * c], x[4 * c + 1], x[4 * c + 2], x[4 * c + 3]);
      asm volatile("bar.sync 2, 64;" ::: "memory");
      {
        const int c2 = 2 * (tid - 64);  // channels c2, c2 + 1
        float mx0 = -INFINITY, mn0 = INFINITY, mx1 = -INFINITY, mn1 = INFINITY;
#pragma unroll 8
        for (int t = 0; t < 32; t += 2) {
          const float2 a = *reinterpret_cast<const float2*>(Rk + t * kRkLd + c2);
          const float2 b2 = *reinterpret_cast<const float2*>(Rk + (t + 1) * kRkLd + c2);
          mx0 = max3(mx0, a.x, b2.x);
          mn0 = min3(mn0, a.x, b2.x);
          mx1 = max3(mx1, a.y, b2.y);
          mn1 = min3(mn1, a.y, b2.y);
        }
        const float s0 = __fdiv_rn(__fsub_rn(mx0, mn0), (float)maxc), s1 = __fdiv_rn(__fsub_rn(mx1, mn1), (float)maxc);
        *reinterpret_cast<float4*>(kzr + c2) =
            make_float4(mn0, s0 != 0.0f ? __frcp_rn(s0) : 0.0f, mn1, s1 != 0.0f ? __frcp_rn(s1) : 0.0f);
        *reinterpret_cast<float2*>(kss + c2) = make_float2(s0, s1);
        float* ksg = reinterpret_cast<float*>(sub + g.off_ks);
        float* kzg = reinterpret_cast<float*>(sub + g.off_kz);
        ksg[ksc_pos(c2)] = s0;
        ksg[ksc_pos(c2 + 1)] = s1;
        kzg[ksc_pos(c2)] = mn0;
        kzg[ksc_pos(c2 + 1)] = mn1;
      }
      asm volatile("bar.sync 2, 64;" ::: "memory");
      const float4* kz4 = reinterpret_cast<const float4*>(kzr + 64 * hh);  // (z, 1/s) of two channels
      const bool clean = codes64(x, pcode, [&](int i2, float& z0, float& z1, float& r0, float& r1) {
        const float4 q = kz4[i2];
        z0 = q.x; r0 = q.y; z1 = q.z; r1 = q.w;
      });
      if (!clean) {
#pragma unroll
        for (int i2 = 0; i2 < 32; ++i2) {
          const int c = 64 * hh + 2 * i2;
          const uint32_t c0 = exact_code(x[2 * i2], kzr[c].x, kss[c], maxc);
          const uint32_t c1 = exact_code(x[2 * i2 + 1], kzr[c + 1].x, kss[c + 1], maxc);
          pcode[i2] = (c0 << 8) | 0x80u | (c1 << 24) | 0x800000u;
        }
      }
    }

    // ---- 16-bit codes over this lane's half of its (already consumed) input row
#pragma unroll
    for (int c = 0; c < 8; ++c)
      *reinterpret_cast<uint4*>(rows + hh * 4096 + swz(row, c)) =
          make_uint4(pcode[4 * c], pcode[4 * c + 1], pcode[4 * c + 2], pcode[4 * c + 3]);
    if (isV) asm volatile("bar.sync 1, 64;" ::: "memory");
    else asm volatile("bar.sync 2, 64;" ::: "memory");

    // ---- words in the page's fragment order: lane = MMA lane, this warp's four words per chunk
    {
      const int q = warp & 1;
      uint32_t* blk = reinterpret_cast<uint32_t*>(sub + (isV ? g.off_vc : 0));
      const int mi = lane >> 3, ri8 = lane & 7;
      const int nchunk = g.bits == 2 ? 1 : 2;  // 16-byte chunks of four words per lane and warp
      for (int cq = 0; cq < nchunk; ++cq) {
        const int wq = (g.bits == 2 ? q : 2 * q + cq);  // chunk index: words 4 wq .. 4 wq + 3
        uint32_t wd[4] = {0u, 0u, 0u, 0u};
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int w = 4 * wq + u;
          // the (up to) two 16 x 16 tiles of word w and their slot offsets
#pragma unroll
          for (int tt = 0; tt < 2; ++tt) {
            if (g.bits == 4 && tt == 1) continue;
            int tile;
            if (g.bits == 2) tile = 2 * w + tt;
            else tile = w;
            int rt, ct;  // row tile (16 rows of the code matrix) and column tile
            if (isV) { rt = tile >> 1; ct = tile & 1; }   // V: rows = channels, 2 column tiles of tokens
            else { rt = tile >> 3; ct = tile & 7; }       // K: rows = tokens, 8 column tiles of channels
            uint32_t a0, a1, a2, a3;
            if (isV) {
              // stored [token][channel]: the transposed load gives rows = channels, columns = tokens
              const int tok = 16 * ct + 8 * (mi >> 1) + ri8, ch = 16 * rt + 8 * (mi & 1);
              ldsm4t(s32(stage + buf * kStageBytes) + elem_off(tok, ch), a0, a1, a2, a3);
            } else {
              const int tok = 16 * rt + 8 * (mi & 1) + ri8, ch = 16 * ct + 8 * (mi >> 1);
              ldsm4(s32(stage + buf * kStageBytes + 8192) + elem_off(tok, ch), a0, a1, a2, a3);
            }
            const uint32_t av[4] = {a0, a1, a2, a3};
#pragma unroll
            for (int rg = 0; rg < 4; ++rg) {
              if (g.bits == 2) {
                const int s = 4 * tt + rg;  // 2-bit slot: codes at bits 2s and 16 + 2s
                const uint32_t v = av[rg] & 0x03000300u;
                wd[u] |= s < 4 ? v >> (8 - 2 * s) : v << (2 * s - 8);
              } else {
                const int s = rg;  // 4-bit slot: codes at bits 4s and 16 + 4s
                const uint32_t v = av[rg] & 0x0F000F00u;
                wd[u] |= s < 2 ? v >> (8 - 4 * s) : v << (4 * s - 8);
              }
            }
          }
        }
        *reinterpret_cast<uint4*>(blk + wq * 128 + lane * 4) = make_uint4(wd[0], wd[1], wd[2], wd[3]);
      }
    }

    // ---- stage free: issue the task after next into it (the generic accesses of this task to the
    // stage ordered before the tensor copy that overwrites it)
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    __syncthreads();
    const int64_t after = nxt < t1 ? next_valid(nxt + 1) : t1;
    if (tid == 0 && after < t1) issue(after, buf);
    cur = nxt;
    nxt = after;
  }
  // drain (after a timeout): the newest copy issued into each stage must land before the CTA
  // exits; phases complete in order, so that covers the older ones
  if (tid == 0 && timed_out) {
    for (int b2 = 0; b2 < 2; ++b2)
      if (n_issued[b2] > 0 && !fb_wait(&full[b2], (n_issued[b2] - 1u) & 1u)) set_status(g.status, KVQ_DEV_TIMEOUT);
  }
}

}  // namespace

bool append_full_eligible(const Geom& g, int n_new) {
  return !g.tx && g.P <= 128 && n_new >= kG && g.B > 0 && (g.dtype == KVQ_BF16 || g.dtype == KVQ_F16);
}

cudaError_t launch_append_full(const Geom& g, const void* k_new, const void* v_new, int n_new, const void* probe,
                               const void* pv, cudaStream_t st) {
  const int F = n_new / kG + 1;  // most pages a sequence can fill completely in this call
  const int64_t T = (int64_t)g.H * g.B * F;
  const FullSmem sp = full_smem(g.P);
  int dev = 0, sms = 148, occ = 1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  auto kern = g.dtype == KVQ_BF16 ? append_full_kernel<KVQ_BF16> : append_full_kernel<KVQ_F16>;
  if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, sp.total)) != cudaSuccess) return e;
  if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, kFThreads, sp.total)) != cudaSuccess) return e;
  const int64_t ctas = std::max<int64_t>(1, std::min<int64_t>(T, (int64_t)std::max(occ, 1) * sms));
  const int64_t per = (T + ctas - 1) / ctas;
  // K / V input as (128 channels, KV heads, tokens of all sequences), boxes of 64 channels x 32 tokens
  CUtensorMap kmap, vmap;
  const CUtensorMapDataType dt = g.dtype == KVQ_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  const cuuint64_t dims[3] = {(cuuint64_t)kD, (cuuint64_t)g.H, (cuuint64_t)g.B * n_new};
  const cuuint64_t strides[2] = {(cuuint64_t)kD * 2, (cuuint64_t)g.H * kD * 2};
  const cuuint32_t box[3] = {64, 1, 32};
  if ((e = encode_tiled_map(&kmap, dt, 3, k_new, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B)) != cudaSuccess ||
      (e = encode_tiled_map(&vmap, dt, 3, v_new, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B)) != cudaSuccess)
    return e;
  kern<<<(unsigned)((T + per - 1) / per), kFThreads, sp.total, st>>>(kmap, vmap, g, (const int32_t*)probe,
                                                                     (const float*)pv, n_new, F, per);
  return cudaGetLastError();
}

}  // namespace kvq
