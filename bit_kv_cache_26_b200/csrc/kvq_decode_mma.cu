#include <algorithm>
#include <cmath>
// Split-K decode attention over the quantized paged cache on tensor cores
// ("PatternKV", Section 3.4: pattern-index restoration, dequantization and the
// QK^T / P.V products fused into the attention kernel).
//
// Design (per CTA: one (sequence, KV head, split); 4 warps, each streaming its own
// pages through a ring of shared-memory stages filled by cp.async.bulk):
//
//   K side, per 32-token page with per-channel scale s_d, zero z_d:
//     q.k_t = sum_d (q_d s_d) code_td + sum_d q_d z_d + T[idx_t],  T_j = q . M_K[j]
//   The codes are turned into exact bf16 integers and used as the A operand of
//   m16n8k16 MMAs (rows = tokens); B = q (.) s split into bf16 hi + lo parts by
//   truncation (columns = query head x {hi, lo}), so each product keeps 16 bits
//   (relative error below 2^-15) with no conversion instructions at all.
//
//   V side, per token with per-group scale s_tg and zero z_tg:
//     sum_t p_t v_t = sum_t (p_t s_tg) code_td + sum_t p_t z_tg + sum_j W_j M_V[j]
//   A = codes (rows = channels), B = p (.) s split into bf16 hi + lo parts (columns =
//   query head x {hi, lo}; a single 8- or 11-bit part loses too much once the
//   cancellation between residual and zero-point terms amplifies it),
//   W_j = sum of p over tokens with V pattern j (shared-memory atomics), the z term
//   in registers.
//
// The page layout (include/kvq.h) stores every lane's MMA operands contiguously.
// Online softmax runs in base 2 in the MMA accumulator layout; the newest
// incomplete group (exact keys in the K tail) is folded in on CUDA cores by the
// last split.  Each CTA folds its pattern term sum_j W_j M_V[j] into its partial o, so the
// partials are (m, l, o); the CTA that finishes a group's last split merges them.
#include <cstdlib>

#include "kvq_common.cuh"
#include "kvq_internal.h"

namespace kvq {

namespace {

constexpr uint32_t kSpinLimit = 1u << 22;

__device__ __forceinline__ uint32_t smem_u32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_u32(dst)),
               "l"(src), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}
// Bounded wait on an mbarrier phase: false if the phase did not complete within `limit` tries.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t phase, uint32_t limit = kSpinLimit) {
  const uint32_t addr = smem_u32(bar);
  for (uint32_t it = 0; it < limit; ++it) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(addr), "r"(phase)
        : "memory");
    if (ok) return true;
  }
  return false;
}

__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Packed fp32 pairs (sm_100a f32x2 instructions).
__device__ __forceinline__ unsigned long long pk(float a, float b) {
  unsigned long long r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ void upk(unsigned long long r, float& a, float& b) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(r));
}
__device__ __forceinline__ unsigned long long mul2(unsigned long long a, unsigned long long b) {
  unsigned long long r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ unsigned long long fma2(unsigned long long a, unsigned long long b, unsigned long long c) {
  unsigned long long r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}

// bf16 pair (lo half = first value) of the hi parts (fp32 truncated to bf16) or, on lanes with
// lo_sel = 1, of the truncated remainders v - hi.  hi + lo keeps 16 significant bits.
__device__ __forceinline__ uint32_t split_bf16(unsigned long long v, unsigned long long neg_sel) {
  float v0, v1;
  upk(v, v0, v1);
  const float t0 = __uint_as_float(__float_as_uint(v0) & 0xFFFF0000u);
  const float t1 = __uint_as_float(__float_as_uint(v1) & 0xFFFF0000u);
  float r0, r1;
  upk(fma2(neg_sel, pk(t0, t1), v), r0, r1);  // v - sel * trunc(v), exact
  return __byte_perm(__float_as_uint(r0), __float_as_uint(r1), 0x7632);
}

// Two codes at bit `S` of each 16-bit half of `src` -> bf16 pair of the exact integers:
// (src & mask) | 0x4300 puts 128 + code * 2^S in each half; one bf16 FMA removes the
// bias and the 2^S factor exactly.  Needs code * 2^S < 128.
template <int BITS, int S>
__device__ __forceinline__ uint32_t code_pair(uint32_t src) {
  static_assert((((1 << BITS) - 1) << S) < 128, "code does not fit the bf16 mantissa");
  constexpr uint32_t mask = ((1u << BITS) - 1u) * 0x00010001u << S;
  uint32_t v;
  asm("lop3.b32 %0, %1, %2, %3, 0xea;" : "=r"(v) : "r"(src), "r"(mask), "r"(0x43004300u));  // (a & b) | c
  constexpr uint32_t kScale = S == 0 ? 0x3F803F80u : (S == 2 ? 0x3E803E80u : 0x3D803D80u);
  constexpr uint32_t kBias = S == 0 ? 0xC300C300u : (S == 2 ? 0xC200C200u : 0xC100C100u);
  uint32_t r;
  asm("fma.rn.bf16x2 %0, %1, %2, %3;" : "=r"(r) : "r"(v), "r"(kScale), "r"(kBias));
  return r;
}

// A operand registers {a0a1, a2a3, a4a5, a6a7} for the 4 consecutive code slots starting at
// SLOT0 of lane word w (slot k holds bits [BITS*k, BITS*k + BITS) of each half).
template <int BITS, int SLOT0>
__device__ __forceinline__ void frag_a(uint32_t w, uint32_t (&a)[4]) {
  if constexpr (BITS == 2) {
    const uint32_t w6 = w >> 6, w12 = w >> 12;
    if constexpr (SLOT0 == 0) {
      a[0] = code_pair<2, 0>(w); a[1] = code_pair<2, 2>(w); a[2] = code_pair<2, 4>(w); a[3] = code_pair<2, 0>(w6);
    } else {
      a[0] = code_pair<2, 2>(w6); a[1] = code_pair<2, 4>(w6); a[2] = code_pair<2, 0>(w12); a[3] = code_pair<2, 2>(w12);
    }
  } else {
    a[0] = code_pair<4, 0>(w); a[1] = code_pair<4, 0>(w >> 4); a[2] = code_pair<4, 0>(w >> 8);
    a[3] = code_pair<4, 0>(w >> 12);
  }
}

template <int BITS>
struct Cfg {
  static constexpr int kWordsPerLane = BITS * 4;  // 32-bit code words per lane per K/V block
};

// Shared memory carve-up (bytes) for one CTA.
struct Smem {
  int ring, bars, qk, qraw, T, W, pex;
  int total;
};
constexpr int kPexLd = 36;  // padded row of the p exchange (floats): conflict-free 16-byte reads

__host__ __device__ inline Smem smem_plan(int sub_bytes, int stages, int NT, int P, int kWarps) {
  Smem s;
  int o = 0;
  // the ring; the merge at the end reuses this region, so it is at least as large as the merge
  const int merge = (kWarps * NT * 4 * kD + 2 * kWarps * NT * 4 + kWarps * NT * 4 * 4 + P * NT * 4 + NT * 4 * kWarps) * 4;
  const int ring = kWarps * stages * sub_bytes;
  s.ring = o; o += ring > merge ? ring : merge;
  o = (o + 15) & ~15;
  s.bars = o; o += kWarps * stages * 8;
  s.qk = o; o += NT * 4 * kD * 4;          // query in the quantized space, per padded head, KSC order
  s.qraw = o; o += NT * 4 * kD * 4;        // raw query (exact tail keys), natural order
  s.T = o; o += NT * 4 * P * 4;            // T[h][j] = q . M_K[j]
  s.W = o; o += kWarps * NT * 4 * (P + 1) * 4;  // per-warp pattern weights (+1: tokens stored raw)
  s.pex = o; o += kWarps * NT * 4 * kPexLd * 4;  // per-warp p exchange
  s.total = o;
  return s;
}

// Combine of one (sequence, KV head) group, run by the CTA that finished the group's last
// split: log-sum-exp merge of the splits' (m, l, o) (each o already holds its pattern term)
// and the inverse pre-transform.  Warp w takes query heads w, w + warps, ...; lane l holds
// channels l + 32 k.  Lane s computes the weight of split s (32 splits at a time) and the
// weights are broadcast, so the loads of consecutive splits are independent and overlap.
// The partials come from other CTAs, so they are read through L2 (after the fence that
// follows the arrival counter).  A non-finite output (an operand outside the fp32 / bf16
// range upstream) sets KVQ_DEV_RANGE.
__device__ void combine_group(const Geom& g, int Hq, int nsplit, int b, int h_kv, int Gq, int set,
                              const float* part_ml, const float* part_o, float* out) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  const float2* ml2 = reinterpret_cast<const float2*>(part_ml);
  for (int hh = warp; hh < Gq; hh += nwarps) {
    const int row = b * Hq + h_kv * Gq + hh;
    const size_t base = (size_t)row * nsplit;
    float* outp = out + (size_t)row * kD;
    float M = -INFINITY;
    for (int s = lane; s < nsplit; s += 32) M = fmaxf(M, __ldcg(part_ml + 2 * (base + s)));
    M = warp_max(M);
    if (M == -INFINITY) {  // no tokens
#pragma unroll
      for (int k = 0; k < 4; ++k) outp[lane + 32 * k] = 0.f;
      continue;
    }
    float Lsum = 0.f, o[4] = {0.f, 0.f, 0.f, 0.f};
    for (int s0 = 0; s0 < nsplit; s0 += 32) {
      float fs = 0.f;
      if (s0 + lane < nsplit) {
        const float2 ml = __ldcg(ml2 + base + s0 + lane);
        fs = ml.x == -INFINITY ? 0.f : exp2f(ml.x - M);
        Lsum = fmaf(fs, ml.y, Lsum);
      }
      const int n = min(32, nsplit - s0);
      const float* po = part_o + (base + s0) * kD + lane;
#pragma unroll 4
      for (int i = 0; i < n; ++i) {
        const float f = __shfl_sync(kFull, fs, i);
#pragma unroll
        for (int k = 0; k < 4; ++k) o[k] = fmaf(f, __ldcg(po + (size_t)i * kD + 32 * k), o[k]);
      }
    }
    Lsum = warp_sum(Lsum);
    const float inv = 1.0f / Lsum;
#pragma unroll
    for (int k = 0; k < 4; ++k) o[k] *= inv;
    if (g.tx) {
      const float* cV = g.vcol + ((size_t)set * g.H + h_kv) * kD;
#pragma unroll
      for (int k = 0; k < 4; ++k) o[k] *= cV[lane + 32 * k];
      fwht_warp(o, lane);
#pragma unroll
      for (int k = 0; k < 4; ++k) o[k] *= 0.0078125f;
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      if (!isfinite(o[k])) set_status(g.status, KVQ_DEV_RANGE);
      outp[lane + 32 * k] = o[k];
    }
  }
}

// ---- one-token append of a decode step (the last split's CTA, before its page copies) ----------
//
// The same definitions as the bulk append ("PatternKV", Section 3.2, Eq. 6 and Eq. 1; Section
// 3.3 for V; Section 3.1, Eq. 5 for the window), for one new token of sequence b and KV head h at
// position L: the exact min-max argmin over the Pe patterns in use (two threads per pattern, a
// channel half each, lowest index on ties), the V codes merged into the page's words (atomicOr:
// two channels of a token share a word), the raw key into the K tail; when the token completes
// its page, the page's 32 keys are assigned (four threads per key) and quantized per channel.
// With decode-time insertion, the window's running min / max take the token and, when L + 1 is a
// multiple of the window length, the Chebyshev centers become pattern Pe of the sequence's set.
// Scratch: the first bytes of the CTA's page ring (unused until the page copies start).
constexpr int kYLd = kD + 4;

__device__ __forceinline__ unsigned long long min_key(unsigned long long a, unsigned long long b2) {
  return a < b2 ? a : b2;
}
__device__ __forceinline__ unsigned long long dkey_s(float d, int j) {
  return ((unsigned long long)__float_as_uint(d) << 32) | (uint32_t)j;
}

// nearest pattern of the vector y (shared, 128 channels) among M[0..Pe): exact fp32 d_mm, key
// (d bits << 32 | j) of the minimum; all 128 threads of the CTA take part, every thread gets it
__device__ unsigned long long nearest_dmm_cta(const float* y, const float* __restrict__ M, int Pe,
                                              unsigned long long* red) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, half = tid & 1;
  unsigned long long best = ~0ull;
  for (int j0 = 0; j0 < Pe; j0 += 64) {
    const int j = j0 + (tid >> 1);
    float mx = -INFINITY, mn = INFINITY;
    if (j < Pe) {
      const float4* m4 = reinterpret_cast<const float4*>(M + (size_t)j * kD + 64 * half);
      const float4* y4 = reinterpret_cast<const float4*>(y + 64 * half);
#pragma unroll 4
      for (int c = 0; c < 16; ++c) {
        const float4 m = __ldg(m4 + c), a = y4[c];
        float r0, r1, r2, r3;
        sub2(a.x, a.y, m.x, m.y, r0, r1);
        sub2(a.z, a.w, m.z, m.w, r2, r3);
        mx = max3(mx, r0, r1);
        mn = min3(mn, r0, r1);
        mx = max3(mx, r2, r3);
        mn = min3(mn, r2, r3);
      }
    }
    mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 1));
    mn = fminf(mn, __shfl_xor_sync(kFull, mn, 1));
    if (j < Pe) best = min_key(best, dkey_s(__fsub_rn(mx, mn), j));
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) best = min_key(best, __shfl_xor_sync(kFull, best, o));
  if (lane == 0) red[warp] = best;
  __syncthreads();
  best = min_key(min_key(red[0], red[1]), min_key(red[2], red[3]));
  __syncthreads();
  return best;
}

template <int BITS>
__device__ void step_append(const Geom& g, int b, int h, int L, int set, int Pe, const uint16_t* __restrict__ k_new,
                            const uint16_t* __restrict__ v_new, uint8_t* scratch) {
  constexpr int maxc = (1 << BITS) - 1;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int slot = L % kG, pg = L / kG;
  const size_t sh = (size_t)set * g.H + h;
  const float* MK = g.kpat + sh * g.P * kD;
  const float* MV = g.vpat + sh * g.P * kD;
  uint8_t* sub = g.pool + (size_t)g.page_table[(size_t)b * g.maxp + pg] * g.page_bytes + (size_t)h * g.sub_bytes;
  float* yv = reinterpret_cast<float*>(scratch);             // [128]
  float* yk = yv + kD;                                       // [32][kYLd] keys of the page (sealing) or [1]
  float* rowf = yk + kG * kYLd;                              // [33] row factors: keys 0..31, then V
  unsigned long long* red = reinterpret_cast<unsigned long long*>(rowf + 40);  // [4]
  float* vstat = reinterpret_cast<float*>(red + 4);          // [2] range of y_v
  int* kbest = reinterpret_cast<int*>(vstat + 4);            // [32]
  float* kz = reinterpret_cast<float*>(kbest + kG);          // [128] K zero, then [128] K scale
  const uint16_t* kin = k_new + ((size_t)b * g.H + h) * kD;
  const uint16_t* vin = v_new + ((size_t)b * g.H + h) * kD;
  const bool seal = slot == kG - 1;

  // ---- the new vectors (and, when the page seals, its other 31 keys from the K tail), pre-transformed
  uint16_t* tail = g.k_tail + ((size_t)b * g.H + h) * kG * kD;
  for (int r = warp; r < 2 + (seal ? kG - 1 : 0); r += 4) {
    // r = 0: V; r = 1: the new key (page slot `slot`); r >= 2: key of slot r - 2 from the tail
    const uint16_t* src = r == 0 ? vin : r == 1 ? kin : tail + (size_t)(r - 2) * kD;
    float y[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) y[k] = bits_to_float(src[lane + 32 * k], g.dtype);  // plain loads: the tail is written here
    float rr = 1.0f;
    if (g.tx) transform_row_warp(y, r == 0 ? g.vcol + sh * kD : g.kcol + sh * kD, rr, lane);
    float* dst = r == 0 ? yv : yk + (size_t)(r == 1 ? (seal ? slot : 0) : r - 2) * kYLd;
#pragma unroll
    for (int k = 0; k < 4; ++k) dst[lane + 32 * k] = y[k];
    if (lane == 0) rowf[r == 0 ? kG : (r == 1 ? (seal ? slot : 0) : r - 2)] = rr;
    if (r == 0) {
      float mx = -INFINITY, mn = INFINITY;
#pragma unroll
      for (int k = 0; k < 4; ++k) { mx = fmaxf(mx, y[k]); mn = fminf(mn, y[k]); }
      mx = warp_max(mx);
      mn = warp_min(mn);
      if (lane == 0) vstat[0] = __fsub_rn(mx, mn);
    }
  }
  // the raw key joins the K tail
  if (tid < kD) tail[(size_t)slot * kD + tid] = kin[tid];
  if (slot == 0) {
    // a fresh page: the V part of the page starts from zeros (tokens not yet appended are zero)
    uint32_t* w = reinterpret_cast<uint32_t*>(sub + g.off_vc);
    for (int i = tid; i < g.cb / 4; i += blockDim.x) w[i] = 0u;
    float* vs = reinterpret_cast<float*>(sub + g.off_vs);
    for (int i = tid; i < 2 * 128; i += blockDim.x) vs[i] = 0.f;  // V scales then V zeros (512 B each)
    if (tid < kG / 4) reinterpret_cast<uint32_t*>(sub + g.off_vidx)[tid] = 0u;
    if (g.tx && tid < kG) reinterpret_cast<float*>(sub + g.off_vrow)[tid] = 0.f;
  }
  __syncthreads();

  // ---- decode-time insertion: the window's running min / max take the new vectors; at the
  // window's end the centers are written as pattern Pe (its count is raised at the very end,
  // after this token's own assignments, which use the Pe patterns present)
  const bool emit = g.gwin > 0 && g.window && (L + 1) % g.gwin == 0 && Pe < g.P;
  if (g.gwin > 0 && g.window) {
    float* wnd = g.window + ((size_t)b * g.H + h) * 4 * kD;
    const int c = tid;
    const float kk = yk[(size_t)(seal ? slot : 0) * kYLd + c], v = yv[c];
    const float kmn = fminf(wnd[c], kk), kmx = fmaxf(wnd[kD + c], kk);
    const float vmn = fminf(wnd[2 * kD + c], v), vmx = fmaxf(wnd[3 * kD + c], v);
    if ((L + 1) % g.gwin == 0) {
      if (emit) {
        // (the pattern buffers are the caller's; with insertion on, steps write their rows Pe .. P - 1)
        const_cast<float*>(g.kpat)[(sh * g.P + Pe) * kD + c] = __fmul_rn(__fadd_rn(kmn, kmx), 0.5f);
        const_cast<float*>(g.vpat)[(sh * g.P + Pe) * kD + c] = __fmul_rn(__fadd_rn(vmn, vmx), 0.5f);
      }
      wnd[c] = INFINITY;
      wnd[kD + c] = -INFINITY;
      wnd[2 * kD + c] = INFINITY;
      wnd[3 * kD + c] = -INFINITY;
    } else {
      wnd[c] = kmn;
      wnd[kD + c] = kmx;
      wnd[2 * kD + c] = vmn;
      wnd[3 * kD + c] = vmx;
    }
  }

  // ---- V: nearest pattern, adaptive threshold, residual, 4 groups of 32 channels (warp = group)
  {
    const unsigned long long kv = nearest_dmm_cta(yv, MV, Pe, red);
    const int j = (int)(kv & 0xffffffffu);
    const bool keep = v_keep_pattern(g.vrho, __uint_as_float((uint32_t)(kv >> 32)), vstat[0]);
    const int c = 32 * warp + lane;
    const float R = keep ? __fsub_rn(yv[c], __ldg(MV + (size_t)j * kD + c)) : yv[c];
    float s, z;
    int code = quant_warp(R, BITS, s, z);
    int wd, bt;
    frag_pos(BITS, 2, c, slot, wd, bt);
    atomicOr(reinterpret_cast<unsigned int*>(sub + g.off_vc) + wd, (unsigned)code << bt);
    if (lane == 0) {
      reinterpret_cast<float*>(sub + g.off_vs)[vsc_pos(slot, warp)] = s;
      reinterpret_cast<float*>(sub + g.off_vz)[vzc_pos(slot, warp)] = z;
    }
    if (tid == 0) {
      sub[g.off_vidx + tok_pos(slot)] = keep ? (uint8_t)j : (uint8_t)kRawIndex;
      if (g.tx) reinterpret_cast<float*>(sub + g.off_vrow)[tok_pos(slot)] = rowf[kG];
    }
  }

  // ---- K: the page seals: its 32 keys, nearest patterns (4 threads per key), per-channel groups
  if (seal) {
    {
      const int r = tid >> 2, q = tid & 3;  // key r, channels 32 q .. 32 q + 31
      const float* y = yk + (size_t)r * kYLd + 32 * q;
      unsigned long long best = ~0ull;
      for (int j = 0; j < Pe; ++j) {
        const float4* m4 = reinterpret_cast<const float4*>(MK + (size_t)j * kD + 32 * q);
        const float4* y4 = reinterpret_cast<const float4*>(y);
        float mx = -INFINITY, mn = INFINITY;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const float4 m = __ldg(m4 + c), a = y4[c];
          float r0, r1, r2, r3;
          sub2(a.x, a.y, m.x, m.y, r0, r1);
          sub2(a.z, a.w, m.z, m.w, r2, r3);
          mx = max3(mx, r0, r1);
          mn = min3(mn, r0, r1);
          mx = max3(mx, r2, r3);
          mn = min3(mn, r2, r3);
        }
        mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 1));
        mn = fminf(mn, __shfl_xor_sync(kFull, mn, 1));
        mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 2));
        mn = fminf(mn, __shfl_xor_sync(kFull, mn, 2));
        best = min_key(best, dkey_s(__fsub_rn(mx, mn), j));
      }
      if (q == 0) kbest[r] = (int)(best & 0xffffffffu);
    }
    __syncthreads();
    // residuals in place, then scale / zero per channel (thread = channel)
    for (int i = tid; i < kG * kD; i += blockDim.x) {
      const int r = i / kD, c = i % kD;
      yk[(size_t)r * kYLd + c] = __fsub_rn(yk[(size_t)r * kYLd + c], __ldg(MK + (size_t)kbest[r] * kD + c));
    }
    __syncthreads();
    {
      const int c = tid;
      float mx = -INFINITY, mn = INFINITY;
      for (int r = 0; r < kG; ++r) { mx = fmaxf(mx, yk[(size_t)r * kYLd + c]); mn = fminf(mn, yk[(size_t)r * kYLd + c]); }
      const float s = __fdiv_rn(__fsub_rn(mx, mn), (float)maxc);
      kz[c] = mn;
      kz[kD + c] = s;
      reinterpret_cast<float*>(sub + g.off_ks)[ksc_pos(c)] = s;
      reinterpret_cast<float*>(sub + g.off_kz)[ksc_pos(c)] = mn;
    }
    __syncthreads();
    // every 32-bit word of the K block, codes by the definition
    for (int wd = tid; wd < g.cb / 4; wd += blockDim.x) {
      uint32_t word = 0u;
      constexpr int SPW = 16 / BITS;
      for (int sl = 0; sl < SPW; ++sl)
        for (int odd = 0; odd < 2; ++odd) {
          int r, c;
          frag_elem(BITS, 8, wd, sl, odd, r, c);
          const float R = yk[(size_t)r * kYLd + c], sc = kz[kD + c];
          uint32_t code = 0u;
          if (sc != 0.0f) code = (uint32_t)min(max(__float2int_rn(__fdiv_rn(__fsub_rn(R, kz[c]), sc)), 0), maxc);
          word |= code << (BITS * sl + 16 * odd);
        }
      reinterpret_cast<uint32_t*>(sub)[wd] = word;
    }
    if (tid < kG) {
      sub[g.off_kidx + tok_pos(tid)] = (uint8_t)kbest[tid];
      if (g.tx) reinterpret_cast<float*>(sub + g.off_krow)[tok_pos(tid)] = rowf[tid];
    }
  }

  // the new pattern rows before the raised count (readers of the count then see the rows)
  if (emit) {
    __threadfence();
    __syncthreads();
    if (tid == 0) g.counts[sh] = Pe + 1;
  }
  // the page writes above before the tensor / bulk copies of this CTA read the sealed page
  __threadfence();
  asm volatile("fence.proxy.async.global;" ::: "memory");
  __syncthreads();
}

// STEP: a decode step -- the last split's CTA of each (sequence, KV head) first appends the
// sequence's new token (step_append), then decodes over every token including it; the other
// splits decode the pages complete before the step.  The CTA that starts last among a
// sequence's CTAs advances its seq_len (all of them have read the old length by then).
template <int BITS, int NT, int STAGES, int kWarps, bool STEP>
__global__ void __launch_bounds__(kWarps * 32, (kWarps == 4 ? (STAGES <= 2 && NT == 1 ? 4 : 3) : 2))
    decode_mma_kernel(Geom g, const uint16_t* __restrict__ q, int Hq, float scale_log2, int nsplit,
                      float* __restrict__ part_ml, float* __restrict__ part_o, int* __restrict__ arrivals,
                      float* __restrict__ out, const uint16_t* __restrict__ k_new, const uint16_t* __restrict__ v_new,
                      int* __restrict__ seqcnt) {
  constexpr int NH = NT * 4;  // padded heads
  constexpr int WPL = Cfg<BITS>::kWordsPerLane;
  extern __shared__ __align__(16) uint8_t smem[];
  const int split = blockIdx.x, h_kv = blockIdx.y, b = blockIdx.z;
  const int Gq = Hq / g.H;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int gq = lane >> 2, tig = lane & 3;
  const float lo_sel = (gq & 1) ? 1.0f : 0.0f;
  const unsigned long long nsel = pk(-lo_sel, -lo_sel);
  const int P = g.P;
  const uint32_t sub_bytes = (uint32_t)g.sub_bytes;
  const Smem sp = smem_plan((int)sub_bytes, STAGES, NT, P, kWarps);

  uint8_t* ring = smem + sp.ring + warp * STAGES * sub_bytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + sp.bars) + warp * STAGES;
  float* qk = reinterpret_cast<float*>(smem + sp.qk);     // [NH][128] KSC order
  float* qraw = reinterpret_cast<float*>(smem + sp.qraw); // [NH][128]
  float* T = reinterpret_cast<float*>(smem + sp.T);       // [NH][P]
  float* Wall = reinterpret_cast<float*>(smem + sp.W);
  const int P1 = P + 1;                                   // W slot P: V tokens stored raw (index 255)
  float* Ww = Wall + warp * NH * P1;                      // this warp's [NH][P + 1]
  float* pex = reinterpret_cast<float*>(smem + sp.pex) + warp * NH * kPexLd;

  int L = g.seq_len[b];
  bool seq_ok = true;  // a sequence with a bad length or set is decoded as empty and left unchanged
  if (L < 0 || L > g.maxp * kG) {
    if (threadIdx.x == 0 && split == 0) set_status(g.status, KVQ_DEV_OVERFLOW);
    L = 0;
    seq_ok = false;
  }
  int set = g.seq_to_set ? g.seq_to_set[b] : 0;
  if (set < 0 || set >= g.S) {
    if (threadIdx.x == 0 && split == 0) set_status(g.status, KVQ_DEV_BAD_SET);
    set = 0;
    L = 0;
    seq_ok = false;
  }
  // a decode step appends one token: it needs room in the page table and a valid page
  bool app = false;
  if constexpr (STEP) {
    if (!seq_ok) {
    } else if (L + 1 > g.maxp * kG) {
      if (threadIdx.x == 0 && split == 0 && h_kv == 0) set_status(g.status, KVQ_DEV_OVERFLOW);
    } else {
      const int phys = g.page_table[(size_t)b * g.maxp + L / kG];
      app = phys >= 0 && phys < g.npages;
      if (!app && threadIdx.x == 0 && split == 0 && h_kv == 0) set_status(g.status, KVQ_DEV_BAD_PAGE);
    }
    if (threadIdx.x == 0) {
      // every CTA of sequence b has read its old length once the counter reaches H * nsplit
      if (atomicAdd(seqcnt + b, 1) == g.H * nsplit - 1) {
        seqcnt[b] = 0;
        if (app) g.seq_len[b] = L + 1;
      }
    }
  }
  const int nfull = L / kG;
  const int per = (nfull + nsplit - 1) / nsplit;
  const int p0 = min(nfull, split * per);
  // the last split also takes the page the step's token completes (and the tail after it)
  const int p1 = (STEP && app && split == nsplit - 1) ? (L + 1) / kG : min(nfull, p0 + per);
  const int ntail = (STEP && app) ? (L + 1) % kG : L % kG;
  const size_t sh = (size_t)set * g.H + h_kv;
  const float* MK = g.kpat + sh * P * kD;
  const int Pe = p_eff(g, (int)sh);  // patterns in use by this set (rows beyond are capacity)
  if constexpr (STEP) {
    if (app && split == nsplit - 1) step_append<BITS>(g, b, h_kv, L, set, Pe, k_new, v_new, ring - warp * STAGES * sub_bytes);
  }
  const float* cK = g.tx ? g.kcol + sh * kD : nullptr;

  // ---- the first STAGES page copies of each warp go out before the setup below
  // pages of this warp: p0 + warp + kWarps*i.  Their physical ids are read 32 at a time (lane l
  // holds page 32w + l of window w), one window ahead, so no page-table load sits between a
  // page and the copy of the page STAGES ahead.
  const int my_n = (p1 - p0 - warp + kWarps - 1) / kWarps;
  auto load_ids = [&](int base) -> int {
    const int i = base + lane;
    return i < my_n ? g.page_table[(size_t)b * g.maxp + p0 + warp + kWarps * i] : -1;
  };
  int ids = load_ids(0), ids_next = load_ids(32);
  auto page_src = [&](int phys, bool& ok) -> const uint8_t* {
    ok = phys >= 0 && phys < g.npages;
    return g.pool + (size_t)(ok ? phys : 0) * g.page_bytes + (size_t)h_kv * g.sub_bytes;
  };
  uint32_t bad_mask = 0;  // lane 0: stages whose page id was invalid
  if (lane < STAGES) mbar_init(&bars[lane], 1);
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  __syncwarp();
  int first_ids[STAGES];
#pragma unroll
  for (int i = 0; i < STAGES; ++i) first_ids[i] = __shfl_sync(kFull, ids, i);
  if (lane == 0) {
    for (int i = 0; i < min(STAGES, my_n); ++i) {
      bool ok;
      const uint8_t* src = page_src(first_ids[i], ok);
      if (ok) {
        mbar_expect_tx(&bars[i], sub_bytes);
        bulk_g2s(ring + i * sub_bytes, src, sub_bytes, &bars[i]);
      } else {
        set_status(g.status, KVQ_DEV_BAD_PAGE);
        bad_mask |= 1u << i;
        mbar_arrive(&bars[i]);
      }
    }
  }
  __syncwarp();

  // ---- setup (overlapping the first copies): queries, T table, zeroed W
  for (int hh = warp; hh < NH; hh += kWarps) {
    float v[4];
    const bool real = hh < Gq;
    const uint16_t* src = q + ((size_t)b * Hq + h_kv * Gq + min(hh, Gq - 1)) * kD;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      v[k] = real ? load_elem(src + lane + 32 * k, g.dtype) : 0.f;
      qraw[hh * kD + lane + 32 * k] = v[k];
    }
    if (g.tx) {
      fwht_warp(v, lane);
#pragma unroll
      for (int k = 0; k < 4; ++k) v[k] = v[k] * __ldg(cK + lane + 32 * k) * 0.0078125f;
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) qk[hh * kD + ksc_pos(lane + 32 * k)] = v[k];
  }
  for (int i = threadIdx.x; i < kWarps * NH * P1; i += blockDim.x) Wall[i] = 0.f;
  // the transformed query comes from shared memory (after this barrier); the plain one straight
  // from global memory, so that its loads and the pattern rows' below share one round trip
  if (g.tx) __syncthreads();
  // T[hh][j] = q_hh . M_K[j] (transformed space): warp w takes patterns w, w + warps, ...;
  // lane l holds channels 4l .. 4l + 3 of four query heads and reads the pattern row with one
  // coalesced 16-byte load; the four head sums are reduced across the warp
#pragma unroll 1
  for (int hg = 0; hg < NT; ++hg) {
    float qv[4][4];
#pragma unroll
    for (int a = 0; a < 4; ++a) {
      const int hh = 4 * hg + a;
      if (g.tx) {
#pragma unroll
        for (int e = 0; e < 4; ++e) qv[a][e] = qk[hh * kD + ksc_pos(4 * lane + e)];
      } else {
        const uint16_t* src = q + ((size_t)b * Hq + h_kv * Gq + min(hh, Gq - 1)) * kD + 4 * lane;
#pragma unroll
        for (int e = 0; e < 4; ++e) qv[a][e] = hh < Gq ? load_elem(src + e, g.dtype) : 0.f;
      }
    }
    // sixteen pattern rows' loads in flight at a time
    for (int j0 = warp; j0 < Pe; j0 += 16 * kWarps) {
      float4 m4[16];
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        const int j = j0 + u * kWarps;
        m4[u] = j < Pe ? __ldg(reinterpret_cast<const float4*>(MK + (size_t)j * kD) + lane) : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        const int j = j0 + u * kWarps;
        float t[4];
#pragma unroll
        for (int a = 0; a < 4; ++a)
          t[a] = fmaf(qv[a][3], m4[u].w, fmaf(qv[a][2], m4[u].z, fmaf(qv[a][1], m4[u].y, qv[a][0] * m4[u].x)));
#pragma unroll
        for (int off = 16; off > 0; off >>= 1)
#pragma unroll
          for (int a = 0; a < 4; ++a) t[a] += __shfl_xor_sync(kFull, t[a], off);
        if (lane < 4 && j < Pe) T[(4 * hg + lane) * P + j] = lane == 0 ? t[0] : lane == 1 ? t[1] : lane == 2 ? t[2] : t[3];
      }
    }
  }
  __syncthreads();


  // ---- per-thread state (head of n-tile j: 4j + tig)
  float accv[NT][8][4];
  float zacc[NT][4];
  float mrun[NT], lrun[NT];
#pragma unroll
  for (int j = 0; j < NT; ++j) {
    mrun[j] = -INFINITY;
    lrun[j] = 0.f;
#pragma unroll
    for (int u = 0; u < 4; ++u) zacc[j][u] = 0.f;
#pragma unroll
    for (int mt = 0; mt < 8; ++mt)
#pragma unroll
      for (int u = 0; u < 4; ++u) accv[j][mt][u] = 0.f;
  }

  int stuck_at = -1;
  for (int i = 0; i < my_n; ++i) {
    const int st = i % STAGES;
    const uint32_t phase = (i / STAGES) & 1;
    const bool ok = mbar_wait(&bars[st], phase, g.wait_limit);
    if (!__all_sync(kFull, ok)) { stuck_at = i; break; }
    const bool skip = __shfl_sync(kFull, (bad_mask >> st) & 1, 0);
    const uint8_t* pgp = ring + st * sub_bytes;
    if (!skip) {
      // ---------------- K side: scores of 32 tokens for the query heads
      uint32_t kw[WPL];
#pragma unroll
      for (int c = 0; c < WPL / 4; ++c) {
        const uint4 t = reinterpret_cast<const uint4*>(pgp + c * 512)[lane];
        kw[4 * c] = t.x; kw[4 * c + 1] = t.y; kw[4 * c + 2] = t.z; kw[4 * c + 3] = t.w;
      }
      const float4* ks4 = reinterpret_cast<const float4*>(pgp + g.off_ks) + tig;
      const float4* kz4 = reinterpret_cast<const float4*>(pgp + g.off_kz) + tig;
      float sc[NT][4];
#pragma unroll
      for (int j = 0; j < NT; ++j) {
        float accs[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
        unsigned long long zk2 = 0ull;
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          const float4 s4 = ks4[ks * 4];
          const float4 z4 = kz4[ks * 4];
          // query of this lane's B column (head 4j + gq/2), channels of k-step ks, from shared memory
          const float4 q4 = reinterpret_cast<const float4*>(qk + (4 * j + (gq >> 1)) * kD)[ks * 4 + tig];
          const unsigned long long qa = pk(q4.x, q4.y), qb = pk(q4.z, q4.w);
          zk2 = fma2(qa, pk(z4.x, z4.y), zk2);
          zk2 = fma2(qb, pk(z4.z, z4.w), zk2);
          const uint32_t b0 = split_bf16(mul2(qa, pk(s4.x, s4.y)), nsel);
          const uint32_t b1 = split_bf16(mul2(qb, pk(s4.z, s4.w)), nsel);
#pragma unroll
          for (int mt = 0; mt < 2; ++mt) {
            uint32_t a[4];
            if constexpr (BITS == 2) {
              const uint32_t w = kw[mt * 4 + ks / 2];
              if (ks & 1) frag_a<2, 4>(w, a); else frag_a<2, 0>(w, a);
            } else {
              frag_a<4, 0>(kw[mt * 8 + ks], a);
            }
            mma16816(accs[mt], a, b0, b1);
          }
        }
        // K zero term of head 4j + gq/2: reduce over the 4 tig lanes, then fetch for head 4j + tig
        float za, zb;
        upk(zk2, za, zb);
        float zk = za + zb;
        zk += __shfl_xor_sync(kFull, zk, 1);
        zk += __shfl_xor_sync(kFull, zk, 2);
        zk = __shfl_sync(kFull, zk, 8 * tig);
        sc[j][0] = accs[0][0] + accs[0][1] + zk;
        sc[j][1] = accs[0][2] + accs[0][3] + zk;
        sc[j][2] = accs[1][0] + accs[1][1] + zk;
        sc[j][3] = accs[1][2] + accs[1][3] + zk;
      }
      const uint32_t kidx4 = *reinterpret_cast<const uint32_t*>(pgp + g.off_kidx + gq * 4);
      const uint32_t vidx4 = *reinterpret_cast<const uint32_t*>(pgp + g.off_vidx + gq * 4);
      float krow[4] = {1.f, 1.f, 1.f, 1.f}, vrow[4] = {1.f, 1.f, 1.f, 1.f};
      if (g.tx) {
        const float4 kr = *reinterpret_cast<const float4*>(pgp + g.off_krow + gq * 16);
        const float4 vr = *reinterpret_cast<const float4*>(pgp + g.off_vrow + gq * 16);
        krow[0] = kr.x; krow[1] = kr.y; krow[2] = kr.z; krow[3] = kr.w;
        vrow[0] = vr.x; vrow[1] = vr.y; vrow[2] = vr.z; vrow[3] = vr.w;
      }
      const float4* vz4 = reinterpret_cast<const float4*>(pgp + g.off_vz) + gq;
      const float4 vz[4] = {vz4[0], vz4[8], vz4[16], vz4[24]};

      // ---------------- online softmax (base 2), per head 4j + tig over the 32 tokens
#pragma unroll
      for (int j = 0; j < NT; ++j) {
        const int hh = 4 * j + tig;
        const bool real = hh < Gq;
        float pm = -INFINITY;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int idx = min((int)((kidx4 >> (8 * u)) & 0xff), Pe - 1);
          sc[j][u] = (sc[j][u] + T[hh * P + idx]) * krow[u] * scale_log2;
          pm = fmaxf(pm, sc[j][u]);
        }
        pm = fmaxf(pm, __shfl_xor_sync(kFull, pm, 4));
        pm = fmaxf(pm, __shfl_xor_sync(kFull, pm, 8));
        pm = fmaxf(pm, __shfl_xor_sync(kFull, pm, 16));
        const float mnew = fmaxf(mrun[j], pm);
        const float alpha = ex2(mrun[j] - mnew);
        if (__any_sync(kFull, alpha != 1.0f)) {
          lrun[j] *= alpha;
#pragma unroll
          for (int u = 0; u < 4; ++u) zacc[j][u] *= alpha;
#pragma unroll
          for (int mt = 0; mt < 8; ++mt)
#pragma unroll
            for (int u = 0; u < 4; ++u) accv[j][mt][u] *= alpha;
          for (int jj = gq; jj < Pe; jj += 8) Ww[hh * P1 + jj] *= alpha;
          __syncwarp();
        }
        mrun[j] = mnew;
        float pv[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const float p = real ? ex2(sc[j][u] - mnew) : 0.f;
          lrun[j] += p;
          pv[u] = p * vrow[u];
          if (real) atomicAdd(&Ww[hh * P1 + min((int)((vidx4 >> (8 * u)) & 0xff), P)], pv[u]);
          zacc[j][0] = fmaf(pv[u], vz[u].x, zacc[j][0]);
          zacc[j][1] = fmaf(pv[u], vz[u].y, zacc[j][1]);
          zacc[j][2] = fmaf(pv[u], vz[u].z, zacc[j][2]);
          zacc[j][3] = fmaf(pv[u], vz[u].w, zacc[j][3]);
        }
        *reinterpret_cast<float4*>(pex + hh * kPexLd + gq * 4) = make_float4(pv[0], pv[1], pv[2], pv[3]);
      }
      __syncwarp();

      // ---------------- V side: p-weighted residual codes for the query heads
      uint32_t vw[WPL];
#pragma unroll
      for (int c = 0; c < WPL / 4; ++c) {
        const uint4 t = reinterpret_cast<const uint4*>(pgp + g.off_vc + c * 512)[lane];
        vw[4 * c] = t.x; vw[4 * c + 1] = t.y; vw[4 * c + 2] = t.z; vw[4 * c + 3] = t.w;
      }
      const float4* vs4 = reinterpret_cast<const float4*>(pgp + g.off_vs) + tig;
#pragma unroll
      for (int j = 0; j < NT; ++j) {
        const float* prow = pex + (4 * j + (gq >> 1)) * kPexLd;
        const float4 pa = *reinterpret_cast<const float4*>(prow + (2 * tig) * 4);
        const float4 pb = *reinterpret_cast<const float4*>(prow + (2 * tig + 1) * 4);
#pragma unroll
        for (int ks = 0; ks < 2; ++ks) {
          const unsigned long long p01 = ks ? pk(pa.z, pb.z) : pk(pa.x, pb.x);  // tokens e=0, e=1
          const unsigned long long p23 = ks ? pk(pa.w, pb.w) : pk(pa.y, pb.y);  // tokens e=2, e=3
          // V scales of tokens (ks, e = 0..3), the 4 channel groups each
          const float4 s0 = vs4[(ks * 4 + 0) * 4], s1 = vs4[(ks * 4 + 1) * 4], s2 = vs4[(ks * 4 + 2) * 4],
                       s3 = vs4[(ks * 4 + 3) * 4];
#pragma unroll
          for (int grp = 0; grp < 4; ++grp) {
            const uint32_t b0 = split_bf16(mul2(p01, pk((&s0.x)[grp], (&s1.x)[grp])), nsel);
            const uint32_t b1 = split_bf16(mul2(p23, pk((&s2.x)[grp], (&s3.x)[grp])), nsel);
#pragma unroll
            for (int mh = 0; mh < 2; ++mh) {
              const int mt = grp * 2 + mh;
              uint32_t a[4];
              if constexpr (BITS == 2) {
                if (ks) frag_a<2, 4>(vw[mt], a); else frag_a<2, 0>(vw[mt], a);
              } else {
                frag_a<4, 0>(vw[mt * 2 + ks], a);
              }
              mma16816(accv[j][mt], a, b0, b1);
            }
          }
        }
      }
    }
    __syncwarp();
    // refill this stage with the page STAGES ahead
    const int nxt = i + STAGES;
    if ((nxt & 31) == 0 && nxt > 0) {  // next window of page ids
      ids = ids_next;
      ids_next = load_ids(nxt + 32);
    }
    const int nxt_phys = __shfl_sync(kFull, ids, nxt & 31);
    if (lane == 0 && nxt < my_n) {
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      bool okp;
      const uint8_t* src = page_src(nxt_phys, okp);
      bad_mask &= ~(1u << st);
      if (okp) {
        mbar_expect_tx(&bars[st], sub_bytes);
        bulk_g2s(ring + st * sub_bytes, src, sub_bytes, &bars[st]);
      } else {
        set_status(g.status, KVQ_DEV_BAD_PAGE);
        bad_mask |= 1u << st;
        mbar_arrive(&bars[st]);
      }
    }
    __syncwarp();
  }
  if (stuck_at >= 0) {
    if (lane == 0) set_status(g.status, KVQ_DEV_TIMEOUT);
    // give the copies already issued (pages stuck_at .. stuck_at + STAGES - 1) a bounded
    // chance to land before the CTA's shared memory is reused or released
    for (int i = stuck_at; i < my_n && i < stuck_at + STAGES; ++i)
      (void)mbar_wait(&bars[i % STAGES], (i / STAGES) & 1);
  }

  // ---- newest incomplete group: exact keys from the K tail, values from the partial page
  if (split == nsplit - 1 && warp == 0 && ntail > 0) {
    const int phys = g.page_table[(size_t)b * g.maxp + nfull];
    if (phys >= 0 && phys < g.npages) {
      const uint8_t* sub = g.pool + (size_t)phys * g.page_bytes + (size_t)h_kv * g.sub_bytes;
      const uint32_t* vwords = reinterpret_cast<const uint32_t*>(sub + g.off_vc);
      const float* vs = reinterpret_cast<const float*>(sub + g.off_vs);
      const float* vz = reinterpret_cast<const float*>(sub + g.off_vz);
      const float* vr = reinterpret_cast<const float*>(sub + g.off_vrow);
      for (int t = 0; t < ntail; ++t) {
        const uint16_t* kt = g.k_tail + (((size_t)b * g.H + h_kv) * kG + t) * kD;
        float kv[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) kv[k] = bits_to_float(kt[lane + 32 * k], g.dtype);  // plain: a step writes the tail
        const int vidx = min((int)sub[g.off_vidx + tok_pos(t)], P);  // P: stored raw
        const float vrow = g.tx ? vr[tok_pos(t)] : 1.0f;
#pragma unroll
        for (int j = 0; j < NT; ++j) {
          // score of head 4j + tig (every lane computes the tile's 4 heads, keeps its own)
          float myscore = 0.f;
#pragma unroll
          for (int hl = 0; hl < 4; ++hl) {
            const int hh = 4 * j + hl;
            float part = 0.f;
#pragma unroll
            for (int k = 0; k < 4; ++k) part = fmaf(qraw[hh * kD + lane + 32 * k], kv[k], part);
            part = warp_sum(part) * scale_log2;
            if (hl == tig) myscore = part;
          }
          const int hh = 4 * j + tig;
          const bool real = hh < Gq;
          const float mnew = fmaxf(mrun[j], myscore);
          const float alpha = ex2(mrun[j] - mnew);
          if (__any_sync(kFull, alpha != 1.0f)) {
            lrun[j] *= alpha;
#pragma unroll
            for (int u = 0; u < 4; ++u) zacc[j][u] *= alpha;
#pragma unroll
            for (int mt = 0; mt < 8; ++mt)
#pragma unroll
              for (int u = 0; u < 4; ++u) accv[j][mt][u] *= alpha;
            for (int jj = gq; jj < Pe; jj += 8) Ww[hh * P1 + jj] *= alpha;
          }
          mrun[j] = mnew;
          __syncwarp();
          const float p = real ? ex2(myscore - mnew) : 0.f;
          const float pv = p * vrow;
          if (gq == 0) {
            lrun[j] += p;
            if (real) Ww[hh * P1 + vidx] += pv;
#pragma unroll
            for (int u = 0; u < 4; ++u) zacc[j][u] = fmaf(pv, vz[vzc_pos(t, u)], zacc[j][u]);
          }
          // residual codes of this thread's 16 channels
#pragma unroll
          for (int mt = 0; mt < 8; ++mt)
#pragma unroll
            for (int rh = 0; rh < 2; ++rh) {
              const int d = 16 * mt + 8 * rh + gq;
              int w, bt;
              frag_pos(BITS, 2, d, t, w, bt);
              const int code = (vwords[w] >> bt) & ((1 << BITS) - 1);
              accv[j][mt][2 * rh] = fmaf(pv * vs[vsc_pos(t, mt >> 1)], (float)code, accv[j][mt][2 * rh]);
            }
          __syncwarp();
        }
      }
    } else if (lane == 0) {
      set_status(g.status, KVQ_DEV_BAD_PAGE);
    }
  }

  // ---- merge the warps and write the partials
#pragma unroll
  for (int j = 0; j < NT; ++j) {
    float l = lrun[j];
    l += __shfl_xor_sync(kFull, l, 4);
    l += __shfl_xor_sync(kFull, l, 8);
    l += __shfl_xor_sync(kFull, l, 16);
    lrun[j] = l;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      float z = zacc[j][u];
      z += __shfl_xor_sync(kFull, z, 4);
      z += __shfl_xor_sync(kFull, z, 8);
      z += __shfl_xor_sync(kFull, z, 16);
      zacc[j][u] = z;
    }
  }
  __syncthreads();  // every warp is done with its ring: reuse it for the merge
  float* mo = reinterpret_cast<float*>(smem + sp.ring);   // [kWarps][NH][128]
  float* mm = mo + kWarps * NH * kD;                      // [kWarps][NH] max
  float* ml = mm + kWarps * NH;                           // [kWarps][NH] sum
  float* mz = ml + kWarps * NH;                           // [kWarps][NH][4]
#pragma unroll
  for (int j = 0; j < NT; ++j) {
    const int hh = 4 * j + tig;
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) {
      mo[(warp * NH + hh) * kD + 16 * mt + gq] = accv[j][mt][0] + accv[j][mt][1];
      mo[(warp * NH + hh) * kD + 16 * mt + gq + 8] = accv[j][mt][2] + accv[j][mt][3];
    }
    if (gq == 0) {
      mm[warp * NH + hh] = mrun[j];
      ml[warp * NH + hh] = lrun[j];
#pragma unroll
      for (int u = 0; u < 4; ++u) mz[(warp * NH + hh) * 4 + u] = zacc[j][u];
    }
  }
  float* wc = mz + kWarps * NH * 4;                       // [P][NH] merged pattern weights
  float* fsh = wc + P * NH;                               // [NH][kWarps] warp weights
  __syncthreads();
  for (int hh = warp; hh < Gq; hh += kWarps) {
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) M = fmaxf(M, mm[w * NH + hh]);
    float f[kWarps], Ls = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      const float mw = mm[w * NH + hh];
      f[w] = (mw == -INFINITY) ? 0.f : ex2(mw - M);
      Ls += f[w] * ml[w * NH + hh];
      if (lane == w) fsh[hh * kWarps + w] = f[w];
    }
    const size_t base = ((size_t)b * Hq + h_kv * Gq + hh) * nsplit + split;
    if (lane == 0) { part_ml[2 * base] = M; part_ml[2 * base + 1] = Ls; }
    for (int jj = lane; jj < Pe; jj += 32) {
      float Wv = 0.f;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) Wv += f[w] * Wall[(w * NH + hh) * P1 + jj];
      wc[jj * NH + hh] = Wv;
    }
  }
  __syncthreads();
  // o = sum_w f_w (residual + zero terms of warp w) + sum_j W_j M_V[j]: thread = channel c,
  // query heads hg, hg + HG, ...; each M_V value is read once per CTA
  {
    constexpr int HG = kWarps * 32 / kD;
    constexpr int NA = NH / HG;
    const int c = threadIdx.x % kD, hg = threadIdx.x / kD;
    const float* mv = g.vpat + sh * P * kD + c;
    float acc[NA];
#pragma unroll
    for (int i = 0; i < NA; ++i) acc[i] = 0.f;
#pragma unroll 8
    for (int j = 0; j < Pe; ++j) {
      const float m = __ldg(mv + (size_t)j * kD);
#pragma unroll
      for (int i = 0; i < NA; ++i) acc[i] = fmaf(wc[j * NH + hg + HG * i], m, acc[i]);
    }
#pragma unroll
    for (int i = 0; i < NA; ++i) {
      const int hh = hg + HG * i;
      if (hh >= Gq) continue;
      float o = acc[i];
#pragma unroll
      for (int w = 0; w < kWarps; ++w)
        o = fmaf(fsh[hh * kWarps + w], mo[(w * NH + hh) * kD + c] + mz[(w * NH + hh) * 4 + (c >> 5)], o);
      part_o[(((size_t)b * Hq + h_kv * Gq + hh) * nsplit + split) * kD + c] = o;
    }
  }

  // ---- the CTA that completes a (sequence, KV head) group merges its splits into `out`
  __shared__ int last;
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) {
    last = atomicAdd(arrivals + (size_t)b * g.H + h_kv, 1) == nsplit - 1;
    if (last) arrivals[(size_t)b * g.H + h_kv] = 0;  // every split has arrived: ready for the next call
  }
  __syncthreads();
  if (!last) return;
  __threadfence();
  combine_group(g, Hq, nsplit, b, h_kv, Gq, set, part_ml, part_o, out);
}

template <int BITS, int NT, int STAGES, int NW, bool STEP = false>
struct Launcher {
  using Step = Launcher<BITS, NT, STAGES, NW, true>;  // the decode-step variant of this configuration
  static auto kernel() { return decode_mma_kernel<BITS, NT, STAGES, NW, STEP>; }
  static int smem(const Geom& g) { return smem_plan((int)g.sub_bytes, STAGES, NT, g.P, NW).total; }
  static int occupancy(const Geom& g) {
    int n = 0;
    if (cudaFuncSetAttribute(kernel(), cudaFuncAttributeMaxDynamicSharedMemorySize, smem(g)) != cudaSuccess) return 1;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel(), NW * 32, smem(g)) != cudaSuccess) return 1;
    return n > 0 ? n : 1;
  }
  static cudaError_t launch(const Geom& g, const void* q, int Hq, float scale_log2, int nsplit, float* ml, float* o,
                            int* arrivals, float* out, const void* k_new, const void* v_new, int* seqcnt,
                            cudaStream_t st) {
    const int total = smem(g);
    cudaError_t e = cudaFuncSetAttribute(kernel(), cudaFuncAttributeMaxDynamicSharedMemorySize, total);
    if (e != cudaSuccess) return e;
    dim3 grid(nsplit, g.H, g.B);
    kernel()<<<grid, NW * 32, total, st>>>(g, (const uint16_t*)q, Hq, scale_log2, nsplit, ml, o, arrivals, out,
                                           (const uint16_t*)k_new, (const uint16_t*)v_new, seqcnt);
    return cudaGetLastError();
  }
};

// Dispatch on (bits, n-tiles, pipeline configuration) with a functor receiving the Launcher
// type.  Configurations (stages per warp, warps per CTA): 0 = (3, 4), 1 = (2, 4), 2 = (2, 8),
// 3 = (3, 8); the query-head tiles beyond the first use configuration 0 or 1.
template <typename F>
auto dispatch(const Geom& g, int Hq, int cfg, F&& f) {
  const int NT = (Hq / g.H + 3) / 4;
#define KVQ_CFG(B)                                                   \
  if (NT == 1) {                                                     \
    switch (cfg) {                                                   \
      case 1: return f(Launcher<B, 1, 2, 4>{});                      \
      case 2: return f(Launcher<B, 1, 2, 8>{});                      \
      case 3: return f(Launcher<B, 1, 3, 8>{});                      \
      default: return f(Launcher<B, 1, 3, 4>{});                     \
    }                                                                \
  }                                                                  \
  if (cfg == 1) {                                                    \
    switch (NT) {                                                    \
      case 2: return f(Launcher<B, 2, 2, 4>{});                      \
      case 3: return f(Launcher<B, 3, 2, 4>{});                      \
      default: return f(Launcher<B, 4, 2, 4>{});                     \
    }                                                                \
  }                                                                  \
  switch (NT) {                                                      \
    case 2: return f(Launcher<B, 2, 3, 4>{});                        \
    case 3: return f(Launcher<B, 3, 3, 4>{});                        \
    default: return f(Launcher<B, 4, 3, 4>{});                       \
  }
  if (g.bits == 2) { KVQ_CFG(2) } else { KVQ_CFG(4) }
#undef KVQ_CFG
}

int decode_stages() {
  const char* s = getenv("KVQ_DECODE_CFG");
  const int v = s ? atoi(s) : 1;
  return (v >= 0 && v <= 3) ? v : 1;
}

}  // namespace

// Number of splits of the token axis.  Model: a CTA costs a fixed setup (the query and the
// q.M_K table, the combine: about 40 pages' worth, measured) plus its pages; each SM takes
// ceil(CTAs / SMs) of the CTAs, `occ` at a time, and a round of k concurrent CTAs takes
// max(k, 3) CTA-times (fewer than 3 CTAs do not saturate an SM).  The page count is the capacity
// (the lengths are on the device).  Fitted to the measured best split count of four shapes
// (one B200): 64 groups of 1024 pages -> 9 splits (2-bit) and 13 (4-bit, fewer CTAs per SM),
// 512 groups of 512 -> 2, 256 groups of ~300 (the decode-step loop) -> 2.
int decode_mma_splits(const Geom& g, int Hq, int num_sms) {
  const int occ = std::max(1, dispatch(g, Hq, decode_stages(), [&](auto L) { return decltype(L)::occupancy(g); }));
  const int units = g.B * g.H > 0 ? g.B * g.H : 1;
  const int pages = g.maxp > 1 ? g.maxp : 1;
  const int maxns = pages < 256 ? pages : 256;
  const int sms = num_sms > 0 ? num_sms : 1;
  int best = 1;
  double best_cost = 1e300;
  for (int ns = 1; ns <= maxns; ++ns) {
    const int64_t per_sm = ((int64_t)units * ns + sms - 1) / sms;  // CTAs of the busiest SM
    const int64_t full = per_sm / occ, rem = per_sm % occ;
    const double slots = (double)full * std::max(occ, 3) + (rem ? std::max<int64_t>(rem, 3) : 0);
    const double cost = slots * (40.0 + std::ceil((double)pages / ns));
    if (cost < best_cost * (1.0 - 1e-9)) { best_cost = cost; best = ns; }
  }
  return best;
}

size_t decode_mma_smem(const Geom& g, int Hq) {
  return (size_t)dispatch(g, Hq, decode_stages(), [&](auto L) { return decltype(L)::smem(g); });
}

cudaError_t launch_decode_mma(const Geom& g, const void* q, int Hq, float scale_log2, int nsplit, float* ml,
                              float* o, int* arrivals, float* out, cudaStream_t st) {
  return dispatch(g, Hq, decode_stages(), [&](auto L) {
    return decltype(L)::launch(g, q, Hq, scale_log2, nsplit, ml, o, arrivals, out, nullptr, nullptr, nullptr, st);
  });
}

cudaError_t launch_decode_step_mma(const Geom& g, const void* k_new, const void* v_new, const void* q, int Hq,
                                   float scale_log2, int nsplit, float* ml, float* o, int* arrivals, int* seqcnt,
                                   float* out, cudaStream_t st) {
  return dispatch(g, Hq, decode_stages(), [&](auto L) {
    return decltype(L)::Step::launch(g, q, Hq, scale_log2, nsplit, ml, o, arrivals, out, k_new, v_new, seqcnt, st);
  });
}

}  // namespace kvq
