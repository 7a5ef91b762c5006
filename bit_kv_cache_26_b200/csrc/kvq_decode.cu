// Decode attention over the quantized paged cache ("PatternKV", Section 3.4:
// pattern-index restoration, dequantization and the QK^T / P.V products fused
// into the attention kernels), split-K over the token axis, then a log-sum-exp
// combine that also adds the pattern term and undoes the pre-transform.
//
// Partial results per (sequence, query head, split):
//   m  running max of the base-2 logits, l  sum of 2^(logit - m),
//   o[128]  sum of p * (s*q + z) [+ pattern] in the quantized space,
//   W[P]    sum of p over the tokens that use each V pattern.
#include "kvq_common.cuh"
#include "kvq_internal.h"

namespace kvq {

namespace {

constexpr float kLog2e = 1.4426950408889634f;

// ---------------------------------------------------------------------------
// Reference-structure decode kernel: one warp per token at a time, lanes over
// channels.  Used for every shape; simple and exact in structure.
// ---------------------------------------------------------------------------
constexpr int kSimpleThreads = 128;
constexpr int kMaxGq = 16;

__global__ void __launch_bounds__(kSimpleThreads) decode_simple_kernel(Geom g, const uint16_t* __restrict__ q,
                                                                       int Hq, float scale_log2, int nsplit,
                                                                       float* __restrict__ part_ml,
                                                                       float* __restrict__ part_o,
                                                                       float* __restrict__ part_w) {
  const int split = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int Gq = Hq / g.H;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  int L = g.seq_len[b];
  if (L < 0 || L > g.maxp * kG) {  // corrupt length: never read outside the page table
    if (threadIdx.x == 0 && split == 0) set_status(g.status, KVQ_DEV_OVERFLOW);
    L = 0;
  }
  const int nfull = L / kG, ntail = L % kG;
  const int per = (nfull + nsplit - 1) / nsplit;
  const int p0 = min(nfull, split * per), p1 = min(nfull, p0 + per);
  const bool do_tail = (split == nsplit - 1) && ntail > 0;
  int set = g.seq_to_set ? g.seq_to_set[b] : 0;
  const bool bad_set = set < 0 || set >= g.S;
  if (bad_set) set = 0;

  __shared__ float wm[4][kMaxGq], wl[4][kMaxGq];
  extern __shared__ float dyn[];
  float (*qt)[kD] = reinterpret_cast<float (*)[kD]>(dyn);               // [Gq][128] query, quantized space
  float (*qr)[kD] = reinterpret_cast<float (*)[kD]>(dyn + Gq * kD);      // [Gq][128] raw query (tail keys)
  float* wo = dyn + 2 * Gq * kD;                                         // [4][Gq][128]
  float* wW = dyn + 6 * Gq * kD;                                         // [4][Gq][P]

  const float* MK = g.kpat + ((size_t)set * g.H + h) * g.P * kD;
  const float* cK = g.tx ? g.kcol + ((size_t)set * g.H + h) * kD : nullptr;

  // queries
  for (int hh = warp; hh < Gq; hh += nwarps) {
    const uint16_t* src = q + ((size_t)b * Hq + h * Gq + hh) * kD;
    float v[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      v[k] = load_elem(src + lane + 32 * k, g.dtype);
      qr[hh][lane + 32 * k] = v[k];
    }
    if (g.tx) {
      fwht_warp(v, lane);
#pragma unroll
      for (int k = 0; k < 4; ++k) v[k] = v[k] * __ldg(cK + lane + 32 * k) * 0.0078125f;
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) qt[hh][lane + 32 * k] = v[k];
  }
  for (int i = threadIdx.x; i < 4 * Gq * g.P; i += blockDim.x) wW[i] = 0.f;
  __syncthreads();

  float m[kMaxGq], l[kMaxGq], acc[kMaxGq][4];
  for (int hh = 0; hh < Gq; ++hh) {
    m[hh] = -INFINITY; l[hh] = 0.f;
#pragma unroll
    for (int k = 0; k < 4; ++k) acc[hh][k] = 0.f;
  }
  float* myW = wW + (size_t)warp * Gq * g.P;

  auto process = [&](const uint8_t* sub, int slot, bool key_exact, const uint16_t* kraw) {
    // key
    float kv[4];
    float krow = 1.0f;
    if (key_exact) {
#pragma unroll
      for (int k = 0; k < 4; ++k) kv[k] = load_elem(kraw + lane + 32 * k, g.dtype);
    } else {
      const uint32_t* words = reinterpret_cast<const uint32_t*>(sub);
      const float* ks = reinterpret_cast<const float*>(sub + g.off_ks);
      const float* kz = reinterpret_cast<const float*>(sub + g.off_kz);
      int idx = min((int)sub[g.off_kidx + tok_pos(slot)], g.P - 1);
      if (g.tx) krow = reinterpret_cast<const float*>(sub + g.off_krow)[tok_pos(slot)];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        int d = lane + 32 * k, w, bt;
        frag_pos(g.bits, 8, slot, d, w, bt);
        int code = (words[w] >> bt) & ((1 << g.bits) - 1);
        kv[k] = ks[ksc_pos(d)] * (float)code + kz[ksc_pos(d)] + MK[(size_t)idx * kD + d];
      }
    }
    // value (always quantized)
    const uint32_t* vwords = reinterpret_cast<const uint32_t*>(sub + g.off_vc);
    const float* vs = reinterpret_cast<const float*>(sub + g.off_vs);
    const float* vz = reinterpret_cast<const float*>(sub + g.off_vz);
    int vidx = min((int)sub[g.off_vidx + tok_pos(slot)], g.P - 1);
    float vrow = g.tx ? reinterpret_cast<const float*>(sub + g.off_vrow)[tok_pos(slot)] : 1.0f;
    float vv[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      int d = lane + 32 * k, w, bt;
      frag_pos(g.bits, 2, d, slot, w, bt);
      int code = (vwords[w] >> bt) & ((1 << g.bits) - 1);
      vv[k] = vs[vsc_pos(slot, k)] * (float)code + vz[vzc_pos(slot, k)];
    }
    for (int hh = 0; hh < Gq; ++hh) {
      const float* qq = key_exact ? qr[hh] : qt[hh];
      float part = 0.f;
#pragma unroll
      for (int k = 0; k < 4; ++k) part += qq[lane + 32 * k] * kv[k];
      float sc = warp_sum(part) * krow * scale_log2;
      float mn = fmaxf(m[hh], sc);
      float alpha = exp2f(m[hh] - mn);
      float p = exp2f(sc - mn);
      l[hh] = l[hh] * alpha + p;
      float pv = p * vrow;
#pragma unroll
      for (int k = 0; k < 4; ++k) acc[hh][k] = acc[hh][k] * alpha + pv * vv[k];
      if (alpha != 1.0f)
        for (int j = lane; j < g.P; j += 32) myW[hh * g.P + j] *= alpha;
      __syncwarp();
      if (lane == 0) myW[hh * g.P + vidx] += pv;
      __syncwarp();
      m[hh] = mn;
    }
  };

  if (!bad_set) {
    for (int pg = p0 + warp; pg < p1; pg += nwarps) {
      int phys = g.page_table[(size_t)b * g.maxp + pg];
      if (phys < 0 || phys >= g.npages) { if (lane == 0) set_status(g.status, KVQ_DEV_BAD_PAGE); continue; }
      const uint8_t* sub = g.pool + (size_t)phys * g.page_bytes + (size_t)h * g.sub_bytes;
      for (int slot = 0; slot < kG; ++slot) process(sub, slot, false, nullptr);
    }
    if (do_tail && warp == 0) {
      int phys = g.page_table[(size_t)b * g.maxp + nfull];
      if (phys < 0 || phys >= g.npages) {
        if (lane == 0) set_status(g.status, KVQ_DEV_BAD_PAGE);
      } else {
        const uint8_t* sub = g.pool + (size_t)phys * g.page_bytes + (size_t)h * g.sub_bytes;
        for (int slot = 0; slot < ntail; ++slot)
          process(sub, slot, true, g.k_tail + (((size_t)b * g.H + h) * kG + slot) * kD);
      }
    }
  } else if (threadIdx.x == 0) {
    set_status(g.status, KVQ_DEV_BAD_SET);
  }

  // merge the warps
  for (int hh = 0; hh < Gq; ++hh) {
    if (lane == 0) { wm[warp][hh] = m[hh]; wl[warp][hh] = l[hh]; }
#pragma unroll
    for (int k = 0; k < 4; ++k) wo[((size_t)warp * Gq + hh) * kD + lane + 32 * k] = acc[hh][k];
  }
  __syncthreads();
  for (int hh = warp; hh < Gq; hh += nwarps) {
    float M = -INFINITY;
    for (int w = 0; w < nwarps; ++w) M = fmaxf(M, wm[w][hh]);
    float f[4], L2 = 0.f;
    for (int w = 0; w < nwarps; ++w) {
      f[w] = (wm[w][hh] == -INFINITY) ? 0.f : exp2f(wm[w][hh] - M);
      L2 += f[w] * wl[w][hh];
    }
    size_t base = ((size_t)b * Hq + h * Gq + hh) * nsplit + split;
    if (lane == 0) { part_ml[2 * base] = M; part_ml[2 * base + 1] = L2; }
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      float o = 0.f;
      for (int w = 0; w < nwarps; ++w) o += f[w] * wo[((size_t)w * Gq + hh) * kD + lane + 32 * k];
      part_o[base * kD + lane + 32 * k] = o;
    }
    for (int j = lane; j < g.P; j += 32) {
      float W = 0.f;
      for (int w = 0; w < nwarps; ++w) W += f[w] * wW[((size_t)w * Gq + hh) * g.P + j];
      part_w[base * g.P + j] = W;
    }
  }
}

// ---------------------------------------------------------------------------
// Combine: log-sum-exp merge of the splits, pattern term, inverse transform.
// One warp per (sequence, query head).
// ---------------------------------------------------------------------------
__global__ void decode_combine_kernel(Geom g, int Hq, int nsplit, const float* __restrict__ part_ml,
                                      const float* __restrict__ part_o, const float* __restrict__ part_w,
                                      float* __restrict__ out) {
  const int lane = threadIdx.x & 31;
  const int row = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (row >= g.B * Hq) return;
  const int b = row / Hq, hq = row % Hq, h = hq / (Hq / g.H);
  int set = g.seq_to_set ? g.seq_to_set[b] : 0;
  if (set < 0 || set >= g.S) set = 0;
  const size_t base = (size_t)row * nsplit;
  float M = -INFINITY;
  for (int s = 0; s < nsplit; ++s) M = fmaxf(M, part_ml[2 * (base + s)]);
  float o[4] = {0.f, 0.f, 0.f, 0.f};
  float* outp = out + (size_t)row * kD;
  if (M == -INFINITY) {
#pragma unroll
    for (int k = 0; k < 4; ++k) outp[lane + 32 * k] = 0.f;
    return;
  }
  float Lsum = 0.f;
  for (int s = 0; s < nsplit; ++s) {
    float ms = part_ml[2 * (base + s)];
    if (ms == -INFINITY) continue;
    float f = exp2f(ms - M);
    Lsum += f * part_ml[2 * (base + s) + 1];
#pragma unroll
    for (int k = 0; k < 4; ++k) o[k] += f * part_o[(base + s) * kD + lane + 32 * k];
  }
  const float* MV = g.vpat + ((size_t)set * g.H + h) * g.P * kD;
  for (int j = 0; j < g.P; ++j) {
    float W = 0.f;
    for (int s = 0; s < nsplit; ++s) {
      float ms = part_ml[2 * (base + s)];
      if (ms == -INFINITY) continue;
      W += exp2f(ms - M) * part_w[(base + s) * g.P + j];
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) o[k] += W * MV[(size_t)j * kD + lane + 32 * k];
  }
  float inv = 1.0f / Lsum;
#pragma unroll
  for (int k = 0; k < 4; ++k) o[k] *= inv;
  if (g.tx) {
    const float* cV = g.vcol + ((size_t)set * g.H + h) * kD;
#pragma unroll
    for (int k = 0; k < 4; ++k) o[k] *= cV[lane + 32 * k];
    fwht_warp(o, lane);
#pragma unroll
    for (int k = 0; k < 4; ++k) o[k] *= 0.0078125f;
  }
#pragma unroll
  for (int k = 0; k < 4; ++k) outp[lane + 32 * k] = o[k];
}

}  // namespace

int decode_num_splits(const Geom& g, int num_sms) {
  int units = max(1, g.B * g.H);
  int want = (4 * num_sms + units - 1) / units;
  return max(1, min(want, max(1, g.maxp)));
}

size_t decode_workspace(const Geom& g, int Hq, int nsplit) {
  size_t rows = (size_t)g.B * Hq * nsplit;
  return rows * (2 + kD + g.P) * sizeof(float) + 256;
}

cudaError_t launch_decode(const Geom& g, const void* q, int Hq, float sm_scale, float* out, void* ws, int nsplit,
                          cudaStream_t st) {
  if (g.B == 0) return cudaSuccess;
  size_t rows = (size_t)g.B * Hq * nsplit;
  float* part_ml = reinterpret_cast<float*>(ws);
  float* part_o = part_ml + 2 * rows;
  float* part_w = part_o + kD * rows;
  const int Gq = Hq / g.H;
  dim3 grid(nsplit, g.H, g.B);
  size_t smem = ((size_t)6 * Gq * kD + (size_t)4 * Gq * g.P) * sizeof(float);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(decode_simple_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  decode_simple_kernel<<<grid, kSimpleThreads, smem, st>>>(g, (const uint16_t*)q, Hq, sm_scale * kLog2e, nsplit,
                                                          part_ml, part_o, part_w);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  int rows_total = g.B * Hq;
  decode_combine_kernel<<<(rows_total + 7) / 8, 256, 0, st>>>(g, Hq, nsplit, part_ml, part_o, part_w, out);
  return cudaGetLastError();
}

}  // namespace kvq
