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
// Combine: log-sum-exp merge of the splits, pattern term sum_j W_j M_V[j], inverse
// pre-transform.  One CTA of 128 threads (thread = channel) per (sequence, query head).
// A non-finite output (an operand outside the fp32 / bf16 range upstream) sets
// KVQ_DEV_RANGE.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(128) decode_combine_kernel(Geom g, int Hq, int nsplit,
                                                             const float* __restrict__ part_ml,
                                                             const float* __restrict__ part_o,
                                                             const float* __restrict__ part_w, float* __restrict__ out) {
  __shared__ float Wsh[256];
  __shared__ float osh[kD];
  const int row = blockIdx.x, d = threadIdx.x;
  const int b = row / Hq, hq = row % Hq, h = hq / (Hq / g.H);
  int set = g.seq_to_set ? g.seq_to_set[b] : 0;
  if (set < 0 || set >= g.S) set = 0;
  const size_t base = (size_t)row * nsplit;
  float M = -INFINITY;
  for (int s = 0; s < nsplit; ++s) M = fmaxf(M, part_ml[2 * (base + s)]);
  float* outp = out + (size_t)row * kD;
  if (M == -INFINITY) {  // no tokens
    outp[d] = 0.f;
    return;
  }
  float Lsum = 0.f, o = 0.f;
  for (int s = 0; s < nsplit; ++s) {
    const float ms = part_ml[2 * (base + s)];
    if (ms == -INFINITY) continue;
    const float f = exp2f(ms - M);
    Lsum += f * part_ml[2 * (base + s) + 1];
    o += f * part_o[(base + s) * kD + d];
  }
  for (int j = d; j < g.P; j += blockDim.x) {
    float W = 0.f;
    for (int s = 0; s < nsplit; ++s) {
      const float ms = part_ml[2 * (base + s)];
      if (ms == -INFINITY) continue;
      W += exp2f(ms - M) * part_w[(base + s) * g.P + j];
    }
    Wsh[j] = W;
  }
  __syncthreads();
  const float* MV = g.vpat + ((size_t)set * g.H + h) * g.P * kD;
  for (int j = 0; j < g.P; ++j) o = fmaf(Wsh[j], __ldg(MV + (size_t)j * kD + d), o);
  o *= 1.0f / Lsum;
  if (g.tx) {
    const float* cV = g.vcol + ((size_t)set * g.H + h) * kD;
    osh[d] = o * cV[d];
    __syncthreads();
    if (d < 32) {
      float v[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) v[k] = osh[d + 32 * k];
      fwht_warp(v, d);
#pragma unroll
      for (int k = 0; k < 4; ++k) osh[d + 32 * k] = v[k] * 0.0078125f;
    }
    __syncthreads();
    o = osh[d];
  }
  if (!isfinite(o)) set_status(g.status, KVQ_DEV_RANGE);
  outp[d] = o;
}

}  // namespace

int decode_num_splits(const Geom& g, int Hq, int num_sms) { return decode_mma_splits(g, Hq, num_sms); }

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
  cudaError_t e = launch_decode_mma(g, q, Hq, sm_scale * kLog2e, nsplit, part_ml, part_o, part_w, st);
  if (e != cudaSuccess) return e;
  decode_combine_kernel<<<g.B * Hq, 128, 0, st>>>(g, Hq, nsplit, part_ml, part_o, part_w, out);
  return cudaGetLastError();
}

}  // namespace kvq
