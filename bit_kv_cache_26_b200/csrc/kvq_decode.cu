// Decode attention over the quantized paged cache ("PatternKV", Section 3.4:
// pattern-index restoration, dequantization and the QK^T / P.V products fused
// into the attention kernels), split-K over the token axis; the CTA that completes
// the last split of a (sequence, KV head) group runs the log-sum-exp combine, which
// also adds the pattern term and undoes the pre-transform (kvq_decode_mma.cu).
//
// Partial results per (sequence, query head, split):
//   m  running max of the base-2 logits, l  sum of 2^(logit - m),
//   o[128]  sum of p * (s*code + z) + sum_j W_j M_V[j] in the quantized space, with
//           W_j the sum of p over the split's tokens that use V pattern j.
#include <algorithm>
#include <cstdlib>

#include "kvq_common.cuh"
#include "kvq_internal.h"

namespace kvq {

namespace {

constexpr float kLog2e = 1.4426950408889634f;

}  // namespace

int decode_num_splits(const Geom& g, int Hq, int num_sms) { return decode_mma_splits(g, Hq, num_sms); }

size_t decode_workspace(const Geom& g, int Hq, int nsplit) {
  const size_t rows = (size_t)g.B * Hq * nsplit;
  return rows * (2 + kD) * sizeof(float) + (size_t)g.B * g.H * sizeof(int) + 256;
}

// Iteration limit of the page-copy waits: the default, or KVQ_TEST_WAIT_LIMIT (read once) for
// tests that make the waits expire on purpose.
uint32_t page_wait_limit(uint32_t dflt) {
  static const long long v = [] {
    const char* e = getenv("KVQ_TEST_WAIT_LIMIT");
    return e ? atoll(e) : -1LL;
  }();
  return v >= 0 ? (uint32_t)std::min<long long>(v, 0xffffffffLL) : dflt;
}

// Split partials, then the per-(sequence, KV head) arrival counters (zeroed here, on the stream).
cudaError_t launch_decode(const Geom& g0, const void* q, int Hq, float sm_scale, float* out, void* ws, int nsplit,
                          cudaStream_t st) {
  if (g0.B == 0) return cudaSuccess;
  Geom g = g0;
  g.wait_limit = page_wait_limit(g0.wait_limit);
  const size_t rows = (size_t)g.B * Hq * nsplit;
  float* part_ml = reinterpret_cast<float*>(ws);
  float* part_o = part_ml + 2 * rows;
  int* arrivals = reinterpret_cast<int*>(part_o + kD * rows);
  cudaError_t e = cudaMemsetAsync(arrivals, 0, (size_t)g.B * g.H * sizeof(int), st);
  if (e != cudaSuccess) return e;
  return launch_decode_mma(g, q, Hq, sm_scale * kLog2e, nsplit, part_ml, part_o, arrivals, out, st);
}

// Decode step: partials, the per-(sequence, KV head) arrival counters, then one counter per
// sequence.  No memset: the kernel leaves every counter at zero (the caller zeroes the workspace
// once, before its first use).
size_t step_workspace(const Geom& g, int Hq, int nsplit) {
  return decode_workspace(g, Hq, nsplit) + (size_t)g.B * sizeof(int) + 256;
}

cudaError_t launch_decode_step(const Geom& g0, const void* k_new, const void* v_new, const void* q, int Hq,
                               float sm_scale, float* out, void* ws, int nsplit, cudaStream_t st) {
  if (g0.B == 0) return cudaSuccess;
  Geom g = g0;
  g.wait_limit = page_wait_limit(g0.wait_limit);
  const size_t rows = (size_t)g.B * Hq * nsplit;
  float* part_ml = reinterpret_cast<float*>(ws);
  float* part_o = part_ml + 2 * rows;
  int* arrivals = reinterpret_cast<int*>(part_o + kD * rows);
  int* seqcnt = arrivals + (size_t)g.B * g.H;
  return launch_decode_step_mma(g, k_new, v_new, q, Hq, sm_scale * kLog2e, nsplit, part_ml, part_o, arrivals, seqcnt,
                                out, st);
}

}  // namespace kvq
