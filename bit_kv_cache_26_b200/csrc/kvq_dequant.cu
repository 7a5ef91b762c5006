// Reconstruction of cached tokens ("PatternKV", Section 3.2: fetch the pattern by
// its stored index and add the dequantized residual, s*q + z of Eq. 1), mapped
// back through the inverse pre-transform when it is enabled.  Verification and
// export path.
#include "kvq_common.cuh"
#include "kvq_internal.h"

namespace kvq {

namespace {

// One warp per (token, KV head).
__global__ void dequant_kernel(Geom g, int b, int start, int count, float* __restrict__ k_out,
                               float* __restrict__ v_out) {
  const int lane = threadIdx.x & 31;
  const int item = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (item >= count * g.H) return;
  const int ti = item / g.H, h = item % g.H, t = start + ti;
  const int L = g.seq_len[b];
  const int sealed = (L / kG) * kG;
  int set = g.seq_to_set ? g.seq_to_set[b] : 0;
  if (set < 0 || set >= g.S) { if (lane == 0) set_status(g.status, KVQ_DEV_BAD_SET); return; }
  const int pg = t / kG, slot = t % kG;
  const int phys = g.page_table[(size_t)b * g.maxp + pg];
  if (phys < 0 || phys >= g.npages) { if (lane == 0) set_status(g.status, KVQ_DEV_BAD_PAGE); return; }
  const uint8_t* sub = g.pool + (size_t)phys * g.page_bytes + (size_t)h * g.sub_bytes;
  const size_t sh = ((size_t)set * g.H + h);
  const int mask = (1 << g.bits) - 1;

  if (k_out) {
    float v[4];
    float* dst = k_out + ((size_t)ti * g.H + h) * kD;
    if (t >= sealed) {
      const uint16_t* src = g.k_tail + (((size_t)b * g.H + h) * kG + slot) * kD;
#pragma unroll
      for (int k = 0; k < 4; ++k) dst[lane + 32 * k] = load_elem(src + lane + 32 * k, g.dtype);
    } else {
      const uint32_t* words = reinterpret_cast<const uint32_t*>(sub);
      const float* ks = reinterpret_cast<const float*>(sub + g.off_ks);
      const float* kz = reinterpret_cast<const float*>(sub + g.off_kz);
      const int idx = min((int)sub[g.off_kidx + tok_pos(slot)], p_eff(g, (int)sh) - 1);
      const float* M = g.kpat + (sh * g.P + idx) * kD;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        int d = lane + 32 * k, w, bt;
        frag_pos(g.bits, 8, slot, d, w, bt);
        int code = (words[w] >> bt) & mask;
        v[k] = ks[ksc_pos(d)] * (float)code + kz[ksc_pos(d)] + M[d];
      }
      if (g.tx) {
        float r = reinterpret_cast<const float*>(sub + g.off_krow)[tok_pos(slot)];
        const float* c = g.kcol + sh * kD;
#pragma unroll
        for (int k = 0; k < 4; ++k) v[k] = r * (v[k] * c[lane + 32 * k]);
        fwht_warp(v, lane);
#pragma unroll
        for (int k = 0; k < 4; ++k) v[k] *= 0.0078125f;
      }
#pragma unroll
      for (int k = 0; k < 4; ++k) dst[lane + 32 * k] = v[k];
    }
  }
  if (v_out) {
    const uint32_t* words = reinterpret_cast<const uint32_t*>(sub + g.off_vc);
    const float* vs = reinterpret_cast<const float*>(sub + g.off_vs);
    const float* vz = reinterpret_cast<const float*>(sub + g.off_vz);
    const int vi = sub[g.off_vidx + tok_pos(slot)];
    const float* M = vi == kRawIndex ? nullptr : g.vpat + (sh * g.P + min(vi, p_eff(g, (int)sh) - 1)) * kD;  // 255: raw
    float v[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      int d = lane + 32 * k, w, bt;
      frag_pos(g.bits, 2, d, slot, w, bt);
      int code = (words[w] >> bt) & mask;
      v[k] = vs[vsc_pos(slot, k)] * (float)code + vz[vzc_pos(slot, k)] + (M ? M[d] : 0.0f);
    }
    if (g.tx) {
      float r = reinterpret_cast<const float*>(sub + g.off_vrow)[tok_pos(slot)];
      const float* c = g.vcol + sh * kD;
#pragma unroll
      for (int k = 0; k < 4; ++k) v[k] = r * (v[k] * c[lane + 32 * k]);
      fwht_warp(v, lane);
#pragma unroll
      for (int k = 0; k < 4; ++k) v[k] *= 0.0078125f;
    }
    float* dst = v_out + ((size_t)ti * g.H + h) * kD;
#pragma unroll
    for (int k = 0; k < 4; ++k) dst[lane + 32 * k] = v[k];
  }
}

}  // namespace

cudaError_t launch_dequant(const Geom& g, int seq, int start, int count, float* k_out, float* v_out,
                           cudaStream_t st) {
  if (count <= 0) return cudaSuccess;
  int items = count * g.H;
  dequant_kernel<<<(items + 7) / 8, 256, 0, st>>>(g, seq, start, count, k_out, v_out);
  return cudaGetLastError();
}

}  // namespace kvq
