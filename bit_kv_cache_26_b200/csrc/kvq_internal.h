// Internal host-side interfaces between the C-ABI layer (kvq_api.cu) and the
// kernel translation units.  Not installed, not part of the ABI.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace kvq {

struct Geom;

// quantize-append (kvq_append.cu)
size_t append_workspace(const Geom& g);
cudaError_t launch_append(const Geom& g, const void* k_new, const void* v_new, int n_new, void* ws, cudaStream_t st);

// decode attention (kvq_decode.cu)
int decode_num_splits(const Geom& g, int Hq, int num_sms);
size_t decode_workspace(const Geom& g, int Hq, int nsplit);
cudaError_t launch_decode(const Geom& g, const void* q, int Hq, float sm_scale, float* out, void* ws, int nsplit,
                          cudaStream_t st);
cudaError_t launch_decode_mma(const Geom& g, const void* q, int Hq, float scale_log2, int nsplit, float* ml,
                              float* o, int* arrivals, float* out, cudaStream_t st);
size_t decode_mma_smem(const Geom& g, int Hq);
// decode step: one-token append + decode in one launch (the workspace's counters reset themselves)
size_t step_workspace(const Geom& g, int Hq, int nsplit);
cudaError_t launch_decode_step(const Geom& g, const void* k_new, const void* v_new, const void* q, int Hq,
                               float sm_scale, float* out, void* ws, int nsplit, cudaStream_t st);
cudaError_t launch_decode_step_mma(const Geom& g, const void* k_new, const void* v_new, const void* q, int Hq,
                                   float scale_log2, int nsplit, float* ml, float* o, int* arrivals, int* seqcnt,
                                   float* out, cudaStream_t st);
int decode_mma_splits(const Geom& g, int Hq, int num_sms);

// dequantize (kvq_dequant.cu)
cudaError_t launch_dequant(const Geom& g, int seq, int start, int count, float* k_out, float* v_out,
                           cudaStream_t st);

// pattern mining (kvq_mine.cu)
struct MineArgs {
  const void* x;
  int dtype;
  int64_t n;
  int sets, heads;
  int64_t tok_stride, head_stride, set_stride;
  int P, iters, transform;
  float* patterns;
  float* colscale;
  int32_t* assign;
};
size_t mine_workspace(int64_t n, int sets, int heads, int P, int transform);

// Tiled TMA tensor map (cuTensorMapEncodeTiled through the runtime's driver entry point; loads
// past the end read as zeros).  kvq_mine.cu.
cudaError_t encode_tiled_map(CUtensorMap* map, CUtensorMapDataType dt, int rank, const void* base,
                             const cuuint64_t* dims, const cuuint64_t* strides, const cuuint32_t* box,
                             CUtensorMapSwizzle swz);

cudaError_t launch_mine(const MineArgs& a, void* ws, size_t ws_bytes, cudaStream_t st);

}  // namespace kvq
