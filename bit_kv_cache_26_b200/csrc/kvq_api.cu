// C-ABI entry points of libkvq (declared in include/kvq.h): host-side argument
// validation, workspace sizing and kernel launches.  No exception crosses the
// ABI; nothing here allocates device memory.
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "kvq_common.cuh"
#include "kvq_internal.h"

namespace {

thread_local char g_err[512] = "";

kvq_status fail(kvq_status st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return st;
}

kvq_status cuda_fail(cudaError_t e, const char* where) {
  return fail(KVQ_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

bool aligned(const void* p, size_t a) { return ((uintptr_t)p % a) == 0; }

int num_sms() {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return sms > 0 ? sms : 148;
}

kvq_status check_cache(const kvq_cache* c) {
  if (!c) return fail(KVQ_ERR_INVALID_ARG, "cache is NULL");
  if (c->head_dim != 128) return fail(KVQ_ERR_UNSUPPORTED, "head_dim %d unsupported (only 128)", c->head_dim);
  if (c->group != 32) return fail(KVQ_ERR_UNSUPPORTED, "group %d unsupported (only 32)", c->group);
  if (c->bits != 2 && c->bits != 4) return fail(KVQ_ERR_UNSUPPORTED, "bits %d unsupported (2 or 4)", c->bits);
  if (c->num_patterns < 1 || c->num_patterns > 255)
    return fail(KVQ_ERR_UNSUPPORTED, "num_patterns %d outside 1..255", c->num_patterns);
  if (c->dtype != KVQ_F16 && c->dtype != KVQ_BF16) return fail(KVQ_ERR_UNSUPPORTED, "dtype %d", c->dtype);
  if (c->transform != KVQ_TX_NONE && c->transform != KVQ_TX_HADAMARD_VARNORM)
    return fail(KVQ_ERR_UNSUPPORTED, "transform %d", c->transform);
  if (!(c->v_rho >= 0.0f) || !(c->v_rho < INFINITY))
    return fail(KVQ_ERR_INVALID_ARG, "v_rho must be finite and >= 0 (0 = adaptive threshold off)");
  if (c->reserved != 0) return fail(KVQ_ERR_INVALID_ARG, "reserved field must be 0");
  if (c->pattern_window_len < 0) return fail(KVQ_ERR_INVALID_ARG, "pattern_window_len %d < 0", c->pattern_window_len);
  if (c->pattern_window_len > 0 && (!c->pattern_counts || !c->pattern_window))
    return fail(KVQ_ERR_INVALID_ARG, "pattern insertion needs pattern_counts and pattern_window");
  if (c->num_seqs < 0 || c->num_kv_heads < 1 || c->num_sets < 1 || c->max_pages_per_seq < 0 || c->num_pages < 0)
    return fail(KVQ_ERR_INVALID_ARG, "negative or zero size in cache (seqs %d heads %d sets %d pages %d/%d)",
                c->num_seqs, c->num_kv_heads, c->num_sets, c->max_pages_per_seq, c->num_pages);
  // sequences and KV heads index the z and y dimensions of the launch grids
  if (c->num_seqs > 65535 || c->num_kv_heads > 65535)
    return fail(KVQ_ERR_CAPACITY, "%d sequences / %d KV heads exceed the 65535 the launch grids allow", c->num_seqs,
                c->num_kv_heads);
  if (c->num_seqs > 0) {
    if (!c->page_pool || !c->page_table || !c->seq_len || !c->k_tail || !c->k_patterns || !c->v_patterns ||
        !c->status)
      return fail(KVQ_ERR_INVALID_ARG, "a required cache pointer is NULL");
    if (!aligned(c->page_pool, 256)) return fail(KVQ_ERR_INVALID_ARG, "page_pool must be 256-byte aligned");
    if (!aligned(c->k_tail, 16) || !aligned(c->k_patterns, 16) || !aligned(c->v_patterns, 16))
      return fail(KVQ_ERR_INVALID_ARG, "k_tail / patterns must be 16-byte aligned");
    if (c->transform && (!c->k_colscale || !c->v_colscale))
      return fail(KVQ_ERR_INVALID_ARG, "transform enabled but colscale pointers are NULL");
  }
  return KVQ_OK;
}

}  // namespace

extern "C" {

const char* kvq_last_error(void) { return g_err; }

const char* kvq_version(void) { return "kvq 0.1 (sm_100a)"; }

float kvq_v_rho_star(int32_t head_dim, double alpha) {
  if (!(alpha > 0.0) || !(alpha < 0.5) || head_dim < 1) return 0.0f;
  // z = Phi^-1(1 - alpha) by bisection on the upper tail 0.5 erfc(z / sqrt 2)
  double lo = 0.0, hi = 40.0;
  for (int it = 0; it < 200; ++it) {
    const double mid = 0.5 * (lo + hi);
    (0.5 * erfc(mid / sqrt(2.0)) > alpha ? lo : hi) = mid;
  }
  const double z = 0.5 * (lo + hi);
  // Eq. 10 with equality, u = rho^2, k = 2 z / sqrt(5 d): (1 - k^2) u^2 - 2 u + (1 - k^2) = 0
  const double k = 2.0 * z / sqrt(5.0 * head_dim), a = 1.0 - k * k;
  if (!(a > 0.0)) return 0.0f;
  const double u = (1.0 - sqrt(1.0 - a * a)) / a;
  return (float)sqrt(u);
}

size_t kvq_subblock_bytes(int32_t bits, int32_t transform) {
  if (bits != 2 && bits != 4) return 0;
  return (size_t)kvq::subblock_bytes_of(bits, transform ? 1 : 0);
}

size_t kvq_page_bytes(const kvq_cache* c) {
  if (!c || c->num_kv_heads < 1) return 0;
  size_t s = kvq_subblock_bytes(c->bits, c->transform);
  return s * (size_t)c->num_kv_heads;
}

size_t kvq_mine_workspace_bytes(int64_t n, int32_t num_sets, int32_t num_kv_heads, int32_t P, int32_t transform) {
  if (n < 0 || num_sets < 0 || num_kv_heads < 0 || P < 1) return 0;
  return kvq::mine_workspace(n, num_sets, num_kv_heads, P, transform ? 1 : 0);
}

kvq_status kvq_mine_patterns(const void* x, int32_t dtype, int64_t n, int32_t num_sets, int32_t num_kv_heads,
                             int64_t tok_stride, int64_t head_stride, int64_t set_stride, int32_t P,
                             int32_t iters, int32_t transform, float* patterns_out, float* colscale_out,
                             int32_t* assign_out, void* ws, size_t ws_bytes, kvq_stream_t stream) {
  g_err[0] = 0;
  if (dtype != KVQ_F16 && dtype != KVQ_BF16) return fail(KVQ_ERR_UNSUPPORTED, "dtype %d", dtype);
  if (transform != KVQ_TX_NONE && transform != KVQ_TX_HADAMARD_VARNORM)
    return fail(KVQ_ERR_UNSUPPORTED, "transform %d", transform);
  if (P < 1 || P > 255) return fail(KVQ_ERR_UNSUPPORTED, "P %d outside 1..255", P);
  if (num_sets < 0 || num_kv_heads < 0 || iters < 0 || n < 0)
    return fail(KVQ_ERR_INVALID_ARG, "negative size (n %lld sets %d heads %d iters %d)", (long long)n, num_sets,
                num_kv_heads, iters);
  if (num_sets == 0 || num_kv_heads == 0) return KVQ_OK;
  if (n < P) return fail(KVQ_ERR_INVALID_ARG, "n = %lld tokens is fewer than P = %d patterns", (long long)n, P);
  if (n > (int64_t)1 << 31) return fail(KVQ_ERR_CAPACITY, "n = %lld exceeds 2^31", (long long)n);
  // (set, KV head) problems index the y / z dimension of the mining grids
  if ((int64_t)num_sets * num_kv_heads > 65535)
    return fail(KVQ_ERR_CAPACITY, "%d sets x %d KV heads exceed the 65535 problems the launch grids allow", num_sets,
                num_kv_heads);
  if (!x || !patterns_out) return fail(KVQ_ERR_INVALID_ARG, "x / patterns_out is NULL");
  if (transform && !colscale_out) return fail(KVQ_ERR_INVALID_ARG, "transform needs colscale_out");
  if (tok_stride < 0 || head_stride < 0 || set_stride < 0)
    return fail(KVQ_ERR_INVALID_ARG, "negative stride");
  if (!aligned(x, 16) || tok_stride % 8 || head_stride % 8 || set_stride % 8)
    return fail(KVQ_ERR_INVALID_ARG, "x must be 16-byte aligned and its strides multiples of 8 elements");
  size_t need = kvq::mine_workspace(n, num_sets, num_kv_heads, P, transform);
  if (ws_bytes < need || (!ws && need))
    return fail(KVQ_ERR_WORKSPACE, "mine workspace %zu < %zu bytes", ws_bytes, need);
  if (!aligned(ws, 256)) return fail(KVQ_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  if ((size_t)P * 128 * sizeof(float) > 200 * 1024) return fail(KVQ_ERR_UNSUPPORTED, "P too large");
  kvq::MineArgs a{x, dtype, n, num_sets, num_kv_heads, tok_stride, head_stride, set_stride, P, iters, transform,
                  patterns_out, colscale_out, assign_out};
  cudaError_t e = kvq::launch_mine(a, ws, ws_bytes, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "kvq_mine_patterns");
  return KVQ_OK;
}

size_t kvq_append_workspace_bytes(const kvq_cache* cache, int32_t n_new) {
  (void)n_new;
  if (!cache || cache->num_kv_heads < 1 || cache->num_sets < 1 || cache->num_patterns < 1) return 0;
  return kvq::append_workspace(kvq::make_geom(*cache));
}

kvq_status kvq_quantize_append(const kvq_cache* cache, const void* k_new, const void* v_new, int32_t n_new,
                               void* ws, size_t ws_bytes, kvq_stream_t stream) {
  g_err[0] = 0;
  kvq_status s = check_cache(cache);
  if (s != KVQ_OK) return s;
  if (n_new < 0) return fail(KVQ_ERR_INVALID_ARG, "n_new %d < 0", n_new);
  if (n_new == 0 || cache->num_seqs == 0) return KVQ_OK;
  if ((int64_t)n_new > (int64_t)cache->max_pages_per_seq * 32)
    return fail(KVQ_ERR_CAPACITY, "n_new %d exceeds the page table capacity %d", n_new,
                cache->max_pages_per_seq * 32);
  if (!k_new || !v_new) return fail(KVQ_ERR_INVALID_ARG, "k_new / v_new is NULL");
  if (!aligned(k_new, 16) || !aligned(v_new, 16)) return fail(KVQ_ERR_INVALID_ARG, "k_new / v_new must be 16-byte aligned");
  kvq::Geom g = kvq::make_geom(*cache);
  const size_t need = kvq::append_workspace(g);
  if (ws_bytes < need || !ws) return fail(KVQ_ERR_WORKSPACE, "append workspace %zu < %zu bytes", ws_bytes, need);
  if (!aligned(ws, 256)) return fail(KVQ_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  cudaError_t e = kvq::launch_append(g, k_new, v_new, n_new, ws, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "kvq_quantize_append");
  return KVQ_OK;
}

size_t kvq_decode_workspace_bytes(const kvq_cache* cache, int32_t num_q_heads) {
  if (!cache || num_q_heads < 1 || cache->num_kv_heads < 1) return 0;
  kvq::Geom g = kvq::make_geom(*cache);
  return kvq::decode_workspace(g, num_q_heads, kvq::decode_num_splits(g, num_q_heads, num_sms()));
}

kvq_status kvq_decode_attention(const kvq_cache* cache, const void* q, int32_t num_q_heads, float sm_scale,
                                float* out, void* ws, size_t ws_bytes, kvq_stream_t stream) {
  g_err[0] = 0;
  kvq_status s = check_cache(cache);
  if (s != KVQ_OK) return s;
  if (num_q_heads < 1 || num_q_heads % cache->num_kv_heads)
    return fail(KVQ_ERR_UNSUPPORTED, "num_q_heads %d is not a multiple of num_kv_heads %d", num_q_heads,
                cache->num_kv_heads);
  if (num_q_heads / cache->num_kv_heads > 16)
    return fail(KVQ_ERR_UNSUPPORTED, "more than 16 query heads per KV head");
  if (cache->num_seqs == 0) return KVQ_OK;
  if (!q || !out) return fail(KVQ_ERR_INVALID_ARG, "q / out is NULL");
  if (!aligned(q, 16) || !aligned(out, 16)) return fail(KVQ_ERR_INVALID_ARG, "q / out must be 16-byte aligned");
  if (!(sm_scale > 0.0f)) return fail(KVQ_ERR_INVALID_ARG, "sm_scale must be positive");
  kvq::Geom g = kvq::make_geom(*cache);
  int nsplit = kvq::decode_num_splits(g, num_q_heads, num_sms());
  size_t need = kvq::decode_workspace(g, num_q_heads, nsplit);
  if (ws_bytes < need || !ws) return fail(KVQ_ERR_WORKSPACE, "decode workspace %zu < %zu bytes", ws_bytes, need);
  if (!aligned(ws, 256)) return fail(KVQ_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  cudaError_t e = kvq::launch_decode(g, q, num_q_heads, sm_scale, out, ws, nsplit, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "kvq_decode_attention");
  return KVQ_OK;
}

size_t kvq_step_workspace_bytes(const kvq_cache* cache, int32_t num_q_heads) {
  if (!cache || num_q_heads < 1 || cache->num_kv_heads < 1) return 0;
  kvq::Geom g = kvq::make_geom(*cache);
  return kvq::step_workspace(g, num_q_heads, kvq::decode_num_splits(g, num_q_heads, num_sms()));
}

kvq_status kvq_decode_step(const kvq_cache* cache, const void* k_new, const void* v_new, const void* q,
                           int32_t num_q_heads, float sm_scale, float* out, void* ws, size_t ws_bytes,
                           kvq_stream_t stream) {
  g_err[0] = 0;
  kvq_status s = check_cache(cache);
  if (s != KVQ_OK) return s;
  if (num_q_heads < 1 || num_q_heads % cache->num_kv_heads)
    return fail(KVQ_ERR_UNSUPPORTED, "num_q_heads %d is not a multiple of num_kv_heads %d", num_q_heads,
                cache->num_kv_heads);
  if (num_q_heads / cache->num_kv_heads > 16)
    return fail(KVQ_ERR_UNSUPPORTED, "more than 16 query heads per KV head");
  if (cache->num_seqs == 0) return KVQ_OK;
  if (!q || !out || !k_new || !v_new) return fail(KVQ_ERR_INVALID_ARG, "q / out / k_new / v_new is NULL");
  if (!aligned(q, 16) || !aligned(out, 16) || !aligned(k_new, 16) || !aligned(v_new, 16))
    return fail(KVQ_ERR_INVALID_ARG, "q / out / k_new / v_new must be 16-byte aligned");
  if (!(sm_scale > 0.0f)) return fail(KVQ_ERR_INVALID_ARG, "sm_scale must be positive");
  if (cache->max_pages_per_seq < 1) return fail(KVQ_ERR_CAPACITY, "the page table has no column");
  kvq::Geom g = kvq::make_geom(*cache);
  const int nsplit = kvq::decode_num_splits(g, num_q_heads, num_sms());
  const size_t need = kvq::step_workspace(g, num_q_heads, nsplit);
  if (ws_bytes < need || !ws) return fail(KVQ_ERR_WORKSPACE, "step workspace %zu < %zu bytes", ws_bytes, need);
  if (!aligned(ws, 256)) return fail(KVQ_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  cudaError_t e = kvq::launch_decode_step(g, k_new, v_new, q, num_q_heads, sm_scale, out, ws, nsplit, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "kvq_decode_step");
  return KVQ_OK;
}

kvq_status kvq_dequantize(const kvq_cache* cache, int32_t seq, int32_t seq_len_host, int32_t start, int32_t count,
                          float* k_out, float* v_out, kvq_stream_t stream) {
  g_err[0] = 0;
  kvq_status s = check_cache(cache);
  if (s != KVQ_OK) return s;
  if (seq < 0 || seq >= cache->num_seqs) return fail(KVQ_ERR_INVALID_ARG, "seq %d out of range", seq);
  if (start < 0 || count < 0 || (int64_t)start + count > seq_len_host)
    return fail(KVQ_ERR_INVALID_ARG, "token range [%d, %d) outside the sequence length %d", start, start + count,
                seq_len_host);
  if ((int64_t)seq_len_host > (int64_t)cache->max_pages_per_seq * 32)
    return fail(KVQ_ERR_CAPACITY, "seq_len_host %d exceeds the page table", seq_len_host);
  if (count == 0) return KVQ_OK;
  kvq::Geom g = kvq::make_geom(*cache);
  cudaError_t e = kvq::launch_dequant(g, seq, start, count, k_out, v_out, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "kvq_dequantize");
  return KVQ_OK;
}

kvq_status kvq_mine_read_status(const void* ws, int32_t* bits_out, kvq_stream_t stream) {
  g_err[0] = 0;
  if (!ws || !bits_out) return fail(KVQ_ERR_INVALID_ARG, "NULL argument");
  cudaStream_t st = (cudaStream_t)stream;
  int32_t v = 0;
  cudaError_t e = cudaMemcpyAsync(&v, ws, sizeof(int32_t), cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail(e, "kvq_mine_read_status");
  *bits_out = v;
  if (v) return fail(KVQ_ERR_DEVICE, "mining status bits 0x%x", v);
  return KVQ_OK;
}

kvq_status kvq_read_status(const kvq_cache* cache, int32_t* bits_out, int32_t clear, kvq_stream_t stream) {
  g_err[0] = 0;
  if (!cache || !cache->status || !bits_out) return fail(KVQ_ERR_INVALID_ARG, "NULL argument");
  cudaStream_t st = (cudaStream_t)stream;
  int32_t v = 0;
  cudaError_t e = cudaMemcpyAsync(&v, cache->status, sizeof(int32_t), cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail(e, "kvq_read_status");
  if (clear) {
    e = cudaMemsetAsync(cache->status, 0, sizeof(int32_t), st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return cuda_fail(e, "kvq_read_status (clear)");
  }
  *bits_out = v;
  if (v) return fail(KVQ_ERR_DEVICE, "device status bits 0x%x", v);
  return KVQ_OK;
}

// ---- allocation-free decode: the split partials in a file-scope device array ----------
namespace {
__device__ __align__(256) uint8_t g_decode_scratch[KVQ_DECODE_STATIC_SCRATCH_BYTES];
constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_addr[kMaxDevices];  // per device, resolved on first use
}  // namespace

kvq_status kvq_decode_attention_static(const kvq_cache* cache, const void* q, int32_t num_q_heads, float sm_scale,
                                       float* out, kvq_stream_t stream) {
  g_err[0] = 0;
  kvq_status s = check_cache(cache);
  if (s != KVQ_OK) return s;
  if (num_q_heads < 1 || num_q_heads % cache->num_kv_heads)
    return fail(KVQ_ERR_UNSUPPORTED, "num_q_heads %d is not a multiple of num_kv_heads %d", num_q_heads,
                cache->num_kv_heads);
  if (num_q_heads / cache->num_kv_heads > 16)
    return fail(KVQ_ERR_UNSUPPORTED, "more than 16 query heads per KV head");
  if (cache->num_seqs == 0) return KVQ_OK;
  if (!q || !out) return fail(KVQ_ERR_INVALID_ARG, "q / out is NULL");
  if (!aligned(q, 16) || !aligned(out, 16)) return fail(KVQ_ERR_INVALID_ARG, "q / out must be 16-byte aligned");
  if (!(sm_scale > 0.0f)) return fail(KVQ_ERR_INVALID_ARG, "sm_scale must be positive");
  kvq::Geom g = kvq::make_geom(*cache);
  const int nsplit = kvq::decode_num_splits(g, num_q_heads, num_sms());
  const size_t need = kvq::decode_workspace(g, num_q_heads, nsplit);
  if (need > KVQ_DECODE_STATIC_SCRATCH_BYTES)
    return fail(KVQ_ERR_WORKSPACE, "decode partials need %zu bytes; the static scratch holds %zu", need,
                (size_t)KVQ_DECODE_STATIC_SCRATCH_BYTES);
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "kvq_decode_attention_static (cudaGetDevice)");
  if (dev < 0 || dev >= kMaxDevices) return fail(KVQ_ERR_UNSUPPORTED, "device %d beyond %d", dev, kMaxDevices);
  void* ws;
  {
    std::lock_guard<std::mutex> lk(g_scratch_mu);
    if (!g_scratch_addr[dev]) {
      e = cudaGetSymbolAddress(&g_scratch_addr[dev], g_decode_scratch);
      if (e != cudaSuccess) {
        g_scratch_addr[dev] = nullptr;
        return cuda_fail(e, "kvq_decode_attention_static (cudaGetSymbolAddress)");
      }
    }
    ws = g_scratch_addr[dev];
  }
  e = kvq::launch_decode(g, q, num_q_heads, sm_scale, out, ws, nsplit, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "kvq_decode_attention_static");
  return KVQ_OK;
}

}  // extern "C"
