/*
 * kvq.h -- C ABI of libkvq: pattern-aligned residual 2/4-bit KV-cache
 * quantization and decode attention over the quantized, paged cache, on one
 * NVIDIA B200 (sm_100a).
 *
 * Method sources (page title, section / equation):
 *   [PKV]   "PatternKV: Flattening KV Representation Expands Quantization Headroom"
 *           Section 2.1 Eq. 1 (asymmetric n-bit quantizer), Section 3.1 Eq. 4
 *           (pattern mining by k-means), Section 3.2 + Eq. 6 (min-max distance,
 *           nearest pattern, residual, index-based reconstruction), Section 3.4
 *           (fused reconstruction + attention kernels), Section 4.1 (K per channel,
 *           V per token, patterns on post-RoPE keys).
 *   [KVarN] "KVarN: Variance-Normalized KV-Cache Quantization Mitigates Error
 *           Accumulation in Reasoning Tasks", abstract (Hadamard rotation + dual-axis
 *           variance normalisation as a pre-transform).
 *
 * Conventions for every entry point
 *   - Pointers named in a struct or argument list are DEVICE pointers owned by the
 *     caller unless the comment says "host".  The library allocates no device
 *     memory: scratch space is the caller's workspace (`ws`, `ws_bytes`).
 *   - Calls are asynchronous and ordered on the caller's `stream`; arguments are
 *     validated on the host before anything is enqueued.  On a host-side error the
 *     call enqueues nothing and returns a non-zero status; kvq_last_error() then
 *     holds a message (thread-local).
 *   - Errors that only the device can see (a page id outside the pool, a sequence
 *     that would outgrow its page table, a set index outside the pattern sets) are
 *     OR-ed into the caller's device status word `cache->status` as KVQ_DEV_* bits;
 *     the offending sequence is left unchanged.  kvq_read_status() fetches it.
 *   - Supported: head_dim 128, group 32 (tokens per page = 32), bits 2 or 4,
 *     1 <= num_patterns <= 255, fp16 or bf16 inputs, query heads a multiple of the
 *     KV heads.  Other values return KVQ_ERR_UNSUPPORTED.  At most 65535 sequences and
 *     65535 KV heads per cache (launch-grid limits; more returns KVQ_ERR_CAPACITY).
 *   - Every device-side wait is bounded (a counted mbarrier.try_wait loop).  For tests of
 *     this failure path only, the environment variable KVQ_TEST_WAIT_LIMIT (read once per
 *     process) replaces the iteration limit of decode attention's page-copy waits; 0 makes
 *     every such wait expire at once.  The kernel then flags KVQ_DEV_TIMEOUT and still waits,
 *     under the normal limit, for the copies it issued before it exits.
 *
 * Cache layout in HBM
 *   A page holds 32 consecutive tokens of one sequence for every KV head.  Page p
 *   starts at page_pool + p * kvq_page_bytes(); inside it the sub-block of KV head h
 *   starts at h * kvq_subblock_bytes().  With CB = 32*128*bits/8 (1024 or 2048):
 *     [0, CB)                K codes    fragment order, rows = tokens (MT=2, KS=8)
 *     [CB, CB+512)           K scales s fp32, channel order KSC
 *     [CB+512, CB+1024)      K zeros z  fp32, channel order KSC
 *     [CB+1024, 2CB+1024)    V codes    fragment order, rows = channels (MT=8, KS=2)
 *     [2CB+1024, 2CB+1536)   V scales s fp32, (token, channel group) order VSC
 *     [2CB+1536, 2CB+2048)   V zeros z  fp32, order VZC
 *     [2CB+2048, 2CB+2080)   K pattern index per token, u8, order TOK
 *     [2CB+2080, 2CB+2112)   V pattern index per token, u8, order TOK
 *     transform only: [2CB+2112, 2CB+2240) K row factors, [2CB+2240, 2CB+2368) V row
 *     factors, fp32, order TOK.
 *   Sub-block size: 4160 B (2-bit) / 6208 B (4-bit), +256 B with the transform;
 *   that is 130 / 194 / 138 bytes per token and KV head.
 *
 *   Fragment order of a (16*MT) x (16*KS) code matrix X (K: X[token][channel];
 *   V: X[channel][token]): element (row, col) belongs to
 *       lane = ((row % 16) % 8) * 4 + ((col % 16) % 8) / 2,   odd = col % 2,
 *       reg  = ((row / 16) * KS + col / 16) * 4 + (row % 16) / 8 + 2 * ((col % 16) / 8)
 *   and to the lane's word w = reg/8 at bit 2*(reg%8) + 16*odd (2-bit), or w = reg/4 at
 *   bit 4*(reg%4) + 16*odd (4-bit).  A lane's words are stored in 16-byte chunks that
 *   interleave the lanes: word w of lane l is the little-endian 32-bit word number
 *       (w / 4) * 128 + l * 4 + (w % 4)
 *   of the code block.  (The register order of the A operand of a 16x8x16 tensor-core
 *   MMA: each lane reads its operands with conflict-free 16-byte loads.)
 *   Orders of the per-channel / per-token fields (i = position in the field):
 *       KSC: i = ks*16 + tig*4 + e            -> channel 16*ks + 2*tig + (e&1) + 8*(e>>1)
 *       VSC: i = ((ks*4 + e)*4 + tig)*4 + grp -> token 16*ks + 2*tig + (e&1) + 8*(e>>1),
 *                                                channel group grp (channels 32*grp..32*grp+31)
 *       VZC: i = (j*8 + g)*4 + grp            -> token g + 8*j, channel group grp
 *       TOK: i = g*4 + j                      -> token g + 8*j
 *   Entries of tokens not yet appended are zero.  The K part of a page (codes,
 *   scales, indices, row factors) is written when its 32nd token arrives; until
 *   then those tokens' keys live unquantized in the K tail.
 *
 *   K tail: k_tail[seq][kv_head][slot][128] in the input dtype; token t of the
 *   newest, incomplete group is in slot t % 32.
 *
 * Numerics (what the kernels compute; identical to the CPU oracle's contract)
 *   - Alignment, residual and quantization are fp32 operations in a fixed order:
 *       r_jd = fl32(x_d - M_jd),  d_j = fl32(max_d r_jd - min_d r_jd),
 *       k* = lowest j with minimal d_j,  R = r_{k*},
 *       per group: s = fl32(fl32(max R - min R) / (2^bits - 1)), z = min R,
 *       q = s == 0 ? 0 : clamp(rne(fl32(fl32(R - z) / s)), 0, 2^bits - 1).
 *     Indices and codes are therefore reproducible bit for bit.
 *   - V groups: 4 groups of 32 channels per token.  K groups: per channel, the
 *     32 tokens of a page.
 *   - Reconstruction: x_hat = s*q + z + M_{k*}; with the transform, x = r * (y (.) c) H / 128.
 *   - Pre-transform (KVARN): x' = x H (unnormalised Sylvester Walsh-Hadamard, fp32
 *     butterfly with strides 1..64); u = fl32(x'/c); r = population std of u in fp32
 *     (halving sums); y = fl32(u / r) (r = 1 when the std is 0).  c is fitted per
 *     (set, head) on the prefill by 3 alternating row / column std passes in float64 (the
 *     GPU recomputes each row per pass instead of storing it, a few ulps from the sequential
 *     divisions, and gives the same c on every run).
 *   - Mining: Lloyd k-means, strided initialisation M_j = x[floor(j*n/P)], float64
 *     squared distances (lowest index on ties), centroid = fl32(float64 mean),
 *     empty clusters keep their pattern.
 *   - V adaptive threshold (cache->v_rho > 0): with v the (pre-transformed) V vector and
 *     M* its nearest pattern, R_flat = d_mm(v, M*), R_raw = fl32(max v - min v); the
 *     pattern is used iff R_flat <= fl32(v_rho * R_raw), else index 255 and R = v.
 */
#ifndef KVQ_H
#define KVQ_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define KVQ_API __attribute__((visibility("default")))
#else
#define KVQ_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* kvq_stream_t; /* a cudaStream_t; NULL = legacy default stream */

typedef enum {
  KVQ_OK = 0,
  KVQ_ERR_INVALID_ARG = 1,   /* null pointer, negative size, misaligned pointer */
  KVQ_ERR_UNSUPPORTED = 2,   /* a shape or mode this build does not implement */
  KVQ_ERR_CAPACITY = 3,      /* a size exceeds what the cache or a limit allows */
  KVQ_ERR_WORKSPACE = 4,     /* ws_bytes smaller than the matching kvq_*_workspace_bytes() */
  KVQ_ERR_CUDA = 5,          /* a CUDA runtime call failed (message in kvq_last_error) */
  KVQ_ERR_DEVICE = 6         /* kvq_read_status found device-side error bits */
} kvq_status;

/* Device status bits OR-ed into cache->status. */
#define KVQ_DEV_BAD_PAGE 0x1   /* page_table entry outside [0, num_pages) */
#define KVQ_DEV_OVERFLOW 0x2   /* seq_len + n_new > max_pages_per_seq * 32 */
#define KVQ_DEV_BAD_SET 0x4    /* seq_to_set entry outside [0, num_sets) */
#define KVQ_DEV_TIMEOUT 0x8    /* a bounded wait for a page copy expired; that step's output is invalid */
#define KVQ_DEV_RANGE 0x10     /* decode: |q_d * s_d| or a V scale exceeded the fp16 operand range (~3e4) */

typedef enum { KVQ_F16 = 0, KVQ_BF16 = 1 } kvq_dtype;
typedef enum { KVQ_TX_NONE = 0, KVQ_TX_HADAMARD_VARNORM = 1 } kvq_transform;

/*
 * The paged cache.  All pointers are device pointers owned by the caller; the
 * library reads and writes through them but never frees or reallocates them.
 */
typedef struct kvq_cache {
  int32_t num_seqs;           /* sequences sharing this cache */
  int32_t num_kv_heads;       /* KV heads (each page stores all of them) */
  int32_t head_dim;           /* must be 128 */
  int32_t group;              /* must be 32: tokens per K group = tokens per page; channels per V group */
  int32_t bits;               /* 2 or 4 */
  int32_t num_patterns;       /* P, 1..255 */
  int32_t num_sets;           /* pattern sets (1 = one set per KV head shared by all sequences) */
  int32_t max_pages_per_seq;  /* columns of page_table */
  int32_t num_pages;          /* pages in page_pool */
  int32_t dtype;              /* kvq_dtype of K/V/q inputs and of k_tail */
  int32_t transform;          /* kvq_transform */
  float v_rho;                /* V adaptive threshold rho* ([PKV] Section 3.3, Eq. 7-10): a V vector
                                 keeps its pattern iff d_mm(v, M*) <= fl32(v_rho * (max v - min v)),
                                 else it is quantized raw and stores index 255.  0 = off (always use
                                 the pattern).  kvq_v_rho_star() gives the value for (d, alpha). */
  void* page_pool;            /* num_pages * kvq_page_bytes() bytes, 256-byte aligned */
  const int32_t* page_table;  /* [num_seqs][max_pages_per_seq] physical page ids */
  int32_t* seq_len;           /* [num_seqs] tokens held per sequence (updated by append) */
  void* k_tail;               /* [num_seqs][num_kv_heads][32][128] dtype */
  const float* k_patterns;    /* [num_sets][num_kv_heads][P][128] fp32 (kvq_decode_step with pattern insertion
                                 writes rows pattern_counts[..] .. P - 1; nothing else writes them) */
  const float* v_patterns;    /* [num_sets][num_kv_heads][P][128] fp32 (same) */
  const int32_t* seq_to_set;  /* [num_seqs] pattern set of each sequence, or NULL (all set 0) */
  const float* k_colscale;    /* [num_sets][num_kv_heads][128] fp32; transform only, else NULL */
  const float* v_colscale;    /* [num_sets][num_kv_heads][128] fp32; transform only, else NULL */
  int32_t* status;            /* one int32, device-side error bits (KVQ_DEV_*); caller zeroes it */
  /* Decode-time pattern insertion ([PKV] Section 3.1 "Decoding Stage", Eq. 5); all optional. */
  int32_t* pattern_counts;    /* [num_sets][num_kv_heads] patterns in use per set, 1..num_patterns (the rest
                                 of the P rows are capacity), or NULL: every set uses num_patterns */
  float* pattern_window;      /* [num_seqs][num_kv_heads][4][128] fp32: running minimum and maximum of the K
                                 vectors, then of the V vectors, of the current window; the caller sets them to
                                 +inf / -inf before the first step.  NULL unless pattern_window_len > 0 */
  int32_t pattern_window_len; /* G_pattern: each time a sequence's length reaches a multiple of it during
                                 kvq_decode_step, the window's Chebyshev centers fl32(fl32(min + max) * 0.5)
                                 become the next K and V pattern of the sequence's set (while its count is
                                 below num_patterns) and the window restarts.  0 = off.  Needs
                                 pattern_counts, and sequences that do not share a pattern set. */
  int32_t reserved;           /* must be 0 */
} kvq_cache;

/* rho*(d, alpha) of [PKV] Eq. 10 rounded to fp32: the root in (0, 1) of
 * 1 - rho^2 = 2 z_{1-alpha} / sqrt(5 d) * sqrt(1 + rho^4) (closed form of the quadratic in
 * rho^2), z the standard normal quantile.  Host only; 0 for alpha <= 0 (threshold off) or
 * arguments without a root (d < 1, alpha >= 0.5). */
KVQ_API float kvq_v_rho_star(int32_t head_dim, double alpha);

/* Bytes of one page (all KV heads) and of one KV head's sub-block.  Host only; 0 if unsupported. */
KVQ_API size_t kvq_page_bytes(const kvq_cache* cache);
KVQ_API size_t kvq_subblock_bytes(int32_t bits, int32_t transform);

/*
 * kvq_mine_patterns -- prefill pattern mining ([PKV] Section 3.1, Eq. 4; Section 3.4
 * "fully GPU-parallel KMeans"), optionally after fitting the [KVarN] pre-transform.
 *
 * For every set s < num_sets and KV head h < num_kv_heads independently, the n
 * vectors x(s, i, h) at  x + s*set_stride + i*tok_stride + h*head_stride  (element
 * strides, multiples of 8; x 16-byte aligned; 128 contiguous elements each, dtype
 * fp16/bf16) are clustered into P
 * patterns with `iters` Lloyd iterations.  With transform = KVQ_TX_HADAMARD_VARNORM
 * the column factors are fitted first and written to colscale_out, and the
 * clustering runs on the normalised vectors y.
 *   patterns_out  [num_sets][num_kv_heads][P][128] fp32
 *   colscale_out  [num_sets][num_kv_heads][128] fp32 (transform only, else NULL)
 *   assign_out    [num_sets][num_kv_heads][n] int32, optional (NULL): the Euclidean
 *                 assignment of the last iteration (made against the patterns that
 *                 iteration started from)
 * Requires n >= P and num_sets * num_kv_heads <= 65535 (else KVQ_ERR_CAPACITY).
 * Workspace: kvq_mine_workspace_bytes(), 256-byte aligned.  Its first 4 bytes are the call's
 * device status word: the call zeroes it when it starts, and a mining kernel whose bounded
 * wait expired ORs KVQ_DEV_TIMEOUT into it (that call's patterns are then unreliable);
 * kvq_mine_read_status() fetches it.
 */
KVQ_API size_t kvq_mine_workspace_bytes(int64_t n, int32_t num_sets, int32_t num_kv_heads, int32_t P,
                                int32_t transform);
KVQ_API kvq_status kvq_mine_patterns(const void* x, int32_t dtype, int64_t n, int32_t num_sets, int32_t num_kv_heads,
                             int64_t tok_stride, int64_t head_stride, int64_t set_stride, int32_t P,
                             int32_t iters, int32_t transform, float* patterns_out, float* colscale_out,
                             int32_t* assign_out, void* ws, size_t ws_bytes, kvq_stream_t stream);

/* Synchronise `stream` and copy the status word of the mining call that used workspace `ws`
 * (device pointer) to *bits_out (host).  Returns KVQ_ERR_DEVICE if any bit is set, else KVQ_OK. */
KVQ_API kvq_status kvq_mine_read_status(const void* ws, int32_t* bits_out, kvq_stream_t stream);

/*
 * kvq_quantize_append -- append n_new tokens to every sequence ([PKV] Section 3.2:
 * align each vector to its nearest pattern under the min-max distance, quantize
 * only the residual; Eq. 1; Section 4.1 granularity).
 *   k_new, v_new  [num_seqs][n_new][num_kv_heads][128] dtype
 * V is quantized per token at once.  K tokens join the K tail; every K group that
 * reaches 32 tokens is quantized per channel and written to its page.  seq_len is
 * advanced by n_new (a sequence that would overflow its page table is left
 * unchanged and flags KVQ_DEV_OVERFLOW).  n_new = 0 is a no-op.
 * Workspace: kvq_append_workspace_bytes() (per-call pattern tables: the 32 channels whose
 * values differ most across the patterns and every pattern's values there, used to prune
 * the exact assignment; 128 + 128 P bytes per (set, KV head) and K / V); 256-byte aligned.
 */
KVQ_API size_t kvq_append_workspace_bytes(const kvq_cache* cache, int32_t n_new);
KVQ_API kvq_status kvq_quantize_append(const kvq_cache* cache, const void* k_new, const void* v_new, int32_t n_new,
                               void* ws, size_t ws_bytes, kvq_stream_t stream);

/*
 * kvq_decode_attention -- one decode step of attention over the quantized cache
 * ([PKV] Section 3.4: pattern-index restoration, dequantization and the QK^T and
 * P.V products fused into the attention kernels).
 *   q    [num_seqs][num_q_heads][128] dtype; query head hq reads KV head hq / (num_q_heads / num_kv_heads)
 *   out  [num_seqs][num_q_heads][128] fp32 = softmax(sm_scale * q . K_hat^T) V_hat over
 *        every token of the sequence: reconstructed keys of complete groups, the exact
 *        keys of the K tail, reconstructed values of all tokens.  A sequence with no
 *        tokens gets zeros.
 * Split-K over the token axis; partial results go to the workspace
 * (kvq_decode_workspace_bytes()).  The environment variable KVQ_DECODE_CFG (read per call,
 * 0..3) selects the kernel's pipeline form, (ring stages per warp, warps per CTA) =
 * (3, 4), (2, 4), (2, 8), (3, 8); the default 1 measured fastest on one B200.  The forms
 * merge their per-warp partials in different orders, so outputs agree to rounding.
 */
KVQ_API size_t kvq_decode_workspace_bytes(const kvq_cache* cache, int32_t num_q_heads);
KVQ_API kvq_status kvq_decode_attention(const kvq_cache* cache, const void* q, int32_t num_q_heads, float sm_scale,
                                float* out, void* ws, size_t ws_bytes, kvq_stream_t stream);

/*
 * kvq_decode_attention_static -- kvq_decode_attention without a caller workspace.
 * This entry point has no counterpart in the method's description.  It is for callers
 * that cannot hand the library a scratch buffer: a runtime whose device memory is
 * partitioned up front with no pool left over for per-call scratch, or code that must
 * not call back into its framework's allocator at this point.  It allocates nothing.
 *   Same arguments, layout and result as kvq_decode_attention, minus ws / ws_bytes.
 *   The split partials live in one file-scope device array of
 *   KVQ_DECODE_STATIC_SCRATCH_BYTES (16 MiB) per device, shared by every call on that
 *   device.  Calls whose partials need more (kvq_decode_workspace_bytes() larger than
 *   the array) return KVQ_ERR_WORKSPACE before launching anything.
 *   Overlapping calls race: two calls in flight at once on one device (different
 *   streams, or different host threads) write the same array and corrupt each other's
 *   results.  Calls issued to one stream run one after another and are safe.
 *   The first call on each device resolves the array's address (cudaGetSymbolAddress,
 *   once per device, under a lock); make that first call before any stream capture is
 *   started on that device.
 */
#define KVQ_DECODE_STATIC_SCRATCH_BYTES ((size_t)16 << 20)
KVQ_API kvq_status kvq_decode_attention_static(const kvq_cache* cache, const void* q, int32_t num_q_heads,
                                               float sm_scale, float* out, kvq_stream_t stream);

/*
 * kvq_decode_step -- one step of decoding in a single launch: kvq_quantize_append of one new
 * token per sequence (n_new = 1) followed by kvq_decode_attention over every token including it
 * ([PKV] Section 3.4: the fused decode kernels; Section 3.2 / Eq. 6 and Eq. 1 for the append;
 * Section 3.3 for V).  With cache->pattern_window_len > 0 the step also runs the decode-time
 * pattern insertion of [PKV] Section 3.1, Eq. 5 (see kvq_cache).
 *   k_new, v_new  [num_seqs][num_kv_heads][128] dtype: the new token's key and value
 *   q             [num_seqs][num_q_heads][128] dtype;  out [num_seqs][num_q_heads][128] fp32
 * Same results (page bytes, K tail, seq_len, out) as the two calls in a row.  The new key and
 * value are assigned among the patterns in use (a brute-force exact min-max argmin: one token per
 * sequence and head); when the token completes a page, the page's 32 keys are assigned and
 * quantized in the same launch.  A sequence whose page table is full, or whose next page id is
 * invalid, flags KVQ_DEV_OVERFLOW / KVQ_DEV_BAD_PAGE, appends nothing and is decoded as it was.
 * Workspace: kvq_step_workspace_bytes(), 256-byte aligned, ZERO-FILLED before its first use:
 * besides the split partials it holds counters that every call leaves at zero again (no memset
 * per step, so a step can be captured in a CUDA graph as one kernel node).  Two steps in flight
 * at once on one workspace race.
 */
KVQ_API size_t kvq_step_workspace_bytes(const kvq_cache* cache, int32_t num_q_heads);
KVQ_API kvq_status kvq_decode_step(const kvq_cache* cache, const void* k_new, const void* v_new, const void* q,
                                   int32_t num_q_heads, float sm_scale, float* out, void* ws, size_t ws_bytes,
                                   kvq_stream_t stream);

/*
 * kvq_dequantize -- reconstruct tokens [start, start+count) of sequence `seq`
 * ([PKV] Section 3.2: pattern by index + dequantized residual; Eq. 1 inverted),
 * in the original space (the pre-transform is undone).
 *   k_out, v_out  [count][num_kv_heads][128] fp32 (either may be NULL)
 * Keys of tokens still in the K tail are copied exactly.  Requires
 * 0 <= start, start + count <= the sequence's length, which the caller asserts
 * through `seq_len_host` (the host-side copy of seq_len[seq]).
 */
KVQ_API kvq_status kvq_dequantize(const kvq_cache* cache, int32_t seq, int32_t seq_len_host, int32_t start, int32_t count,
                          float* k_out, float* v_out, kvq_stream_t stream);

/* Synchronise `stream`, copy cache->status to *bits_out (host), optionally clear it.
 * Returns KVQ_ERR_DEVICE if any bit is set, else KVQ_OK. */
KVQ_API kvq_status kvq_read_status(const kvq_cache* cache, int32_t* bits_out, int32_t clear, kvq_stream_t stream);

/* Message of the last failed call on this thread ("" if none). */
KVQ_API const char* kvq_last_error(void);

/* Library version string. */
KVQ_API const char* kvq_version(void);

#ifdef __cplusplus
}
#endif
#endif /* KVQ_H */
