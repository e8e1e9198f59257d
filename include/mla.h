/*
 * mla.h — C ABI of the B200 (sm_100a) Multi-head Latent Attention decode path.
 *
 * One MLA attention layer of DeepSeek-V2, in the absorbed inference form:
 *   c^KV_t = W^DKV h_t                       (eq 9)
 *   k^R_t  = RoPE_t(W^KR h_t)                (decoupled RoPE key, taken from h_t)
 *   c^Q_t  = W^DQ h_t  (or h_t, no compression)   (eq 12)
 *   q^C_t  = W^UQ c^Q_t                      (eq 13)
 *   q^R_t  = RoPE_t(W^QR c^Q_t), per head
 *   q_lat_{t,i} = (W^UK_i)^T q^C_{t,i}       (W^UK absorbed into the query)
 *   s_j    = scale (q_lat_i . c^KV_j + q^R_i . k^R_j),  scale = factor / sqrt(d_h + d_h^R)
 *   o_lat_i = sum_j softmax_j(s) c^KV_j      (eq 7 over the latent cache)
 *   u_t    = W^O [W^UV_1 o_lat_1; ...; W^UV_nh o_lat_nh]   (eqs 8, 11; W^UV absorbed)
 * Equations (1)-(13) as printed in the "DeepSeek-V2" reading notes
 * (irregular6612.github.io), sections 2.1.1-2.1.2; the decoupled RoPE, the
 * concatenated query/key and the absorption of W^UK and W^UV follow the
 * DeepSeek-V2 explainer (adg.csdn.net), section 2.2.2; the cached row
 * [c^KV ; k^R] of d_c + d_h^R values per token, shared by every head, is the
 * explainer's section 2.2.2 cache formula.
 *
 * Conventions (all calls):
 *  - Every tensor argument is a DEVICE pointer owned by the caller; structs
 *    (mla_layer_desc, mla_weights, mla_paged_cache) live in HOST memory and
 *    hold device pointers.  The library never allocates or frees device
 *    memory at call time; scratch comes from the caller's `ws` of at least
 *    mla_workspace_size() bytes (256-byte aligned).  The one exception is
 *    mla_decode_attn_noalloc, whose scratch is a fixed 32 MiB array that the
 *    library holds on every device that loads it.
 *  - Row-major layouts.  Weights are [out, in] (the y = W x convention).
 *    Element type is float for MLA_F32 layers and bfloat16 for MLA_BF16
 *    layers, except where a float type is written out (lse, u).
 *  - Calls are asynchronous on `stream` (a cudaStream_t passed as void*).
 *    Host-detectable errors return immediately and launch nothing.  Kernels
 *    that detect a bad page id or give up a bounded wait record it in a
 *    device error word read by mla_get_last_error().
 *  - There is no CPU fallback and no dispatch to other devices: a shape the
 *    kernels do not support returns MLA_ERR_UNSUPPORTED.
 *  - Results are deterministic for fixed arguments (no atomics in reductions).
 *  - bf16 kernels launch with programmatic stream serialisation: each may
 *    start (set-up, L2 prefetch of weights) while the previous kernel on the
 *    stream is finishing, but reads no buffer and writes nothing before that
 *    kernel has completed, so any stream-ordered producer of an argument —
 *    weights included — is safe.
 *
 * Supported shapes.
 *  MLA_F32 (exact fp32 SIMT kernels): d_hr even, block_size >= 1, any d, n_h,
 *    d_h, d_c, d_cq.
 *  MLA_BF16 (tcgen05 tensor-core kernels): block_size == 64, d_c == 512,
 *    d_hr == 64, d_h % 64 == 0, d % 64 == 0, d_cq % 64 == 0, n_h in {16, 32,
 *    64, 128}.
 *  MLA_CACHE_FP8_E4M3: MLA_BF16 layers; the latent attention
 *    (mla_decode_attn, mla_decode_attn_noalloc, mla_decode_attn_partial,
 *    mla_prefill_attn) reads FP8 rows at every supported n_h (128-head
 *    layers on CTA pairs, as with native rows); the un-absorbed prefill
 *    returns MLA_ERR_UNSUPPORTED.
 */
#ifndef MLA_H
#define MLA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MLA_OK = 0,
  MLA_ERR_INVALID_ARG = 1,     /* null pointer, non-positive size, bad desc field */
  MLA_ERR_UNSUPPORTED = 2,     /* valid but not implemented (shape / dtype) */
  MLA_ERR_CAPACITY = 3,        /* workspace too small, page id out of range */
  MLA_ERR_CUDA = 4,            /* a CUDA runtime call failed */
  MLA_ERR_DEVICE_TIMEOUT = 5   /* a kernel gave up a bounded wait */
} mla_status_t;

typedef enum { MLA_F32 = 0, MLA_BF16 = 1 } mla_dtype_t;

/* Storage of the latent cache rows (mla_layer_desc.cache_dtype). */
typedef enum {
  MLA_CACHE_NATIVE = 0,   /* [c^KV | k^R] in the layer's element type */
  MLA_CACHE_FP8_E4M3 = 1  /* FP8 rows, MLA_BF16 layers only (see mla_paged_cache) */
} mla_cache_dtype_t;

/* Layer description, in the pages' notation. */
typedef struct {
  int d;            /* model width (input h_t has d values) */
  int n_h;          /* attention heads */
  int d_h;          /* per-head dimension of q^C, k^C, v^C */
  int d_c;          /* KV latent dimension (c^KV) */
  int d_cq;         /* query latent dimension d_c'; 0 = queries read h directly */
  int d_hr;         /* decoupled RoPE dimension d_h^R (q^R per head, shared k^R) */
  int block_size;   /* tokens per cache page */
  mla_dtype_t dtype;
  double rope_base;          /* theta_k = rope_base^(-2k/d_hr) */
  double yarn_scale;         /* s; 1 = plain RoPE */
  int yarn_orig_ctx;         /* original context window of the YaRN blend */
  double yarn_alpha, yarn_beta;
  double attn_logit_factor;  /* multiplies every logit; 1 when YaRN is off */
  /* RMSNorm after the compressed latents and a scale factor at each of these
   * width bottlenecks (DeepSeek-V2 explainer, section 3.1.1):
   *   c^KV <- scale_kv * g_kv * c^KV / sqrt(mean(c^KV^2) + norm_eps), before it is cached
   *   c^Q  <- scale_q  * g_q  * c^Q  / sqrt(mean(c^Q^2)  + norm_eps), before W^UQ, W^QR
   * (c^Q only when d_cq > 0).  0 = off: the other three fields are ignored. */
  int latent_norm;
  double norm_eps;           /* >= 0 */
  double scale_kv, scale_q;  /* > 0 */
  /* mla_cache_dtype_t.  The KV cache is quantised for serving (DeepSeek-V2
   * explainer, section 3.1.4); MLA_CACHE_FP8_E4M3 stores c^KV as FP8 codes
   * with one power-of-two scale per row and keeps k^R in bf16. */
  int cache_dtype;
} mla_layer_desc;

/* Projection matrices, [out, in] row-major, element type = desc.dtype.
 *   w_dkv [d_c, d]            w_kr [d_hr, d]          w_dq [d_cq, d] (NULL if d_cq == 0)
 *   w_uq  [n_h*d_h, q_in]     w_qr [n_h*d_hr, q_in]   (q_in = d_cq, or d when d_cq == 0)
 *   w_uk  [n_h*d_h, d_c]      w_uv [n_h*d_h, d_c]     (head i = rows i*d_h .. i*d_h+d_h-1)
 *   w_o   [d, n_h*d_h]
 *   g_kv  [d_c], g_q [d_cq]   RMSNorm gains of the latents (read only when
 *                             desc.latent_norm; g_q only when d_cq > 0)        */
typedef struct {
  const void *w_dkv, *w_kr, *w_dq, *w_uq, *w_qr, *w_uk, *w_uv, *w_o;
  const void *g_kv, *g_q;
} mla_weights;

/* Paged latent cache: pool [num_blocks, block_size, row]; token j of
 * sequence b lives at pool[block_table[b*max_blocks + j/block_size]][j % block_size].
 * Slots that no sequence has written may hold any bits (NaN included): the
 * attention kernels never let them reach a result.
 * Row (mla_cache_row_bytes bytes):
 *   MLA_CACHE_NATIVE    [c^KV (d_c) | k^R (d_hr)] in the layer's element type
 *   MLA_CACHE_FP8_E4M3  bytes [0, d_c)               E4M3 codes q of c^KV
 *                       bytes [d_c, d_c + 2 d_hr)    k^R, bf16
 *                       bytes [d_c + 2 d_hr, +4)     fp32 scale 2^e
 *                       zero padding to a multiple of 16 bytes (656 bytes at
 *                       d_c = 512, d_hr = 64)
 *     c^KV = q * 2^e, E4M3 = OCP 8-bit float (sign, 4 exponent bits with bias
 *     7, 3 mantissa bits, subnormals, largest finite 448); e is the smallest
 *     integer with max|c^KV| <= 448 * 2^e, codes are rounded to nearest even
 *     and saturated.  The attention multiplies with c^KV = q * 2^e exactly. */
typedef struct {
  void* pool;
  int num_blocks;
  const int32_t* block_table;  /* [B, max_blocks] int32 */
  int max_blocks;
} mla_paged_cache;

/* Bytes of one cache row of this layer (0 for an invalid desc). */
size_t mla_cache_row_bytes(const mla_layer_desc* desc);

/* Encode n bf16 cache rows [n, d_c + d_hr] (e.g. a whole pool of
 * num_blocks * block_size rows) as FP8 rows [n, mla_cache_row_bytes] in the
 * format above; desc.cache_dtype must be MLA_CACHE_FP8_E4M3.  A NaN element
 * (an unwritten slot) becomes a NaN code and is left out of its row's
 * maximum.  src and dst must not overlap. */
mla_status_t mla_cache_quantize(const mla_layer_desc* desc, const void* src, long long n, void* dst, void* stream);

/* Bytes of scratch that every call below needs for T tokens per projection
 * call and B sequences of at most max_kv_len cached tokens per attention call
 * (prefill: B sequences x q_per_seq queries count as B*q_per_seq rows). */
size_t mla_workspace_size(const mla_layer_desc* desc, int T, int B, int max_kv_len);

/* Compress and append T new tokens (eq 9 + decoupled RoPE key).
 *   h       [T, d]        hidden states
 *   seq_idx [T] int32     sequence of each token (row of block_table)
 *   pos     [T] int32     position of each token; its page must already be
 *                         in block_table (pos / block_size < max_blocks)
 * Writes cache->pool rows [c^KV (d_c) | RoPE_pos(W^KR h) (d_hr)] (FP8 rows:
 * the E4M3 codes of c^KV with the row's scale, see mla_paged_cache).
 * A page id outside [0, num_blocks) sets MLA_ERR_CAPACITY in the device error
 * word and the row is skipped.  Workspace: mla_workspace_size(desc, T, 0, 0)
 * (used with the latent norm or FP8 rows). */
mla_status_t mla_compress_append(const mla_layer_desc* desc, const mla_weights* w,
                                 const void* h, const int32_t* seq_idx, const int32_t* pos, int T,
                                 mla_paged_cache* cache, void* ws, size_t ws_bytes, void* stream);

/* Absorbed queries of T tokens (eqs 12-13, decoupled RoPE query, W^UK folded in).
 *   h      [T, d]; pos [T] int32
 *   q_lat  [T, n_h, d_c]   out: (W^UK_i)^T W^UQ_i c^Q
 *   q_rope [T, n_h, d_hr]  out: RoPE_pos(W^QR_i c^Q)                      */
mla_status_t mla_absorb_q(const mla_layer_desc* desc, const mla_weights* w,
                          const void* h, const int32_t* pos, int T,
                          void* q_lat, void* q_rope, void* ws, size_t ws_bytes, void* stream);

/* mla_compress_append then mla_absorb_q of the same T tokens in one call (same
 * arguments, results and scratch bound as the two calls).  With query
 * compression (d_cq > 0) the projections of h by W^DKV, W^KR and W^DQ share
 * one GEMM launch, so the weights of both steps stream in a single pass. */
mla_status_t mla_compress_append_absorb_q(const mla_layer_desc* desc, const mla_weights* w, const void* h,
                                          const int32_t* seq_idx, const int32_t* pos, int T,
                                          mla_paged_cache* cache, void* q_lat, void* q_rope, void* ws,
                                          size_t ws_bytes, void* stream);

/* Decode attention over the latent cache, one query per sequence.
 *   q_lat [B, n_h, d_c], q_rope [B, n_h, d_hr]
 *   kv_len [B] int32     rows attended by sequence b (including the token just
 *                        appended), 1 <= kv_len[b] <= max_blocks*block_size
 *   num_splits           how the KV rows are cut into work units:
 *                        0 = automatic: the 128-row tiles of all sequences,
 *                        in sequence order, are dealt to one wave of CTAs
 *                        (CTA pairs for 128 heads) as equal contiguous
 *                        ranges, so a sequence is cut wherever a range
 *                        boundary falls inside it; S > 0 = every sequence
 *                        cut into min(S, its tiles) parts, one per CTA.
 *                        Cut sequences are merged by a log-sum-exp combine.
 *                        1 needs no workspace.
 *   o_lat [B, n_h, d_c]  out: softmax-weighted sum of c^KV (desc dtype)
 *   lse   [B, n_h] float out (may be NULL): natural-log sum of exp(s_j)      */
mla_status_t mla_decode_attn(const mla_layer_desc* desc, const void* q_lat, const void* q_rope,
                             const mla_paged_cache* cache, const int32_t* kv_len, int B,
                             void* ws, size_t ws_bytes, int num_splits,
                             void* o_lat, float* lse, void* stream);

/* mla_decode_attn without a caller workspace (the pages have no counterpart:
 * this is a deployment variant, not part of the method).
 * For callers that cannot allocate device memory at call time — code running
 * inside a region that forbids allocation (a captured or replayed command
 * stream, a real-time serving loop whose memory was fixed at start-up, a
 * plug-in that may not touch the host framework's allocator) and that has no
 * spare buffer to lend as workspace.
 * Same arguments and results as mla_decode_attn, minus the workspace.  The
 * work-unit list and split partials live in a library-owned device array of
 * 32 MiB (every device that loads the library holds it until the process
 * exits); with num_splits == 0 the automatic plan is made for the largest
 * number of CTAs (CTA pairs) whose unit list and partials fit (63 pairs
 * instead of 74 for 128 heads at batch 64), an explicit num_splits whose
 * unit list and partials need
 * more than 32 MiB (about num_splits * B * (n_h * 2052 + 16) bytes, bf16
 * layers) returns MLA_ERR_CAPACITY,
 * as does an fp32 layer whose score scratch (B * n_h * max_blocks *
 * block_size * 4 bytes) exceeds it.  No device memory is allocated or freed.
 * The first call on a device looks up the array's address on that device (a
 * host-side runtime query): make that first call before any stream capture.
 * All calls share the one array and every partial is written before it is
 * read, so nothing needs clearing; calls that may run concurrently on the
 * GPU (different streams, or two devices' work racing on one device) race on
 * it and must be serialised by the caller. */
mla_status_t mla_decode_attn_noalloc(const mla_layer_desc* desc, const void* q_lat, const void* q_rope,
                                     const mla_paged_cache* cache, const int32_t* kv_len, int B, int num_splits,
                                     void* o_lat, float* lse, void* stream);

/* Context parallelism for long decodes (the pages' 128K-context setting, DeepSeek-V2
 * explainer section 3.1.3): the pages of one sequence are spread over R GPUs,
 * each attends to the rows it holds, and the ranks' results are merged by
 * log-sum-exp after one exchange of n_h * (d_c + 1) floats per sequence.
 *
 * mla_decode_attn_partial: decode attention over rows [kv_begin[b], kv_end[b])
 * of each sequence only (the rows this GPU holds; pages outside the range are
 * never read, so block_table may leave them unset).
 *   kv_begin [B] int32   a multiple of 128 (0 <= kv_begin <= kv_end); a bad
 *                        value empties the row and sets MLA_ERR_CAPACITY in
 *                        the device error word
 *   kv_end   [B] int32   <= max_blocks * block_size; kv_end == kv_begin is an
 *                        empty range: o_part = 0, lse_part = -inf
 *   o_part   [B, n_h, d_c] float  out: softmax-weighted sum of c^KV over the range
 *   lse_part [B, n_h] float       out: log sum over the range of exp(s_j)
 * Workspace: mla_workspace_size(desc, 0, B, max kv_end).  bf16 layers only
 * (MLA_ERR_UNSUPPORTED for MLA_F32).
 *
 * mla_lse_merge: merges R partials of the same B rows,
 *   lse = log sum_r exp(lse_r),  o = sum_r exp(lse_r - lse) o_r   (lse_r = -inf: weight 0)
 *   o_parts [R, B, n_h, d_c] float, lse_parts [R, B, n_h] float (rank-major, as an
 *   all-gather lays them out); o_lat [B, n_h, d_c] desc dtype, lse [B, n_h]
 *   float (may be NULL). */
mla_status_t mla_decode_attn_partial(const mla_layer_desc* desc, const void* q_lat, const void* q_rope,
                                     const mla_paged_cache* cache, const int32_t* kv_begin, const int32_t* kv_end,
                                     int B, void* ws, size_t ws_bytes, float* o_part, float* lse_part, void* stream);
mla_status_t mla_lse_merge(const mla_layer_desc* desc, const float* o_parts, const float* lse_parts, int R, int B,
                           void* o_lat, float* lse, void* stream);

/* Causal attention of a chunk of q_per_seq new queries per sequence (chunked
 * prefill, after mla_compress_append of the chunk).  Query q of sequence b
 * sits at position q_start[b] + q and attends rows 0 .. q_start[b] + q.
 *   q_lat [B*q_per_seq, n_h, d_c], q_rope [B*q_per_seq, n_h, d_hr]
 *   o_lat [B*q_per_seq, n_h, d_c], lse [B*q_per_seq, n_h] float (may be NULL) */
mla_status_t mla_prefill_attn(const mla_layer_desc* desc, const void* q_lat, const void* q_rope,
                              const mla_paged_cache* cache, const int32_t* q_start, int q_per_seq, int B,
                              void* ws, size_t ws_bytes, void* o_lat, float* lse, void* stream);

/* Chunked prefill in the un-absorbed form (the reading notes' eqs 10-11: per-head
 * keys k^C_i = W^UK_i c^KV and values v^C_i = W^UV_i c^KV decompressed once per
 * chunk, then causal attention with q_i = [q^C_i ; q^R_i], k_i = [k^C_i ; k^R]).
 * Per (query, key) pair it costs 2 n_h (d_h + d_h^R + d_h) FLOP against
 * 2 n_h (2 d_c + d_h^R) in the latent form, plus the decompression of every
 * cached row of the chunk's sequences: cheaper for long chunks.
 *
 * mla_queries: q_c [T, n_h, d_h] and q_rope [T, n_h, d_hr] (eqs 12-13, decoupled
 *   query), without the W^UK absorption.  Workspace as mla_absorb_q's.
 * mla_prefill_attn_unabsorbed: after mla_compress_append of the chunk, query q
 *   of sequence b at position q_start[b] + q attends rows 0 .. q_start[b] + q.
 *   Decompresses the pages of rows 0 .. q_start[b] + q_per_seq - 1 of each
 *   sequence into the workspace (mla_prefill_unabsorbed_workspace_size bytes:
 *   2 n_h d_h bf16 values per pool row), then runs the attention.
 *   q_c, q_rope [B*q_per_seq, n_h, ...] from mla_queries; o [B*q_per_seq, n_h,
 *   d_h] bf16 out; lse [B*q_per_seq, n_h] float out (may be NULL).  bf16 layers
 *   with d_h == 128 and MLA_CACHE_NATIVE rows.
 * mla_out_proj_unabsorbed: u [T, d] float = W^O o (eq 8) for o [T, n_h, d_h]. */
size_t mla_prefill_unabsorbed_workspace_size(const mla_layer_desc* desc, int num_blocks, int B, int max_blocks);
mla_status_t mla_queries(const mla_layer_desc* desc, const mla_weights* w, const void* h, const int32_t* pos, int T,
                         void* q_c, void* q_rope, void* ws, size_t ws_bytes, void* stream);
mla_status_t mla_prefill_attn_unabsorbed(const mla_layer_desc* desc, const mla_weights* w, const void* q_c,
                                         const void* q_rope, const mla_paged_cache* cache, const int32_t* q_start,
                                         int q_per_seq, int B, void* ws, size_t ws_bytes, void* o, float* lse,
                                         void* stream);
mla_status_t mla_out_proj_unabsorbed(const mla_layer_desc* desc, const mla_weights* w, const void* o, int T, float* u,
                                     void* stream);

/* Output projection (eq 8 with W^UV absorbed): u = W^O [W^UV_i o_lat_i]_i.
 *   o_lat [T, n_h, d_c]; u [T, d] float                                     */
mla_status_t mla_out_proj(const mla_layer_desc* desc, const mla_weights* w, const void* o_lat, int T,
                          float* u, void* ws, size_t ws_bytes, void* stream);

/* Synchronises `stream`, then returns and clears the device error word
 * (MLA_ERR_CAPACITY for a bad page id, MLA_ERR_DEVICE_TIMEOUT for an
 * abandoned wait) or MLA_ERR_CUDA if the stream reported a CUDA error. */
mla_status_t mla_get_last_error(void* stream);

/* Measurement hook.  With non-NULL handles (cudaEvent_t values), every
 * later bf16 attention call (decode, no-alloc, partial, latent prefill)
 * records `before` on its stream right before its attention kernel (after
 * the work plan) and `after` right after it (before the combine), so that
 * the kernel can be timed alone; the events separate the kernel from its
 * neighbours on the stream, so a timed run with them set is not the
 * pipelined step.  NULL, NULL turns it off.  Process-wide, not thread-safe:
 * for benchmarks only. */
void mla_debug_attention_events(void* before, void* after);

/* Test hook for the bounded waits.  Sets the process-wide wait limit of the
 * kernels to `limit_ns` (1 .. 100,000,000 ns) on `stream`, runs one kernel
 * whose single thread waits on a shared-memory barrier that nothing arrives
 * on (the kernels' own wait routine, so it gives up after the limit and
 * records MLA_ERR_DEVICE_TIMEOUT in the device error word; no copy or MMA is
 * in flight), then puts the previous limit back on the same stream.  Returns
 * MLA_ERR_INVALID_ARG for a limit out of range, MLA_ERR_CUDA if a copy or the
 * launch failed, else MLA_OK; the timeout itself is read with
 * mla_get_last_error(stream).  Kernels on other streams that run meanwhile
 * see the lowered limit: for tests only. */
mla_status_t mla_debug_wait_probe(long long limit_ns, void* stream);

/* Static string for a status code. */
const char* mla_status_string(mla_status_t status);

/* Library version, for the loader check: (major << 16) | minor. */
int mla_version(void);

/* Number of kernels this library has launched in this process (all devices,
 * all streams), for accounting in benchmarks. */
unsigned long long mla_launch_count(void);

#ifdef __cplusplus
}
#endif
#endif /* MLA_H */
