// mla_lib.cu — the C ABI of include/mla.h (one translation unit).
//
// Host side of every entry point: argument validation, workspace carving,
// TMA descriptor creation and kernel launches on the caller's stream.  The
// kernels themselves live in the included .cuh files.
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>
#include <string.h>

#include <mutex>

#include "../../include/mla.h"
#include "common.cuh"
#include "rope.cuh"
#include "simt_f32.cuh"
#include "tc_kernels.cuh"

using namespace mla;

namespace {

constexpr int kVersionMajor = 0, kVersionMinor = 1;

inline cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

// A bounded wait that runs out: one thread waits on a barrier that nothing
// arrives on, with the kernels' own wait (mbar_wait), so the give-up path
// (error word, status) can be exercised without stopping a pipeline that has
// copies or MMAs in flight.
constexpr long long kProbeMaxNs = 100000000LL;  // 0.1 s
__global__ void mla_wait_probe_kernel() {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
    mbar_wait(&bar, 0, nullptr, 901);
  }
}

mla_status_t check_launch() {
  return cudaGetLastError() == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

bool desc_valid(const mla_layer_desc* D) {
  if (!D) return false;
  if (D->d <= 0 || D->n_h <= 0 || D->d_h <= 0 || D->d_c <= 0 || D->d_cq < 0 || D->d_hr < 0) return false;
  if (D->d_hr % 2 != 0 || D->block_size <= 0) return false;
  if (!(D->rope_base > 0.0) || !(D->yarn_scale >= 1.0) || !(D->attn_logit_factor > 0.0)) return false;
  if (D->yarn_scale > 1.0 && (D->yarn_orig_ctx <= 0 || !(D->yarn_beta > D->yarn_alpha))) return false;
  if (D->latent_norm && (!(D->norm_eps >= 0.0) || !(D->scale_kv > 0.0) || !(D->scale_q > 0.0))) return false;
  if (D->cache_dtype != MLA_CACHE_NATIVE && !(D->cache_dtype == MLA_CACHE_FP8_E4M3 && D->dtype == MLA_BF16))
    return false;
  return D->dtype == MLA_F32 || D->dtype == MLA_BF16;
}

// Every latent attention path reads both row formats (both attention kernels
// have an FP8 form).
bool attn_cache_supported(const mla_layer_desc*) { return true; }

// Shapes the tcgen05 kernels are written for.
bool bf16_supported(const mla_layer_desc* D) {
  return D->block_size == 64 && D->d_c == 512 && D->d_hr == 64 && D->d_h % 64 == 0 && D->d % 64 == 0 &&
         D->d_cq % 64 == 0 && (D->n_h == 16 || D->n_h == 32 || D->n_h == 64 || D->n_h == 128);
}

RopeParams rope_params(const mla_layer_desc* D) {
  RopeParams r;
  r.base = D->rope_base;
  r.yarn_scale = D->yarn_scale;
  r.yarn_alpha = D->yarn_alpha;
  r.yarn_beta = D->yarn_beta;
  r.yarn_orig_ctx = D->yarn_orig_ctx;
  return r;
}

double softmax_scale(const mla_layer_desc* D) { return D->attn_logit_factor / sqrt((double)(D->d_h + D->d_hr)); }

F32Layer f32_layer(const mla_layer_desc* D) {
  F32Layer L;
  L.d = D->d;
  L.n_h = D->n_h;
  L.d_h = D->d_h;
  L.d_c = D->d_c;
  L.d_cq = D->d_cq;
  L.d_hr = D->d_hr;
  L.block_size = D->block_size;
  L.rope = rope_params(D);
  L.scale_log2 = (float)(softmax_scale(D) * 1.4426950408889634);
  L.latent_norm = D->latent_norm ? 1 : 0;
  L.norm_eps = (float)D->norm_eps;
  L.scale_kv = (float)D->scale_kv;
  L.scale_q = (float)D->scale_q;
  return L;
}

bool cache_valid(const mla_paged_cache* c) {
  return c && c->pool && c->block_table && c->num_blocks > 0 && c->max_blocks > 0;
}

size_t f32_attn_ws(const mla_layer_desc* D, int rows, int max_len) {
  return (size_t)rows * D->n_h * (size_t)max_len * sizeof(float);
}

}  // namespace

// ---------------------------------------------------------------------------
// Scratch for mla_decode_attn_noalloc: a fixed device array owned by this
// library instead of a caller workspace.  Every device that loads the library
// holds it until the process exits.  Host code may not use the symbol itself
// as a device address; the address is looked up per device.
// ---------------------------------------------------------------------------
constexpr size_t kNoAllocScratchBytes = 32u << 20;  // 32 MiB
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mutex;
void* g_noalloc_ptr[kMaxDevices] = {};

// Device address of g_noalloc_scratch on the current device (looked up once
// per device, with that device current).  nullptr if the lookup fails.
void* noalloc_scratch() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  if (!g_noalloc_ptr[dev]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess) return nullptr;
    g_noalloc_ptr[dev] = ptr;
  }
  return g_noalloc_ptr[dev];
}
}  // namespace

extern "C" {

int mla_version(void) { return (kVersionMajor << 16) | kVersionMinor; }

unsigned long long mla_launch_count(void) { return launch_counter(); }

const char* mla_status_string(mla_status_t s) {
  switch (s) {
    case MLA_OK: return "ok";
    case MLA_ERR_INVALID_ARG: return "invalid argument";
    case MLA_ERR_UNSUPPORTED: return "unsupported shape or dtype";
    case MLA_ERR_CAPACITY: return "capacity exceeded (workspace or page id)";
    case MLA_ERR_CUDA: return "CUDA error";
    case MLA_ERR_DEVICE_TIMEOUT: return "device wait timed out";
  }
  return "unknown status";
}

size_t mla_cache_row_bytes(const mla_layer_desc* D) {
  if (!desc_valid(D)) return 0;
  if (D->dtype == MLA_F32) return (size_t)(D->d_c + D->d_hr) * sizeof(float);
  return (size_t)cache_row_bytes(D);
}

mla_status_t mla_cache_quantize(const mla_layer_desc* D, const void* src, long long n, void* dst, void* stream) {
  if (!desc_valid(D) || !src || !dst || n < 0 || !fp8_cache(D)) return MLA_ERR_INVALID_ARG;
  if (n == 0) return MLA_OK;
  if (!bf16_supported(D)) return MLA_ERR_UNSUPPORTED;
  if (!aligned16(src) || !aligned16(dst)) return MLA_ERR_INVALID_ARG;
  const char* s0 = (const char*)src;
  const char* d0 = (const char*)dst;
  if (s0 < d0 + n * cache_row_bytes(D) && d0 < s0 + n * (D->d_c + D->d_hr) * 2) return MLA_ERR_INVALID_ARG;
  const long long blocks = (n + CVT_ROWS_PER_BLOCK - 1) / CVT_ROWS_PER_BLOCK;
  if (blocks > 0x7FFFFFFFLL) return MLA_ERR_UNSUPPORTED;
  return launch_pdl(mla_cache_to_fp8_kernel, dim3((unsigned)blocks), dim3(32 * CVT_ROWS_PER_BLOCK), 0,
                    as_stream(stream), 1, (const __nv_bfloat16*)src, n, (uint8_t*)dst, cache_row_bytes(D)) ==
                 cudaSuccess
             ? MLA_OK
             : MLA_ERR_CUDA;
}

size_t mla_workspace_size(const mla_layer_desc* D, int T, int B, int max_kv_len) {
  if (!desc_valid(D) || T < 0 || B < 0 || max_kv_len < 0) return 0;
  if (D->dtype == MLA_F32) {
    const int cap = (max_kv_len + D->block_size - 1) / D->block_size * D->block_size;
    return f32_attn_ws(D, B, cap) + 256;
  }
  return tc_workspace_size(D, T, B, max_kv_len);
}

mla_status_t mla_compress_append(const mla_layer_desc* D, const mla_weights* w, const void* h, const int32_t* seq_idx,
                                 const int32_t* pos, int T, mla_paged_cache* cache, void* ws, size_t ws_bytes,
                                 void* stream) {
  if (!desc_valid(D) || !w || !w->w_dkv || !w->w_kr || !h || !seq_idx || !pos || T < 0 || !cache_valid(cache) ||
      (D->latent_norm && !w->g_kv))
    return MLA_ERR_INVALID_ARG;
  if (T == 0) return MLA_OK;
  if (D->dtype == MLA_F32) {
    F32Layer L = f32_layer(D);
    const size_t smem = (size_t)(D->d + D->d_c + D->d_hr) * sizeof(float);
    if (smem > 200 * 1024) return MLA_ERR_UNSUPPORTED;
    MLA_COUNT_LAUNCH();
    f32_compress_append_kernel<<<T, 256, smem, as_stream(stream)>>>(
        L, (const float*)h, (const float*)w->w_dkv, (const float*)w->w_kr, (const float*)w->g_kv, seq_idx, pos,
        (float*)cache->pool,
        cache->num_blocks, cache->block_table, cache->max_blocks);
    return check_launch();
  }
  if (!bf16_supported(D)) return MLA_ERR_UNSUPPORTED;
  return tc_compress_append(D, w, h, seq_idx, pos, T, cache, ws, ws_bytes, as_stream(stream));
}

mla_status_t mla_absorb_q(const mla_layer_desc* D, const mla_weights* w, const void* h, const int32_t* pos, int T,
                          void* q_lat, void* q_rope, void* ws, size_t ws_bytes, void* stream) {
  if (!desc_valid(D) || !w || !w->w_uq || !w->w_qr || !w->w_uk || (D->d_cq && !w->w_dq) || !h || !pos || T < 0 ||
      !q_lat || !q_rope || (D->latent_norm && D->d_cq && !w->g_q))
    return MLA_ERR_INVALID_ARG;
  if (T == 0) return MLA_OK;
  if (D->dtype == MLA_F32) {
    F32Layer L = f32_layer(D);
    const int q_in = D->d_cq ? D->d_cq : D->d;
    const size_t smem = (size_t)(D->d + q_in + D->n_h * D->d_h + D->n_h * D->d_hr) * sizeof(float);
    if (smem > 200 * 1024) return MLA_ERR_UNSUPPORTED;
    if (smem > 48 * 1024)
      cudaFuncSetAttribute(f32_absorb_q_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    MLA_COUNT_LAUNCH();
    f32_absorb_q_kernel<<<T, 256, smem, as_stream(stream)>>>(L, (const float*)h, (const float*)w->w_dq,
                                                               (const float*)w->g_q, (const float*)w->w_uq,
                                                               (const float*)w->w_qr,
                                                               (const float*)w->w_uk, pos, (float*)q_lat,
                                                               (float*)q_rope);
    return check_launch();
  }
  if (!bf16_supported(D)) return MLA_ERR_UNSUPPORTED;
  return tc_absorb_q(D, w, h, pos, T, q_lat, q_rope, ws, ws_bytes, as_stream(stream));
}

mla_status_t mla_compress_append_absorb_q(const mla_layer_desc* D, const mla_weights* w, const void* h,
                                          const int32_t* seq_idx, const int32_t* pos, int T, mla_paged_cache* cache,
                                          void* q_lat, void* q_rope, void* ws, size_t ws_bytes, void* stream) {
  if (!desc_valid(D) || !w || !w->w_dkv || !w->w_kr || !w->w_uq || !w->w_qr || !w->w_uk || (D->d_cq && !w->w_dq) ||
      !h || !seq_idx || !pos || T < 0 || !cache_valid(cache) || !q_lat || !q_rope ||
      (D->latent_norm && (!w->g_kv || (D->d_cq && !w->g_q))))
    return MLA_ERR_INVALID_ARG;
  if (T == 0) return MLA_OK;
  if (D->dtype == MLA_F32) {
    const mla_status_t s = mla_compress_append(D, w, h, seq_idx, pos, T, cache, ws, ws_bytes, stream);
    return s != MLA_OK ? s : mla_absorb_q(D, w, h, pos, T, q_lat, q_rope, ws, ws_bytes, stream);
  }
  if (!bf16_supported(D)) return MLA_ERR_UNSUPPORTED;
  return tc_compress_absorb(D, w, h, seq_idx, pos, T, cache, q_lat, q_rope, ws, ws_bytes, as_stream(stream));
}

static mla_status_t f32_attention(const mla_layer_desc* D, const void* q_lat, const void* q_rope,
                                  const mla_paged_cache* cache, const int32_t* kv_len, const int32_t* q_start,
                                  int q_per_seq, int rows, void* ws, size_t ws_bytes, void* o_lat, float* lse,
                                  cudaStream_t stream) {
  const int max_len = cache->max_blocks * D->block_size;
  if (!ws || ws_bytes < f32_attn_ws(D, rows, max_len)) return MLA_ERR_CAPACITY;
  F32Layer L = f32_layer(D);
  dim3 grid(rows, D->n_h);
  MLA_COUNT_LAUNCH();
  f32_attn_kernel<<<grid, 128, 0, stream>>>(L, (const float*)q_lat, (const float*)q_rope, (const float*)cache->pool,
                                            cache->num_blocks, cache->block_table, cache->max_blocks, kv_len,
                                            q_start, q_per_seq, (float*)ws, max_len, (float*)o_lat, lse);
  return check_launch();
}

mla_status_t mla_decode_attn(const mla_layer_desc* D, const void* q_lat, const void* q_rope,
                             const mla_paged_cache* cache, const int32_t* kv_len, int B, void* ws, size_t ws_bytes,
                             int num_splits, void* o_lat, float* lse, void* stream) {
  if (!desc_valid(D) || !q_lat || !q_rope || !cache_valid(cache) || !kv_len || B < 0 || num_splits < 0 || !o_lat)
    return MLA_ERR_INVALID_ARG;
  if (B == 0) return MLA_OK;
  if (D->dtype == MLA_F32)
    return f32_attention(D, q_lat, q_rope, cache, kv_len, nullptr, 1, B, ws, ws_bytes, o_lat, lse,
                         as_stream(stream));
  if (!bf16_supported(D) || !attn_cache_supported(D)) return MLA_ERR_UNSUPPORTED;
  return tc_attention(D, q_lat, q_rope, cache, kv_len, nullptr, 1, B, ws, ws_bytes, num_splits, o_lat, lse,
                      as_stream(stream));
}

mla_status_t mla_decode_attn_noalloc(const mla_layer_desc* D, const void* q_lat, const void* q_rope,
                                     const mla_paged_cache* cache, const int32_t* kv_len, int B, int num_splits,
                                     void* o_lat, float* lse, void* stream) {
  if (!desc_valid(D) || !q_lat || !q_rope || !cache_valid(cache) || !kv_len || B < 0 || num_splits < 0 || !o_lat)
    return MLA_ERR_INVALID_ARG;
  if (B == 0) return MLA_OK;
  void* scratch = noalloc_scratch();
  if (!scratch) return MLA_ERR_CUDA;
  // Every partial the kernels read back is written first in the same call,
  // so the array needs no clearing between calls.
  const int max_len = cache->max_blocks * D->block_size;
  if (D->dtype == MLA_F32) {
    if (f32_attn_ws(D, B, max_len) > kNoAllocScratchBytes) return MLA_ERR_CAPACITY;
    return f32_attention(D, q_lat, q_rope, cache, kv_len, nullptr, 1, B, scratch, kNoAllocScratchBytes, o_lat, lse,
                         as_stream(stream));
  }
  if (!bf16_supported(D) || !attn_cache_supported(D)) return MLA_ERR_UNSUPPORTED;
  // The plan's unit list and partials must fit the array: an explicit split
  // count that does not fit is refused; the automatic plan deals the tiles
  // out to the largest number of CTAs (CTA pairs) whose plan fits.
  const size_t cap = kNoAllocScratchBytes - 256;
  int workers = 0;
  if (num_splits > 0) {
    if (ws_attn(D, B, plan_attn(D, B, max_len, num_splits)) > cap) return MLA_ERR_CAPACITY;
  } else {
    // the largest worker count whose plan fits (host arithmetic only)
    workers = attn_wave_workers(D);
    while (workers > 1 && ws_attn(D, B, plan_attn(D, B, max_len, 0, workers)) > cap) --workers;
    if (ws_attn(D, B, plan_attn(D, B, max_len, 0, workers)) > cap) return MLA_ERR_CAPACITY;
  }
  return tc_attention(D, q_lat, q_rope, cache, kv_len, nullptr, 1, B, scratch, kNoAllocScratchBytes, num_splits,
                      o_lat, lse, as_stream(stream), workers);
}

mla_status_t mla_decode_attn_partial(const mla_layer_desc* D, const void* q_lat, const void* q_rope,
                                     const mla_paged_cache* cache, const int32_t* kv_begin, const int32_t* kv_end,
                                     int B, void* ws, size_t ws_bytes, float* o_part, float* lse_part, void* stream) {
  if (!desc_valid(D) || !q_lat || !q_rope || !cache_valid(cache) || !kv_begin || !kv_end || B < 0 || !o_part ||
      !lse_part)
    return MLA_ERR_INVALID_ARG;
  if (B == 0) return MLA_OK;
  if (D->dtype != MLA_BF16 || !bf16_supported(D) || !attn_cache_supported(D)) return MLA_ERR_UNSUPPORTED;
  return tc_attention(D, q_lat, q_rope, cache, kv_end, nullptr, 1, B, ws, ws_bytes, 0, nullptr, lse_part,
                      as_stream(stream), 0, kv_begin, o_part);
}

mla_status_t mla_lse_merge(const mla_layer_desc* D, const float* o_parts, const float* lse_parts, int R, int B,
                           void* o_lat, float* lse, void* stream) {
  if (!desc_valid(D) || !o_parts || !lse_parts || R < 1 || B < 0 || !o_lat) return MLA_ERR_INVALID_ARG;
  if (B == 0) return MLA_OK;
  if (D->dtype == MLA_BF16 && !bf16_supported(D)) return MLA_ERR_UNSUPPORTED;
  return tc_lse_merge(D, o_parts, lse_parts, R, B, o_lat, lse, as_stream(stream));
}

size_t mla_prefill_unabsorbed_workspace_size(const mla_layer_desc* D, int num_blocks, int B, int max_blocks) {
  if (!desc_valid(D) || num_blocks < 0 || B < 0 || max_blocks < 0) return 0;
  return ws_prefill_unabsorbed(D, num_blocks, B, max_blocks);
}

mla_status_t mla_queries(const mla_layer_desc* D, const mla_weights* w, const void* h, const int32_t* pos, int T,
                         void* q_c, void* q_rope, void* ws, size_t ws_bytes, void* stream) {
  if (!desc_valid(D) || !w || !w->w_uq || !w->w_qr || (D->d_cq && !w->w_dq) || !h || !pos || T < 0 || !q_c ||
      !q_rope || (D->latent_norm && D->d_cq && !w->g_q))
    return MLA_ERR_INVALID_ARG;
  if (T == 0) return MLA_OK;
  if (D->dtype != MLA_BF16 || !bf16_supported(D)) return MLA_ERR_UNSUPPORTED;
  return tc_absorb_q(D, w, h, pos, T, nullptr, q_rope, ws, ws_bytes, as_stream(stream), q_c);
}

mla_status_t mla_prefill_attn_unabsorbed(const mla_layer_desc* D, const mla_weights* w, const void* q_c,
                                         const void* q_rope, const mla_paged_cache* cache, const int32_t* q_start,
                                         int q_per_seq, int B, void* ws, size_t ws_bytes, void* o, float* lse,
                                         void* stream) {
  if (!desc_valid(D) || !w || !w->w_uk || !w->w_uv || !q_c || !q_rope || !cache_valid(cache) || !q_start ||
      q_per_seq <= 0 || B < 0 || !o)
    return MLA_ERR_INVALID_ARG;
  if (B == 0) return MLA_OK;
  if ((long long)B * q_per_seq > (1 << 30)) return MLA_ERR_UNSUPPORTED;
  if (D->dtype != MLA_BF16 || !bf16_supported(D) || fp8_cache(D)) return MLA_ERR_UNSUPPORTED;
  return tc_prefill_unabsorbed(D, w, q_c, q_rope, cache, q_start, q_per_seq, B, ws, ws_bytes, o, lse,
                               as_stream(stream));
}

mla_status_t mla_out_proj_unabsorbed(const mla_layer_desc* D, const mla_weights* w, const void* o, int T, float* u,
                                     void* stream) {
  if (!desc_valid(D) || !w || !w->w_o || !o || T < 0 || !u) return MLA_ERR_INVALID_ARG;
  if (T == 0) return MLA_OK;
  if (D->dtype != MLA_BF16 || !bf16_supported(D)) return MLA_ERR_UNSUPPORTED;
  return tc_out_proj(D, w, o, T, u, nullptr, 0, as_stream(stream), /*from_o=*/true);
}

mla_status_t mla_prefill_attn(const mla_layer_desc* D, const void* q_lat, const void* q_rope,
                              const mla_paged_cache* cache, const int32_t* q_start, int q_per_seq, int B, void* ws,
                              size_t ws_bytes, void* o_lat, float* lse, void* stream) {
  if (!desc_valid(D) || !q_lat || !q_rope || !cache_valid(cache) || !q_start || q_per_seq <= 0 || B < 0 || !o_lat)
    return MLA_ERR_INVALID_ARG;
  if (B == 0) return MLA_OK;
  const long long rows = (long long)B * q_per_seq;
  if (rows > (1 << 30)) return MLA_ERR_UNSUPPORTED;
  if (D->dtype == MLA_F32)
    return f32_attention(D, q_lat, q_rope, cache, nullptr, q_start, q_per_seq, (int)rows, ws, ws_bytes, o_lat, lse,
                         as_stream(stream));
  if (!bf16_supported(D) || !attn_cache_supported(D)) return MLA_ERR_UNSUPPORTED;
  return tc_attention(D, q_lat, q_rope, cache, nullptr, q_start, q_per_seq, (int)rows, ws, ws_bytes, 1, o_lat, lse,
                      as_stream(stream));
}

mla_status_t mla_out_proj(const mla_layer_desc* D, const mla_weights* w, const void* o_lat, int T, float* u, void* ws,
                          size_t ws_bytes, void* stream) {
  if (!desc_valid(D) || !w || !w->w_uv || !w->w_o || !o_lat || T < 0 || !u) return MLA_ERR_INVALID_ARG;
  if (T == 0) return MLA_OK;
  if (D->dtype == MLA_F32) {
    F32Layer L = f32_layer(D);
    const size_t smem = (size_t)(D->n_h * D->d_c + D->n_h * D->d_h) * sizeof(float);
    if (smem > 200 * 1024) return MLA_ERR_UNSUPPORTED;
    if (smem > 48 * 1024)
      cudaFuncSetAttribute(f32_out_proj_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    MLA_COUNT_LAUNCH();
    f32_out_proj_kernel<<<T, 256, smem, as_stream(stream)>>>(L, (const float*)o_lat, (const float*)w->w_uv,
                                                               (const float*)w->w_o, u);
    return check_launch();
  }
  if (!bf16_supported(D)) return MLA_ERR_UNSUPPORTED;
  return tc_out_proj(D, w, o_lat, T, u, ws, ws_bytes, as_stream(stream));
}

#ifdef MLA_TRACE
// Trace builds only: copy the device trace buffer to `dst` (host) and clear it.
int mla_trace_read(void* dst, size_t bytes) {
  if (bytes > sizeof(g_trace)) bytes = sizeof(g_trace);
  if (cudaDeviceSynchronize() != cudaSuccess) return -1;
  if (cudaMemcpyFromSymbol(dst, g_trace, bytes) != cudaSuccess) return -1;
  static unsigned long long zeros[MLA_TRACE_UNITS][MLA_TRACE_EVENTS][MLA_TRACE_TILES];
  return cudaMemcpyToSymbol(g_trace, zeros, sizeof(zeros)) == cudaSuccess ? (int)bytes : -1;
}
#endif

mla_status_t mla_debug_wait_probe(long long limit_ns, void* stream) {
  if (limit_ns <= 0 || limit_ns > kProbeMaxNs) return MLA_ERR_INVALID_ARG;
  cudaStream_t st = as_stream(stream);
  unsigned long long prev = 0;
  const unsigned long long lim = (unsigned long long)limit_ns;
  if (cudaMemcpyFromSymbol(&prev, g_spin_limit_ns, sizeof(prev)) != cudaSuccess) return MLA_ERR_CUDA;
  // pageable sources: each copy is staged before the call returns
  if (cudaMemcpyToSymbolAsync(g_spin_limit_ns, &lim, sizeof(lim), 0, cudaMemcpyHostToDevice, st) != cudaSuccess)
    return MLA_ERR_CUDA;
  mla_wait_probe_kernel<<<1, 32, 0, st>>>();
  const cudaError_t e = cudaGetLastError();
  // the process-wide limit goes back whatever the launch did
  const cudaError_t r = cudaMemcpyToSymbolAsync(g_spin_limit_ns, &prev, sizeof(prev), 0, cudaMemcpyHostToDevice, st);
  return e == cudaSuccess && r == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

void mla_debug_attention_events(void* before, void* after) {
  g_attn_ev_before = reinterpret_cast<cudaEvent_t>(before);
  g_attn_ev_after = reinterpret_cast<cudaEvent_t>(after);
}

mla_status_t mla_get_last_error(void* stream) {
  if (cudaStreamSynchronize(as_stream(stream)) != cudaSuccess) return MLA_ERR_CUDA;
  int code = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&code, g_error_code, sizeof(int)) != cudaSuccess) return MLA_ERR_CUDA;
  if (code != 0) {
    cudaMemcpyToSymbol(g_error_code, &zero, sizeof(int));
    cudaMemcpyToSymbol(g_error_site, &zero, sizeof(int));
    return code == ERR_TIMEOUT ? MLA_ERR_DEVICE_TIMEOUT : MLA_ERR_CAPACITY;
  }
  return cudaGetLastError() == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

}  // extern "C"
