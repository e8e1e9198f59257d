// tc_kernels.cuh — host side of the bf16 tensor-core path.
//
// Builds TMA descriptors over the caller's buffers, plans the projections'
// K splits (thread-block clusters) and the attention's work plan from the SM
// count, carves the caller's workspace and launches the GEMM, plan, attention
// and combine kernels on the caller's stream with programmatic dependent
// launch.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <mutex>
#include <utility>

#include "../../include/mla.h"
#include "common.cuh"
#include "norm.cuh"
#include "rope.cuh"
#include "tc_attn.cuh"
#include "tc_attn2.cuh"
#include "tc_gemm.cuh"
#include "tc_prefill.cuh"
#include "tc_gemm_heads.cuh"

namespace mla {

// ---------------------------------------------------------------------------
// device properties and TMA descriptor encoding
// ---------------------------------------------------------------------------
inline int num_sms() {
  int dev = 0, n = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

// the layer's cache rows are FP8 (E4M3 codes of c^KV, bf16 k^R, a scale)
inline bool fp8_cache(const mla_layer_desc* D) { return D->cache_dtype == MLA_CACHE_FP8_E4M3; }

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 2D bf16 map: `outer` rows of `inner` elements, rows `row_bytes` apart,
// box = box_outer rows x box_inner elements, 128-byte swizzle.
inline bool map_2d(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer, uint64_t row_bytes,
                   uint32_t box_inner, uint32_t box_outer) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t es[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The paged cache as a 3D map {row values, slot, block}; box = one page of
// 64 slots x 64 values.  Block coordinates past num_blocks read zeros.
inline bool map_cache(CUtensorMap* m, const void* pool, int num_blocks, int row) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {(cuuint64_t)row, 64, (cuuint64_t)num_blocks};
  cuuint64_t strides[2] = {(cuuint64_t)row * 2, (cuuint64_t)row * 2 * 64};
  cuuint32_t box[3] = {64, 64, 1};
  cuuint32_t es[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(pool), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The paged cache as a 4D map {column in chunk, slot, 64-column chunk, block}
// (the chunk stride, 128 bytes, is smaller than the slot stride): a box of
// `chunks` chunks of one page lands chunk-major, 8 KB per chunk, so one TMA
// instruction moves up to a whole page.
inline bool map_cache_chunks(CUtensorMap* m, const void* pool, int num_blocks, int row, int chunks) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[4] = {64, 64, (cuuint64_t)(row / 64), (cuuint64_t)num_blocks};
  cuuint64_t strides[3] = {(cuuint64_t)row * 2, 128, (cuuint64_t)row * 2 * 64};
  cuuint32_t box[4] = {64, 64, (cuuint32_t)chunks, 1};
  cuuint32_t es[4] = {1, 1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(pool), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// FP8 cache rows (row_bytes each) as bf16 elements in 128-byte chunks
// {column in chunk, slot, chunk, block}: chunk d_c / 128 is k^R (64 x 64
// boxes, 128-byte swizzle), the layout of map_cache_chunks' RoPE box.
inline bool map_fp8_rope_chunks(CUtensorMap* m, const void* pool, int num_blocks, int row_bytes) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[4] = {64, 64, (cuuint64_t)(row_bytes / 128), (cuuint64_t)num_blocks};
  cuuint64_t strides[3] = {(cuuint64_t)row_bytes, 128, (cuuint64_t)row_bytes * 64};
  cuuint32_t box[4] = {64, 64, 1, 1};
  cuuint32_t es[4] = {1, 1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(pool), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// FP8 cache rows (row_bytes each) as bytes {byte, slot, block}; box = box_bytes
// x 64 slots of one page, no swizzle (the codes of 128 latent columns, or a
// row's 16-byte scale field).
inline bool map_cache_bytes(CUtensorMap* m, const void* pool, int num_blocks, int row_bytes, uint32_t box_bytes) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {(cuuint64_t)row_bytes, 64, (cuuint64_t)num_blocks};
  cuuint64_t strides[2] = {(cuuint64_t)row_bytes, (cuuint64_t)row_bytes * 64};
  cuuint32_t box[3] = {box_bytes, 64, 1};
  cuuint32_t es[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(pool), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The same FP8 rows as bf16 elements {value, slot, block} (row_bytes / 2
// values per row): 64 x 64 boxes with the 128-byte swizzle, for k^R.
inline bool map_cache_bf16_view(CUtensorMap* m, const void* pool, int num_blocks, int row_bytes) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {(cuuint64_t)row_bytes / 2, 64, (cuuint64_t)num_blocks};
  cuuint64_t strides[2] = {(cuuint64_t)row_bytes, (cuuint64_t)row_bytes * 64};
  cuuint32_t box[3] = {64, 64, 1};
  cuuint32_t es[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(pool), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// A row-major bf16 matrix (`rows` rows of `inner` elements, rows `row_bytes`
// apart) as a 3D map {column in chunk, row, 64-column chunk}: a box of
// box_rows rows x kc chunks lands chunk-major (each chunk box_rows x 128 B,
// 128-byte swizzle), i.e. exactly kc consecutive 2D boxes of 64 columns.
inline bool map_rows_chunks(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows, uint64_t row_bytes,
                            uint32_t box_rows, uint32_t kc) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {64, rows, inner / 64};
  cuuint64_t strides[2] = {row_bytes, 128};
  cuuint32_t box[3] = {64, box_rows, kc};
  cuuint32_t es[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// ---------------------------------------------------------------------------
// workspace carving
// ---------------------------------------------------------------------------
struct Carver {
  uint8_t* base;
  size_t cap, used = 0;
  void* take(size_t bytes) {
    used = (used + 255) & ~size_t(255);
    void* p = base ? base + used : nullptr;
    used += bytes;
    return p;
  }
  bool ok() const { return used <= cap; }
};

// ---------------------------------------------------------------------------
// GEMM planning and launch
// ---------------------------------------------------------------------------
// Launch with programmatic stream serialisation (the kernel calls pdl_wait()
// before it touches anything an earlier kernel writes) and, for cluster > 1,
// a thread-block cluster of that many CTAs along x.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                              int cluster, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute at[2];
  int n = 0;
  at[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[n].val.programmaticStreamSerializationAllowed = 1;
  ++n;
  if (cluster > 1) {
    at[n].id = cudaLaunchAttributeClusterDimension;
    at[n].val.clusterDim.x = (unsigned)cluster;
    at[n].val.clusterDim.y = 1;
    at[n].val.clusterDim.z = 1;
    ++n;
  }
  cfg.attrs = at;
  cfg.numAttrs = n;
  MLA_COUNT_LAUNCH();
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

struct GemmPlan {
  int tn, n_tiles, splits, kcs;
  bool deep;  // one deep-pipelined CTA per SM (else two per SM)
};

inline int pick_tn(int T) { return T <= 32 ? 32 : T <= 64 ? 64 : T <= 128 ? 128 : 256; }
inline int gemm_kc(bool a_mn) { return a_mn ? 1 : MLA_GEMM_KC; }

// Tiles that fit one wave of SMs run one deep-pipelined CTA per SM, their K
// split over a cluster of up to 8 CTAs to fill the wave; more tiles than SMs
// run two CTAs per SM (token tiles of at most 64) with no split.
inline GemmPlan plan_gemm(int m_tiles, int Z, int T, int K, bool a_mn = false) {
  GemmPlan p;
  p.tn = pick_tn(T);
  p.n_tiles = (T + p.tn - 1) / p.tn;
  const int kc = K / GEMM_BK;
  const int kcb = gemm_kc(a_mn);  // chunks per stage: splits cover whole stages
  const long long tiles = (long long)m_tiles * p.n_tiles * Z;
  const int sms = num_sms();
  p.deep = tiles <= sms || p.tn > 64;
  const long long slots = (long long)sms * (p.deep ? 1 : 2);
  int s = (int)std::max<long long>(1, std::min<long long>(8, slots / std::max<long long>(tiles, 1)));
  s = std::max(1, std::min(s, kc / (2 * kcb)));
  p.kcs = ((kc + s - 1) / s + kcb - 1) / kcb * kcb;
  p.splits = (kc + p.kcs - 1) / p.kcs;
  return p;
}

template <int TN, bool A_MN, bool DEEP>
inline cudaError_t launch_gemm_t(const CUtensorMap& A0, const CUtensorMap& A1, const CUtensorMap& A2,
                                 const CUtensorMap& B, const GemmArgs& g, dim3 grid, cudaStream_t st) {
  constexpr int KC = A_MN ? 1 : MLA_GEMM_KC;
  auto kfn = gemm_bf16_kernel<TN, A_MN, KC, DEEP>;
  constexpr int smem = GemmCfg<TN, KC, DEEP>::SMEM;
  cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  return launch_pdl(kfn, grid, dim3(GEMM_THREADS), smem, st, g.splits, A0, A1, A2, B, g);
}

template <bool A_MN, bool DEEP>
inline cudaError_t launch_gemm_tn(int tn, const CUtensorMap& A0, const CUtensorMap& A1, const CUtensorMap& A2,
                                  const CUtensorMap& B, const GemmArgs& g, dim3 grid, cudaStream_t st) {
  switch (tn) {
    case 32: return launch_gemm_t<32, A_MN, DEEP>(A0, A1, A2, B, g, grid, st);
    case 64: return launch_gemm_t<64, A_MN, DEEP>(A0, A1, A2, B, g, grid, st);
    case 128: return launch_gemm_t<128, A_MN, true>(A0, A1, A2, B, g, grid, st);
    default: return launch_gemm_t<256, A_MN, true>(A0, A1, A2, B, g, grid, st);
  }
}

// One projection: Y = epilogue(A X) over up to three weight segments (rows0
// of A0, rows1 of A1, rows2 of A2), K contraction, Z batches.
struct GemmCall {
  const void* a0;
  int rows0;
  const void* a1;  // may be null
  int rows1;
  const void* a2;  // may be null (only with a1)
  int rows2;
  long long a_row_elems;  // row pitch of A in elements (K-major: K; MN-major: features)
  bool a_mn;              // A stored [k][n] (n contiguous)
  int a_mn_rows;          // MN-major: total K rows of the map (Z * K)
  const void* x;
  long long x_rows, x_row_elems;  // X map: x_rows rows of x_row_elems
  int K, T, Z, a_z_rows, b_z_cols;
  const int32_t* b_tile_row;  // optional page-indexed token tiles (see GemmArgs)
  int n_tiles_override;       // with b_tile_row: the number of token tiles
};

inline mla_status_t run_gemm(const GemmCall& c, const GemmEpi& e, const GemmPlan& p, cudaStream_t st) {
  CUtensorMap A0, A1, A2, B;
  bool ok;
  const uint32_t kc = (uint32_t)gemm_kc(c.a_mn);
  if (!c.a_mn) {
    ok = map_rows_chunks(&A0, c.a0, (uint64_t)c.K, (uint64_t)c.rows0 * c.Z, (uint64_t)c.a_row_elems * 2, 128, kc);
    ok = ok && map_rows_chunks(&A1, c.a1 ? c.a1 : c.a0, (uint64_t)c.K, (uint64_t)(c.a1 ? c.rows1 : c.rows0) * c.Z,
                               (uint64_t)c.a_row_elems * 2, 128, kc);
    if (c.a1 && c.a2)
      ok = ok && map_rows_chunks(&A2, c.a2, (uint64_t)c.K, (uint64_t)c.rows2 * c.Z, (uint64_t)c.a_row_elems * 2, 128,
                                 kc);
    else
      A2 = A0;
  } else {
    ok = map_2d(&A0, c.a0, (uint64_t)c.rows0, (uint64_t)c.a_mn_rows, (uint64_t)c.a_row_elems * 2, 64, 64);
    A1 = A2 = A0;
  }
  ok = ok && map_rows_chunks(&B, c.x, (uint64_t)c.x_row_elems, (uint64_t)c.x_rows, (uint64_t)c.x_row_elems * 2,
                             (uint32_t)p.tn, kc);
  if (!ok) return MLA_ERR_CUDA;
  GemmArgs g;
  g.k_chunks = c.K / GEMM_BK;
  g.k_chunks_split = p.kcs;
  g.splits = p.splits;
  g.m_tiles0 = (c.rows0 + GEMM_BM - 1) / GEMM_BM;
  g.m_tiles1 = c.a1 ? (c.rows1 + GEMM_BM - 1) / GEMM_BM : 0;
  g.n_out0 = c.rows0;
  g.n_out1 = c.a1 ? c.rows1 : 0;
  g.n_out2 = c.a1 && c.a2 ? c.rows2 : 0;
  g.T = c.T;
  g.a_z_rows = c.a_z_rows;
  g.b_z_cols = c.b_z_cols;
  g.b_tile_row = c.b_tile_row;
  g.e = e;
  const int m_tiles = g.m_tiles0 + g.m_tiles1 + (g.n_out2 + GEMM_BM - 1) / GEMM_BM;
  dim3 grid(m_tiles * p.splits, c.b_tile_row ? c.n_tiles_override : p.n_tiles, c.Z);
  cudaError_t err;
  if (c.a_mn)
    err = p.deep ? launch_gemm_tn<true, true>(p.tn, A0, A1, A2, B, g, grid, st)
                 : launch_gemm_tn<true, false>(p.tn, A0, A1, A2, B, g, grid, st);
  else
    err = p.deep ? launch_gemm_tn<false, true>(p.tn, A0, A1, A2, B, g, grid, st)
                 : launch_gemm_tn<false, false>(p.tn, A0, A1, A2, B, g, grid, st);
  return err == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

// A GEMM whose token tiles are cache pages (c.b_tile_row): X rows are
// x_row_bytes apart (the pool's [c^KV | k^R] rows), the plan is the caller's.
inline mla_status_t run_gemm_paged(const GemmCall& c, const GemmEpi& e, const GemmPlan& p, uint64_t x_row_bytes,
                                   cudaStream_t st) {
  CUtensorMap A0, A1, B;
  bool ok = map_rows_chunks(&A0, c.a0, (uint64_t)c.K, (uint64_t)c.rows0, (uint64_t)c.a_row_elems * 2, 128, 1);
  ok = ok && map_rows_chunks(&A1, c.a1, (uint64_t)c.K, (uint64_t)c.rows1, (uint64_t)c.a_row_elems * 2, 128, 1);
  ok = ok && map_rows_chunks(&B, c.x, (uint64_t)c.x_row_elems, (uint64_t)c.x_rows, x_row_bytes, 64, 1);
  if (!ok) return MLA_ERR_CUDA;
  GemmArgs g;
  g.k_chunks = c.K / GEMM_BK;
  g.k_chunks_split = p.kcs;
  g.splits = 1;
  g.m_tiles0 = (c.rows0 + GEMM_BM - 1) / GEMM_BM;
  g.m_tiles1 = (c.rows1 + GEMM_BM - 1) / GEMM_BM;
  g.n_out0 = c.rows0;
  g.n_out1 = c.rows1;
  g.n_out2 = 0;
  g.T = c.T;
  g.a_z_rows = 0;
  g.b_z_cols = 0;
  g.b_tile_row = c.b_tile_row;
  g.e = e;
  const int m_tiles = g.m_tiles0 + (c.rows1 + GEMM_BM - 1) / GEMM_BM;
  const cudaError_t err = launch_gemm_t<64, false, false>(A0, A1, A0, B, g, dim3(m_tiles, p.n_tiles, 1), st);
  return err == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

inline RopeParams rope_of(const mla_layer_desc* D) {
  RopeParams r;
  r.base = D->rope_base;
  r.yarn_scale = D->yarn_scale;
  r.yarn_alpha = D->yarn_alpha;
  r.yarn_beta = D->yarn_beta;
  r.yarn_orig_ctx = D->yarn_orig_ctx;
  return r;
}

// ---------------------------------------------------------------------------
// per-op workspace needs (same carving order as the ops below)
// ---------------------------------------------------------------------------
inline GemmPlan plan_compress(const mla_layer_desc* D, int T) {
  return plan_gemm((D->d_c + 127) / 128 + (D->d_hr + 127) / 128, 1, T, D->d);
}
inline GemmPlan plan_q1(const mla_layer_desc* D, int T) { return plan_gemm((D->d_cq + 127) / 128, 1, T, D->d); }
inline GemmPlan plan_compress_q(const mla_layer_desc* D, int T) {
  return plan_gemm((D->d_c + 127) / 128 + (D->d_hr + 127) / 128 + (D->d_cq + 127) / 128, 1, T, D->d);
}
inline GemmPlan plan_q2(const mla_layer_desc* D, int T) {
  const int q_in = D->d_cq ? D->d_cq : D->d;
  return plan_gemm((D->n_h * D->d_h + 127) / 128 + (D->n_h * D->d_hr + 127) / 128, 1, T, q_in);
}
inline GemmPlan plan_o1(const mla_layer_desc* D, int T) { return plan_gemm((D->d_h + 127) / 128, D->n_h, T, D->d_c); }
inline GemmPlan plan_o2(const mla_layer_desc* D, int T) {
  return plan_gemm((D->d + 127) / 128, 1, T, D->n_h * D->d_h);
}

// Workspace of the projections: only the bf16 intermediates between two
// GEMMs (K splits are reduced inside each GEMM's cluster).
// bytes of one cache row: [c^KV | k^R] in bf16, or the FP8 row (codes, bf16
// k^R, scale, padding)
inline int cache_row_bytes(const mla_layer_desc* D) {
  return fp8_cache(D) ? fp8_row_bytes(D->d_c, D->d_hr) : (D->d_c + D->d_hr) * 2;
}
inline size_t ws_compress(const mla_layer_desc* D, int T) {
  return D->latent_norm || fp8_cache(D) ? (size_t)T * D->d_c * 4 + 256 : 0;
}
inline size_t ws_absorb(const mla_layer_desc* D, int T) {
  Carver c{nullptr, 0};
  if (D->d_cq) c.take((size_t)T * D->d_cq * 2);
  c.take((size_t)T * D->n_h * D->d_h * 2);
  if (D->d_cq && D->latent_norm) c.take((size_t)T * D->d_cq * 4);
  return c.used;
}
inline size_t ws_compress_absorb(const mla_layer_desc* D, int T) {
  Carver c{nullptr, 0};
  if (D->d_cq) c.take((size_t)T * D->d_cq * 2);
  c.take((size_t)T * D->n_h * D->d_h * 2);
  if (D->d_cq && D->latent_norm) c.take((size_t)T * D->d_cq * 4);
  if (D->latent_norm || fp8_cache(D)) c.take((size_t)T * D->d_c * 4);
  return c.used;
}
inline size_t ws_out(const mla_layer_desc* D, int T) {
  Carver c{nullptr, 0};
  c.take((size_t)T * D->n_h * D->d_h * 2);
  return c.used;
}

inline int heads_per_cta(const mla_layer_desc* D) { return D->n_h == 16 ? 16 : 32; }
// 128-head layers run on CTA pairs (tc_attn2.cuh), one pair per (row,
// split), over bf16 or FP8 rows.  MLA_FP8_PAIR=0 sends 128-head layers over
// FP8 rows to the one-CTA kernel instead, as four 32-head groups per worker
// side by side on the same tiles (L2 serves the other three groups).
#ifndef MLA_FP8_PAIR
#define MLA_FP8_PAIR 1
#endif
inline bool use_pair_kernel(const mla_layer_desc* D) { return D->n_h == 128 && (MLA_FP8_PAIR || !fp8_cache(D)); }

// Host side of the attention work plan (the device side is
// mla_attn_plan_kernel).  Automatic decode plans deal the tiles of all rows
// out to one wave of CTAs (or CTA pairs) in equal contiguous ranges; explicit
// split counts cut every row into that many segments, one per CTA; prefill
// (and decode with num_splits == 1) runs one CTA per row with no plan at all.
// The host bounds the segment and slot counts for the grid and the workspace;
// the plan kernel fills in the actual lists from kv_len.
struct AttnPlan {
  bool use_plan;  // false: CTA w = row w, nothing to combine
  int splits;     // explicit segments per row (> 0) or 0 (automatic)
  int workers;    // CTAs (CTA pairs) the plan is made for = grid size / head groups
  int max_units, max_slots;
};
inline int attn_groups(const mla_layer_desc* D) { return use_pair_kernel(D) ? 1 : D->n_h / heads_per_cta(D); }
// One wave: one CTA per SM, or one CTA pair per two SMs.
inline int attn_wave_workers(const mla_layer_desc* D) {
  return std::max(1, use_pair_kernel(D) ? num_sms() / 2 : num_sms() / attn_groups(D));
}
// force: every segment gets a partial slot (partial decode: all rows go out in fp32 through the combine)
inline AttnPlan plan_attn(const mla_layer_desc* D, int rows, int max_len, int requested, int workers = 0,
                          bool force = false) {
  AttnPlan p{};
  const int max_tiles = std::max(1, (max_len + ATT_TILE - 1) / ATT_TILE);
  if (requested == 1) {
    p.use_plan = false;
    p.splits = 1;
    p.workers = rows;
    return p;
  }
  p.use_plan = true;
  if (requested > 1) {
    p.splits = std::min(requested, max_tiles);
    p.max_units = rows * p.splits;
    p.workers = p.max_units;
    p.max_slots = (p.splits > 1 || force) ? p.max_units : 0;
    return p;
  }
  p.splits = 0;
  p.workers = workers > 0 ? workers : attn_wave_workers(D);
  // each range boundary cuts at most one row: segments <= rows + workers - 1,
  // and the segments of cut rows number at most 2 * (workers - 1)
  p.max_units = rows + p.workers;
  p.max_slots = force ? p.max_units : std::min(p.max_units, 2 * p.workers);
  return p;
}
// Workspace carve of one plan: segment list, row table, CTA table, partials.
struct AttnWs {
  int4* units;
  int4* row_info;
  int* work;
  int* n_units;
  float* o_part;
  float* lse_part;
};
inline bool carve_attn(Carver& c, const mla_layer_desc* D, int rows, const AttnPlan& p, AttnWs* w) {
  *w = AttnWs{};
  if (!p.use_plan) return true;
  w->units = (int4*)c.take((size_t)p.max_units * sizeof(int4));
  w->row_info = (int4*)c.take((size_t)rows * sizeof(int4));
  w->work = (int*)c.take((size_t)(p.workers + 1) * sizeof(int));
  w->n_units = (int*)c.take(16);
  if (p.max_slots > 0) {
    w->o_part = (float*)c.take((size_t)p.max_slots * D->n_h * ATT_DC * 4);
    w->lse_part = (float*)c.take((size_t)p.max_slots * D->n_h * 4);
  }
  return c.ok();
}
inline size_t ws_attn(const mla_layer_desc* D, int rows, const AttnPlan& p) {
  Carver c{nullptr, 0};
  AttnWs w;
  carve_attn(c, D, rows, p, &w);
  return c.used;
}

}  // namespace mla

using namespace mla;

static size_t tc_workspace_size(const mla_layer_desc* D, int T, int B, int max_kv_len) {
  size_t w = 0;
  if (T > 0) w = std::max({ws_compress(D, T), ws_absorb(D, T), ws_compress_absorb(D, T), ws_out(D, T)});
  if (B > 0 && max_kv_len > 0) {
    const int max_len = (max_kv_len + 63) / 64 * 64;
    // the automatic plan, or any explicit split count up to 16
    w = std::max(w, ws_attn(D, B, plan_attn(D, B, max_len, 0)));
    w = std::max(w, ws_attn(D, B, plan_attn(D, B, max_len, 0, 0, /*force=*/true)));  // partial decode
    w = std::max(w, ws_attn(D, B, plan_attn(D, B, max_len, 16)));
  }
  return w + 256;
}

static Carver carve(void* ws, size_t ws_bytes) {
  uint8_t* b = reinterpret_cast<uint8_t*>(ws);
  const uintptr_t a = (reinterpret_cast<uintptr_t>(b) + 255) & ~uintptr_t(255);
  const size_t lost = b ? a - reinterpret_cast<uintptr_t>(b) : 0;
  return Carver{b ? reinterpret_cast<uint8_t*>(a) : nullptr, ws_bytes > lost ? ws_bytes - lost : 0};
}

// Epilogue of the GEMM that writes new cache rows: [c^KV ; k^R] with RoPE on
// k^R scattered into the paged cache, or (lat non-null) c^KV parked in fp32
// for the second pass and only k^R written.
static GemmEpi cache_epi(const mla_layer_desc* D, const int32_t* seq_idx, const int32_t* pos,
                         const mla_paged_cache* cache, float* lat) {
  GemmEpi e{};
  e.kind = EPI_CACHE;
  e.rope = rope_table(rope_of(D), D->d_hr);
  e.pos = pos;
  e.d_hr = D->d_hr;
  e.d_c = D->d_c;
  e.seq_idx = seq_idx;
  e.pool = (uint8_t*)cache->pool;
  e.num_blocks = cache->num_blocks;
  e.max_blocks = cache->max_blocks;
  e.block_size = D->block_size;
  e.row_bytes = cache_row_bytes(D);
  e.rope_off = fp8_cache(D) ? D->d_c : 2 * D->d_c;
  e.table = cache->block_table;
  e.lat_f32 = lat;
  return e;
}

// Second pass over the parked fp32 c^KV: c^KV <- scale_kv * g_kv * c^KV /
// rms(c^KV) (with the norm), into the cache row as bf16 or as E4M3 codes with
// the row's scale.
static mla_status_t kv_second_pass(const mla_layer_desc* D, const mla_weights* w, const float* lat,
                                   const int32_t* seq_idx, const int32_t* pos, int T, const mla_paged_cache* cache,
                                   cudaStream_t st) {
  NormArgs na{};
  na.x = lat;
  na.n = D->d_c;
  na.do_norm = D->latent_norm ? 1 : 0;
  na.gain = (const __nv_bfloat16*)w->g_kv;
  na.eps = (float)D->norm_eps;
  na.scale = (float)D->scale_kv;
  na.pool = (uint8_t*)cache->pool;
  na.table = cache->block_table;
  na.seq_idx = seq_idx;
  na.pos = pos;
  na.num_blocks = cache->num_blocks;
  na.max_blocks = cache->max_blocks;
  na.block_size = D->block_size;
  na.row_bytes = cache_row_bytes(D);
  na.fp8 = fp8_cache(D) ? 1 : 0;
  na.scale_off = fp8_scale_off(D->d_c, D->d_hr);
  return launch_pdl(mla_latent_norm_kernel, dim3(T), dim3(NORM_THREADS), 0, st, 1, na) == cudaSuccess ? MLA_OK
                                                                                                      : MLA_ERR_CUDA;
}

// c^Q <- scale_q * g_q * c^Q / rms(c^Q), fp32 in, bf16 out.
static mla_status_t cq_norm_pass(const mla_layer_desc* D, const mla_weights* w, const float* cq32, __nv_bfloat16* cq,
                                 int T, cudaStream_t st) {
  NormArgs na{};
  na.x = cq32;
  na.n = D->d_cq;
  na.do_norm = 1;
  na.gain = (const __nv_bfloat16*)w->g_q;
  na.eps = (float)D->norm_eps;
  na.scale = (float)D->scale_q;
  na.out = cq;
  na.out_t = D->d_cq;
  return launch_pdl(mla_latent_norm_kernel, dim3(T), dim3(NORM_THREADS), 0, st, 1, na) == cudaSuccess ? MLA_OK
                                                                                                      : MLA_ERR_CUDA;
}

// Scratch of the query path: c^Q (bf16), q^C, fp32 c^Q (latent norm) and, when
// the append shares the first GEMM, the fp32 c^KV of the second pass.
struct QueryWs {
  __nv_bfloat16 *cq, *qc;
  float *cq32, *lat;
};
static bool carve_queries(Carver& cv, const mla_layer_desc* D, int T, bool own_qc, bool with_lat, QueryWs* q) {
  q->cq = D->d_cq ? (__nv_bfloat16*)cv.take((size_t)T * D->d_cq * 2) : nullptr;
  q->qc = own_qc ? (__nv_bfloat16*)cv.take((size_t)T * D->n_h * D->d_h * 2) : nullptr;
  q->cq32 = D->d_cq && D->latent_norm ? (float*)cv.take((size_t)T * D->d_cq * 4) : nullptr;
  q->lat = with_lat && (D->latent_norm || fp8_cache(D)) ? (float*)cv.take((size_t)T * D->d_c * 4) : nullptr;
  return cv.ok();
}

static mla_status_t tc_compress_append(const mla_layer_desc* D, const mla_weights* w, const void* h,
                                       const int32_t* seq_idx, const int32_t* pos, int T, mla_paged_cache* cache,
                                       void* ws, size_t ws_bytes, cudaStream_t st) {
  if (!aligned16(h) || !aligned16(w->w_dkv) || !aligned16(w->w_kr) || !aligned16(cache->pool) ||
      (D->latent_norm && !aligned16(w->g_kv)))
    return MLA_ERR_INVALID_ARG;
  float* lat = nullptr;  // fp32 c^KV for the second pass (latent RMSNorm, FP8 encoding)
  if (D->latent_norm || fp8_cache(D)) {
    Carver cv = carve(ws, ws_bytes);
    lat = (float*)cv.take((size_t)T * D->d_c * 4);
    if (!ws || !cv.ok()) return MLA_ERR_CAPACITY;
  }
  // [c^KV ; k^R] = [W^DKV ; W^KR] h  (eq 9 + decoupled key), RoPE on k^R,
  // bf16 rows scattered into the paged cache (with the second pass: k^R only)
  GemmCall c{};
  c.a0 = w->w_dkv;
  c.rows0 = D->d_c;
  c.a1 = w->w_kr;
  c.rows1 = D->d_hr;
  c.a_row_elems = D->d;
  c.x = h;
  c.x_rows = T;
  c.x_row_elems = D->d;
  c.K = D->d;
  c.T = T;
  c.Z = 1;
  mla_status_t s = run_gemm(c, cache_epi(D, seq_idx, pos, cache, lat), plan_compress(D, T), st);
  if (s != MLA_OK || !lat) return s;
  return kv_second_pass(D, w, lat, seq_idx, pos, T, cache, st);
}

// Per-head projection out[t][i][0 .. 128 m_tiles) on one persistent CTA per
// SM (tc_gemm_heads.cuh).  A: W^UK read MN-major (A_MN) or W^UV K-major;
// B: the activations [T][n_h * K].
template <bool A_MN>
static mla_status_t run_heads(const void* w, int a_rows, int a_cols, int a_rows_per_head, const void* x, int n_h,
                              int K, int T, int m_tiles, void* out, cudaStream_t st) {
  CUtensorMap mA, mB;
  const bool ok = (A_MN ? map_2d(&mA, w, (uint64_t)a_cols, (uint64_t)a_rows, (uint64_t)a_cols * 2, 64, 64)
                        : map_rows_chunks(&mA, w, (uint64_t)a_cols, (uint64_t)a_rows, (uint64_t)a_cols * 2, 128, 1)) &&
                  map_rows_chunks(&mB, x, (uint64_t)n_h * K, (uint64_t)T, (uint64_t)n_h * K * 2,
                                  (uint32_t)HeadsCfg::TN, 1);
  if (!ok) return MLA_ERR_CUDA;
  HeadsArgs ha;
  ha.n_h = n_h;
  ha.T = T;
  ha.a_rows_per_head = a_rows_per_head;
  ha.k_chunks = K / 64;
  ha.m_tiles = m_tiles;
  ha.n_tiles = (T + HeadsCfg::TN - 1) / HeadsCfg::TN;
  ha.units = n_h * ha.m_tiles * ha.n_tiles;
  ha.out_rows = m_tiles * 128;
  ha.out = (__nv_bfloat16*)out;
  auto kfn = mla_heads_gemm_kernel<A_MN>;
  cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, HeadsCfg::SMEM);
  const int grid = std::min(ha.units, num_sms());
  return launch_pdl(kfn, dim3(grid), dim3(HeadsCfg::THREADS), HeadsCfg::SMEM, st, 1, mA, mB, ha) == cudaSuccess
             ? MLA_OK
             : MLA_ERR_CUDA;
}

// [q^C ; q^R] = [W^UQ ; W^QR] c^Q (eq 13 + decoupled query, RoPE on q^R), then
// (q_lat non-null) q_lat_i = (W^UK_i)^T q^C_i.
static mla_status_t queries_from_cq(const mla_layer_desc* D, const mla_weights* w, const void* qsrc,
                                    const int32_t* pos, int T, __nv_bfloat16* qc, void* q_lat, void* q_rope,
                                    cudaStream_t st) {
  const int nq = D->n_h * D->d_h, nr = D->n_h * D->d_hr;
  const int q_in = D->d_cq ? D->d_cq : D->d;
  mla_status_t s;
  {
    GemmCall c{};
    c.a0 = w->w_uq;
    c.rows0 = nq;
    c.a1 = w->w_qr;
    c.rows1 = nr;
    c.a_row_elems = q_in;
    c.x = qsrc;
    c.x_rows = T;
    c.x_row_elems = q_in;
    c.K = q_in;
    c.T = T;
    c.Z = 1;
    GemmEpi e{};
    e.kind = EPI_Q;
    e.rope = rope_table(rope_of(D), D->d_hr);
    e.pos = pos;
    e.d_hr = D->d_hr;
    e.nq = nq;
    e.n_h = D->n_h;
    e.q_c = qc;
    e.q_rope = (__nv_bfloat16*)q_rope;
    if ((s = run_gemm(c, e, plan_q2(D, T), st)) != MLA_OK) return s;
  }
  if (!q_lat) return MLA_OK;  // queries only (the un-absorbed prefill reads q^C)
  // q_lat_i = (W^UK_i)^T q^C_i : per head, A = W^UK_i viewed MN-major (its
  // [d_h][d_c] block), all (head, row tile, token tile) units on one
  // persistent CTA per SM; d_c is a multiple of 128 for the bf16 kernels
  return run_heads<true>(w->w_uk, nq, D->d_c, D->d_h, qc, D->n_h, D->d_h, T, D->d_c / 128, q_lat, st);
}

// q_c_out: write q^C [T, n_h, d_h] there (the un-absorbed prefill's queries);
// q_lat may then be null (no W^UK absorption).
static mla_status_t tc_absorb_q(const mla_layer_desc* D, const mla_weights* w, const void* h, const int32_t* pos,
                                int T, void* q_lat, void* q_rope, void* ws, size_t ws_bytes, cudaStream_t st,
                                void* q_c_out = nullptr) {
  if (!aligned16(h) || !aligned16(w->w_uq) || !aligned16(w->w_qr) || !aligned16(w->w_uk) ||
      (D->d_cq && !aligned16(w->w_dq)) || !aligned16(q_lat) || !aligned16(q_rope) ||
      (D->d_cq && D->latent_norm && !aligned16(w->g_q)) || (q_c_out && !aligned16(q_c_out)))
    return MLA_ERR_INVALID_ARG;
  Carver cv = carve(ws, ws_bytes);
  QueryWs q;
  if (!carve_queries(cv, D, T, !q_c_out, false, &q) || !ws) return MLA_ERR_CAPACITY;
  __nv_bfloat16* qc = q_c_out ? (__nv_bfloat16*)q_c_out : q.qc;
  mla_status_t s;
  if (D->d_cq) {  // c^Q = W^DQ h   (eq 12)
    GemmCall c{};
    c.a0 = w->w_dq;
    c.rows0 = D->d_cq;
    c.a_row_elems = D->d;
    c.x = h;
    c.x_rows = T;
    c.x_row_elems = D->d;
    c.K = D->d;
    c.T = T;
    c.Z = 1;
    GemmEpi e{};
    e.kind = q.cq32 ? EPI_F32 : EPI_BF16;  // fp32 c^Q: the latent RMSNorm writes the bf16 c^Q
    e.out = q.cq32 ? (void*)q.cq32 : (void*)q.cq;
    e.out_t = D->d_cq;
    if ((s = run_gemm(c, e, plan_q1(D, T), st)) != MLA_OK) return s;
    if (q.cq32 && (s = cq_norm_pass(D, w, q.cq32, q.cq, T, st)) != MLA_OK) return s;
  }
  return queries_from_cq(D, w, D->d_cq ? (const void*)q.cq : h, pos, T, qc, q_lat, q_rope, st);
}

// mla_compress_append followed by mla_absorb_q on the same tokens, with
// W^DQ sharing the first GEMM with [W^DKV ; W^KR] (all three multiply h):
// one launch of 5 + 12 row tiles at V2 shapes instead of two.
static mla_status_t tc_compress_absorb(const mla_layer_desc* D, const mla_weights* w, const void* h,
                                       const int32_t* seq_idx, const int32_t* pos, int T, mla_paged_cache* cache,
                                       void* q_lat, void* q_rope, void* ws, size_t ws_bytes, cudaStream_t st) {
  if (!D->d_cq) {
    mla_status_t s = tc_compress_append(D, w, h, seq_idx, pos, T, cache, ws, ws_bytes, st);
    return s != MLA_OK ? s : tc_absorb_q(D, w, h, pos, T, q_lat, q_rope, ws, ws_bytes, st);
  }
  if (!aligned16(h) || !aligned16(w->w_dkv) || !aligned16(w->w_kr) || !aligned16(w->w_dq) ||
      !aligned16(cache->pool) || !aligned16(w->w_uq) || !aligned16(w->w_qr) || !aligned16(w->w_uk) ||
      !aligned16(q_lat) || !aligned16(q_rope) || (D->latent_norm && (!aligned16(w->g_kv) || !aligned16(w->g_q))))
    return MLA_ERR_INVALID_ARG;
  Carver cv = carve(ws, ws_bytes);
  QueryWs q;
  if (!carve_queries(cv, D, T, true, true, &q) || !ws) return MLA_ERR_CAPACITY;
  // [c^KV ; k^R ; c^Q] = [W^DKV ; W^KR ; W^DQ] h  (eqs 9, 12 + decoupled key)
  GemmCall c{};
  c.a0 = w->w_dkv;
  c.rows0 = D->d_c;
  c.a1 = w->w_kr;
  c.rows1 = D->d_hr;
  c.a2 = w->w_dq;
  c.rows2 = D->d_cq;
  c.a_row_elems = D->d;
  c.x = h;
  c.x_rows = T;
  c.x_row_elems = D->d;
  c.K = D->d;
  c.T = T;
  c.Z = 1;
  GemmEpi e = cache_epi(D, seq_idx, pos, cache, q.lat);
  e.cq_out = q.cq32 ? (void*)q.cq32 : (void*)q.cq;
  e.cq_f32 = q.cq32 ? 1 : 0;
  e.d_cq = D->d_cq;
  mla_status_t s = run_gemm(c, e, plan_compress_q(D, T), st);
  if (s != MLA_OK) return s;
  if (q.lat && (s = kv_second_pass(D, w, q.lat, seq_idx, pos, T, cache, st)) != MLA_OK) return s;
  if (q.cq32 && (s = cq_norm_pass(D, w, q.cq32, q.cq, T, st)) != MLA_OK) return s;
  return queries_from_cq(D, w, q.cq, pos, T, q.qc, q_lat, q_rope, st);
}

// from_o: the input is o [T, n_h, d_h] itself (un-absorbed prefill): W^O only.
static mla_status_t tc_out_proj(const mla_layer_desc* D, const mla_weights* w, const void* o_lat, int T, float* u,
                                void* ws, size_t ws_bytes, cudaStream_t st, bool from_o = false) {
  if (!aligned16(o_lat) || !aligned16(w->w_uv) || !aligned16(w->w_o)) return MLA_ERR_INVALID_ARG;
  Carver cv = carve(ws, ws_bytes);
  const int nq = D->n_h * D->d_h;
  __nv_bfloat16* o = from_o ? (__nv_bfloat16*)o_lat : (__nv_bfloat16*)cv.take((size_t)T * nq * 2);
  if (!from_o && (!ws || !cv.ok())) return MLA_ERR_CAPACITY;
  mla_status_t s;
  // With enough heads, o_i = W^UV_i o_lat_i (eq 11 absorbed) runs as one
  // persistent CTA per SM over the (head, row tile) units, A = W^UV_i
  // [d_h, d_c] read K-major; few heads (V2-Lite: 16 tiles) keep the batched
  // GEMM, whose K split over a cluster covers the SMs.
  const bool per_head = D->d_h % 128 == 0 && D->n_h * (D->d_h / 128) * 2 >= num_sms();
  if (!from_o && per_head) {
    if ((s = run_heads<false>(w->w_uv, nq, D->d_c, D->d_h, o_lat, D->n_h, D->d_c, T, D->d_h / 128, o, st)) !=
        MLA_OK)
      return s;
  } else if (!from_o) {  // o_i = W^UV_i o_lat_i as a batched GEMM over the heads
    GemmCall c{};
    c.a0 = w->w_uv;
    c.rows0 = D->d_h;
    c.a_row_elems = D->d_c;
    c.x = o_lat;
    c.x_rows = T;
    c.x_row_elems = (long long)D->n_h * D->d_c;
    c.K = D->d_c;
    c.T = T;
    c.Z = D->n_h;
    c.a_z_rows = D->d_h;
    c.b_z_cols = D->d_c;
    GemmEpi e{};  // o[t][head][d_h]
    e.kind = EPI_BF16;
    e.out = o;
    e.out_z = D->d_h;
    e.out_t = nq;
    if ((s = run_gemm(c, e, plan_o1(D, T), st)) != MLA_OK) return s;
  }
  {  // u = W^O o   (eq 8)
    GemmCall c{};
    c.a0 = w->w_o;
    c.rows0 = D->d;
    c.a_row_elems = nq;
    c.x = o;
    c.x_rows = T;
    c.x_row_elems = nq;
    c.K = nq;
    c.T = T;
    c.Z = 1;
    GemmEpi e{};
    e.kind = EPI_F32;
    e.out = u;
    e.out_t = D->d;
    if ((s = run_gemm(c, e, plan_o2(D, T), st)) != MLA_OK) return s;
  }
  return MLA_OK;
}

// Merge R partials [R][rows][n_h][d_c] (+ lse [R][rows][n_h]) into o (desc dtype) and lse.
static mla_status_t tc_lse_merge(const mla_layer_desc* D, const float* o_parts, const float* lse_parts, int R, int rows,
                                 void* o, float* lse, cudaStream_t st) {
  if (D->dtype == MLA_F32 || D->d_c != ATT_DC || D->n_h % COMBINE_HEADS != 0) {
    MLA_COUNT_LAUNCH();
    mla_lse_merge_any_kernel<<<rows * D->n_h, 128, 0, st>>>(o_parts, lse_parts, R, rows, D->n_h, D->d_c, (float*)o,
                                                             lse);
    return cudaGetLastError() == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
  }
  if (!aligned16(o_parts) || !aligned16(o)) return MLA_ERR_INVALID_ARG;
  const int blocks = rows * (D->n_h / COMBINE_HEADS);
  const int cs = blocks >= 2 * num_sms() ? 1 : blocks >= num_sms() ? 2 : 4;
  auto kfn = cs == 1 ? mla_lse_merge_kernel<1> : cs == 2 ? mla_lse_merge_kernel<2> : mla_lse_merge_kernel<4>;
  return launch_pdl(kfn, dim3(blocks, cs), dim3(COMBINE_THREADS), 0, st, 1, o_parts, lse_parts, R, rows, D->n_h,
                    (__nv_bfloat16*)o, (float*)nullptr, lse) == cudaSuccess
             ? MLA_OK
             : MLA_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// un-absorbed chunked prefill (tc_prefill.cuh)
// ---------------------------------------------------------------------------
// rows[b * max_blocks + j]: first pool row of page j of sequence b, or -1 past
// the sequence's end after the chunk (q_start[b] + q_per_seq rows)
__global__ void mla_page_rows_kernel(const int32_t* __restrict__ table, const int32_t* __restrict__ q_start,
                                     int q_per_seq, int B, int max_blocks, int num_blocks, int32_t* __restrict__ rows) {
  pdl_trigger();
  pdl_wait();
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= B * max_blocks) return;
  const int b = i / max_blocks, j = i % max_blocks;
  int r = -1;
  if (j * 64 < q_start[b] + q_per_seq) {
    const int blk = table[i];
    if (blk >= 0 && blk < num_blocks) r = blk * 64;
    else record_error(ERR_CAPACITY, 704);
  }
  rows[i] = r;
}

// Scratch of the un-absorbed prefill: page rows and the decompressed keys
// and values of every pool row, [num_blocks * 64][2 * n_h * d_h] bf16.
inline size_t ws_prefill_unabsorbed(const mla_layer_desc* D, int num_blocks, int B, int max_blocks) {
  Carver c{nullptr, 0};
  c.take((size_t)B * max_blocks * 4);
  c.take((size_t)num_blocks * 64 * 2 * D->n_h * D->d_h * 2);
  return c.used + 256;
}

static mla_status_t tc_prefill_unabsorbed(const mla_layer_desc* D, const mla_weights* w, const void* q_c,
                                          const void* q_rope, const mla_paged_cache* cache, const int32_t* q_start,
                                          int q_per_seq, int B, void* ws, size_t ws_bytes, void* o, float* lse,
                                          cudaStream_t st) {
  if (D->d_h != 128 || !aligned16(q_c) || !aligned16(q_rope) || !aligned16(o) || !aligned16(w->w_uk) ||
      !aligned16(w->w_uv) || !aligned16(cache->pool))
    return D->d_h != 128 ? MLA_ERR_UNSUPPORTED : MLA_ERR_INVALID_ARG;
  Carver cv = carve(ws, ws_bytes);
  int32_t* rows = (int32_t*)cv.take((size_t)B * cache->max_blocks * 4);
  __nv_bfloat16* kv = (__nv_bfloat16*)cv.take((size_t)cache->num_blocks * 64 * 2 * D->n_h * D->d_h * 2);
  if (!ws || !cv.ok()) return MLA_ERR_CAPACITY;
  const int n_pages = B * cache->max_blocks;
  if (launch_pdl(mla_page_rows_kernel, dim3((n_pages + 255) / 256), dim3(256), 0, st, 1, cache->block_table, q_start,
                 q_per_seq, B, cache->max_blocks, cache->num_blocks, rows) != cudaSuccess)
    return MLA_ERR_CUDA;
  const int nq = D->n_h * D->d_h;
  {  // [k^C ; v^C] of every page of the chunk's sequences: [W^UK ; W^UV] c^KV (eqs 10-11)
    GemmCall c{};
    c.a0 = w->w_uk;
    c.rows0 = nq;
    c.a1 = w->w_uv;
    c.rows1 = nq;
    c.a_row_elems = D->d_c;
    c.x = cache->pool;
    c.x_rows = (long long)cache->num_blocks * 64;
    c.x_row_elems = D->d_c;  // the c^KV columns of each [c^KV | k^R] row
    c.K = D->d_c;
    c.T = cache->num_blocks * 64;
    c.Z = 1;
    c.b_tile_row = rows;
    c.n_tiles_override = n_pages;
    GemmEpi e{};
    e.kind = EPI_BF16;
    e.out = kv;
    e.out_t = 2LL * nq;
    GemmPlan p;
    p.tn = 64;  // one cache page per token tile
    p.n_tiles = n_pages;
    p.deep = false;
    p.splits = 1;
    p.kcs = D->d_c / GEMM_BK;
    mla_status_t s = run_gemm_paged(c, e, p, (uint64_t)(D->d_c + D->d_hr) * 2, st);
    if (s != MLA_OK) return s;
  }
  CUtensorMap mq, mr, mkv, mkr;
  const long long T = (long long)B * q_per_seq;
  bool ok = map_2d(&mq, q_c, (uint64_t)nq, (uint64_t)T, (uint64_t)nq * 2, 64, 128);
  ok = ok && map_2d(&mr, q_rope, (uint64_t)D->n_h * D->d_hr, (uint64_t)T, (uint64_t)D->n_h * D->d_hr * 2, 64, 128);
  ok = ok && map_2d(&mkv, kv, 2ULL * nq, (uint64_t)cache->num_blocks * 64, 4ULL * nq, 64, 64);
  ok = ok && map_2d(&mkr, cache->pool, (uint64_t)(D->d_c + D->d_hr), (uint64_t)cache->num_blocks * 64,
                    (uint64_t)(D->d_c + D->d_hr) * 2, 64, 64);
  if (!ok) return MLA_ERR_CUDA;
  PrefillArgs a;
  a.n_h = D->n_h;
  a.q_per_seq = q_per_seq;
  a.num_blocks = cache->num_blocks;
  a.max_blocks = cache->max_blocks;
  a.scale_log2 = (float)(D->attn_logit_factor / sqrt((double)(D->d_h + D->d_hr)) * 1.4426950408889634);
  a.table = cache->block_table;
  a.q_start = q_start;
  a.o = (__nv_bfloat16*)o;
  a.lse = lse;
  cudaFuncSetAttribute(mla_prefill_unabsorbed_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, PfCfg::SMEM);
  const dim3 grid((q_per_seq + 127) / 128, D->n_h, B);
  return launch_pdl(mla_prefill_unabsorbed_kernel, grid, dim3(PfCfg::THREADS), PfCfg::SMEM, st, 1, mq, mr, mkv, mkr,
                    a) == cudaSuccess
             ? MLA_OK
             : MLA_ERR_CUDA;
}

template <int H>
static cudaError_t launch_attn(const CUtensorMap& mq, const CUtensorMap& mr, const CUtensorMap& mc,
                               const CUtensorMap& mr8, const CUtensorMap& ms8, bool f8, const AttnArgs& a, dim3 grid,
                               cudaStream_t st) {
  if (f8) {
    auto kfn = mla_attn_kernel<H, true>;
    constexpr int smem = AttnCfg<H, true>::SMEM;
    cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    return launch_pdl(kfn, grid, dim3(AttnCfg<H, true>::THREADS), smem, st, 1, mq, mr, mc, mr8, ms8, a);
  }
  auto kfn = mla_attn_kernel<H, false>;
  constexpr int smem = AttnCfg<H, false>::SMEM;
  cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  return launch_pdl(kfn, grid, dim3(AttnCfg<H, false>::THREADS), smem, st, 1, mq, mr, mc, mc, mc, a);
}

// Measurement hook (mla_debug_attention_events): events recorded on the
// attention call's stream right before and after its attention kernel (after
// the work plan, before the combine), so that the kernel alone can be timed.
inline cudaEvent_t g_attn_ev_before = nullptr, g_attn_ev_after = nullptr;

// kv_begin (partial decode): rows [kv_begin[b], kv_len[b]) only, every row
// written in fp32 to o_f32 (o_lat unused) with its lse.
static mla_status_t tc_attention(const mla_layer_desc* D, const void* q_lat, const void* q_rope,
                                 const mla_paged_cache* cache, const int32_t* kv_len, const int32_t* q_start,
                                 int q_per_seq, int rows, void* ws, size_t ws_bytes, int num_splits, void* o_lat,
                                 float* lse, cudaStream_t st, int workers = 0, const int32_t* kv_begin = nullptr,
                                 float* o_f32 = nullptr) {
  if (!aligned16(q_lat) || !aligned16(q_rope) || !aligned16(cache->pool) || !aligned16(kv_begin ? o_f32 : o_lat))
    return MLA_ERR_INVALID_ARG;
  const int H = heads_per_cta(D);
  const int max_len = cache->max_blocks * 64;
  const bool partial = kv_begin != nullptr;
  const AttnPlan p = plan_attn(D, rows, max_len, kv_len ? (partial && num_splits == 1 ? 0 : num_splits) : 1, workers,
                               partial);
  Carver cv = carve(ws, ws_bytes);
  AttnWs aw{};
  if (p.use_plan && (!ws || !carve_attn(cv, D, rows, p, &aw))) return MLA_ERR_CAPACITY;
  if (p.use_plan) {
    const int threads = std::min(1024, std::max(32, (rows + 31) / 32 * 32));
    if (launch_pdl(mla_attn_plan_kernel, dim3(1), dim3(threads), 0, st, 1, kv_len, q_start, q_per_seq, rows,
                   max_len, p.workers, p.splits, p.max_units, p.max_slots, aw.units, aw.row_info, aw.work,
                   aw.n_units, kv_begin, partial ? 1 : 0) != cudaSuccess)
      return MLA_ERR_CUDA;
  }
  const bool pair = use_pair_kernel(D);
  const uint32_t q_box = pair ? 64u : (uint32_t)H;  // query rows per CTA
  CUtensorMap mq, mr, mc;
  bool ok = map_2d(&mq, q_lat, ATT_DC, (uint64_t)rows * D->n_h, ATT_DC * 2, 64, q_box);
  ok = ok && map_2d(&mr, q_rope, ATT_DR, (uint64_t)rows * D->n_h, ATT_DR * 2, 64, q_box);
  const bool f8 = fp8_cache(D);
  CUtensorMap mr8, ms8;  // FP8 rows: k^R view and scales (m_cache: the codes)
  if (f8) {
    const int rb = cache_row_bytes(D);
    ok = ok && map_cache_bytes(&mc, cache->pool, cache->num_blocks, rb, 128);
    ok = ok && map_cache_bf16_view(&mr8, cache->pool, cache->num_blocks, rb);
    ok = ok && map_cache_bytes(&ms8, cache->pool, cache->num_blocks, rb, 16);
  } else {
    ok = ok && map_cache(&mc, cache->pool, cache->num_blocks, ATT_DC + ATT_DR);
    mr8 = ms8 = mc;
  }
  if (!ok) return MLA_ERR_CUDA;
  AttnArgs a;
  a.n_h = D->n_h;
  a.rows = rows;
  a.q_per_seq = q_per_seq;
  a.num_blocks = cache->num_blocks;
  a.max_blocks = cache->max_blocks;
  a.scale_log2 = (float)(D->attn_logit_factor / sqrt((double)(D->d_h + D->d_hr)) * 1.4426950408889634);
  a.table = cache->block_table;
  a.pool = (const uint8_t*)cache->pool;
  a.kv_len = kv_len;
  a.kv_begin = kv_begin;
  a.q_start = q_start;
  a.o_lat = (__nv_bfloat16*)o_lat;
  a.lse = lse;
  a.units = aw.units;
  a.work = aw.work;
  a.o_part = aw.o_part;
  a.lse_part = aw.lse_part;
  cudaError_t e;
  if (g_attn_ev_before && cudaEventRecord(g_attn_ev_before, st) != cudaSuccess) return MLA_ERR_CUDA;
  if (pair) {
    dim3 grid(2 * p.workers);
    // cluster dimensions are compiled in (__cluster_dims__)
    if (f8) {
      // RoPE chunks through a bf16 view of the rows; the codes as bytes (mc)
      CUtensorMap m1;
      if (!map_fp8_rope_chunks(&m1, cache->pool, cache->num_blocks, cache_row_bytes(D))) return MLA_ERR_CUDA;
      using PC = PairCfgT<true>;
      cudaFuncSetAttribute(mla_attn_pair_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, PC::SMEM);
      e = launch_pdl(mla_attn_pair_kernel<true>, grid, dim3(PC::THREADS), PC::SMEM, st, 1, mq, mr, m1, mc, a);
    } else {
      CUtensorMap m1, m2;
      if (!map_cache_chunks(&m1, cache->pool, cache->num_blocks, ATT_DC + ATT_DR, 1) ||
          !map_cache_chunks(&m2, cache->pool, cache->num_blocks, ATT_DC + ATT_DR, 2))
        return MLA_ERR_CUDA;
      cudaFuncSetAttribute(mla_attn_pair_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, PairCfg::SMEM);
      e = launch_pdl(mla_attn_pair_kernel<false>, grid, dim3(PairCfg::THREADS), PairCfg::SMEM, st, 1, mq, mr, m1, m2,
                     a);
    }
  } else {
    dim3 grid(p.workers * attn_groups(D));
    e = H == 16 ? launch_attn<16>(mq, mr, mc, mr8, ms8, f8, a, grid, st)
                : launch_attn<32>(mq, mr, mc, mr8, ms8, f8, a, grid, st);
  }
  if (e != cudaSuccess) return MLA_ERR_CUDA;
  if (g_attn_ev_after && cudaEventRecord(g_attn_ev_after, st) != cudaSuccess) return MLA_ERR_CUDA;
  if (p.max_slots > 0) {
    // enough blocks for two per SM: split the latent columns when there are few rows
    const int blocks = rows * (D->n_h / COMBINE_HEADS);
    const int cs = blocks >= 2 * num_sms() ? 1 : blocks >= num_sms() ? 2 : 4;
    const dim3 grid(blocks, cs);
    auto kfn = cs == 1 ? mla_combine_kernel<1> : cs == 2 ? mla_combine_kernel<2> : mla_combine_kernel<4>;
    if (launch_pdl(kfn, grid, dim3(COMBINE_THREADS), 0, st, 1, (const float*)aw.o_part, (const float*)aw.lse_part,
                   (const int4*)aw.row_info, D->n_h, (__nv_bfloat16*)o_lat, lse, o_f32, kv_begin, kv_len) !=
        cudaSuccess)
      return MLA_ERR_CUDA;
  }
  return MLA_OK;
}
