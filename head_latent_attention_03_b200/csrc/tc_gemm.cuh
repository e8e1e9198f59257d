// tc_gemm.cuh — weight-streaming bf16 GEMM on the 5th-generation tensor cores,
// with the K-split reduction and the projection's epilogue fused in.
//
//   Y[z][t][n] = epilogue( sum_k A_z[n][k] * X_z[t][k] )
//
// A holds weight rows (output features n, on the MMA's M = 128), X holds the
// token activations (tokens t on the MMA's N).  Putting the weights on M keeps
// the 128-lane accumulator full at decode batch sizes (T = 32 or 64 tokens),
// where every projection of the MLA layer is bound by streaming its weights.
//
// A tile's K range is split over the S CTAs of one thread-block cluster
// (S <= 8), so that a wave of CTAs covers the GPU even when a projection has
// few 128-row tiles.  Each CTA accumulates its K slice in TMEM, parks the fp32
// tile in its own shared memory, and after a cluster barrier CTA s sums rows
// [128 s / S, 128 (s+1) / S) of all S tiles over distributed shared memory, in
// rank order (deterministic), and applies the epilogue: bf16 or fp32 store,
// RoPE of the decoupled key/query features, or the paged-cache scatter of
// [c^KV | k^R].  No partial sums reach global memory.
//
// Warps (192 threads):
//   warp 0      TMA producer (A and X tiles, 64-wide K chunks, SW128)
//   warp 1      MMA issuer (one elected thread) and TMEM owner
//   warps 2..5  TMEM -> shared memory; all six warps share the reduction
// Launched with programmatic stream serialisation: set-up and an L2 prefetch
// of the first weight tiles overlap the previous kernel of the step; every
// load into shared memory and every output store waits for it.
// A is K-major ([n][k] rows) or, for the per-head absorbed W^UK, MN-major
// (memory [k][n], n contiguous).  Up to three weight segments that multiply
// the same activations (e.g. W^DKV, W^KR and W^DQ, all applied to h) share one
// launch: M tiles below m_tiles0 read map A0, the next m_tiles1 map A1, the
// rest A2; the epilogue sees the features of the segments one after another.
#pragma once

#include "common.cuh"
#include "rope.cuh"

namespace mla {

enum GemmEpiKind : int {
  EPI_F32 = 0,    // fp32 y[z][t][n]
  EPI_BF16 = 1,   // bf16 y[z][t][n]
  EPI_CACHE = 2,  // features [0, d_c): c^KV; [d_c, d_c + d_hr): RoPE_pos(k^R); bf16 into the paged cache;
                  // [d_c + d_hr, d_c + d_hr + d_cq): c^Q (bf16 or fp32 [t][d_cq]) when W^DQ shares the launch
  EPI_Q = 3,      // features [0, nq): q^C (bf16 [t][nq]); [nq, nq + n_h d_hr): RoPE_pos(q^R) (bf16)
};

struct GemmEpi {
  int kind;
  void* out;                 // EPI_F32 / EPI_BF16
  long long out_z, out_t;    // element strides of y (feature stride 1)
  RopeTable rope;            // EPI_CACHE / EPI_Q: theta_k of the layer
  const int32_t* pos;        // [T]
  int d_hr;
  // EPI_CACHE
  int d_c;
  float* lat_f32;            // non-null: c^KV goes here ([t][d_c] fp32) for the second pass (latent
                             // RMSNorm, FP8 encoding), not to the cache
  const int32_t* seq_idx;    // [T]
  uint8_t* pool;             // rows of row_bytes; k^R (bf16) at byte rope_off of its row
  int num_blocks, max_blocks, block_size, row_bytes, rope_off;
  const int32_t* table;
  void* cq_out;              // c^Q of the W^DQ segment: bf16, or fp32 when cq_f32
  int cq_f32, d_cq;
  // EPI_Q
  int nq, n_h;
  __nv_bfloat16* q_c;
  __nv_bfloat16* q_rope;
};

struct GemmArgs {
  int k_chunks;        // K / 64 (whole contraction)
  int k_chunks_split;  // chunks per split
  int splits;          // CTAs per cluster (K splits of one tile)
  int m_tiles0, m_tiles1;      // M tiles of segments 0 and 1 (segment 2 has the rest)
  int n_out0, n_out1, n_out2;  // rows of the segments (0: the segment is absent)
  int T;               // tokens
  int a_z_rows;        // per-batch row offset into A (K-major: output rows; MN-major: K rows)
  int b_z_cols;        // per-batch column offset into X
  // optional: token tile nt reads (and writes) rows b_tile_row[nt] .. + TN of
  // X and Y (cache pages scattered over the pool); nullptr: rows nt * TN ..
  const int32_t* b_tile_row;
  GemmEpi e;
};

constexpr int GEMM_THREADS = 192;
constexpr int GEMM_BM = 128, GEMM_BK = 64;

#ifndef MLA_GEMM_KC
#define MLA_GEMM_KC 1  // 64-column K chunks per weight TMA box (K-major weights)
#endif

// A stage holds KC consecutive 64-wide K chunks of the weight tile and of the
// activations, each fetched by one TMA box (rows x KC chunks).  DEEP: one CTA
// per SM with up to 8 stages in flight (projections whose tiles fit one wave
// of SMs); otherwise two CTAs per SM with about 100 KB each (projections with
// more tiles than SMs).
template <int TN, int KC, bool DEEP>
struct GemmCfg {
  static constexpr int A_CHUNK = GEMM_BM * GEMM_BK * 2;  // 16 KB
  static constexpr int B_CHUNK = TN * GEMM_BK * 2;
  static constexpr int A_BYTES = KC * A_CHUNK;
  static constexpr int B_BYTES = KC * B_CHUNK;
  static constexpr int STAGE = A_BYTES + B_BYTES;
  static constexpr bool TWO = !DEEP && TN <= 64 && 2 * STAGE <= 104 * 1024;
  static constexpr int BUDGET = TWO ? 104 * 1024 : 200 * 1024;
  static constexpr int NST = (BUDGET / STAGE) < 8 ? (BUDGET / STAGE) : 8;
  static constexpr int RED_BYTES = TN * GEMM_BM * 4;     // fp32 tile, [t][row]
  static constexpr int TMEM_COLS = TN <= 32 ? 32 : TN <= 64 ? 64 : TN <= 128 ? 128 : 256;
  static constexpr int SMEM = NST * STAGE + 1024 /*align*/ + 256 /*barriers*/;
  static constexpr int CTAS_PER_SM = TWO ? 2 : 1;
  static_assert(NST >= 2, "pipeline depth");
  static_assert(RED_BYTES <= NST * STAGE, "the reduction tile reuses the pipeline stages");
};

// Final value of features (n, n+1) of token t in batch z.
__device__ __forceinline__ void gemm_epilogue(const GemmEpi& e, int z, int t, int n, float2 v) {
  switch (e.kind) {
    case EPI_F32:
      *reinterpret_cast<float2*>(reinterpret_cast<float*>(e.out) + z * e.out_z + t * e.out_t + n) = v;
      break;
    case EPI_BF16:
      *reinterpret_cast<__nv_bfloat162*>(reinterpret_cast<__nv_bfloat16*>(e.out) + z * e.out_z + t * e.out_t + n) =
          __floats2bfloat162_rn(v.x, v.y);
      break;
    case EPI_CACHE: {
      if (n >= e.d_c + e.d_hr) {  // c^Q (eq 12), the W^DQ segment
        const long long o = (long long)t * e.d_cq + (n - e.d_c - e.d_hr);
        if (e.cq_f32)
          *reinterpret_cast<float2*>(reinterpret_cast<float*>(e.cq_out) + o) = v;
        else
          *reinterpret_cast<__nv_bfloat162*>(reinterpret_cast<__nv_bfloat16*>(e.cq_out) + o) =
              __floats2bfloat162_rn(v.x, v.y);
        break;
      }
      const long long p = e.pos[t];
      if (n < e.d_c && e.lat_f32) {
        *reinterpret_cast<float2*>(e.lat_f32 + (long long)t * e.d_c + n) = v;
        break;
      }
      if (n >= e.d_c) {
        float c, s;
        rope_cos_sin_reduced(e.rope.theta[(n - e.d_c) / 2], p, &c, &s);
        const float a = v.x, b = v.y;
        v.x = a * c - b * s;
        v.y = a * s + b * c;
      }
      const int page = (int)(p / e.block_size);
      const int blk = (page >= 0 && page < e.max_blocks) ? e.table[(long long)e.seq_idx[t] * e.max_blocks + page] : -1;
      if (blk < 0 || blk >= e.num_blocks) {
        if (n == 0) record_error(ERR_CAPACITY, 301);
        break;
      }
      uint8_t* rowp = e.pool + ((long long)blk * e.block_size + p % e.block_size) * e.row_bytes;
      uint8_t* dst = n < e.d_c ? rowp + 2 * n : rowp + e.rope_off + 2 * (n - e.d_c);
      *reinterpret_cast<__nv_bfloat162*>(dst) = __floats2bfloat162_rn(v.x, v.y);
      break;
    }
    case EPI_Q: {
      if (n < e.nq) {
        *reinterpret_cast<__nv_bfloat162*>(e.q_c + (long long)t * e.nq + n) = __floats2bfloat162_rn(v.x, v.y);
        break;
      }
      const int r = n - e.nq;  // = head * d_hr + 2k
      float c, s;
      rope_cos_sin_reduced(e.rope.theta[(r % e.d_hr) / 2], e.pos[t], &c, &s);
      const float a = v.x, b = v.y;
      *reinterpret_cast<__nv_bfloat162*>(e.q_rope + (long long)t * e.n_h * e.d_hr + r) =
          __floats2bfloat162_rn(a * c - b * s, a * s + b * c);
      break;
    }
    default:
      break;
  }
}

// Grid: x = M tile * splits + split (clusters of `splits` along x), y = token
// tile, z = batch.
template <int TN, bool A_MN, int KC, bool DEEP>
__global__ void __launch_bounds__(GEMM_THREADS, GemmCfg<TN, KC, DEEP>::CTAS_PER_SM)
    gemm_bf16_kernel(const __grid_constant__ CUtensorMap mA0, const __grid_constant__ CUtensorMap mA1,
                     const __grid_constant__ CUtensorMap mA2,
                     const __grid_constant__ CUtensorMap mB, const GemmArgs g) {
  using C = GemmCfg<TN, KC, DEEP>;
  static_assert(TN % 16 == 0 && TN >= 16 && TN <= 256, "token tile");
  static_assert(!A_MN || KC == 1, "MN-major weights load one chunk per stage");
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::NST * C::STAGE);
  uint64_t* empty = full + C::NST;
  uint64_t* done = empty + C::NST;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* red = reinterpret_cast<float*>(smem);  // [TN][128] fp32 after the main loop

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int S = g.splits;
  const int mt = blockIdx.x / S, ks = blockIdx.x % S;  // ks = rank in the cluster
  const int nt = blockIdx.y, z = blockIdx.z;
  const int kc0 = ks * g.k_chunks_split;
  int nk = max(0, min(g.k_chunks_split, g.k_chunks - kc0));
  if (g.b_tile_row) {
    // a page-indexed token tile with row -1 (past its sequence) does nothing
    pdl_wait();
    if (g.b_tile_row[nt] < 0) nk = 0;
  }
  const int seg = mt < g.m_tiles0 ? 0 : mt < g.m_tiles0 + g.m_tiles1 ? 1 : 2;
  const CUtensorMap* mA = seg == 0 ? &mA0 : seg == 1 ? &mA1 : &mA2;
  const int m_row0 = (mt - (seg == 0 ? 0 : seg == 1 ? g.m_tiles0 : g.m_tiles0 + g.m_tiles1)) * GEMM_BM;
  const int n_base = seg == 0 ? 0 : seg == 1 ? g.n_out0 : g.n_out0 + g.n_out1;  // first feature of the segment

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::NST; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    mbar_init(done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(tmem_slot, C::TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_trigger();  // after the TMEM allocation: a dependent CTA on this SM allocates after it

  bool ok = true;
  if (warp == 0) {
    if (elect_one()) {
      tma_prefetch_desc(mA);
      tma_prefetch_desc(&mB);
      // stage i covers chunks [kc0 + KC i, kc0 + KC (i+1)); chunks past this
      // split's range are fetched (or zero-filled past K) but not multiplied
      const int ns = (nk + KC - 1) / KC;
      auto load_a = [&](int i, uint8_t* sa) {
        const int kc = kc0 + i * KC;
        if (!A_MN) {
          tma_load_3d(sa, mA, &full[i % C::NST], 0, z * g.a_z_rows + m_row0, kc);
        } else {
          tma_load_2d(sa, mA, &full[i % C::NST], m_row0, z * g.a_z_rows + kc * GEMM_BK);
          tma_load_2d(sa + 8192, mA, &full[i % C::NST], m_row0 + 64, z * g.a_z_rows + kc * GEMM_BK);
        }
      };
      int b_row0 = nt * TN;  // a page-indexed tile's row is read after pdl_wait below
      auto load_b = [&](int i, uint8_t* sb) {
        tma_load_3d(sb, &mB, &full[i % C::NST], 0, b_row0, z * g.b_z_cols / GEMM_BK + kc0 + i * KC);
      };
      // While the previous kernel finishes, pull this CTA's first weight
      // tiles into L2; every load into shared memory waits for it.
      const int pre = min(ns, C::NST);
      for (int i = 0; i < pre; ++i) {
        const int kc = kc0 + i * KC;
        if (!A_MN) {
          tma_prefetch_l2_3d(mA, 0, z * g.a_z_rows + m_row0, kc);
        } else {
          tma_prefetch_l2_2d(mA, m_row0, z * g.a_z_rows + kc * GEMM_BK);
          tma_prefetch_l2_2d(mA, m_row0 + 64, z * g.a_z_rows + kc * GEMM_BK);
        }
      }
      pdl_wait();
      if (g.b_tile_row) b_row0 = g.b_tile_row[nt];
      for (int i = 0; i < pre; ++i) {
        mbar_expect_tx(&full[i], C::STAGE);
        load_a(i, smem + i * C::STAGE);
        load_b(i, smem + i * C::STAGE + C::A_BYTES);
      }
      for (int i = pre; i < ns; ++i) {
        const int s = i % C::NST;
        if (!mbar_wait(&empty[s], ((i / C::NST) - 1) & 1, abort_flag, 201)) break;
        uint8_t* sa = smem + s * C::STAGE;
        mbar_expect_tx(&full[s], C::STAGE);
        load_a(i, sa);
        load_b(i, sa + C::A_BYTES);
      }
    }
  } else if (warp == 1) {
    if (elect_one()) {
      const uint32_t idesc = idesc_bf16_f32(GEMM_BM, TN, A_MN, false);
      const int ns = (nk + KC - 1) / KC;
      for (int i = 0; i < ns; ++i) {
        const int s = i % C::NST;
        if (!mbar_wait(&full[s], (i / C::NST) & 1, abort_flag, 202)) break;
        tc_fence_after();
        const uint32_t sa = smem_u32(smem + s * C::STAGE);
        const uint32_t sb = sa + C::A_BYTES;
        const int nc = min(KC, nk - i * KC);
        for (int c = 0; c < nc; ++c) {
#pragma unroll
          for (int kk = 0; kk < GEMM_BK / 16; ++kk) {
            const uint64_t ad = A_MN ? smem_desc(sa + kk * 2048, 8192, 1024, SW128)
                                     : smem_desc(sa + c * C::A_CHUNK + kk * 32, 16, 1024, SW128);
            const uint64_t bd = smem_desc(sb + c * C::B_CHUNK + kk * 32, 16, 1024, SW128);
            mma_bf16_ss(tmem, ad, bd, idesc, (i | c | kk) != 0);
          }
        }
        mma_commit(&empty[s]);
      }
      mma_commit(done);
    }
  } else {
    // TMEM -> shared memory: warp w reads TMEM lanes 32*(w%4) .. +31 (tile rows)
    const int q = warp & 3;
    const int row = q * 32 + lane;
    ok = mbar_wait(done, 0, abort_flag, 203);
    tc_fence_after();
#pragma unroll 1
    for (int c0 = 0; c0 < TN; c0 += 16) {
      float v[16];
      tmem_ld32<16>(tmem + ((uint32_t)(q * 32) << 16) + c0, v);
      tmem_wait_ld();
#pragma unroll
      for (int j = 0; j < 16; ++j) red[(c0 + j) * GEMM_BM + row] = nk > 0 ? v[j] : 0.f;
    }
  }
  __syncwarp();
  tc_fence_before();
  // every CTA of the cluster has its partial tile in shared memory
  if (S > 1)
    cluster_sync_all();
  else
    __syncthreads();
  ok = __syncthreads_and(ok ? 1 : 0) != 0;
  pdl_wait();  // outputs may be read by the previous kernel until it has finished

  // this CTA's rows of the tile, summed over the cluster in rank order
  const int r0 = ((ks * GEMM_BM) / S) & ~1, r1 = ks == S - 1 ? GEMM_BM : (((ks + 1) * GEMM_BM) / S) & ~1;
  const int n_pairs = (r1 - r0) / 2;
  const int n_seg = seg == 0 ? g.n_out0 : seg == 1 ? g.n_out1 : g.n_out2;
  const uint32_t red_addr = smem_u32(red);
  if (ok) {
    // E elements per thread and round: all their S remote loads are issued
    // before any is summed, so the DSMEM latency is paid once per round
    constexpr int E = 4, SMAX = 8;
    const int n_el = n_pairs * TN;
    for (int e0 = threadIdx.x; e0 < n_el; e0 += E * GEMM_THREADS) {
      float2 part[E][SMAX];
      uint32_t off[E];
#pragma unroll
      for (int q = 0; q < E; ++q) {
        const int e = e0 + q * GEMM_THREADS;
        const int t_loc = e / n_pairs, rr = r0 + 2 * (e % n_pairs);
        off[q] = (uint32_t)(t_loc * GEMM_BM + rr) * 4u;
        if (e >= n_el) continue;
        if (S == 1) {
          part[q][0] = *reinterpret_cast<const float2*>(reinterpret_cast<const uint8_t*>(red) + off[q]);
        } else {
#pragma unroll
          for (int sr = 0; sr < SMAX; ++sr)
            if (sr < S) part[q][sr] = ld_cluster_f2(mapa_shared(red_addr + off[q], (uint32_t)sr));
        }
      }
#pragma unroll
      for (int q = 0; q < E; ++q) {
        const int e = e0 + q * GEMM_THREADS;
        if (e >= n_el) continue;
        const int t_loc = e / n_pairs, rr = r0 + 2 * (e % n_pairs);
        const int t = (g.b_tile_row ? g.b_tile_row[nt] : nt * TN) + t_loc;
        const int n_in_seg = m_row0 + rr;
        if (t >= g.T || n_in_seg >= n_seg || (g.b_tile_row && g.b_tile_row[nt] < 0)) continue;
        float2 v = part[q][0];
#pragma unroll
        for (int sr = 1; sr < SMAX; ++sr)
          if (sr < S) {
            v.x += part[q][sr].x;
            v.y += part[q][sr].y;
          }
        gemm_epilogue(g.e, z, t, n_base + n_in_seg, v);
      }
    }
  }
  // keep this CTA's tile alive until every CTA of the cluster has read it
  if (S > 1) cluster_sync_all();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) tmem_dealloc(tmem, C::TMEM_COLS);
}

}  // namespace mla
