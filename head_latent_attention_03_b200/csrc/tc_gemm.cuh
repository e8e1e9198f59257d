// tc_gemm.cuh — weight-streaming bf16 GEMM on the 5th-generation tensor cores.
//
//   P[ks][z][t][n] = sum_{k in split ks} A_z[n][k] * X_z[t][k]      (fp32)
//
// A holds weight rows (output features n, on the MMA's M = 128), X holds the
// token activations (tokens t on the MMA's N).  Putting the weights on M keeps
// the 128-lane accumulator full at decode batch sizes (T = 32 or 64 tokens),
// where every projection of the MLA layer is bound by streaming its weights.
// One CTA computes one 128 x TN tile over one K split:
//   warp 0      TMA producer (A and X tiles, 64-wide K chunks, SW128)
//   warp 1      MMA issuer (one elected thread) and TMEM owner
//   warps 2..5  epilogue: tcgen05.ld of the accumulator, fp32 stores
// A is K-major ([n][k] rows) or, for the per-head absorbed W^UK, MN-major
// (memory [k][n], n contiguous).  Two weight segments (e.g. W^DKV and W^KR)
// can share one launch: M tiles below m_tiles0 read map A0, the rest A1.
#pragma once

#include "common.cuh"

namespace mla {

struct GemmArgs {
  int k_chunks;        // K / 64 (whole contraction)
  int k_chunks_split;  // chunks per split
  int n_tiles;         // token tiles
  int m_tiles0;        // M tiles of segment 0
  int n_out0, n_out1;  // rows of segment 0 / segment 1 (n_out1 = 0: one segment)
  int T;               // tokens
  int a_z_rows;        // per-batch row offset into A (K-major: output rows; MN-major: K rows)
  int b_z_cols;        // per-batch column offset into X
  float* out;          // fp32 partials
  long long out_split, out_z, out_t;  // element strides (feature stride is 1)
};

constexpr int GEMM_THREADS = 192;
constexpr int GEMM_BM = 128, GEMM_BK = 64;

template <int TN>
struct GemmCfg {
  static constexpr int A_BYTES = GEMM_BM * GEMM_BK * 2;  // 16 KB
  static constexpr int B_BYTES = TN * GEMM_BK * 2;
  static constexpr int STAGE = A_BYTES + B_BYTES;
  static constexpr int NST = (196 * 1024 / STAGE) < 6 ? (196 * 1024 / STAGE) : 6;
  static constexpr int TMEM_COLS = TN <= 32 ? 32 : TN <= 64 ? 64 : TN <= 128 ? 128 : 256;
  static constexpr int SMEM = NST * STAGE + 1024 /*align*/ + 256 /*barriers*/;
};

template <int TN, bool A_MN>
__global__ void __launch_bounds__(GEMM_THREADS, 1)
    gemm_bf16_kernel(const __grid_constant__ CUtensorMap mA0, const __grid_constant__ CUtensorMap mA1,
                     const __grid_constant__ CUtensorMap mB, const GemmArgs g) {
  using C = GemmCfg<TN>;
  static_assert(TN % 16 == 0 && TN >= 16 && TN <= 256, "token tile");
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::NST * C::STAGE);
  uint64_t* empty = full + C::NST;
  uint64_t* done = empty + C::NST;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int mt = blockIdx.x;
  const int nt = blockIdx.y % g.n_tiles, ks = blockIdx.y / g.n_tiles, z = blockIdx.z;
  const int kc0 = ks * g.k_chunks_split;
  const int nk = min(g.k_chunks_split, g.k_chunks - kc0);
  const bool seg1 = mt >= g.m_tiles0;
  const CUtensorMap* mA = seg1 ? &mA1 : &mA0;
  const int m_row0 = (seg1 ? mt - g.m_tiles0 : mt) * GEMM_BM;  // first row inside the segment

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

  if (warp == 0) {
    if (elect_one()) {
      tma_prefetch_desc(mA);
      tma_prefetch_desc(&mB);
      for (int i = 0; i < nk; ++i) {
        const int s = i % C::NST;
        if (i >= C::NST && !mbar_wait(&empty[s], ((i / C::NST) - 1) & 1, abort_flag, 201)) break;
        uint8_t* sa = smem + s * C::STAGE;
        uint8_t* sb = sa + C::A_BYTES;
        mbar_expect_tx(&full[s], C::STAGE);
        const int kx = (kc0 + i) * GEMM_BK;
        if (!A_MN) {
          tma_load_2d(sa, mA, &full[s], kx, z * g.a_z_rows + m_row0);
        } else {
          tma_load_2d(sa, mA, &full[s], m_row0, z * g.a_z_rows + kx);
          tma_load_2d(sa + 8192, mA, &full[s], m_row0 + 64, z * g.a_z_rows + kx);
        }
        tma_load_2d(sb, &mB, &full[s], z * g.b_z_cols + kx, nt * TN);
      }
    }
  } else if (warp == 1) {
    if (elect_one()) {
      const uint32_t idesc = idesc_bf16_f32(GEMM_BM, TN, A_MN, false);
      for (int i = 0; i < nk; ++i) {
        const int s = i % C::NST;
        if (!mbar_wait(&full[s], (i / C::NST) & 1, abort_flag, 202)) break;
        tc_fence_after();
        const uint32_t sa = smem_u32(smem + s * C::STAGE);
        const uint32_t sb = sa + C::A_BYTES;
#pragma unroll
        for (int kk = 0; kk < GEMM_BK / 16; ++kk) {
          const uint64_t ad = A_MN ? smem_desc(sa + kk * 2048, 8192, 1024, SW128)
                                   : smem_desc(sa + kk * 32, 16, 1024, SW128);
          const uint64_t bd = smem_desc(sb + kk * 32, 16, 1024, SW128);
          mma_bf16_ss(tmem, ad, bd, idesc, (i | kk) != 0);
        }
        mma_commit(&empty[s]);
      }
      mma_commit(done);
    }
  } else {
    // epilogue warps 2..5: warp w reads TMEM lanes 32*(w%4) .. +31
    const int q = warp & 3;
    const int row = q * 32 + lane;  // output feature inside the tile
    const int n_seg = seg1 ? g.n_out1 : g.n_out0;
    const int n_in_seg = m_row0 + row;
    const int n_out = (seg1 ? g.n_out0 : 0) + n_in_seg;
    const bool ok = mbar_wait(done, 0, abort_flag, 203) && nk > 0;
    tc_fence_after();
    float* dst = g.out + (long long)ks * g.out_split + (long long)z * g.out_z + n_out;
#pragma unroll 1
    for (int c0 = 0; c0 < TN; c0 += 16) {
      float v[16];
      tmem_ld32<16>(tmem + ((uint32_t)(q * 32) << 16) + c0, v);
      tmem_wait_ld();
      if (ok && n_in_seg < n_seg) {
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const int t = nt * TN + c0 + j;
          if (t < g.T) dst[(long long)t * g.out_t] = v[j];
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) tmem_dealloc(tmem, C::TMEM_COLS);
}

// ---------------------------------------------------------------------------
// finishing kernels: sum the K splits (fixed order, deterministic) and apply
// the step's epilogue.  Each thread owns one adjacent pair of features so that
// a RoPE pair (2k, 2k+1) stays in one thread.
// ---------------------------------------------------------------------------
__device__ __forceinline__ float2 sum_splits(const float* p, int splits, long long split_stride) {
  float2 a = *reinterpret_cast<const float2*>(p);
  for (int s = 1; s < splits; ++s) {
    const float2 b = *reinterpret_cast<const float2*>(p + s * split_stride);
    a.x += b.x;
    a.y += b.y;
  }
  return a;
}

// compress_append: [c^KV | RoPE_pos(k^R)] -> bf16 cache slot of (seq_idx[t], pos[t]).
__global__ void finish_compress_kernel(const float* __restrict__ part, int splits, long long split_stride, int T,
                                       int d_c, int d_hr, RopeParams rp, const int32_t* __restrict__ seq_idx,
                                       const int32_t* __restrict__ pos, __nv_bfloat16* __restrict__ pool,
                                       int num_blocks, const int32_t* __restrict__ table, int max_blocks,
                                       int block_size) {
  const int row = d_c + d_hr;
  const int pairs = row / 2;
  const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (long long)T * pairs) return;
  const int t = (int)(idx / pairs), e = 2 * (int)(idx % pairs);
  float2 v = sum_splits(part + (long long)t * row + e, splits, split_stride);
  const long long p = pos[t];
  if (e >= d_c) {
    float c, s;
    rope_cos_sin(rp, d_hr, (e - d_c) / 2, p, &c, &s);
    const float a = v.x, b = v.y;
    v.x = a * c - b * s;
    v.y = a * s + b * c;
  }
  const int page = (int)(p / block_size);
  const int blk = (page >= 0 && page < max_blocks) ? table[(long long)seq_idx[t] * max_blocks + page] : -1;
  if (blk < 0 || blk >= num_blocks) {
    if (e == 0) record_error(ERR_CAPACITY, 301);
    return;
  }
  __nv_bfloat16* dst = pool + ((long long)blk * block_size + p % block_size) * row + e;
  *reinterpret_cast<__nv_bfloat162*>(dst) = __floats2bfloat162_rn(v.x, v.y);
}

// plain conversion: y[z][t][n] (bf16) = sum of splits, n < n_out.
__global__ void finish_bf16_kernel(const float* __restrict__ part, int splits, long long split_stride, int Z, int T,
                                   int n_out, long long in_z, long long in_t, __nv_bfloat16* __restrict__ y,
                                   long long y_z, long long y_t) {
  const int pairs = n_out / 2;
  const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (long long)Z * T * pairs) return;
  const int e = 2 * (int)(idx % pairs);
  const long long zt = idx / pairs;
  const int t = (int)(zt % T), z = (int)(zt / T);
  const float2 v = sum_splits(part + z * in_z + t * in_t + e, splits, split_stride);
  *reinterpret_cast<__nv_bfloat162*>(y + z * y_z + t * y_t + e) = __floats2bfloat162_rn(v.x, v.y);
}

// absorb_q second projection: features [0, nq) are q^C (bf16 copy), features
// [nq, nq + n_h*d_hr) are q^R of head (n-nq)/d_hr, rotated at pos[t].
__global__ void finish_q_kernel(const float* __restrict__ part, int splits, long long split_stride, int T, int nq,
                                int n_h, int d_hr, RopeParams rp, const int32_t* __restrict__ pos,
                                __nv_bfloat16* __restrict__ q_c, __nv_bfloat16* __restrict__ q_rope) {
  const int n_all = nq + n_h * d_hr;
  const int pairs = n_all / 2;
  const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (long long)T * pairs) return;
  const int t = (int)(idx / pairs), e = 2 * (int)(idx % pairs);
  float2 v = sum_splits(part + (long long)t * n_all + e, splits, split_stride);
  if (e < nq) {
    *reinterpret_cast<__nv_bfloat162*>(q_c + (long long)t * nq + e) = __floats2bfloat162_rn(v.x, v.y);
    return;
  }
  const int r = e - nq;  // = head * d_hr + 2k
  float c, s;
  rope_cos_sin(rp, d_hr, (r % d_hr) / 2, pos[t], &c, &s);
  const float a = v.x, b = v.y;
  *reinterpret_cast<__nv_bfloat162*>(q_rope + (long long)t * n_h * d_hr + r) =
      __floats2bfloat162_rn(a * c - b * s, a * s + b * c);
}

// fp32 output: u[t][n] = sum of splits.
__global__ void finish_f32_kernel(const float* __restrict__ part, int splits, long long split_stride, int T,
                                  int n_out, float* __restrict__ u) {
  const int pairs = n_out / 2;
  const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (long long)T * pairs) return;
  const int t = (int)(idx / pairs), e = 2 * (int)(idx % pairs);
  const float2 v = sum_splits(part + (long long)t * n_out + e, splits, split_stride);
  *reinterpret_cast<float2*>(u + (long long)t * n_out + e) = v;
}

}  // namespace mla
