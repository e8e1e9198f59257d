// tc_gemm_heads.cuh — the per-head projections of the absorbed form as one
// persistent tcgen05 kernel:
//
//   q_lat[t][i][n] = sum_k W^UK[i d_h + k][n] q^C[t][i d_h + k]   (A_MN: W^UK read MN-major)
//   o[t][i][r]     = sum_c W^UV[i d_h + r][c] o_lat[t][i][c]      (W^UV read K-major)
// (q_lat_i = (W^UK_i)^T q^C_i and o_i = W^UV_i o_lat_i: W^UK absorbed into the
// query, W^UV applied before W^O — DeepSeek-V2 explainer, adg.csdn.net,
// section 2.2.2; "DeepSeek-V2" reading notes, eq 11.)
//
// Each head contributes a few output tiles of 128 rows: q_lat has d_c / 128
// tiles per head over a short contraction (K = d_h = 128, 512 tiles of 32 KB
// of W^UK at V2 shapes); o has one tile per head over K = d_c.  Launched one
// CTA per tile they spend their life in set-up; here 1 CTA per SM walks a
// contiguous range of (head, row tile, token tile) units, the weight loads
// stream through one ring of stages across unit boundaries, and the
// accumulator is double-buffered in TMEM so that a unit's epilogue overlaps
// the next unit's MMAs.
//
// Operands: A = W^UK_i read MN-major (two 64-column SW128 boxes per 64-row K
// chunk: the head's [d_h][d_c] block is the transposed A) or W^UV_i read
// K-major (one 128-row x 64-column box per chunk); B = the head's slice of
// the activations (K-major, token rows).  Tokens on N = 64.
//
// Warps (192 threads):
//   0     TMA producer
//   1     MMA issuer (one thread) and TMEM owner
//   2..5  epilogue: TMEM -> bf16 -> shared staging [token][row] -> 16-byte
//         stores of the output rows
// All waits are bounded.
#pragma once

#include "common.cuh"

namespace mla {

struct HeadsArgs {
  int n_h, T;             // heads, tokens
  int a_rows_per_head;    // rows of A per head: K (MN-major, W^UK: d_h) or M (K-major, W^UV: d_h)
  int k_chunks;           // K / 64
  int m_tiles, n_tiles;   // output row tiles per head (of 128), ceil(T / 64) token tiles
  int units;              // n_h * m_tiles * n_tiles
  int out_rows;           // output rows per head (m_tiles * 128)
  __nv_bfloat16* out;     // [T][n_h][out_rows]
};

struct HeadsCfg {
  static constexpr int THREADS = 192;
  static constexpr int TN = 64;
  static constexpr int A_BYTES = 128 * 64 * 2;  // 128 latent rows x one 64-wide K chunk
  static constexpr int B_BYTES = TN * 64 * 2;   // 64 tokens x one K chunk
  static constexpr int STAGE = A_BYTES + B_BYTES;
  static constexpr int NST = 8;
  static constexpr int OUT_BYTES = TN * 128 * 2;  // bf16 staging [token][row]
  static constexpr int OFF_OUT = NST * STAGE;
  static constexpr int OFF_BAR = OFF_OUT + OUT_BYTES;
  static constexpr int N_BAR = 2 * NST + 2 + 2 + 1;
  static constexpr int SMEM = OFF_BAR + N_BAR * 8 + 16 + 1024;
  static constexpr int TMEM_COLS = 2 * TN;
  static_assert(SMEM <= 227 * 1024, "shared memory");
};

template <bool A_MN>
__global__ void __launch_bounds__(HeadsCfg::THREADS, 1)
    mla_heads_gemm_kernel(const __grid_constant__ CUtensorMap mA, const __grid_constant__ CUtensorMap mB,
                          const HeadsArgs a) {
  using C = HeadsCfg;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* full = bar;
  uint64_t* empty = full + C::NST;
  uint64_t* acc_full = empty + C::NST;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* grp_bar = acc_empty + 2;  // 128-thread barrier of the epilogue warps
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(grp_bar + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  // this CTA's units: a contiguous range, so that the units of one head
  // (and the rows of one W^UK block) follow each other
  const int u0 = (int)((long long)blockIdx.x * a.units / gridDim.x);
  const int u1 = (int)((long long)(blockIdx.x + 1) * a.units / gridDim.x);
  auto unit = [&](int u, int* z, int* m, int* nt) {
    *nt = u % a.n_tiles;
    *m = (u / a.n_tiles) % a.m_tiles;
    *z = u / (a.n_tiles * a.m_tiles);
  };

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::NST; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], 128);
    }
    mbar_init(grp_bar, 128);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(tmem_slot, C::TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_trigger();  // after the TMEM allocation

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (elect_one()) {
      tma_prefetch_desc(&mA);
      tma_prefetch_desc(&mB);
      // while the previous kernel finishes: the first weight chunks into L2
      int i = 0;
      for (int u = u0; u < u1 && i < C::NST; ++u) {
        int z, m, nt;
        unit(u, &z, &m, &nt);
        for (int kc = 0; kc < a.k_chunks && i < C::NST; ++kc, ++i) {
          if (A_MN) {
            tma_prefetch_l2_2d(&mA, m * 128, z * a.a_rows_per_head + kc * 64);
            tma_prefetch_l2_2d(&mA, m * 128 + 64, z * a.a_rows_per_head + kc * 64);
          } else {
            tma_prefetch_l2_3d(&mA, 0, z * a.a_rows_per_head + m * 128, kc);
          }
        }
      }
      pdl_wait();  // the activations come from the kernel before
      i = 0;
      bool ok = true;
      for (int u = u0; ok && u < u1; ++u) {
        int z, m, nt;
        unit(u, &z, &m, &nt);
        for (int kc = 0; kc < a.k_chunks; ++kc, ++i) {
          const int s = i % C::NST;
          if (i >= C::NST && !mbar_wait(&empty[s], ((i / C::NST) - 1) & 1, abort_flag, 701)) {
            ok = false;
            break;
          }
          uint8_t* st = smem + s * C::STAGE;
          mbar_expect_tx(&full[s], C::STAGE);
          if (A_MN) {
            tma_load_2d(st, &mA, &full[s], m * 128, z * a.a_rows_per_head + kc * 64);
            tma_load_2d(st + 8192, &mA, &full[s], m * 128 + 64, z * a.a_rows_per_head + kc * 64);
          } else {
            tma_load_3d(st, &mA, &full[s], 0, z * a.a_rows_per_head + m * 128, kc);
          }
          tma_load_3d(st + C::A_BYTES, &mB, &full[s], 0, nt * C::TN, z * a.k_chunks + kc);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (elect_one()) {
      const uint32_t idesc = idesc_bf16_f32(128, C::TN, A_MN, false);
      int i = 0;
      bool ok = true;
      for (int u = u0, ul = 0; ok && u < u1; ++u, ++ul) {
        const int b = ul & 1;
        if (ul >= 2 && !mbar_wait(&acc_empty[b], ((ul / 2) - 1) & 1, abort_flag, 702)) break;
        tc_fence_after();
        for (int kc = 0; kc < a.k_chunks; ++kc, ++i) {
          const int s = i % C::NST;
          if (!mbar_wait(&full[s], (i / C::NST) & 1, abort_flag, 703)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + s * C::STAGE);
          const uint32_t sb = sa + C::A_BYTES;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t ad = A_MN ? smem_desc(sa + kk * 2048, 8192, 1024, SW128)
                                     : smem_desc(sa + kk * 32, 16, 1024, SW128);
            const uint64_t bd = smem_desc(sb + kk * 32, 16, 1024, SW128);
            mma_bf16_ss(tmem + b * C::TN, ad, bd, idesc, (kc | kk) != 0);
          }
          mma_commit(&empty[s]);
        }
        if (ok) mma_commit(&acc_full[b]);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    pdl_wait();  // the output may be read by the kernel before until it has finished
    const int q = warp & 3;
    const int row = q * 32 + (threadIdx.x & 31);  // latent row within the tile (TMEM lane)
    const int et = threadIdx.x - 64;                // 0..127
    __nv_bfloat16* stage_out = reinterpret_cast<__nv_bfloat16*>(smem + C::OFF_OUT);
    uint32_t gphase = 0;
    auto group_sync = [&](int site) -> bool {
      mbar_arrive(grp_bar);
      const bool r = mbar_wait(grp_bar, gphase & 1, abort_flag, site);
      ++gphase;
      return r;
    };
    bool ok = true;
    for (int u = u0, ul = 0; ok && u < u1; ++u, ++ul) {
      int z, m, nt;
      unit(u, &z, &m, &nt);
      const int b = ul & 1;
      if (!mbar_wait(&acc_full[b], (ul / 2) & 1, abort_flag, 704)) break;
      tc_fence_after();
      float v[C::TN];
      tmem_ld32<32>(tmem + b * C::TN + ((uint32_t)(q * 32) << 16), v);
      tmem_ld32<32>(tmem + b * C::TN + 32 + ((uint32_t)(q * 32) << 16), v + 32);
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(&acc_empty[b]);
      // staging [token][row]: for a token the warp writes 32 consecutive rows
#pragma unroll
      for (int t = 0; t < C::TN; ++t) stage_out[t * 128 + row] = __float2bfloat16_rn(v[t]);
      if (!group_sync(705)) break;
      // out[t][z][128 m .. 128 m + 127]: 256 contiguous bytes per token
      for (int idx = et; idx < C::TN * 16; idx += 128) {
        const int t = idx >> 4, part = idx & 15;
        const int tok = nt * C::TN + t;
        if (tok < a.T)
          *reinterpret_cast<uint4*>(a.out + ((long long)tok * a.n_h + z) * a.out_rows + m * 128 + part * 8) =
              *reinterpret_cast<const uint4*>(stage_out + t * 128 + part * 8);
      }
      // the staging is read by every thread before the next unit overwrites it
      ok = group_sync(706);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) tmem_dealloc(tmem, C::TMEM_COLS);
}

}  // namespace mla
