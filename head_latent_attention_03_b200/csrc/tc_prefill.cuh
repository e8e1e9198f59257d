// tc_prefill.cuh — causal attention of a prefill chunk in the un-absorbed form.
//
// The "DeepSeek-V2" reading notes (irregular6612.github.io), section 2.1.2,
// eqs (10)-(11), up-project the cached latent into per-head keys and values,
// k^C_{j,i} = W^UK_i c^KV_j and v^C_{j,i} = W^UV_i c^KV_j; with the decoupled
// RoPE parts (DeepSeek-V2 explainer, adg.csdn.net, section 2.2.2) head i
// attends with
//   q_{t,i} = [q^C_{t,i} ; q^R_{t,i}],  k_{j,i} = [k^C_{j,i} ; k^R_j]   (192 values)
//   o_{t,i} = sum_{j <= t} softmax_j(scale q_{t,i} . k_{j,i}) v^C_{j,i}  (eq 7, causal)
// Per (query, key) pair this is 2 n_h (192 + 128) FLOP against 2 n_h (576 +
// 512) in the latent form, so a long chunk is cheaper un-absorbed once its
// keys have been decompressed (the decompression GEMM writes k^C and v^C of
// every cache page into kv [page row][K of all heads | V of all heads]).
//
// One CTA = one head x 128 consecutive queries of one sequence, looping over
// the 128-key tiles up to its last query (causal tile skipping; the diagonal
// tiles are masked per element).  tcgen05 with cta_group::1, queries on
// M = 128, so a softmax thread owns a whole score row:
//   S[128 q x 128 k] = Q[128 x 192] . K^T     A = Q (smem), B = K tile (smem)
//   O[128 q x 128 d] += P[128 x 128] . V      A = P (TMEM), B = V tile (smem, MN-major)
// TMEM: S double-buffered (2 x 128 columns), O (128), P double-buffered
// (2 x 64, two bf16 per column).  Shared memory: Q (48 KB) and two stages of
// K (48 KB) + V (32 KB).
//
// Warps (192 threads):
//   0     TMA producer: Q once; per tile the K tile (k^C of two pages from kv,
//         k^R from the cache pool) and the V tile, each on its own barrier
//   1     MMA issuer (one thread) and TMEM owner: QK(j), then PV(j-1)
//   2..5  softmax: thread = query row; row max, exp2, P into TMEM, lazy
//         rescale of O; then the epilogue
// Keys past the sequence's end in its last page may be unwritten (any
// bits): their scores are replaced by -inf and their V rows are zeroed in
// shared memory before PV.  All waits are bounded.
#pragma once

#include "common.cuh"

namespace mla {

struct PrefillArgs {
  int n_h, q_per_seq, num_blocks, max_blocks;
  float scale_log2;          // softmax scale * log2(e)
  const int32_t* table;      // [B, max_blocks]
  const int32_t* q_start;    // [B] position of each sequence's first query
  __nv_bfloat16* o;          // [B * q_per_seq, n_h, 128]
  float* lse;                // [B * q_per_seq, n_h] (may be null)
};

struct PfCfg {
  static constexpr int THREADS = 192;
  static constexpr int CHUNK = 128 * 128;          // 128 rows x 64 bf16 columns (SW128)
  static constexpr int Q_BYTES = 3 * CHUNK;        // q^C (2 chunks) + q^R (1)
  static constexpr int K_BYTES = 3 * CHUNK;        // k^C (2 chunks) + k^R (1)
  static constexpr int V_BYTES = 2 * CHUNK;        // v^C (2 chunks of 64 columns)
  static constexpr int NS = 2;                     // stages
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + Q_BYTES;
  static constexpr int OFF_V = OFF_K + NS * K_BYTES;
  static constexpr int OFF_BAR = OFF_V + NS * V_BYTES;
  static constexpr int N_BAR = 1 + 4 * NS + 2 * 2 + 2 * 2;
  static constexpr int OFF_MISC = OFF_BAR + N_BAR * 8;
  static constexpr int SMEM = OFF_MISC + 16 + 1024;
  static constexpr int TMEM_COLS = 512;
  static_assert(SMEM <= 227 * 1024, "shared memory");
};

__device__ __forceinline__ void mma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// m_q: q^C [rows][n_h*128] (box 64 x 128); m_qr: q^R [rows][n_h*64] (box 64 x
// 128); m_kv: kv [pool rows][2*n_h*128] (box 64 x 64); m_kr: cache pool
// [pool rows][576] (box 64 x 64).
__global__ void __launch_bounds__(PfCfg::THREADS, 1)
    mla_prefill_unabsorbed_kernel(const __grid_constant__ CUtensorMap m_q, const __grid_constant__ CUtensorMap m_qr,
                                  const __grid_constant__ CUtensorMap m_kv, const __grid_constant__ CUtensorMap m_kr,
                                  const PrefillArgs a) {
  using C = PfCfg;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* q_full = bar;
  uint64_t* k_full = q_full + 1;       // [NS]
  uint64_t* k_empty = k_full + C::NS;  // [NS] QK has read the K stage
  uint64_t* v_full = k_empty + C::NS;  // [NS]
  uint64_t* v_empty = v_full + C::NS;  // [NS] PV has read the V stage
  uint64_t* s_full = v_empty + C::NS;  // [2] QK(j) done
  uint64_t* s_free = s_full + 2;       // [2] softmax read S(j) (4 warp arrives)
  uint64_t* p_full = s_free + 2;       // [2] P(j) in TMEM (4 warp arrives)
  uint64_t* pv_done = p_full + 2;      // [2] PV(j) done
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qb = blockIdx.x, h = blockIdx.y, b = blockIdx.z;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < C::NS; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&k_empty[i], 1);
      mbar_init(&v_full[i], 1);
      mbar_init(&v_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&s_free[i], 4);
      mbar_init(&p_full[i], 4);
      mbar_init(&pv_done[i], 1);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(tmem_slot, C::TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_trigger();
  pdl_wait();  // q^C, q^R, kv and the cache come from earlier kernels
  const uint32_t tS = tmem, tO = tmem + 256, tP = tmem + 384;

  const int start = a.q_start[b];
  const int q0 = qb * 128;                               // first query of this CTA within the chunk
  const int n_q = min(128, a.q_per_seq - q0);            // queries of this CTA
  const int kv_total = start + a.q_per_seq;              // rows of the sequence after the chunk
  const int last_pos = start + q0 + n_q - 1;             // the CTA's last query position
  const int n_tiles = last_pos / 128 + 1;                // key tiles 0 .. last_pos / 128
  const long long row0 = (long long)b * a.q_per_seq + q0;  // first query row of the chunk

  auto page_row = [&](int page) -> int {  // first pool row of the sequence's page
    if (page * 64 >= kv_total || page >= a.max_blocks) return a.num_blocks * 64;  // reads zeros
    const int blk = a.table[(long long)b * a.max_blocks + page];
    if (blk < 0 || blk >= a.num_blocks) {
      record_error(ERR_CAPACITY, 701);
      return a.num_blocks * 64;
    }
    return blk * 64;
  };

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (elect_one()) {
      mbar_expect_tx(q_full, C::Q_BYTES);
      tma_load_2d(smem + C::OFF_Q, &m_q, q_full, h * 128, (int)row0);
      tma_load_2d(smem + C::OFF_Q + C::CHUNK, &m_q, q_full, h * 128 + 64, (int)row0);
      tma_load_2d(smem + C::OFF_Q + 2 * C::CHUNK, &m_qr, q_full, h * 64, (int)row0);
      for (int j = 0; j < n_tiles; ++j) {
        const int s = j % C::NS, u = j / C::NS;
        const int r0 = page_row(2 * j), r1 = page_row(2 * j + 1);
        if (u >= 1 && !mbar_wait(&k_empty[s], (u - 1) & 1, abort_flag, 702)) break;
        uint8_t* kd = smem + C::OFF_K + s * C::K_BYTES;
        mbar_expect_tx(&k_full[s], C::K_BYTES);
        for (int c = 0; c < 2; ++c) {
          tma_load_2d(kd + c * C::CHUNK, &m_kv, &k_full[s], h * 128 + c * 64, r0);
          tma_load_2d(kd + c * C::CHUNK + 8192, &m_kv, &k_full[s], h * 128 + c * 64, r1);
        }
        tma_load_2d(kd + 2 * C::CHUNK, &m_kr, &k_full[s], 512, r0);
        tma_load_2d(kd + 2 * C::CHUNK + 8192, &m_kr, &k_full[s], 512, r1);
        if (u >= 1 && !mbar_wait(&v_empty[s], (u - 1) & 1, abort_flag, 703)) break;
        uint8_t* vd = smem + C::OFF_V + s * C::V_BYTES;
        mbar_expect_tx(&v_full[s], C::V_BYTES);
        for (int c = 0; c < 2; ++c) {
          tma_load_2d(vd + c * C::CHUNK, &m_kv, &v_full[s], a.n_h * 128 + h * 128 + c * 64, r0);
          tma_load_2d(vd + c * C::CHUNK + 8192, &m_kv, &v_full[s], a.n_h * 128 + h * 128 + c * 64, r1);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (elect_one()) {
      const uint32_t id_qk = idesc_bf16_f32(128, 128, false, false);
      const uint32_t id_pv = idesc_bf16_f32(128, 128, false, true);
      const uint32_t q_base = smem_u32(smem + C::OFF_Q);
      bool ok = mbar_wait(q_full, 0, abort_flag, 711);
      auto pv = [&](int j) -> bool {
        const int s = j % C::NS, u = j / C::NS;
        if (!mbar_wait(&p_full[j & 1], (j >> 1) & 1, abort_flag, 712)) return false;
        if (!mbar_wait(&v_full[s], u & 1, abort_flag, 713)) return false;
        tc_fence_after();
        const uint32_t vb = smem_u32(smem + C::OFF_V + s * C::V_BYTES);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t bd = smem_desc(vb + kk * 2048, C::CHUNK, 1024, SW128);
          mma_bf16_ts(tO, tP + (j & 1) * 64 + 8 * kk, bd, id_pv, (j > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(&v_empty[s]);
        mma_commit(&pv_done[j & 1]);
        return true;
      };
      for (int j = 0; ok && j < n_tiles; ++j) {
        const int s = j % C::NS, u = j / C::NS;
        if (j >= 2 && !mbar_wait(&s_free[j & 1], ((j >> 1) - 1) & 1, abort_flag, 714)) break;
        if (!mbar_wait(&k_full[s], u & 1, abort_flag, 715)) break;
        tc_fence_after();
        const uint32_t kb = smem_u32(smem + C::OFF_K + s * C::K_BYTES);
#pragma unroll
        for (int c = 0; c < 3; ++c) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t ad = smem_desc(q_base + c * C::CHUNK + kk * 32, 16, 1024, SW128);
            const uint64_t bd = smem_desc(kb + c * C::CHUNK + kk * 32, 16, 1024, SW128);
            mma_bf16_ss(tS + (j & 1) * 128, ad, bd, id_qk, (c | kk) != 0 ? 1u : 0u);
          }
        }
        mma_commit(&k_empty[s]);
        mma_commit(&s_full[j & 1]);
        if (j >= 1 && !pv(j - 1)) break;
        if (j == n_tiles - 1 && !pv(j)) break;
      }
    }
  } else {
    // ------------------------------------------------------------ softmax + epilogue
    const int q = warp & 3;
    const int r = q * 32 + lane;                 // query row of the CTA (TMEM lane)
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    const int pos = start + q0 + r;              // this row's position
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    for (int j = 0; ok && j < n_tiles; ++j) {
      if (!mbar_wait(&s_full[j & 1], (j >> 1) & 1, abort_flag, 721)) {
        ok = false;
        break;
      }
      tc_fence_after();
      float s[128];
#pragma unroll
      for (int cc = 0; cc < 128; cc += 32) tmem_ld32<32>(tS + (j & 1) * 128 + cc + lane_off, s + cc);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s_free[j & 1]);
      // causal mask: key j*128 + c is visible to the query at `pos` iff it is not after it
      const int k0 = j * 128;
      const int nvalid = min(128, max(0, pos - k0 + 1));
      float tmax = -INFINITY;
#pragma unroll
      for (int c = 0; c < 128; ++c) {
        s[c] = c < nvalid ? s[c] * a.scale_log2 : -INFINITY;
        tmax = fmaxf(tmax, s[c]);
      }
      const float m_new = fmaxf(m_run, tmax);
      // lazy rescale: only when the max grows by more than 2^8 (warp-uniform
      // decision, since the O rescale is a warp-wide TMEM access)
      const bool grow = __any_sync(0xffffffffu, j > 0 && m_new > m_run + ATT_RESCALE_LOG2);
      float alpha = 1.f;
      if (j == 0) {
        m_run = m_new;
      } else if (grow && m_new > m_run) {
        alpha = exp2_approx(m_run - m_new);
        l_run *= alpha;
        m_run = m_new;
      }
      // a row with no visible key in this tile keeps p = 0 (m_run may still be -inf
      // for rows past the chunk's queries: use 0 then)
      const float mref = m_run == -INFINITY ? 0.f : m_run;
      uint32_t pk[64];
#pragma unroll
      for (int c = 0; c < 64; ++c) {
        const float p0 = exp2_approx(s[2 * c] - mref), p1 = exp2_approx(s[2 * c + 1] - mref);
        l_run += p0 + p1;
        pk[c] = pack_bf16(p0, p1);
      }
      // P(j)'s buffer was read by PV(j-2); a rescale of O needs PV(j-1)
      if (j >= 2 || (grow && j >= 1)) {
        const int jw = grow ? j - 1 : j - 2;
        if (!mbar_wait(&pv_done[jw & 1], (jw >> 1) & 1, abort_flag, 722)) {
          ok = false;
          break;
        }
        tc_fence_after();
      }
      if (grow) {
#pragma unroll 1
        for (int cc = 0; cc < 128; cc += 16) {
          float o[16];
          tmem_ld32<16>(tO + cc + lane_off, o);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 16; ++e) o[e] *= alpha;
          tmem_st32<16>(tO + cc + lane_off, o);
        }
        tmem_wait_st();
      }
      tmem_st32<32>(tP + (j & 1) * 64 + lane_off, reinterpret_cast<const float*>(pk));
      tmem_st32<32>(tP + (j & 1) * 64 + 32 + lane_off, reinterpret_cast<const float*>(pk + 32));
      tmem_wait_st();
      // keys past the sequence's end in its last page may hold any bits:
      // zero their V rows before PV multiplies them by p = 0
      if ((j + 1) * 128 > kv_total) {
        const int st = j % C::NS;
        if (!mbar_wait(&v_full[st], (j / C::NS) & 1, abort_flag, 723)) {
          ok = false;
          break;
        }
        uint8_t* vd = smem + C::OFF_V + st * C::V_BYTES;
        const int first = max(0, kv_total - k0);  // first key row of the tile to clear
        for (int e = first * 8 + r; e < 128 * 8; e += 128) {
          const int row = e >> 3, ch = e & 7;
          for (int c = 0; c < 2; ++c)
            *reinterpret_cast<uint4*>(vd + c * C::CHUNK + row * 128 + ch * 16) = make_uint4(0, 0, 0, 0);
        }
        fence_proxy_async_smem();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[j & 1]);
    }
    // ---------------------------------------------------------- epilogue
    const int jl = n_tiles - 1;
    ok = ok && mbar_wait(&pv_done[jl & 1], (jl >> 1) & 1, abort_flag, 724);
    tc_fence_after();
    const float inv_l = l_run > 0.f ? 1.f / l_run : 0.f;
    const bool write = ok && r < n_q;
    __nv_bfloat16* dst = a.o + ((row0 + r) * a.n_h + h) * 128;
#pragma unroll 1
    for (int cc = 0; cc < 128; cc += 16) {
      float o[16];
      tmem_ld32<16>(tO + cc + lane_off, o);
      tmem_wait_ld();
      if (!write) continue;
      *reinterpret_cast<uint4*>(dst + cc) =
          make_uint4(pack_bf16(o[0] * inv_l, o[1] * inv_l), pack_bf16(o[2] * inv_l, o[3] * inv_l),
                     pack_bf16(o[4] * inv_l, o[5] * inv_l), pack_bf16(o[6] * inv_l, o[7] * inv_l));
      *reinterpret_cast<uint4*>(dst + cc + 8) =
          make_uint4(pack_bf16(o[8] * inv_l, o[9] * inv_l), pack_bf16(o[10] * inv_l, o[11] * inv_l),
                     pack_bf16(o[12] * inv_l, o[13] * inv_l), pack_bf16(o[14] * inv_l, o[15] * inv_l));
    }
    if (write && a.lse) a.lse[(row0 + r) * a.n_h + h] = (m_run + log2f(l_run)) * 0.69314718055994531f;
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) tmem_dealloc(tmem, C::TMEM_COLS);
}

}  // namespace mla
