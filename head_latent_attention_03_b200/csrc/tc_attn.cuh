// tc_attn.cuh — latent-cache attention on the 5th-generation tensor cores.
//
// Absorbed MLA attention (DeepSeek-V2 explainer, adg.csdn.net, section 2.2.2):
// for every head i of a query row,
//   s_j = scale * (q_lat_i . c^KV_j + q^R_i . k^R_j),   o_lat_i = sum_j softmax(s)_j c^KV_j
// over the shared paged cache rows [c^KV_j | k^R_j] (d_c = 512, d_h^R = 64).
//
// Work unit: (query row r, group of H heads, KV split).  Both contractions run
// as tcgen05 MMAs with the cached tokens on M = 128 ("swap-AB"): the group's
// H heads are the N dimension, so one 128-token cache tile feeds
//   S^T[128 tok x H]   = Kt[128 x 576]   . Q^T      (A = tile, K-major)
//   O^T[512 x H]      += V^T[512 x 128] . P^T      (A = same tile, MN-major)
// The 576-wide cache row is read from HBM once per unit and used by both
// products straight from shared memory.  S^T and O^T live in TMEM
// (2*H + 4*H fp32 columns).
//
// Roles (192 threads):
//   warp 0      TMA producer: Q once, then per tile one 16 KB RoPE slot and
//               four 32 KB latent slots (2 pages x 128 latent columns)
//   warp 1      MMA issuer (one thread) and TMEM owner; QK(j+1) runs while
//               the softmax of tile j does, PV(j) as soon as P(j) is written
//   warps 2..5  softmax: thread = token row of the tile.  Tile max per head by
//               redux.sync + a 4-warp exchange; lazy rescale of O^T in TMEM
//               (only when a head's max grows by more than 2^8); P^T written
//               as bf16 into an MN-major swizzled buffer; per-thread partial
//               sums, reduced once at the end.  Then the epilogue.
// Rows of the last tile past kv_len are masked to -inf, and their cache rows
// are zeroed in shared memory before PV: unwritten slots may hold NaN bits.
#pragma once

#include "common.cuh"

namespace mla {

constexpr int ATT_THREADS = 192;
constexpr int ATT_TILE = 128;        // cached tokens per tile (MMA M)
constexpr int ATT_DC = 512, ATT_DR = 64;
constexpr float ATT_RESCALE_LOG2 = 8.0f;

template <int H>
struct AttnCfg {
  static constexpr int Q_CHUNK = H * 128;              // one 64-column chunk of H rows
  static constexpr int Q_BYTES = 9 * Q_CHUNK;
  static constexpr int P_BYTES = ATT_TILE * 2 * H;     // P^T[128 tokens x H] bf16
  static constexpr int LAT_SLOT = 32768;               // 2 pages x 128 latent cols
  static constexpr int ROPE_SLOT = 16384;              // 2 pages x 64 rope cols
  static constexpr int NR = 2;
  static constexpr int NL = H == 16 ? 5 : 4;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_P = OFF_Q + Q_BYTES;
  static constexpr int OFF_ROPE = OFF_P + 2 * P_BYTES;
  static constexpr int OFF_LAT = OFF_ROPE + NR * ROPE_SLOT;
  static constexpr int OFF_BAR = OFF_LAT + NL * LAT_SLOT;
  static constexpr int N_BAR = 2 * NL + 2 * NR + 1 + 2 + 2 + 2 + 2 + 1;
  static constexpr int OFF_RED = OFF_BAR + N_BAR * 8 + 16;
  static constexpr int SMEM = OFF_RED + 2 * 4 * H * 4 + 1024;
  static constexpr int TMEM_COLS = 6 * H <= 128 ? 128 : 256;
  static constexpr uint32_t P_LAYOUT = H == 16 ? SW32 : SW64;
  static_assert(OFF_P % 1024 == 0 && OFF_ROPE % 1024 == 0 && OFF_LAT % 1024 == 0, "1 KB alignment");
  static_assert(SMEM <= 227 * 1024, "shared memory");
};

struct AttnArgs {
  int n_h, rows, q_per_seq, span, n_splits, num_blocks, max_blocks;
  float scale_log2;
  const int32_t* table;
  const int32_t* kv_len;   // decode: per row; nullptr for prefill
  const int32_t* q_start;  // prefill: per sequence
  __nv_bfloat16* o_lat;    // final output (single split)
  float* lse;              // final lse (may be null)
  float* o_part;           // [split][row][head][512] partials (multi split)
  float* lse_part;         // [split][row][head]
};

__device__ __forceinline__ int att_kv_len(const AttnArgs& a, int r) {
  if (a.kv_len) return a.kv_len[r];
  return a.q_start[r / a.q_per_seq] + r % a.q_per_seq + 1;
}

template <int H>
__global__ void __launch_bounds__(ATT_THREADS, 1)
    mla_attn_kernel(const __grid_constant__ CUtensorMap m_qlat, const __grid_constant__ CUtensorMap m_qrope,
                    const __grid_constant__ CUtensorMap m_cache, const AttnArgs a) {
  using C = AttnCfg<H>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* lat_full = bar;
  uint64_t* lat_empty = lat_full + C::NL;
  uint64_t* rope_full = lat_empty + C::NL;
  uint64_t* rope_empty = rope_full + C::NR;
  uint64_t* q_full = rope_empty + C::NR;
  uint64_t* s_full = q_full + 1;
  uint64_t* s_free = s_full + 2;
  uint64_t* p_full = s_free + 2;
  uint64_t* pv_done = p_full + 2;
  uint64_t* grp_bar = pv_done + 2;  // 128-thread barrier of the softmax warps
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(grp_bar + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* red = reinterpret_cast<float*>(smem + C::OFF_RED);  // [2][4][H]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int split = blockIdx.x, grp = blockIdx.y, r = blockIdx.z;
  const int kv = att_kv_len(a, r);
  const int seq = r / a.q_per_seq;
  const int t_begin = split * a.span;
  const int t_end = min(t_begin + a.span, kv);
  const int n_tiles = t_end > t_begin ? (t_end - t_begin + ATT_TILE - 1) / ATT_TILE : 0;
  const bool direct = a.n_splits == 1;
  const int head0 = grp * H;

  if (kv < 1 || kv > a.max_blocks * 64) {
    if (threadIdx.x == 0) record_error(ERR_CAPACITY, 401);
    return;
  }
  if (n_tiles == 0) {
    // empty split: contributes nothing to the combine
    if (!direct) {
      for (int e = threadIdx.x; e < H; e += blockDim.x)
        a.lse_part[((long long)split * a.rows + r) * a.n_h + head0 + e] = -INFINITY;
    }
    return;
  }

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::NL; ++i) {
      mbar_init(&lat_full[i], 1);
      mbar_init(&lat_empty[i], 1);
    }
    for (int i = 0; i < C::NR; ++i) {
      mbar_init(&rope_full[i], 1);
      mbar_init(&rope_empty[i], 1);
    }
    mbar_init(q_full, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&s_free[i], 128);
      mbar_init(&p_full[i], 128);
      mbar_init(&pv_done[i], 1);
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
  const uint32_t tS = tmem;            // S^T buffers at columns [0, 2H)
  const uint32_t tO = tmem + 2 * H;    // O^T M-block m at columns 2H + m*H

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (elect_one()) {
      tma_prefetch_desc(&m_cache);
      const int qrow = r * a.n_h + head0;
      mbar_expect_tx(q_full, C::Q_BYTES);
      for (int c = 0; c < 8; ++c) tma_load_2d(smem + C::OFF_Q + c * C::Q_CHUNK, &m_qlat, q_full, c * 64, qrow);
      tma_load_2d(smem + C::OFF_Q + 8 * C::Q_CHUNK, &m_qrope, q_full, 0, qrow);
      const int* trow = a.table + (long long)seq * a.max_blocks;
      int li = 0;  // latent slot uses so far
      for (int j = 0; j < n_tiles; ++j) {
        const int tok = t_begin + j * ATT_TILE;
        int blk[2];
        for (int p = 0; p < 2; ++p) {
          const int page = tok / 64 + p;
          int b = a.num_blocks;  // out of range -> TMA fills zeros
          if (page * 64 < kv) {
            b = trow[page];
            if (b < 0 || b >= a.num_blocks) {
              record_error(ERR_CAPACITY, 402);
              b = a.num_blocks;
            }
          }
          blk[p] = b;
        }
        const int rs = j % C::NR;
        if (j >= C::NR && !mbar_wait(&rope_empty[rs], ((j / C::NR) - 1) & 1, abort_flag, 404)) break;
        uint8_t* rdst = smem + C::OFF_ROPE + rs * C::ROPE_SLOT;
        mbar_expect_tx(&rope_full[rs], C::ROPE_SLOT);
        for (int p = 0; p < 2; ++p) tma_load_3d(rdst + p * 8192, &m_cache, &rope_full[rs], ATT_DC, 0, blk[p]);
        bool ok = true;
        for (int m = 0; m < 4 && ok; ++m, ++li) {
          const int s = li % C::NL;
          if (li >= C::NL && !mbar_wait(&lat_empty[s], ((li / C::NL) - 1) & 1, abort_flag, 403)) {
            ok = false;
            break;
          }
          uint8_t* dst = smem + C::OFF_LAT + s * C::LAT_SLOT;
          mbar_expect_tx(&lat_full[s], C::LAT_SLOT);
          for (int hh = 0; hh < 2; ++hh)
            for (int p = 0; p < 2; ++p)
              tma_load_3d(dst + hh * 16384 + p * 8192, &m_cache, &lat_full[s], m * 128 + hh * 64, 0, blk[p]);
        }
        if (!ok) break;
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // One thread polls both queues and issues whatever is ready: QK chunks of
    // the next tile as their cache slots land, PV(j) as soon as P(j) is
    // written.  PV(j) frees the slots that QK(j+1) waits for, so neither may
    // block the other.
    if (elect_one()) {
      const uint32_t id_qk = idesc_bf16_f32(ATT_TILE, H, false, false);
      const uint32_t id_pv = idesc_bf16_f32(ATT_TILE, H, true, true);
      const uint32_t q_base = smem_u32(smem + C::OFF_Q);
      const uint32_t lat_base = smem_u32(smem + C::OFF_LAT);
      const uint32_t rope_base = smem_u32(smem + C::OFF_ROPE);
      const uint32_t p_base = smem_u32(smem + C::OFF_P);
      bool ok = mbar_wait(q_full, 0, abort_flag, 411);
      int jq = 0, cq = 0;    // next QK tile and chunk
      bool sbuf_ok = false;  // S buffer of tile jq released by the softmax
      int jp = 0;            // next PV tile
      uint64_t t_idle = 0;
      uint32_t spins = 0;
      while (ok && jp < n_tiles) {
        bool prog = false;
        if (jp < jq && mbar_test(smem_u32(&p_full[jp & 1]), (jp >> 1) & 1)) {
          tc_fence_after();
          const int pb = jp & 1;
          for (int m = 0; m < 4; ++m) {
            const int s = (jp * 4 + m) % C::NL;
            const uint32_t va = lat_base + s * C::LAT_SLOT;
#pragma unroll
            for (int kk = 0; kk < ATT_TILE / 16; ++kk) {
              const uint64_t ad = smem_desc(va + kk * 2048, 16384, 1024, SW128);
              const uint64_t bd = smem_desc(p_base + pb * C::P_BYTES + kk * 16 * 2 * H, C::P_BYTES, 8 * 2 * H,
                                            C::P_LAYOUT);
              mma_bf16_ss(tO + m * H, ad, bd, id_pv, (jp > 0 || kk > 0) ? 1u : 0u);
            }
            mma_commit(&lat_empty[s]);
          }
          mma_commit(&pv_done[pb]);
          ++jp;
          prog = true;
        }
        if (jq < n_tiles) {
          const int sb = jq & 1;
          if (!sbuf_ok) sbuf_ok = jq < 2 || mbar_test(smem_u32(&s_free[sb]), ((jq >> 1) - 1) & 1);
          if (sbuf_ok) {
            bool ready;
            uint32_t ka;
            int qchunk;  // chunk of Q: 0..7 latent, 8 rope
            if (cq == 0) {
              const int rs = jq % C::NR;
              ready = mbar_test(smem_u32(&rope_full[rs]), (jq / C::NR) & 1);
              ka = rope_base + rs * C::ROPE_SLOT;
              qchunk = 8;
            } else {
              const int c = cq - 1;
              const int li = jq * 4 + c / 2;
              const int s = li % C::NL;
              ready = (c & 1) || mbar_test(smem_u32(&lat_full[s]), (li / C::NL) & 1);
              ka = lat_base + s * C::LAT_SLOT + (c & 1) * 16384;
              qchunk = c;
            }
            if (ready) {
              tc_fence_after();
#pragma unroll
              for (int kk = 0; kk < 4; ++kk) {
                const uint64_t ad = smem_desc(ka + kk * 32, 16, 1024, SW128);
                const uint64_t bd = smem_desc(q_base + qchunk * C::Q_CHUNK + kk * 32, 16, 1024, SW128);
                mma_bf16_ss(tS + sb * H, ad, bd, id_qk, (cq | kk) != 0 ? 1u : 0u);
              }
              if (cq == 0) mma_commit(&rope_empty[jq % C::NR]);
              if (++cq == 9) {
                mma_commit(&s_full[sb]);
                ++jq;
                cq = 0;
                sbuf_ok = false;
              }
              prog = true;
            }
          }
        }
        if (prog) {
          t_idle = 0;
          spins = 0;
        } else if ((++spins & 63u) != 0) {
          __nanosleep(64);  // back off: the barrier words are also updated by TMA and MMA completions
        } else {
          if (*abort_flag) break;
          const uint64_t now = globaltimer_ns();
          if (t_idle == 0) {
            t_idle = now;
          } else if (now - t_idle > g_spin_limit_ns) {
            record_error(ERR_TIMEOUT, 412);
            *abort_flag = 1;
            break;
          }
        }
      }
    }
  } else {
    // ------------------------------------------------------------ softmax + epilogue
    const int q = warp & 3;                 // TMEM sub-partition of this warp
    const int sw = warp - 2;                // softmax warp index 0..3
    const int tr = q * 32 + lane;           // token row within a tile (TMEM lane)
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    float m_run[H], l_part[H];
#pragma unroll
    for (int h = 0; h < H; ++h) {
      m_run[h] = -INFINITY;
      l_part[h] = 0.f;
    }
    uint8_t* p_smem = smem + C::OFF_P;
    uint32_t gphase = 0;
    // bounded 128-thread barrier (a bar.sync could wait forever on a warp
    // that gave up a timed-out wait)
    auto group_sync = [&](int site) -> bool {
      mbar_arrive(grp_bar);
      const bool r = mbar_wait(grp_bar, gphase & 1, abort_flag, site);
      ++gphase;
      return r;
    };
    bool ok = true;
    for (int j = 0; j < n_tiles; ++j) {
      const int sb = j & 1;
      if (!mbar_wait(&s_full[sb], (j >> 1) & 1, abort_flag, 421)) {
        ok = false;
        break;
      }
      tc_fence_after();
      float s[H];
      tmem_ld32<H>(tS + sb * H + lane_off, s);
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(&s_free[sb]);
      const int tok = t_begin + j * ATT_TILE + tr;
      const bool valid = tok < t_end;
      // tile max per head: warp redux, then exchange across the 4 warps
      float* rb = red + (j & 1) * 4 * H;
#pragma unroll
      for (int h = 0; h < H; ++h) {
        s[h] = valid ? s[h] * a.scale_log2 : -INFINITY;
        const float wm = warp_max(s[h]);
        if (lane == (h & 31)) rb[sw * H + h] = wm;
      }
      if (!group_sync(425)) {
        ok = false;
        break;
      }
      bool grow = false;
      float m_new[H];
#pragma unroll
      for (int h = 0; h < H; ++h) {
        const float tm = fmaxf(fmaxf(rb[h], rb[H + h]), fmaxf(rb[2 * H + h], rb[3 * H + h]));
        m_new[h] = fmaxf(m_run[h], tm);
        grow |= (m_new[h] > m_run[h] + ATT_RESCALE_LOG2);
      }
      if (j == 0) {
#pragma unroll
        for (int h = 0; h < H; ++h) m_run[h] = m_new[h];
      } else if (grow) {
        // O^T must hold PV(j-1) complete before it is rescaled
        if (!mbar_wait(&pv_done[(j - 1) & 1], ((j - 1) >> 1) & 1, abort_flag, 422)) {
          ok = false;
          break;
        }
        tc_fence_after();
        float alpha[H];
#pragma unroll
        for (int h = 0; h < H; ++h) {
          alpha[h] = exp2_approx(m_run[h] - m_new[h]);
          l_part[h] *= alpha[h];
          m_run[h] = m_new[h];
        }
#pragma unroll 1
        for (int m = 0; m < 4; ++m) {
          float o[H];
          tmem_ld32<H>(tO + m * H + lane_off, o);
          tmem_wait_ld();
#pragma unroll
          for (int h = 0; h < H; ++h) o[h] *= alpha[h];
          tmem_st32<H>(tO + m * H + lane_off, o);
        }
        tmem_wait_st();
      }
      // P^T row of this token (bf16), l partial sums
      uint32_t pk[H / 2];
#pragma unroll
      for (int h = 0; h < H; h += 2) {
        const float p0 = valid ? exp2_approx(s[h] - m_run[h]) : 0.f;
        const float p1 = valid ? exp2_approx(s[h + 1] - m_run[h + 1]) : 0.f;
        l_part[h] += p0;
        l_part[h + 1] += p1;
        pk[h / 2] = pack_bf16(p0, p1);
      }
      // the P buffer was last read by PV(j-2)
      if (j >= 2 && !mbar_wait(&pv_done[sb], ((j - 2) >> 1) & 1, abort_flag, 423)) {
        ok = false;
        break;
      }
      uint8_t* prow = p_smem + sb * C::P_BYTES;
#pragma unroll
      for (int c = 0; c < H / 8; ++c) {
        const uint32_t off = swizzle_off((uint32_t)(tr * 2 * H + c * 16), C::P_LAYOUT);
        *reinterpret_cast<uint4*>(prow + off) = make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
      }
      if (j == n_tiles - 1 && t_begin + j * ATT_TILE + ATT_TILE > kv) {
        // last tile: zero the latent rows past kv_len before PV reads them
        const int first = kv - (t_begin + j * ATT_TILE);
        for (int m = 0; m < 4; ++m) {
          uint8_t* slot = smem + C::OFF_LAT + ((j * 4 + m) % C::NL) * C::LAT_SLOT;
          for (int e = first * 8 + tr; e < ATT_TILE * 8; e += 128) {
            const int row = e >> 3, ch = e & 7;  // 128-byte row, 16-byte chunk
            const int page = row >> 6, slot_row = row & 63;
            for (int hh = 0; hh < 2; ++hh)
              *reinterpret_cast<uint4*>(slot + hh * 16384 + page * 8192 + slot_row * 128 + ch * 16) =
                  make_uint4(0, 0, 0, 0);
          }
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&p_full[sb]);
    }
    // ------------------------------------------------------------ epilogue
    // l per head: sum of the per-thread partials over the 128 token rows
    ok = ok && group_sync(426);
    float* lred = red;  // reuse [4][H]
#pragma unroll
    for (int h = 0; h < H; ++h) {
      const float ws = warp_sum(l_part[h]);
      if (ok && lane == (h & 31)) lred[sw * H + h] = ws;
    }
    ok = group_sync(427) && ok;
    float l_tot[H];
#pragma unroll
    for (int h = 0; h < H; ++h) l_tot[h] = lred[h] + lred[H + h] + lred[2 * H + h] + lred[3 * H + h];
    const int last = n_tiles - 1;
    ok = ok && mbar_wait(&pv_done[last & 1], (last >> 1) & 1, abort_flag, 424);
    tc_fence_after();
    // thread = latent row d = 128*m + tr of O^T, registers = heads
#pragma unroll 1
    for (int m = 0; m < 4; ++m) {
      float o[H];
      tmem_ld32<H>(tO + m * H + lane_off, o);
      tmem_wait_ld();
      if (!ok) continue;
      const int d = m * 128 + tr;
#pragma unroll
      for (int h = 0; h < H; ++h) {
        const float val = o[h] / l_tot[h];
        const long long oi = ((long long)r * a.n_h + head0 + h) * ATT_DC + d;
        if (direct) {
          a.o_lat[oi] = __float2bfloat16_rn(val);
        } else {
          a.o_part[(long long)split * a.rows * a.n_h * ATT_DC + oi] = val;
        }
      }
    }
    if (ok && sw == 0 && lane < H) {
      float mm = 0.f, ll = 0.f;
#pragma unroll
      for (int h = 0; h < H; ++h)
        if (h == lane) {
          mm = m_run[h];
          ll = l_tot[h];
        }
      const float lse = (mm + log2f(ll)) * 0.69314718055994531f;
      const long long li = (long long)r * a.n_h + head0 + lane;
      if (direct) {
        if (a.lse) a.lse[li] = lse;
      } else {
        a.lse_part[(long long)split * a.rows * a.n_h + li] = lse;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) tmem_dealloc(tmem, C::TMEM_COLS);
}

// Merge split partials: lse = log sum_s e^{lse_s}, o = sum_s e^{lse_s - lse} o_s.
__global__ void mla_combine_kernel(const float* __restrict__ o_part, const float* __restrict__ lse_part, int n_splits,
                                   int rows, int n_h, __nv_bfloat16* __restrict__ o_lat, float* __restrict__ lse) {
  const int rh = blockIdx.x;  // row * n_h + head
  const long long stride_o = (long long)rows * n_h * ATT_DC;
  const long long stride_l = (long long)rows * n_h;
  float mx = -INFINITY;
  for (int s = 0; s < n_splits; ++s) mx = fmaxf(mx, lse_part[s * stride_l + rh]);
  float tot = 0.f;
  for (int s = 0; s < n_splits; ++s) {
    const float v = lse_part[s * stride_l + rh];
    tot += v == -INFINITY ? 0.f : expf(v - mx);
  }
  const float lse_all = mx + logf(tot);
  for (int d = threadIdx.x * 4; d < ATT_DC; d += blockDim.x * 4) {
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int s = 0; s < n_splits; ++s) {
      const float v = lse_part[s * stride_l + rh];
      if (v == -INFINITY) continue;
      const float wgt = expf(v - lse_all);
      const float4 x = *reinterpret_cast<const float4*>(o_part + s * stride_o + (long long)rh * ATT_DC + d);
      acc.x += wgt * x.x;
      acc.y += wgt * x.y;
      acc.z += wgt * x.z;
      acc.w += wgt * x.w;
    }
    __nv_bfloat16* dst = o_lat + (long long)rh * ATT_DC + d;
    *reinterpret_cast<__nv_bfloat162*>(dst) = __floats2bfloat162_rn(acc.x, acc.y);
    *reinterpret_cast<__nv_bfloat162*>(dst + 2) = __floats2bfloat162_rn(acc.z, acc.w);
  }
  if (lse && threadIdx.x == 0) lse[rh] = lse_all;
}

}  // namespace mla
