// tc_attn.cuh — latent-cache attention on the 5th-generation tensor cores.
//
// Absorbed MLA attention (DeepSeek-V2 explainer, adg.csdn.net, section 2.2.2):
// for every head i of a query row,
//   s_j = scale * (q_lat_i . c^KV_j + q^R_i . k^R_j),   o_lat_i = sum_j softmax(s)_j c^KV_j
// over the shared paged cache rows [c^KV_j | k^R_j] (d_c = 512, d_h^R = 64).
//
// This file holds the attention work plan (mla_attn_plan_kernel: rows cut
// into segments of 128-token tiles, dealt to CTAs), the one-CTA attention
// kernel for layers of up to 64 heads, and the LSE combine; 128-head layers
// use the CTA-pair kernel of tc_attn2.cuh on the same plan.
//
// One-CTA kernel.  A CTA = one group of H heads walking its list of segments
// (query row, token range).  Both contractions run as tcgen05 MMAs with the
// cached tokens on M = 128 ("swap-AB"): the group's H heads are the N
// dimension, so one 128-token cache tile feeds
//   S^T[128 tok x H]   = Kt[128 x 576]   . Q^T      (A = tile, K-major)
//   O^T[512 x H]      += V^T[512 x 128] . P^T      (A = same tile, MN-major)
// The 576-wide cache row is read from HBM once per CTA and used by both
// products straight from shared memory.  S^T and O^T live in TMEM
// (2*H + 4*H fp32 columns).
//
// Roles (192 threads):
//   warp 0      TMA producer: Q once per segment, then per tile one 16 KB
//               RoPE slot and four 32 KB latent slots (2 pages x 128 latent
//               columns)
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

// F8: the cache rows are FP8 (E4M3 codes of c^KV, bf16 k^R, a power-of-two
// scale per row); four more warps turn the codes into the bf16 tile.
template <int H, bool F8 = false>
struct AttnCfg {
  static constexpr int THREADS = F8 ? ATT_THREADS + 128 : ATT_THREADS;
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
  static constexpr int SC_SLOT = 2048;                 // F8: 2 pages x 64 rows x 16 bytes (scale + padding)
  static constexpr int NSC = F8 ? 2 : 0;               // F8: scale slots (by tile parity)
  static constexpr int CONV = F8 ? NL : 0;             // F8: "slot converted" barriers
  static constexpr int OFF_SCALE = OFF_LAT + NL * LAT_SLOT;
  static constexpr int OFF_BAR = OFF_SCALE + NSC * SC_SLOT;
  static constexpr int N_BAR = 2 * NL + 2 * NR + 1 + 2 + 2 + 2 + 2 + 1 + CONV + 2 * NSC + (F8 ? 1 : 0);
  static constexpr int OFF_RED = OFF_BAR + N_BAR * 8 + 16;
  static constexpr int SMEM = OFF_RED + 2 * 4 * H * 4 + 1024;
  static constexpr int TMEM_COLS = 6 * H <= 128 ? 128 : 256;
  static constexpr uint32_t P_LAYOUT = H == 16 ? SW32 : SW64;
  static_assert(OFF_P % 1024 == 0 && OFF_ROPE % 1024 == 0 && OFF_LAT % 1024 == 0 && OFF_SCALE % 1024 == 0,
                "1 KB alignment");
  static_assert(SMEM <= 227 * 1024, "shared memory");
};

#ifndef ATT_PREFETCH
#define ATT_PREFETCH 0  // tiles of cache pages prefetched into L2 ahead of their load (0: none;
                        // measured slower for the one-CTA kernel)
#endif

struct AttnArgs {
  int n_h, rows, q_per_seq, num_blocks, max_blocks;
  float scale_log2;
  const int32_t* table;
  const uint8_t* pool;     // cache pages, 64 rows x 1152 bytes each (L2 prefetch)
  const int32_t* kv_len;   // decode: per row (the end of the row's range); nullptr for prefill
  const int32_t* kv_begin; // partial decode: first row of each row's range (multiple of 128); else nullptr
  const int32_t* q_start;  // prefill: per sequence
  const int4* units;       // [segment] {row, first token, end token, partial slot or -1 (whole row)};
                           // nullptr: CTA w does all of row w
  const int* work;         // [CTA + 1]: first segment of each CTA (or CTA pair)
  __nv_bfloat16* o_lat;    // final output (rows done by one unit)
  float* lse;              // final lse (may be null)
  float* o_part;           // [slot][head][512] partials of rows split over several units
  float* lse_part;         // [slot][head]
};

__device__ __forceinline__ int att_kv_len(const AttnArgs& a, int r) {
  if (a.kv_len) return a.kv_len[r];
  return a.q_start[r / a.q_per_seq] + r % a.q_per_seq + 1;
}

// Work of CTA (or CTA pair) w: segments [x, y) of the plan.  Without a plan
// CTA w does all of row w.
__device__ __forceinline__ int2 att_work(const AttnArgs& a, int w) {
  if (!a.units) return make_int2(w, w + 1);
  return make_int2(a.work[w], a.work[w + 1]);
}
// Segment s: {row, first token, end token, partial slot or -1}.
__device__ __forceinline__ int4 att_seg(const AttnArgs& a, int s) {
  if (a.units) return a.units[s];
  return make_int4(s, 0, att_kv_len(a, s), -1);
}

// One segment as the kernels see it; n_tiles == 0 marks a segment to skip
// (its row's kv_len is out of range: recorded as MLA_ERR_CAPACITY).
struct SegInfo {
  int r, t_begin, t_end, pslot, kv, n_tiles;
};
__device__ __forceinline__ SegInfo att_seg_info(const AttnArgs& a, int s) {
  const int4 u = att_seg(a, s);
  SegInfo S;
  S.r = u.x;
  S.t_begin = u.y;
  S.t_end = u.z;
  S.pslot = u.w;
  S.kv = att_kv_len(a, S.r);
  // a partial decode may give a row an empty range (kv_end == kv_begin, 0 included)
  const bool ok = S.kv >= (a.kv_begin ? 0 : 1) && S.kv <= a.max_blocks * 64;
  if (!ok) record_error(ERR_CAPACITY, 401);
  S.n_tiles = ok && S.t_end > S.t_begin ? (S.t_end - S.t_begin + ATT_TILE - 1) / ATT_TILE : 0;
  return S;
}

// Walks the tiles of a CTA's segments in order.  Every role of a kernel keeps
// its own cursor; g (the tile count over all segments) indexes the pipeline's
// barrier phases, so they run on unchanged across segment boundaries.
struct TileCursor {
  int s, s_end;  // current segment, end of the list
  int j, g;      // tile within the segment, tile overall
  int n;         // segments entered so far - 1
  SegInfo S;
  __device__ __forceinline__ void init(const AttnArgs& a, int2 range) {
    s = range.x - 1;
    s_end = range.y;
    g = 0;
    n = -1;
    next_segment(a);
  }
  __device__ __forceinline__ void next_segment(const AttnArgs& a) {
    j = 0;
    while (++s < s_end) {
      S = att_seg_info(a, s);
      if (S.n_tiles > 0) {
        ++n;
        return;
      }
    }
  }
  __device__ __forceinline__ bool done() const { return s >= s_end; }
  __device__ __forceinline__ void step(const AttnArgs& a) {
    ++g;
    if (++j >= S.n_tiles) next_segment(a);
  }
  __device__ __forceinline__ bool first() const { return j == 0; }
  __device__ __forceinline__ bool last() const { return j == S.n_tiles - 1; }
  __device__ __forceinline__ int tok() const { return S.t_begin + j * ATT_TILE; }
  // the tile reaches past kv_len: rows to zero before PV
  __device__ __forceinline__ bool zero() const { return tok() + ATT_TILE > S.kv; }
};

// Work plan (one block).  A segment is a run of 128-token tiles of one row,
// and every CTA (or CTA pair) works through its own list of segments.
//   automatic (splits == 0): the tiles of all rows, taken in row order, are
//     dealt out to `workers` CTAs as equal contiguous ranges, so each CTA
//     gets the same number of tiles (+-1) whatever the length mix; a row
//     that straddles range boundaries becomes several segments.
//   explicit (splits > 0): every row cut into min(splits, its tiles) equal
//     segments, one per CTA.
// With kv_begin (partial decode) row b covers rows [kv_begin[b], kv_len[b])
// only, in tiles from kv_begin[b] (a multiple of 128), and force_slots gives
// every segment a partial slot: the combine then writes every row in fp32.
// Segments of rows cut in several get partial slots (merged by the combine
// kernel); the others write their output directly.  Outputs:
//   units[u]    = {row, first token, end token, slot or -1}   (row order)
//   row_info[b] = {first segment, segments of the row, first slot, 0}
//   work[w]     = first segment of CTA w, work[workers] = segment count
__global__ void mla_attn_plan_kernel(const int32_t* __restrict__ kv_len, const int32_t* __restrict__ q_start,
                                     int q_per_seq, int rows, int max_len, int workers, int splits, int max_units,
                                     int max_slots, int4* __restrict__ units, int4* __restrict__ row_info,
                                     int* __restrict__ work, int* __restrict__ n_units,
                                     const int32_t* __restrict__ kv_begin, int force_slots) {
  __shared__ long long s_sum[32];
  __shared__ int s_scan[3][1024];
  __shared__ int s_lastw[1024];
  __shared__ int s_per;
  const int tid = threadIdx.x, nt = blockDim.x;
  pdl_trigger();
  pdl_wait();  // kv_len may come from the previous kernel; the workspace may still be in its use
  auto kv_of = [&](int b) -> int {
    const int kv = kv_len ? kv_len[b] : q_start[b / q_per_seq] + b % q_per_seq + 1;
    return min(max(kv, 0), max_len);
  };
  // first row of b's range; a kv_begin that is not a multiple of 128 or lies
  // outside [0, kv] empties the row and is reported
  auto kb_of = [&](int b) -> int {
    if (!kv_begin) return 0;
    const int kb = kv_begin[b], kv = kv_of(b);
    if (kb < 0 || kb % ATT_TILE != 0 || kb > kv) {
      record_error(ERR_CAPACITY, 404);
      return kv;
    }
    return kb;
  };
  auto tiles_of = [&](int b) -> int {
    const int kb = kb_of(b);
    return (kv_of(b) - kb + ATT_TILE - 1) / ATT_TILE;
  };
  long long local = 0;
  for (int b = tid; b < rows; b += nt) local += tiles_of(b);
  for (int o = 16; o > 0; o >>= 1) local += __shfl_xor_sync(0xffffffffu, local, o);
  if ((tid & 31) == 0) s_sum[tid >> 5] = local;
  __syncthreads();
  if (tid == 0) {
    long long tot = 0;
    for (int w = 0; w < nt / 32; ++w) tot += s_sum[w];
    s_per = (int)max(1LL, (tot + workers - 1) / max(workers, 1));  // tiles per CTA (automatic)
  }
  __syncthreads();
  const int per = s_per;
  int run_tiles = 0, run_units = 0, run_slots = 0, run_lastw = -1;
  bool bad = false;
  for (int base = 0; base < rows; base += nt) {
    const int b = base + tid;
    const int tiles = b < rows ? tiles_of(b) : 0;
    // inclusive scan of the tiles: global position of every row's first tile
    s_scan[0][tid] = tiles;
    __syncthreads();
    for (int off = 1; off < nt; off <<= 1) {
      const int a0 = tid >= off ? s_scan[0][tid - off] : 0;
      __syncthreads();
      s_scan[0][tid] += a0;
      __syncthreads();
    }
    const int cum = run_tiles + s_scan[0][tid] - tiles;
    int parts = 0, per_seg = 1, w0 = 0, lastw = -1;
    if (b < rows) {
      if (splits > 0) {
        parts = max(1, min(splits, tiles));
        per_seg = max(1, (tiles + parts - 1) / parts);
        parts = max(1, (tiles + per_seg - 1) / per_seg);  // no empty segments
      } else if (tiles > 0) {
        w0 = cum / per;
        lastw = (cum + tiles - 1) / per;
        parts = lastw - w0 + 1;
      } else {
        w0 = lastw = min(cum / per, workers - 1);  // a row with no tiles (bad kv_len) still gets a segment
        parts = 1;
      }
    }
    s_lastw[tid] = lastw;
    __syncthreads();
    const int t_last = s_scan[0][nt - 1];
    __syncthreads();
    s_scan[1][tid] = parts;
    s_scan[2][tid] = (parts > 1 || force_slots) ? parts : 0;
    __syncthreads();
    for (int off = 1; off < nt; off <<= 1) {
      const int a1 = tid >= off ? s_scan[1][tid - off] : 0;
      const int a2 = tid >= off ? s_scan[2][tid - off] : 0;
      __syncthreads();
      s_scan[1][tid] += a1;
      s_scan[2][tid] += a2;
      __syncthreads();
    }
    const int u0 = run_units + s_scan[1][tid] - parts;
    const bool slotted = parts > 1 || force_slots;
    const int sl0 = slotted ? run_slots + s_scan[2][tid] - parts : -1;
    const bool over = b < rows && (u0 + parts > max_units || sl0 + parts > max_slots ||
                                   (splits == 0 && lastw >= workers));
    if (over) record_error(ERR_CAPACITY, 402);  // beyond the host's bounds: cannot happen for a valid plan
    bad |= over;
    if (b < rows && !over) {
      row_info[b] = make_int4(u0, parts, sl0, 0);
      const int kv = kv_of(b), kb = kb_of(b);
      if (splits > 0) {
        for (int q = 0; q < parts; ++q) {
          const int t0 = min(kb + q * per_seg * ATT_TILE, kv), t1 = min(kb + (q + 1) * per_seg * ATT_TILE, kv);
          units[u0 + q] = make_int4(b, t0, t1, slotted ? sl0 + q : -1);
        }
      } else {
        // CTAs after the previous row's last one and up to this row's first
        // start with this row's first segment
        const int prev_w = tid > 0 ? s_lastw[tid - 1] : run_lastw;
        for (int w = prev_w + 1; w <= w0; ++w) work[w] = u0;
        for (int q = 0; q < parts; ++q) {
          const int w = w0 + q;
          if (q > 0) work[w] = u0 + q;
          const int g0 = max(cum, w * per), g1 = min(cum + tiles, (w + 1) * per);
          const int t0 = min(kb + (g0 - cum) * ATT_TILE, kv), t1 = min(kb + (g1 - cum) * ATT_TILE, kv);
          units[u0 + q] = make_int4(b, t0, t1, slotted ? sl0 + q : -1);
        }
      }
    }
    run_tiles += t_last;
    run_units += s_scan[1][nt - 1];
    run_slots += s_scan[2][nt - 1];
    const int chunk_last = min(nt, rows - base) - 1;
    run_lastw = s_lastw[chunk_last];
    __syncthreads();
  }
  bad = __syncthreads_or(bad);
  const int n = bad ? 0 : run_units;
  if (splits > 0) {
    for (int w = tid; w <= workers; w += nt) work[w] = min(w, n);
  } else {
    // CTAs past the last row's last one (and all of them after an error) get nothing
    for (int w = (bad ? 0 : run_lastw + 1) + tid; w <= workers; w += nt) work[w] = n;
  }
  if (tid == 0) *n_units = n;
}

// m_cache: bf16 rows as {value, slot, block} (64 x 64 boxes); F8: the rows'
// bytes as {byte, slot, block} (128-byte x 64 boxes of codes, no swizzle),
// with m_rope8 (bf16 view of the same rows, k^R boxes) and m_scale8 (16-byte
// x 64 boxes of the scales).
template <int H, bool F8>
__global__ void __launch_bounds__(AttnCfg<H, F8>::THREADS, 1)
    mla_attn_kernel(const __grid_constant__ CUtensorMap m_qlat, const __grid_constant__ CUtensorMap m_qrope,
                    const __grid_constant__ CUtensorMap m_cache, const __grid_constant__ CUtensorMap m_rope8,
                    const __grid_constant__ CUtensorMap m_scale8, const AttnArgs a) {
  using C = AttnCfg<H, F8>;
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
  uint64_t* lat_conv = grp_bar + 1;  // F8: latent slot converted to bf16 (128 converter arrivals)
  uint64_t* sc_full = lat_conv + C::CONV;
  uint64_t* sc_empty = sc_full + C::NSC;
  uint64_t* q_conv = sc_empty + C::NSC;  // F8: the segment's queries converted to f16 (128 arrivals)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(q_conv + (F8 ? 1 : 0));
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* red = reinterpret_cast<float*>(smem + C::OFF_RED);  // [2][4][H]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // blockIdx.x = worker * (n_h / H) + head group: the head groups of one
  // worker run side by side and share its cache tiles in L2
  const int n_grp = a.n_h / H;
  const int worker = blockIdx.x / n_grp, grp = blockIdx.x % n_grp;
  const int head0 = grp * H;

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
    for (int i = 0; i < C::CONV; ++i) mbar_init(&lat_conv[i], 128);
    for (int i = 0; i < C::NSC; ++i) {
      mbar_init(&sc_full[i], 1);
      mbar_init(&sc_empty[i], 128);
    }
    if (F8) mbar_init(q_conv, 128);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(tmem_slot, C::TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_trigger();  // after the TMEM allocation
  pdl_wait();     // the plan, the queries and the cache come from earlier kernels
  // nothing written by an earlier kernel is read above this line
  const int2 range = att_work(a, worker);
  const uint32_t tS = tmem;            // S^T buffers at columns [0, 2H)
  const uint32_t tO = tmem + 2 * H;    // O^T M-block m at columns 2H + m*H

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (elect_one()) {
      tma_prefetch_desc(&m_cache);
      // cache block of page `page` of the cursor's row; past the row:
      // num_blocks (out of range: TMA reads zeros)
      auto page_block = [&](const TileCursor& c, int page) -> int {
        int b = a.num_blocks;
        if (page * 64 < c.S.kv) {
          b = a.table[(long long)(c.S.r / a.q_per_seq) * a.max_blocks + page];
          if (b < 0 || b >= a.num_blocks) {
            record_error(ERR_CAPACITY, 402);
            b = a.num_blocks;
          }
        }
        return b;
      };
      // Pages are prefetched into L2 ATT_PREFETCH tiles ahead of their TMA
      // loads, which then see L2 rather than HBM latency.
      constexpr uint32_t PAGE_BYTES = 64u * (F8 ? fp8_row_bytes(ATT_DC, ATT_DR) : (ATT_DC + ATT_DR) * 2);
      TileCursor c, cf;
      c.init(a, range);
      cf = c;
      auto prefetch = [&]() {
        if (ATT_PREFETCH > 0 && !cf.done()) {
          for (int p = 0; p < 2; ++p) {
            const int b = page_block(cf, cf.tok() / 64 + p);
            if (b < a.num_blocks) prefetch_l2_bulk(a.pool + (size_t)b * PAGE_BYTES, PAGE_BYTES);
          }
          cf.step(a);
        }
      };
      if (!cf.done()) cf.step(a);
      for (int i = 0; i < ATT_PREFETCH; ++i) prefetch();
      bool ok = true;
      while (ok && !c.done()) {
        const int g = c.g;
        if (c.first()) {
          // the queries of the segment's row; the buffer is free once the
          // previous segment's last QK is done
          if (g >= 1 && !mbar_wait(&s_full[(g - 1) & 1], ((g - 1) >> 1) & 1, abort_flag, 405)) break;
          const int qrow = c.S.r * a.n_h + head0;
          mbar_expect_tx(q_full, C::Q_BYTES);
          for (int k = 0; k < 8; ++k) tma_load_2d(smem + C::OFF_Q + k * C::Q_CHUNK, &m_qlat, q_full, k * 64, qrow);
          tma_load_2d(smem + C::OFF_Q + 8 * C::Q_CHUNK, &m_qrope, q_full, 0, qrow);
        }
        prefetch();
        int blk[2];
        for (int p = 0; p < 2; ++p) blk[p] = page_block(c, c.tok() / 64 + p);
        if (F8) {
          // the rows' scales, read by the converter warps first
          const int ss = g % 2;
          if (g >= 2 && !mbar_wait(&sc_empty[ss], ((g / 2) - 1) & 1, abort_flag, 406)) break;
          uint8_t* sdst = smem + C::OFF_SCALE + ss * C::SC_SLOT;
          mbar_expect_tx(&sc_full[ss], C::SC_SLOT);
          for (int p = 0; p < 2; ++p)
            tma_load_3d(sdst + p * 1024, &m_scale8, &sc_full[ss], fp8_scale_off(ATT_DC, ATT_DR), 0, blk[p]);
        }
        const int rs = g % C::NR;
        if (g >= C::NR && !mbar_wait(&rope_empty[rs], ((g / C::NR) - 1) & 1, abort_flag, 404)) break;
        uint8_t* rdst = smem + C::OFF_ROPE + rs * C::ROPE_SLOT;
        mbar_expect_tx(&rope_full[rs], C::ROPE_SLOT);
        for (int p = 0; p < 2; ++p)
          tma_load_3d(rdst + p * 8192, F8 ? &m_rope8 : &m_cache, &rope_full[rs], F8 ? ATT_DC / 2 : ATT_DC, 0, blk[p]);
        for (int m = 0; m < 4; ++m) {
          const int li = 4 * g + m;  // latent slot uses so far
          const int s = li % C::NL;
          if (li >= C::NL && !mbar_wait(&lat_empty[s], ((li / C::NL) - 1) & 1, abort_flag, 403)) {
            ok = false;
            break;
          }
          uint8_t* dst = smem + C::OFF_LAT + s * C::LAT_SLOT;
          if (F8) {
            // the codes of latent columns [128 m, 128 m + 128) of both pages
            // land in the slot's upper half, where the converters expand them
            mbar_expect_tx(&lat_full[s], C::LAT_SLOT / 2);
            for (int p = 0; p < 2; ++p) tma_load_3d(dst + 16384 + p * 8192, &m_cache, &lat_full[s], m * 128, 0, blk[p]);
          } else {
            mbar_expect_tx(&lat_full[s], C::LAT_SLOT);
            for (int hh = 0; hh < 2; ++hh)
              for (int p = 0; p < 2; ++p)
                tma_load_3d(dst + hh * 16384 + p * 8192, &m_cache, &lat_full[s], m * 128 + hh * 64, 0, blk[p]);
          }
        }
        c.step(a);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // One thread polls both queues and issues whatever is ready: QK chunks of
    // the next tile as their cache slots land, PV(j) as soon as P(j) is
    // written.  PV(j) frees the slots that QK(j+1) waits for, so neither may
    // block the other.
    if (elect_one()) {
      // F8: the latent tile, Q's latent chunks and P are f16; the RoPE chunk stays bf16
      const uint32_t id_qr = idesc_bf16_f32(ATT_TILE, H, false, false);
      const uint32_t id_qk = F8 ? idesc_f16_f32(ATT_TILE, H, false, false) : id_qr;
      const uint32_t id_pv = F8 ? idesc_f16_f32(ATT_TILE, H, true, true) : idesc_bf16_f32(ATT_TILE, H, true, true);
      const uint32_t q_base = smem_u32(smem + C::OFF_Q);
      const uint32_t lat_base = smem_u32(smem + C::OFF_LAT);
      const uint32_t rope_base = smem_u32(smem + C::OFF_ROPE);
      const uint32_t p_base = smem_u32(smem + C::OFF_P);
      TileCursor cq, cp;  // next QK tile, next PV tile
      cq.init(a, range);
      cp = cq;
      int kq = 0;            // next QK chunk of tile cq
      bool sbuf_ok = false;  // S buffer of tile cq released by the softmax
      int q_seen = -1;       // segment whose queries have landed
      bool ok = true;
      uint64_t t_idle = 0;
      uint32_t spins = 0;
      while (ok && !cp.done()) {
        bool prog = false;
        const int jp = cp.g;
        if (jp < cq.g && mbar_test(smem_u32(&p_full[jp & 1]), (jp >> 1) & 1)) {
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
              mma_bf16_ss(tO + m * H, ad, bd, id_pv, (cp.j > 0 || kk > 0) ? 1u : 0u);
            }
            mma_commit(&lat_empty[s]);
          }
          mma_commit(&pv_done[pb]);
          cp.step(a);
          prog = true;
        }
        if (!cq.done()) {
          const int jq = cq.g;
          const int sb = jq & 1;
          if (!sbuf_ok) sbuf_ok = jq < 2 || mbar_test(smem_u32(&s_free[sb]), ((jq >> 1) - 1) & 1);
          if (q_seen != cq.n && mbar_test(smem_u32(F8 ? q_conv : q_full), cq.n & 1)) q_seen = cq.n;
          if (sbuf_ok && q_seen == cq.n) {
            bool ready;
            uint32_t ka;
            int qchunk;  // chunk of Q: 0..7 latent, 8 rope
            if (kq == 0) {
              const int rs = jq % C::NR;
              ready = mbar_test(smem_u32(&rope_full[rs]), (jq / C::NR) & 1);
              ka = rope_base + rs * C::ROPE_SLOT;
              qchunk = 8;
            } else {
              const int c = kq - 1;
              const int li = jq * 4 + c / 2;
              const int s = li % C::NL;
              ready = (c & 1) || mbar_test(smem_u32(F8 ? &lat_conv[s] : &lat_full[s]), (li / C::NL) & 1);
              ka = lat_base + s * C::LAT_SLOT + (c & 1) * 16384;
              qchunk = c;
            }
            if (ready) {
              tc_fence_after();
#pragma unroll
              for (int kk = 0; kk < 4; ++kk) {
                const uint64_t ad = smem_desc(ka + kk * 32, 16, 1024, SW128);
                const uint64_t bd = smem_desc(q_base + qchunk * C::Q_CHUNK + kk * 32, 16, 1024, SW128);
                mma_bf16_ss(tS + sb * H, ad, bd, kq == 0 ? id_qr : id_qk, (kq | kk) != 0 ? 1u : 0u);
              }
              if (kq == 0) mma_commit(&rope_empty[jq % C::NR]);
              if (++kq == 9) {
                mma_commit(&s_full[sb]);
                cq.step(a);
                kq = 0;
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
            ok = false;
          }
        }
      }
    }
  } else if (F8 && warp >= 6) {
    // ------------------------------------------------------------ F8 converters
    // Per segment: the queries' latent chunks, bf16 -> f16 in place.  Per
    // tile: thread = (page p, token row r) of every latent slot; it reads the
    // row's 128 codes from the slot's upper half and writes code * 2^e as f16
    // into both halves in the MMA's SW128 layout (codes of columns 0..63 ->
    // the lower half, 64..127 -> the upper half, over exactly the bytes this
    // thread just read, so no other thread's input is touched).  The f16
    // values are exact for scales 2^e with -15 <= e <= 7 (latent values of
    // magnitude 2^-6 .. 2^15 at the row maximum).
    const int ct = threadIdx.x - ATT_THREADS;
    const int p = ct >> 6, r = ct & 63;
    TileCursor c;
    c.init(a, range);
    bool ok = true;
    while (ok && !c.done()) {
      const int g = c.g;
      if (c.first()) {
        if (!mbar_wait(q_full, c.n & 1, abort_flag, 433)) break;
        uint4* q = reinterpret_cast<uint4*>(smem + C::OFF_Q);
        for (int i = ct; i < 8 * C::Q_CHUNK / 16; i += 128) {
          const uint4 w = q[i];
          q[i] = make_uint4(f16x2_from_bf16x2(w.x), f16x2_from_bf16x2(w.y), f16x2_from_bf16x2(w.z),
                            f16x2_from_bf16x2(w.w));
        }
        fence_proxy_async_smem();
        mbar_arrive(q_conv);
      }
      const int ss = g % 2;
      if (!mbar_wait(&sc_full[ss], (g / 2) & 1, abort_flag, 431)) break;
      const float scale = *reinterpret_cast<const float*>(smem + C::OFF_SCALE + ss * C::SC_SLOT + p * 1024 + r * 16);
      mbar_arrive(&sc_empty[ss]);
      // 2^e in both f16 halves (a zero-filled row past the cache has scale 0:
      // its codes are zero as well)
      const uint32_t sc2 = pack_f16(scale, scale);
      for (int m = 0; m < 4 && ok; ++m) {
        const int li = 4 * g + m, s = li % C::NL;
        if (!mbar_wait(&lat_full[s], (li / C::NL) & 1, abort_flag, 432)) {
          ok = false;
          break;
        }
        uint8_t* slot = smem + C::OFF_LAT + s * C::LAT_SLOT + p * 8192 + r * 128;
        const uint4* in = reinterpret_cast<const uint4*>(slot + 16384);
        // thread r takes its row's 16-byte chunks in the order r, r+1, ...
        // (mod 8), so the 32 rows of a warp spread over all banks
        uint4 v[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) v[j] = in[(j + r) & 7];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          // codes 16k .. 16k+15: f16 columns 16(k%4) .. +15 of half k/4, 16-byte units 2(k%4), 2(k%4)+1
          const int k = (j + r) & 7;
          uint8_t* half = slot + (k >> 2) * 16384;
          const uint32_t u0 = 2u * (k & 3);
          const uint4 lo = make_uint4(f16x2_from_e4m3x2((uint16_t)v[j].x, sc2),
                                      f16x2_from_e4m3x2((uint16_t)(v[j].x >> 16), sc2),
                                      f16x2_from_e4m3x2((uint16_t)v[j].y, sc2),
                                      f16x2_from_e4m3x2((uint16_t)(v[j].y >> 16), sc2));
          const uint4 hi = make_uint4(f16x2_from_e4m3x2((uint16_t)v[j].z, sc2),
                                      f16x2_from_e4m3x2((uint16_t)(v[j].z >> 16), sc2),
                                      f16x2_from_e4m3x2((uint16_t)v[j].w, sc2),
                                      f16x2_from_e4m3x2((uint16_t)(v[j].w >> 16), sc2));
          *reinterpret_cast<uint4*>(half + ((u0 ^ (uint32_t)(r & 7)) << 4)) = lo;
          *reinterpret_cast<uint4*>(half + (((u0 + 1) ^ (uint32_t)(r & 7)) << 4)) = hi;
        }
        fence_proxy_async_smem();  // the tensor core reads what these threads wrote
        mbar_arrive(&lat_conv[s]);
      }
      c.step(a);
    }
  } else {
    // ------------------------------------------------------------ softmax + epilogue
    const int q = warp & 3;                 // TMEM sub-partition of this warp
    const int sw = warp - 2;                // softmax warp index 0..3
    const int tr = q * 32 + lane;           // token row within a tile (TMEM lane)
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    float m_run[H], l_part[H];
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
    TileCursor c;
    c.init(a, range);
    while (ok && !c.done()) {
      const int j = c.g;
      const int sb = j & 1;
      if (c.first()) {
#pragma unroll
        for (int h = 0; h < H; ++h) {
          m_run[h] = -INFINITY;
          l_part[h] = 0.f;
        }
      }
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
      const int tok = c.tok() + tr;
      const bool valid = tok < c.S.t_end;
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
      if (c.first()) {
        // PV of a segment's first tile overwrites O^T
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
        pk[h / 2] = F8 ? pack_f16(p0, p1) : pack_bf16(p0, p1);
      }
      // the P buffer was last read by PV(j-2)
      if (j >= 2 && !mbar_wait(&pv_done[sb], ((j - 2) >> 1) & 1, abort_flag, 423)) {
        ok = false;
        break;
      }
      uint8_t* prow = p_smem + sb * C::P_BYTES;
#pragma unroll
      for (int cc = 0; cc < H / 8; ++cc) {
        const uint32_t off = swizzle_off((uint32_t)(tr * 2 * H + cc * 16), C::P_LAYOUT);
        *reinterpret_cast<uint4*>(prow + off) =
            make_uint4(pk[4 * cc], pk[4 * cc + 1], pk[4 * cc + 2], pk[4 * cc + 3]);
      }
      if (c.zero()) {
        // the row's last tile: zero the latent rows past kv_len before PV reads them
        const int first = c.S.kv - c.tok();
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
      if (c.last()) {
        // ---------------------------------------------------------- epilogue of the segment
        // O^T is read out before this thread writes the next segment's first
        // P, which is what PV of that tile (overwriting O^T) waits for.
        const SegInfo& S = c.S;
        const bool direct = S.pslot < 0;
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
        ok = ok && mbar_wait(&pv_done[j & 1], (j >> 1) & 1, abort_flag, 424);
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
            if (direct) {
              a.o_lat[((long long)S.r * a.n_h + head0 + h) * ATT_DC + d] = __float2bfloat16_rn(val);
            } else {
              a.o_part[((long long)S.pslot * a.n_h + head0 + h) * ATT_DC + d] = val;
            }
          }
        }
        tc_fence_before();
        if (ok && sw == 0 && lane < H) {
          float mm = 0.f, ll = 0.f;
#pragma unroll
          for (int h = 0; h < H; ++h)
            if (h == lane) {
              mm = m_run[h];
              ll = l_tot[h];
            }
          const float lse = (mm + log2f(ll)) * 0.69314718055994531f;
          if (direct) {
            if (a.lse) a.lse[(long long)S.r * a.n_h + head0 + lane] = lse;
          } else {
            a.lse_part[(long long)S.pslot * a.n_h + head0 + lane] = lse;
          }
        }
        // the 4 x H sums are read by every thread before the red buffer is reused
        ok = group_sync(428) && ok;
      }
      c.step(a);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) tmem_dealloc(tmem, C::TMEM_COLS);
}

// Merge the partials of rows cut into several units:
// lse = log sum_s e^{lse_s}, o = sum_s e^{lse_s - lse} o_s.
// Block = (row, 8 heads, 1/CS of the latent columns), 256 threads; thread =
// (head, 16/CS columns).  All loads of a part are independent and issued
// together, so a thread pays the L2 latency about once per four parts; CS
// > 1 spreads rows of few sequences (long contexts) over more blocks.
constexpr int COMBINE_THREADS = 256, COMBINE_HEADS = 8;
// With o_f32 (partial decode) every row is written, in fp32: rows of one
// segment are copied, rows with an empty range get o = 0 and lse = -inf.
template <int CS>
__global__ void __launch_bounds__(COMBINE_THREADS)
    mla_combine_kernel(const float* __restrict__ o_part, const float* __restrict__ lse_part,
                       const int4* __restrict__ row_info, int n_h, __nv_bfloat16* __restrict__ o_lat,
                       float* __restrict__ lse, float* __restrict__ o_f32, const int32_t* __restrict__ kv_begin,
                       const int32_t* __restrict__ kv_len) {
  constexpr int CPT = 16 / CS;  // columns per thread
  pdl_trigger();
  pdl_wait();
  const int groups = n_h / COMBINE_HEADS;
  const int r = blockIdx.x / groups;
  const int h = (blockIdx.x % groups) * COMBINE_HEADS + threadIdx.x / 32;
  const int c0 = blockIdx.y * (ATT_DC / CS) + (threadIdx.x & 31) * CPT;
  const int4 info = row_info[r];
  const int n_parts = info.y, slot0 = info.z;
  if (n_parts <= (o_f32 ? 0 : 1)) return;  // written directly by its unit
  if (o_f32 && kv_len[r] <= kv_begin[r]) {
    // an empty range: no rows, no weight
    float4* dst = reinterpret_cast<float4*>(o_f32 + ((long long)r * n_h + h) * ATT_DC + c0);
#pragma unroll
    for (int q = 0; q < CPT / 4; ++q) dst[q] = make_float4(0.f, 0.f, 0.f, 0.f);
    if (lse && c0 == 0) lse[(long long)r * n_h + h] = -INFINITY;
    return;
  }
  // online log-sum-exp over the parts' lse
  float mx = -INFINITY, tot = 0.f;
  for (int s = 0; s < n_parts; ++s) {
    const float l = lse_part[(long long)(slot0 + s) * n_h + h];
    const float m2 = fmaxf(mx, l);
    tot = tot * expf(mx - m2) + expf(l - m2);
    mx = m2;
  }
  const float lse_all = mx + logf(tot);
  float acc[CPT];
#pragma unroll
  for (int e = 0; e < CPT; ++e) acc[e] = 0.f;
#pragma unroll 4
  for (int s = 0; s < n_parts; ++s) {
    const float wgt = expf(lse_part[(long long)(slot0 + s) * n_h + h] - lse_all);
    const float4* src = reinterpret_cast<const float4*>(o_part + ((long long)(slot0 + s) * n_h + h) * ATT_DC + c0);
    float4 x[CPT / 4];
#pragma unroll
    for (int q = 0; q < CPT / 4; ++q) x[q] = src[q];
#pragma unroll
    for (int q = 0; q < CPT / 4; ++q) {
      acc[4 * q] += wgt * x[q].x;
      acc[4 * q + 1] += wgt * x[q].y;
      acc[4 * q + 2] += wgt * x[q].z;
      acc[4 * q + 3] += wgt * x[q].w;
    }
  }
  if (o_f32) {
    float4* dst = reinterpret_cast<float4*>(o_f32 + ((long long)r * n_h + h) * ATT_DC + c0);
#pragma unroll
    for (int q = 0; q < CPT / 4; ++q) dst[q] = make_float4(acc[4 * q], acc[4 * q + 1], acc[4 * q + 2], acc[4 * q + 3]);
  } else {
    uint2* dst = reinterpret_cast<uint2*>(o_lat + ((long long)r * n_h + h) * ATT_DC + c0);
#pragma unroll
    for (int q = 0; q < CPT / 4; ++q)
      dst[q] = make_uint2(pack_bf16(acc[4 * q], acc[4 * q + 1]), pack_bf16(acc[4 * q + 2], acc[4 * q + 3]));
  }
  if (lse && c0 == 0) lse[(long long)r * n_h + h] = lse_all;
}

// Context-parallel merge of R ranks' partials of the same rows:
// lse = log sum_r e^{lse_r}, o = sum_r e^{lse_r - lse} o_r.  A rank whose range
// was empty contributes lse = -inf (weight 0).  Same block layout as the
// combine (rows x 8 heads x column share).
template <int CS>
__global__ void __launch_bounds__(COMBINE_THREADS)
    mla_lse_merge_kernel(const float* __restrict__ o_parts, const float* __restrict__ lse_parts, int R, int rows,
                         int n_h, __nv_bfloat16* __restrict__ o_bf16, float* __restrict__ o_f32,
                         float* __restrict__ lse) {
  constexpr int CPT = 16 / CS;
  pdl_trigger();
  pdl_wait();
  const int groups = n_h / COMBINE_HEADS;
  const int r = blockIdx.x / groups;
  const int h = (blockIdx.x % groups) * COMBINE_HEADS + threadIdx.x / 32;
  const int c0 = blockIdx.y * (ATT_DC / CS) + (threadIdx.x & 31) * CPT;
  const long long stride = (long long)rows * n_h;  // one rank's lse block
  float mx = -INFINITY;
  for (int k = 0; k < R; ++k) mx = fmaxf(mx, lse_parts[k * stride + (long long)r * n_h + h]);
  float tot = 0.f;
  for (int k = 0; k < R; ++k) {
    const float l = lse_parts[k * stride + (long long)r * n_h + h];
    tot += l == -INFINITY ? 0.f : expf(l - mx);
  }
  const float lse_all = mx + logf(tot);
  float acc[CPT];
#pragma unroll
  for (int e = 0; e < CPT; ++e) acc[e] = 0.f;
  for (int k = 0; k < R; ++k) {
    const float l = lse_parts[k * stride + (long long)r * n_h + h];
    if (l == -INFINITY) continue;
    const float wgt = expf(l - lse_all);
    const float4* src = reinterpret_cast<const float4*>(o_parts + (k * stride + (long long)r * n_h + h) * ATT_DC + c0);
#pragma unroll
    for (int q = 0; q < CPT / 4; ++q) {
      const float4 x = src[q];
      acc[4 * q] += wgt * x.x;
      acc[4 * q + 1] += wgt * x.y;
      acc[4 * q + 2] += wgt * x.z;
      acc[4 * q + 3] += wgt * x.w;
    }
  }
  const long long ob = ((long long)r * n_h + h) * ATT_DC + c0;
  if (o_f32) {
#pragma unroll
    for (int q = 0; q < CPT / 4; ++q)
      reinterpret_cast<float4*>(o_f32 + ob)[q] = make_float4(acc[4 * q], acc[4 * q + 1], acc[4 * q + 2], acc[4 * q + 3]);
  } else {
#pragma unroll
    for (int q = 0; q < CPT / 4; ++q)
      reinterpret_cast<uint2*>(o_bf16 + ob)[q] =
          make_uint2(pack_bf16(acc[4 * q], acc[4 * q + 1]), pack_bf16(acc[4 * q + 2], acc[4 * q + 3]));
  }
  if (lse && c0 == 0) lse[(long long)r * n_h + h] = lse_all;
}

// The same merge for any d_c (fp32 layers): one block per (row, head).
__global__ void mla_lse_merge_any_kernel(const float* __restrict__ o_parts, const float* __restrict__ lse_parts, int R,
                                         int rows, int n_h, int d_c, float* __restrict__ o_f32,
                                         float* __restrict__ lse) {
  const int r = blockIdx.x / n_h, h = blockIdx.x % n_h;
  const long long stride = (long long)rows * n_h;
  float mx = -INFINITY;
  for (int k = 0; k < R; ++k) mx = fmaxf(mx, lse_parts[k * stride + (long long)r * n_h + h]);
  float tot = 0.f;
  for (int k = 0; k < R; ++k) {
    const float l = lse_parts[k * stride + (long long)r * n_h + h];
    tot += l == -INFINITY ? 0.f : expf(l - mx);
  }
  const float lse_all = mx + logf(tot);
  for (int c = threadIdx.x; c < d_c; c += blockDim.x) {
    float acc = 0.f;
    for (int k = 0; k < R; ++k) {
      const float l = lse_parts[k * stride + (long long)r * n_h + h];
      if (l != -INFINITY) acc += expf(l - lse_all) * o_parts[(k * stride + (long long)r * n_h + h) * d_c + c];
    }
    o_f32[((long long)r * n_h + h) * d_c + c] = acc;
  }
  if (lse && threadIdx.x == 0) lse[(long long)r * n_h + h] = lse_all;
}

}  // namespace mla
