// tc_attn2.cuh — latent-cache attention of 128-head layers on a CTA pair.
//
// Same arithmetic as tc_attn.cuh (absorbed MLA, DeepSeek-V2 explainer,
// adg.csdn.net, section 2.2.2), laid out for n_h = 128: the two CTAs of a
// cluster each own 64 heads and together issue tcgen05.mma.cta_group::2 with
// the heads on M = 128.  Per 128-token tile (two cache pages, page r is
// CTA r's "own" page):
//   S[128 heads x 128 tok] = Q[128 x 576] . K^T    B split by page
//   O[128 heads x 512]    += P[128 x 128] . V      B split by latent column:
//                                                  CTA r holds columns 256i + [128r, 128r+128)
// In the pair layout each CTA's TMEM holds its 64 heads folded over 128
// lanes (lanes 64..127 carry the second half of the N columns), so S takes 64
// columns and O 256: the fp32 O of all 128 heads (256 KB) no longer has to fit
// one SM.  Q of 64 heads (72 KB) stays resident in shared memory.
//
// P lives in TMEM as the A operand of PV (two buffers, by tile parity), so
// the softmax of tile j+1 never waits for PV(j).  A 2-SM M = 128 MMA reads A
// from both lane halves of each CTA (lanes r and 64 + r hold row r with the
// instruction's whole K), while a softmax thread computes one page of its
// head; the two threads of a head swap halves through a 16 KB shared-memory
// staging buffer and both store all 128 tokens.
//
// Cache data flow.  Each CTA loads its own page's row once, as a RoPE chunk
// and four latent "pairs" (chunks 2k, 2k+1: 16 KB), and QK reads them.  PV
// instruction (i, p) — latent columns of instruction i, tokens of page p —
// reads pair slot k = 2i + p in BOTH CTAs (one descriptor for the pair): one
// CTA already holds the right columns of its own page there, the other
// overwrites its own (already multiplied) pair with the columns it needs from
// the other page.  So every cached byte crosses into shared memory once per
// CTA that needs it (104 KB per CTA per tile), and the eight 16 KB pair slots
// keep two tiles in flight.  Slots recycle one at a time: the own-page pair
// for slot s of tile j+2 is loaded as soon as PV(j) has read slot s (a commit
// per slot), and QK(j+2) starts on the first pair to land, so the chain
// load -> QK -> refill -> PV overlaps across the four pairs of a tile
// instead of running tile by tile.  The cache is read through a 4D view
// {column, slot, chunk, block}: per tile and CTA, one RoPE box and four
// 2-chunk own-page boxes, plus two 2-chunk refill boxes.
//
// Warps (224 threads per CTA, 480 over FP8 rows):
//   0    own-page producer (four latent pairs per tile as their slots free
//        up, then the RoPE chunk once QK of the previous tile is done)
//   1    MMA issuer (leader CTA only, one thread) and TMEM owner (both CTAs)
//   2-5  softmax: thread = (head, page half of the tile)
//   6    other-page producer: refills the pair slots PV needs once QK is done
//        with them; zeroes rows past kv_len in the last tile (bf16 rows)
//   7-14 FP8 rows only: converters.  The producers then load each pair's
//        128 codes per token (8 KB per page) into the upper half of its slot
//        and the converters expand them to f16 over the whole slot, own
//        pages before QK and refills before PV, zeroing rows past kv_len;
//        QK's latent chunks and PV run as f16 MMAs on f16 queries and P, the
//        RoPE chunk as a bf16 MMA into the same accumulator.
// TMA pair loads complete their bytes on the leader's barriers, for which the
// leader alone posts the byte count; the other CTA's only arrives on the
// leader's barriers are "S read" (one per tile), "P written" (one per softmax
// warp and tile) and the last tile's zeroing, all with CTA-scope release.
// All waits are bounded.
#pragma once

#include "common.cuh"
#include "tc_attn.cuh"

namespace mla {

// Signals from the non-leader CTA to the leader's barriers (S consumed, P
// written, last tile zeroed) announce data in the signalling CTA's own shared
// memory / TMEM, consumed by its own tensor core: CTA-scope release and
// acquire suffice (PAIR_CLUSTER_SCOPE = 1 selects cluster scope).
#ifndef PAIR_CLUSTER_SCOPE
#define PAIR_CLUSTER_SCOPE 0
#endif
#if PAIR_CLUSTER_SCOPE
#define PAIR_ARRIVE(a) mbar_arrive_cluster(a)
#define PAIR_TEST(a, p) mbar_test_cluster(a, p)
#else
#define PAIR_ARRIVE(a) mbar_arrive_remote(a)
#define PAIR_TEST(a, p) mbar_test(a, p)
#endif

#ifndef PAIR_WARP_ARRIVE
#define PAIR_WARP_ARRIVE 1  // P written: one arrive per softmax warp instead of a group barrier
#endif
#ifndef PAIR_BACKOFF_NS
#define PAIR_BACKOFF_NS 32  // MMA issuer's back-off between fruitless polls
#endif

#ifndef PAIR_SM_SPIN
#define PAIR_SM_SPIN 0  // 1: the softmax warps poll their barriers without suspending
#endif
#if PAIR_SM_SPIN
#define PAIR_SM_WAIT mbar_wait_spin
#else
#define PAIR_SM_WAIT mbar_wait
#endif

#ifndef PAIR_QK_CUTIN
#define PAIR_QK_CUTIN 0  // 1: the MMA issuer re-checks PV between the latent pairs of a QK
#endif

#ifndef PAIR_PREFETCH
#define PAIR_PREFETCH 1  // own pages are prefetched into L2 this many tiles ahead of their load (>= 1)
#endif

#ifndef PAIR_CONV_WARPS
#define PAIR_CONV_WARPS 8  // F8: converter warps per CTA (4 or 8)
#endif

// F8: the cache rows are FP8 (E4M3 codes of c^KV, bf16 k^R, a power-of-two
// scale per row); PAIR_CONV_WARPS more warps expand the codes into f16 pair
// slots.
template <bool F8>
struct PairCfgT {
#if defined(MLA_TRACE) && defined(MLA_TRACE_OBSERVER)
  static constexpr int BASE_THREADS = 256;  // + a barrier-observer warp
#else
  static constexpr int BASE_THREADS = 224;
#endif
  static constexpr int CONV_WARPS = PAIR_CONV_WARPS;
  static_assert(CONV_WARPS == 4 || CONV_WARPS == 8, "converter warps");
  static constexpr int THREADS = BASE_THREADS + (F8 ? 32 * CONV_WARPS : 0);
  static constexpr int CONV_WARP0 = BASE_THREADS / 32;  // F8: first converter warp
  static constexpr int Q_CHUNK = 64 * 128;        // 64 heads x 64 columns
  static constexpr int Q_BYTES = 9 * Q_CHUNK;     // 72 KB
  static constexpr int P_BYTES = 2 * 64 * 128;    // staging: 64 heads x 2 pages x 64 tokens (bf16 or f16)
  static constexpr int PAIR = 16384;              // one page x 2 latent chunks
  static constexpr int CODES = 8192;              // F8: one page x 128 codes, in the slot's upper half
  static constexpr int ROPE = 8192;               // one page x 64 RoPE columns
  static constexpr int NP = 8;                    // pair slots (two tiles)
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_P = OFF_Q + Q_BYTES;
  static constexpr int OFF_ROPE = OFF_P + P_BYTES;
  static constexpr int OFF_PAIR = OFF_ROPE + ROPE;
  static constexpr int OFF_BAR = OFF_PAIR + NP * PAIR;
  // own_full, oth_full, qk_done, pv_slot [NP]; rope_full, q_full, grp_bar;
  // s_full, s_free, p_full, pv_done [2]; then either last_ready, z_land [2]
  // (bf16 rows) or own_land, oth_land [NP] and q_land (F8 rows)
  static constexpr int N_BAR = 4 * NP + 3 + 4 * 2 + (F8 ? 2 * NP + 1 : 2 * 2);
  static constexpr int OFF_MISC = OFF_BAR + N_BAR * 8;
  static constexpr int OFF_RED = OFF_MISC + 16;
  static constexpr int SMEM = OFF_RED + 3 * 128 * 4 + 1024;
  static constexpr int TMEM_COLS = 512;
  static_assert(OFF_P % 1024 == 0 && OFF_ROPE % 1024 == 0 && OFF_PAIR % 1024 == 0, "1 KB alignment");
  static_assert(SMEM <= 227 * 1024, "shared memory");
};
using PairCfg = PairCfgT<false>;

// m_page1: RoPE chunks of the cached rows (bf16, 128-byte chunks of a row);
// m_page2: bf16 rows as 4D {column, slot, chunk, block} (2-chunk boxes), or
// F8 rows as bytes {byte, slot, block} (128-code boxes, no swizzle).
template <bool F8>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(PairCfgT<F8>::THREADS, 1)
    mla_attn_pair_kernel(const __grid_constant__ CUtensorMap m_qlat, const __grid_constant__ CUtensorMap m_qrope,
                         const __grid_constant__ CUtensorMap m_page1, const __grid_constant__ CUtensorMap m_page2,
                         const AttnArgs a) {
  using C = PairCfgT<F8>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  // Pair commits per tile: one qk_done per pair slot (QK has read it: the
  // other CTA may refill it), one pv_slot per pair slot (PV has read it: the
  // next own-page load may overwrite it), s_full (S ready; the RoPE slot is
  // free) and pv_done (O is stable, the tile's P buffer is free).  s_full and
  // pv_done have one instance per tile parity so that a waiter is never two
  // phases behind.  With F8 rows own_full, oth_full and q_full count the
  // converter warps that finished the slot (the codes land on each CTA's own
  // own_land / oth_land / q_land).
  uint64_t* own_full = bar;                   // leader [NP]: own-page pair ready in the slot
  uint64_t* oth_full = own_full + C::NP;      // leader [NP]: other-page refill ready
  uint64_t* qk_done = oth_full + C::NP;       // both [NP]: pair commit once QK has read the slot
  uint64_t* pv_slot = qk_done + C::NP;        // both [NP]: pair commit once PV has read the slot
  uint64_t* rope_full = pv_slot + C::NP;      // leader
  uint64_t* q_full = rope_full + 1;           // leader
  uint64_t* grp_bar = q_full + 1;             // local: 128 softmax threads
  uint64_t* s_full = grp_bar + 1;             // both [2]: pair commit after QK(j)
  uint64_t* s_free = s_full + 2;              // leader [2]: one arrive per CTA
  uint64_t* p_full = s_free + 2;              // leader [2]: P(j) in TMEM, one arrive per softmax warp
  uint64_t* pv_done = p_full + 2;             // both [2]: pair commit after PV(j)
  uint64_t* last_ready = pv_done + 2;         // bf16 rows, leader [2]: both CTAs zeroed the last tile
  uint64_t* z_land = last_ready + 2;          // bf16 rows, local [2]: last tile's other-page refills
  uint64_t* own_land = pv_done + 2;           // F8 rows, local [NP]: own-page codes landed
  uint64_t* oth_land = own_land + C::NP;      // F8 rows, local [NP]: other-page codes landed
  uint64_t* q_land = oth_land + C::NP;        // F8 rows, local: the segment's queries landed
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);
  float* red = reinterpret_cast<float*>(smem + C::OFF_RED);  // [3][128]: tile max x2, final sums
  (void)last_ready;
  (void)z_land;
  (void)own_land;
  (void)oth_land;
  (void)q_land;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  // both CTAs of the pair walk the same segment list
  const int worker = blockIdx.x >> 1;
  const int head0 = (int)rank * 64;
  const int tunit = rank == 0 ? worker : -1;  // trace slot (leader only)
  (void)tunit;

  if (threadIdx.x == 0) {
    // F8: a slot or the queries are ready once both CTAs' converter warps of
    // that kind arrived (a slot is expanded by two warps: per CTA for its own
    // page, by the one CTA that refills it for the other page)
    for (int i = 0; i < C::NP; ++i) {
      mbar_init(&own_full[i], F8 ? 4 : 1);
      mbar_init(&oth_full[i], F8 ? 2 : 1);
      mbar_init(&qk_done[i], 1);
      mbar_init(&pv_slot[i], 1);
    }
    mbar_init(rope_full, 1);
    mbar_init(q_full, F8 ? C::CONV_WARPS : 1);  // F8: the own-page half of the converter warps, both CTAs
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&s_free[i], 2);
      mbar_init(&pv_done[i], 1);
      mbar_init(&p_full[i], PAIR_WARP_ARRIVE ? 8 : 2);
    }
    if (F8) {
      for (int i = 0; i < C::NP; ++i) {
        mbar_init(&own_land[i], 1);
        mbar_init(&oth_land[i], 1);
      }
      mbar_init(q_land, 1);
    } else {
      for (int i = 0; i < 2; ++i) {
        mbar_init(&z_land[i], 1);
        mbar_init(&last_ready[i], 2);
      }
    }
    mbar_init(grp_bar, 128);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc_pair(tmem_slot, C::TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // peer barriers initialised before any remote arrive
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_trigger();  // after the TMEM allocation
  pdl_wait();     // the plan, the queries and the cache come from earlier kernels
  // nothing written by an earlier kernel is read above this line
  const int2 range = att_work(a, worker);
  if (threadIdx.x == 0) MLA_TRACE_EVENT(tunit, 0, 0);
  const uint32_t tS = tmem;         // S buffers: columns [0,64) and [64,128)
  const uint32_t tO = tmem + 128;   // O: columns [128,256) (d_c 0..255) and [256,384) (256..511)
  const uint32_t tP = tmem + 384;   // P buffers (bf16 / F8: f16, A operand of PV): columns [384,448) and [448,512)

  // cache block of page `page` of the cursor's row; past the row: num_blocks
  // (out of range: TMA reads zeros)
  auto page_block = [&](const TileCursor& c, int page) -> int {
    int b = a.num_blocks;
    if (page * 64 < c.S.kv) {
      b = a.table[(long long)(c.S.r / a.q_per_seq) * a.max_blocks + page];
      if (b < 0 || b >= a.num_blocks) {
        record_error(ERR_CAPACITY, 502);
        b = a.num_blocks;
      }
    }
    return b;
  };
  // pair slot of latent pair k of tile g, and how often that slot was used before
  auto slot_of = [](int g, int k) -> int { return (4 * g + k) % C::NP; };
  auto use_of = [](int g, int k) -> int { return (4 * g + k) / C::NP; };
  // Pair k of a tile serves PV instruction k >> 1 over the tokens of page k & 1.
  // The CTA whose own page is k & 1 keeps its own columns there; the other CTA
  // refills the slot with columns 2*(2*(k>>1) + rank) .. +1 of page k & 1.

#if defined(MLA_TRACE) && defined(MLA_TRACE_OBSERVER)
  if (warp == 7) {
    if (lane != 0 || rank != 0) {
    } else {
    // trace-only observer: completion times of each tile's first and last
    // own pair, first refill, S, P and PV (leader barriers), polled for two
    // tiles at a time without blocking anyone
    TileCursor c;
    c.init(a, range);
    TileCursor c2 = c;
    if (!c2.done()) c2.step(a);
    uint32_t seen[2] = {0, 0};
    const uint64_t t_start = globaltimer_ns();
    while (!c.done() && !*abort_flag && globaltimer_ns() - t_start < 20000000ull) {
      for (int w = 0; w < 2; ++w) {
        const TileCursor& cc = w == 0 ? c : c2;
        if (cc.done()) continue;
        const int g = cc.g;
        const int s0 = slot_of(g, 0), u0 = use_of(g, 0), s3 = slot_of(g, 3), u3 = use_of(g, 3);
        uint32_t& m = seen[w];
        if (cc.zero()) m |= 2u;
        if (!(m & 1u) && mbar_test(smem_u32(&own_full[s0]), u0 & 1)) { m |= 1u; MLA_TRACE_EVENT(tunit, 3, g); }
        if (!(m & 2u) && mbar_test(smem_u32(&oth_full[s0]), u0 & 1)) { m |= 2u; MLA_TRACE_EVENT(tunit, 4, g); }
        if (!(m & 4u) && mbar_test_cluster(smem_u32(&p_full[g & 1]), (g >> 1) & 1)) { m |= 4u; MLA_TRACE_EVENT(tunit, 15, g); }
        if (!(m & 8u) && mbar_test(smem_u32(&own_full[s3]), u3 & 1)) { m |= 8u; MLA_TRACE_EVENT(tunit, 18, g); }
        if (!(m & 16u) && mbar_test(smem_u32(&s_full[g & 1]), (g >> 1) & 1)) { m |= 16u; MLA_TRACE_EVENT(tunit, 16, g); }
        if (!(m & 32u) && mbar_test(smem_u32(&pv_done[g & 1]), (g >> 1) & 1)) { m |= 32u; MLA_TRACE_EVENT(tunit, 17, g); }
      }
      if (seen[0] == 63u) {
        c = c2;
        seen[0] = seen[1];
        seen[1] = 0;
        if (!c2.done()) c2.step(a);
      }
    }
    }
  } else
#endif
  if (warp == 0) {
    // ------------------------------------------------------------ own-page producer
    // Per tile two TMA instructions: the RoPE chunk (8 KB) and all eight
    // latent chunks of the own page (64 KB, landing in the tile's four
    // consecutive pair slots); per segment the queries of its row.
    if (elect_one()) {
      tma_prefetch_desc(&m_page2);
      const uint32_t lq = mapa_shared(smem_u32(q_full), 0);
      const uint32_t l_rope = mapa_shared(smem_u32(rope_full), 0);
      // Own pages are prefetched into L2 PAIR_PREFETCH tiles ahead (one tile
      // measured best): the loads below, and the other CTA's refills from
      // this page, then see L2 rather than HBM latency.
      constexpr uint32_t PAGE_BYTES = 64u * (F8 ? fp8_row_bytes(ATT_DC, ATT_DR) : (ATT_DC + ATT_DR) * 2u);
      constexpr int ROPE_CHUNK = (F8 ? ATT_DC : 2 * ATT_DC) / 128;  // the 128-byte chunk of a row holding k^R
      TileCursor c, cf;
      c.init(a, range);
      cf = c;
      auto prefetch = [&]() {
        if (!cf.done()) {
          const int page = cf.tok() / 64 + (int)rank;
          const int b = page_block(cf, page);
          if (b < a.num_blocks) prefetch_l2_bulk(a.pool + (size_t)b * PAGE_BYTES, PAGE_BYTES);
          cf.step(a);
        }
      };
      if (!cf.done()) cf.step(a);
      for (int i = 1; i < PAIR_PREFETCH; ++i) prefetch();
      while (!c.done()) {
        const int g = c.g;
        prefetch();
        const int blk = page_block(c, c.tok() / 64 + (int)rank);
        // the own page pair by pair, each into its slot as soon as PV(g-2)
        // has read that slot: QK(g) starts on the first pair to land.  These
        // loads wait for nothing else, so tile g streams in while QK(g-1)
        // still runs.
        bool ok = true;
        for (int k = 0; k < 4 && ok; ++k) {
          const int s = slot_of(g, k), u = use_of(g, k);
          if (u >= 1 && !mbar_wait(&pv_slot[s], (u - 1) & 1, abort_flag, 504)) {
            ok = false;
            break;
          }
          if (F8) {
            // the codes of latent columns 128k .. 128k+127 into the slot's upper half
            mbar_expect_tx(&own_land[s], C::CODES);
            tma_load_3d(smem + C::OFF_PAIR + s * C::PAIR + C::CODES, &m_page2, &own_land[s], 128 * k, 0, blk);
          } else {
            if (rank == 0) mbar_expect_tx(&own_full[s], 2 * C::PAIR);
            tma_load_4d_pair(smem + C::OFF_PAIR + s * C::PAIR, &m_page2, mapa_shared(smem_u32(&own_full[s]), 0), 0,
                             0, 2 * k, blk);
          }
          if (k == 0) MLA_TRACE_EVENT(tunit, 1, g);
          if (k == 3) MLA_TRACE_EVENT(tunit, 2, g);
        }
        if (!ok) break;
        // the RoPE slot, and at a segment's start the Q buffer, are free once
        // QK(g-1) is done (QK reads the RoPE chunk last)
        if (g >= 1 && !mbar_wait(&s_full[(g - 1) & 1], ((g - 1) >> 1) & 1, abort_flag, 503)) break;
        if (c.first()) {
          const int qrow = c.S.r * a.n_h + head0;
          if (F8) {
            // each CTA's own queries, turned into f16 by its converters
            mbar_expect_tx(q_land, C::Q_BYTES);
            for (int k = 0; k < 8; ++k) tma_load_2d(smem + C::OFF_Q + k * C::Q_CHUNK, &m_qlat, q_land, k * 64, qrow);
            tma_load_2d(smem + C::OFF_Q + 8 * C::Q_CHUNK, &m_qrope, q_land, 0, qrow);
          } else {
            if (rank == 0) mbar_expect_tx(q_full, 2 * C::Q_BYTES);
            for (int k = 0; k < 8; ++k)
              tma_load_2d_pair(smem + C::OFF_Q + k * C::Q_CHUNK, &m_qlat, lq, k * 64, qrow);
            tma_load_2d_pair(smem + C::OFF_Q + 8 * C::Q_CHUNK, &m_qrope, lq, 0, qrow);
          }
        }
        if (rank == 0) mbar_expect_tx(rope_full, 2 * C::ROPE);
        tma_load_4d_pair(smem + C::OFF_ROPE, &m_page1, l_rope, 0, 0, ROPE_CHUNK, blk);
        MLA_TRACE_EVENT(tunit, 19, g);
        c.step(a);
      }
    }
  } else if (warp == 6) {
    // ------------------------------------------------------------ other-page producer
    TileCursor c;
    c.init(a, range);
    int nz = 0;  // zero tiles so far (phase of z_land)
    const int tunit6 = rank == 0 ? worker : 256 + worker;  // trace slot of this CTA's refills
    (void)tunit6;
    bool ok = true;
    while (ok && !c.done()) {
      const int g = c.g;
      // F8: the converters zero the rows past kv_len of every slot they write
      const bool zero = !F8 && c.zero();
      if (lane == 0) {
        int zk = 0;  // refills of this tile that land on z_land
        for (int k = 0; k < 4 && ok; ++k) {
          const int s = slot_of(g, k), u = use_of(g, k);
          if ((k & 1) == (int)rank) continue;  // kept by this CTA
          ok = mbar_wait(&qk_done[s], u & 1, abort_flag, 505);  // QK(g) has read this pair
          if (!ok) break;
          MLA_TRACE_EVENT(tunit6, zk == 0 && k < 2 ? 12 : 13, g);
          const int b = page_block(c, c.tok() / 64 + (k & 1));
          const int c0 = 2 * (2 * (k >> 1) + (int)rank);  // columns this CTA multiplies in instruction k >> 1
          uint8_t* dst = smem + C::OFF_PAIR + s * C::PAIR;
          if (F8) {
            // the codes of those columns into the slot's upper half, for this CTA's converters
            mbar_expect_tx(&oth_land[s], C::CODES);
            tma_load_3d(dst + C::CODES, &m_page2, &oth_land[s], 64 * c0, 0, b);
          } else if (!zero) {
            if (rank == 0) mbar_expect_tx(&oth_full[s], C::PAIR);  // the peer's are posted by the MMA issuer
            tma_load_4d_pair(dst, &m_page2, mapa_shared(smem_u32(&oth_full[s]), 0), 0, 0, c0, b);
          } else {
            mbar_expect_tx(&z_land[zk], C::PAIR);
            tma_load_4d(dst, &m_page2, &z_land[zk], 0, 0, c0, b);
            ++zk;
          }
        }
      }
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      if (!ok) break;
      if (zero) {
        // every pair this CTA presents to PV — refilled ones once landed, kept
        // ones once QK is done with them — gets its rows past kv_len zeroed
        const int first = c.S.kv - c.tok();
        int zi = 0;
        for (int k = 0; k < 4 && ok; ++k) {
          const int s = slot_of(g, k);
          const bool refilled = (k & 1) != (int)rank;
          if (lane == 0)
            ok = refilled ? mbar_wait(&z_land[zi], nz & 1, abort_flag, 506)
                          : mbar_wait(&qk_done[s], use_of(g, k) & 1, abort_flag, 507);
          if (refilled) ++zi;
          ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
          if (!ok) break;
          const int lo = max(0, first - 64 * (k & 1));  // first row of this page to clear
          uint8_t* dst = smem + C::OFF_PAIR + s * C::PAIR;
          for (int e = lo * 8 + lane; e < 64 * 8; e += 32) {
            const int row = e >> 3, ch = e & 7;
            *reinterpret_cast<uint4*>(dst + row * 128 + ch * 16) = make_uint4(0, 0, 0, 0);
            *reinterpret_cast<uint4*>(dst + 8192 + row * 128 + ch * 16) = make_uint4(0, 0, 0, 0);
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0 && ok) PAIR_ARRIVE(mapa_shared(smem_u32(&last_ready[nz & 1]), 0));
        ++nz;
      }
      c.step(a);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (leader)
    if (rank == 0 && elect_one()) {
      // F8: the latent chunks of Q and K, P and V are f16; the RoPE chunk stays bf16
      const uint32_t id_qr = idesc_bf16_f32(128, 128, false, false);
      const uint32_t id_qk = F8 ? idesc_f16_f32(128, 128, false, false) : id_qr;
      const uint32_t id_pv = F8 ? idesc_f16_f32(128, 256, false, true) : idesc_bf16_f32(128, 256, false, true);
      const uint32_t q_base = smem_u32(smem + C::OFF_Q);
      const uint32_t rope_base = smem_u32(smem + C::OFF_ROPE);
      const uint32_t pair0 = smem_u32(smem + C::OFF_PAIR);
      TileCursor cq, cp, cpost;  // next QK tile, next PV tile, PV tile + 2
      cq.init(a, range);
      cp = cq;
      cpost = cq;
      // Byte counts of the refills the peer performs (pairs k = 0, 2) are
      // posted here, each as soon as the slot's previous refill has been
      // consumed by PV; the leader's own refills post theirs themselves.
      auto post_peer_refill = [&](int k) {
        if (!F8 && !cpost.done() && !cpost.zero()) mbar_expect_tx(&oth_full[slot_of(cpost.g, k)], C::PAIR);
      };
      for (int t = 0; t < 2; ++t) {
        post_peer_refill(0);
        post_peer_refill(2);
        if (!cpost.done()) cpost.step(a);
      }
      // Work is issued in batches (a tile's 32 latent QK MMAs at once, PV pair
      // by pair): every barrier probe between MMAs costs issue slots.
      int pv_k = 0;  // next pair of PV(cp)
      int qk_k = 0;  // next pair of QK(cq)
      int q_seen = -1;  // segment whose queries have landed
      int nz = 0;       // zero tiles passed by PV (phase of last_ready)
      bool sbuf_ok = false, rope_pending = false, p_ok = false, ok = true;
      uint64_t t_idle = 0;
      uint32_t spins = 0;
      while (ok && !cp.done()) {
        bool prog = false;
        // PV first: it frees the slots that later tiles' loads wait for
        if (cp.g < cq.g) {
          const int jp = cp.g;
          if (!p_ok) {
            p_ok = PAIR_TEST(smem_u32(&p_full[jp & 1]), (jp >> 1) & 1);
            if (p_ok) MLA_TRACE_EVENT(tunit, 15, jp);
          }
          if (p_ok) {
            const bool zero = !F8 && cp.zero();
            while (pv_k < 4) {
              const int s = slot_of(jp, pv_k), u = use_of(jp, pv_k);
              const bool ready = zero ? PAIR_TEST(smem_u32(&last_ready[nz & 1]), (nz >> 1) & 1)
                                      : mbar_test(smem_u32(&oth_full[s]), u & 1);
              if (!ready) break;
              if (pv_k == 0) MLA_TRACE_EVENT(tunit, 14, jp);
              if (pv_k == 1) MLA_TRACE_EVENT(tunit, 20, jp);
              if (pv_k == 2) MLA_TRACE_EVENT(tunit, 21, jp);
              tc_fence_after();
              const int i = pv_k >> 1, p = pv_k & 1;
              const uint32_t pb = pair0 + s * C::PAIR;
              // P of page p, tokens 16kk..16kk+15: columns 32p + 8kk of the tile's P buffer
              const uint32_t pa = tP + (jp & 1) * 64 + 32 * p;
#pragma unroll
              for (int kk = 0; kk < 4; ++kk) {
                const uint64_t bd = smem_desc(pb + kk * 2048, 8192, 1024, SW128);
                mma_bf16_pair_ts(tO + 128 * i, pa + 8 * kk, bd, id_pv, (cp.j > 0 || p > 0 || kk > 0) ? 1u : 0u);
              }
              mma_commit_pair(&pv_slot[s]);
              // a zero tile's slots had no refill on oth_full: close that phase
              if (zero) mbar_arrive(&oth_full[s]);
              if ((pv_k & 1) == 0) post_peer_refill(pv_k);
              ++pv_k;
              prog = true;
            }
            if (pv_k == 4) {
              MLA_TRACE_EVENT(tunit, 5, jp);
              mma_commit_pair(&pv_done[jp & 1]);
              if (zero) ++nz;
              cp.step(a);
              if (!cpost.done()) cpost.step(a);
              pv_k = 0;
              p_ok = false;
            }
          }
        }
        if (!cq.done()) {
          const int jq = cq.g;
          if (!rope_pending) {
            if (!sbuf_ok) sbuf_ok = jq < 2 || PAIR_TEST(smem_u32(&s_free[jq & 1]), ((jq >> 1) - 1) & 1);
            if (q_seen != cq.n && mbar_test(smem_u32(q_full), cq.n & 1)) q_seen = cq.n;
            // the latent chunks pair by pair as their slots land; each pair's
            // commit lets the other CTA refill that slot
            while (sbuf_ok && q_seen == cq.n && qk_k < 4) {
              const int s = slot_of(jq, qk_k);
              if (!mbar_test(smem_u32(&own_full[s]), use_of(jq, qk_k) & 1)) break;
              if (qk_k == 0) MLA_TRACE_EVENT(tunit, 6, jq);
              tc_fence_after();
              const uint32_t kb = pair0 + s * C::PAIR;
#pragma unroll
              for (int h2 = 0; h2 < 2; ++h2) {
                const int k = 2 * qk_k + h2;
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                  const uint64_t ad = smem_desc(q_base + k * C::Q_CHUNK + kk * 32, 16, 1024, SW128);
                  const uint64_t bd = smem_desc(kb + h2 * 8192 + kk * 32, 16, 1024, SW128);
                  mma_bf16_pair(tS + (jq & 1) * 64, ad, bd, id_qk, (k | kk) != 0 ? 1u : 0u);
                }
              }
              mma_commit_pair(&qk_done[s]);
              ++qk_k;
              prog = true;
              if (PAIR_QK_CUTIN && cp.g < cq.g) break;  // let PV of an older tile cut in
            }
            if (qk_k == 4) {
              rope_pending = true;
              qk_k = 0;
            }
          }
          if (rope_pending && mbar_test(smem_u32(rope_full), jq & 1)) {
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const uint64_t ad = smem_desc(q_base + 8 * C::Q_CHUNK + kk * 32, 16, 1024, SW128);
              const uint64_t bd = smem_desc(rope_base + kk * 32, 16, 1024, SW128);
              mma_bf16_pair(tS + (jq & 1) * 64, ad, bd, id_qr, 1u);
            }
            MLA_TRACE_EVENT(tunit, 7, jq);
            mma_commit_pair(&s_full[jq & 1]);
            cq.step(a);
            rope_pending = false;
            sbuf_ok = false;
            prog = true;
          }
        }
        if (prog) {
          t_idle = 0;
          spins = 0;
        } else if ((++spins & 63u) != 0) {
          if (PAIR_BACKOFF_NS > 0) __nanosleep(PAIR_BACKOFF_NS);
        } else {
          if (*abort_flag) break;
          const uint64_t now = globaltimer_ns();
          if (t_idle == 0) {
            t_idle = now;
          } else if (now - t_idle > g_spin_limit_ns) {
            record_error(ERR_TIMEOUT, 512);
            *abort_flag = 1;
            ok = false;
          }
        }
      }
    }
  } else if (F8 && warp >= C::CONV_WARP0) {
    // ------------------------------------------------------------ F8 converters
    // Units of two warps, thread = token row r of a page.  The first half of
    // the units expands the four own-page pairs of every tile (and, per
    // segment, turns the queries' latent chunks into f16 in place); the
    // second half expands the two pairs this CTA refills from the other page.
    // With two units per half, unit i of a half takes every second pair.  A
    // thread reads its row's 128 codes from the slot's upper half and writes
    // code * 2^e as f16 into both halves in the MMA's SW128 layout: columns
    // 0..63 to the lower half, 64..127 over exactly the bytes it has just
    // read.  Rows past kv_len are written as zeros (PV multiplies them by
    // P = 0, and a stale code may be a NaN).  The values are exact for row
    // scales 2^e, -15 <= e <= 7.
    constexpr int NU = C::CONV_WARPS / 4;  // units per half
    const int ct = threadIdx.x - 32 * C::CONV_WARP0;
    const int unit = ct >> 6, r = ct & 63;
    const bool own_half = unit < NU;
    const int sg = unit % NU;
    constexpr int ROWB = fp8_row_bytes(ATT_DC, ATT_DR);
    auto row_scale = [&](int blk, int nvalid) -> float {
      if (r >= nvalid || blk >= a.num_blocks) return 0.f;
      return *reinterpret_cast<const float*>(a.pool + ((size_t)blk * 64 + r) * ROWB + fp8_scale_off(ATT_DC, ATT_DR));
    };
    auto expand = [&](int s, uint32_t sc2, bool valid) {
      uint8_t* row = smem + C::OFF_PAIR + s * C::PAIR + r * 128;
      const uint4* in = reinterpret_cast<const uint4*>(row + C::CODES);
      // thread r takes its row's 16-byte units in the order r, r+1, ... (mod
      // 8), so the rows of a warp spread over all banks
      uint4 v[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) v[j] = in[(j + r) & 7];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        // codes 16k .. 16k+15: f16 columns 16(k%4) .. +15 of half k/4, 16-byte units 2(k%4), 2(k%4)+1
        const int k = (j + r) & 7;
        uint8_t* half = row + (k >> 2) * C::CODES;
        const uint32_t u0 = 2u * (k & 3);
        uint4 lo = make_uint4(0, 0, 0, 0), hi = make_uint4(0, 0, 0, 0);
        if (valid) {
          lo = make_uint4(f16x2_from_e4m3x2((uint16_t)v[j].x, sc2), f16x2_from_e4m3x2((uint16_t)(v[j].x >> 16), sc2),
                          f16x2_from_e4m3x2((uint16_t)v[j].y, sc2), f16x2_from_e4m3x2((uint16_t)(v[j].y >> 16), sc2));
          hi = make_uint4(f16x2_from_e4m3x2((uint16_t)v[j].z, sc2), f16x2_from_e4m3x2((uint16_t)(v[j].z >> 16), sc2),
                          f16x2_from_e4m3x2((uint16_t)v[j].w, sc2), f16x2_from_e4m3x2((uint16_t)(v[j].w >> 16), sc2));
        }
        *reinterpret_cast<uint4*>(half + ((u0 ^ (uint32_t)(r & 7)) << 4)) = lo;
        *reinterpret_cast<uint4*>(half + (((u0 + 1) ^ (uint32_t)(r & 7)) << 4)) = hi;
      }
    };
    // one arrive per warp on the leader's barrier, after every lane's writes
    // are visible to the tensor core
    auto announce = [&](uint64_t* b) {
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        if (rank == 0)
          mbar_arrive(b);
        else
          PAIR_ARRIVE(mapa_shared(smem_u32(b), 0));
      }
    };
    TileCursor c;
    c.init(a, range);
    bool ok = true;
    while (ok && !c.done()) {
      const int g = c.g;
      if (own_half) {
        if (c.first()) {
          // every lane leaves a wait before its warp's __syncwarp: give up as a warp
          if (!__all_sync(0xffffffffu, mbar_wait(q_land, c.n & 1, abort_flag, 531))) break;
          uint4* qv = reinterpret_cast<uint4*>(smem + C::OFF_Q);
          for (int i = ct; i < 8 * C::Q_CHUNK / 16; i += 64 * NU) {
            const uint4 w = qv[i];
            qv[i] = make_uint4(f16x2_from_bf16x2(w.x), f16x2_from_bf16x2(w.y), f16x2_from_bf16x2(w.z),
                               f16x2_from_bf16x2(w.w));
          }
          announce(q_full);
        }
        const int page = c.tok() / 64 + (int)rank;
        const int blk = page_block(c, page);
        const int nvalid = min(64, max(0, c.S.kv - 64 * page));
        const float sc = row_scale(blk, nvalid);
        const uint32_t sc2 = pack_f16(sc, sc);
        for (int k = sg; k < 4; k += NU) {
          const int s = slot_of(g, k);
          if (!__all_sync(0xffffffffu, mbar_wait(&own_land[s], use_of(g, k) & 1, abort_flag, 532))) {
            ok = false;
            break;
          }
          expand(s, sc2, r < nvalid);
          announce(&own_full[s]);
        }
      } else {
        // this CTA refills pairs k with (k & 1) != rank: the other page's tokens
        const int page = c.tok() / 64 + (int)(rank ^ 1u);
        const int blk = page_block(c, page);
        const int nvalid = min(64, max(0, c.S.kv - 64 * page));
        const float sc = row_scale(blk, nvalid);
        const uint32_t sc2 = pack_f16(sc, sc);
        for (int k = (int)(rank ^ 1u) + 2 * sg; k < 4; k += 2 * NU) {
          const int s = slot_of(g, k);
          if (!__all_sync(0xffffffffu, mbar_wait(&oth_land[s], use_of(g, k) & 1, abort_flag, 533))) {
            ok = false;
            break;
          }
          expand(s, sc2, r < nvalid);
          announce(&oth_full[s]);
        }
      }
      c.step(a);
    }
  } else {
    // ------------------------------------------------------------ softmax + epilogue
    const int q = warp & 3;
    const int L = q * 32 + lane;     // TMEM lane
    const int h = L & 63;            // head within this CTA
    const int g = L >> 6;            // which page of the tile this thread's scores cover
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    const uint32_t l_sfree[2] = {mapa_shared(smem_u32(&s_free[0]), 0), mapa_shared(smem_u32(&s_free[1]), 0)};
    const uint32_t l_pfull[2] = {mapa_shared(smem_u32(&p_full[0]), 0), mapa_shared(smem_u32(&p_full[1]), 0)};
    uint32_t gphase = 0;
    auto group_sync = [&](int site) -> bool {
      mbar_arrive(grp_bar);
      const bool ok2 = PAIR_SM_WAIT(grp_bar, gphase & 1, abort_flag, site);
      ++gphase;
      return ok2;
    };
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    const int tunit_sm = rank == 0 ? worker : 256 + worker;  // trace slot of this CTA's softmax
    (void)tunit_sm;
    TileCursor c;
    c.init(a, range);
    while (ok && !c.done()) {
      const int j = c.g;
      if (c.first()) {
        m_run = -INFINITY;
        l_run = 0.f;
      }
      if (!PAIR_SM_WAIT(&s_full[j & 1], (j >> 1) & 1, abort_flag, 521)) {
        ok = false;
        break;
      }
      if (L == 0) MLA_TRACE_EVENT(tunit_sm, 8, j);
      tc_fence_after();
      float s[64];
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) tmem_ld32<16>(tS + (j & 1) * 64 + cc * 16 + lane_off, s + 16 * cc);
      tmem_wait_ld();
      tc_fence_before();
      const int tok0 = c.tok() + 64 * g;
      const int nvalid = min(64, max(0, c.S.t_end - tok0));
      float pmax = -INFINITY;
#pragma unroll
      for (int cc = 0; cc < 64; ++cc) {
        s[cc] = cc < nvalid ? s[cc] * a.scale_log2 : -INFINITY;
        pmax = fmaxf(pmax, s[cc]);
      }
      float* rb = red + (j & 1) * 128;
      rb[L] = pmax;
      if (!group_sync(522)) {
        ok = false;
        break;
      }
      if (L == 0) MLA_TRACE_EVENT(tunit_sm, 22, j);
      // every thread's TMEM reads of S(j) are complete: release the buffer
      if (L == 0) {
        if (rank == 0)
          mbar_arrive(&s_free[j & 1]);
        else
          PAIR_ARRIVE(l_sfree[j & 1]);
      }
      const float m_new = fmaxf(m_run, fmaxf(pmax, rb[L ^ 64]));
      // Warps q and q+2 hold the two page halves of the same 32 heads with
      // equal (m_new, m_run), so both take the same decision.
      const bool grow = __any_sync(0xffffffffu, m_new > m_run + ATT_RESCALE_LOG2);
      float alpha = 1.f;
      bool rescale = false;
      if (c.first()) {
        m_run = m_new;  // PV of a segment's first tile overwrites O
      } else if (grow) {
        alpha = exp2_approx(m_run - m_new);
        l_run *= alpha;
        m_run = m_new;
        rescale = true;
      }
      // P of this tile in registers; its store into the tile's TMEM P buffer
      // waits for PV(j-2), a rescale of O for PV(j-1)
      uint32_t pk[8][4];
#pragma unroll
      for (int cc = 0; cc < 8; ++cc) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float p0 = exp2_approx(s[8 * cc + 2 * e] - m_run);
          const float p1 = exp2_approx(s[8 * cc + 2 * e + 1] - m_run);
          l_run += p0 + p1;
          pk[cc][e] = F8 ? pack_f16(p0, p1) : pack_bf16(p0, p1);
        }
      }
      // Both TMEM lanes of a head (h and 64 + h) must hold P over all 128
      // tokens of the tile (the duplicated A layout of the 2-SM MMA), but
      // each thread computed one page: swap halves with the partner thread
      // (same head, other page) through the staging buffer.  Its reuse by the
      // next tile comes after that tile's max exchange, which every thread
      // reaches only after reading this tile's halves.
      uint4* stg = reinterpret_cast<uint4*>(smem + C::OFF_P);  // [page][8][64 heads]
#pragma unroll
      for (int cc = 0; cc < 8; ++cc) stg[(g * 8 + cc) * 64 + h] = make_uint4(pk[cc][0], pk[cc][1], pk[cc][2], pk[cc][3]);
      if (!group_sync(526)) {
        ok = false;
        break;
      }
      if (L == 0) MLA_TRACE_EVENT(tunit_sm, 23, j);
      uint32_t po[8][4];
#pragma unroll
      for (int cc = 0; cc < 8; ++cc) {
        const uint4 v = stg[((g ^ 1) * 8 + cc) * 64 + h];
        po[cc][0] = v.x;
        po[cc][1] = v.y;
        po[cc][2] = v.z;
        po[cc][3] = v.w;
      }
      // the P buffer of this tile was last read by PV(j-2); a rescale of O
      // needs PV(j-1) complete
      if (j >= 2 || (rescale && j >= 1)) {
        const int jw = rescale ? j - 1 : j - 2;
        if (!mbar_wait(&pv_done[jw & 1], (jw >> 1) & 1, abort_flag, 523)) {
          ok = false;
          break;
        }
        if (L == 0) MLA_TRACE_EVENT(tunit_sm, 9, j);
        tc_fence_after();
      }
      if (rescale) {
#pragma unroll 1
        for (int cc = 0; cc < 256; cc += 16) {
          float o[16];
          tmem_ld32<16>(tO + cc + lane_off, o);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 16; ++e) o[e] *= alpha;
          tmem_st32<16>(tO + cc + lane_off, o);
        }
        tmem_wait_st();
      }
      {
        // columns [0,32): page 0's tokens, [32,64): page 1's; two tokens per column
        const uint32_t pt = tP + (j & 1) * 64 + lane_off;
        tmem_st32<32>(pt + 32 * g, reinterpret_cast<const float*>(&pk[0][0]));
        tmem_st32<32>(pt + 32 * (g ^ 1), reinterpret_cast<const float*>(&po[0][0]));
        tmem_wait_st();
      }
      tc_fence_before();
#if PAIR_WARP_ARRIVE
      // each warp announces its own stores (p_full counts 4 warps x 2 CTAs)
      __syncwarp();
      if (lane == 0) {
        if (rank == 0)
          mbar_arrive(&p_full[j & 1]);
        else
          PAIR_ARRIVE(l_pfull[j & 1]);
        if (L == 0) MLA_TRACE_EVENT(tunit_sm, 10, j);
        if (L == 32) MLA_TRACE_EVENT(tunit_sm, 24, j);
        if (L == 64) MLA_TRACE_EVENT(tunit_sm, 25, j);
        if (L == 96) MLA_TRACE_EVENT(tunit_sm, 26, j);
      }
#else
      if (!group_sync(528)) {
        ok = false;
        break;
      }
      if (L == 0) {
        if (rank == 0)
          mbar_arrive(&p_full[j & 1]);
        else
          PAIR_ARRIVE(l_pfull[j & 1]);
        MLA_TRACE_EVENT(tunit_sm, 10, j);
      }
#endif
      if (c.last()) {
        // ---------------------------------------------------------- epilogue of the segment
        // O is read out before this thread writes the next segment's first P,
        // which is what PV of that tile (overwriting O) waits for.
        const SegInfo& S = c.S;
        float* lred = red + 256;
        lred[L] = l_run;
        ok = group_sync(524) && ok;
        const float l_tot = l_run + lred[L ^ 64];
        ok = ok && mbar_wait(&pv_done[j & 1], (j >> 1) & 1, abort_flag, 525);
        tc_fence_after();
        const float inv_l = 1.f / l_tot;
        const long long ob = ((long long)S.r * a.n_h + head0 + h) * ATT_DC;
        const bool direct = S.pslot < 0;
#pragma unroll 1
        for (int cc = 0; cc < 256; cc += 16) {
          float o[16];
          tmem_ld32<16>(tO + cc + lane_off, o);
          tmem_wait_ld();
          if (!ok) continue;
          // TMEM column cc of this lane: latent index 256*(cc/128) + 128*g + cc%128
          const int d = 256 * (cc >> 7) + 128 * g + (cc & 127);
          if (direct) {
            uint4 v0 = make_uint4(pack_bf16(o[0] * inv_l, o[1] * inv_l), pack_bf16(o[2] * inv_l, o[3] * inv_l),
                                  pack_bf16(o[4] * inv_l, o[5] * inv_l), pack_bf16(o[6] * inv_l, o[7] * inv_l));
            uint4 v1 = make_uint4(pack_bf16(o[8] * inv_l, o[9] * inv_l), pack_bf16(o[10] * inv_l, o[11] * inv_l),
                                  pack_bf16(o[12] * inv_l, o[13] * inv_l), pack_bf16(o[14] * inv_l, o[15] * inv_l));
            uint4* dst = reinterpret_cast<uint4*>(a.o_lat + ob + d);
            dst[0] = v0;
            dst[1] = v1;
          } else {
            float4* dst =
                reinterpret_cast<float4*>(a.o_part + ((long long)S.pslot * a.n_h + head0 + h) * ATT_DC + d);
#pragma unroll
            for (int e = 0; e < 4; ++e)
              dst[e] = make_float4(o[4 * e] * inv_l, o[4 * e + 1] * inv_l, o[4 * e + 2] * inv_l,
                                   o[4 * e + 3] * inv_l);
          }
        }
        tc_fence_before();
        if (ok && g == 0) {
          const float lse = (m_run + log2f(l_tot)) * 0.69314718055994531f;
          if (direct) {
            if (a.lse) a.lse[(long long)S.r * a.n_h + head0 + h] = lse;
          } else {
            a.lse_part[(long long)S.pslot * a.n_h + head0 + h] = lse;
          }
        }
      }
      c.step(a);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0) MLA_TRACE_EVENT(tunit, 11, 0);
  // A role of this CTA gave up a wait: its peer's roles may be waiting for
  // this CTA's signals, so raise the peer's abort flag too (their waits poll
  // it) rather than let each of them run into its own time limit.
  if (threadIdx.x == 0 && *abort_flag)
    st_cluster_u32(mapa_shared(smem_u32(const_cast<int*>(abort_flag)), rank ^ 1u), 1u);
  cluster_sync_all();  // the peer's MMAs, TMA signals and arrives are done
  if (warp == 1) tmem_dealloc_pair(tmem, C::TMEM_COLS);
}

}  // namespace mla
