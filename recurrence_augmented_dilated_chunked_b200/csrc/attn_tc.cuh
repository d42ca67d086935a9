// attn_tc.cuh -- dilated (+ windowed) prefill attention on the 5th-generation
// tensor cores (TMA + tcgen05.mma, accumulators and P in tensor memory).
//
// Computes, for every (b, h, t), softmax attention of q[b,t,h] over the
// recurrent keys/values at K_h(t) = {j < t : j mod D_h = D_h-1} U {t}
// U {t-W < j <= t} (RAT+ abstract: dilated attention with optional local
// windows; write-up section 6: dense heads D_h = 1).  bf16 in, fp32
// accumulate, head dim 128.
//
// Work item = (b, h, 128-query tile).  Its keys come in 64-key tiles of two
// kinds, both fetched by plain tiled TMA boxes:
//   * dilated tiles: slots s..s+63 of the strided view of hk/hv whose row s
//     is position s*D + D - 1 (base offset D-1 rows, row stride D rows), so the
//     gather is an ordinary box of the strided tensor map; a dense head reads
//     the positional view instead (slot = position);
//   * window tiles (dilated heads only): positions of [t0 - W' + 1, t_last],
//     W' = max(W, 1), so W = 0 still supplies the self key t.
// Each key is counted once by splitting the set at the window: row t takes
// every window position t-W'+1..t and only the dilated slots whose position
// lies before the window, s < floor((t - W' + 1) / D).  So per-row validity is
// a prefix (dilated; dense: s <= t) or a contiguous range (window), applied as
// bit masks per 32-column chunk.
//
// Items are listed segment by segment; a segment is a product set (samples x
// heads) of one dilation: samples whose D is 1 with every head, the other
// samples with the dense heads (both dense), then, per dilation D_c > 1 in
// ascending order, the samples of D_c with the dilated heads.  One dilation
// for the whole batch (the per-head hybrid) is the case of a single dilated
// segment; several (per-sample D, the batch composition of the write-up's
// section 2.2, where half the samples run dense and half at D = 64) take one
// strided tensor-map pair each.  Within a dense segment, late query tiles come
// first across all of its (b, h); a dilated segment runs (b, h) by (b, h),
// late query tiles first, so that its dilated rows stay in L2.
//
// Two CTAs per SM, persistent over items blockIdx.x, +G, +2G, ... (G = grid
// size = 2 x SMs; dense segments, the heaviest items, come first).  When a
// launch mixes segments (dense and dilated items, whose costs differ by up to
// ~D x), every other round is dealt in reverse CTA order, so that the CTAs
// that drew the heaviest items in one round draw the lightest in the next
// (7.6B hybrid layer: 797 -> 753 us; a single segment keeps plain rounds,
// which measured 2.6% faster on an all-dense layer).  Given a workspace, a
// mixed launch instead hands out items from a counter as CTAs become free
// (attn_kernel<false, true>, through the same item ring as the fused prefill).  Per CTA, tensor memory holds S (64 columns), two P buffers (bf16
// pairs, 32 columns each) and O (128 columns): 256 columns, half an SM's.
// Because S and P are separate, S = Q K^T of tile n+1 is issued as soon as
// the softmax has read S of tile n, so the tensor core computes the next
// scores while the softmax of the current tile runs; O += P V of tile n
// follows the softmax.  The other CTA on the SM fills the remaining gaps.
//
// Roles (192 threads per CTA):
//   warps 0-3  softmax: one thread per query row (warp w reads TMEM lanes
//              32w..32w+31), all 64 key columns of the row.  Reads S, frees
//              it, masks, takes the row max, writes P = 2^(s - m) as bf16 pairs
//              into P buffer n%2, rescales O in TMEM only when the running max
//              grew by more than 2^8, and after the item's last tile
//              normalises O and stores the output rows.
//   warp 4     one lane: TMA producer of Q (one buffer), K and V (two stages
//              each);
//   warp 5     allocates TMEM and one lane issues S = Q K^T (M=128, N=64,
//              K=128; Q and K K-major in smem) and O += P V (M=128, N=128,
//              K=64; P K-major in TMEM, V MN-major in smem) as tcgen05.mma with
//              K=16 steps, from precomputed descriptors.  Per item: S(0), then
//              S(j) and P V(j-1) for j >= 1, then P V of the last tile.
// Every mbarrier wait is bounded; on expiry the CTA records RATP_ERR_TIMEOUT,
// all roles drain out (copies and MMAs in flight are waited for), and TMEM
// is released.
//
// attn_kernel<true> is the fused prefill (fused.cuh): 256 threads per CTA;
// the first CTAs to start scan the recurrence, the others run the pipeline
// above (warps 6-7 idle) over query tiles in ascending order, waiting per
// item for the scanned chunks it reads.  Its tiles end at the item's last
// row: window tiles end at t_last and start at or before the window's first
// row, the dilated tiles end at the item's last dilated slot (the first ones
// may start before slot 0, which TMA fills with zeros), so no tile loads a
// row after the item's last query.
#pragma once
#include "sm100.cuh"
#include "fused.cuh"

namespace ratp {
namespace attn_tc {

constexpr int BM = 128;          // queries per tile
constexpr int BN = 64;           // keys per tile
constexpr int DH = 128;          // head dim
constexpr int kCtasPerSm = 2;
constexpr int kSoftmaxWarps = 4;
constexpr int kProducerWarp = 4;
constexpr int kMmaWarp = 5;
constexpr int kThreads = 192;
// The fused prefill's CTAs have the chunk scan's 256 threads.
constexpr int kThreadsFused = 256;
constexpr uint32_t kQHalf = BM * 64 * 2;       // Q: 128 rows x 64 columns: 16 KB
constexpr uint32_t kQTile = 2 * kQHalf;        // 32 KB
constexpr uint32_t kKHalf = BN * 64 * 2;       // K/V: 64 rows x 64 columns: 8 KB
constexpr uint32_t kKTile = 2 * kKHalf;        // 16 KB
constexpr uint32_t kOffQ = 0;
constexpr uint32_t kOffK = kOffQ + kQTile;     // 2 stages
constexpr uint32_t kOffV = kOffK + 2 * kKTile; // 2 stages
constexpr uint32_t kOffBar = kOffV + 2 * kKTile;
// barriers: qfull qempty kfull[2] kempty[2] vfull[2] sfull sfree pfull[2] pvdone[2] final item[8]
constexpr uint32_t kNumBars = 23;
constexpr int kItemRing = 8;       // fused: item indices handed from the producer to the other roles
// after the barriers: TMEM address, abort flag, item ring; then alignment slack
constexpr uint32_t kCtlBytes = 8 + 4 * kItemRing;
constexpr uint32_t kSmemBytes = kOffBar + kNumBars * 8 + kCtlBytes + 1024;
// fused: a scan CTA stages its chunk tiles from the same (1024-aligned) base;
// the barriers and control words lie past them, since the CTA goes on to
// attend after its scan
constexpr uint32_t kScanBytes = scan::Smem<__nv_bfloat16, 2>::kBytes;
constexpr uint32_t kOffBarFused = (kScanBytes + 7) & ~7u;
constexpr uint32_t kSmemBytesFused = kOffBarFused + kNumBars * 8 + kCtlBytes + 1024;
static_assert(kOffBarFused >= kOffBar, "fused layout");
constexpr uint32_t kTmemCols = 256;
constexpr uint32_t kColS = 0;      // S: 64 columns
constexpr uint32_t kColP = 64;     // P buffer b at 64 + 32 b
constexpr uint32_t kColO = 128;    // O: 128 columns
constexpr float kRescaleThreshold = 8.0f;   // log2 units
// The O rescale and the epilogue run once per item or less often: their
// loops stay rolled, which keeps the softmax loop's code compact (measured
// 2% faster than unrolling them).
constexpr int kColdUnroll = 1;
static_assert(kCtasPerSm * (kSmemBytesFused + 1024) <= 233472, "two CTAs per SM");

constexpr int kMaxDil = 4;                 // distinct dilations D > 1 in one launch
constexpr int kMaxSeg = 2 + kMaxDil;
constexpr int kMaxSamples = 1024;          // batch size with per-sample dilation

// Head sets a segment ranges over
constexpr int kHeadsDense = 0, kHeadsDil = 1, kHeadsAll = 2;

struct Segment {
  int begin;        // first item index of the segment
  int n_b, n_h;     // samples x heads
  int b_off;        // samples[b_off + i] is sample i; -1: sample i is b = i
  int8_t heads;     // kHeadsDense / kHeadsDil / kHeadsAll
  int8_t cls;       // -1: dense; c >= 0: dilation dil_D[c], tensor maps k[c], v[c]
  int tail;         // dilated: (b, h) pairs from this one on are interleaved
};

// Strided ("dilated") views of hk and hv, one pair per dilation class: row s
// of class c is position s * dil_D[c] + dil_D[c] - 1.
struct DilMaps {
  CUtensorMap k[kMaxDil];
  CUtensorMap v[kMaxDil];
};

struct Params {
  __nv_bfloat16* o;
  int B, T, H, W_eff, NQ;
  int n_items, n_seg, n_cls;
  int alternate;          // deal every other round of items in reverse CTA order
  float scale_log2;
  int o_align32;          // output base 32-byte aligned (rows are 256 bytes)
  int dil_D[kMaxDil];
  Segment seg[kMaxSeg];
  uint8_t dense_list[RATP_MAX_HEADS];
  uint8_t dil_list[RATP_MAX_HEADS];
  uint16_t samples[kMaxSamples];   // samples grouped by dilation (per-sample mode)
  // fused prefill: items in ascending order (query tile major, then b, h),
  // head h dense where bit h of dense_bits is set, else dilation dil_D[0]
  unsigned long long dense_bits[RATP_MAX_HEADS / 64];
  fused::Scan scan;                // chunk scan of x_k, x_v with g into h_k, h_v
  fused::Control ctl;
};

// The fused prefill's scan inputs: [B][T][H*128] views of g, x_k, x_v, box
// 64 channels x 256 tokens.
struct ScanMaps {
  CUtensorMap g, xk, xv;
};

struct Item {
  int b, h, t0, t_last, Dd, n_win, n_tiles, p_start, cls;
  int win0;         // first row of the first window tile
  int dil0;         // first slot of the first dilated tile (< 0: zero-filled rows)
  bool dense;
};

template <bool FUSED, bool DYN>
__device__ __forceinline__ Item make_item(const Params& p, int idx) {
  Item it;
  if (FUSED) {
    // ascending: every unit an item reads is scanned by an item that comes
    // no later in this order
    const int per = p.B * p.H;
    const int qi = idx / per;
    const int rem = idx - qi * per;
    it.b = rem / p.H;
    it.h = rem - it.b * p.H;
    it.cls = 0;
    it.dense = ((p.dense_bits[it.h >> 6] >> (it.h & 63)) & 1ull) != 0ull || p.dil_D[0] == 1;
    it.t0 = qi * BM;
  } else {
    int s = 0;
    while (s + 1 < p.n_seg && idx >= p.seg[s + 1].begin) ++s;
    const Segment& g = p.seg[s];
    idx -= g.begin;
    // dense segments: query tile major (the heaviest items, late query tiles,
    // first across all of the segment's (b, h)); dilated segments: (b, h)
    // major, late query tiles first within each (b, h), so that the few
    // (b, h) in flight at a time keep their dilated rows in L2 (measured on
    // the 7.6B hybrid layer: DRAM reads 2.18 -> 0.83 GB, 826 -> 787 us)
    // With dynamic dealing (DYN) the last (b, h) pairs of a dilated segment
    // (from g.tail on) are interleaved, late query tiles first across them, so
    // that the launch ends on light items (at most 32 pairs' rows in flight).
    int qi, bi, hi;
    if (g.cls >= 0) {
      int pair;
      if (!DYN || idx < g.tail * p.NQ) {
        pair = idx / p.NQ;
        qi = idx - pair * p.NQ;
      } else {
        const int j = idx - g.tail * p.NQ;
        const int n_t = g.n_b * g.n_h - g.tail;
        qi = j / n_t;
        pair = g.tail + (j - qi * n_t);
      }
      bi = pair / g.n_h;
      hi = pair - bi * g.n_h;
    } else {
      const int per = g.n_b * g.n_h;
      qi = idx / per;
      const int rem = idx - qi * per;
      bi = rem / g.n_h;
      hi = rem - bi * g.n_h;
    }
    it.b = g.b_off < 0 ? bi : (int)p.samples[g.b_off + bi];
    it.h = g.heads == kHeadsDense ? (int)p.dense_list[hi] : g.heads == kHeadsDil ? (int)p.dil_list[hi] : hi;
    it.cls = g.cls < 0 ? 0 : g.cls;
    it.dense = g.cls < 0;
    it.t0 = (p.NQ - 1 - qi) * BM;
  }
  it.t_last = min(it.t0 + BM - 1, p.T - 1);
  if (it.dense) {
    it.Dd = 1;
    it.n_win = 0;
    it.p_start = 0;
    it.n_tiles = (it.t_last + 1 + BN - 1) / BN;
  } else {
    it.Dd = p.dil_D[it.cls];
    const int n_dil = max(0, it.t_last - p.W_eff + 1) / it.Dd;   // slots before the last row's window
    const int n_dt = (n_dil + BN - 1) / BN;
    it.p_start = max(0, it.t0 - p.W_eff + 1);
    it.n_win = (it.t_last - it.p_start + 1 + BN - 1) / BN;
    it.n_tiles = it.n_win + n_dt;
    // the fused prefill's tiles end at the item's last row / slot; the
    // others start at the window's first row and at slot 0
    it.win0 = FUSED ? it.t_last + 1 - it.n_win * BN : it.p_start;
    it.dil0 = FUSED ? n_dil - n_dt * BN : 0;
  }
  if (it.dense) {
    it.win0 = 0;
    it.dil0 = 0;
  }
  return it;
}


// Waits (whole warp) until the scan has stored every row that the item's
// tiles load: with the fused prefill's tile placement all of them lie at or
// before t_last, and chunks complete in sequence order per chain, so the done
// flags of t_last's chunk in the head's two 64-channel chains suffice (lanes
// 0 and 1 poll one each).  Rows a tile loads but no query attends to still
// enter O += P V with P = 0, so they must hold finite values, which an
// unscanned part of h_k/h_v need not.  Then the TMA loads that lane 0 issues
// next see the scan's stores.  False if the wait ran out or another CTA
// aborted.
__device__ __forceinline__ bool wait_chunks(const Params& p, const Item& it, unsigned int tag, int lane,
                                            volatile int* s_abort) {
  const fused::Scan& sc = p.scan;
  const int chunk = min(it.t_last / scan::Shape<__nv_bfloat16>::kChunk, sc.n_chunks_t - 1);
  const long long chain = (long long)it.b * sc.slabs + 2 * it.h + (lane & 1);
  const long long desc = chain * sc.n_chunks_t + chunk;
  const unsigned long long t0 = global_ns();
  unsigned int polls = 0;
  bool done = lane >= 2;
  while (true) {
    if (!done && RATP_IN(desc, 1, (long long)sc.n_chains * sc.n_chunks_t))
      done = fused::ld_acquire(sc.done + desc) == tag;
    if (__all_sync(0xffffffffu, done)) break;
    bool expired = false, give_up = false;
    if ((++polls & 15u) == 0u) {
      expired = global_ns() - t0 > spin_timeout();
      give_up = expired || *s_abort || fused::aborted(sc.ws.abort);
    }
    if (__any_sync(0xffffffffu, give_up)) {
      if (__any_sync(0xffffffffu, expired) && lane == 0) raise_error(RATP_ERR_TIMEOUT);
      if (lane == 0) {
        *s_abort = 1;
        fused::abort_all(sc.ws.abort);
      }
      return false;
    }
    __nanosleep(32);
  }
  __syncwarp();
  if (lane == 0) {
    asm volatile("fence.acq_rel.gpu;" ::: "memory");
    asm volatile("fence.proxy.async.global;" ::: "memory");
  }
  __syncwarp();
  return true;
}

// DYN: a mixed non-fused launch given a workspace; its items are drawn from
// the counter ctl.items (a separate instance, so that the static kernel's
// code is unchanged: the larger body cost the static path instruction
// fetches, T=16K +4% cycles).
template <bool FUSED, bool DYN = false>
__global__ void __launch_bounds__(FUSED ? kThreadsFused : kThreads, kCtasPerSm)
attn_kernel(const __grid_constant__ CUtensorMap tm_q,
            const __grid_constant__ CUtensorMap tm_kpos,
            const __grid_constant__ CUtensorMap tm_vpos,
            const __grid_constant__ DilMaps tm_dil,
            const __grid_constant__ ScanMaps tm_scan,
            const __grid_constant__ Params p) {
  using namespace sm100;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_u32(smem);
  const uint32_t sQ = sb + kOffQ, sK = sb + kOffK, sV = sb + kOffV;
  constexpr uint32_t off_bar = FUSED ? kOffBarFused : kOffBar;
  const uint32_t bar0 = sb + off_bar;
  const uint32_t b_qfull = bar0 + 0 * 8;    // Q landed
  const uint32_t b_qempty = bar0 + 1 * 8;   // last S = Q K^T of an item done
  const uint32_t b_kfull = bar0 + 2 * 8;    // [2] K stage landed
  const uint32_t b_kempty = bar0 + 4 * 8;   // [2] S = Q K^T read the K stage
  const uint32_t b_vfull = bar0 + 6 * 8;    // [2] V stage landed
  const uint32_t b_sfull = bar0 + 8 * 8;    // S = Q K^T done
  const uint32_t b_sfree = bar0 + 9 * 8;    // S read by the softmax (128 threads)
  const uint32_t b_pfull = bar0 + 10 * 8;   // [2] P buffer written (128 threads)
  const uint32_t b_pvdone = bar0 + 12 * 8;  // [2] O += P V done: P buffer and V stage free
  const uint32_t b_final = bar0 + 14 * 8;
  const uint32_t b_item = bar0 + 15 * 8;    // [kItemRing] fused: item index written
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + off_bar + kNumBars * 8);
  volatile int* s_abort = reinterpret_cast<volatile int*>(smem + off_bar + kNumBars * 8 + 4);
  volatile int* s_items = reinterpret_cast<volatile int*>(smem + off_bar + kNumBars * 8 + 8);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(b_qfull, 1);
    mbar_init(b_qempty, 1);
    mbar_init(b_sfull, 1);
    mbar_init(b_sfree, kSoftmaxWarps * 32);
    for (int i = 0; i < 2; ++i) {
      mbar_init(b_kfull + 8 * i, 1);
      mbar_init(b_kempty + 8 * i, 1);
      mbar_init(b_vfull + 8 * i, 1);
      mbar_init(b_pfull + 8 * i, kSoftmaxWarps * 32);
      mbar_init(b_pvdone + 8 * i, 1);
    }
    mbar_init(b_final, 1);
    for (int i = 0; i < kItemRing; ++i) mbar_init(b_item + 8 * i, 1);
    *s_abort = 0;
    fence_barrier_init();
  }
  // every CTA allocates its tensor memory and gives up the allocation permit
  // at once (a fused scan CTA attends after its scan)
  if (warp == kMmaWarp) {
    tmem_alloc(smem_u32(s_tmem), kTmemCols);
    tmem_relinquish();
  }
  if (warp == kProducerWarp && lane == 0) {
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_kpos);
    prefetch_tmap(&tm_vpos);
    for (int c = 0; c < p.n_cls; ++c) {
      prefetch_tmap(&tm_dil.k[c]);
      prefetch_tmap(&tm_dil.v[c]);
    }
  }
  unsigned int tag = 0u;
  __shared__ unsigned int s_start, s_tag;
  if (FUSED && threadIdx.x == 0) {
    // the role comes from the order in which the CTAs start (fused.cuh);
    // every CTA draws exactly one ticket, which also returns the launch tag
    unsigned int tk;
    s_tag = scan::draw_ticket(p.scan.ws, (unsigned int)p.ctl.n_ctas, &tk);
    s_start = tk;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s_tmem;
  if (FUSED) {
    tag = s_tag;
    if ((int)s_start < p.ctl.n_scan) {
      // scan until the chunk tickets run out, then attend like the others
      fused::scan_role(tm_scan.g, tm_scan.xk, tm_scan.xv, p.scan, p.ctl, smem, tag);
      __syncthreads();
    }
  }
  // This CTA's items: FUSED (and a DYN launch) draws them one by
  // one from the launch's item counter, the producer passing each index on
  // through the ring (an index >= n_items ends the loop); otherwise
  // blockIdx.x, +G, +2G, ... (every other round reversed with p.alternate).
  // The producer runs at most a few items ahead of the MMA issuer and the
  // softmax (it waits for O += P V of tile n-2 before it loads tile n), far
  // less than the ring's depth.
  auto item_of = [&](int li) -> int {           // static dealing, round li
    const int G = (int)gridDim.x, c = (int)blockIdx.x;
    return (p.alternate && (li & 1)) ? (li + 1) * G - 1 - c : c + li * G;
  };
  auto item_at = [&](int li) -> int {
    if (!FUSED && !DYN) return item_of(li);
    if (!mbar_wait(b_item + 8 * (li % kItemRing), (uint32_t)(li / kItemRing) & 1u, s_abort)) return -1;
    return s_items[li % kItemRing];
  };

  if (warp == kProducerWarp) {
    // ------------------------------------------------------------ producer
    // Tile n (stage n%2): K once S = Q K^T of tile n-2 read the stage; at an
    // item's first tile then Q, once the previous item's last S = Q K^T is
    // done (its K load is already under way); V once O += P V of tile n-2
    // read the stage.  The fused prefill draws the item, passes its index on
    // and first waits (whole warp) for the scanned chunks the item reads.
    int n = 0, nq = 0;
    int last_k[2] = {-1, -1}, last_v[2] = {-1, -1};   // last tile loaded per stage
    bool ok = true;
    for (int li = 0;; ++li) {
      int idx;
      if (FUSED || DYN) {
        if (lane == 0) {
          idx = ok ? (int)min(atomicAdd(p.ctl.items, 1u), (unsigned int)p.n_items) : p.n_items;
          s_items[li % kItemRing] = idx;           // n_items: no more items
          mbar_arrive(b_item + 8 * (li % kItemRing));
        }
        idx = __shfl_sync(0xffffffffu, idx, 0);
      } else {
        idx = item_of(li);
      }
      if (!ok || idx >= p.n_items) break;
      const Item it = make_item<FUSED, DYN>(p, idx);
      if (FUSED && !wait_chunks(p, it, tag, lane, s_abort)) ok = false;
      if (ok && lane == 0) {
        for (int j = 0; j < it.n_tiles; ++j, ++n) {
          const int st = n & 1;
          const bool pos = (j < it.n_win) || it.dense;
          const int row = (j < it.n_win) ? it.win0 + j * BN : it.dil0 + (j - it.n_win) * BN;
          if (n >= 2 && !mbar_wait(b_kempty + 8 * st, ((n - 2) >> 1) & 1, s_abort)) { ok = false; break; }
          if (!(blockIdx.x == 0 && (long long)n == g_fault_attn_ktile)) {   // else: planted failure
            const CUtensorMap* m = pos ? &tm_kpos : &tm_dil.k[it.cls];
            const uint32_t fb = b_kfull + 8 * st;
            mbar_arrive_expect_tx(fb, kKTile);
            tma_load_4d(sK + st * kKTile, m, fb, 0, it.h, row, it.b);
            tma_load_4d(sK + st * kKTile + kKHalf, m, fb, 64, it.h, row, it.b);
            last_k[st] = n;
          }
          if (j == 0) {
            if (li > 0 && !mbar_wait(b_qempty, (li - 1) & 1, s_abort)) { ok = false; break; }
            mbar_arrive_expect_tx(b_qfull, kQTile);
            tma_load_4d(sQ, &tm_q, b_qfull, 0, it.h, it.t0, it.b);
            tma_load_4d(sQ + kQHalf, &tm_q, b_qfull, 64, it.h, it.t0, it.b);
            ++nq;
          }
          if (n >= 2 && !mbar_wait(b_pvdone + 8 * st, ((n - 2) >> 1) & 1, s_abort)) { ok = false; break; }
          const CUtensorMap* m = pos ? &tm_vpos : &tm_dil.v[it.cls];
          const uint32_t fb = b_vfull + 8 * st;
          mbar_arrive_expect_tx(fb, kKTile);
          tma_load_4d(sV + st * kKTile, m, fb, 0, it.h, row, it.b);
          tma_load_4d(sV + st * kKTile + kKHalf, m, fb, 64, it.h, row, it.b);
          last_v[st] = n;
        }
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
    }
    // let the copies in flight land before the CTA ends (after an abort
    // they may never have been consumed)
    if (lane == 0) {
      if (nq > 0) mbar_drain(b_qfull, (nq - 1) & 1);
      for (int st = 0; st < 2; ++st) {
        if (last_k[st] >= 0) mbar_drain(b_kfull + 8 * st, (last_k[st] >> 1) & 1);
        if (last_v[st] >= 0) mbar_drain(b_vfull + 8 * st, (last_v[st] >> 1) & 1);
      }
    }
    __syncwarp();
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16_f32(BM, BN, 0, 0);    // Q K^T: both K-major
      constexpr uint32_t idPV = idesc_bf16_f32(BM, DH, 0, 1);   // P V: P K-major (TMEM), V MN-major
      const uint64_t dq = sw128_desc(sQ, 16, 1024);
      const uint64_t dk0 = sw128_desc(sK, 16, 1024);
      const uint64_t dv0 = sw128_desc(sV, kKHalf, 1024);
      constexpr uint64_t kStageDesc = kKTile >> 4;      // descriptor step between stages
      const uint32_t tS = tmem + kColS, tP = tmem + kColP, tO = tmem + kColO;
      int n = 0;
      bool ok = true;
      // S = Q K^T of tile n (its S columns were read by the softmax of n-1)
      auto issue_s = [&](int nn) -> bool {
        const int st = nn & 1;
        if (nn > 0 && !mbar_wait(b_sfree, (nn - 1) & 1, s_abort)) return false;
        if (!mbar_wait(b_kfull + 8 * st, (nn >> 1) & 1, s_abort)) return false;
        tc_fence_after();
        const uint64_t dk = dk0 + st * kStageDesc;
#pragma unroll
        for (int k = 0; k < DH / 16; ++k) {
          const uint64_t oa = (uint64_t)(((k >> 2) * kQHalf + (k & 3) * 32) >> 4);
          const uint64_t ob = (uint64_t)(((k >> 2) * kKHalf + (k & 3) * 32) >> 4);
          umma_f16(tS, dq + oa, dk + ob, idS, k > 0 ? 1u : 0u);
        }
        umma_commit(b_sfull);
        umma_commit(b_kempty + 8 * st);
        return true;
      };
      // O += P V of tile nn (first = the item's first tile: O is overwritten)
      auto issue_pv = [&](int nn, bool first) -> bool {
        const int st = nn & 1;
        if (!mbar_wait(b_pfull + 8 * st, (nn >> 1) & 1, s_abort)) return false;
        if (!mbar_wait(b_vfull + 8 * st, (nn >> 1) & 1, s_abort)) return false;
        tc_fence_after();
        const uint64_t dv = dv0 + st * kStageDesc;
        const uint32_t aP = tP + st * (BN / 2);
        umma_f16_ts(tO, aP, dv, idPV, first ? 0u : 1u);
#pragma unroll
        for (int k = 1; k < BN / 16; ++k)
          umma_f16_ts(tO, aP + k * 8, dv + (uint64_t)((k * 16 * 128) >> 4), idPV, 1u);
        umma_commit(b_pvdone + 8 * st);
        return true;
      };
      for (int li = 0; ok; ++li) {
        const int idx = item_at(li);
        if (idx < 0) { ok = false; break; }
        if (idx >= p.n_items) break;
        const int n_tiles = make_item<FUSED, DYN>(p, idx).n_tiles;
        if (!mbar_wait(b_qfull, li & 1, s_abort)) { ok = false; break; }
        if (!issue_s(n)) { ok = false; break; }
        for (int j = 1; j < n_tiles; ++j) {
          if (!issue_s(n + j) || !issue_pv(n + j - 1, j == 1)) { ok = false; break; }
        }
        if (!ok) break;
        umma_commit(b_qempty);                       // all of this item's S = Q K^T issued
        if (!issue_pv(n + n_tiles - 1, n_tiles == 1)) { ok = false; break; }
        n += n_tiles;
      }
      // every MMA issued has completed before TMEM is released
      umma_commit(b_final);
      mbar_drain(b_final, 0);
    }
    __syncwarp();
  } else if (warp < kSoftmaxWarps) {
    // ------------------------------------------------------------ softmax
    const int r = warp * 32 + lane;                  // query row within the tile (TMEM lane)
    const uint32_t tl = tmem + ((uint32_t)(warp * 32) << 16);
    const uint32_t colS = tl + kColS, colP = tl + kColP, colO = tl + kColO;
    const float sc = p.scale_log2;
    // After a failed (timed-out or aborted) wait the warp leaves the loop;
    // every wait is warp-uniform, so warp-collective tcgen05 instructions are
    // always executed by the whole warp.
    int n = 0;                                       // tiles so far
    bool ok = true;
    for (int li = 0; ok; ++li) {
      const int idx = item_at(li);
      if (!warp_all(idx >= 0)) { ok = false; break; }
      if (idx >= p.n_items) break;
      const Item it = make_item<FUSED, DYN>(p, idx);
      const int t = it.t0 + r;
      const int lim_dil = it.dense ? (t + 1) : (max(0, t - p.W_eff + 1) / it.Dd);
      const int w_lo = max(t - p.W_eff + 1, 0);
      float m_used = -1e30f, l = 0.f;
      for (int j = 0; j < it.n_tiles; ++j, ++n) {
        const int pb = n & 1;
        if (!warp_all(mbar_wait(b_sfull, n & 1, s_abort))) { ok = false; break; }
        tc_fence_after();
        uint32_t sr[BN];
        tmem_ld32(colS, sr);
        tmem_ld32(colS + 32, sr + 32);
        tmem_wait_ld();
        tc_fence_before();
        mbar_arrive(b_sfree);                        // S may be overwritten now

        // valid columns [lo, hi) of this row in this tile, as 32-bit chunk masks
        int lo, hi;
        if (j < it.n_win) {
          const int base = it.win0 + j * BN;
          lo = w_lo - base;
          hi = t - base + 1;
        } else {
          const int base = it.dil0 + (j - it.n_win) * BN;   // < 0: leading zero-filled slots
          lo = -base;
          hi = lim_dil - base;
        }
        uint32_t vm[2];
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          const int clo = min(max(lo - 32 * c, 0), 32);
          const int chi = min(max(hi - 32 * c, 0), 32);
          vm[c] = (chi >= 32 ? 0xffffffffu : ((1u << chi) - 1u)) & ~(clo >= 32 ? 0xffffffffu : ((1u << clo) - 1u));
        }
        // mask in place (invalid -> -inf), then the row max of raw scores
        float mx = -INFINITY;
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          if (!__all_sync(0xffffffffu, vm[c] == 0xffffffffu)) {
#pragma unroll
            for (int i = 0; i < 32; ++i)
              sr[32 * c + i] = ((vm[c] >> i) & 1u) ? sr[32 * c + i] : 0xff800000u;
          }
          float m3[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
          for (int i = 0; i < 32; i += 8) {
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const float a = __uint_as_float(sr[32 * c + i + 2 * u]);
              const float b = __uint_as_float(sr[32 * c + i + 2 * u + 1]);
              asm("max.f32 %0, %1, %2, %3;" : "=f"(m3[u]) : "f"(m3[u]), "f"(a), "f"(b));
            }
          }
          float m01, m23;
          asm("max.f32 %0, %1, %2, %3;" : "=f"(m01) : "f"(mx), "f"(m3[0]), "f"(m3[1]));
          asm("max.f32 %0, %1, %2, %3;" : "=f"(m23) : "f"(m01), "f"(m3[2]), "f"(m3[3]));
          mx = m23;
        }
        const float mxs = mx * sc;                   // -inf stays -inf
        // O is rescaled only when some row's running max grew by more than
        // 2^kRescaleThreshold; tcgen05.ld/st are warp-collective, so the
        // decision is per warp and rows that do not need it scale by 1.
        const bool need = (j > 0) && (mxs > m_used + kRescaleThreshold);
        if (j == 0) m_used = fmaxf(mxs, -1e30f);
        const bool rescale = __any_sync(0xffffffffu, need);
        const float alpha = need ? exp2f(m_used - mxs) : 1.f;
        if (need) {
          l *= alpha;
          m_used = mxs;
        }
        // p = 2^(s*scale - m) as bf16 pairs
        const float2 sc2 = make_float2(sc, sc);
        const float2 nm2 = make_float2(-m_used, -m_used);
        float2 ls[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
        uint32_t w[BN / 2];
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          if (__all_sync(0xffffffffu, vm[c] == 0u)) {
#pragma unroll
            for (int i = 0; i < 16; ++i) w[16 * c + i] = 0u;
          } else {
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const float2 x = fma2(make_float2(__uint_as_float(sr[32 * c + 2 * i]),
                                                __uint_as_float(sr[32 * c + 2 * i + 1])), sc2, nm2);
              const float2 e = make_float2(exp2f(x.x), exp2f(x.y));
              ls[i & 1] = add2(ls[i & 1], e);
              w[16 * c + i] = pack_bf16x2(e.x, e.y);
            }
          }
        }
        l += (ls[0].x + ls[0].y) + (ls[1].x + ls[1].y);
        // P buffer pb was last read by O += P V of tile n-2
        if (n >= 2 && !warp_all(mbar_wait(b_pvdone + 8 * pb, ((n - 2) >> 1) & 1, s_abort))) { ok = false; break; }
        tc_fence_after();
        tmem_st32(colP + pb * (BN / 2), w);
        if (rescale) {
          // O must hold P V of tile n-1 before it is scaled
          if (!warp_all(mbar_wait(b_pvdone + 8 * (pb ^ 1), ((n - 1) >> 1) & 1, s_abort))) { ok = false; break; }
          tc_fence_after();
#pragma unroll kColdUnroll
          for (int c = 0; c < 4; ++c) {
            uint32_t o32[32];
            tmem_ld32(colO + 32 * c, o32);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) o32[i] = __float_as_uint(__uint_as_float(o32[i]) * alpha);
            tmem_st32(colO + 32 * c, o32);
          }
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(b_pfull + 8 * pb);
      }
      if (!ok) break;
      // epilogue: wait for the item's last P V, normalise, store
      const int nl = n - 1;
      if (!warp_all(mbar_wait(b_pvdone + 8 * (nl & 1), (nl >> 1) & 1, s_abort))) { ok = false; break; }
      tc_fence_after();
      const float inv = 1.f / l;
      __nv_bfloat16* orow = p.o + (((size_t)it.b * p.T + t) * p.H + it.h) * DH;
#pragma unroll kColdUnroll
      for (int c = 0; c < 4; ++c) {
        uint32_t o32[32];
        tmem_ld32(colO + 32 * c, o32);
        tmem_wait_ld();
        if (t < p.T) {
#pragma unroll
          for (int v = 0; v < 2; ++v) {
            uint32_t q[8];
#pragma unroll
            for (int i = 0; i < 8; ++i)
              q[i] = pack_bf16x2(__uint_as_float(o32[16 * v + 2 * i]) * inv, __uint_as_float(o32[16 * v + 2 * i + 1]) * inv);
            if (!RATP_IN((orow - p.o) + 32 * c + 16 * v, 16, (long long)p.B * p.T * p.H * DH)) continue;
            if (p.o_align32) {                       // one 32-byte store per 16 values
              asm volatile("st.global.v8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};"
                           :: "l"(orow + 32 * c + 16 * v), "r"(q[0]), "r"(q[1]), "r"(q[2]), "r"(q[3]),
                              "r"(q[4]), "r"(q[5]), "r"(q[6]), "r"(q[7]) : "memory");
            } else {                                 // output only 16-byte aligned
              *reinterpret_cast<uint4*>(orow + 32 * c + 16 * v) = make_uint4(q[0], q[1], q[2], q[3]);
              *reinterpret_cast<uint4*>(orow + 32 * c + 16 * v + 8) = make_uint4(q[4], q[5], q[6], q[7]);
            }
          }
        }
      }
      tc_fence_before();
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace attn_tc
}  // namespace ratp
