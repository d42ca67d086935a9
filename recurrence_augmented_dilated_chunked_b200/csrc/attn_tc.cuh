// attn_tc.cuh -- dilated (+ windowed) prefill attention on the 5th-generation
// tensor cores (TMA + tcgen05.mma, accumulators in tensor memory).
//
// Computes, for every (b, h, t), softmax attention of q[b,t,h] over the
// recurrent keys/values at K_h(t) = {j < t : j mod D_h = D_h-1} U {t}
// U {t-W < j <= t} (RAT+ abstract: dilated attention with optional local
// windows; write-up section 6: dense heads D_h = 1).  bf16 in, fp32
// accumulate, head dim 128.
//
// Work item = (b, h, 128-query tile).  Its keys come in 128-key tiles of two
// kinds, both fetched by plain tiled TMA boxes:
//   * dilated tiles: slots s..s+127 of the strided view of hk/hv whose row s
//     is position s*D + D - 1 (base offset D-1 rows, row stride D rows), so the
//     gather is an ordinary box of the strided tensor map; a dense head reads
//     the positional view instead (slot = position);
//   * window tiles (dilated heads only): positions of [t0 - W' + 1, t_last],
//     W' = max(W, 1), so W = 0 still supplies the self key t.
// Each key is counted once by splitting the set at the window: row t takes
// every window position t-W'+1..t and only the dilated slots whose position
// lies before the window, s < floor((t - W' + 1) / D).  So per-row validity is
// a prefix (dilated; dense: s <= t) or a contiguous range (window), evaluated
// as bit masks per 32-column chunk.
//
// Roles (352 threads, one CTA per SM, persistent over items in heavy-first
// order -- dense heads and late query tiles first, round-robin over CTAs):
//   warps 0-7  softmax: warps w and w+4 share query rows 32(w%4)..+31 (TMEM
//              lanes) and split the 128 key columns in halves.  Each reads its
//              half of S from TMEM, masks it per 32-column chunk with a bit
//              mask (all-valid and all-masked chunks take fast paths), the
//              pair exchanges the row max through shared memory, the running
//              max is kept with O rescaled in TMEM only when it grows by more
//              than 2^8, and P (bf16) is written into one of two 128B-swizzled
//              K-major smem tiles.  An item's epilogue (normalise half an O
//              row, store) runs after the softmax of the next item's first
//              tile, so waiting for its last P V overlaps useful work.
//   warp 8     TMA producer of Q and of a 2-stage K ring (a K stage is freed
//              as soon as its S = Q K^T completes);
//   warp 10    TMA producer of a 2-stage V ring (freed when P V completes);
//   warp 9     allocates TMEM (512 columns: S ping-pong 2x128, O ping-pong
//              2x128, one O per work item in flight) and one
//              lane issues S = Q K^T (SS, K-major) and O += P V (P K-major,
//              V MN-major) as 128x128x16 tcgen05.mma; completions signal
//              mbarriers via tcgen05.commit.
// Every mbarrier wait is bounded; on expiry the CTA records RATP_ERR_TIMEOUT,
// all roles drain out, and TMEM is released.
#pragma once
#include "sm100.cuh"

namespace ratp {
namespace attn_tc {

constexpr int BM = 128;          // queries per tile
constexpr int BN = 128;          // keys per tile
constexpr int DH = 128;          // head dim
constexpr int NST = 2;           // K/V pipeline stages
constexpr int kSoftmaxWarps = 8;
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;
constexpr int kVProducerWarp = 10;
constexpr int kThreads = 352;
constexpr uint32_t kHalf = BN * 64 * 2;        // one 64-column half tile: 16 KB
constexpr uint32_t kTile = 2 * kHalf;          // 128 x 128 bf16: 32 KB
constexpr uint32_t kOffQ = 0;                  // Q
constexpr uint32_t kOffK = kOffQ + kTile;
constexpr uint32_t kOffV = kOffK + NST * kTile;
constexpr uint32_t kOffP = kOffV + NST * kTile;  // 2 P buffers
constexpr uint32_t kOffBar = kOffP + 2 * kTile;
constexpr uint32_t kNumBars = 18;
constexpr uint32_t kOffXchg = kOffBar + kNumBars * 8 + 16;     // row-max / row-sum exchange
constexpr uint32_t kXchgBytes = 2 * BM * 4;                    // [2 halves][128] f32
constexpr uint32_t kSmemBytes = kOffXchg + kXchgBytes + 1024;  // + alignment slack
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0;      // S buffers at columns 0 and 128
constexpr uint32_t kColO = 256;    // O double buffer at columns 256..383 and 384..511
constexpr float kRescaleThreshold = 8.0f;   // log2 units

struct Params {
  __nv_bfloat16* o;
  int B, T, H, D, W_eff, NQ;
  int n_dense, n_dil;
  int n_items_dense, n_items;
  float scale_log2;
  uint8_t dense_list[RATP_MAX_HEADS];
  uint8_t dil_list[RATP_MAX_HEADS];
};

struct Item {
  int b, h, t0, t_last, Dd, n_win, n_tiles, p_start;
  bool dense;
};

__device__ __forceinline__ Item make_item(const Params& p, int idx) {
  Item it;
  int per, qi, rem;
  if (idx < p.n_items_dense) {
    per = p.B * p.n_dense;
    qi = idx / per;
    rem = idx - qi * per;
    it.b = rem / p.n_dense;
    it.h = p.dense_list[rem - it.b * p.n_dense];
    it.dense = true;
  } else {
    idx -= p.n_items_dense;
    per = p.B * p.n_dil;
    qi = idx / per;
    rem = idx - qi * per;
    it.b = rem / p.n_dil;
    it.h = p.dil_list[rem - it.b * p.n_dil];
    it.dense = false;
  }
  it.t0 = (p.NQ - 1 - qi) * BM;
  it.t_last = min(it.t0 + BM - 1, p.T - 1);
  if (it.dense) {
    it.Dd = 1;
    it.n_win = 0;
    it.p_start = 0;
    it.n_tiles = (it.t_last + 1 + BN - 1) / BN;
  } else {
    it.Dd = p.D;
    const int n_dil = max(0, it.t_last - p.W_eff + 1) / p.D;   // slots before the last row's window
    it.p_start = max(0, it.t0 - p.W_eff + 1);
    it.n_win = (it.t_last - it.p_start + 1 + BN - 1) / BN;
    it.n_tiles = it.n_win + (n_dil + BN - 1) / BN;
  }
  return it;
}

__global__ void __launch_bounds__(kThreads, 1)
attn_kernel(const __grid_constant__ CUtensorMap tm_q,
            const __grid_constant__ CUtensorMap tm_kpos,
            const __grid_constant__ CUtensorMap tm_vpos,
            const __grid_constant__ CUtensorMap tm_kdil,
            const __grid_constant__ CUtensorMap tm_vdil,
            const __grid_constant__ Params p) {
  using namespace sm100;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_u32(smem);
  const uint32_t sQ = sb + kOffQ, sK = sb + kOffK, sV = sb + kOffV, sP = sb + kOffP;
  const uint32_t bar0 = sb + kOffBar;
  // barrier map
  const uint32_t b_qfull = bar0 + 0 * 8;
  const uint32_t b_qempty = bar0 + 1 * 8;
  const uint32_t b_kfull = bar0 + 2 * 8;    // [NST]
  const uint32_t b_kempty = bar0 + 4 * 8;   // [NST]
  const uint32_t b_sfull = bar0 + 6 * 8;    // [2]
  const uint32_t b_sfree = bar0 + 8 * 8;    // [2]
  const uint32_t b_pfull = bar0 + 10 * 8;   // [2]
  const uint32_t b_pvdone = bar0 + 12 * 8;  // [2]
  const uint32_t b_vfull = bar0 + 14 * 8;   // [NST]
  const uint32_t b_vempty = bar0 + 16 * 8;  // [NST]
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + kOffBar + kNumBars * 8);
  volatile int* s_abort = reinterpret_cast<volatile int*>(smem + kOffBar + kNumBars * 8 + 4);
  float* s_xchg = reinterpret_cast<float*>(smem + kOffXchg);     // [2 halves][128 rows]

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(b_qfull, 1);
    mbar_init(b_qempty, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(b_sfull + 8 * i, 1);
      mbar_init(b_sfree + 8 * i, kSoftmaxWarps * 32);
      mbar_init(b_pfull + 8 * i, kSoftmaxWarps * 32);
      mbar_init(b_pvdone + 8 * i, 1);
    }
    for (int i = 0; i < NST; ++i) {
      mbar_init(b_kfull + 8 * i, 1);
      mbar_init(b_kempty + 8 * i, 1);
      mbar_init(b_vfull + 8 * i, 1);
      mbar_init(b_vempty + 8 * i, 1);
    }
    *s_abort = 0;
    fence_barrier_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(smem_u32(s_tmem), kTmemCols);
    tmem_relinquish();
  }
  if (warp == kProducerWarp && lane == 0) {
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_kpos);
    prefetch_tmap(&tm_vpos);
    prefetch_tmap(&tm_kdil);
    prefetch_tmap(&tm_vdil);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s_tmem;

  if (warp == kProducerWarp || warp == kVProducerWarp) {
    // ------------------------------------------------------------ producers
    // warp kProducerWarp: Q and K tiles; warp kVProducerWarp: V tiles.  Both
    // walk the same item/tile sequence.
    const bool is_k = (warp == kProducerWarp);
    if (lane == 0) {
      const uint32_t ring = is_k ? sK : sV;
      const uint32_t b_full = is_k ? b_kfull : b_vfull;
      const uint32_t b_empty = is_k ? b_kempty : b_vempty;
      int g = 0, li = 0;
      bool ok = true;
      for (int idx = blockIdx.x; ok && idx < p.n_items; idx += gridDim.x, ++li) {
        const Item it = make_item(p, idx);
        if (is_k) {
          if (li >= 1 && !mbar_wait(b_qempty, (li - 1) & 1, s_abort)) break;
          mbar_arrive_expect_tx(b_qfull, kTile);
          tma_load_4d(sQ, &tm_q, b_qfull, 0, it.h, it.t0, it.b);
          tma_load_4d(sQ + kHalf, &tm_q, b_qfull, 64, it.h, it.t0, it.b);
        }
        for (int j = 0; j < it.n_tiles; ++j, ++g) {
          const int st = g % NST;
          if (g >= NST && !mbar_wait(b_empty + 8 * st, ((g / NST) - 1) & 1, s_abort)) {
            ok = false;
            break;
          }
          const CUtensorMap* m;
          int row;
          if (j < it.n_win) {
            m = is_k ? &tm_kpos : &tm_vpos;
            row = it.p_start + j * BN;
          } else {
            row = (j - it.n_win) * BN;
            if (it.dense) m = is_k ? &tm_kpos : &tm_vpos;
            else m = is_k ? &tm_kdil : &tm_vdil;
          }
          if (is_k && blockIdx.x == 0 && (long long)g == g_fault_attn_ktile) continue;   // planted failure
          const uint32_t fb = b_full + 8 * st;
          mbar_arrive_expect_tx(fb, kTile);
          tma_load_4d(ring + st * kTile, m, fb, 0, it.h, row, it.b);
          tma_load_4d(ring + st * kTile + kHalf, m, fb, 64, it.h, row, it.b);
        }
      }
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16_f32(BM, BN, 0, 0);    // Q K^T: both K-major
      constexpr uint32_t idPV = idesc_bf16_f32(BM, DH, 0, 1);   // P V: V is MN-major
      int g = 0, li = 0;
      bool pend = false;
      int pg = 0, pst = 0, pacc = 0, pob = 0;
      bool ok = true;
      auto issue_pv = [&](int gg, int stg, int acc, int ob) -> bool {
        const int pb = gg & 1;
        if (!mbar_wait(b_pfull + 8 * pb, (gg >> 1) & 1, s_abort)) return false;
        if (!mbar_wait(b_vfull + 8 * stg, (gg / NST) & 1, s_abort)) return false;
        tc_fence_after();
#pragma unroll
        for (int k = 0; k < BN / 16; ++k) {
          const uint64_t a = sw128_desc(sP + pb * kTile + (k >> 2) * kHalf + (k & 3) * 32, 16, 1024);
          const uint64_t bdesc = sw128_desc(sV + stg * kTile + k * 16 * 128, kHalf, 1024);
          umma_f16(tmem + kColO + ob * DH, a, bdesc, idPV, (acc || k > 0) ? 1u : 0u);
        }
        umma_commit(b_vempty + 8 * stg);
        umma_commit(b_pvdone + 8 * pb);
        return true;
      };
      for (int idx = blockIdx.x; ok && idx < p.n_items; idx += gridDim.x, ++li) {
        const Item it = make_item(p, idx);
        if (!mbar_wait(b_qfull, li & 1, s_abort)) { ok = false; break; }
        for (int j = 0; j < it.n_tiles; ++j, ++g) {
          const int st = g % NST;
          const int sbuf = g & 1;
          if (!mbar_wait(b_kfull + 8 * st, (g / NST) & 1, s_abort)) { ok = false; break; }
          if (g >= 2 && !mbar_wait(b_sfree + 8 * sbuf, ((g >> 1) - 1) & 1, s_abort)) { ok = false; break; }
          tc_fence_after();
#pragma unroll
          for (int k = 0; k < DH / 16; ++k) {
            const uint32_t koff = (k >> 2) * kHalf + (k & 3) * 32;
            const uint64_t a = sw128_desc(sQ + koff, 16, 1024);
            const uint64_t bdesc = sw128_desc(sK + st * kTile + koff, 16, 1024);
            umma_f16(tmem + kColS + sbuf * BN, a, bdesc, idS, k > 0 ? 1u : 0u);
          }
          umma_commit(b_sfull + 8 * sbuf);
          umma_commit(b_kempty + 8 * st);
          if (j == it.n_tiles - 1) umma_commit(b_qempty);
          if (pend && !issue_pv(pg, pst, pacc, pob)) { ok = false; break; }
          pend = true;
          pg = g; pst = st; pacc = (j > 0); pob = li & 1;
        }
      }
      if (ok && pend) issue_pv(pg, pst, pacc, pob);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax
    const int r = (warp & 3) * 32 + lane;            // query row within the tile (TMEM lane)
    const int half = warp >> 2;                      // key/output column half
    const int c_base = half * 64;
    const uint32_t bar_id = 1 + (warp & 3);          // named barrier of the warp pair
    const uint32_t tl = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    float* x_mine = s_xchg + half * BM + r;
    const float* x_other = s_xchg + (1 - half) * BM + r;
    auto pair_sync = [&]() {
      asm volatile("bar.sync %0, %1;" :: "r"(bar_id), "r"(64) : "memory");
    };
    // The two warps of a pair meet at named barriers, so neither may leave the
    // schedule early: after a failed (timed-out or aborted) wait the warps
    // carry on with whatever tensor memory holds; every later wait fails fast
    // and the error word already records the timeout.
    // deferred epilogue of the previous item (-1: none): its item index, its
    // O buffer, its last tile and this thread's partial row sum
    int pend_idx = -1, pend_ob = 0, pend_gl = 0;
    float pend_l = 0.f;
    auto epilogue = [&](int e_idx, int e_ob, int e_gl, float e_l) {
      const Item e = make_item(p, e_idx);
      const int e_t = e.t0 + r;
      warp_all(mbar_wait(b_pvdone + 8 * (e_gl & 1), (e_gl >> 1) & 1, s_abort));
      tc_fence_after();
      *x_mine = e_l;
      pair_sync();
      const float inv = 1.f / (e_l + *x_other);
      pair_sync();
      __nv_bfloat16* orow = p.o + (((size_t)e.b * p.T + e_t) * p.H + e.h) * DH + c_base;
      const uint32_t ocol = kColO + e_ob * DH + c_base;
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t o32[32];
        tmem_ld32(tl + ocol + c * 32, o32);
        tmem_wait_ld();
        if (e_t < p.T) {
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            uint4 pk;
            pk.x = pack_bf16x2(__uint_as_float(o32[8 * v + 0]) * inv, __uint_as_float(o32[8 * v + 1]) * inv);
            pk.y = pack_bf16x2(__uint_as_float(o32[8 * v + 2]) * inv, __uint_as_float(o32[8 * v + 3]) * inv);
            pk.z = pack_bf16x2(__uint_as_float(o32[8 * v + 4]) * inv, __uint_as_float(o32[8 * v + 5]) * inv);
            pk.w = pack_bf16x2(__uint_as_float(o32[8 * v + 6]) * inv, __uint_as_float(o32[8 * v + 7]) * inv);
            *reinterpret_cast<uint4*>(orow + c * 32 + v * 8) = pk;
          }
        }
      }
      tc_fence_before();
    };
    int g = 0, li = 0;
    for (int idx = blockIdx.x; idx < p.n_items; idx += gridDim.x, ++li) {
      const Item it = make_item(p, idx);
      const int ob = li & 1;
      const uint32_t ocol_item = kColO + ob * DH + c_base;
      const int t = it.t0 + r;
      const int lim_dil = it.dense ? (t + 1) : (max(0, t - p.W_eff + 1) / it.Dd);
      const int w_lo = max(t - p.W_eff + 1, 0);
      float m_used = -1e30f, l = 0.f;
      for (int j = 0; j < it.n_tiles; ++j, ++g) {
        const int sbuf = g & 1;
        warp_all(mbar_wait(b_sfull + 8 * sbuf, (g >> 1) & 1, s_abort));
        tc_fence_after();
        uint32_t sr[64];
        tmem_ld32(tl + kColS + sbuf * BN + c_base, sr);
        tmem_ld32(tl + kColS + sbuf * BN + c_base + 32, sr + 32);
        tmem_wait_ld();
        tc_fence_before();
        mbar_arrive(b_sfree + 8 * sbuf);

        // validity bit masks of the two 32-column chunks of this half
        uint32_t vm[2];
        {
          const int lim_lo = (j < it.n_win) ? (w_lo - (it.p_start + j * BN) - c_base) : 0;
          const int lim_hi = (j < it.n_win) ? (t - (it.p_start + j * BN) - c_base + 1)
                                            : (lim_dil - (j - it.n_win) * BN - c_base);
#pragma unroll
          for (int k = 0; k < 2; ++k) {
            const int lo = min(max(lim_lo - 32 * k, 0), 32);   // first valid column of the chunk
            const int hi = min(max(lim_hi - 32 * k, 0), 32);   // one past the last valid column
            vm[k] = (hi >= 32 ? 0xffffffffu : ((1u << hi) - 1u)) & ~(lo >= 32 ? 0xffffffffu : ((1u << lo) - 1u));
          }
        }
        // masked row max of this half (raw scores)
        // (four independent accumulators per chunk keep the chain short)
        float mx = -INFINITY;
#pragma unroll
        for (int k = 0; k < 2; ++k) {
          float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
          if (vm[k] == 0xffffffffu) {
#pragma unroll
            for (int i = 0; i < 32; ++i) m4[i & 3] = fmaxf(m4[i & 3], __uint_as_float(sr[32 * k + i]));
          } else if (vm[k] != 0u) {
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const float v = __uint_as_float(sr[32 * k + i]);
              m4[i & 3] = fmaxf(m4[i & 3], ((vm[k] >> i) & 1u) ? v : -INFINITY);
            }
          }
          mx = fmaxf(mx, fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3])));
        }
        // combine with the partner half of the row
        *x_mine = mx;
        pair_sync();
        mx = fmaxf(mx, *x_other);
        pair_sync();
        const float mxs = mx * p.scale_log2;               // -inf stays -inf
        // P buffer g&1 was last read by P.V of tile g-2
        if (g >= 2) warp_all(mbar_wait(b_pvdone + 8 * sbuf, ((g >> 1) - 1) & 1, s_abort));
        // O is rescaled only when some row's running max grew by more than
        // 2^kRescaleThreshold; tcgen05.ld/st are warp-collective, so the
        // decision is per warp (both warps of a pair decide alike) and rows
        // that do not need it scale by 1.  P.V of tile g-1 must be complete.
        const bool need = (j > 0) && (mxs > m_used + kRescaleThreshold);
        if (j == 0) m_used = fmaxf(mxs, -1e30f);
        if (__any_sync(0xffffffffu, need)) {
          const int pb1 = (g - 1) & 1;
          warp_all(mbar_wait(b_pvdone + 8 * pb1, ((g - 1) >> 1) & 1, s_abort));
          tc_fence_after();
          const float alpha = need ? exp2f(m_used - mxs) : 1.f;
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            uint32_t o32[32];
            tmem_ld32(tl + ocol_item + c * 32, o32);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) o32[i] = __float_as_uint(__uint_as_float(o32[i]) * alpha);
            tmem_st32(tl + ocol_item + c * 32, o32);
          }
          tmem_wait_st();
          if (need) {
            l *= alpha;
            m_used = mxs;
          }
        }
        // p = 2^(s*scale - m), bf16 into the swizzled P tile (keys c_base..c_base+63)
        const uint32_t prow = sP + sbuf * kTile + half * kHalf + r * 128;
        const float neg_m = -m_used;
        float rs[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int k = 0; k < 2; ++k) {
          uint32_t w[16];
          if (vm[k] == 0u) {
#pragma unroll
            for (int i = 0; i < 16; ++i) w[i] = 0u;
          } else if (vm[k] == 0xffffffffu) {
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const float e0 = exp2f(fmaf(__uint_as_float(sr[32 * k + 2 * i]), p.scale_log2, neg_m));
              const float e1 = exp2f(fmaf(__uint_as_float(sr[32 * k + 2 * i + 1]), p.scale_log2, neg_m));
              rs[i & 3] += e0 + e1;
              w[i] = pack_bf16x2(e0, e1);
            }
          } else {
            // exponentiate every column, then select: no per-element branches
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              float e0 = exp2f(fmaf(__uint_as_float(sr[32 * k + 2 * i]), p.scale_log2, neg_m));
              float e1 = exp2f(fmaf(__uint_as_float(sr[32 * k + 2 * i + 1]), p.scale_log2, neg_m));
              e0 = ((vm[k] >> (2 * i)) & 1u) ? e0 : 0.f;
              e1 = ((vm[k] >> (2 * i + 1)) & 1u) ? e1 : 0.f;
              rs[i & 3] += e0 + e1;
              w[i] = pack_bf16x2(e0, e1);
            }
          }
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            const uint32_t chunk = (uint32_t)(4 * k + v);                 // 16-byte chunk in the half row
            const uint32_t addr = prow + ((chunk ^ ((uint32_t)r & 7u)) << 4);
            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};"
                         :: "r"(addr), "r"(w[4 * v]), "r"(w[4 * v + 1]), "r"(w[4 * v + 2]), "r"(w[4 * v + 3])
                         : "memory");
          }
        }
        l += (rs[0] + rs[1]) + (rs[2] + rs[3]);
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(b_pfull + 8 * sbuf);
        if (j == 0 && pend_idx >= 0) {
          epilogue(pend_idx, pend_ob, pend_gl, pend_l);
          pend_idx = -1;
        }
      }
      pend_idx = idx;
      pend_ob = ob;
      pend_gl = g - 1;
      pend_l = l;
    }
    if (pend_idx >= 0) epilogue(pend_idx, pend_ob, pend_gl, pend_l);
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
