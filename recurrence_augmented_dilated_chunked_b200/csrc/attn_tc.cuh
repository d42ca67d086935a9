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
//     W' = max(W, 1), so W = 0 still supplies the self key t; window keys that
//     are also dilated keys (j mod D = D-1, j < t) are masked out.
// Per-row validity is a prefix (dilated: s < floor(t / D_h), dense: s <= t) or
// a range minus a periodic pattern (window), evaluated in registers.
//
// Roles (192 threads, one CTA per SM, persistent over items in heavy-first
// order -- dense heads and late query tiles first, round-robin over CTAs):
//   warps 0-3  softmax: thread r owns query row r = TMEM lane r.  Reads S from
//              TMEM, masks, keeps the running max (rescaling O in TMEM only
//              when the max grows by more than 2^8), writes P (bf16) into a
//              128B-swizzled K-major smem tile, and finally normalises O.
//   warp 4     TMA producer: Q (double-buffered) and a 2-stage K/V ring.
//   warp 5     allocates TMEM (512 columns: S ping-pong 2x128, O 128) and one
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
constexpr int kThreads = 192;
constexpr uint32_t kHalf = BN * 64 * 2;        // one 64-column half tile: 16 KB
constexpr uint32_t kTile = 2 * kHalf;          // 128 x 128 bf16: 32 KB
constexpr uint32_t kOffQ = 0;                  // 2 Q buffers
constexpr uint32_t kOffK = kOffQ + 2 * kTile;
constexpr uint32_t kOffV = kOffK + NST * kTile;
constexpr uint32_t kOffP = kOffV + NST * kTile;
constexpr uint32_t kOffBar = kOffP + kTile;
constexpr uint32_t kNumBars = 14;
constexpr uint32_t kSmemBytes = kOffBar + kNumBars * 8 + 16 + 1024;   // + alignment slack
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0;      // S buffers at columns 0 and 128
constexpr uint32_t kColO = 256;    // O at columns 256..383
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
    const int n_dil = it.t_last / p.D;
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
  const uint32_t b_qfull = bar0 + 0 * 8;    // [2]
  const uint32_t b_qempty = bar0 + 2 * 8;   // [2]
  const uint32_t b_kvfull = bar0 + 4 * 8;   // [NST]
  const uint32_t b_kvempty = bar0 + 6 * 8;  // [NST]
  const uint32_t b_sfull = bar0 + 8 * 8;    // [2]
  const uint32_t b_sfree = bar0 + 10 * 8;   // [2]
  const uint32_t b_pfull = bar0 + 12 * 8;
  const uint32_t b_pvdone = bar0 + 13 * 8;
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + kOffBar + kNumBars * 8);
  volatile int* s_abort = reinterpret_cast<volatile int*>(smem + kOffBar + kNumBars * 8 + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(b_qfull + 8 * i, 1);
      mbar_init(b_qempty + 8 * i, 1);
      mbar_init(b_sfull + 8 * i, 1);
      mbar_init(b_sfree + 8 * i, 128);
    }
    for (int i = 0; i < NST; ++i) {
      mbar_init(b_kvfull + 8 * i, 1);
      mbar_init(b_kvempty + 8 * i, 1);
    }
    mbar_init(b_pfull, 128);
    mbar_init(b_pvdone, 1);
    *s_abort = 0;
    fence_barrier_init();
  }
  if (warp == 5) {
    tmem_alloc(smem_u32(s_tmem), kTmemCols);
    tmem_relinquish();
  }
  if (warp == 4 && lane == 0) {
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

  if (warp == 4) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int g = 0, li = 0;
      for (int idx = blockIdx.x; idx < p.n_items; idx += gridDim.x, ++li) {
        const Item it = make_item(p, idx);
        const int qb = li & 1;
        if (li >= 2 && !mbar_wait(b_qempty + 8 * qb, ((li >> 1) - 1) & 1, s_abort)) break;
        mbar_arrive_expect_tx(b_qfull + 8 * qb, kTile);
        tma_load_4d(sQ + qb * kTile, &tm_q, b_qfull + 8 * qb, 0, it.h, it.t0, it.b);
        tma_load_4d(sQ + qb * kTile + kHalf, &tm_q, b_qfull + 8 * qb, 64, it.h, it.t0, it.b);
        bool ok = true;
        for (int j = 0; j < it.n_tiles; ++j, ++g) {
          const int st = g % NST;
          if (g >= NST && !mbar_wait(b_kvempty + 8 * st, ((g / NST) - 1) & 1, s_abort)) {
            ok = false;
            break;
          }
          const CUtensorMap* mk;
          const CUtensorMap* mv;
          int row;
          if (j < it.n_win) {
            mk = &tm_kpos; mv = &tm_vpos;
            row = it.p_start + j * BN;
          } else {
            row = (j - it.n_win) * BN;
            if (it.dense) { mk = &tm_kpos; mv = &tm_vpos; }
            else { mk = &tm_kdil; mv = &tm_vdil; }
          }
          const uint32_t fb = b_kvfull + 8 * st;
          mbar_arrive_expect_tx(fb, 2 * kTile);
          tma_load_4d(sK + st * kTile, mk, fb, 0, it.h, row, it.b);
          tma_load_4d(sK + st * kTile + kHalf, mk, fb, 64, it.h, row, it.b);
          tma_load_4d(sV + st * kTile, mv, fb, 0, it.h, row, it.b);
          tma_load_4d(sV + st * kTile + kHalf, mv, fb, 64, it.h, row, it.b);
        }
        if (!ok) break;
      }
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16_f32(BM, BN, 0, 0);    // Q K^T: both K-major
      constexpr uint32_t idPV = idesc_bf16_f32(BM, DH, 0, 1);   // P V: V is MN-major
      int g = 0, li = 0;
      bool pend = false;
      int pg = 0, pst = 0, pacc = 0;
      bool ok = true;
      auto issue_pv = [&](int gg, int stg, int acc) -> bool {
        if (!mbar_wait(b_pfull, gg & 1, s_abort)) return false;
        tc_fence_after();
#pragma unroll
        for (int k = 0; k < BN / 16; ++k) {
          const uint64_t a = sw128_desc(sP + (k >> 2) * kHalf + (k & 3) * 32, 16, 1024);
          const uint64_t bdesc = sw128_desc(sV + stg * kTile + k * 16 * 128, kHalf, 1024);
          umma_f16(tmem + kColO, a, bdesc, idPV, (acc || k > 0) ? 1u : 0u);
        }
        umma_commit(b_kvempty + 8 * stg);
        umma_commit(b_pvdone);
        return true;
      };
      for (int idx = blockIdx.x; ok && idx < p.n_items; idx += gridDim.x, ++li) {
        const Item it = make_item(p, idx);
        const int qb = li & 1;
        if (!mbar_wait(b_qfull + 8 * qb, (li >> 1) & 1, s_abort)) { ok = false; break; }
        for (int j = 0; j < it.n_tiles; ++j, ++g) {
          const int st = g % NST;
          const int sbuf = g & 1;
          if (!mbar_wait(b_kvfull + 8 * st, (g / NST) & 1, s_abort)) { ok = false; break; }
          if (g >= 2 && !mbar_wait(b_sfree + 8 * sbuf, ((g >> 1) - 1) & 1, s_abort)) { ok = false; break; }
          tc_fence_after();
#pragma unroll
          for (int k = 0; k < DH / 16; ++k) {
            const uint32_t koff = (k >> 2) * kHalf + (k & 3) * 32;
            const uint64_t a = sw128_desc(sQ + qb * kTile + koff, 16, 1024);
            const uint64_t bdesc = sw128_desc(sK + st * kTile + koff, 16, 1024);
            umma_f16(tmem + kColS + sbuf * BN, a, bdesc, idS, k > 0 ? 1u : 0u);
          }
          umma_commit(b_sfull + 8 * sbuf);
          if (j == it.n_tiles - 1) umma_commit(b_qempty + 8 * qb);
          if (pend && !issue_pv(pg, pst, pacc)) { ok = false; break; }
          pend = true;
          pg = g; pst = st; pacc = (j > 0);
        }
      }
      if (ok && pend) issue_pv(pg, pst, pacc);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax
    const int r = threadIdx.x;                       // query row within the tile
    const uint32_t tl = tmem + ((uint32_t)(warp * 32) << 16);
    int g = 0;
    bool ok = true;
    for (int idx = blockIdx.x; ok && idx < p.n_items; idx += gridDim.x) {
      const Item it = make_item(p, idx);
      const int t = it.t0 + r;
      const bool row_ok = t < p.T;
      const int lim_dil = it.dense ? (t + 1) : (t / it.Dd);
      const int w_lo = max(t - p.W_eff + 1, 0);
      float m_used = -1e30f, l = 0.f;
      for (int j = 0; j < it.n_tiles; ++j, ++g) {
        const int sbuf = g & 1;
        if (!warp_all(mbar_wait(b_sfull + 8 * sbuf, (g >> 1) & 1, s_abort))) { ok = false; break; }
        tc_fence_after();
        uint32_t sr[BN];
#pragma unroll
        for (int c = 0; c < BN / 32; ++c) tmem_ld32(tl + kColS + sbuf * BN + c * 32, sr + c * 32);
        tmem_wait_ld();
        tc_fence_before();
        mbar_arrive(b_sfree + 8 * sbuf);

        float x[BN];
        float mx = -INFINITY;
        if (j < it.n_win) {
          const int p0 = it.p_start + j * BN;
          int rm = p0 % it.Dd;
#pragma unroll
          for (int c = 0; c < BN; ++c) {
            const int pos = p0 + c;
            const bool dup = (rm == it.Dd - 1) && (pos < t);
            const bool ok_c = (pos >= w_lo) && (pos <= t) && !dup;
            x[c] = ok_c ? __uint_as_float(sr[c]) * p.scale_log2 : -INFINITY;
            mx = fmaxf(mx, x[c]);
            rm = (rm + 1 == it.Dd) ? 0 : rm + 1;
          }
        } else {
          const int lim = lim_dil - (j - it.n_win) * BN;
#pragma unroll
          for (int c = 0; c < BN; ++c) {
            x[c] = (c < lim) ? __uint_as_float(sr[c]) * p.scale_log2 : -INFINITY;
            mx = fmaxf(mx, x[c]);
          }
        }
        // previous P.V must be complete before P is overwritten / O rescaled
        if (g > 0 && !warp_all(mbar_wait(b_pvdone, (g - 1) & 1, s_abort))) { ok = false; break; }
        tc_fence_after();
        // O is rescaled only when some row's running max grew by more than
        // 2^kRescaleThreshold.  tcgen05.ld/st are warp-collective, so the
        // decision is taken per warp and rows that do not need it use alpha 1.
        const bool need = (j > 0) && (mx > m_used + kRescaleThreshold);
        if (j == 0) m_used = fmaxf(mx, -1e30f);
        if (__any_sync(0xffffffffu, need)) {
          const float alpha = need ? exp2f(m_used - mx) : 1.f;
#pragma unroll
          for (int c = 0; c < DH / 32; ++c) {
            uint32_t o32[32];
            tmem_ld32(tl + kColO + c * 32, o32);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) o32[i] = __float_as_uint(__uint_as_float(o32[i]) * alpha);
            tmem_st32(tl + kColO + c * 32, o32);
          }
          tmem_wait_st();
          if (need) {
            l *= alpha;
            m_used = mx;
          }
        }
        float rowsum = 0.f;
#pragma unroll
        for (int cc = 0; cc < BN / 8; ++cc) {
          uint32_t w[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float e0 = exp2f(x[cc * 8 + 2 * i] - m_used);
            const float e1 = exp2f(x[cc * 8 + 2 * i + 1] - m_used);
            w[i] = pack_bf16x2(e0, e1);
            rowsum += __uint_as_float(w[i] << 16) + __uint_as_float(w[i] & 0xffff0000u);
          }
          const uint32_t addr = sP + (cc >> 3) * kHalf + r * 128 + ((((uint32_t)cc & 7u) ^ ((uint32_t)r & 7u)) << 4);
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};"
                       :: "r"(addr), "r"(w[0]), "r"(w[1]), "r"(w[2]), "r"(w[3]) : "memory");
        }
        l += rowsum;
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(b_pfull);
      }
      if (!ok) break;
      // ---- epilogue: O / l -> bf16 -> global
      if (!warp_all(mbar_wait(b_pvdone, (g - 1) & 1, s_abort))) { ok = false; break; }
      tc_fence_after();
      const float inv = 1.f / l;
      __nv_bfloat16* orow = p.o + (((size_t)it.b * p.T + t) * p.H + it.h) * DH;
#pragma unroll
      for (int c = 0; c < DH / 32; ++c) {
        uint32_t o32[32];
        tmem_ld32(tl + kColO + c * 32, o32);
        tmem_wait_ld();
        if (row_ok) {
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
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace attn_tc
}  // namespace ratp
