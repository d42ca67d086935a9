// window.cuh -- fixed look-back recurrence over the key and value streams.
//
// h_t = the forget-gate recurrence h = g h + (1 - g) x started from zero at
// position max(0, t - L + 1) and run to t: each token's recurrent state covers
// exactly the L tokens up to itself (zhichai.net "RAT+ 深度拆解", section 2.1:
// the fixed recurrence window L* = 64 of the RAT+ design before the full
// sequence).  One gate tensor serves both streams.
//
// A sliding window of a linear recurrence has no stable O(1) update (dropping
// the oldest token would divide by a product of gates), so the kernel uses a
// block form.  Cut the sequence into blocks of L positions (block k starts at
// c = kL).  For t = c + o:
//   h_t = loc_t + A_t * S(o)
//   loc_t = the recurrence from zero at c, run to t (this block's part),
//   A_t   = g_c * ... * g_t (decay from the block start to t),
//   S(o)  = the previous block's positions c-L+o+1 .. c-1 run from zero to c-1
//           (the part of the window in the previous block).
// S(o) for all o is one backward pass over the previous block:
//   S(L-1) = 0;  S(o-1) = S(o) + P (1 - g_{c-L+o}) x_{c-L+o},  P *= g_{c-L+o}
// with P the product of the gates after that position up to c-1.  Every term
// is a non-negative combination, so there is no cancellation.
//
// Decomposition: a CTA owns 256 tokens x 32 channels of one batch item, for
// both streams.  TMA stages the gate and the two inputs for rows
// [t0 - 64, t0 + 256) (the 64-row halo holds the previous block of the
// chunk's first block; rows before 0 or past T are filled with zeros, which
// contribute nothing).  A thread owns a channel pair (bf16x2 or float2 loads
// from shared memory, packed f32x2 arithmetic, 4- or 8-byte stores) of one
// stream and runs, for blocks blane, blane + 4, ... of the chunk, the
// backward pass of the previous block (S of both channels in registers) and
// the forward pass of its own block.  No CTA depends on another: there is no
// look-back and no workspace.  The one wait (the TMA tiles) is bounded.
// Thread 0 also prefetches into L2 the tiles of the CTA one SM count of
// blocks later, so that the loads of later CTAs mostly hit L2.
#pragma once
#include "common.cuh"
#include "sm100.cuh"

namespace ratp {
namespace window {

constexpr int kThreads = 128;  // 16 channel pairs x 2 streams x 4 block lanes
constexpr int kChunk = 256;    // tokens per CTA
constexpr int kCh = 32;        // channels per CTA
constexpr int kHalo = 64;      // rows staged before the chunk (>= L)
constexpr int kRows = kHalo + kChunk;
constexpr int kBox = 64;       // TMA box rows

template <typename T>
struct Smem {
  static constexpr int kTile = kRows * kCh * (int)sizeof(T);   // one tensor
  static constexpr int kBytes = 3 * kTile + 128;               // g, x_k, x_v + alignment
};

template <typename T>
struct Params {
  T* h[2];                 // h_k, h_v
  int B, Tn, C;            // Tn tokens, C = H * Dh channels per token
  int slabs;               // C / 32
  int n_chunks_t;          // chunks along T
  int l2_ahead;            // L2 prefetch distance in CTAs (0: none)
};

// a channel pair of one staged row, as fp32
__device__ __forceinline__ float2 ld_pair(const float* p) { return *reinterpret_cast<const float2*>(p); }
__device__ __forceinline__ float2 ld_pair(const __nv_bfloat16* p) {
  const uint32_t w = *reinterpret_cast<const uint32_t*>(p);
  return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
}
__device__ __forceinline__ void st_pair(float* p, float2 v) { __stcs(reinterpret_cast<float2*>(p), v); }
__device__ __forceinline__ void st_pair(__nv_bfloat16* p, float2 v) {
  __stcs(reinterpret_cast<unsigned int*>(p), pack_bf16x2(v.x, v.y));
}

// Three CTAs per SM (61.5 KB of tiles each for bf16), 128 threads each: a
// thread keeps the L backward-pass sums of its two channels in registers.
template <typename T, int L>
__global__ void __launch_bounds__(kThreads, 3)
window_kernel(const __grid_constant__ CUtensorMap tm_g, const __grid_constant__ CUtensorMap tm_x0,
              const __grid_constant__ CUtensorMap tm_x1, const __grid_constant__ Params<T> p) {
  static_assert(L >= 1 && L <= kHalo && kChunk % L == 0, "block length");
  using SM = Smem<T>;
  constexpr int NB = kChunk / L;          // blocks per chunk
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
  __shared__ __align__(8) uint64_t s_bar;

  const int tid = threadIdx.x;
  const int chunk = blockIdx.x % p.n_chunks_t;
  const int rest = blockIdx.x / p.n_chunks_t;
  const int slab = rest % p.slabs;
  const int b = rest / p.slabs;
  const int t0 = chunk * kChunk;
  const uint32_t bar = sm100::smem_u32(&s_bar);
  if (tid == 0) {
    sm100::mbar_init(bar, 1);
    sm100::fence_barrier_init();
  }
  __syncthreads();
  if (tid == 0) {
    sm100::mbar_arrive_expect_tx(bar, 3 * SM::kTile);
    const uint32_t dst = sm100::smem_u32(smem);
    const CUtensorMap* maps[3] = {&tm_g, &tm_x0, &tm_x1};
#pragma unroll
    for (int m = 0; m < 3; ++m)
#pragma unroll
      for (int r = 0; r < kRows / kBox; ++r)   // rows t0 - 64 + 64 r (the first box may start before 0)
        sm100::tma_load_3d(dst + m * SM::kTile + r * kBox * kCh * (int)sizeof(T), maps[m], bar,
                           slab * kCh, t0 - kHalo + r * kBox, b);
    // warm L2 with the chunk of the CTA l2_ahead blocks later (its halo is
    // this range's tail, fetched already), so that DRAM keeps streaming
    // while the resident CTAs compute
    const long long nb = (long long)blockIdx.x + p.l2_ahead;
    if (p.l2_ahead > 0 && nb < (long long)p.B * p.slabs * p.n_chunks_t) {
      const int ck = (int)(nb % p.n_chunks_t);
      const long long rs = nb / p.n_chunks_t;
      const int sl = (int)(rs % p.slabs), bb = (int)(rs / p.slabs);
#pragma unroll
      for (int m = 0; m < 3; ++m)
#pragma unroll
        for (int r = 1; r < kRows / kBox; ++r)
          sm100::tma_prefetch_l2_3d(maps[m], sl * kCh, ck * kChunk - kHalo + r * kBox, bb);
    }
  }
  bool ok = true;
  if (tid == 0) {
    unsigned long long tw = 0;
    unsigned int n = 0;
    while (!sm100::mbar_try_wait(bar, 0)) {
      if ((++n & 63u) == 0u) {
        const unsigned long long now = global_ns();
        if (tw == 0) tw = now;
        else if (now - tw > spin_timeout()) { ok = false; break; }
      }
    }
    if (!ok) raise_error(RATP_ERR_TIMEOUT);
  }
  if (!__syncthreads_and(ok)) {
    // the tiles never arrived: let any copy still in flight land before the
    // shared memory is released (bounded), then give up
    if (tid == 0) {
      unsigned long long t1 = global_ns();
      while (!sm100::mbar_try_wait(bar, 0) && global_ns() - t1 < spin_timeout()) {}
    }
    __syncthreads();
    return;
  }

  const T* sg = reinterpret_cast<const T*>(smem);
  const int cp = 2 * (tid & 15);                // first channel of this thread's pair
  const int s = (tid >> 4) & 1;                 // stream
  const int bl = tid >> 5;                      // block lane
  const T* sx = reinterpret_cast<const T*>(smem + (1 + s) * SM::kTile);
  T* out = p.h[s] + ((long long)b * p.Tn) * p.C + (long long)slab * kCh + cp;

  for (int k = bl; k < NB; k += kThreads / 32) {
    const int cur = kHalo + k * L;              // smem row of the block start
    const int prev = cur - L;                   // smem row of the previous block
    // backward pass over the previous block: S[o] = its positions o+1 .. L-1
    float2 S[L];
    S[L - 1] = make_float2(0.f, 0.f);
    {
      float2 suf = make_float2(0.f, 0.f), P = make_float2(1.f, 1.f);
#pragma unroll
      for (int o = L - 1; o >= 1; --o) {
        const float2 gj = ld_pair(sg + (prev + o) * kCh + cp);
        const float2 xj = ld_pair(sx + (prev + o) * kCh + cp);
        suf = fma2(P, fma2(make_float2(-gj.x, -gj.y), xj, xj), suf);   // + P (1 - g) x
        P = mul2(P, gj);
        S[o - 1] = suf;
      }
    }
    // forward pass over this block
    const int tb = t0 + k * L;                  // first token of the block
    T* dst = out + (long long)tb * p.C;
    const bool whole = tb + L <= p.Tn;          // warp-uniform: no per-token bound check
    float2 loc = make_float2(0.f, 0.f), A = make_float2(1.f, 1.f);
#pragma unroll
    for (int o = 0; o < L; ++o) {
      const float2 gj = ld_pair(sg + (cur + o) * kCh + cp);
      const float2 xj = ld_pair(sx + (cur + o) * kCh + cp);
      loc = fma2(gj, sub2(loc, xj), xj);
      A = mul2(A, gj);
      if ((whole || tb + o < p.Tn) &&
          RATP_IN((dst - p.h[s]), 2, (long long)p.B * p.Tn * p.C))
        st_pair(dst, fma2(A, S[o], loc));
      dst += p.C;
    }
  }
}

}  // namespace window
}  // namespace ratp
