// scan.cuh -- single-pass chunked scan of the RAT+ forget-gate recurrence.
//
// h_t = g_t * h_{t-1} + (1 - g_t) * x_t per channel, h_{-1} = 0, over the full
// sequence (zhichai.net "RAT+ 深度拆解", section 2.1: forget-gate recurrence,
// associative scan in parallel at prefill).  Each step is the affine map
// h -> a h + b with a = g, b = (1 - g) x; maps compose associatively:
// (a2, b2) o (a1, b1) = (a2 a1, a2 b1 + b2).
//
// Decomposition (B200-first, HBM bound):
//   * a "chain" is one batch item x one slab of 64 contiguous channels; a
//     chunk is L consecutive tokens of one chain (L = 128 for bf16, 64 for
//     fp32).  One CTA of 256 threads owns one chunk.  Lanes cover contiguous
//     channels with 16-byte vectors, so every load instruction of a warp reads
//     whole 128-byte lines; each thread holds R = 4 consecutive tokens.
//   * in registers: each thread reduces its 4 tokens to one affine map; the
//     row groups of the CTA are combined by a shuffle scan in shared memory.
//   * across chunks: decoupled look-back.  Chunk tickets come from an atomic
//     counter in launch order, so a CTA only waits on chunks whose CTAs have
//     started.  A CTA publishes its aggregate map at once, then warp 0 polls
//     up to 32 predecessors in parallel and composes their aggregates until it
//     meets a published inclusive state.  Inputs stay in registers while it
//     waits, so x and g are read from HBM exactly once.
//   * every wait is bounded (kSpinTimeoutNs); on expiry the kernel records
//     RATP_ERR_TIMEOUT and finishes with a zero carry.
#pragma once
#include "common.cuh"
#include "sm100.cuh"

namespace ratp {
namespace scan {

constexpr int kThreads = 256;
constexpr int kSlab = 64;   // channels per chain
constexpr int kRows = 4;    // tokens per thread

template <typename T>
struct Shape {
  static constexpr int kVec = Elem<T>::kVec;             // channels per 16 B
  static constexpr int kLanes = kSlab / kVec;            // threads per token row
  static constexpr int kGroups = kThreads / kLanes;      // row groups per CTA
  static constexpr int kChunk = kGroups * kRows;         // tokens per chunk
};

// Workspace layout (bytes), given n = total chunks and NS streams:
//   [0, 256)                ticket counter (u32)
//   flags  u32 [n]          0 empty, 1 aggregate ready, 2 inclusive ready
//   agg    f32 [n][1+NS][64] aggregate map (a, b_stream...)
//   incl   f32 [n][NS][64]   inclusive state at the chunk's last token
struct Workspace {
  unsigned int* counter;
  unsigned int* flags;
  float* agg;
  float* incl;
};

__host__ __device__ inline size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

inline size_t workspace_bytes(long long n_chunks, int NS) {
  size_t b = 256;
  b += align256(sizeof(unsigned int) * n_chunks);
  b += align256(sizeof(float) * n_chunks * (1 + NS) * kSlab);
  b += align256(sizeof(float) * n_chunks * NS * kSlab);
  return b;
}

inline Workspace carve(void* base, long long n_chunks, int NS) {
  char* p = static_cast<char*>(base);
  Workspace w;
  w.counter = reinterpret_cast<unsigned int*>(p);
  p += 256;
  w.flags = reinterpret_cast<unsigned int*>(p);
  p += align256(sizeof(unsigned int) * n_chunks);
  w.agg = reinterpret_cast<float*>(p);
  p += align256(sizeof(float) * n_chunks * (1 + NS) * kSlab);
  w.incl = reinterpret_cast<float*>(p);
  return w;
}

// Bytes to zero before each launch: counter + flags.
inline size_t reset_bytes(long long n_chunks) {
  return 256 + align256(sizeof(unsigned int) * n_chunks);
}

template <typename T, int NS>
struct Params {
  T* h[NS];
  float* final_state;     // nullable: [NS][B][C]
  Workspace ws;
  int B, Tn, C;           // Tn tokens, C = H * Dh channels per token
  int slabs;              // C / 64
  int n_chains;           // B * slabs
  int n_chunks_t;         // chunks along T
};

// Dynamic shared memory: (1 + NS) tiles of [chunk][64] elements filled by TMA
// (the gate tile first), then the row-group maps of the intra-chunk scan.
template <typename T, int NS>
struct Smem {
  static constexpr int kTile = Shape<T>::kChunk * kSlab * (int)sizeof(T);   // 16 KB
  static constexpr int kData = (1 + NS) * kTile;
  static constexpr int kScan = Shape<T>::kGroups * kSlab * (1 + NS) * 4;
  static constexpr int kBytes = kData + kScan + 128;                       // + alignment
};

// Compose the affine maps of up to 8 predecessor chunks (nearest first) into
// the running composite x -> ca*x + cb, with all loads issued before use.
template <int NS>
__device__ __forceinline__ void compose_batch(const float* agg, long long d0, int n, int c0,
                                              float& ca0, float& ca1, float (&cb0)[NS],
                                              float (&cb1)[NS]) {
  float2 pa[8], pb[NS][8];
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    if (u < n) {
      const float* src = agg + (d0 - u) * (1 + NS) * kSlab;
      pa[u] = __ldcg(reinterpret_cast<const float2*>(src + c0));
#pragma unroll
      for (int s = 0; s < NS; ++s) pb[s][u] = __ldcg(reinterpret_cast<const float2*>(src + (1 + s) * kSlab + c0));
    }
  }
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    if (u < n) {
#pragma unroll
      for (int s = 0; s < NS; ++s) {
        cb0[s] = fmaf(ca0, pb[s][u].x, cb0[s]);
        cb1[s] = fmaf(ca1, pb[s][u].y, cb1[s]);
      }
      ca0 *= pa[u].x;
      ca1 *= pa[u].y;
    }
  }
}

template <typename T, int NS>
__global__ void __launch_bounds__(kThreads, 3)
scan_kernel(const __grid_constant__ CUtensorMap tm_g, const __grid_constant__ CUtensorMap tm_x0,
            const __grid_constant__ CUtensorMap tm_x1, const __grid_constant__ Params<T, NS> p) {
  using S = Shape<T>;
  using SM = Smem<T, NS>;
  constexpr int V = S::kVec, LANES = S::kLanes, G = S::kGroups, L = S::kChunk;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
  const T* s_g = reinterpret_cast<const T*>(smem);
  float* s_a = reinterpret_cast<float*>(smem + SM::kData);            // [G][64]
  float* s_b = s_a + G * kSlab;                                        // [NS][G][64]
  __shared__ __align__(8) uint64_t s_bar;
  __shared__ unsigned int s_ticket;
  __shared__ float s_tot_a[kSlab];
  __shared__ float s_tot_b[NS][kSlab];
  __shared__ float s_carry[NS][kSlab];

  const int tid = threadIdx.x;
  const uint32_t bar = sm100::smem_u32(&s_bar);
  if (tid == 0) {
    s_ticket = atomicAdd(p.ws.counter, 1u);
    sm100::mbar_init(bar, 1);
    sm100::fence_barrier_init();
  }
  __syncthreads();
  const unsigned int ticket = s_ticket;
  const int chunk = ticket / p.n_chains;     // chunk-major: predecessors started earlier
  const int chain = ticket % p.n_chains;
  const int b = chain / p.slabs;
  const int slab = chain % p.slabs;
  const long long desc = (long long)chain * p.n_chunks_t + chunk;   // descriptor index

  // ---- TMA: gate and input tiles of this chunk (rows past T read as zero) ----
  if (tid == 0) {
    sm100::mbar_arrive_expect_tx(bar, SM::kData);
    const uint32_t dst = sm100::smem_u32(smem);
    sm100::tma_load_3d(dst, &tm_g, bar, slab * kSlab, chunk * L, b);
    sm100::tma_load_3d(dst + SM::kTile, &tm_x0, bar, slab * kSlab, chunk * L, b);
    if (NS == 2) sm100::tma_load_3d(dst + 2 * SM::kTile, &tm_x1, bar, slab * kSlab, chunk * L, b);
  }

  const int lane_c = tid % LANES;            // 16-byte column within the slab
  const int grp = tid / LANES;               // row group
  const int t0 = chunk * L + grp * kRows;    // first token of this thread
  const int nrows = max(0, min(kRows, p.Tn - t0));   // valid tokens of this thread
  const long long row_stride = p.C;
  const long long base = ((long long)b * p.Tn) * row_stride + (long long)slab * kSlab + lane_c * V;
  const int soff = grp * kRows * kSlab + lane_c * V;   // element offset of row 0 in a tile

  {
    // bounded wait for the tiles (uniform outcome across the CTA)
    const unsigned long long tw = global_ns();
    bool ok = true;
    while (!sm100::mbar_try_wait(bar, 0)) {
      if (global_ns() - tw > kSpinTimeoutNs) { ok = false; break; }
    }
    if (!__syncthreads_and(ok)) {
      // publish a zero state so that successors do not wait on this chunk
      if (tid < 32) {
        for (int i = tid; i < NS * kSlab; i += 32) __stcg(p.ws.incl + desc * NS * kSlab + i, 0.f);
        __threadfence();
        __syncwarp();
        if (tid == 0) {
          raise_error(RATP_ERR_TIMEOUT);
          st_release_gpu(p.ws.flags + (long long)chain * p.n_chunks_t + chunk, 2u);
        }
      }
      return;
    }
  }

  // ---- thread-local aggregate of its tokens ----
  float la[V], lb[NS][V];
#pragma unroll
  for (int i = 0; i < V; ++i) la[i] = 1.f;
#pragma unroll
  for (int s = 0; s < NS; ++s)
#pragma unroll
    for (int i = 0; i < V; ++i) lb[s][i] = 0.f;
#pragma unroll
  for (int r = 0; r < kRows; ++r) {
    if (r < nrows) {
      float gf[V];
      Elem<T>::unpack(*reinterpret_cast<const uint4*>(s_g + soff + r * kSlab), gf);
#pragma unroll
      for (int s = 0; s < NS; ++s) {
        float xf[V];
        Elem<T>::unpack(*reinterpret_cast<const uint4*>(s_g + (1 + s) * L * kSlab + soff + r * kSlab), xf);
#pragma unroll
        for (int i = 0; i < V; ++i) lb[s][i] = fmaf(gf[i], lb[s][i] - xf[i], xf[i]);
      }
#pragma unroll
      for (int i = 0; i < V; ++i) la[i] *= gf[i];
    }
  }
#pragma unroll
  for (int i = 0; i < V; ++i) {
    s_a[grp * kSlab + lane_c * V + i] = la[i];
#pragma unroll
    for (int s = 0; s < NS; ++s) s_b[(s * G + grp) * kSlab + lane_c * V + i] = lb[s][i];
  }
  __syncthreads();

  // ---- exclusive scan over the G row groups, per channel (shuffle scan) ----
  {
    constexpr int kBlocks = kThreads / G;          // channel blocks
    const int gi = tid % G;                        // row group handled
    const int cb = tid / G;
    for (int c = cb; c < kSlab; c += kBlocks) {
      float a = s_a[gi * kSlab + c];
      float bb[NS];
#pragma unroll
      for (int s = 0; s < NS; ++s) bb[s] = s_b[(s * G + gi) * kSlab + c];
#pragma unroll
      for (int d = 1; d < G; d <<= 1) {
        const float ua = __shfl_up_sync(0xffffffffu, a, d, G);
        float ub[NS];
#pragma unroll
        for (int s = 0; s < NS; ++s) ub[s] = __shfl_up_sync(0xffffffffu, bb[s], d, G);
        if (gi >= d) {
#pragma unroll
          for (int s = 0; s < NS; ++s) bb[s] = fmaf(a, ub[s], bb[s]);   // self o up
          a *= ua;
        }
      }
      float ea = __shfl_up_sync(0xffffffffu, a, 1, G);
      float eb[NS];
#pragma unroll
      for (int s = 0; s < NS; ++s) eb[s] = __shfl_up_sync(0xffffffffu, bb[s], 1, G);
      if (gi == 0) {
        ea = 1.f;
#pragma unroll
        for (int s = 0; s < NS; ++s) eb[s] = 0.f;
      }
      if (gi == G - 1) {
        s_tot_a[c] = a;
#pragma unroll
        for (int s = 0; s < NS; ++s) s_tot_b[s][c] = bb[s];
      }
      s_a[gi * kSlab + c] = ea;
#pragma unroll
      for (int s = 0; s < NS; ++s) s_b[(s * G + gi) * kSlab + c] = eb[s];
    }
  }
  __syncthreads();

  // ---- publish, look back, publish inclusive (warp 0) ----
  if (tid < 32) {
    const int lane = tid;
    unsigned int* flags = p.ws.flags + (long long)chain * p.n_chunks_t;
    const float* agg = p.ws.agg;
    float* incl = p.ws.incl;
    const int c0 = lane * 2;                  // two channels per lane
    if (chunk == 0) {
#pragma unroll
      for (int s = 0; s < NS; ++s) {
        s_carry[s][c0] = 0.f;
        s_carry[s][c0 + 1] = 0.f;
        __stcg(reinterpret_cast<float2*>(incl + (desc * NS + s) * kSlab + c0),
               make_float2(s_tot_b[s][c0], s_tot_b[s][c0 + 1]));
      }
      __threadfence();
      __syncwarp();
      if (lane == 0) st_release_gpu(flags + chunk, 2u);
    } else {
      {
        float* dst = p.ws.agg + desc * (1 + NS) * kSlab;
        __stcg(reinterpret_cast<float2*>(dst + c0), make_float2(s_tot_a[c0], s_tot_a[c0 + 1]));
#pragma unroll
        for (int s = 0; s < NS; ++s)
          __stcg(reinterpret_cast<float2*>(dst + (1 + s) * kSlab + c0),
                 make_float2(s_tot_b[s][c0], s_tot_b[s][c0 + 1]));
      }
      __threadfence();
      __syncwarp();
      if (lane == 0) st_release_gpu(flags + chunk, 1u);

      // composite map of the predecessors seen so far: x -> ca x + cb
      float ca0 = 1.f, ca1 = 1.f;
      float cb0[NS], cb1[NS];
#pragma unroll
      for (int s = 0; s < NS; ++s) { cb0[s] = 0.f; cb1[s] = 0.f; }
      int top = chunk - 1;                     // nearest predecessor not yet composed
      const unsigned long long t_start = global_ns();
      while (true) {
        const int k = top - lane;
        const unsigned int f = (k >= 0) ? ld_acquire_gpu(flags + k) : 3u;   // 3: before start
        const unsigned int incl_mask = __ballot_sync(0xffffffffu, f >= 2u);
        const unsigned int empty_mask = __ballot_sync(0xffffffffu, f == 0u);
        int upto = -1;                          // compose lanes [0, upto)
        bool found = false;
        if (incl_mask != 0u) {
          const int jl = __ffs(incl_mask) - 1;
          const unsigned int below = (jl == 0) ? 0u : ((1u << jl) - 1u);
          if ((empty_mask & below) == 0u) { upto = jl; found = true; }
        } else if (empty_mask == 0u) {
          upto = 32;                            // 32 aggregates: compose, go further back
        }
        if (upto < 0) {
          const bool expired = (global_ns() - t_start) > kSpinTimeoutNs;
          if (__any_sync(0xffffffffu, expired)) {
            if (lane == 0) raise_error(RATP_ERR_TIMEOUT);
            ca0 = ca1 = 0.f;                     // give up: zero carry
#pragma unroll
            for (int s = 0; s < NS; ++s) { cb0[s] = 0.f; cb1[s] = 0.f; }
            break;
          }
          __nanosleep(32);
          continue;
        }
        __syncwarp();
        __threadfence();
        // inclusive state of the chunk that ends the look-back (issued first)
        float v0[NS], v1[NS];
#pragma unroll
        for (int s = 0; s < NS; ++s) { v0[s] = 0.f; v1[s] = 0.f; }
        const int kin = top - upto;
        if (found && kin >= 0) {
          const long long dk = (long long)chain * p.n_chunks_t + kin;
#pragma unroll
          for (int s = 0; s < NS; ++s) {
            const float2 pv = __ldcg(reinterpret_cast<const float2*>(incl + (dk * NS + s) * kSlab + c0));
            v0[s] = pv.x; v1[s] = pv.y;
          }
        }
        const long long dtop = (long long)chain * p.n_chunks_t + top;
        for (int m0 = 0; m0 < upto; m0 += 8)
          compose_batch<NS>(agg, dtop - m0, min(8, upto - m0), c0, ca0, ca1, cb0, cb1);
        if (found) {
#pragma unroll
          for (int s = 0; s < NS; ++s) {
            cb0[s] = fmaf(ca0, v0[s], cb0[s]);   // carry = composite(inclusive)
            cb1[s] = fmaf(ca1, v1[s], cb1[s]);
          }
          break;
        }
        top -= 32;
      }
      // cb now holds the state entering this chunk
#pragma unroll
      for (int s = 0; s < NS; ++s) {
        s_carry[s][c0] = cb0[s];
        s_carry[s][c0 + 1] = cb1[s];
        const float e0 = fmaf(s_tot_a[c0], cb0[s], s_tot_b[s][c0]);
        const float e1 = fmaf(s_tot_a[c0 + 1], cb1[s], s_tot_b[s][c0 + 1]);
        __stcg(reinterpret_cast<float2*>(incl + (desc * NS + s) * kSlab + c0), make_float2(e0, e1));
      }
      __threadfence();
      __syncwarp();
      if (lane == 0) st_release_gpu(flags + chunk, 2u);
    }
  }
  __syncthreads();

  // ---- recompute the tokens from the carry and store ----
  float hs[NS][V];
#pragma unroll
  for (int i = 0; i < V; ++i) {
    const int c = lane_c * V + i;
    const float ea = s_a[grp * kSlab + c];
#pragma unroll
    for (int s = 0; s < NS; ++s) hs[s][i] = fmaf(ea, s_carry[s][c], s_b[(s * G + grp) * kSlab + c]);
  }
#pragma unroll
  for (int r = 0; r < kRows; ++r) {
    if (r < nrows) {
      const int t = t0 + r;
      float gf[V];
      Elem<T>::unpack(*reinterpret_cast<const uint4*>(s_g + soff + r * kSlab), gf);
#pragma unroll
      for (int s = 0; s < NS; ++s) {
        float xf[V];
        Elem<T>::unpack(*reinterpret_cast<const uint4*>(s_g + (1 + s) * L * kSlab + soff + r * kSlab), xf);
#pragma unroll
        for (int i = 0; i < V; ++i) hs[s][i] = fmaf(gf[i], hs[s][i] - xf[i], xf[i]);
        const long long off = base + (long long)t * row_stride;
        __stcs(reinterpret_cast<uint4*>(p.h[s] + off), Elem<T>::pack(hs[s]));
        if (t == p.Tn - 1 && p.final_state != nullptr) {
          float* fs = p.final_state + ((long long)s * p.B + b) * p.C + slab * kSlab + lane_c * V;
#pragma unroll
          for (int i = 0; i < V; ++i) fs[i] = hs[s][i];
        }
      }
    }
  }
}

}  // namespace scan
}  // namespace ratp
