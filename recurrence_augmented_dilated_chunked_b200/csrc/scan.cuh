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
  const T* x[NS];
  const T* g;
  T* h[NS];
  float* final_state;     // nullable: [NS][B][C]
  Workspace ws;
  int B, Tn, C;           // Tn tokens, C = H * Dh channels per token
  int slabs;              // C / 64
  int n_chains;           // B * slabs
  int n_chunks_t;         // chunks along T
};

template <typename T, int NS>
__global__ void __launch_bounds__(kThreads, 2)
scan_kernel(const Params<T, NS> p) {
  using S = Shape<T>;
  constexpr int V = S::kVec, LANES = S::kLanes, G = S::kGroups, L = S::kChunk;

  __shared__ unsigned int s_ticket;
  __shared__ float s_a[G][kSlab];            // per row-group maps, then exclusive prefix
  __shared__ float s_b[NS][G][kSlab];
  __shared__ float s_tot_a[kSlab];           // chunk aggregate
  __shared__ float s_tot_b[NS][kSlab];
  __shared__ float s_carry[NS][kSlab];       // state entering the chunk
  __shared__ int s_timeout;

  const int tid = threadIdx.x;
  if (tid == 0) {
    s_ticket = atomicAdd(p.ws.counter, 1u);
    s_timeout = 0;
  }
  __syncthreads();
  const unsigned int ticket = s_ticket;
  const int chunk = ticket / p.n_chains;     // chunk-major: predecessors started earlier
  const int chain = ticket % p.n_chains;
  const int b = chain / p.slabs;
  const int slab = chain % p.slabs;
  const long long desc = (long long)chain * p.n_chunks_t + chunk;   // descriptor index

  const int lane_c = tid % LANES;            // 16-byte column within the slab
  const int grp = tid / LANES;               // row group
  const int t0 = chunk * L + grp * kRows;    // first token of this thread
  const long long row_stride = p.C;
  const long long base = ((long long)b * p.Tn) * row_stride + (long long)slab * kSlab + lane_c * V;

  // ---- load 4 tokens x (x streams, g): all loads issued before any use ----
  uint4 rg[kRows], rx[NS][kRows];
#pragma unroll
  for (int r = 0; r < kRows; ++r) {
    const int t = t0 + r;
    if (t < p.Tn) {
      const long long off = base + (long long)t * row_stride;
      rg[r] = __ldcs(reinterpret_cast<const uint4*>(p.g + off));
#pragma unroll
      for (int s = 0; s < NS; ++s) rx[s][r] = __ldcs(reinterpret_cast<const uint4*>(p.x[s] + off));
    } else {
      // padding tokens act as the identity map: a = 1, b = 0
      float one[V], zero[V];
#pragma unroll
      for (int i = 0; i < V; ++i) { one[i] = 1.f; zero[i] = 0.f; }
      rg[r] = Elem<T>::pack(one);
#pragma unroll
      for (int s = 0; s < NS; ++s) rx[s][r] = Elem<T>::pack(zero);
    }
  }

  // ---- thread-local aggregate of 4 tokens ----
  float la[V], lb[NS][V];
#pragma unroll
  for (int i = 0; i < V; ++i) { la[i] = 1.f; }
#pragma unroll
  for (int s = 0; s < NS; ++s)
#pragma unroll
    for (int i = 0; i < V; ++i) lb[s][i] = 0.f;
#pragma unroll
  for (int r = 0; r < kRows; ++r) {
    float gf[V];
    Elem<T>::unpack(rg[r], gf);
#pragma unroll
    for (int s = 0; s < NS; ++s) {
      float xf[V];
      Elem<T>::unpack(rx[s][r], xf);
#pragma unroll
      for (int i = 0; i < V; ++i) lb[s][i] = fmaf(gf[i], lb[s][i] - xf[i], xf[i]);
    }
#pragma unroll
    for (int i = 0; i < V; ++i) la[i] *= gf[i];
  }
#pragma unroll
  for (int i = 0; i < V; ++i) {
    s_a[grp][lane_c * V + i] = la[i];
#pragma unroll
    for (int s = 0; s < NS; ++s) s_b[s][grp][lane_c * V + i] = lb[s][i];
  }
  __syncthreads();

  // ---- exclusive scan over the G row groups, per channel (shuffle scan) ----
  {
    constexpr int kBlocks = kThreads / G;          // channel blocks
    const int gi = tid % G;                        // row group handled
    const int cb = tid / G;
    for (int c = cb; c < kSlab; c += kBlocks) {
      float a = s_a[gi][c];
      float bb[NS];
#pragma unroll
      for (int s = 0; s < NS; ++s) bb[s] = s_b[s][gi][c];
#pragma unroll
      for (int d = 1; d < G; d <<= 1) {
        float ua = __shfl_up_sync(0xffffffffu, a, d, G);
        float ub[NS];
#pragma unroll
        for (int s = 0; s < NS; ++s) ub[s] = __shfl_up_sync(0xffffffffu, bb[s], d, G);
        if (gi >= d) {
#pragma unroll
          for (int s = 0; s < NS; ++s) bb[s] = fmaf(a, ub[s], bb[s]);   // self o up
          a *= ua;
        }
      }
      // inclusive -> exclusive
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
      __syncwarp();
      s_a[gi][c] = ea;
#pragma unroll
      for (int s = 0; s < NS; ++s) s_b[s][gi][c] = eb[s];
    }
  }
  __syncthreads();

  // ---- publish, look back, publish inclusive (warp 0) ----
  if (tid < 32) {
    const int lane = tid;
    unsigned int* flags = p.ws.flags + (long long)chain * p.n_chunks_t;
    float* agg = p.ws.agg;
    float* incl = p.ws.incl;
    const int c0 = lane * 2;                  // two channels per lane
    if (chunk == 0) {
#pragma unroll
      for (int s = 0; s < NS; ++s) {
        s_carry[s][c0] = 0.f;
        s_carry[s][c0 + 1] = 0.f;
        float* dst = incl + (desc * NS + s) * kSlab;
        __stcg(reinterpret_cast<float2*>(dst + c0), make_float2(s_tot_b[s][c0], s_tot_b[s][c0 + 1]));
      }
      __syncwarp();
      if (lane == 0) st_release_gpu(flags + chunk, 2u);
    } else {
      {
        float* dst = agg + desc * (1 + NS) * kSlab;
        __stcg(reinterpret_cast<float2*>(dst + c0), make_float2(s_tot_a[c0], s_tot_a[c0 + 1]));
#pragma unroll
        for (int s = 0; s < NS; ++s)
          __stcg(reinterpret_cast<float2*>(dst + (1 + s) * kSlab + c0),
                 make_float2(s_tot_b[s][c0], s_tot_b[s][c0 + 1]));
      }
      __syncwarp();
      if (lane == 0) st_release_gpu(flags + chunk, 1u);

      // composite map of the predecessors seen so far: x -> ca x + cb
      float ca0 = 1.f, ca1 = 1.f;
      float cb0[NS], cb1[NS];
#pragma unroll
      for (int s = 0; s < NS; ++s) { cb0[s] = 0.f; cb1[s] = 0.f; }
      int top = chunk - 1;                     // nearest predecessor not yet composed
      const unsigned long long t_start = global_ns();
      bool done = false;
      while (!done) {
        const int k = top - lane;
        unsigned int f = (k >= 0) ? ld_acquire_gpu(flags + k) : 3u;   // 3: before start
        const unsigned int incl_mask = __ballot_sync(0xffffffffu, f >= 2u);
        const unsigned int empty_mask = __ballot_sync(0xffffffffu, f == 0u);
        int upto;                               // compose lanes [0, upto)
        bool found;
        if (incl_mask != 0u) {
          const int jl = __ffs(incl_mask) - 1;
          const unsigned int below = (jl == 0) ? 0u : ((1u << jl) - 1u);
          if ((empty_mask & below) != 0u) {
            upto = -1; found = false;            // a gap: wait
          } else {
            upto = jl; found = true;
          }
        } else if (empty_mask == 0u) {
          upto = 32; found = false;              // 32 aggregates: compose, go further back
        } else {
          upto = -1; found = false;
        }
        if (upto < 0) {
          if (global_ns() - t_start > kSpinTimeoutNs) {
            if (lane == 0) { raise_error(RATP_ERR_TIMEOUT); s_timeout = 1; }
            ca0 = ca1 = 0.f;                     // give up: zero carry
#pragma unroll
            for (int s = 0; s < NS; ++s) { cb0[s] = 0.f; cb1[s] = 0.f; }
            break;
          }
          __nanosleep(64);
          continue;
        }
        __syncwarp();
        // compose aggregates of predecessors top, top-1, ..., top-upto+1
        for (int m = 0; m < upto; ++m) {
          const long long dk = (long long)chain * p.n_chunks_t + (top - m);
          const float* src = agg + dk * (1 + NS) * kSlab;
          const float2 pa = __ldcg(reinterpret_cast<const float2*>(src + c0));
#pragma unroll
          for (int s = 0; s < NS; ++s) {
            const float2 pb = __ldcg(reinterpret_cast<const float2*>(src + (1 + s) * kSlab + c0));
            cb0[s] = fmaf(ca0, pb.x, cb0[s]);
            cb1[s] = fmaf(ca1, pb.y, cb1[s]);
          }
          ca0 *= pa.x;
          ca1 *= pa.y;
        }
        if (found) {
          const int kin = top - upto;
          float v0[NS], v1[NS];
          if (kin >= 0) {
            const long long dk = (long long)chain * p.n_chunks_t + kin;
#pragma unroll
            for (int s = 0; s < NS; ++s) {
              const float2 pv = __ldcg(reinterpret_cast<const float2*>(incl + (dk * NS + s) * kSlab + c0));
              v0[s] = pv.x; v1[s] = pv.y;
            }
          } else {
#pragma unroll
            for (int s = 0; s < NS; ++s) { v0[s] = 0.f; v1[s] = 0.f; }
          }
#pragma unroll
          for (int s = 0; s < NS; ++s) {
            cb0[s] = fmaf(ca0, v0[s], cb0[s]);   // carry = composite(incl)
            cb1[s] = fmaf(ca1, v1[s], cb1[s]);
          }
          done = true;
        } else {
          top -= 32;
        }
      }
      // cb now holds the state entering this chunk
#pragma unroll
      for (int s = 0; s < NS; ++s) {
        s_carry[s][c0] = cb0[s];
        s_carry[s][c0 + 1] = cb1[s];
        const float e0 = fmaf(s_tot_a[c0], cb0[s], s_tot_b[s][c0]);
        const float e1 = fmaf(s_tot_a[c0 + 1], cb1[s], s_tot_b[s][c0 + 1]);
        float* dst = incl + (desc * NS + s) * kSlab;
        __stcg(reinterpret_cast<float2*>(dst + c0), make_float2(e0, e1));
      }
      __syncwarp();
      if (lane == 0) st_release_gpu(flags + chunk, 2u);
    }
  }
  __syncthreads();

  // ---- recompute the 4 tokens from the carry and store ----
  float hs[NS][V];
#pragma unroll
  for (int i = 0; i < V; ++i) {
    const int c = lane_c * V + i;
    const float ea = s_a[grp][c];
#pragma unroll
    for (int s = 0; s < NS; ++s) hs[s][i] = fmaf(ea, s_carry[s][c], s_b[s][grp][c]);
  }
#pragma unroll
  for (int r = 0; r < kRows; ++r) {
    const int t = t0 + r;
    float gf[V];
    Elem<T>::unpack(rg[r], gf);
#pragma unroll
    for (int s = 0; s < NS; ++s) {
      float xf[V];
      Elem<T>::unpack(rx[s][r], xf);
#pragma unroll
      for (int i = 0; i < V; ++i) hs[s][i] = fmaf(gf[i], hs[s][i] - xf[i], xf[i]);
      if (t < p.Tn) {
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
