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
//     chunk is L consecutive tokens of one chain.  One CTA of 256 threads owns
//     one chunk, staged by TMA into shared memory (gate tile + one tile per
//     stream).  A thread holds R consecutive tokens x 8 (bf16; 4 for fp32)
//     contiguous channels, works on channel pairs with packed f32x2
//     arithmetic, and reduces its tokens to one affine map per channel.
//   * within the chunk: the row groups of a warp are combined by a shuffle
//     scan, the 8 warp totals by one warp through shared memory.
//   * across chunks: decoupled look-back.  Chunk tickets come from an atomic
//     counter in launch order, so a CTA only waits on chunks whose CTAs have
//     started.  Each lane of warp 0 owns two channels of the chunk's
//     descriptor: it publishes its part of the aggregate map at once as
//     tagged 64-bit words, then reads two predecessors per round trip
//     and composes their aggregates until it meets an inclusive state.  x and
//     g are read from HBM exactly once.
//   * DRAM keeps streaming while CTAs compute: thread 0 of the CTA with ticket
//     k also prefetches into L2 the tiles of ticket k + l2_ahead (about one
//     ticket per SM ahead), so the TMA loads of later CTAs mostly hit L2.
//   * every wait is bounded (spin_timeout()); on expiry the kernel records
//     RATP_ERR_TIMEOUT, sets a kernel-wide abort word so that no other CTA
//     keeps waiting, and finishes with a zero carry.
//
// Chunk-local variant (RESET; the original RAT that section 2.1 of the same
// write-up contrasts with RAT+, where a token recurs only inside its block of
// reset_L tokens): the step of a token t with t mod reset_L == 0 becomes the
// map (0, (1 - g) x).  Only those steps change; the composition, the in-chunk
// scan and the look-back are the same maps.  A chunk whose first token
// restarts needs no carry and skips the look-back; otherwise the look-back
// stops at the predecessor holding the last restart (its aggregate slope is
// exactly 0), so no chain waits further back than one block.
#pragma once
#include "common.cuh"
#include "sm100.cuh"

namespace ratp {
namespace scan {

constexpr int kThreads = 256;
constexpr int kSlab = 64;   // channels per chain
// Tokens per thread: 8 gives 256-token bf16 chunks (96 KB of tiles, two CTAs
// per SM); 4 (128-token chunks, four CTAs per SM, twice the look-backs)
// measured 25% slower.
constexpr int kRows = 8;

template <typename T, int R = kRows>
struct Shape {
  static constexpr int kVec = Elem<T>::kVec;             // channels per 16 B
  static constexpr int kLanes = kSlab / kVec;            // threads per token row
  static constexpr int kGroups = kThreads / kLanes;      // row groups per CTA
  static constexpr int kChunk = kGroups * R;             // tokens per chunk
};

// Workspace layout (bytes), given n = total chunks and NS streams:
//   [0, 256)                       header: ticket word (u64 at byte 0: launch
//                                  tag in the high 32 bits, ticket counter in
//                                  the low 32), kept across launches; abort
//                                  word (u32 at byte 128), zeroed before each
//                                  launch
//   agg  u64 [n][2(1+NS)][32]      aggregate map words, lane-minor
//   incl u64 [n][2 NS][32]         inclusive-state words, lane-minor
// Lane l of warp 0 owns channels 2l, 2l+1 of a chunk; word w of lane l holds
// {tag (high 32 bits), fp32 value (low 32 bits)}.  A 64-bit word is written
// and read in one access, so a reader that sees the current launch's tag also
// sees its value: the descriptors need no flags, fences or reset, only a zero
// fill before the workspace's first use (tag 0 is never issued).
// The tag lives on the device: every CTA draws its ticket with one 64-bit
// atomic add on the ticket word, which also returns the tag stored there; the
// launch uses the next tag (1, 2, ..., 2^32 - 1, 1, ...).  The CTA that draws
// the last ticket stores {next tag, counter 0}; every other CTA's add comes
// before that store in the word's order, so all of them saw the old tag, and
// the next launch finds its counter at zero.  A launch replayed from a CUDA
// graph therefore gets a fresh tag too, which a tag fixed in the kernel
// parameters at capture time would not.
struct Workspace {
  unsigned long long* ticket;
  unsigned int* abort;
  unsigned long long* agg;
  unsigned long long* incl;
};

__host__ __device__ inline size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

constexpr int kDescLanes = 32;

inline size_t workspace_bytes(long long n_chunks, int NS) {
  size_t b = 256;
  b += align256(sizeof(unsigned long long) * n_chunks * 2 * (1 + NS) * kDescLanes);
  b += align256(sizeof(unsigned long long) * n_chunks * 2 * NS * kDescLanes);
  return b;
}

inline Workspace carve(void* base, long long n_chunks, int NS) {
  char* p = static_cast<char*>(base);
  Workspace w;
  w.ticket = reinterpret_cast<unsigned long long*>(p);
  w.abort = reinterpret_cast<unsigned int*>(p + 128);
  p += 256;
  w.agg = reinterpret_cast<unsigned long long*>(p);
  p += align256(sizeof(unsigned long long) * n_chunks * 2 * (1 + NS) * kDescLanes);
  w.incl = reinterpret_cast<unsigned long long*>(p);
  return w;
}

// Zeroed before each launch: the abort word (the ticket word is kept).
constexpr size_t kResetOffset = 128, kResetBytes = 64;

__device__ __forceinline__ void put_word(unsigned long long* p, float v, unsigned int tag) {
  const unsigned long long w = ((unsigned long long)tag << 32) | __float_as_uint(v);
  asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" :: "l"(p), "l"(w) : "memory");
}

__device__ __forceinline__ unsigned long long get_word(const unsigned long long* p) {
  unsigned long long w;
  asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(w) : "l"(p) : "memory");
  return w;
}

__device__ __forceinline__ bool word_ok(unsigned long long w, unsigned int tag) {
  return (unsigned int)(w >> 32) == tag;
}

__device__ __forceinline__ float word_val(unsigned long long w) {
  return __uint_as_float((unsigned int)w);
}

// Draws this CTA's ticket and returns the launch tag (see Workspace).
__device__ __forceinline__ unsigned int draw_ticket(const Workspace& ws, unsigned int n_tickets,
                                                    unsigned int* ticket) {
  unsigned long long old;
  asm volatile("atom.relaxed.gpu.global.add.u64 %0, [%1], 1;" : "=l"(old) : "l"(ws.ticket) : "memory");
  const unsigned int t = (unsigned int)old, stored = (unsigned int)(old >> 32);
  const unsigned int tag = stored == 0xffffffffu ? 1u : stored + 1u;
  if (t == n_tickets - 1u)
    asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" :: "l"(ws.ticket), "l"((unsigned long long)tag << 32)
                 : "memory");
  *ticket = t;
  return tag;
}

template <typename T, int NS>
struct Params {
  T* h[NS];
  float* final_state;     // nullable: [NS][B][C]
  Workspace ws;
  int B, Tn, C;           // Tn tokens, C = H * Dh channels per token
  int reset_L;            // chunk-local block length (RESET kernels only, >= 1)
  int l2_ahead;           // L2 prefetch distance in tickets (0: none)
  int slabs;              // C / 64
  int n_chains;           // B * slabs
  int n_chunks_t;         // chunks along T
  unsigned int* done;     // fused prefill only: per-chunk done flags (see scan_chunk)
};

// Dynamic shared memory: (1 + NS) tiles of [chunk][64] elements filled by TMA
// (the gate tile first), then the per-warp totals of the intra-chunk scan.
template <typename T, int NS, int R = kRows>
struct Smem {
  static constexpr int kTile = Shape<T, R>::kChunk * kSlab * (int)sizeof(T);
  static constexpr int kData = (1 + NS) * kTile;
  static constexpr int kScan = (kThreads / 32) * (1 + NS) * kSlab * 4;
  static constexpr int kBytes = kData + kScan + 128;                       // + alignment
};

// One chunk (the chunk of `ticket`) by the whole CTA: its tiles are staged
// into `smem` (128-byte aligned, Smem::kBytes) through the mbarrier `bar`,
// whose phase `parity` this call completes.  Returns false when a bounded
// wait ran out or another CTA aborted; a CTA that goes on using `smem` must
// then first let the copies in flight on `bar` land.
// FUSED (the fused prefill, whose attention reads h_k/h_v right after the
// scan): the stores keep their lines in L2 (no streaming hint), and once all
// of the chunk is stored, after its predecessor in the chain, the chunk's done
// flag p.done[desc] takes the launch tag.  Flags therefore complete in
// sequence order per chain: a reader that sees chunk c done may read every
// row of the chain up to the end of chunk c.
template <typename T, int NS, int R, bool RESET, bool FUSED>
__device__ __forceinline__ bool scan_chunk(const CUtensorMap& tm_g, const CUtensorMap& tm_x0,
                                           const CUtensorMap& tm_x1, const Params<T, NS>& p, uint8_t* smem,
                                           uint32_t bar, uint32_t parity, unsigned int ticket, unsigned int tag) {
  using S = Shape<T, R>;
  using SM = Smem<T, NS, R>;
  constexpr int V = S::kVec, V2 = V / 2, LANES = S::kLanes, L = S::kChunk;
  constexpr int NW = kThreads / 32;

  const T* s_g = reinterpret_cast<const T*>(smem);
  float* s_w = reinterpret_cast<float*>(smem + SM::kData);            // [NW][1 + NS][64]
  __shared__ float s_tot_a[kSlab];
  __shared__ float s_tot_b[NS][kSlab];
  __shared__ float s_carry[NS][kSlab];
  static_assert(32 % LANES == 0, "row groups of a warp must share channels");

  const int tid = threadIdx.x;
  auto aborted = [&]() -> bool {
    unsigned int v;
    asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p.ws.abort) : "memory");
    return v != 0u;
  };
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
    // warm L2 with the tiles of the chunk l2_ahead tickets later, so that
    // DRAM keeps streaming while the resident CTAs compute
    {
      const long long nt = (long long)ticket + p.l2_ahead;
      if (p.l2_ahead > 0 && nt < (long long)p.n_chains * p.n_chunks_t) {
        const int ck = (int)(nt / p.n_chains), chn = (int)(nt % p.n_chains);
        const int b2 = chn / p.slabs, s2 = chn % p.slabs;
        sm100::tma_prefetch_l2_3d(&tm_g, s2 * kSlab, ck * L, b2);
        sm100::tma_prefetch_l2_3d(&tm_x0, s2 * kSlab, ck * L, b2);
        if (NS == 2) sm100::tma_prefetch_l2_3d(&tm_x1, s2 * kSlab, ck * L, b2);
      }
    }
  }

  const int lane_c = tid % LANES;            // 16-byte column within the slab
  const int grp = tid / LANES;               // row group
  const int t0 = chunk * L + grp * R;        // first token of this thread
  const int nrows = max(0, min(R, p.Tn - t0));   // valid tokens of this thread
  const long long row_stride = p.C;
  const long long base = ((long long)b * p.Tn) * row_stride + (long long)slab * kSlab + lane_c * V;
  const int soff = grp * R * kSlab + lane_c * V;   // element offset of row 0 in a tile
  // rows r of this thread whose token restarts the recurrence (bit r)
  unsigned int rmask = 0u;
  if (RESET) {
    for (int r = (p.reset_L - t0 % p.reset_L) % p.reset_L; r < R; r += p.reset_L) rmask |= 1u << r;
  }

  {
    // one thread waits for the tiles (bounded; the clock and the abort word
    // are read every 64 polls), the others sleep in the barrier
    bool ok = true;
    if (tid == 0) {
      unsigned long long tw = 0;
      unsigned int n = 0;
      while (!sm100::mbar_try_wait(bar, parity)) {
        if ((++n & 63u) == 0u) {
          const unsigned long long now = global_ns();
          if (tw == 0) tw = now;
          else if (now - tw > spin_timeout() || aborted()) { ok = false; break; }
        }
      }
    }
    if (!__syncthreads_and(ok)) {
      // give up: publish a zero state for this chunk and make every other
      // CTA stop waiting
      if (tid < 32 && RATP_IN(desc, 1, (long long)p.n_chains * p.n_chunks_t)) {
#pragma unroll
        for (int w = 0; w < 2 * NS; ++w)
          put_word(p.ws.incl + (desc * 2 * NS + w) * kDescLanes + tid, 0.f, tag);
        if (tid == 0) {
          raise_error(RATP_ERR_TIMEOUT);
          atomicExch(p.ws.abort, 1u);
        }
      }
      return false;
    }
  }

  // ---- thread-local aggregate of its tokens (channel pairs) ----
  float2 la[V2], lb[NS][V2];
#pragma unroll
  for (int i = 0; i < V2; ++i) {
    la[i] = make_float2(1.f, 1.f);
#pragma unroll
    for (int s = 0; s < NS; ++s) lb[s][i] = make_float2(0.f, 0.f);
  }
#pragma unroll
  for (int r = 0; r < R; ++r) {
    if (r < nrows) {
      if (RESET && ((rmask >> r) & 1u)) {    // restart: forget the rows before
#pragma unroll
        for (int i = 0; i < V2; ++i) {
          la[i] = make_float2(0.f, 0.f);
#pragma unroll
          for (int s = 0; s < NS; ++s) lb[s][i] = make_float2(0.f, 0.f);
        }
      }
      float2 gf[V2];
      Elem<T>::unpack2(*reinterpret_cast<const uint4*>(s_g + soff + r * kSlab), gf);
#pragma unroll
      for (int s = 0; s < NS; ++s) {
        float2 xf[V2];
        Elem<T>::unpack2(*reinterpret_cast<const uint4*>(s_g + (1 + s) * L * kSlab + soff + r * kSlab), xf);
#pragma unroll
        for (int i = 0; i < V2; ++i) lb[s][i] = fma2(gf[i], sub2(lb[s][i], xf[i]), xf[i]);
      }
#pragma unroll
      for (int i = 0; i < V2; ++i) la[i] = mul2(la[i], gf[i]);
    }
  }

  // ---- intra-chunk scan over row groups, hierarchical ----
  // (1) the row groups of one warp hold the same channels in lanes
  //     lane_c, lane_c + LANES, ...: a shuffle scan over them (stride LANES)
  //     gives each thread the map of the warp's rows up to and including its
  //     own; (2) lane group GW-1 publishes the warp total, warp 0 scans the NW
  //     totals per channel; (3) each thread composes its exclusive prefix.
  constexpr int GW = 32 / LANES;             // row groups per warp
  const int lane = tid & 31, wid = tid >> 5;
  const int gw = lane / LANES;               // row group within the warp
  float2 ia[V2], ib[NS][V2];                 // inclusive map within the warp
#pragma unroll
  for (int i = 0; i < V2; ++i) {
    ia[i] = la[i];
#pragma unroll
    for (int s = 0; s < NS; ++s) ib[s][i] = lb[s][i];
  }
#pragma unroll
  for (int d = 1; d < GW; d <<= 1) {
#pragma unroll
    for (int i = 0; i < V2; ++i) {
      float2 ua, ub[NS];
      ua.x = __shfl_up_sync(0xffffffffu, ia[i].x, d * LANES);
      ua.y = __shfl_up_sync(0xffffffffu, ia[i].y, d * LANES);
#pragma unroll
      for (int s = 0; s < NS; ++s) {
        ub[s].x = __shfl_up_sync(0xffffffffu, ib[s][i].x, d * LANES);
        ub[s].y = __shfl_up_sync(0xffffffffu, ib[s][i].y, d * LANES);
      }
      if (gw >= d) {
#pragma unroll
        for (int s = 0; s < NS; ++s) ib[s][i] = fma2(ia[i], ub[s], ib[s][i]);   // self o up
        ia[i] = mul2(ia[i], ua);
      }
    }
  }
  if (gw == GW - 1) {                        // warp total
#pragma unroll
    for (int i = 0; i < V2; ++i) {
      const int c = lane_c * V + 2 * i;
      *reinterpret_cast<float2*>(s_w + (wid * (1 + NS)) * kSlab + c) = ia[i];
#pragma unroll
      for (int s = 0; s < NS; ++s) *reinterpret_cast<float2*>(s_w + (wid * (1 + NS) + 1 + s) * kSlab + c) = ib[s][i];
    }
  }
  __syncthreads();
  if (tid < 32) {
    // exclusive prefix over warps (in place) and the chunk total, 2 channels per lane
    const int c = 2 * tid;
    float2 pa = make_float2(1.f, 1.f), pb[NS];
#pragma unroll
    for (int s = 0; s < NS; ++s) pb[s] = make_float2(0.f, 0.f);
#pragma unroll
    for (int w = 0; w < NW; ++w) {
      float2* wa = reinterpret_cast<float2*>(s_w + (w * (1 + NS)) * kSlab + c);
      const float2 va = *wa;
      *wa = pa;
#pragma unroll
      for (int s = 0; s < NS; ++s) {
        float2* wb = reinterpret_cast<float2*>(s_w + (w * (1 + NS) + 1 + s) * kSlab + c);
        const float2 vb = *wb;
        *wb = pb[s];
        pb[s] = fma2(va, pb[s], vb);         // warp w applied after the prefix
      }
      pa = mul2(pa, va);
    }
    s_tot_a[c] = pa.x;
    s_tot_a[c + 1] = pa.y;
#pragma unroll
    for (int s = 0; s < NS; ++s) {
      s_tot_b[s][c] = pb[s].x;
      s_tot_b[s][c + 1] = pb[s].y;
    }
  }
  __syncthreads();
  // exclusive map of this thread's row group: (within-warp exclusive) o (warp prefix)
  float2 ea[V2], eb[NS][V2];
#pragma unroll
  for (int i = 0; i < V2; ++i) {
    float2 xa, xb[NS];
    xa.x = __shfl_up_sync(0xffffffffu, ia[i].x, LANES);
    xa.y = __shfl_up_sync(0xffffffffu, ia[i].y, LANES);
#pragma unroll
    for (int s = 0; s < NS; ++s) {
      xb[s].x = __shfl_up_sync(0xffffffffu, ib[s][i].x, LANES);
      xb[s].y = __shfl_up_sync(0xffffffffu, ib[s][i].y, LANES);
    }
    if (gw == 0) {
      xa = make_float2(1.f, 1.f);
#pragma unroll
      for (int s = 0; s < NS; ++s) xb[s] = make_float2(0.f, 0.f);
    }
    const int c = lane_c * V + 2 * i;
    const float2 wa = *reinterpret_cast<const float2*>(s_w + (wid * (1 + NS)) * kSlab + c);
#pragma unroll
    for (int s = 0; s < NS; ++s) {
      const float2 wb = *reinterpret_cast<const float2*>(s_w + (wid * (1 + NS) + 1 + s) * kSlab + c);
      eb[s][i] = fma2(xa, wb, xb[s]);
    }
    ea[i] = mul2(xa, wa);
  }

  // ---- publish, look back, publish inclusive (warp 0) ----
  // Lane l of warp 0 owns channels c0 = 2l, 2l+1: it writes its aggregate
  // words, walks back over predecessor chunks of the chain reading the same
  // lane's words (two predecessors per round trip), composing aggregates until
  // it meets an inclusive state, then writes its own inclusive words.
  if (tid < 32) {
    const int lane = tid;
    const bool drop = (long long)ticket == g_fault_scan_ticket;   // planted failure: publish nothing
    constexpr int WA = 2 * (1 + NS), WI = 2 * NS;   // words per lane
    const unsigned long long* agg = p.ws.agg;
    const unsigned long long* incl = p.ws.incl;
    const long long chain0 = (long long)chain * p.n_chunks_t;   // descriptor of chunk 0
    const int c0 = lane * 2;
    float cb0[NS], cb1[NS];
#pragma unroll
    for (int s = 0; s < NS; ++s) { cb0[s] = 0.f; cb1[s] = 0.f; }
    [[maybe_unused]] const long long n_desc = (long long)p.n_chains * p.n_chunks_t;
    if (chunk > 0 && !drop && RATP_IN(desc, 1, n_desc)) {
      unsigned long long* dst = p.ws.agg + desc * WA * kDescLanes + lane;
      put_word(dst + 0 * kDescLanes, s_tot_a[c0], tag);
      put_word(dst + 1 * kDescLanes, s_tot_a[c0 + 1], tag);
#pragma unroll
      for (int s = 0; s < NS; ++s) {
        put_word(dst + (2 + 2 * s) * kDescLanes, s_tot_b[s][c0], tag);
        put_word(dst + (3 + 2 * s) * kDescLanes, s_tot_b[s][c0 + 1], tag);
      }
    }
    // a chunk whose first token restarts the recurrence needs no carry
    const bool restart = RESET && ((long long)chunk * L) % p.reset_L == 0;
    if (chunk > 0 && !restart) {
      // composite map of the predecessors composed so far: x -> ca x + cb
      float ca0 = 1.f, ca1 = 1.f;
      int top = chunk - 1;                      // nearest predecessor not yet composed
      const unsigned long long t_start = global_ns();
      while (top >= 0) {
        // words of predecessors top and top-1, all loads issued together
        unsigned long long wi[2][WI], wa[2][WA];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const long long d = chain0 + (top - u);
          const bool exists = (top - u) >= 0 && RATP_IN(d, 1, n_desc);
#pragma unroll
          for (int w = 0; w < WI; ++w) wi[u][w] = exists ? get_word(incl + (d * WI + w) * kDescLanes + lane) : 0ull;
#pragma unroll
          for (int w = 0; w < WA; ++w) wa[u][w] = exists ? get_word(agg + (d * WA + w) * kDescLanes + lane) : 0ull;
        }
        bool inc[2], ag[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          inc[u] = true;
          ag[u] = true;
#pragma unroll
          for (int w = 0; w < WI; ++w) inc[u] = inc[u] && word_ok(wi[u][w], tag);
#pragma unroll
          for (int w = 0; w < WA; ++w) ag[u] = ag[u] && word_ok(wa[u][w], tag);
        }
        // how far this round gets: compose n aggregates, then maybe an inclusive
        int n = -1;
        bool found = false;
        if (inc[0]) { n = 0; found = true; }
        else if (ag[0]) {
          if (top >= 1 && inc[1]) { n = 1; found = true; }
          else if (top >= 1 && ag[1]) n = 2;
          else n = 1;
        }
        if (n < 0) {
          if (global_ns() - t_start > spin_timeout() || aborted()) {
            raise_error(RATP_ERR_TIMEOUT);
            atomicExch(p.ws.abort, 1u);
            ca0 = ca1 = 0.f;                     // give up: zero carry
#pragma unroll
            for (int s = 0; s < NS; ++s) { cb0[s] = 0.f; cb1[s] = 0.f; }
            break;
          }
          __nanosleep(20);
          continue;
        }
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          if (u < n) {
#pragma unroll
            for (int s = 0; s < NS; ++s) {
              cb0[s] = fmaf(ca0, word_val(wa[u][2 + 2 * s]), cb0[s]);
              cb1[s] = fmaf(ca1, word_val(wa[u][3 + 2 * s]), cb1[s]);
            }
            ca0 *= word_val(wa[u][0]);
            ca1 *= word_val(wa[u][1]);
          }
        }
        if (found) {
#pragma unroll
          for (int s = 0; s < NS; ++s) {                           // carry = composite(inclusive)
            const unsigned long long i0 = (n == 0) ? wi[0][2 * s] : wi[1][2 * s];
            const unsigned long long i1 = (n == 0) ? wi[0][2 * s + 1] : wi[1][2 * s + 1];
            cb0[s] = fmaf(ca0, word_val(i0), cb0[s]);
            cb1[s] = fmaf(ca1, word_val(i1), cb1[s]);
          }
          break;
        }
        if (RESET && ca0 == 0.f && ca1 == 0.f) break;   // composed the last restart
        top -= n;
      }
    }
    // publish the inclusive state of this chunk
    if (!drop && RATP_IN(desc, 1, n_desc)) {
      unsigned long long* dst = p.ws.incl + desc * (2 * NS) * kDescLanes + lane;
#pragma unroll
      for (int s = 0; s < NS; ++s) {
        put_word(dst + (2 * s) * kDescLanes, fmaf(s_tot_a[c0], cb0[s], s_tot_b[s][c0]), tag);
        put_word(dst + (2 * s + 1) * kDescLanes, fmaf(s_tot_a[c0 + 1], cb1[s], s_tot_b[s][c0 + 1]), tag);
      }
    }
#pragma unroll
    for (int s = 0; s < NS; ++s) {
      s_carry[s][c0] = cb0[s];
      s_carry[s][c0 + 1] = cb1[s];
    }
  }
  __syncthreads();

  // ---- recompute the tokens from the carry and store ----
  float2 hs[NS][V2];
#pragma unroll
  for (int i = 0; i < V2; ++i) {
    const int c = lane_c * V + 2 * i;
#pragma unroll
    for (int s = 0; s < NS; ++s) hs[s][i] = fma2(ea[i], make_float2(s_carry[s][c], s_carry[s][c + 1]), eb[s][i]);
  }
#pragma unroll
  for (int r = 0; r < R; ++r) {
    if (r < nrows) {
      const int t = t0 + r;
      if (RESET && ((rmask >> r) & 1u)) {
#pragma unroll
        for (int s = 0; s < NS; ++s)
#pragma unroll
          for (int i = 0; i < V2; ++i) hs[s][i] = make_float2(0.f, 0.f);
      }
      float2 gf[V2];
      Elem<T>::unpack2(*reinterpret_cast<const uint4*>(s_g + soff + r * kSlab), gf);
#pragma unroll
      for (int s = 0; s < NS; ++s) {
        float2 xf[V2];
        Elem<T>::unpack2(*reinterpret_cast<const uint4*>(s_g + (1 + s) * L * kSlab + soff + r * kSlab), xf);
#pragma unroll
        for (int i = 0; i < V2; ++i) hs[s][i] = fma2(gf[i], sub2(hs[s][i], xf[i]), xf[i]);
        const long long off = base + (long long)t * row_stride;
        if (RATP_IN(off, V, (long long)p.B * p.Tn * p.C)) {
          if (FUSED) *reinterpret_cast<uint4*>(p.h[s] + off) = Elem<T>::pack2(hs[s]);
          else __stcs(reinterpret_cast<uint4*>(p.h[s] + off), Elem<T>::pack2(hs[s]));
        }
        if (t == p.Tn - 1 && p.final_state != nullptr &&
            RATP_IN(((long long)s * p.B + b) * p.C + slab * kSlab + lane_c * V, V, (long long)NS * p.B * p.C)) {
          float* fs = p.final_state + ((long long)s * p.B + b) * p.C + slab * kSlab + lane_c * V;
#pragma unroll
          for (int i = 0; i < V2; ++i) { fs[2 * i] = hs[s][i].x; fs[2 * i + 1] = hs[s][i].y; }
        }
      }
    }
  }
  if (!FUSED) return true;

  // ---- done flag (fused prefill) ----
  // Every thread orders its stores before the attention's TMA reads (async
  // proxy); after the barrier thread 0 waits (bounded) for the predecessor's
  // flag and releases this chunk's.
  asm volatile("fence.proxy.async.global;" ::: "memory");
  __syncthreads();
  bool ok = true;
  if (tid == 0) {
    [[maybe_unused]] const long long n_desc = (long long)p.n_chains * p.n_chunks_t;
    if (chunk > 0) {
      const unsigned int* prev = p.done + desc - 1;
      const unsigned long long t_start = global_ns();
      unsigned int v = 0u;
      while (true) {
        if (RATP_IN(desc - 1, 1, n_desc))
          asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(prev) : "memory");
        if (v == tag) break;
        if (global_ns() - t_start > spin_timeout() || aborted()) {
          raise_error(RATP_ERR_TIMEOUT);
          atomicExch(p.ws.abort, 1u);
          ok = false;
          break;
        }
        __nanosleep(32);
      }
    }
    if (ok && desc != g_fault_fused_chunk && RATP_IN(desc, 1, n_desc)) {   // else: planted failure
      __threadfence();
      asm volatile("st.release.gpu.global.u32 [%0], %1;" :: "l"(p.done + desc), "r"(tag) : "memory");
    }
  }
  return __syncthreads_and(ok) != 0;
}

template <typename T, int NS, int R = kRows, bool RESET = false>
__global__ void __launch_bounds__(kThreads, 2)
scan_kernel(const __grid_constant__ CUtensorMap tm_g, const __grid_constant__ CUtensorMap tm_x0,
            const __grid_constant__ CUtensorMap tm_x1, const __grid_constant__ Params<T, NS> p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
  __shared__ __align__(8) uint64_t s_bar;
  __shared__ unsigned int s_ticket, s_tag;
  const uint32_t bar = sm100::smem_u32(&s_bar);
  if (threadIdx.x == 0) {
    unsigned int tk;
    s_tag = draw_ticket(p.ws, (unsigned int)(p.n_chains * p.n_chunks_t), &tk);
    s_ticket = tk;
    sm100::mbar_init(bar, 1);
    sm100::fence_barrier_init();
  }
  __syncthreads();
  // one chunk per CTA; after a failed wait, the copies still in flight land
  // (bounded) before the CTA's shared memory is released
  if (!scan_chunk<T, NS, R, RESET, false>(tm_g, tm_x0, tm_x1, p, smem, bar, 0u, s_ticket, s_tag) &&
      threadIdx.x == 0) {
    const unsigned long long t1 = global_ns();
    while (!sm100::mbar_try_wait(bar, 0) && global_ns() - t1 < spin_timeout()) {}
  }
}

}  // namespace scan
}  // namespace ratp
