// fused.cuh -- the recurrence side of the fused prefill: scan warps that run
// inside the attention kernel, ahead of its tensor-core pipeline.
//
// The forget-gate recurrence h_t = g_t * h_{t-1} + (1 - g_t) * x_t over the
// key and value streams (zhichai.net "RAT+ 深度拆解", section 2.1: the
// full-sequence recurrence whose keys and values the dilated attention of
// section 1 reads) is computed unit by unit.  A unit is one (b, h) and the
// 128 positions of one work item of the attention kernel (a 128-query tile),
// all 128 channels of the head, both streams with one gate.  Two warps scan a
// unit: warp w takes positions 64w .. 64w+63 of it, lane l channels
// 4l .. 4l+3 (8-byte loads of bf16).
//   pass 1  each warp reduces its 64 positions to one affine map per channel
//           (h -> a h + b, a = prod g); warp 1 composes the unit's map;
//   publish warp 1 writes the unit's map as tagged 64-bit words (the launch
//           tag in the high half, the fp32 value in the low half: a word that
//           carries the current tag is this launch's value, with no flag);
//   carry   warp 1 walks back over the unit's predecessors of the same (b, h),
//           composing their maps until it meets an inclusive state (a
//           decoupled look-back), then publishes the unit's inclusive state;
//   pass 2  each warp runs its positions again from its carry and stores
//           h_k, h_v (bf16) and, at position T-1, the fp32 final state;
//   done    after a proxy fence (the attention reads h_k/h_v with TMA) and a
//           release store, the unit's flag holds the launch tag.
// The attention producer acquires the flags of every unit its item reads
// before it loads a key tile.  Every wait is bounded.
#pragma once
#include "common.cuh"

namespace ratp {
namespace fused {

constexpr int kUnit = 128;            // positions per unit (one attention work item)
constexpr int kHalfUnit = 64;         // positions per scan warp
constexpr int kAggWords = 12;         // per lane: a, b_k, b_v of 4 channels
constexpr int kInclWords = 8;         // per lane: h_k, h_v of 4 channels
constexpr int kBatch = 4;             // positions in flight per lane (loads issued together)

// Workspace layout (bytes), n_units = B * H * ceil(T / 128):
//   [0, 256)       header: ticket word (u64 at byte 0, launch tag in the high
//                  32 bits, CTA counter in the low 32), kept across launches;
//                  abort word (u32 at byte 128), zeroed before each launch
//   flags  u32 [n_units]                unit done (holds the launch tag)
//   agg    u64 [n_units][12][32]        aggregate map words, lane-minor
//   incl   u64 [n_units][8][32]         inclusive-state words, lane-minor
struct Workspace {
  unsigned long long* ticket;
  unsigned int* abort;
  unsigned int* flags;
  unsigned long long* agg;
  unsigned long long* incl;
};

__host__ __device__ inline size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

inline size_t workspace_bytes(long long n_units) {
  return 256 + align256(4 * (size_t)n_units) + align256(8 * (size_t)n_units * kAggWords * 32) +
         align256(8 * (size_t)n_units * kInclWords * 32);
}

inline Workspace carve(void* base, long long n_units) {
  char* p = static_cast<char*>(base);
  Workspace w;
  w.ticket = reinterpret_cast<unsigned long long*>(p);
  w.abort = reinterpret_cast<unsigned int*>(p + 128);
  p += 256;
  w.flags = reinterpret_cast<unsigned int*>(p);
  p += align256(4 * (size_t)n_units);
  w.agg = reinterpret_cast<unsigned long long*>(p);
  p += align256(8 * (size_t)n_units * kAggWords * 32);
  w.incl = reinterpret_cast<unsigned long long*>(p);
  return w;
}
constexpr size_t kResetOffset = 128, kResetBytes = 64;   // the abort word

struct ScanParams {
  const __nv_bfloat16* xk;
  const __nv_bfloat16* xv;
  const __nv_bfloat16* g;
  __nv_bfloat16* hk;
  __nv_bfloat16* hv;
  float* final_state;     // nullable: [2][B][H][128]
  Workspace ws;
  int NQ;                 // units per (b, h)
};

// ---- tagged words and flags ---------------------------------------------------
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
__device__ __forceinline__ float word_val(unsigned long long w) { return __uint_as_float((unsigned int)w); }

__device__ __forceinline__ unsigned int ld_acquire(const unsigned int* p) {
  unsigned int v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_release(unsigned int* p, unsigned int v) {
  asm volatile("st.release.gpu.global.u32 [%0], %1;" :: "l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ unsigned int ld_relaxed(const unsigned int* p) {
  unsigned int v;
  asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
// Orders this thread's generic-proxy memory accesses with its later
// async-proxy (TMA) ones, and the reverse.
__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

// Every CTA of a launch calls this once (one thread): returns the launch tag
// (1, 2, ..., 2^32-1, 1, ...).  The last CTA to arrive stores the next tag and
// a zero counter; every other CTA's add precedes that store in the word's
// order, so all of them read the same stored tag.
__device__ __forceinline__ unsigned int draw_tag(const Workspace& ws, unsigned int n_ctas) {
  unsigned long long old;
  asm volatile("atom.relaxed.gpu.global.add.u64 %0, [%1], 1;" : "=l"(old) : "l"(ws.ticket) : "memory");
  const unsigned int stored = (unsigned int)(old >> 32);
  const unsigned int tag = stored == 0xffffffffu ? 1u : stored + 1u;
  if ((unsigned int)old == n_ctas - 1u)
    asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" :: "l"(ws.ticket), "l"((unsigned long long)tag << 32)
                 : "memory");
  return tag;
}

__device__ __forceinline__ bool aborted(const Workspace& ws) { return ld_relaxed(ws.abort) != 0u; }
__device__ __forceinline__ void abort_all(const Workspace& ws) {
  raise_error(RATP_ERR_TIMEOUT);
  atomicExch(ws.abort, 1u);
}

// ---- the unit scan ----------------------------------------------------------
// 4 channels of bf16 in 8 bytes <-> two fp32 pairs
__device__ __forceinline__ void unpack4(uint2 v, float2& lo, float2& hi) {
  lo = make_float2(__uint_as_float(v.x << 16), __uint_as_float(v.x & 0xffff0000u));
  hi = make_float2(__uint_as_float(v.y << 16), __uint_as_float(v.y & 0xffff0000u));
}
__device__ __forceinline__ uint2 pack4(float2 lo, float2 hi) {
  return make_uint2(pack_bf16x2(lo.x, lo.y), pack_bf16x2(hi.x, hi.y));
}
__device__ __forceinline__ uint2 ld_nc8(const __nv_bfloat16* p) {
  uint2 v;
  asm volatile("ld.global.nc.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "l"(p));
  return v;
}

// Scans unit (b, h, u) with the two scan warps (sw = 0, 1 in the caller's
// numbering, 64 threads); bar_id names the barrier the two warps share.
// s_map: shared scratch of 20 floats per lane (640 floats): warp 0's map,
// then the unit's carry.
// Returns false if a wait ran out (the kernel-wide abort word is then set).
__device__ __forceinline__ bool scan_unit(const ScanParams& p, int B, int T, int H, int b, int h, int u,
                                          int sw, int lane, unsigned int tag, float* s_map, int bar_id) {
  const int p0 = u * kUnit + sw * kHalfUnit;           // first position of this warp
  const int p1 = min(p0 + kHalfUnit, T);               // end (exclusive)
  const long long row = (long long)H * 128;            // elements per position
  const long long off = ((long long)b * T) * row + (long long)h * 128 + 4 * lane;
  const long long unit = ((long long)b * H + h) * p.NQ + u;
  [[maybe_unused]] const long long n_el = (long long)B * T * row;

  // ---- pass 1: this warp's map over its positions ----
  float2 a[2] = {make_float2(1.f, 1.f), make_float2(1.f, 1.f)};
  float2 bk[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
  float2 bv[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
  for (int t = p0; t < p1; t += kBatch) {
    uint2 G[kBatch], XK[kBatch], XV[kBatch];
#pragma unroll
    for (int i = 0; i < kBatch; ++i) {
      if (t + i < p1 && RATP_IN(off + (long long)(t + i) * row, 4, n_el)) {
        const long long o = off + (long long)(t + i) * row;
        G[i] = ld_nc8(p.g + o);
        XK[i] = ld_nc8(p.xk + o);
        XV[i] = ld_nc8(p.xv + o);
      }
    }
#pragma unroll
    for (int i = 0; i < kBatch; ++i) {
      if (t + i < p1) {
        float2 g2[2], k2[2], v2[2];
        unpack4(G[i], g2[0], g2[1]);
        unpack4(XK[i], k2[0], k2[1]);
        unpack4(XV[i], v2[0], v2[1]);
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          bk[c] = fma2(g2[c], sub2(bk[c], k2[c]), k2[c]);
          bv[c] = fma2(g2[c], sub2(bv[c], v2[c]), v2[c]);
          a[c] = mul2(a[c], g2[c]);
        }
      }
    }
  }

  // ---- the unit's map: warp 1's map applied after warp 0's ----
  float* m0 = s_map + lane;                            // warp 0's map, 12 floats strided by 32
  if (sw == 0) {
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      m0[(4 * c + 0) * 32] = a[c].x;  m0[(4 * c + 1) * 32] = a[c].y;
      m0[(4 * c + 2) * 32] = bk[c].x; m0[(4 * c + 3) * 32] = bk[c].y;
      m0[(8 + 2 * c) * 32] = bv[c].x; m0[(9 + 2 * c) * 32] = bv[c].y;
    }
  }
  asm volatile("bar.sync %0, 64;" :: "r"(bar_id) : "memory");
  float2 a0[2], bk0[2], bv0[2];
#pragma unroll
  for (int c = 0; c < 2; ++c) {
    a0[c] = make_float2(m0[(4 * c + 0) * 32], m0[(4 * c + 1) * 32]);
    bk0[c] = make_float2(m0[(4 * c + 2) * 32], m0[(4 * c + 3) * 32]);
    bv0[c] = make_float2(m0[(8 + 2 * c) * 32], m0[(9 + 2 * c) * 32]);
  }
  bool ok = true;
  float* cs = s_map + 12 * 32 + lane;                  // carry into the unit: 8 floats strided by 32
  if (sw == 1) {
    // unit map U = (a1 a0, a1 b0 + b1)
    float ua[4], uk[4], uv[4];
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      const float2 ta = mul2(a[c], a0[c]);
      const float2 tk = fma2(a[c], bk0[c], bk[c]);
      const float2 tv = fma2(a[c], bv0[c], bv[c]);
      ua[2 * c] = ta.x; ua[2 * c + 1] = ta.y;
      uk[2 * c] = tk.x; uk[2 * c + 1] = tk.y;
      uv[2 * c] = tv.x; uv[2 * c + 1] = tv.y;
    }
    [[maybe_unused]] const long long n_units = (long long)B * H * p.NQ;
    if (u > 0 && RATP_IN(unit, 1, n_units)) {
      unsigned long long* dst = p.ws.agg + unit * kAggWords * 32 + lane;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        put_word(dst + (0 + c) * 32, ua[c], tag);
        put_word(dst + (4 + c) * 32, uk[c], tag);
        put_word(dst + (8 + c) * 32, uv[c], tag);
      }
    }
    // look back: carry = A_{u-1}(A_{u-2}(... (inclusive state of some j)))
    float ca[4] = {1.f, 1.f, 1.f, 1.f}, ck[4] = {0.f, 0.f, 0.f, 0.f}, cv[4] = {0.f, 0.f, 0.f, 0.f};
    int j = u - 1;
    const unsigned long long t_start = global_ns();
    unsigned int polls = 0;
    while (j >= 0) {
      const long long d = unit - (u - j);
      if (!RATP_IN(d, 1, n_units)) break;
      unsigned long long wi[kInclWords];
#pragma unroll
      for (int w = 0; w < kInclWords; ++w) wi[w] = get_word(p.ws.incl + (d * kInclWords + w) * 32 + lane);
      bool inc = true;
#pragma unroll
      for (int w = 0; w < kInclWords; ++w) inc = inc && word_ok(wi[w], tag);
      if (inc) {
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          ck[c] = fmaf(ca[c], word_val(wi[c]), ck[c]);
          cv[c] = fmaf(ca[c], word_val(wi[4 + c]), cv[c]);
        }
        break;
      }
      unsigned long long wa[kAggWords];
#pragma unroll
      for (int w = 0; w < kAggWords; ++w) wa[w] = get_word(p.ws.agg + (d * kAggWords + w) * 32 + lane);
      bool ag = j > 0;        // unit 0 of a chain publishes no aggregate (its inclusive state is its map)
#pragma unroll
      for (int w = 0; w < kAggWords; ++w) ag = ag && word_ok(wa[w], tag);
      if (ag) {
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          ck[c] = fmaf(ca[c], word_val(wa[4 + c]), ck[c]);
          cv[c] = fmaf(ca[c], word_val(wa[8 + c]), cv[c]);
          ca[c] *= word_val(wa[c]);
        }
        --j;
        continue;
      }
      if ((++polls & 15u) == 0u && (global_ns() - t_start > spin_timeout() || aborted(p.ws))) {
        abort_all(p.ws);
        ok = false;
#pragma unroll
        for (int c = 0; c < 4; ++c) { ck[c] = 0.f; cv[c] = 0.f; }   // give up: zero carry
        break;
      }
      __nanosleep(20);
    }
    // inclusive state of the unit = U(carry)
    if (RATP_IN(unit, 1, n_units)) {
      unsigned long long* dst = p.ws.incl + unit * kInclWords * 32 + lane;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        put_word(dst + c * 32, fmaf(ua[c], ck[c], uk[c]), tag);
        put_word(dst + (4 + c) * 32, fmaf(ua[c], cv[c], uv[c]), tag);
      }
    }
#pragma unroll
    for (int c = 0; c < 4; ++c) { cs[c * 32] = ck[c]; cs[(4 + c) * 32] = cv[c]; }
  }
  asm volatile("bar.sync %0, 64;" :: "r"(bar_id) : "memory");

  // ---- pass 2: positions again from the carry; store h_k, h_v ----
  float2 hk2[2], hv2[2];
#pragma unroll
  for (int c = 0; c < 2; ++c) {
    const float2 ck = make_float2(cs[(2 * c) * 32], cs[(2 * c + 1) * 32]);
    const float2 cv = make_float2(cs[(4 + 2 * c) * 32], cs[(5 + 2 * c) * 32]);
    if (sw == 0) {
      hk2[c] = ck;
      hv2[c] = cv;
    } else {                                           // warp 1 starts after warp 0's positions
      hk2[c] = fma2(a0[c], ck, bk0[c]);
      hv2[c] = fma2(a0[c], cv, bv0[c]);
    }
  }
  for (int t = p0; t < p1; t += kBatch) {
    uint2 G[kBatch], XK[kBatch], XV[kBatch];
#pragma unroll
    for (int i = 0; i < kBatch; ++i) {
      if (t + i < p1 && RATP_IN(off + (long long)(t + i) * row, 4, n_el)) {
        const long long o = off + (long long)(t + i) * row;
        G[i] = ld_nc8(p.g + o);
        XK[i] = ld_nc8(p.xk + o);
        XV[i] = ld_nc8(p.xv + o);
      }
    }
#pragma unroll
    for (int i = 0; i < kBatch; ++i) {
      if (t + i < p1) {
        float2 g2[2], k2[2], v2[2];
        unpack4(G[i], g2[0], g2[1]);
        unpack4(XK[i], k2[0], k2[1]);
        unpack4(XV[i], v2[0], v2[1]);
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          hk2[c] = fma2(g2[c], sub2(hk2[c], k2[c]), k2[c]);
          hv2[c] = fma2(g2[c], sub2(hv2[c], v2[c]), v2[c]);
        }
        const long long o = off + (long long)(t + i) * row;
        if (RATP_IN(o, 4, n_el)) {
          *reinterpret_cast<uint2*>(p.hk + o) = pack4(hk2[0], hk2[1]);
          *reinterpret_cast<uint2*>(p.hv + o) = pack4(hv2[0], hv2[1]);
        }
        if (t + i == T - 1 && p.final_state != nullptr) {
          const long long fo = ((long long)b * H + h) * 128 + 4 * lane;
          const long long fn = 2ll * B * H * 128;
          if (RATP_IN(fo, 4, fn) && RATP_IN(fn / 2 + fo, 4, fn)) {
            *reinterpret_cast<float4*>(p.final_state + fo) = make_float4(hk2[0].x, hk2[0].y, hk2[1].x, hk2[1].y);
            *reinterpret_cast<float4*>(p.final_state + fn / 2 + fo) =
                make_float4(hv2[0].x, hv2[0].y, hv2[1].x, hv2[1].y);
          }
        }
      }
    }
  }
  // publish: the stores above are visible to the TMA loads of any CTA that
  // acquires the flag
  fence_proxy_async_global();
  __threadfence();
  asm volatile("bar.sync %0, 64;" :: "r"(bar_id) : "memory");
  if (sw == 0 && lane == 0 && unit != g_fault_fused_unit && RATP_IN(unit, 1, (long long)B * H * p.NQ))
    st_release(p.ws.flags + unit, tag);
  return ok;
}

}  // namespace fused
}  // namespace ratp
