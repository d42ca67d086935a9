// decode.cuh -- D-compressed KV cache: prefill hand-off and the fused decode
// step (RAT+ abstract: the KV cache shrinks by the dilation D; write-up
// section 2.1: the recurrence is a one-step state update at decode; write-up
// section 6: dense heads).
//
// Decode step for token t = len[b] of every sequence, one launch:
//   grid: one CTA per (b, h, split).  The keys of (b, h) form a virtual list: the cached
//   dilated slots whose positions lie before the window, s < (t-W+1) / D_h
//   (all s < t / D_h without a window; Kc/Vc rows), then every window position
//   t-W < p < t (ring rows), so each key appears once.  Split i streams keys
//   [i*split_keys, (i+1)*split_keys) with 16-byte loads, a half-warp per key
//   (Dh = 128) and an fp32 online softmax per half-warp.
//   Split 0 additionally performs the recurrence step for the k and v streams
//   (fp32 state, in place; with a chunk-local recurrence of block reset_L the
//   state is taken as zero at t mod reset_L == 0), appends the bf16-rounded new key/value to Kc/Vc
//   when t mod D_h = D_h-1, writes it into ring row t mod W, and attends to it
//   (the query's own key).  None of these rows is read by any CTA of the
//   same step, so there is no intra-step race.
//   Splits publish (m, l, acc) partials; the last split of (b, h) to finish
//   (atomic counter) merges them and writes o.  The last CTA of batch item b
//   advances len[b].  Counters return to zero, so no per-step reset is needed.
#pragma once
#include "common.cuh"

namespace ratp {
namespace decode {

constexpr int kThreads = 128;
// cached rows per split warmed into L2 before the step waits for the previous
// kernel (measured per step: 32 rows 58.0 / 31.5 us, 64 rows 57.5 / 31.5 us,
// 128 rows 58.2 / 33.1 us, none 59.1 / 32.5 us for the 32K-context and the
// hybrid decode)
constexpr int kPrefetchRows = 64;

// L2 prefetch of `bytes` (a multiple of 16) at a 16-byte aligned address
__device__ __forceinline__ void bulk_prefetch_l2(const void* ptr, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" :: "l"(ptr), "r"(bytes) : "memory");
}

struct Params {
  const __nv_bfloat16* q;
  const __nv_bfloat16* xk;
  const __nv_bfloat16* xv;
  const __nv_bfloat16* g;
  __nv_bfloat16* o;
  float* state;                 // [2][B][H][Dh]
  __nv_bfloat16* Kc;
  __nv_bfloat16* Vc;
  __nv_bfloat16* Kw;
  __nv_bfloat16* Vw;
  int32_t* len;
  float* partial;               // [B][H][max_splits][Dh + 2]
  uint32_t* counters;           // [B*H] per (b, h), then [B] per batch item
  long long rows_per_b;
  int B, H, D, W, T_max, split_keys, max_splits;
  int reset_L;                  // chunk-local recurrence: state restarts at t mod reset_L == 0; 0 = never
  int window_L;                 // fixed look-back window (0 = none); inputs ring in in_ring
  __nv_bfloat16* in_ring;       // [3][B][H][window_L][DH]: x_k, x_v, g of the last window_L positions
  float scale_log2;
  int splits_per_b;             // CTAs per batch item: sum over heads of split_base
  int split_base[RATP_MAX_HEADS + 1];   // first CTA (within a batch item) of each head
  unsigned long long dense_bits[RATP_MAX_HEADS / 64];
};

__device__ __forceinline__ bool is_dense(const unsigned long long* bits, int h) {
  return (bits[h >> 6] >> (h & 63)) & 1ull;
}

// Row offset of head h inside one batch item: sum of capacities of heads < h.
__device__ __forceinline__ long long head_offset(const unsigned long long* bits, int h,
                                                 int T_max, int D) {
  int nd = 0;
  for (int w = 0; w < (h >> 6); ++w) nd += __popcll(bits[w]);
  if (h & 63) nd += __popcll(bits[h >> 6] & ((1ull << (h & 63)) - 1ull));
  return (long long)nd * T_max + (long long)(h - nd) * (T_max / D);
}

template <int DH>
__global__ void __launch_bounds__(kThreads, 7)
decode_kernel(const Params p) {
  constexpr int LPK = DH / 8;                    // lanes per key (8 bf16 per lane)
  constexpr int KPW = 32 / LPK;                  // keys per warp per step
  constexpr int NG = (kThreads / 32) * KPW;      // key groups per CTA
  constexpr int UNROLL = 4;

  __shared__ float s_self_k[DH], s_self_v[DH];
  __shared__ float s_m[NG], s_l[NG];
  __shared__ float s_acc[NG][DH];
  __shared__ int s_last;

  // 1-D grid: batch item, then head (each head gets the splits its largest
  // key count can need), then split
  const int b = blockIdx.x / p.splits_per_b;
  const int rem = blockIdx.x - b * p.splits_per_b;
  int h = 0;
  {
    int lo = 0, hi = p.H - 1;                    // last head with split_base[h] <= rem
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (p.split_base[mid] <= rem) lo = mid; else hi = mid - 1;
    }
    h = lo;
  }
  const int split = rem - p.split_base[h];
  const int tid = threadIdx.x;

  // Launched as a programmatic dependent of the previous kernel in the
  // stream: let the next step be scheduled now.  Before waiting for the
  // previous kernel, warm L2 with the first cached rows of this split's range:
  // they depend on nothing that kernel writes (a row it may append is read
  // after the wait, from L2 or memory as it then stands; a prefetch returns no
  // data), so their fetch overlaps the previous step's tail.  Then wait until
  // everything before this step has completed and is visible.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  if (tid == 0) {
    const int cap = is_dense(p.dense_bits, h) ? p.T_max : p.T_max / p.D;
    const int first = split * p.split_keys;
    const int n = min(kPrefetchRows, cap - first);
    const long long row = (long long)b * p.rows_per_b + head_offset(p.dense_bits, h, p.T_max, p.D) + first;
    if (n > 0 && RATP_IN(row * DH, (long long)n * DH, (long long)p.B * p.rows_per_b * DH)) {
      bulk_prefetch_l2(p.Kc + row * DH, (uint32_t)n * DH * 2);
      bulk_prefetch_l2(p.Vc + row * DH, (uint32_t)n * DH * 2);
    }
  }
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int t = p.len[b];
  const bool dense = is_dense(p.dense_bits, h);
  const int Dd = dense ? 1 : p.D;
  bool active = true;
  int n_slots = 0, w_lo = 0, n_win = 0, n_keys = 0, n_used = 1, app_slot = 0;
  if (t >= p.T_max) {
    active = false;
    if (split == 0 && h == 0 && tid == 0) raise_error(RATP_ERR_CAPACITY);
  } else {
    app_slot = t / Dd;                           // slot of position t if it is a dilated one
    n_slots = app_slot;
    if (p.W > 0 && !dense) {
      w_lo = max(0, t - p.W + 1);
      n_win = t - w_lo;
      n_slots = w_lo / Dd;                       // dilated slots before the window
    }
    n_keys = n_slots + n_win;
    n_used = max(1, (n_keys + p.split_keys - 1) / p.split_keys);
    if (split >= n_used) active = false;
  }

  if (active) {
    const long long bh = (long long)b * p.H + h;
    [[maybe_unused]] const long long n_tok = (long long)p.B * p.H * DH;              // q, x, g, o elements
    [[maybe_unused]] const long long n_dil = (long long)p.B * p.rows_per_b * DH;     // Kc / Vc elements
    [[maybe_unused]] const long long n_ring = (long long)p.B * p.H * p.W * DH;       // Kw / Vw elements
    const __nv_bfloat16* qrow = p.q + bh * DH;
    const long long cache_row0 = (long long)b * p.rows_per_b + head_offset(p.dense_bits, h, p.T_max, p.D);

    // ---- split 0: recurrence step, append, ring write, self key ----
    if (split == 0) {
      const int WL = p.window_L;
      [[maybe_unused]] const long long n_in = 3ll * p.B * p.H * (long long)WL * DH;    // input-ring elements
      if (WL > 0) {
        // this step's inputs into slot t mod WL; the window is then
        // positions max(0, t - WL + 1) .. t of the ring
        for (int c = tid; c < 3 * DH; c += kThreads) {
          const int s3 = c / DH, ch = c % DH;
          const __nv_bfloat16* src = (s3 == 0 ? p.xk : s3 == 1 ? p.xv : p.g) + bh * DH + ch;
          const long long dst = (((long long)s3 * p.B * p.H + bh) * WL + t % WL) * DH + ch;
          if (RATP_IN(dst, 1, n_in) && RATP_IN(bh * DH + ch, 1, n_tok)) p.in_ring[dst] = *src;
        }
        __syncthreads();
      }
      for (int c = tid; c < 2 * DH; c += kThreads) {
        const int s = c / DH, ch = c % DH;
        if (!RATP_IN(((long long)s * p.B * p.H + bh) * DH + ch, 1, 2 * n_tok) ||
            !RATP_IN(bh * DH + ch, 1, n_tok)) continue;
        float* st = p.state + ((long long)s * p.B * p.H + bh) * DH + ch;
        const float x = __bfloat162float((s == 0 ? p.xk : p.xv)[bh * DH + ch]);
        const float gg = __bfloat162float(p.g[bh * DH + ch]);
        float hn;
        if (WL > 0) {
          // fixed look-back: the recurrence from zero over the window
          const __nv_bfloat16* rx = p.in_ring + ((long long)s * p.B * p.H + bh) * WL * DH + ch;
          const __nv_bfloat16* rg = p.in_ring + ((long long)2 * p.B * p.H + bh) * WL * DH + ch;
          float acc_h = 0.f;
          const int j0 = max(0, t - WL + 1);
          if (!RATP_IN(((long long)2 * p.B * p.H + bh) * WL * DH, (long long)WL * DH, n_in)) continue;
#pragma unroll 4
          for (int j = j0; j <= t; ++j) {
            const int slot = j % WL;
            const float gj = __bfloat162float(rg[(long long)slot * DH]);
            const float xj = __bfloat162float(rx[(long long)slot * DH]);
            acc_h = fmaf(gj, acc_h - xj, xj);
          }
          hn = acc_h;
        } else {
          const float prev = (p.reset_L > 0 && t % p.reset_L == 0) ? 0.f : *st;
          hn = fmaf(gg, prev - x, x);
        }
        *st = hn;
        const __nv_bfloat16 hb = __float2bfloat16_rn(hn);
        (s == 0 ? s_self_k : s_self_v)[ch] = __bfloat162float(hb);
        if (t % Dd == Dd - 1 && app_slot < p.T_max / Dd && RATP_IN((cache_row0 + app_slot) * DH + ch, 1, n_dil))
          (s == 0 ? p.Kc : p.Vc)[(cache_row0 + app_slot) * DH + ch] = hb;
        if (p.W > 0 && RATP_IN((bh * p.W + t % p.W) * DH + ch, 1, n_ring))
          (s == 0 ? p.Kw : p.Vw)[(bh * p.W + t % p.W) * DH + ch] = hb;
      }
      if (t % Dd == Dd - 1 && app_slot >= p.T_max / Dd && tid == 0) raise_error(RATP_ERR_CAPACITY);
      __syncthreads();
    }

    // ---- stream this split's keys ----
    const int warp = tid >> 5, lane = tid & 31;
    const int sub = lane / LPK, li = lane % LPK;
    const int grp = warp * KPW + sub;
    const unsigned int sub_mask = (LPK == 32) ? 0xffffffffu : (((1u << LPK) - 1u) << (sub * LPK));
    float qf[8];
    {
      const uint4 qv = RATP_IN(bh * DH + li * 8, 8, n_tok) ? *reinterpret_cast<const uint4*>(qrow + li * 8)
                                                             : make_uint4(0u, 0u, 0u, 0u);
      Elem<__nv_bfloat16>::unpack(qv, qf);
#pragma unroll
      for (int i = 0; i < 8; ++i) qf[i] *= p.scale_log2;
    }
    float m = -INFINITY, l = 0.f, acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.f;

    const int k_begin = split * p.split_keys;
    const int k_end = min(n_keys, k_begin + p.split_keys);
    for (int k0 = k_begin + grp; k0 < k_end; k0 += NG * UNROLL) {
      uint4 kv[UNROLL], vv[UNROLL];
      bool use[UNROLL];
#pragma unroll
      for (int u = 0; u < UNROLL; ++u) {
        const int k = k0 + u * NG;
        use[u] = false;
        if (k < k_end) {
          const __nv_bfloat16 *kr, *vr;
          if (k < n_slots) {
            kr = p.Kc + (cache_row0 + k) * DH;
            vr = p.Vc + (cache_row0 + k) * DH;
            use[u] = RATP_IN((cache_row0 + k) * DH, DH, n_dil);
          } else {
            const int pos = w_lo + (k - n_slots);
            const long long rr = (bh * p.W + pos % p.W) * DH;
            kr = p.Kw + rr;
            vr = p.Vw + rr;
            use[u] = RATP_IN(rr, DH, n_ring);
          }
          if (use[u]) {
            kv[u] = __ldcs(reinterpret_cast<const uint4*>(kr + li * 8));
            vv[u] = __ldcs(reinterpret_cast<const uint4*>(vr + li * 8));
          }
        }
      }
      // scores of the block's keys, then one max and one rescale per block
      float sc_[UNROLL];
      float m_blk = m;
#pragma unroll
      for (int u = 0; u < UNROLL; ++u) {
        float kf[8];
        Elem<__nv_bfloat16>::unpack(kv[u], kf);
        float s = 0.f;
#pragma unroll
        for (int i = 0; i < 8; ++i) s = fmaf(qf[i], kf[i], s);
#pragma unroll
        for (int off = LPK / 2; off > 0; off >>= 1) s += __shfl_xor_sync(sub_mask, s, off, LPK);
        sc_[u] = use[u] ? s : -INFINITY;
        m_blk = fmaxf(m_blk, sc_[u]);
      }
      if (m_blk != -INFINITY) {
        const float alpha = exp2f(m - m_blk);      // m = -inf on the first block: alpha = 0
        l *= alpha;
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] *= alpha;
        m = m_blk;
#pragma unroll
        for (int u = 0; u < UNROLL; ++u) {
          if (use[u]) {
            float vf[8];
            Elem<__nv_bfloat16>::unpack(vv[u], vf);
            const float pj = exp2f(sc_[u] - m);
            l += pj;
#pragma unroll
            for (int i = 0; i < 8; ++i) acc[i] = fmaf(pj, vf[i], acc[i]);
          }
        }
      }
    }
    // the query's own key, once, in group 0 of split 0
    if (split == 0 && grp == 0) {
      float s = 0.f;
#pragma unroll
      for (int i = 0; i < 8; ++i) s = fmaf(qf[i], s_self_k[li * 8 + i], s);
#pragma unroll
      for (int off = LPK / 2; off > 0; off >>= 1) s += __shfl_xor_sync(sub_mask, s, off, LPK);
      const float m_new = fmaxf(m, s);
      const float alpha = exp2f(m - m_new);
      const float pj = exp2f(s - m_new);
      l = l * alpha + pj;
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] = fmaf(acc[i], alpha, pj * s_self_v[li * 8 + i]);
      m = m_new;
    }
    // ---- merge the key groups of this CTA ----
    if (li == 0) { s_m[grp] = m; s_l[grp] = l; }
#pragma unroll
    for (int i = 0; i < 8; ++i) s_acc[grp][li * 8 + i] = acc[i];
    __syncthreads();
    float M = -INFINITY;
#pragma unroll
    for (int gi = 0; gi < NG; ++gi) M = fmaxf(M, s_m[gi]);
    const bool single = (n_used == 1);
    [[maybe_unused]] const long long n_part = (long long)p.B * p.H * p.max_splits * (DH + 2);
    const bool part_ok = single || RATP_IN((bh * p.max_splits + split) * (DH + 2), DH + 2, n_part);
    float* part = p.partial + (bh * p.max_splits + split) * (DH + 2);
    for (int c = tid; c < DH; c += kThreads) {
      float L = 0.f, A = 0.f;
#pragma unroll
      for (int gi = 0; gi < NG; ++gi) {
        const float w = (s_m[gi] == -INFINITY) ? 0.f : exp2f(s_m[gi] - M);
        L = fmaf(s_l[gi], w, L);
        A = fmaf(s_acc[gi][c], w, A);
      }
      if (single) {
        if (RATP_IN(bh * DH + c, 1, n_tok)) p.o[bh * DH + c] = __float2bfloat16_rn(A / L);
      } else if (part_ok) {
        __stcg(part + 2 + c, A);
        if (c == 0) { __stcg(part, M); __stcg(part + 1, L); }
      }
    }
    if (!single) {
      __threadfence();
      __syncthreads();
      if (tid == 0) {
        const unsigned int prev = atomicAdd(p.counters + bh, 1u);
        s_last = (prev == (unsigned int)(n_used - 1));
      }
      __syncthreads();
      if (s_last) {
        __threadfence();
        const float* pb = p.partial + bh * p.max_splits * (DH + 2);
        const bool pb_ok = RATP_IN(bh * p.max_splits * (DH + 2), (long long)n_used * (DH + 2), n_part);
        float MM = -INFINITY;
        for (int i = 0; i < n_used; ++i) MM = fmaxf(MM, __ldcg(pb + i * (DH + 2)));
        for (int c = tid; pb_ok && c < DH; c += kThreads) {
          float L = 0.f, A = 0.f;
          for (int i = 0; i < n_used; ++i) {
            const float mi = __ldcg(pb + i * (DH + 2));
            const float w = (mi == -INFINITY) ? 0.f : exp2f(mi - MM);
            L = fmaf(__ldcg(pb + i * (DH + 2) + 1), w, L);
            A = fmaf(__ldcg(pb + i * (DH + 2) + 2 + c), w, A);
          }
          if (RATP_IN(bh * DH + c, 1, n_tok)) p.o[bh * DH + c] = __float2bfloat16_rn(A / L);
        }
        if (tid == 0) p.counters[bh] = 0u;
      }
    }
  }

  // ---- the last CTA of batch item b advances len[b] ----
  // (one counter per batch item, so the step's closing atomics spread over
  // B addresses instead of one)
  __syncthreads();
  if (tid == 0) {
    __threadfence();
    uint32_t* cnt = p.counters + (long long)p.B * p.H + b;
    const unsigned int prev = atomicAdd(cnt, 1u);
    if (prev == (unsigned int)p.splits_per_b - 1u) {
      __threadfence();
      const int tb = p.len[b];
      if (tb < p.T_max) p.len[b] = tb + 1;
      *cnt = 0u;
      __threadfence();
    }
  }
}

// ---- prefill -> cache hand-off --------------------------------------------
struct PackParams {
  const __nv_bfloat16* hk;
  const __nv_bfloat16* hv;
  __nv_bfloat16* Kc;
  __nv_bfloat16* Vc;
  __nv_bfloat16* Kw;
  __nv_bfloat16* Vw;
  int32_t* len;
  long long rows_per_b;
  int B, T, H, D, W, T_max;
  unsigned long long dense_bits[RATP_MAX_HEADS / 64];
};

// grid (ceil(rows / rows_per_block), H, B); Dh/8 threads per row, 16 B each.
template <int DH>
__global__ void __launch_bounds__(256)
pack_kernel(const PackParams p) {
  constexpr int TPR = DH / 8;
  constexpr int RPB = 256 / TPR;
  const int h = blockIdx.y, b = blockIdx.z;
  const int r = blockIdx.x * RPB + threadIdx.x / TPR;
  const int li = threadIdx.x % TPR;
  const bool dense = is_dense(p.dense_bits, h);
  const int Dd = dense ? 1 : p.D;
  const int n_dil = p.T / Dd;
  const int w_lo = max(0, p.T - p.W);
  const int n_ring = (p.W > 0) ? (p.T - w_lo) : 0;
  if (blockIdx.x == 0 && h == 0 && threadIdx.x == 0) p.len[b] = p.T;
  const long long src_base = (long long)b * p.T * p.H * DH + (long long)h * DH + li * 8;
  [[maybe_unused]] const long long n_src = (long long)p.B * p.T * p.H * DH;
  if (r < n_dil) {
    const int pos = r * Dd + Dd - 1;
    const long long src = src_base + (long long)pos * p.H * DH;
    const long long dst = ((long long)b * p.rows_per_b + head_offset(p.dense_bits, h, p.T_max, p.D) + r) * DH + li * 8;
    if (!RATP_IN(src, 8, n_src) || !RATP_IN(dst, 8, (long long)p.B * p.rows_per_b * DH)) return;
    *reinterpret_cast<uint4*>(p.Kc + dst) = *reinterpret_cast<const uint4*>(p.hk + src);
    *reinterpret_cast<uint4*>(p.Vc + dst) = *reinterpret_cast<const uint4*>(p.hv + src);
  } else if (r < n_dil + n_ring) {
    const int pos = w_lo + (r - n_dil);
    const long long src = src_base + (long long)pos * p.H * DH;
    const long long dst = (((long long)b * p.H + h) * p.W + pos % p.W) * DH + li * 8;
    if (!RATP_IN(src, 8, n_src) || !RATP_IN(dst, 8, (long long)p.B * p.H * p.W * DH)) return;
    *reinterpret_cast<uint4*>(p.Kw + dst) = *reinterpret_cast<const uint4*>(p.hk + src);
    *reinterpret_cast<uint4*>(p.Vw + dst) = *reinterpret_cast<const uint4*>(p.hv + src);
  }
}

// prefill -> decode hand-off of the look-back inputs: positions
// max(0, T - WL) .. T-1 of x_k, x_v, g into ring slots p mod WL.
// grid (ceil(rows / rows_per_block), H, B); Dh/8 threads per row.
struct PackInputsParams {
  const __nv_bfloat16* x[3];    // x_k, x_v, g: [B][T][H][Dh]
  __nv_bfloat16* in_ring;       // [3][B][H][WL][Dh]
  int B, T, H, WL;
};

template <int DH>
__global__ void __launch_bounds__(256)
pack_inputs_kernel(const PackInputsParams p) {
  constexpr int TPR = DH / 8;
  constexpr int RPB = 256 / TPR;
  const int h = blockIdx.y, b = blockIdx.z;
  const int r = blockIdx.x * RPB + threadIdx.x / TPR;
  const int li = threadIdx.x % TPR;
  const int lo = max(0, p.T - p.WL);
  if (r >= p.T - lo) return;
  const int pos = lo + r;
  const long long src = (((long long)b * p.T + pos) * p.H + h) * DH + li * 8;
  [[maybe_unused]] const long long n_src = (long long)p.B * p.T * p.H * DH;
  [[maybe_unused]] const long long n_ring = 3ll * p.B * p.H * p.WL * DH;
#pragma unroll
  for (int s = 0; s < 3; ++s) {
    const long long dst = (((long long)s * p.B * p.H + (long long)b * p.H + h) * p.WL + pos % p.WL) * DH + li * 8;
    if (RATP_IN(src, 8, n_src) && RATP_IN(dst, 8, n_ring))
      *reinterpret_cast<uint4*>(p.in_ring + dst) = *reinterpret_cast<const uint4*>(p.x[s] + src);
  }
}

}  // namespace decode
}  // namespace ratp
