// ratp.cu -- C ABI of the RAT+ sequence-mixer library (one translation unit).
//
// Host-side argument checks, workspace/cache carving, TMA tensor-map encoding
// and kernel launches.  The kernels live in the included headers:
//   scan.cuh       single-pass chunked scan of the forget-gate recurrence
//   attn_tc.cuh    tensor-core (TMA + tcgen05) dilated/windowed attention
//   attn_simt.cuh  CUDA-core attention for fp32 / head dim 64
//   decode.cuh     cache pack and the fused decode step
//   window.cuh     fixed look-back recurrence (window of the last L tokens)
#include <cuda.h>
#include <cuda_runtime.h>
#include <string.h>

#include <algorithm>
#include <mutex>
#include <set>
#include <utility>

#include "ratp.h"
#include "common.cuh"
#include "scan.cuh"
#include "window.cuh"

#ifdef RATP_GUARDED
namespace ratp {
// Self-test of the guard: asks for element 4 of a 4-element array.  The
// guard refuses it (the store never executes) and records RATP_ERR_BOUNDS.
__device__ int g_guard_probe_buf[4];
__global__ void guard_probe_kernel() {
  const int i = 4;
  if (RATP_IN(i, 1, 4)) g_guard_probe_buf[i & 3] = 1;
}
}  // namespace ratp
#endif
#include "sm100.cuh"
#include "attn_tc.cuh"
#include "attn_simt.cuh"
#include "decode.cuh"

using namespace ratp;

namespace {

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline int launch_status() {
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? RATP_OK : RATP_ERR_CUDA;
}

// Opt a kernel into more than 48 KB of dynamic shared memory, once per device.
template <typename F>
bool ensure_smem(F* func, int bytes) {
  static std::mutex mu;
  static std::set<std::pair<const void*, int>> done;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  std::lock_guard<std::mutex> lock(mu);
  const auto key = std::make_pair(reinterpret_cast<const void*>(func), dev);
  if (done.count(key)) return true;
  if (cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess)
    return false;
  done.insert(key);
  return true;
}

int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 148;
  return n;
}

// ---- scan -------------------------------------------------------------------
struct ScanGeom {
  int slabs, n_chains, n_chunks_t;
  long long n_chunks;
};

int scan_geom(int B, int T, int H, int Dh, int dtype, ScanGeom* g) {
  if (B < 0 || T < 0 || H < 0 || Dh < 0) return RATP_ERR_ARG;
  if (dtype != RATP_F32 && dtype != RATP_BF16) return RATP_ERR_ARG;
  const long long C = (long long)H * Dh;
  if (C % scan::kSlab != 0 || C > (1ll << 30)) return RATP_ERR_SHAPE;
  const int chunk = (dtype == RATP_BF16) ? scan::Shape<__nv_bfloat16>::kChunk
                                         : scan::Shape<float>::kChunk;
  g->slabs = (int)(C / scan::kSlab);
  g->n_chains = B * g->slabs;
  g->n_chunks_t = (T + chunk - 1) / chunk;
  g->n_chunks = (long long)g->n_chains * g->n_chunks_t;
  if (g->n_chunks > 0x7fffffffll) return RATP_ERR_SHAPE;
  return RATP_OK;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn encode_fn();

// [B][T][C] view, box of 64 channels x `rows` tokens x 1 sequence, no swizzle.
template <typename T>
bool make_scan_map(CUtensorMap* m, const void* base, int B, int Tn, int C, int rows,
                   int box_ch = scan::kSlab) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const CUtensorMapDataType dt = sizeof(T) == 4 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32
                                                : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  const cuuint64_t dims[3] = {(cuuint64_t)C, (cuuint64_t)Tn, (cuuint64_t)B};
  const cuuint64_t strides[2] = {(cuuint64_t)C * sizeof(T), (cuuint64_t)Tn * C * sizeof(T)};
  const cuuint32_t box[3] = {(cuuint32_t)box_ch, (cuuint32_t)rows, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, dt, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <typename T, int NS, bool RESET>
int launch_scan(const void* const* x, const void* g, void* const* h, float* fs,
                int B, int Tn, int H, int Dh, int reset_L, const ScanGeom& geo,
                void* ws, size_t ws_bytes, cudaStream_t st) {
  if (geo.n_chunks == 0) return RATP_OK;
  if (ws == nullptr || !aligned16(ws)) return ws == nullptr ? RATP_ERR_ARG : RATP_ERR_ALIGN;
  if (ws_bytes < scan::workspace_bytes(geo.n_chunks, NS)) return RATP_ERR_CAPACITY;
  scan::Params<T, NS> p;
  for (int s = 0; s < NS; ++s) p.h[s] = static_cast<T*>(h[s]);
  p.final_state = fs;
  p.ws = scan::carve(ws, geo.n_chunks, NS);
  p.B = B; p.Tn = Tn; p.C = H * Dh;
  p.reset_L = reset_L;
  p.l2_ahead = sm_count();   // about one ticket per SM ahead (measured: 100-200 alike)
  p.slabs = geo.slabs; p.n_chains = geo.n_chains; p.n_chunks_t = geo.n_chunks_t;
  const int C = H * Dh, rows = scan::Shape<T>::kChunk;
  CUtensorMap tg, tx0, tx1;
  if (!make_scan_map<T>(&tg, g, B, Tn, C, rows) || !make_scan_map<T>(&tx0, x[0], B, Tn, C, rows))
    return RATP_ERR_CUDA;
  if (NS == 2) {
    if (!make_scan_map<T>(&tx1, x[1], B, Tn, C, rows)) return RATP_ERR_CUDA;
  } else {
    tx1 = tx0;
  }
  constexpr int smem = scan::Smem<T, NS>::kBytes;
  auto kernel = scan::scan_kernel<T, NS, scan::kRows, RESET>;
  if (!ensure_smem(kernel, smem)) return RATP_ERR_CUDA;
  cudaError_t e = cudaMemsetAsync(static_cast<char*>(ws) + scan::kResetOffset, 0, scan::kResetBytes, st);
  if (e != cudaSuccess) return RATP_ERR_CUDA;
  // one CTA per chunk; chunk tickets, not block indices, fix the order
  kernel<<<(unsigned)geo.n_chunks, scan::kThreads, smem, st>>>(tg, tx0, tx1, p);
  return launch_status();
}

template <typename E, bool RESET>
int launch_scan_ns(int NS, const void* const* x, const void* g, void* const* h, float* fs,
                   int B, int T, int H, int Dh, int reset_L, const ScanGeom& geo,
                   void* ws, size_t ws_bytes, cudaStream_t st) {
  return NS == 1 ? launch_scan<E, 1, RESET>(x, g, h, fs, B, T, H, Dh, reset_L, geo, ws, ws_bytes, st)
                 : launch_scan<E, 2, RESET>(x, g, h, fs, B, T, H, Dh, reset_L, geo, ws, ws_bytes, st);
}

// reset_L: 0 = the full-sequence recurrence, >= 1 = chunk-local blocks of reset_L tokens
template <typename E, int L>
int launch_window(const void* xk, const void* xv, const void* g, void* hk, void* hv,
                  int B, int T, int H, int Dh, cudaStream_t st) {
  window::Params<E> p;
  p.h[0] = static_cast<E*>(hk);
  p.h[1] = static_cast<E*>(hv);
  p.B = B; p.Tn = T; p.C = H * Dh;
  p.slabs = p.C / window::kCh;
  p.n_chunks_t = (T + window::kChunk - 1) / window::kChunk;
  // one block per SM ahead (measured at T = 16K, L = 64: none 149.8 us,
  // 148 blocks 131.5 us, 444 blocks 135.6 us, 888 blocks 166.4 us)
  p.l2_ahead = sm_count();
  const long long grid = (long long)B * p.slabs * p.n_chunks_t;
  if (grid > 0x7fffffffll) return RATP_ERR_SHAPE;
  CUtensorMap tg, tx0, tx1;
  if (!make_scan_map<E>(&tg, g, B, T, p.C, window::kBox, window::kCh) ||
      !make_scan_map<E>(&tx0, xk, B, T, p.C, window::kBox, window::kCh) ||
      !make_scan_map<E>(&tx1, xv, B, T, p.C, window::kBox, window::kCh))
    return RATP_ERR_CUDA;
  constexpr int smem = window::Smem<E>::kBytes;
  auto kernel = window::window_kernel<E, L>;
  if (!ensure_smem(kernel, smem)) return RATP_ERR_CUDA;
  kernel<<<(unsigned)grid, window::kThreads, smem, st>>>(tg, tx0, tx1, p);
  return launch_status();
}

int scan_common(int NS, const void* const* x, const void* g, void* const* h, float* fs,
                int B, int T, int H, int Dh, int dtype, int reset_L,
                void* ws, size_t ws_bytes, void* stream) {
  if (reset_L < 0) return RATP_ERR_ARG;
  ScanGeom geo;
  int rc = scan_geom(B, T, H, Dh, dtype, &geo);
  if (rc) return rc;
  if (geo.n_chunks == 0) return RATP_OK;
  if (g == nullptr) return RATP_ERR_ARG;
  for (int s = 0; s < NS; ++s) {
    if (x[s] == nullptr || h[s] == nullptr) return RATP_ERR_ARG;
    if (!aligned16(x[s]) || !aligned16(h[s])) return RATP_ERR_ALIGN;
  }
  if (!aligned16(g)) return RATP_ERR_ALIGN;
  if (fs != nullptr && !aligned16(fs)) return RATP_ERR_ALIGN;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // a block at least as long as the sequence never restarts after t = 0
  const bool reset = reset_L > 0 && reset_L < T;
  if (dtype == RATP_BF16) {
    return reset ? launch_scan_ns<__nv_bfloat16, true>(NS, x, g, h, fs, B, T, H, Dh, reset_L, geo, ws, ws_bytes, st)
                 : launch_scan_ns<__nv_bfloat16, false>(NS, x, g, h, fs, B, T, H, Dh, 0, geo, ws, ws_bytes, st);
  }
  return reset ? launch_scan_ns<float, true>(NS, x, g, h, fs, B, T, H, Dh, reset_L, geo, ws, ws_bytes, st)
               : launch_scan_ns<float, false>(NS, x, g, h, fs, B, T, H, Dh, 0, geo, ws, ws_bytes, st);
}

// ---- head masks -------------------------------------------------------------
int read_mask(const uint8_t* head_mask, int H, unsigned long long* bits, uint8_t* dense_list,
              int* n_dense, uint8_t* dil_list, int* n_dil) {
  if (H > RATP_MAX_HEADS) return RATP_ERR_SHAPE;
  for (int w = 0; w < RATP_MAX_HEADS / 64; ++w) bits[w] = 0ull;
  int nd = 0, nl = 0;
  for (int h = 0; h < H; ++h) {
    const bool dense = head_mask != nullptr && head_mask[h] != 0;
    if (dense) {
      bits[h >> 6] |= 1ull << (h & 63);
      if (dense_list) dense_list[nd] = (uint8_t)h;
      ++nd;
    } else {
      if (dil_list) dil_list[nl] = (uint8_t)h;
      ++nl;
    }
  }
  if (n_dense) *n_dense = nd;
  if (n_dil) *n_dil = nl;
  return RATP_OK;
}

int check_attn_args(const void* q, const void* hk, const void* hv, void* o,
                    int B, int T, int H, int Dh, int D, int W, int dtype) {
  if (B < 0 || T < 0 || H < 0 || D < 1 || W < 0) return RATP_ERR_ARG;
  if (dtype != RATP_F32 && dtype != RATP_BF16) return RATP_ERR_ARG;
  if (Dh != 64 && Dh != 128) return RATP_ERR_SHAPE;
  if (H > RATP_MAX_HEADS) return RATP_ERR_SHAPE;
  if ((long long)B * T * H == 0) return RATP_OK;
  if (!q || !hk || !hv || !o) return RATP_ERR_ARG;
  if (!aligned16(q) || !aligned16(hk) || !aligned16(hv) || !aligned16(o)) return RATP_ERR_ALIGN;
  if ((long long)B * T * H * Dh > (1ll << 40)) return RATP_ERR_SHAPE;
  return RATP_OK;
}

int launch_attn_simt(const void* q, const void* hk, const void* hv, void* o,
                     int B, int T, int H, int Dh, int D, int W,
                     const uint8_t* head_mask, int dtype, cudaStream_t st) {
  attn_simt::Params p;
  p.q = q; p.hk = hk; p.hv = hv; p.o = o;
  p.B = B; p.T = T; p.H = H; p.D = D; p.W = W;
  p.scale_log2 = 1.4426950408889634f / sqrtf((float)Dh);
  int rc = read_mask(head_mask, H, p.dense_bits, nullptr, nullptr, nullptr, nullptr);
  if (rc) return rc;
  const long long rows = (long long)B * T * H;
  const unsigned grid = (unsigned)((rows + attn_simt::kWarps - 1) / attn_simt::kWarps);
  const int threads = attn_simt::kWarps * 32;
  if (dtype == RATP_BF16) {
    if (Dh == 128) attn_simt::attn_simt_kernel<__nv_bfloat16, 128><<<grid, threads, 0, st>>>(p);
    else attn_simt::attn_simt_kernel<__nv_bfloat16, 64><<<grid, threads, 0, st>>>(p);
  } else {
    if (Dh == 128) attn_simt::attn_simt_kernel<float, 128><<<grid, threads, 0, st>>>(p);
    else attn_simt::attn_simt_kernel<float, 64><<<grid, threads, 0, st>>>(p);
  }
  return launch_status();
}

// ---- TMA tensor maps (driver entry point fetched through the runtime) --------
EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  return fn;
}

// [B][rows][H][128] bf16 view, rows of `row_stride_elems` elements apart,
// starting `base_elems` elements into each batch item; box 64 x 1 x 128 x 1.
bool make_map(CUtensorMap* m, const void* base, long long base_elems, int B, long long rows,
              int H, long long row_stride_elems, long long batch_stride_elems, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[4] = {128, (cuuint64_t)H, (cuuint64_t)rows, (cuuint64_t)B};
  const cuuint64_t strides[3] = {128 * 2, (cuuint64_t)row_stride_elems * 2,
                                 (cuuint64_t)batch_stride_elems * 2};
  const cuuint32_t box[4] = {64, 1, (cuuint32_t)box_rows, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  void* addr = const_cast<char*>(static_cast<const char*>(base)) + base_elems * 2;
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, addr, dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Ds: nullable host array of B per-sample dilations (else every sample has D).
// ws: nullable device workspace (RATP_ATTN_WORKSPACE_BYTES); with it, a
// launch that mixes segments deals its items dynamically.
int launch_attn_tc(const void* q, const void* hk, const void* hv, void* o,
                   int B, int T, int H, const int* Ds, int D, int W, const uint8_t* head_mask,
                   void* ws, cudaStream_t st) {
  using attn_tc::Segment;
  attn_tc::Params p;
  memset(&p, 0, sizeof(p));
  p.o = static_cast<__nv_bfloat16*>(o);
  p.B = B; p.T = T; p.H = H; p.W_eff = W > 0 ? W : 1;
  p.NQ = (T + attn_tc::BM - 1) / attn_tc::BM;
  unsigned long long bits[RATP_MAX_HEADS / 64];
  int n_dense = 0, n_dil = 0;
  int rc = read_mask(head_mask, H, bits, p.dense_list, &n_dense, p.dil_list, &n_dil);
  if (rc) return rc;
  if (Ds != nullptr && B > attn_tc::kMaxSamples) return RATP_ERR_SHAPE;
  auto D_of = [&](int b) { return Ds != nullptr ? Ds[b] : D; };
  // dilation classes: the distinct D > 1, ascending (more keys first)
  for (int b = 0; b < (Ds != nullptr ? B : 1); ++b) {
    const int d = D_of(b);
    if (d < 1) return RATP_ERR_ARG;
    if (d == 1) continue;
    bool seen = false;
    for (int c = 0; c < p.n_cls; ++c) seen = seen || p.dil_D[c] == d;
    if (seen) continue;
    if (p.n_cls == attn_tc::kMaxDil) return RATP_ERR_UNSUPPORTED;
    p.dil_D[p.n_cls++] = d;
  }
  std::sort(p.dil_D, p.dil_D + p.n_cls);
  // segments, heavy first: dense, then each dilation class
  long long items = 0;
  auto add = [&](int n_b, int b_off, int n_h, int heads, int cls) {
    if ((long long)n_b * n_h == 0) return;
    Segment& g = p.seg[p.n_seg++];
    g.begin = (int)items; g.n_b = n_b; g.n_h = n_h; g.b_off = b_off;
    g.heads = (int8_t)heads; g.cls = (int8_t)cls;
    g.tail = n_b * n_h;                      // no interleaved pairs (set below for dynamic dealing)
    items += (long long)n_b * n_h * p.NQ;
  };
  if (Ds == nullptr) {
    if (D == 1) {
      add(B, -1, H, attn_tc::kHeadsAll, -1);
    } else {
      add(B, -1, n_dense, attn_tc::kHeadsDense, -1);
      add(B, -1, n_dil, attn_tc::kHeadsDil, 0);
    }
  } else {
    // samples ordered: dense ones, then class 0, class 1, ...
    int n = 0;
    for (int b = 0; b < B; ++b) if (D_of(b) == 1) p.samples[n++] = (uint16_t)b;
    const int n_ds = n;
    int off[attn_tc::kMaxDil], cnt[attn_tc::kMaxDil];
    for (int c = 0; c < p.n_cls; ++c) {
      off[c] = n;
      for (int b = 0; b < B; ++b) if (D_of(b) == p.dil_D[c]) p.samples[n++] = (uint16_t)b;
      cnt[c] = n - off[c];
    }
    add(n_ds, 0, H, attn_tc::kHeadsAll, -1);
    add(B - n_ds, n_ds, n_dense, attn_tc::kHeadsDense, -1);
    for (int c = 0; c < p.n_cls; ++c) add(cnt[c], off[c], n_dil, attn_tc::kHeadsDil, c);
  }
  if (items > 0x7fffffffll) return RATP_ERR_SHAPE;
  p.n_items = (int)items;
  if (p.n_items == 0) return RATP_OK;
  p.alternate = p.n_seg > 1;
  // Mixed segments (dense and dilated items, whose costs differ by up to ~D x)
  // balance best when each CTA draws its next item when it is free; the last
  // 32 (b, h) pairs of each dilated segment are interleaved so that the launch
  // ends on light items.  A single segment keeps static dealing (dynamic
  // dealing measured 1-8% slower there).
  const bool dynamic = ws != nullptr && p.n_seg > 1;
  if (dynamic) {
    p.ctl.items = static_cast<unsigned int*>(ws);
    for (int i = 0; i < p.n_seg; ++i) {
      Segment& g = p.seg[i];
      if (g.cls >= 0) g.tail = std::max(0, g.n_b * g.n_h - 32);
    }
    if (cudaMemsetAsync(ws, 0, sizeof(unsigned int), st) != cudaSuccess) return RATP_ERR_CUDA;
  }
  p.scale_log2 = 1.4426950408889634f / sqrtf(128.f);
  p.o_align32 = (reinterpret_cast<uintptr_t>(o) & 31u) == 0;
  const long long row = (long long)H * 128, bat = (long long)T * row;
  CUtensorMap tq, tkp, tvp;
  attn_tc::DilMaps dm;
  memset(&dm, 0, sizeof(dm));
  constexpr int qr = attn_tc::BM, kr = attn_tc::BN;
  if (!make_map(&tq, q, 0, B, T, H, row, bat, qr) || !make_map(&tkp, hk, 0, B, T, H, row, bat, kr) ||
      !make_map(&tvp, hv, 0, B, T, H, row, bat, kr))
    return RATP_ERR_CUDA;
  for (int c = 0; c < attn_tc::kMaxDil; ++c) {
    const int d = c < p.n_cls ? p.dil_D[c] : 0;
    const long long n_slots = d > 0 ? T / d : 0;
    if (n_slots >= 1) {
      if (!make_map(&dm.k[c], hk, (long long)(d - 1) * row, B, n_slots, H, (long long)d * row, bat, kr) ||
          !make_map(&dm.v[c], hv, (long long)(d - 1) * row, B, n_slots, H, (long long)d * row, bat, kr))
        return RATP_ERR_CUDA;
    } else {
      dm.k[c] = tkp;   // no dilated slot exists for any query: never read
      dm.v[c] = tvp;
    }
  }
  attn_tc::ScanMaps sm_unused;
  memset(&sm_unused, 0, sizeof(sm_unused));
  auto kernel = dynamic ? attn_tc::attn_kernel<false, true> : attn_tc::attn_kernel<false, false>;
  if (!ensure_smem(kernel, (int)attn_tc::kSmemBytes)) return RATP_ERR_CUDA;
  const int slots = attn_tc::kCtasPerSm * sm_count();
  const int grid = p.n_items < slots ? p.n_items : slots;
  kernel<<<grid, attn_tc::kThreads, attn_tc::kSmemBytes, st>>>(tq, tkp, tvp, dm, sm_unused, p);
  return launch_status();
}

// Fused prefill: the recurrence of both streams and the attention in one
// launch (attn_kernel<true>: scan CTAs and attention CTAs, fused.cuh).
// Share of the launch's CTAs (two per SM) that scan first, in thousandths.
// An SM shared by a scan CTA and an attention CTA runs each at about half
// its two-CTA rate, so overlap gains little; most CTAs scan first, and the
// rest start the attention on the sequence's first tiles (measured at
// T = 16K: 500 -> 335 us, 700 -> 332 us, 850 -> 323 us, 1000 -> 326 us).
#ifndef RATP_FUSED_SCAN_PER_MILLE
#define RATP_FUSED_SCAN_PER_MILLE 850
#endif

int launch_prefill_fused(const void* q, const void* xk, const void* xv, const void* g, void* hk, void* hv,
                         void* o, float* fs, int B, int T, int H, int D, int W, const uint8_t* head_mask,
                         void* ws, size_t ws_bytes, cudaStream_t st) {
  attn_tc::Params p;
  memset(&p, 0, sizeof(p));
  p.o = static_cast<__nv_bfloat16*>(o);
  p.B = B; p.T = T; p.H = H; p.W_eff = W > 0 ? W : 1;
  p.NQ = (T + attn_tc::BM - 1) / attn_tc::BM;
  const long long n_items = (long long)B * H * p.NQ;
  ScanGeom geo;
  int rc = scan_geom(B, T, H, 128, RATP_BF16, &geo);
  if (rc) return rc;
  if (n_items > 0x7fffffffll) return RATP_ERR_SHAPE;
  if (ws_bytes < fused::workspace_bytes(geo.n_chunks)) return RATP_ERR_CAPACITY;
  rc = read_mask(head_mask, H, p.dense_bits, nullptr, nullptr, nullptr, nullptr);
  if (rc) return rc;
  p.n_items = (int)n_items;
  p.n_cls = D > 1 ? 1 : 0;
  p.dil_D[0] = D;
  p.scale_log2 = 1.4426950408889634f / sqrtf(128.f);
  p.o_align32 = (reinterpret_cast<uintptr_t>(o) & 31u) == 0;
  fused::carve(ws, geo.n_chunks, &p.ctl, &p.scan);
  p.scan.h[0] = static_cast<__nv_bfloat16*>(hk);
  p.scan.h[1] = static_cast<__nv_bfloat16*>(hv);
  p.scan.final_state = fs;
  p.scan.B = B; p.scan.Tn = T; p.scan.C = H * 128;
  p.scan.reset_L = 0;
  p.scan.slabs = geo.slabs; p.scan.n_chains = geo.n_chains; p.scan.n_chunks_t = geo.n_chunks_t;
  // CTAs: two per SM; n_scan of them scan first (no more than there are
  // chunks), and no more CTAs than the scan CTAs plus one per item
  const int slots = attn_tc::kCtasPerSm * sm_count();
  long long n_scan = ((long long)slots * RATP_FUSED_SCAN_PER_MILLE + 500) / 1000;
  n_scan = std::max(1ll, std::min(n_scan, std::min(geo.n_chunks, (long long)slots - 1)));
  const long long n_attn = std::min(n_items, (long long)slots - n_scan);
  p.ctl.n_scan = (int)n_scan;
  p.ctl.n_ctas = (int)(n_scan + n_attn);
  p.scan.l2_ahead = (int)n_scan;   // one chunk per scan CTA ahead
  const long long row = (long long)H * 128, bat = (long long)T * row;
  constexpr int qr = attn_tc::BM, kr = attn_tc::BN;
  constexpr int sr = scan::Shape<__nv_bfloat16>::kChunk;
  CUtensorMap tq, tkp, tvp;
  attn_tc::DilMaps dm;
  attn_tc::ScanMaps sm;
  memset(&dm, 0, sizeof(dm));
  if (!make_map(&tq, q, 0, B, T, H, row, bat, qr) || !make_map(&tkp, hk, 0, B, T, H, row, bat, kr) ||
      !make_map(&tvp, hv, 0, B, T, H, row, bat, kr) ||
      !make_scan_map<__nv_bfloat16>(&sm.g, g, B, T, H * 128, sr) ||
      !make_scan_map<__nv_bfloat16>(&sm.xk, xk, B, T, H * 128, sr) ||
      !make_scan_map<__nv_bfloat16>(&sm.xv, xv, B, T, H * 128, sr))
    return RATP_ERR_CUDA;
  const long long n_slots = D > 1 ? T / D : 0;
  if (n_slots >= 1) {
    if (!make_map(&dm.k[0], hk, (long long)(D - 1) * row, B, n_slots, H, (long long)D * row, bat, kr) ||
        !make_map(&dm.v[0], hv, (long long)(D - 1) * row, B, n_slots, H, (long long)D * row, bat, kr))
      return RATP_ERR_CUDA;
  } else {
    dm.k[0] = tkp;   // no dilated slot exists for any query: never read
    dm.v[0] = tvp;
  }
  auto kernel = attn_tc::attn_kernel<true>;
  if (!ensure_smem(kernel, (int)attn_tc::kSmemBytesFused)) return RATP_ERR_CUDA;
  if (cudaMemsetAsync(static_cast<char*>(ws) + fused::kResetOffset, 0, fused::kResetBytes, st) != cudaSuccess)
    return RATP_ERR_CUDA;
  kernel<<<p.ctl.n_ctas, attn_tc::kThreadsFused, attn_tc::kSmemBytesFused, st>>>(tq, tkp, tvp, dm, sm, p);
  return launch_status();
}

// ---- cache ------------------------------------------------------------------
struct CacheLayout {
  long long rows_per_b;
  size_t off_kc, off_vc, off_kw, off_vw, off_len, off_part, off_cnt, total;
  int max_splits, split_keys;
};

// Decode grid sizing: keys per split chosen so that one step is about one
// wave of CTAs (kDecodeCtasPerSm resident per SM), never below kMinSplitKeys.
constexpr int kDecodeCtasPerSm = 6;
constexpr int kMinSplitKeys = 128;

int cache_layout(int B, int H, int Dh, int T_max, int D, int W, const uint8_t* head_mask,
                 CacheLayout* L) {
  if (B < 1 || H < 1 || T_max < 1 || D < 1 || W < 0) return RATP_ERR_ARG;
  if (Dh != 128 && Dh != 64) return RATP_ERR_SHAPE;
  if (H > RATP_MAX_HEADS) return RATP_ERR_SHAPE;
  long long per_b = 0, keys_total = 0;
  int max_keys = 0;
  for (int h = 0; h < H; ++h) {
    const bool dense = head_mask != nullptr && head_mask[h] != 0;
    const int cap = dense ? T_max : T_max / D;
    per_b += cap;
    const int keys = cap + (dense ? 0 : W);
    keys_total += (long long)B * keys;
    if (keys > max_keys) max_keys = keys;
  }
  L->rows_per_b = per_b;
  const long long target_ctas = (long long)sm_count() * kDecodeCtasPerSm;
  long long split = (keys_total + target_ctas - 1) / target_ctas;
  if (split < kMinSplitKeys) split = kMinSplitKeys;
  // Keep every head's split count but even out its splits: the split becomes
  // the largest per-split share among the heads, so no CTA streams more keys
  // than it must (7.6B hybrid: 357 -> 347 keys, 24 and 6 splits per head).
  {
    long long even = kMinSplitKeys;
    for (int h = 0; h < H; ++h) {
      const bool dense = head_mask != nullptr && head_mask[h] != 0;
      const long long keys = (dense ? T_max : T_max / D) + (dense ? 0 : W);
      if (keys == 0) continue;
      const long long n = (keys + split - 1) / split;
      even = std::max(even, (keys + n - 1) / n);
    }
    split = std::min(split, even);
  }
  if (split > (1 << 30)) split = 1 << 30;
  L->split_keys = (int)split;
  L->max_splits = (max_keys + L->split_keys - 1) / L->split_keys;
  if (L->max_splits < 1) L->max_splits = 1;
  const size_t row_bytes = (size_t)Dh * 2;
  size_t off = 0;
  auto take = [&](size_t bytes) { size_t o = off; off += scan::align256(bytes); return o; };
  L->off_kc = take((size_t)B * per_b * row_bytes);
  L->off_vc = take((size_t)B * per_b * row_bytes);
  L->off_kw = take((size_t)B * H * W * row_bytes);
  L->off_vw = take((size_t)B * H * W * row_bytes);
  L->off_len = take((size_t)B * 4);
  L->off_part = take((size_t)B * H * L->max_splits * (Dh + 2) * 4);
  L->off_cnt = take((size_t)(B * H + B) * 4);
  L->total = off;
  return RATP_OK;
}

bool cache_matches(const ratp_cache* c, int D, int W, const uint8_t* head_mask) {
  if (c->D != D || c->W != W) return false;
  for (int h = 0; h < c->H; ++h) {
    const uint8_t want = (head_mask != nullptr && head_mask[h] != 0) ? 1 : 0;
    if (c->dense[h] != want) return false;
  }
  return true;
}

// ---- allocation-free scan scratch ---------------------------------------------
// One fixed array in the device image; its device address is looked up once
// per device (cudaGetSymbolAddress with that device current) and cached.
static __device__ __align__(256) unsigned char g_noalloc_scratch[RATP_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kMaxDevices] = {};

int noalloc_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return RATP_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (g_noalloc_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return RATP_ERR_CUDA;
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return RATP_OK;
}

}  // namespace

// =============================================================================
extern "C" {

const char* ratp_status_string(int status) {
  switch (status) {
    case RATP_OK: return "ok";
    case RATP_ERR_ARG: return "invalid argument";
    case RATP_ERR_SHAPE: return "unsupported shape";
    case RATP_ERR_ALIGN: return "pointer not 16-byte aligned";
    case RATP_ERR_CAPACITY: return "workspace or cache capacity exceeded";
    case RATP_ERR_TIMEOUT: return "bounded device wait expired";
    case RATP_ERR_CUDA: return "CUDA error";
    case RATP_ERR_UNSUPPORTED: return "unsupported dtype/shape combination";
    case RATP_ERR_BOUNDS: return "guarded build: an out-of-range access was skipped";
    default: return "unknown status";
  }
}

int ratp_last_error(void* stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return RATP_ERR_CUDA;
  unsigned int word = 0;
  if (cudaMemcpyFromSymbol(&word, ratp::g_error_word, sizeof(word)) != cudaSuccess) return RATP_ERR_CUDA;
  const unsigned int zero = 0;
  if (cudaMemcpyToSymbol(ratp::g_error_word, &zero, sizeof(zero)) != cudaSuccess) return RATP_ERR_CUDA;
  for (int code = 1; code < 32; ++code)
    if (word & (1u << code)) return code;
  return RATP_OK;
}

int ratp_guard_line(int* line) {
  if (!line) return RATP_ERR_ARG;
  *line = 0;
#ifdef RATP_GUARDED
  if (cudaMemcpyFromSymbol(line, ratp::g_guard_line, sizeof(int)) != cudaSuccess) return RATP_ERR_CUDA;
  const int zero = 0;
  if (cudaMemcpyToSymbol(ratp::g_guard_line, &zero, sizeof(int)) != cudaSuccess) return RATP_ERR_CUDA;
  return RATP_OK;
#else
  return RATP_ERR_UNSUPPORTED;
#endif
}

int ratp_debug_guard_probe(void* stream) {
#ifdef RATP_GUARDED
  ratp::guard_probe_kernel<<<1, 1, 0, static_cast<cudaStream_t>(stream)>>>();
  return launch_status();
#else
  (void)stream;
  return RATP_ERR_UNSUPPORTED;
#endif
}

int ratp_debug_fault(int kind, long long arg) {
  // each kind sets one device variable; RATP_FAULT_NONE restores all four
  const long long none = -1;
  const unsigned long long timeout =
      (kind == RATP_FAULT_SPIN_LIMIT && arg > 0) ? (unsigned long long)arg : ratp::kSpinTimeoutNs;
  bool ok = true;
  switch (kind) {
    case RATP_FAULT_NONE:
      ok = cudaMemcpyToSymbol(ratp::g_spin_timeout_ns, &timeout, sizeof(timeout)) == cudaSuccess &&
           cudaMemcpyToSymbol(ratp::g_fault_scan_ticket, &none, sizeof(none)) == cudaSuccess &&
           cudaMemcpyToSymbol(ratp::g_fault_attn_ktile, &none, sizeof(none)) == cudaSuccess &&
           cudaMemcpyToSymbol(ratp::g_fault_fused_chunk, &none, sizeof(none)) == cudaSuccess;
      break;
    case RATP_FAULT_SPIN_LIMIT:
      ok = cudaMemcpyToSymbol(ratp::g_spin_timeout_ns, &timeout, sizeof(timeout)) == cudaSuccess;
      break;
    case RATP_FAULT_SCAN_DROP:
      ok = cudaMemcpyToSymbol(ratp::g_fault_scan_ticket, &arg, sizeof(arg)) == cudaSuccess;
      break;
    case RATP_FAULT_ATTN_DROP_K:
      ok = cudaMemcpyToSymbol(ratp::g_fault_attn_ktile, &arg, sizeof(arg)) == cudaSuccess;
      break;
    case RATP_FAULT_FUSED_DROP_CHUNK:
      ok = cudaMemcpyToSymbol(ratp::g_fault_fused_chunk, &arg, sizeof(arg)) == cudaSuccess;
      break;
    default:
      return RATP_ERR_ARG;
  }
  return ok ? RATP_OK : RATP_ERR_CUDA;
}

int ratp_device_sm_count(int* sms) {
  if (!sms) return RATP_ERR_ARG;
  *sms = sm_count();
  return RATP_OK;
}

int ratp_scan_workspace_bytes(int B, int T, int H, int Dh, int dtype, size_t* bytes) {
  if (!bytes) return RATP_ERR_ARG;
  ScanGeom geo;
  int rc = scan_geom(B, T, H, Dh, dtype, &geo);
  if (rc) return rc;
  // one size serves both the single- and the two-stream scan
  *bytes = scan::workspace_bytes(geo.n_chunks, 2);
  return RATP_OK;
}

int ratp_scan_prefill(const void* x, const void* g, void* h, float* final_state,
                      int B, int T, int H, int Dh, int dtype,
                      void* workspace, size_t workspace_bytes, void* stream) {
  const void* xs[1] = {x};
  void* hs[1] = {h};
  return scan_common(1, xs, g, hs, final_state, B, T, H, Dh, dtype, 0, workspace, workspace_bytes, stream);
}

int ratp_scan_prefill_chunk_local(const void* x, const void* g, void* h, float* final_state,
                                  int B, int T, int H, int Dh, int dtype, int L,
                                  void* workspace, size_t workspace_bytes, void* stream) {
  const void* xs[1] = {x};
  void* hs[1] = {h};
  return scan_common(1, xs, g, hs, final_state, B, T, H, Dh, dtype, L, workspace, workspace_bytes, stream);
}

int ratp_scan_prefill_kv(const void* xk, const void* xv, const void* g,
                         void* hk, void* hv, float* final_state,
                         int B, int T, int H, int Dh, int dtype,
                         void* workspace, size_t workspace_bytes, void* stream) {
  const void* xs[2] = {xk, xv};
  void* hs[2] = {hk, hv};
  return scan_common(2, xs, g, hs, final_state, B, T, H, Dh, dtype, 0, workspace, workspace_bytes, stream);
}

int ratp_scan_prefill_kv_chunk_local(const void* xk, const void* xv, const void* g,
                                     void* hk, void* hv, float* final_state,
                                     int B, int T, int H, int Dh, int dtype, int L,
                                     void* workspace, size_t workspace_bytes, void* stream) {
  const void* xs[2] = {xk, xv};
  void* hs[2] = {hk, hv};
  return scan_common(2, xs, g, hs, final_state, B, T, H, Dh, dtype, L, workspace, workspace_bytes, stream);
}

int ratp_scan_prefill_kv_window(const void* xk, const void* xv, const void* g,
                                void* hk, void* hv, int B, int T, int H, int Dh, int dtype,
                                int L, void* stream) {
  if (B < 0 || T < 0 || H < 0 || Dh < 0 || L < 1) return RATP_ERR_ARG;
  if (dtype != RATP_F32 && dtype != RATP_BF16) return RATP_ERR_ARG;
  if (L != 16 && L != 32 && L != 64) return RATP_ERR_UNSUPPORTED;
  const long long C = (long long)H * Dh;
  if (C % 64 != 0 || C > (1ll << 30)) return RATP_ERR_SHAPE;
  if ((long long)B * T * C == 0) return RATP_OK;
  if (!xk || !xv || !g || !hk || !hv) return RATP_ERR_ARG;
  if (!aligned16(xk) || !aligned16(xv) || !aligned16(g) || !aligned16(hk) || !aligned16(hv))
    return RATP_ERR_ALIGN;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (dtype == RATP_BF16) {
    switch (L) {
      case 16: return launch_window<__nv_bfloat16, 16>(xk, xv, g, hk, hv, B, T, H, Dh, st);
      case 32: return launch_window<__nv_bfloat16, 32>(xk, xv, g, hk, hv, B, T, H, Dh, st);
      default: return launch_window<__nv_bfloat16, 64>(xk, xv, g, hk, hv, B, T, H, Dh, st);
    }
  }
  switch (L) {
    case 16: return launch_window<float, 16>(xk, xv, g, hk, hv, B, T, H, Dh, st);
    case 32: return launch_window<float, 32>(xk, xv, g, hk, hv, B, T, H, Dh, st);
    default: return launch_window<float, 64>(xk, xv, g, hk, hv, B, T, H, Dh, st);
  }
}

int ratp_scan_prefill_kv_noalloc(const void* xk, const void* xv, const void* g,
                                 void* hk, void* hv, float* final_state,
                                 int B, int T, int H, int Dh, int dtype, void* stream) {
  ScanGeom geo;
  int rc = scan_geom(B, T, H, Dh, dtype, &geo);
  if (rc) return rc;
  if (geo.n_chunks == 0) return RATP_OK;
  if (scan::workspace_bytes(geo.n_chunks, 2) > (size_t)RATP_NOALLOC_SCRATCH_BYTES) return RATP_ERR_CAPACITY;
  void* ws = nullptr;
  rc = noalloc_scratch(&ws);
  if (rc) return rc;
  const void* xs[2] = {xk, xv};
  void* hs[2] = {hk, hv};
  return scan_common(2, xs, g, hs, final_state, B, T, H, Dh, dtype, 0, ws,
                     (size_t)RATP_NOALLOC_SCRATCH_BYTES, stream);
}

int ratp_dilated_attn_prefill_simt(const void* q, const void* hk, const void* hv, void* o,
                                   int B, int T, int H, int Dh, int D, int W,
                                   const uint8_t* head_mask, int dtype, void* stream) {
  int rc = check_attn_args(q, hk, hv, o, B, T, H, Dh, D, W, dtype);
  if (rc) return rc;
  if ((long long)B * T * H == 0) return RATP_OK;
  return launch_attn_simt(q, hk, hv, o, B, T, H, Dh, D, W, head_mask, dtype,
                          static_cast<cudaStream_t>(stream));
}

int ratp_dilated_attn_prefill(const void* q, const void* hk, const void* hv, void* o,
                              int B, int T, int H, int Dh, int D, int W,
                              const uint8_t* head_mask, int dtype, void* stream) {
  int rc = check_attn_args(q, hk, hv, o, B, T, H, Dh, D, W, dtype);
  if (rc) return rc;
  if ((long long)B * T * H == 0) return RATP_OK;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (dtype == RATP_BF16 && Dh == 128)
    return launch_attn_tc(q, hk, hv, o, B, T, H, nullptr, D, W, head_mask, nullptr, st);
  return launch_attn_simt(q, hk, hv, o, B, T, H, Dh, D, W, head_mask, dtype, st);
}

int ratp_prefill_fused_workspace_bytes(int B, int T, int H, int Dh, size_t* bytes) {
  if (!bytes || B < 0 || T < 0 || H < 0) return RATP_ERR_ARG;
  if (Dh != 128) return RATP_ERR_UNSUPPORTED;
  ScanGeom geo;
  const int rc = scan_geom(B, T, H, 128, RATP_BF16, &geo);
  if (rc) return rc;
  *bytes = fused::workspace_bytes(geo.n_chunks);
  return RATP_OK;
}

int ratp_prefill_fused(const void* q, const void* xk, const void* xv, const void* g,
                       void* hk, void* hv, void* o, float* final_state,
                       int B, int T, int H, int Dh, int D, int W, const uint8_t* head_mask, int dtype,
                       void* workspace, size_t workspace_bytes, void* stream) {
  int rc = check_attn_args(q, hk, hv, o, B, T, H, Dh, D, W, dtype);
  if (rc) return rc;
  if (dtype != RATP_BF16 || Dh != 128) return RATP_ERR_UNSUPPORTED;
  if ((long long)B * T * H == 0) return RATP_OK;
  if (!xk || !xv || !g || !workspace) return RATP_ERR_ARG;
  if (!aligned16(xk) || !aligned16(xv) || !aligned16(g) || !aligned16(workspace)) return RATP_ERR_ALIGN;
  if (final_state != nullptr && !aligned16(final_state)) return RATP_ERR_ALIGN;
  return launch_prefill_fused(q, xk, xv, g, hk, hv, o, final_state, B, T, H, D, W, head_mask, workspace,
                              workspace_bytes, static_cast<cudaStream_t>(stream));
}

int ratp_dilated_attn_prefill_per_sample(const void* q, const void* hk, const void* hv, void* o,
                                         int B, int T, int H, int Dh, const int32_t* D_per_sample,
                                         int W, const uint8_t* head_mask, int dtype, void* stream) {
  int rc = check_attn_args(q, hk, hv, o, B, T, H, Dh, 1, W, dtype);
  if (rc) return rc;
  if (B > 0 && D_per_sample == nullptr) return RATP_ERR_ARG;
  for (int b = 0; b < B; ++b)
    if (D_per_sample[b] < 1) return RATP_ERR_ARG;
  if (dtype != RATP_BF16 || Dh != 128) return RATP_ERR_UNSUPPORTED;
  if (B > attn_tc::kMaxSamples) return RATP_ERR_SHAPE;
  if ((long long)B * T * H == 0) return RATP_OK;
  return launch_attn_tc(q, hk, hv, o, B, T, H, D_per_sample, 0, W, head_mask, nullptr,
                        static_cast<cudaStream_t>(stream));
}

int ratp_dilated_attn_prefill_ws(const void* q, const void* hk, const void* hv, void* o,
                                 int B, int T, int H, int Dh, int D, int W,
                                 const uint8_t* head_mask, int dtype, void* workspace, void* stream) {
  if (workspace != nullptr && !aligned16(workspace)) return RATP_ERR_ALIGN;
  int rc = check_attn_args(q, hk, hv, o, B, T, H, Dh, D, W, dtype);
  if (rc) return rc;
  if ((long long)B * T * H == 0) return RATP_OK;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (dtype == RATP_BF16 && Dh == 128)
    return launch_attn_tc(q, hk, hv, o, B, T, H, nullptr, D, W, head_mask, workspace, st);
  return launch_attn_simt(q, hk, hv, o, B, T, H, Dh, D, W, head_mask, dtype, st);
}

int ratp_dilated_attn_prefill_per_sample_ws(const void* q, const void* hk, const void* hv, void* o,
                                            int B, int T, int H, int Dh, const int32_t* D_per_sample,
                                            int W, const uint8_t* head_mask, int dtype, void* workspace,
                                            void* stream) {
  if (workspace != nullptr && !aligned16(workspace)) return RATP_ERR_ALIGN;
  int rc = check_attn_args(q, hk, hv, o, B, T, H, Dh, 1, W, dtype);
  if (rc) return rc;
  if (B > 0 && D_per_sample == nullptr) return RATP_ERR_ARG;
  for (int b = 0; b < B; ++b)
    if (D_per_sample[b] < 1) return RATP_ERR_ARG;
  if (dtype != RATP_BF16 || Dh != 128) return RATP_ERR_UNSUPPORTED;
  if (B > attn_tc::kMaxSamples) return RATP_ERR_SHAPE;
  if ((long long)B * T * H == 0) return RATP_OK;
  return launch_attn_tc(q, hk, hv, o, B, T, H, D_per_sample, 0, W, head_mask, workspace,
                        static_cast<cudaStream_t>(stream));
}

int ratp_cache_bytes(int B, int H, int Dh, int T_max, int D, int W,
                     const uint8_t* head_mask, size_t* bytes) {
  if (!bytes) return RATP_ERR_ARG;
  CacheLayout L;
  int rc = cache_layout(B, H, Dh, T_max, D, W, head_mask, &L);
  if (rc) return rc;
  *bytes = L.total;
  return RATP_OK;
}

int ratp_cache_init(ratp_cache* c, void* buffer, size_t bytes, int B, int H, int Dh, int T_max,
                    int D, int W, const uint8_t* head_mask, void* stream) {
  if (!c || !buffer) return RATP_ERR_ARG;
  if (!aligned16(buffer)) return RATP_ERR_ALIGN;
  CacheLayout L;
  int rc = cache_layout(B, H, Dh, T_max, D, W, head_mask, &L);
  if (rc) return rc;
  if (bytes < L.total) return RATP_ERR_CAPACITY;
  char* base = static_cast<char*>(buffer);
  memset(c, 0, sizeof(*c));
  c->Kc = base + L.off_kc;
  c->Vc = base + L.off_vc;
  c->Kw = W > 0 ? base + L.off_kw : nullptr;
  c->Vw = W > 0 ? base + L.off_vw : nullptr;
  c->len = reinterpret_cast<int32_t*>(base + L.off_len);
  c->partial = reinterpret_cast<float*>(base + L.off_part);
  c->counters = reinterpret_cast<uint32_t*>(base + L.off_cnt);
  c->rows_per_b = L.rows_per_b;
  c->B = B; c->H = H; c->Dh = Dh; c->T_max = T_max; c->D = D; c->W = W;
  c->split_keys = L.split_keys;
  c->max_splits = L.max_splits;
  c->reset_L = 0;
  c->window_L = 0;
  c->in_ring = nullptr;
  for (int h = 0; h < H; ++h) c->dense[h] = (head_mask != nullptr && head_mask[h] != 0) ? 1 : 0;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(c->len, 0, (size_t)B * 4, st) != cudaSuccess) return RATP_ERR_CUDA;
  if (cudaMemsetAsync(c->counters, 0, (size_t)(B * H + B) * 4, st) != cudaSuccess) return RATP_ERR_CUDA;
  return RATP_OK;
}

int ratp_cache_pack(ratp_cache* c, const void* hk, const void* hv, int T, void* stream) {
  if (!c || !hk || !hv) return RATP_ERR_ARG;
  if (T < 0 || T > c->T_max) return RATP_ERR_CAPACITY;
  if (!aligned16(hk) || !aligned16(hv)) return RATP_ERR_ALIGN;
  decode::PackParams p;
  p.hk = static_cast<const __nv_bfloat16*>(hk);
  p.hv = static_cast<const __nv_bfloat16*>(hv);
  p.Kc = static_cast<__nv_bfloat16*>(c->Kc);
  p.Vc = static_cast<__nv_bfloat16*>(c->Vc);
  p.Kw = static_cast<__nv_bfloat16*>(c->Kw);
  p.Vw = static_cast<__nv_bfloat16*>(c->Vw);
  p.len = c->len;
  p.rows_per_b = c->rows_per_b;
  p.B = c->B; p.T = T; p.H = c->H; p.D = c->D; p.W = c->W; p.T_max = c->T_max;
  int rc = read_mask(c->dense, c->H, p.dense_bits, nullptr, nullptr, nullptr, nullptr);
  if (rc) return rc;
  int max_rows = 0;
  for (int h = 0; h < c->H; ++h) {
    const int Dd = c->dense[h] ? 1 : c->D;
    const int rows = T / Dd + (c->W > 0 ? (T < c->W ? T : c->W) : 0);
    if (rows > max_rows) max_rows = rows;
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int rpb = 256 / (c->Dh / 8);
  dim3 grid((unsigned)((max_rows + rpb - 1) / rpb), (unsigned)c->H, (unsigned)c->B);
  if (grid.x == 0) grid.x = 1;   // still sets len
  if (c->Dh == 128) decode::pack_kernel<128><<<grid, 256, 0, st>>>(p);
  else decode::pack_kernel<64><<<grid, 256, 0, st>>>(p);
  return launch_status();
}

int ratp_cache_set_chunk_local(ratp_cache* c, int L) {
  if (!c || L < 0) return RATP_ERR_ARG;
  if (L > 0 && c->window_L > 0) return RATP_ERR_ARG;
  c->reset_L = L;
  return RATP_OK;
}

int ratp_cache_window_bytes(int B, int H, int Dh, int L, size_t* bytes) {
  if (!bytes || B < 1 || H < 1 || L < 1 || L > 256) return RATP_ERR_ARG;
  if (Dh != 128 && Dh != 64) return RATP_ERR_SHAPE;
  *bytes = (size_t)3 * B * H * L * Dh * 2;
  return RATP_OK;
}

int ratp_cache_set_window(ratp_cache* c, void* ring, size_t bytes, int L) {
  if (!c || L < 0 || L > 256) return RATP_ERR_ARG;
  if (L == 0) {
    c->window_L = 0;
    c->in_ring = nullptr;
    return RATP_OK;
  }
  if (!ring || c->reset_L > 0) return RATP_ERR_ARG;
  if (!aligned16(ring)) return RATP_ERR_ALIGN;
  size_t need = 0;
  int rc = ratp_cache_window_bytes(c->B, c->H, c->Dh, L, &need);
  if (rc) return rc;
  if (bytes < need) return RATP_ERR_CAPACITY;
  c->in_ring = ring;
  c->window_L = L;
  return RATP_OK;
}

int ratp_cache_pack_inputs(ratp_cache* c, const void* xk, const void* xv, const void* g, int T,
                           void* stream) {
  if (!c || !xk || !xv || !g || c->window_L <= 0 || !c->in_ring) return RATP_ERR_ARG;
  if (T < 0 || T > c->T_max) return RATP_ERR_CAPACITY;
  if (!aligned16(xk) || !aligned16(xv) || !aligned16(g)) return RATP_ERR_ALIGN;
  if (T == 0) return RATP_OK;
  decode::PackInputsParams p;
  p.x[0] = static_cast<const __nv_bfloat16*>(xk);
  p.x[1] = static_cast<const __nv_bfloat16*>(xv);
  p.x[2] = static_cast<const __nv_bfloat16*>(g);
  p.in_ring = static_cast<__nv_bfloat16*>(c->in_ring);
  p.B = c->B; p.T = T; p.H = c->H; p.WL = c->window_L;
  const int rows = T < c->window_L ? T : c->window_L;
  const int rpb = 256 / (c->Dh / 8);
  dim3 grid((unsigned)((rows + rpb - 1) / rpb), (unsigned)c->H, (unsigned)c->B);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (c->Dh == 128) decode::pack_inputs_kernel<128><<<grid, 256, 0, st>>>(p);
  else decode::pack_inputs_kernel<64><<<grid, 256, 0, st>>>(p);
  return launch_status();
}

}  // extern "C"

namespace {

// One decode step of one layer: the checks and the launch behind
// ratp_decode_step and ratp_decode_step_layers (the cache's own D, W and
// head mask).
int decode_launch(const void* q, const void* xk, const void* xv, const void* g,
                  float* state, const ratp_cache* c, void* o, cudaStream_t st) {
  if (!q || !xk || !xv || !g || !state || !c || !o) return RATP_ERR_ARG;
  if (c->reset_L < 0 || c->window_L < 0 || c->window_L > 256) return RATP_ERR_ARG;
  if (c->window_L > 0 && (c->in_ring == nullptr || c->reset_L > 0)) return RATP_ERR_ARG;
  if (!aligned16(q) || !aligned16(xk) || !aligned16(xv) || !aligned16(g) || !aligned16(state) ||
      !aligned16(o))
    return RATP_ERR_ALIGN;
  decode::Params p;
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.xk = static_cast<const __nv_bfloat16*>(xk);
  p.xv = static_cast<const __nv_bfloat16*>(xv);
  p.g = static_cast<const __nv_bfloat16*>(g);
  p.o = static_cast<__nv_bfloat16*>(o);
  p.state = state;
  p.Kc = static_cast<__nv_bfloat16*>(c->Kc);
  p.Vc = static_cast<__nv_bfloat16*>(c->Vc);
  p.Kw = static_cast<__nv_bfloat16*>(c->Kw);
  p.Vw = static_cast<__nv_bfloat16*>(c->Vw);
  p.len = c->len;
  p.partial = c->partial;
  p.counters = c->counters;
  p.rows_per_b = c->rows_per_b;
  p.B = c->B; p.H = c->H; p.D = c->D; p.W = c->W; p.T_max = c->T_max;
  p.split_keys = c->split_keys;
  p.max_splits = c->max_splits;
  p.reset_L = c->reset_L;
  p.window_L = c->window_L;
  p.in_ring = static_cast<__nv_bfloat16*>(c->in_ring);
  p.scale_log2 = 1.4426950408889634f / sqrtf((float)c->Dh);
  int rc = read_mask(c->dense, c->H, p.dense_bits, nullptr, nullptr, nullptr, nullptr);
  if (rc) return rc;
  // per-head split counts: the most keys head h can hold, over split_keys
  p.split_base[0] = 0;
  for (int h = 0; h < c->H; ++h) {
    const bool dense = (p.dense_bits[h >> 6] >> (h & 63)) & 1ull;
    const long long keys = dense ? (long long)c->T_max : (long long)c->T_max / c->D + c->W;
    long long sp = (keys + c->split_keys - 1) / c->split_keys;
    if (sp < 1) sp = 1;
    if (sp > c->max_splits) sp = c->max_splits;
    p.split_base[h + 1] = p.split_base[h] + (int)sp;
  }
  p.splits_per_b = p.split_base[c->H];
  if ((long long)p.splits_per_b * c->B > 0x7fffffffll) return RATP_ERR_SHAPE;
  dim3 grid((unsigned)(p.splits_per_b * c->B));
  // Programmatic dependent launch: the step may be scheduled while the
  // previous kernel in the stream drains; it waits for that kernel's
  // completion (griddepcontrol.wait) before touching any memory.
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(decode::kThreads);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = (c->Dh == 128) ? cudaLaunchKernelEx(&cfg, decode::decode_kernel<128>, p)
                                 : cudaLaunchKernelEx(&cfg, decode::decode_kernel<64>, p);
  if (e != cudaSuccess) return RATP_ERR_CUDA;
  return launch_status();
}

}  // namespace

extern "C" {

int ratp_decode_step(const void* q, const void* xk, const void* xv, const void* g,
                     float* state, ratp_cache* c, void* o,
                     int D, int W, const uint8_t* head_mask, void* stream) {
  if (!q || !xk || !xv || !g || !state || !c || !o) return RATP_ERR_ARG;
  if (!cache_matches(c, D, W, head_mask)) return RATP_ERR_ARG;
  return decode_launch(q, xk, xv, g, state, c, o, static_cast<cudaStream_t>(stream));
}

int ratp_decode_step_layers(const ratp_decode_layer* layers, int n_layers, void* stream) {
  if (n_layers < 0 || (n_layers > 0 && layers == nullptr)) return RATP_ERR_ARG;
  for (int l = 0; l < n_layers; ++l) {
    const ratp_decode_layer& L = layers[l];
    const int rc = decode_launch(L.q, L.xk, L.xv, L.g, L.state, L.cache, L.o,
                                 static_cast<cudaStream_t>(stream));
    if (rc) return rc;
  }
  return RATP_OK;
}

}  // extern "C"
