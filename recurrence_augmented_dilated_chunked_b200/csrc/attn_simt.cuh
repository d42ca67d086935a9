// attn_simt.cuh -- CUDA-core dilated (+ windowed) prefill attention.
//
// Same operation as the tensor-core kernel (RAT+ abstract: dilated attention
// with optional local windows; write-up section 6: dense heads), for the
// cases it does not cover: fp32 tensors and head dim 64.  One warp per query
// row walks the row's key set in increasing position order -- the dilated
// positions j = D_h-1, 2D_h-1, ... < t, the window positions t-W < j < t that
// are not dilated ones, then j = t -- with an fp32 online softmax.  Each lane
// holds Dh/32 contiguous elements of q, k, v and of the output accumulator.
#pragma once
#include "common.cuh"

namespace ratp {
namespace attn_simt {

constexpr int kWarps = 4;

struct Params {
  const void* q;
  const void* hk;
  const void* hv;
  void* o;
  int B, T, H, D, W;
  float scale_log2;
  unsigned long long dense_bits[RATP_MAX_HEADS / 64];
};

template <typename T, int EPL>
__device__ __forceinline__ void load_lane(const T* row, int lane, float* f) {
#pragma unroll
  for (int i = 0; i < EPL; ++i) f[i] = Elem<T>::load1(row + lane * EPL + i);
}

template <typename T, int DH>
__global__ void __launch_bounds__(kWarps * 32)
attn_simt_kernel(const Params p) {
  constexpr int EPL = DH / 32;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const long long row = (long long)blockIdx.x * kWarps + warp;
  const long long n_rows = (long long)p.B * p.T * p.H;
  if (row >= n_rows) return;
  const int h = (int)(row % p.H);
  const int t = (int)((row / p.H) % p.T);
  const int b = (int)(row / ((long long)p.H * p.T));
  const bool dense = (p.dense_bits[h >> 6] >> (h & 63)) & 1ull;
  const int Dd = dense ? 1 : p.D;

  const T* q = static_cast<const T*>(p.q);
  const T* hk = static_cast<const T*>(p.hk);
  const T* hv = static_cast<const T*>(p.hv);
  const long long bstride = (long long)p.T * p.H * DH;
  const long long tstride = (long long)p.H * DH;
  const T* kbase = hk + b * bstride + (long long)h * DH;
  const T* vbase = hv + b * bstride + (long long)h * DH;

  float qv[EPL], acc[EPL];
  [[maybe_unused]] const long long n_elem = (long long)p.B * bstride;
  if (!RATP_IN(b * bstride + (long long)t * tstride + (long long)h * DH, DH, n_elem)) return;
  load_lane<T, EPL>(q + b * bstride + (long long)t * tstride + (long long)h * DH, lane, qv);
#pragma unroll
  for (int i = 0; i < EPL; ++i) { qv[i] *= p.scale_log2; acc[i] = 0.f; }
  float m = -INFINITY, l = 0.f;

  auto visit = [&](int j) {
    float kf[EPL], vf[EPL];
    if (!RATP_IN(b * bstride + (long long)j * tstride + (long long)h * DH, DH, n_elem)) return;
    load_lane<T, EPL>(kbase + (long long)j * tstride, lane, kf);
    load_lane<T, EPL>(vbase + (long long)j * tstride, lane, vf);
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < EPL; ++i) s = fmaf(qv[i], kf[i], s);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
    const float m_new = fmaxf(m, s);
    const float alpha = exp2f(m - m_new);
    const float pj = exp2f(s - m_new);
    l = l * alpha + pj;
#pragma unroll
    for (int i = 0; i < EPL; ++i) acc[i] = fmaf(acc[i], alpha, pj * vf[i]);
    m = m_new;
  };

  for (int j = Dd - 1; j < t; j += Dd) visit(j);
  if (p.W > 0 && Dd > 1) {
    for (int j = max(0, t - p.W + 1); j < t; ++j)
      if (j % Dd != Dd - 1) visit(j);
  }
  visit(t);

  const float inv = 1.f / l;
  T* out = static_cast<T*>(p.o) + b * bstride + (long long)t * tstride + (long long)h * DH + lane * EPL;
#pragma unroll
  for (int i = 0; i < EPL; ++i) {
    if constexpr (sizeof(T) == 4) out[i] = acc[i] * inv;
    else out[i] = __float2bfloat16_rn(acc[i] * inv);
  }
}

}  // namespace attn_simt
}  // namespace ratp
