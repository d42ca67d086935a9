// common.cuh -- device helpers shared by the RAT+ kernels (sm_100a).
#pragma once
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "ratp.h"

namespace ratp {

// Device error word: kernels OR a RATP_ERR_* bit pattern into it instead of
// trapping; ratp_last_error() reads and clears it.  One word per device.
__device__ unsigned int g_error_word;

__device__ __forceinline__ void raise_error(unsigned int code) {
  atomicOr(&g_error_word, 1u << code);
}

// Guarded debug build (compiled with -DRATP_GUARDED into libratp_guarded.so):
// every global access that a kernel addresses itself (TMA boxes are bounded by
// the hardware) first checks its element range against the buffer's size.
// An access outside it is skipped, RATP_ERR_BOUNDS is set in the error word
// and the first failing source line is kept in g_guard_line, so an index
// error shows up as a status instead of a memory fault.  In the normal build
// RATP_IN(...) is the constant true and costs nothing.
#ifdef RATP_GUARDED
__device__ int g_guard_line;
__device__ __noinline__ bool guard_fail(int line) {
  atomicCAS(&g_guard_line, 0, line);
  raise_error(RATP_ERR_BOUNDS);
  return false;
}
__device__ __forceinline__ bool in_range(long long first, long long count, long long size, int line) {
  return (first >= 0 && count >= 0 && first + count <= size) ? true : guard_fail(line);
}
#define RATP_IN(first, count, size) \
  ::ratp::in_range((long long)(first), (long long)(count), (long long)(size), __LINE__)
#else
#define RATP_IN(first, count, size) true
#endif

// Bound for every spin-wait (ns of %globaltimer).  A wait that runs out sets
// RATP_ERR_TIMEOUT and the kernel carries on to a clean exit.  Tests of the
// failure paths lower it and plant a missing publication (ratp_debug_fault).
constexpr unsigned long long kSpinTimeoutNs = 2000000000ull;
__device__ unsigned long long g_spin_timeout_ns = kSpinTimeoutNs;
__device__ long long g_fault_scan_ticket = -1;    // scan chunk that publishes nothing
__device__ long long g_fault_attn_ktile = -1;     // K tile the first attention CTA skips
__device__ long long g_fault_fused_chunk = -1;    // fused prefill scan chunk whose done flag is never raised

__device__ __forceinline__ unsigned long long spin_timeout() { return g_spin_timeout_ns; }

__device__ __forceinline__ unsigned long long global_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// ---- element conversion -----------------------------------------------------
template <typename T> struct Elem;
template <> struct Elem<float> {
  static constexpr int kVec = 4;  // elements per 16-byte vector
  __device__ static __forceinline__ void unpack2(const uint4& v, float2* f) {
    f[0] = make_float2(__uint_as_float(v.x), __uint_as_float(v.y));
    f[1] = make_float2(__uint_as_float(v.z), __uint_as_float(v.w));
  }
  __device__ static __forceinline__ uint4 pack2(const float2* f) {
    return make_uint4(__float_as_uint(f[0].x), __float_as_uint(f[0].y),
                      __float_as_uint(f[1].x), __float_as_uint(f[1].y));
  }
  __device__ static __forceinline__ void unpack(const uint4& v, float* f) {
    f[0] = __uint_as_float(v.x); f[1] = __uint_as_float(v.y);
    f[2] = __uint_as_float(v.z); f[3] = __uint_as_float(v.w);
  }
  __device__ static __forceinline__ float load1(const float* p) { return *p; }
};
template <> struct Elem<__nv_bfloat16> {
  static constexpr int kVec = 8;
  // 16 bytes <-> four channel pairs
  __device__ static __forceinline__ void unpack2(const uint4& v, float2* f) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) f[i] = make_float2(__uint_as_float(w[i] << 16), __uint_as_float(w[i] & 0xffff0000u));
  }
  __device__ static __forceinline__ uint4 pack2(const float2* f) {
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      __nv_bfloat162 h = __floats2bfloat162_rn(f[i].x, f[i].y);
      w[i] = *reinterpret_cast<uint32_t*>(&h);
    }
    return make_uint4(w[0], w[1], w[2], w[3]);
  }
  __device__ static __forceinline__ void unpack(const uint4& v, float* f) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      f[2 * i] = __uint_as_float(w[i] << 16);
      f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
  }
  __device__ static __forceinline__ float load1(const __nv_bfloat16* p) {
    return __bfloat162float(*p);
  }
};

// ---- packed fp32 pairs (Blackwell f32x2 arithmetic, one instruction per pair)
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
      "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y) : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
  return d;
}
__device__ __forceinline__ float2 mul2(float2 a, float2 b) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rd;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "mul.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y) : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}
__device__ __forceinline__ float2 add2(float2 a, float2 b) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rd;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "add.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y) : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}
__device__ __forceinline__ float2 sub2(float2 a, float2 b) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rd;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "sub.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y) : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

}  // namespace ratp
