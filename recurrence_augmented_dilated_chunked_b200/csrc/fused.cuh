// fused.cuh -- the recurrence side of the fused prefill, and the launch's
// shared control words.
//
// The fused prefill computes the forget-gate recurrence of the key and value
// streams (zhichai.net "RAT+ 深度拆解", section 2.1: the full-sequence
// recurrence) and the dilated / windowed / head-wise hybrid attention over
// its output (RAT+ abstract; the write-up's sections 1 and 6) in one launch.
// Every CTA of the launch allocates its tensor memory and draws a start
// ticket; the first n_scan CTAs to start scan first:
//   * scan: the chunk scan of scan.cuh (256 tokens x 64 channels of one batch
//     item per chunk, staged by TMA, decoupled look-back across chunks) over
//     chunk tickets drawn in sequence order, one chunk after another; each
//     chunk's done flag is raised once its rows are stored, in sequence order
//     per chain;
//   * attention: the tensor-core pipeline of attn_tc.cuh over query tiles
//     drawn one by one from an item counter in ascending order; before an
//     item's key tiles are loaded, the producer waits for the done flags of
//     the chunk holding the item's last row in both 64-channel chains of its
//     head (every row a tile of that item loads lies at or before its last
//     query).
// The other CTAs attend from the start; a scan CTA attends once the chunk
// tickets run out, so the attention of the first query tiles overlaps the
// rest of the scan, and it finds rows of h_k/h_v in L2 soon after the scan
// stored them.
//
// No CTA waits on one that may not be running: a scan CTA waits only on
// chunks of lower tickets (its look-back and its predecessor's done flag),
// which scan CTAs that already run have drawn; the scan CTAs are the first
// CTAs to start; the attention waits only on chunks.  Every wait is bounded;
// on expiry the CTA records RATP_ERR_TIMEOUT and sets the launch's abort word,
// which ends every other wait.
#pragma once
#include "common.cuh"
#include "scan.cuh"

namespace ratp {
namespace fused {

using Scan = scan::Params<__nv_bfloat16, 2>;

// Workspace layout (bytes), n = chunks = B * (H * 128 / 64) * ceil(T / 256):
//   [0, 256)  header: ticket word (u64 at byte 0: launch tag in the high 32
//             bits, CTA counter in the low 32; kept across launches), abort
//             word (u32 at byte 128), chunk counter (u32 at byte 132) and
//             item counter (u32 at byte 136), all zeroed before each launch
//   done u32 [n]                        chunk done flags (hold the launch tag)
//   agg, incl                           the chunk scan's descriptor words for
//                                       two streams (scan::workspace_bytes)
// Only a zero fill before the first use is needed: tag 0 is never issued.
struct Control {
  unsigned long long* ticket;
  unsigned int* counter;     // chunk tickets
  unsigned int* items;       // attention items
  int n_ctas;       // CTAs of the launch
  int n_scan;       // of which scan CTAs (the first to start)
};

__host__ __device__ inline size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

inline size_t workspace_bytes(long long n_chunks) {
  // the scan's own layout after the flags; its 256-byte header is unused
  return 256 + align256(4 * (size_t)n_chunks) + scan::workspace_bytes(n_chunks, 2);
}

// Carves the workspace into the control words, the flags and the scan's
// descriptor arrays.
inline void carve(void* base, long long n_chunks, Control* ctl, Scan* sp) {
  char* p = static_cast<char*>(base);
  ctl->ticket = reinterpret_cast<unsigned long long*>(p);
  ctl->counter = reinterpret_cast<unsigned int*>(p + 132);
  ctl->items = reinterpret_cast<unsigned int*>(p + 136);
  sp->ws = scan::carve(p + 256 + align256(4 * (size_t)n_chunks), n_chunks, 2);
  sp->ws.ticket = ctl->ticket;
  sp->ws.abort = reinterpret_cast<unsigned int*>(p + 128);
  sp->done = reinterpret_cast<unsigned int*>(p + 256);
}
constexpr size_t kResetOffset = 128, kResetBytes = 64;   // abort word and the two counters

__device__ __forceinline__ unsigned int ld_acquire(const unsigned int* p) {
  unsigned int v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ bool aborted(const unsigned int* abort_word) {
  unsigned int v;
  asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(abort_word) : "memory");
  return v != 0u;
}
__device__ __forceinline__ void abort_all(unsigned int* abort_word) { atomicExch(abort_word, 1u); }

// Scan role: the whole CTA (256 threads) scans chunk after chunk until the
// chunk tickets run out or a wait gives up (the abort word is then set).  `smem` is 128-byte aligned and
// holds scan::Smem<bf16, 2>::kBytes.
__device__ __forceinline__ void scan_role(const CUtensorMap& tm_g, const CUtensorMap& tm_xk,
                                          const CUtensorMap& tm_xv, const Scan& sp, const Control& ctl,
                                          uint8_t* smem, unsigned int tag) {
  __shared__ __align__(8) uint64_t s_bar;
  __shared__ unsigned int s_chunk;
  const uint32_t bar = sm100::smem_u32(&s_bar);
  if (threadIdx.x == 0) {
    sm100::mbar_init(bar, 1);
    sm100::fence_barrier_init();
  }
  const unsigned int n_chunks = (unsigned int)(sp.n_chains * sp.n_chunks_t);
  for (uint32_t it = 0;; ++it) {
    // the previous chunk's last barrier (inside scan_chunk) ordered every
    // read of s_chunk and of the staged tiles before this write and the next
    // TMA copy
    if (threadIdx.x == 0) s_chunk = atomicAdd(ctl.counter, 1u);
    __syncthreads();
    const unsigned int c = s_chunk;
    if (c >= n_chunks) break;
    if (!scan::scan_chunk<__nv_bfloat16, 2, scan::kRows, false, true>(tm_g, tm_xk, tm_xv, sp, smem, bar,
                                                                      it & 1u, c, tag)) {
      // copies still in flight land (bounded) before the shared memory is
      // reused
      if (threadIdx.x == 0) {
        const unsigned long long t1 = global_ns();
        while (!sm100::mbar_try_wait(bar, it & 1u) && global_ns() - t1 < spin_timeout()) {}
      }
      break;
    }
  }
}

}  // namespace fused
}  // namespace ratp
