/*
 * ratp.h -- C ABI of the B200 (sm_100a) RAT+ sequence-mixer library.
 *
 * The library computes the data-parallel hot path of RAT+ ("RAT+: Train
 * Dense, Infer Sparse -- Recurrence Augmented Attention for Dilated
 * Inference", arXiv 2602.18196):
 *
 *   1. the full-sequence forget-gate recurrence over the key and value
 *      streams, h_t = g_t * h_{t-1} + (1 - g_t) * x_t per channel, h_{-1} = 0
 *      (zhichai.net write-up "RAT+ 深度拆解", section 2.1: forget-gate
 *      recurrence over the whole sequence, parallel associative scan at
 *      prefill);
 *   2. causal softmax attention of query t over the recurrent keys/values at
 *      S_D(t) = { j < t : j mod D = D-1 } U { t }, optionally united with the
 *      window { j : t-W < j <= t } (RAT+ abstract: dilated attention of
 *      dilation D cuts attention FLOPs and the KV cache by D, optionally with
 *      local windows; write-up section 1);
 *   3. head-wise hybrids: heads flagged in head_mask run dense (D = 1)
 *      (write-up section 6: the first heads dense, the rest dilated).
 *
 * Conventions for every entry point:
 *   - Tensors are dense, row-major, on the current CUDA device, and owned by
 *     the caller.  Prefill tensors are [B][T][H][Dh]; decode tensors are
 *     [B][H][Dh].  Every device pointer must be 16-byte aligned.
 *   - dtype is RATP_F32 or RATP_BF16 for all tensor arguments of one call
 *     (recurrent state and final states are always fp32).  Arithmetic is fp32.
 *   - stream is a cudaStream_t (NULL = legacy default stream).  Calls are
 *     stream-ordered and asynchronous; none synchronises the host except
 *     ratp_last_error().
 *   - Return value: RATP_OK (0) or a ratp_status code.  Argument errors are
 *     detected on the host before any launch and leave outputs untouched.
 *     Asynchronous device-side errors (a bounded wait that ran out, a cache
 *     append beyond capacity) are recorded in a per-device error word that
 *     ratp_last_error() returns.  The library never aborts the process.
 *   - The library allocates no device memory.  Scratch space is passed in by
 *     the caller (sizes from the *_bytes queries).
 */
#ifndef RATP_H_
#define RATP_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum ratp_status {
  RATP_OK = 0,
  RATP_ERR_ARG = 1,         /* null pointer, negative size, bad enum */
  RATP_ERR_SHAPE = 2,       /* unsupported shape (Dh, H, sizes)        */
  RATP_ERR_ALIGN = 3,       /* pointer not 16-byte aligned            */
  RATP_ERR_CAPACITY = 4,    /* workspace/cache too small, cache full  */
  RATP_ERR_TIMEOUT = 5,     /* a bounded device wait ran out          */
  RATP_ERR_CUDA = 6,        /* a CUDA runtime/driver call failed      */
  RATP_ERR_UNSUPPORTED = 7, /* dtype/shape combination not built      */
  RATP_ERR_BOUNDS = 8       /* guarded build only: an access outside its
                               buffer was skipped (ratp_guard_line)    */
} ratp_status;

typedef enum ratp_dtype { RATP_F32 = 0, RATP_BF16 = 1 } ratp_dtype;

/* Largest head count accepted by head_mask-taking calls. */
#define RATP_MAX_HEADS 256

/* Human-readable name of a status code (static string). */
const char* ratp_status_string(int status);

/* Reads and clears the device error word of the current device after
 * synchronising `stream`.  Returns RATP_OK or the lowest-numbered error
 * recorded by any kernel since the previous call. */
int ratp_last_error(void* stream);

/* Number of SMs of the current device (grid sizing). */
int ratp_device_sm_count(int* sms);

/* Failure injection for tests of the error paths; never needed otherwise.
 * Affects launches issued afterwards on the current device.
 *   RATP_FAULT_NONE          restore the defaults (arg ignored);
 *   RATP_FAULT_SPIN_LIMIT    bound, in ns, of every device-side wait
 *                            (default 2e9); arg <= 0 restores the default;
 *   RATP_FAULT_SCAN_DROP     the scan chunk with launch ticket `arg` publishes
 *                            no descriptor, so its successor's wait runs out;
 *   RATP_FAULT_ATTN_DROP_K   the first CTA of the tensor-core attention never
 *                            loads its K tile number `arg`, so the MMA's wait
 *                            runs out;
 *   RATP_FAULT_FUSED_DROP_CHUNK  the fused prefill never raises the done
 *                            flag of scan chunk `arg` (chunk = (b * H*Dh/64
 *                            + channel/64) * ceil(T/256) + t/256), so the
 *                            waits on it run out.
 * A wait that runs out ends its kernel early with RATP_ERR_TIMEOUT in the
 * device error word (outputs are then undefined); the context stays usable.
 * Returns RATP_ERR_ARG for an unknown kind, RATP_ERR_CUDA if the device
 * update fails.  Not thread-safe with concurrent launches. */
enum { RATP_FAULT_NONE = 0, RATP_FAULT_SPIN_LIMIT = 1, RATP_FAULT_SCAN_DROP = 2,
       RATP_FAULT_ATTN_DROP_K = 3, RATP_FAULT_FUSED_DROP_CHUNK = 4 };
int ratp_debug_fault(int kind, long long arg);

/* ------------------------------------------------------------------------
 * Guarded debug build (libratp_guarded.so, compiled with -DRATP_GUARDED; a
 * stand-in for a memory checker).  Every global access a kernel addresses
 * itself is range-checked against its buffer; an access outside it is
 * skipped and RATP_ERR_BOUNDS is set in the device error word.
 * ratp_guard_line: *line receives (and the call clears) the source line of
 *   the first refused access, 0 if none.  Returns RATP_ERR_UNSUPPORTED (and
 *   *line = 0) in the normal build, so a caller can tell the builds apart.
 * ratp_debug_guard_probe: guarded build only; one thread asks for element 4
 *   of a 4-element device array, which the guard refuses (nothing is
 *   written): the error word then holds RATP_ERR_BOUNDS.  The normal build
 *   returns RATP_ERR_UNSUPPORTED and launches nothing.
 * ---------------------------------------------------------------------- */
int ratp_guard_line(int* line);
int ratp_debug_guard_probe(void* stream);

/* ------------------------------------------------------------------------
 * Prefill recurrence (write-up section 2.1).
 *
 * ratp_scan_workspace_bytes: bytes of device scratch that one scan call of
 *   this shape needs (chunk descriptors of the single-pass scan).
 * ratp_scan_prefill: h = scan(x, g) over T for every (b, channel);
 *   x, g, h: [B][T][H][Dh] of dtype.  final_state (nullable): fp32 [B][H][Dh],
 *   receives h_{T-1} in fp32.
 * ratp_scan_prefill_kv: the key and value streams in one pass with one gate
 *   tensor (g is read once): hk = scan(xk, g), hv = scan(xv, g).
 *   final_state (nullable): fp32 [2][B][H][Dh] (k then v) -- the layout of the
 *   decode state.
 * workspace: device scratch of at least ratp_scan_workspace_bytes.  It must
 *   be zero-filled once before its first use; every call leaves it valid for
 *   the next one: each call clears its abort word on `stream` first, its
 *   kernel returns the ticket counter to zero, and it tags the chunk
 *   descriptors with a fresh number kept in the workspace itself (so a call
 *   replayed from a CUDA graph gets a fresh tag as well; tags repeat after
 *   2^32 - 1 calls on one workspace).  Calls sharing one workspace must be
 *   ordered on one stream.
 *   h may alias x (in-place) only when T == 1.
 * Errors: ARG (null, B/T/H/Dh < 0), SHAPE (H*Dh not a multiple of 64), ALIGN,
 *   CAPACITY (workspace too small).  T == 0 or B == 0 is a no-op.
 * ---------------------------------------------------------------------- */
int ratp_scan_workspace_bytes(int B, int T, int H, int Dh, int dtype, size_t* bytes);
int ratp_scan_prefill(const void* x, const void* g, void* h, float* final_state,
                      int B, int T, int H, int Dh, int dtype,
                      void* workspace, size_t workspace_bytes, void* stream);
int ratp_scan_prefill_kv(const void* xk, const void* xv, const void* g,
                         void* hk, void* hv, float* final_state,
                         int B, int T, int H, int Dh, int dtype,
                         void* workspace, size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------
 * Chunk-local recurrence (the original RAT, which section 2.1 of the
 * zhichai.net write-up "RAT+ 深度拆解" describes as the method RAT+ replaces:
 * the sequence is cut into blocks of L tokens and each token recurs only
 * inside its own block; there L = D).
 *
 * h_t = g_t * h_{t-1} + (1 - g_t) * x_t, with h_{t-1} taken as 0 whenever
 * t mod L == 0; positions count from 0 at the first token of x.
 * Arguments, layouts, workspace and errors are those of ratp_scan_prefill /
 * ratp_scan_prefill_kv, plus L: L >= 1 is the block length; L == 0 (or any
 * L >= T) gives the full-sequence recurrence; L < 0 is RATP_ERR_ARG.
 * final_state receives h_{T-1}; a decode that continues from it must use a
 * cache with the same L (ratp_cache_set_chunk_local).
 * ---------------------------------------------------------------------- */
int ratp_scan_prefill_chunk_local(const void* x, const void* g, void* h, float* final_state,
                                  int B, int T, int H, int Dh, int dtype, int L,
                                  void* workspace, size_t workspace_bytes, void* stream);
int ratp_scan_prefill_kv_chunk_local(const void* xk, const void* xv, const void* g,
                                     void* hk, void* hv, float* final_state,
                                     int B, int T, int H, int Dh, int dtype, int L,
                                     void* workspace, size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------
 * Fixed look-back recurrence (section 2.1 of the zhichai.net write-up: the
 * recurrence window L* = 64 of the RAT+ design before it moved to the full
 * sequence).  Prefill only.
 *
 * h_t = the recurrence h = g h + (1 - g) x started from zero at position
 * max(0, t - L + 1) and run to t, for the key and value streams with one
 * gate tensor.  xk, xv, g, hk, hv: [B][T][H][Dh] of dtype (bf16 or fp32),
 * device pointers, 16-byte aligned; hk, hv are written, nothing else is.
 * L: 16, 32 or 64 (L >= T gives the full-sequence recurrence).  No
 * workspace: every 256-token chunk is computed from its own tokens and the
 * L before it.
 * Errors: ARG (L < 1, null pointer, negative size, bad dtype), UNSUPPORTED
 *   (another L), SHAPE (H*Dh not a multiple of 64), ALIGN.  B, T or H == 0
 *   is a no-op.  Decode continues it through a cache with a window attached
 *   (ratp_cache_set_window, ratp_cache_pack_inputs).
 * ---------------------------------------------------------------------- */
int ratp_scan_prefill_kv_window(const void* xk, const void* xv, const void* g,
                                void* hk, void* hv, int B, int T, int H, int Dh, int dtype,
                                int L, void* stream);

/* ------------------------------------------------------------------------
 * Allocation-free variant of ratp_scan_prefill_kv.  The paper has no
 * counterpart: this is a convenience of the library.
 *
 * It serves callers that must not allocate device memory themselves and so
 * cannot hand in the scratch workspace that ratp_scan_prefill_kv needs --
 * for example a plug-in running inside a host application whose memory pool
 * owns every device byte, or a latency-critical path where cudaMalloc's
 * implicit device-wide synchronisation is not acceptable.  The scratch is a
 * fixed array of RATP_NOALLOC_SCRATCH_BYTES (16 MiB) compiled into the
 * library's device image; every device that loads the library holds it until
 * the process exits.  Inputs, outputs and errors are those of
 * ratp_scan_prefill_kv (the caller still provides and owns all tensors), and
 * the call itself performs no allocation of any kind.
 *   - A shape whose scratch would not fit returns RATP_ERR_CAPACITY
 *     (at most 6,553 chunks of 64 channels x 256 tokens for bf16, i.e.
 *     B*T*H*Dh up to ~107 million elements; fp32 chunks hold 128 tokens,
 *     ~53 million elements).
 *   - The first call on a device looks up the array's device address with
 *     that device current; make that first call before any stream capture.
 *     The address is kept for the life of the process: after
 *     cudaDeviceReset() on a device this entry point must not be called on
 *     that device again.
 *   - All calls share the one array, which keeps the previous call's
 *     contents; each call clears, on `stream`, the part that must start at
 *     zero.  Calls that can run at the same time on the GPU (for example on
 *     two unordered streams) race on the array and produce wrong results.
 * ---------------------------------------------------------------------- */
#define RATP_NOALLOC_SCRATCH_BYTES (16u << 20)
int ratp_scan_prefill_kv_noalloc(const void* xk, const void* xv, const void* g,
                                 void* hk, void* hv, float* final_state,
                                 int B, int T, int H, int Dh, int dtype, void* stream);

/* ------------------------------------------------------------------------
 * Dilated (+ windowed) prefill attention (RAT+ abstract; write-up sections 1
 * and 6).
 *
 * o[b][t][h] = sum_{j in K_h(t)} softmax_j(q[b][t][h] . hk[b][j][h] / sqrt(Dh))
 *              * hv[b][j][h]
 * K_h(t) = { j < t : j mod D_h = D_h-1 } U { t } U { j : t-W < j <= t }
 * (each key once), D_h = 1 where head_mask[h] != 0, else D.
 *
 * q, hk, hv, o: [B][T][H][Dh] of dtype.  D >= 1, W >= 0 (0 = no window).
 * head_mask: HOST array of H bytes, or NULL (no dense heads).
 * ratp_dilated_attn_prefill dispatches bf16 with Dh == 128 to the tensor-core
 * kernel (TMA + tcgen05.mma, accumulators in tensor memory) and every other
 * supported case (fp32; Dh 64) to the CUDA-core kernel.
 * ratp_dilated_attn_prefill_simt always runs the CUDA-core kernel
 * (fp32 or bf16, Dh in {64, 128}).
 * Errors: ARG, SHAPE (Dh not 64/128, H > RATP_MAX_HEADS), ALIGN, CUDA.
 * ---------------------------------------------------------------------- */
int ratp_dilated_attn_prefill(const void* q, const void* hk, const void* hv, void* o,
                              int B, int T, int H, int Dh, int D, int W,
                              const uint8_t* head_mask, int dtype, void* stream);
int ratp_dilated_attn_prefill_simt(const void* q, const void* hk, const void* hv, void* o,
                                   int B, int T, int H, int Dh, int D, int W,
                                   const uint8_t* head_mask, int dtype, void* stream);

/* Same computation as ratp_dilated_attn_prefill, with an optional workspace:
 * device memory of at least RATP_ATTN_WORKSPACE_BYTES, 16-byte aligned, no
 * initialisation needed (each call clears what it uses, on `stream`).  With
 * it, a tensor-core launch that mixes dense and dilated work (a head_mask
 * with dense heads and D > 1) hands its work items to CTAs as they become
 * free instead of in fixed rounds, which balances items of very different
 * cost; launches of one kind are unchanged.  NULL behaves as
 * ratp_dilated_attn_prefill.  Calls sharing one workspace must be ordered on
 * one stream.  Errors: as ratp_dilated_attn_prefill; ALIGN for a misaligned
 * workspace. */
#define RATP_ATTN_WORKSPACE_BYTES 256u
int ratp_dilated_attn_prefill_ws(const void* q, const void* hk, const void* hv, void* o,
                                 int B, int T, int H, int Dh, int D, int W,
                                 const uint8_t* head_mask, int dtype, void* workspace, void* stream);

/* ------------------------------------------------------------------------
 * Fused prefill: the recurrence of both streams and the dilated (+ windowed,
 * head-wise hybrid) attention over it in one launch (the full-sequence
 * recurrence of the write-up's section 2.1 feeding the dilated attention of
 * its section 1 and of the RAT+ abstract).
 *
 * Computes what ratp_scan_prefill_kv followed by ratp_dilated_attn_prefill
 * computes: hk = scan(xk, g), hv = scan(xv, g), final_state = the fp32 state
 * at position T-1 ([2][B][H][Dh], k then v; nullable), and o = attention of q
 * over hk, hv with dilation D, window W and head_mask (HOST array of H bytes,
 * nonzero = dense head; or NULL).  Inside the launch, the CTAs that start
 * first run the chunk scan of ratp_scan_prefill_kv (256 tokens x 64 channels
 * per chunk, in sequence order) and raise a done flag per chunk; the others
 * run the tensor-core attention over query tiles in ascending order and wait
 * (bounded) for the flags of the chunks holding the rows they load.  The
 * look-back of the scan composes a timing-dependent number of chunk maps,
 * and the attention places its key tiles differently, so results agree with
 * the two separate calls to rounding, not bit for bit.
 * q, xk, xv, g, hk, hv, o: [B][T][H][Dh] bf16, Dh = 128, device, 16-byte
 * aligned; hk and hv are written (they are outputs, and the attention reads
 * its keys back from them, mostly out of L2).
 * workspace: device scratch of ratp_prefill_fused_workspace_bytes bytes,
 *   zero-filled once before its first use; like the scan workspace it tags
 *   its descriptors and flags with a fresh number per call, kept in the
 *   workspace itself, and calls sharing one workspace must be ordered on one
 *   stream.
 * Errors: ARG, SHAPE, ALIGN, CAPACITY (workspace too small), UNSUPPORTED
 *   (not bf16 or Dh != 128).  B, T or H == 0 is a no-op.  A bounded wait that
 *   ran out sets RATP_ERR_TIMEOUT in the device error word (outputs are then
 *   undefined).
 * ---------------------------------------------------------------------- */
int ratp_prefill_fused_workspace_bytes(int B, int T, int H, int Dh, size_t* bytes);
int ratp_prefill_fused(const void* q, const void* xk, const void* xv, const void* g,
                       void* hk, void* hv, void* o, float* final_state,
                       int B, int T, int H, int Dh, int D, int W, const uint8_t* head_mask, int dtype,
                       void* workspace, size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------
 * Per-sample dilation in one launch (the batch composition of the write-up's
 * section 2.2 "Active Recurrence Learning": in one batch, half the samples
 * run dense, D = 1, and half dilated, D = 64; forward only).
 *
 * o[b] = ratp_dilated_attn_prefill of sample b alone with D = D_per_sample[b]
 * (same W and head_mask for every sample): a sample with D = 1 is dense in
 * every head; in the others, heads with head_mask[h] != 0 stay dense.
 * D_per_sample: host array of B int32 values >= 1, read during the call only.
 * Tensors as for ratp_dilated_attn_prefill; bf16 with Dh = 128 only.
 * Errors: ARG (a D < 1, D_per_sample NULL with B > 0, ...), ALIGN,
 *   SHAPE (B > 1024), UNSUPPORTED (fp32 or Dh = 64, or more than 4 distinct
 *   values D > 1 in one call).  B, T or H == 0 is a no-op.
 * ---------------------------------------------------------------------- */
int ratp_dilated_attn_prefill_per_sample(const void* q, const void* hk, const void* hv, void* o,
                                         int B, int T, int H, int Dh, const int32_t* D_per_sample,
                                         int W, const uint8_t* head_mask, int dtype, void* stream);
/* With the optional workspace of ratp_dilated_attn_prefill_ws (the same
 * rules); a batch that mixes dense and dilated samples is dealt dynamically. */
int ratp_dilated_attn_prefill_per_sample_ws(const void* q, const void* hk, const void* hv, void* o,
                                            int B, int T, int H, int Dh, const int32_t* D_per_sample,
                                            int W, const uint8_t* head_mask, int dtype, void* workspace,
                                            void* stream);

/* ------------------------------------------------------------------------
 * D-compressed KV cache and decode (RAT+ abstract: the KV cache shrinks by D).
 *
 * Layout (all bf16 rows of Dh elements):
 *   Kc/Vc: dilated rows.  Head h keeps the recurrent key/value of position
 *          p = s*D_h + D_h - 1 in slot s < cap_h = T_max / D_h.  Row of
 *          (b, h, s) = b * rows_per_b + sum_{h' < h} cap_{h'} + s.
 *   Kw/Vw: window ring, [B][H][W][Dh]; position p sits in row p mod W.
 *          Absent (NULL) when W == 0.
 *   len:   int32 [B], the number of tokens absorbed per sequence (the
 *          position of the next token).
 *   partial, counters: decode split-K scratch.  counters must be zero when
 *          a decode step starts; ratp_cache_init zeroes them and every step
 *          leaves them zero.
 * The struct is plain data filled by ratp_cache_init; the caller owns the
 * buffer it points into.
 * ---------------------------------------------------------------------- */
typedef struct ratp_cache {
  void* Kc;
  void* Vc;
  void* Kw;
  void* Vw;
  int32_t* len;
  float* partial;
  uint32_t* counters;
  void* in_ring;        /* fixed look-back decode: ring of the last window_L inputs,
                           bf16 [3][B][H][window_L][Dh] (x_k, x_v, g); NULL if unused */
  int64_t rows_per_b;   /* sum_h cap_h */
  int32_t B, H, Dh, T_max, D, W;
  int32_t split_keys;   /* keys per decode split */
  int32_t max_splits;   /* most decode splits any head can need (partial rows per (b, h)) */
  int32_t reset_L;      /* chunk-local recurrence block (0 = full sequence); set by
                           ratp_cache_set_chunk_local */
  int32_t window_L;     /* fixed look-back window (0 = none); set by ratp_cache_set_window */
  uint8_t dense[RATP_MAX_HEADS];
} ratp_cache;

/* Bytes of the single device buffer that holds a cache of this shape. */
int ratp_cache_bytes(int B, int H, int Dh, int T_max, int D, int W,
                     const uint8_t* head_mask, size_t* bytes);

/* Carves `buffer` (device, >= ratp_cache_bytes) into the cache regions,
 * fills *c, and zeroes len and the counters on `stream`.
 * Dh must be 128 or 64, dtype is bf16.  Errors: ARG, SHAPE, ALIGN, CAPACITY. */
int ratp_cache_init(ratp_cache* c, void* buffer, size_t bytes,
                    int B, int H, int Dh, int T_max, int D, int W,
                    const uint8_t* head_mask, void* stream);

/* Prefill -> decode hand-off: copies the dilated rows of hk, hv (bf16
 * [B][T][H][Dh], T <= T_max) into Kc/Vc, the last min(W, T) positions into
 * the ring, and sets len[b] = T.  The recurrent state comes from the scan's
 * final_state (ratp_scan_prefill_kv writes the [2][B][H][Dh] decode layout). */
int ratp_cache_pack(ratp_cache* c, const void* hk, const void* hv, int T, void* stream);

/* Selects the recurrence that ratp_decode_step continues: L == 0 (the
 * default that ratp_cache_init sets) is the full-sequence recurrence; L >= 1
 * is the chunk-local recurrence of ratp_scan_prefill_kv_chunk_local, whose
 * state restarts at every position t with t mod L == 0.  Host-only: writes
 * c->reset_L and launches nothing.  Errors: ARG (null c, L < 0, or L > 0
 * with a look-back window attached). */
int ratp_cache_set_chunk_local(ratp_cache* c, int L);

/* Decode of the fixed look-back recurrence (ratp_scan_prefill_kv_window): the
 * step needs the inputs of the last L positions, kept in a caller-owned ring.
 * ratp_cache_window_bytes: bytes of that ring, 3 * B * H * L * Dh bf16
 *   (x_k, x_v, g; position p in slot p mod L).
 * ratp_cache_set_window: attaches `ring` (device, >= the bytes above,
 *   16-byte aligned) and L (1 <= L <= 256) to the cache; L == 0 detaches.
 *   Host-only.  A cache cannot be both chunk-local and look-back (ARG).
 * ratp_cache_pack_inputs: prefill -> decode hand-off of the inputs: copies
 *   positions max(0, T-L) .. T-1 of xk, xv, g (bf16 [B][T][H][Dh], device)
 *   into the ring (T <= T_max; call after ratp_cache_pack with the same T).
 * With a window attached, ratp_decode_step first writes the step's inputs
 * into slot t mod L, then computes the new recurrent key/value as the
 * recurrence from zero over positions max(0, t-L+1) .. t read from the ring
 * (O(L) per channel, in split 0) instead of the one-step update; it also
 * stores that value in `state`.
 * Errors: ARG, ALIGN, CAPACITY (ring too small, T > T_max). */
int ratp_cache_window_bytes(int B, int H, int Dh, int L, size_t* bytes);
int ratp_cache_set_window(ratp_cache* c, void* ring, size_t bytes, int L);
int ratp_cache_pack_inputs(ratp_cache* c, const void* xk, const void* xv, const void* g, int T,
                           void* stream);

/* One decode token for every sequence (fused): state <- g*state + (1-g)*x for
 * the key and value streams (fp32 state [2][B][H][Dh], in/out; the state is
 * first zeroed where t mod c->reset_L == 0 for a chunk-local cache); the new
 * recurrent key/value is appended to Kc/Vc when t mod D_h == D_h - 1 and
 * always written to the ring; o = attention of q over the cached dilated
 * slots s < t / D_h, the window positions t-W < p < t not among them, and the
 * new key/value itself; len[b] += 1.
 * q, xk, xv, g, o: bf16 [B][H][Dh].  D, W, head_mask must equal the values
 * the cache was initialised with (ERR_ARG otherwise).  A token beyond T_max
 * sets RATP_ERR_CAPACITY in the device error word and leaves that sequence
 * unchanged. */
int ratp_decode_step(const void* q, const void* xk, const void* xv, const void* g,
                     float* state, ratp_cache* c, void* o,
                     int D, int W, const uint8_t* head_mask, void* stream);

/* ------------------------------------------------------------------------
 * Decode token step of a stack of layers (layer-wise hybrid, write-up
 * section 6: a few dense layers, e.g. the input layer 0 and the middle layer
 * 12, among dilated ones).  Each layer has its own cache, so its own D, W,
 * head mask and recurrence (ratp_cache_init, ratp_cache_set_chunk_local);
 * layers may differ in all of them.
 *
 * For l = 0 .. n_layers-1 in order, performs ratp_decode_step on
 * layers[l] with the D, W and head mask of layers[l].cache, all on `stream`
 * (each launch may start while the previous layer's kernel drains and waits
 * for its completion before touching memory).  The whole call is one token
 * step and can be captured into one CUDA graph.  The array and the structs
 * are read on the host during the call only; every pointer in them is a
 * device pointer with the meaning, layout and ownership of ratp_decode_step.
 * Errors: ARG (n_layers < 0, layers NULL with n_layers > 0, a NULL field),
 * ALIGN, SHAPE; on the first failing layer the call returns its status and
 * launches no later layer (earlier layers' launches stand).
 * ---------------------------------------------------------------------- */
typedef struct ratp_decode_layer {
  const void* q;      /* bf16 [B][H][Dh] */
  const void* xk;     /* bf16 [B][H][Dh] */
  const void* xv;     /* bf16 [B][H][Dh] */
  const void* g;      /* bf16 [B][H][Dh], gates in (0, 1) */
  float* state;       /* fp32 [2][B][H][Dh], in/out */
  ratp_cache* cache;  /* this layer's cache (host struct, device buffers) */
  void* o;            /* bf16 [B][H][Dh], out */
} ratp_decode_layer;

int ratp_decode_step_layers(const ratp_decode_layer* layers, int n_layers, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* RATP_H_ */
