/*
 * exactattn.h -- C ABI of the exact IO-aware attention forward for NVIDIA
 * B200 (sm_100a).
 *
 * The operation (Hacker News discussion item 40939398, the answer on GQA and
 * sliding windows; "Flash Attention" concept note (heepie.pages.dev), AS-IS
 * and TO-BE diagrams):
 *
 *     O   = softmax(scale * Q K^T + mask) V
 *     LSE = per-row natural-log log-sum-exp of scale * Q K^T + mask
 *
 * computed tile by tile on chip with a running row maximum and row sum, so
 * the N x N score matrix never reaches device memory (same note, "Tiling";
 * FlashAttention quiz (aiunderstanding.org), questions 3-5).
 *
 * Layouts (row-major, innermost index last, no padding):
 *     q   [B, N, Hq,  d]      k, v [B, N, Hkv, d]
 *     o   [B, N, Hq,  d]      lse  [B, Hq, N]  (fp32)
 * Query head h reads key/value head h / (Hq / Hkv) (grouped-query attention).
 * Mask: key j is visible to query i iff (causal == 0 || j <= i) and
 * (window <= 0 || j > i - window).
 *
 * Element formats (ea_dtype):
 *     EA_BF16      q, k, v bf16; o bf16; fp32 accumulation.
 *     EA_FP8_E4M3  q, k, v e4m3 codes with fp32 per-head scales q_scale[Hq],
 *                  k_scale[Hkv], v_scale[Hkv] (real value = code * scale);
 *                  o bf16.  The probabilities enter the second product as e4m3.
 *     EA_FP32      q, k, v fp32; o fp32.  Each operand is split into a bf16
 *                  high part and a bf16 remainder inside the library and the
 *                  products hi*hi + hi*lo + lo*hi run on the bf16 tensor
 *                  cores (d = 64 only).
 *
 * Ownership: every pointer passed to attn_fwd is a device pointer owned by
 * the caller and must stay valid until the work queued on `stream` has
 * finished.  The library owns only per-device state created on first use: an
 * error word, cached launch attributes, and a device memory pool from which
 * each EA_FP32 call takes its split-operand scratch in stream order (the pool
 * keeps its memory between calls); attn_shutdown() frees all of it.
 *
 * Errors: functions return an ea_status.  Argument errors are detected
 * synchronously before anything is queued.  Launches are asynchronous; a
 * device-side failure (a pipeline wait that ran past its time limit) is
 * recorded in the device error word and reported by attn_get_last_error().
 * No function aborts the process or traps the GPU.
 *
 * Thread safety: calls may come from several host threads.  Creating the
 * per-device state and the one-time launch set-up of each kernel run under
 * internal locks (concurrent first calls on a device do them once); after
 * that, calls take no lock, and launches on one stream are ordered by that
 * stream.  attn_set_option changes process-wide settings and should not race
 * with calls; attn_shutdown must not race with any call.
 */
#ifndef EXACTATTN_H
#define EXACTATTN_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  EA_BF16 = 0,
  EA_FP8_E4M3 = 1,
  EA_FP32 = 2
} ea_dtype;

typedef enum {
  EA_OK = 0,
  EA_EINVAL = -1,          /* bad argument: shape, null/host pointer, scale, window */
  EA_EUNSUPPORTED = -2,    /* valid request this build has no kernel for (e.g. d = 96) */
  EA_EALIGN = -3,          /* a pointer is not 16-byte aligned (needed by the tensor copies) */
  EA_ELAUNCH = -4,         /* the CUDA launch itself failed */
  EA_EDEVICE_TIMEOUT = -5, /* a device-side pipeline wait ran past its limit */
  EA_ECUDA = -6,           /* another CUDA runtime / driver error */
  EA_ENOMEM = -7           /* library scratch could not be allocated */
} ea_status;

/*
 * attn_fwd -- queue one attention forward on `stream`.
 *
 *   q, k, v   device pointers in the layouts above, 16-byte aligned.
 *   o         device output [B, N, Hq, d]: bf16 for EA_BF16 / EA_FP8_E4M3,
 *             fp32 for EA_FP32.  16-byte aligned.
 *   lse       device output [B, Hq, N] fp32 (natural log), 4-byte aligned.
 *   B, Hq, Hkv, N, d   sizes; B, Hq, Hkv, N >= 1, Hq % Hkv == 0.
 *             d in {64, 128} for EA_BF16 and EA_FP8_E4M3, d == 64 for EA_FP32.
 *             Hq * N and Hkv * N must stay below 2^31.
 *   causal    0 or 1.
 *   window    <= 0: no sliding window; else each query sees at most the
 *             `window` most recent keys (with causal) -- keys j > i - window.
 *   scale     finite and > 0 (typically 1/sqrt(d)).
 *   dtype     an ea_dtype value.
 *   q_scale, k_scale, v_scale   device fp32 per-head scales, required for
 *             EA_FP8_E4M3 ([Hq], [Hkv], [Hkv]); must be NULL otherwise.
 *   stream    a cudaStream_t (NULL = legacy default stream).
 *
 * Returns EA_OK once the work is queued, or an error code with nothing
 * queued.
 */
int attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
             int B, int Hq, int Hkv, int N, int d, int causal, int window, float scale,
             int dtype, const float* q_scale, const float* k_scale, const float* v_scale,
             void* stream);

/*
 * attn_fwd_masked -- attn_fwd with a per-row key range on top of the
 * causal and window masks.
 *
 * What it computes: the same O and LSE, where the mask -- what decides which
 * queries see which keys (Hacker News discussion, item 40939398) -- also
 * holds one contiguous range of visible keys per query row, the simplest
 * form of the richer masks of the FlashMask work that "FlashAttention-2
 * (PL)" lists in its literature section.  Query row i of batch b sees key j
 * iff key_lo[b*N + i] <= j < key_hi[b*N + i] and the causal / window
 * conditions of attn_fwd hold.  Examples: packed documents (key_lo = the
 * row's document start, key_hi = its end, causal = 1), a prefix-LM mask
 * (key_lo = 0, key_hi = max(prefix, i + 1), causal = 0), a sliding window
 * that varies by row.
 *
 *   key_lo, key_hi  device int32 arrays [B, N] (row-major), 4-byte aligned,
 *                   owned by the caller, shared by all heads; any values
 *                   (ranges are clipped to [0, N); lo >= hi: no key).
 *   all other arguments as attn_fwd.
 *
 * A row that sees no key gets O = 0 and LSE = -inf.  The cost follows the
 * visible keys: each 128-row query tile visits only the K/V tiles spanned by
 * its rows' ranges (a small kernel reduces the ranges per tile first, into
 * stream-ordered scratch from the library's pool that goes back to the pool
 * after the launch; the same scratch holds the counter from which the CTAs
 * take their work items, see EA_OPT_ITEM_DEAL).
 *
 * Errors: those of attn_fwd, plus EA_EINVAL for a NULL key_lo / key_hi or
 * arrays that are not device allocations of B*N int32, EA_EALIGN for
 * misaligned ones, EA_ENOMEM when the pool cannot supply the tile table.
 */
int attn_fwd_masked(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv, int N,
                    int d, int causal, int window, const int32_t* key_lo, const int32_t* key_hi, float scale,
                    int dtype, const float* q_scale, const float* k_scale, const float* v_scale, void* stream);

/*
 * attn_bwd -- queue the backward pass of attn_fwd (bf16) on `stream`: the
 * gradients dQ, dK, dV of a scalar loss whose gradient with respect to O is
 * dO.
 *
 * What it computes: with P = softmax(scale Q K^T + mask) recomputed tile by
 * tile from Q, K and the forward's LSE (the N x N probabilities are never
 * stored: "Flash Attention" concept note (heepie.pages.dev), "Tiling" and
 * "FLOP != speed"), the chain rule of the forward definition:
 *     dV = P^T dO,  dP = dO V^T,  D = rowsum(dO o O),  dS = P o (dP - D),
 *     dQ = scale dS K,  dK = scale dS^T Q
 * with the query heads of a group summed into their key/value head's dK, dV.
 *
 *   q, k, v   the forward's inputs, bf16, layouts as attn_fwd.
 *   o, lse    the forward's outputs for the same q, k, v, causal, window and
 *             scale: o bf16 [B, N, Hq, d], lse fp32 [B, Hq, N].
 *   dout      dL/dO, bf16 [B, N, Hq, d].
 *   dq        output bf16 [B, N, Hq, d];  dk, dv  outputs bf16 [B, N, Hkv, d].
 *   B, Hq, Hkv, N, d, causal, window, scale   as attn_fwd; dtype must be
 *             EA_BF16; d is 64 or 128.
 *   stream    cudaStream_t (NULL = default stream); the call is asynchronous.
 * All pointers are device pointers owned by the caller; q, k, v, o, dout, dq,
 * dk, dv 16-byte aligned, lse 4-byte aligned.
 *
 * Memory: 8 bytes per query row and head of per-row statistics come
 * stream-ordered from the library's pool and go back to it on the stream.
 * Results are deterministic: every gradient element is accumulated by one
 * CTA in a fixed order (no atomics).
 *
 * Errors (returned synchronously, nothing queued): EA_EINVAL for NULL
 * pointers, non-positive sizes, Hq not a multiple of Hkv, causal not 0/1, a
 * non-positive or non-finite scale, an unknown dtype, sizes past the limits
 * of attn_fwd, or buffers that are not device allocations large enough;
 * EA_EUNSUPPORTED for fp8/fp32 inputs or d other than 64/128; EA_EALIGN;
 * EA_ENOMEM when the pool cannot supply the statistics; EA_ECUDA without a
 * usable sm_100 device; EA_ELAUNCH if a launch fails.  A device-side wait
 * that runs past its limit is reported by attn_get_last_error.
 */
int attn_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dout, void* dq,
             void* dk, void* dv, int B, int Hq, int Hkv, int N, int d, int causal, int window, float scale, int dtype,
             void* stream);

/*
 * attn_bwd_masked -- attn_bwd for a forward run by attn_fwd_masked: the same
 * gradients with the per-row key ranges key_lo / key_hi ([B, N] int32,
 * device, shared by all heads; row i of batch b sees keys key_lo <= j <
 * key_hi, intersected with causal and window) as the mask.  Pass the same
 * ranges as the forward.  Rows that see no key contribute nothing; keys no
 * row sees get dK = dV = 0.  The per-tile ranges (the forward's tile table
 * and, for the dK/dV kernel, the span of query tiles that see each key
 * tile) are computed by two small kernels into pool scratch, which also
 * holds the two kernels' work-item counters (see EA_OPT_ITEM_DEAL).
 * Arguments and errors: those of attn_bwd, plus EA_EINVAL for a NULL range
 * array or one that is not a device allocation of B*N int32, EA_EALIGN for
 * one that is not 4-byte aligned.
 */
int attn_bwd_masked(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dout,
                    void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int N, int d, int causal, int window,
                    const int32_t* key_lo, const int32_t* key_hi, float scale, int dtype, void* stream);

/*
 * attn_get_last_error -- synchronise `stream`, then read and clear the
 * current device's error word.  *device_code receives 0 or the recorded
 * failure kind (1 = wait timed out), *site the pipeline wait that failed
 * (either pointer may be NULL).  Returns EA_OK, EA_EDEVICE_TIMEOUT, or
 * EA_ECUDA if synchronising the stream reported a CUDA error.
 */
int attn_get_last_error(void* stream, int* device_code, int* site);

/* attn_status_string -- static, human-readable name of an ea_status. */
const char* attn_status_string(int status);

/*
 * attn_set_option -- process-wide tuning and test hooks (host state only):
 *   EA_OPT_WAIT_TIMEOUT_NS  limit for every device-side pipeline wait
 *                           (default 2e9 ns).
 *   EA_OPT_MAX_CTAS         cap on persistent CTAs per launch (0 = one per SM).
 *   EA_OPT_SCHEDULE_ORDER   0 = heaviest query blocks first (default),
 *                           1 = lightest first, 2 = with per-row key ranges,
 *                           (batch, query block) pairs ranked by the K/V
 *                           tiles they visit, most first (better balance
 *                           across SMs, less reuse of K/V in L2; otherwise
 *                           as 0).  Results do not depend on it.
 *   EA_OPT_SKIP_ARRIVE_ONCE test hook: the next launch's load warp skips its
 *                           first key/value copy, so the consumer's bounded
 *                           wait runs out and reports EA_EDEVICE_TIMEOUT.
 *   EA_OPT_ITEM_DEAL        0 (default) = with per-row key ranges (forward
 *                           with order 0, and backward), each CTA takes its
 *                           next work item from a global counter when it
 *                           starts one (dynamic deal: the costs of ranged
 *                           items follow no order, so a static deal leaves
 *                           SMs idle); 1 = the static boustrophedon deal
 *                           everywhere.
 *   Results depend on neither the order nor the deal (each work item's
 *   arithmetic is the same wherever it runs).
 * Returns EA_OK or EA_EINVAL.
 */
enum {
  EA_OPT_WAIT_TIMEOUT_NS = 1,
  EA_OPT_MAX_CTAS = 2,
  EA_OPT_SCHEDULE_ORDER = 3,
  EA_OPT_SKIP_ARRIVE_ONCE = 4,
  EA_OPT_ITEM_DEAL = 5
};
int attn_set_option(int option, long long value);

/* attn_shutdown -- free all per-device library state (call after the
 * streams that used it are idle) and forget attn_fwd_fp32_noalloc's
 * per-device set-up.  Returns EA_OK or EA_ECUDA. */
int attn_shutdown(void);

/* attn_version -- library ABI version (major * 10000 + minor * 100 + patch). */
int attn_version(void);

/*
 * attn_fwd_fp32_noalloc -- the EA_FP32 forward of attn_fwd for callers that
 * cannot allocate device memory.  (The pages have no counterpart; this is a
 * deployment variant.)  Such callers include code embedded in a host process
 * whose own memory manager has reserved the device memory and forbids or
 * cannot satisfy allocations from libraries, and runtimes that require a
 * fixed device-memory footprint known at load time.  attn_fwd's fp32 path
 * takes its split operands from a device memory pool that the library
 * creates and grows on demand; this variant keeps them instead in one
 * statically allocated device array of
 * EA_NOALLOC_SCRATCH_BYTES that every GPU which loads the library holds
 * until the process exits.  It calls no cudaMalloc, cudaFree or allocating
 * library routine; the caller still passes all inputs and outputs.
 *
 *   q, k, v, o, lse, B, Hq, Hkv, N, d, causal, window, scale, stream:
 *             as attn_fwd with dtype EA_FP32 (fp32 in, fp32 O, d == 64).
 *   status    optional device int (NULL allowed): cleared on `stream`, then
 *             set to (kind << 16) | site if a device-side pipeline wait runs
 *             past its limit.  attn_get_last_error does not see this variant,
 *             so without a status word such a timeout goes unreported and the
 *             outputs of that call are undefined: pass a status word.
 *
 * Scratch needed: 384 * B*N*Hq + 640 * B*N*Hkv bytes (each of the three
 * parts rounded up to 256 bytes) plus 256; a request above
 * EA_NOALLOC_SCRATCH_BYTES returns EA_EINVAL with nothing queued.
 * The first call on a device is a set-up call: with that device current it
 * looks up the array's device address (with lazy module loading the CUDA
 * runtime places the array on the device at that point) and synchronises
 * the device once; make that first call before any stream capture.
 * attn_shutdown() forgets that set-up, so the next call on each device is a
 * set-up call again.  Every call shares the one array and overwrites the part
 * it uses before reading it, so calls whose work overlaps on the GPU
 * (different streams, or different host threads) race: serialise them.
 */
#define EA_NOALLOC_SCRATCH_BYTES (16u * 1024u * 1024u)
int attn_fwd_fp32_noalloc(const float* q, const float* k, const float* v, float* o, float* lse, int B, int Hq,
                          int Hkv, int N, int d, int causal, int window, float scale, int* status, void* stream);

/*
 * attn_fwd_decode -- the same exact attention for Nq new query rows against a
 * key/value cache of Nk >= Nq rows (a decode step), computed by splitting the
 * keys across warps and merging the parts' results with their log-sum-exps.
 *
 * What it computes: the pages' softmax(scale Q K^T + mask) V with its
 * per-row log-sum-exp ("Flash Attention" concept note, AS-IS diagram; Hacker
 * News discussion, item 40939398), key blocks combined through their
 * normalisation factors ("Flash Attention" note, TO-BE diagram and "Tiling"
 * section), split across parallel workers as in the decoding work the pages
 * list by title (FlashDecoding++).  Query row i is the token at position
 * Nk - Nq + i (the new tokens end the sequence): with causal = 1 it sees keys
 * 0 .. Nk - Nq + i; with window > 0 only keys j > Nk - Nq + i - window.
 *
 * Arguments and layout (all device pointers, d contiguous, caller-owned):
 *   q    [B, Nq, Hq, d]  bf16        o    [B, Nq, Hq, d]  bf16 (written)
 *   k, v [B, Nk, Hkv, d] bf16        lse  [B, Hq, Nq]     fp32 (written, natural log)
 *   dtype must be EA_BF16; d is 64 or 128; (Hq / Hkv) * Nq <= 32 query rows
 *   per key/value head (<= 8 with num_splits > 0; larger query blocks: use
 *   attn_fwd).
 *   num_splits: 0 (recommended) runs the tensor-core kernel: one persistent
 *   CTA per SM, the K/V tiles of all (batch, key/value head) pairs split
 *   into equal contiguous ranges, each pair's query rows in the first rows
 *   of a 128-row tcgen05 tile; > 0 runs the CUDA-core kernel with that many
 *   key ranges per (batch, key/value head).  Results of the two kernels and
 *   of different split counts agree within rounding; each is deterministic
 *   for given sizes.
 *   stream: cudaStream_t (NULL = default stream); the call is asynchronous.
 *
 * Memory: the partial results (per range and query row: 2 + d floats) come
 * stream-ordered from the library's memory pool and go back to it on the
 * stream; attn_shutdown() releases the pool.
 *
 * Errors (returned synchronously, nothing queued): EA_EINVAL for NULL
 * pointers, non-positive sizes, Nq > Nk, Hq not a multiple of Hkv, causal not
 * 0/1, a non-positive or non-finite scale, an unknown dtype, negative
 * num_splits, or a buffer that is not one device allocation large enough;
 * EA_EUNSUPPORTED for fp8/fp32 inputs, d other than 64/128, or more query
 * rows per key/value head than the chosen kernel takes; EA_EALIGN unless q, k, v, o are 16-byte and
 * lse 4-byte aligned; EA_ENOMEM when the pool cannot supply the partials;
 * EA_ECUDA without a usable sm_100 device; EA_ELAUNCH if a launch fails.
 */
int attn_fwd_decode(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv, int Nq,
                    int Nk, int d, int causal, int window, float scale, int dtype, int num_splits, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* EXACTATTN_H */
