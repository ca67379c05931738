/*
 * kvpop.h -- C ABI for KVpop future-attention targets on NVIDIA B200 (sm_100a).
 *
 * KVpop trains a per-KV-head token scorer against a future-attention target:
 * the softmax probability that later queries give a token, counted only from
 * the step at which the token is no longer among the W most recent positions.
 * The target is computed during training by a transposed attention pass, so
 * the dense attention map is never formed
 * (aiweekly article "KVpop shrinks Qwen3 KV cache 88%", second paragraph;
 * KVpop paper summary; French article, second paragraph).  At inference the
 * cache keeps sink tokens, the protected recent window and the scored top-k
 * of the older tokens (Qwen3-8B-KVpop-4x model card, introduction:
 * 4 sink + 3,772 scored + 256 recent = 4,032 entries per head).
 *
 * Definitions used by every call (one packed sequence of length L; positions
 * i, j relative to the sequence's start; G = n_q_heads / n_kv_heads; query
 * head g reads KV head g / G; s = the softmax scale):
 *
 *   lse[g, i]    = ln sum_{j <= i} exp(s * q[i, g, :] . k[j, g/G, :])
 *   target[h, j] = sum_{g : g/G = h} sum_{i = j+W}^{L-1} exp(s * q[i,g,:] . k[j,h,:] - lse[g, i])
 *
 * Key j has left the recent window of W positions exactly when the query is
 * at i >= j + W; target[h, j] = 0 for j >= L - W.
 *
 * Memory layouts (row-major, no padding, element strides as written):
 *   q       bf16  [T, n_q_heads,  head_dim]      T = cu_seqlens[batch]
 *   k       bf16  [T, n_kv_heads, head_dim]
 *   lse     fp32  [n_q_heads,  T]                natural logarithm
 *   target  fp32  [n_kv_heads, T]
 *   keep    uint8 [n_kv_heads, T]                1 = kept, 0 = evicted
 *
 * Ownership: every pointer is owned by the caller.  Device pointers must stay
 * valid until the enqueued work has finished.  Calls are stream-ordered: they
 * validate on the host, enqueue on `stream` (a cudaStream_t, NULL = legacy
 * default stream) on the current device and return without synchronising.
 * Device pointers must point into the current device's memory and `stream`
 * must belong to that device; the library does not look a pointer's device
 * up, so memory of another GPU would be read as a peer address.
 * The library allocates no device memory and keeps no mutable state besides
 * per-device caches (SM count, capability, kernel attributes).
 *
 * Errors: a call returns KVPOP_ERR_INVALID_ARG or KVPOP_ERR_UNSUPPORTED before
 * touching the device when an argument is bad; KVPOP_ERR_CUDA when the CUDA
 * runtime reports an error (cudaGetLastError after the launch).  Kernels that
 * wait on on-chip barriers give every wait a time limit (1 s, or the number
 * of nanoseconds in the environment variable KVPOP_WAIT_NS, 1e3 .. 6e10, when
 * it is set at the call); when one runs out the kernel writes a nonzero code
 * into *dev_status, stops its work early and exits cleanly;
 * kvpop_check_device_status() maps that word to KVPOP_ERR_TIMEOUT.
 * kvpop_last_error() gives a one-line description of the last failure on the
 * calling thread.
 *
 * Tracing: every call that enqueues work wraps its host work and launches in
 * an NVTX range named after the call (seen by Nsight tools when one is
 * attached, a no-op otherwise).
 */
#ifndef KVPOP_H_
#define KVPOP_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define KVPOP_ABI_VERSION 3

#if defined(__GNUC__)
#define KVPOP_API __attribute__((visibility("default")))
#else
#define KVPOP_API
#endif

typedef enum {
  KVPOP_OK = 0,
  KVPOP_ERR_INVALID_ARG = 1,   /* null pointer, bad size, inconsistent cu_seqlens, ... */
  KVPOP_ERR_UNSUPPORTED = 2,   /* head_dim not 64/128, too many sequences or tokens, non-sm_100 device */
  KVPOP_ERR_CUDA = 3,          /* CUDA runtime error (launch, copy, device query) */
  KVPOP_ERR_TIMEOUT = 4,       /* a kernel's bounded on-chip wait ran out (from kvpop_check_device_status) */
  KVPOP_ERR_BOUNDS = 5         /* debug build only: a kernel's index check failed (see kvpop_debug_set_word) */
} kvpop_status;

/* Problem shape.  cu_seqlens (host memory, int32 [batch + 1]) holds the packed
 * sequence offsets: cu_seqlens[0] = 0, non-decreasing, cu_seqlens[batch] =
 * total_tokens.  Zero-length sequences are allowed. */
typedef struct {
  int32_t batch;          /* number of packed sequences, 1 .. 512 */
  int32_t total_tokens;   /* T, >= 0; every sequence at most 131072 tokens */
  int32_t n_q_heads;      /* >= 1, a multiple of n_kv_heads */
  int32_t n_kv_heads;     /* >= 1 */
  int32_t head_dim;       /* 64 or 128 */
} kvpop_shape;

/* Row logsumexp, the normaliser of every causal softmax row (first of the two
 * passes; the transposed pass below needs it to normalise without the row).
 *   q, k        device, bf16, 16-byte aligned, layouts above
 *   cu_seqlens  HOST int32 [batch + 1]
 *   scale       softmax scale s (finite, > 0; 1/sqrt(head_dim) for the workloads)
 *   lse         device fp32 [n_q_heads, T], written for every (g, i)
 *   dev_status  device int32 or NULL; receives a nonzero code if a wait times out
 * Accuracy: the exponentials are fp32, 3 of every 16 from a degree-3
 * polynomial (relative error at most 8.6e-5), the rest from the hardware
 * exp2; sums in fp32.  |lse - exact| stays within 2e-4 (tested on every row
 * of the workloads and edge shapes); a target moves by about that relative
 * amount, well inside its 2e-3 bound.  A row whose scores lie far outside
 * the fp32 range of the fast path (a first key tile summing outside
 * [2^-64, 2^64) at offset 0, or a later tile past 2^64 above the running
 * offset: score spreads beyond ~40-90 nats) takes an exact path for that
 * tile, its scores recomputed on CUDA cores: slower, equally accurate.
 * Runs as CTA pairs: each M = 256 MMA is shared by two SMs.
 */
KVPOP_API kvpop_status kvpop_row_lse(const void* q, const void* k, const int32_t* cu_seqlens,
                           kvpop_shape shape, float scale, float* lse,
                           int32_t* dev_status, void* stream);

/* Device workspace (bytes) of kvpop_future_target and kvpop_future_targets:
 * the normaliser rows of the transposed pass, 16 bytes per (query head,
 * token), rounded up to 256; 0 for T = 0. */
KVPOP_API size_t kvpop_target_workspace_bytes(kvpop_shape shape);

/* Future-attention target: the transposed pass.  Each CTA owns a tile of 128
 * keys of one KV head and streams the query tiles i >= j + W of all G query
 * heads of its group, so the sum over queries and over the GQA group stays
 * inside one thread per key (the pages name the target's computation a
 * transposed attention pass: aiweekly article, second paragraph).  A first small kernel turns lse into the rows
 * that the tensor cores subtract from every score (lse_i / s as three bf16
 * parts, 16 bytes a row); they travel beside each query tile in one bulk copy.
 *   window      W >= 0, the protected recent window
 *   lse         device fp32 [n_q_heads, T] from kvpop_row_lse with the same q, k, scale
 *   target      device fp32 [n_kv_heads, T], written for every (h, j)
 *   workspace   device, >= kvpop_target_workspace_bytes(shape) bytes, 16-byte
 *               aligned; contents on entry are ignored
 * other arguments as for kvpop_row_lse. */
KVPOP_API kvpop_status kvpop_future_target(const void* q, const void* k, const int32_t* cu_seqlens,
                                 kvpop_shape shape, float scale, int32_t window,
                                 const float* lse, float* target, void* workspace,
                                 size_t workspace_bytes, int32_t* dev_status, void* stream);

/* Device workspace (bytes) of kvpop_future_target_split: the normaliser rows
 * (kvpop_target_workspace_bytes) followed by n_q_heads * 4 * T floats of
 * partial sums (per query head and softmax column group). */
KVPOP_API size_t kvpop_target_split_workspace_bytes(kvpop_shape shape);

/* kvpop_future_target with one work item per (key tile, query head) instead
 * of per (key tile, KV head): for few KV heads per call (a group of heads, a
 * tensor-parallel shard) the G-fold larger item count keeps every SM busy.
 * Each item writes per-head partial sums to the workspace; a second kernel
 * adds them in the order the one-item-per-KV-head pass uses, so `target` is
 * bit-identical to kvpop_future_target's.  With G = 1 it is that call.
 *   workspace  device, >= kvpop_target_split_workspace_bytes(shape) bytes,
 *              16-byte aligned; contents on entry are ignored
 * Other arguments as for kvpop_future_target. */
KVPOP_API kvpop_status kvpop_future_target_split(const void* q, const void* k, const int32_t* cu_seqlens,
                                                 kvpop_shape shape, float scale, int32_t window, const float* lse,
                                                 float* target, void* workspace, size_t workspace_bytes,
                                                 int32_t* dev_status, void* stream);

/* Sink + top-k + recent-window keep set (model card, introduction; French
 * article, second paragraph).  Per sequence b and KV head h: keep p < sinks,
 * keep p >= L - window, and among p in [sinks, L - window) keep the
 * budget[b] - sinks - window largest scores, equal scores going to the
 * smaller position first and NaN ranking below every number (-0 equals +0).
 * Everything is kept when L <= budget[b].
 *   score    device fp32 [n_kv_heads, T] (any values; normally the target)
 *   budgets  HOST int32 [batch], each >= sinks + window
 *   keep     device uint8 [n_kv_heads, T]
 * This kernel has no on-chip waits and takes no status word. */
KVPOP_API kvpop_status kvpop_keep_mask(const float* score, const int32_t* cu_seqlens, kvpop_shape shape,
                             int32_t window, int32_t sinks, const int32_t* budgets,
                             uint8_t* keep, void* stream);

/* Prefix top-k eviction thresholds (model card, "Usage" note: the scorer's
 * "prefix top-k thresholds").  At decoding step t (relative to the sequence
 * start) the tokens p in [sinks, t - window] have left the recent window and
 * compete for the k = budget[b] - sinks - window scored slots.  Per sequence
 * b, KV head h and step t the threshold is the k-th best of them in the keep
 * order (higher score first, then smaller position; NaN below every number,
 * -0 equal to +0); a token is kept at step t iff it ranks at or above it.
 * With fixed scores this equals online eviction of the worst token whenever
 * the scored slots overflow, and at the last step it selects the same tokens
 * as kvpop_keep_mask.
 *   score      device fp32 [n_kv_heads, T]
 *   budgets    HOST int32 [batch], each >= sinks + window
 *   thr_score  device fp32 [n_kv_heads, T]: the threshold token's score
 *              (-0 reported as +0); -inf while fewer than k tokens compete
 *              (nothing evicted yet); +inf when k = 0 (nothing kept)
 *   thr_pos    device int32 [n_kv_heads, T]: its position relative to the
 *              sequence start, or -1 in the two cases above
 * No on-chip waits, no status word. */
KVPOP_API kvpop_status kvpop_prefix_topk_thresholds(const float* score, const int32_t* cu_seqlens,
                                                    kvpop_shape shape, int32_t window, int32_t sinks,
                                                    const int32_t* budgets, float* thr_score,
                                                    int32_t* thr_pos, void* stream);

/* Static fixed-budget cache (model card, "Cache backends": a cache of fixed
 * size whose slots hold the same three shares as the keep mask: sinks, the
 * scored top-k and the recent window). */
typedef struct {
  int32_t batch;          /* sequences, 1 .. 512 */
  int32_t n_q_heads;      /* a multiple of n_kv_heads, at most 16 per KV head, group a power of two */
  int32_t n_kv_heads;
  int32_t head_dim;       /* 64 or 128 */
  int32_t capacity;       /* cache slots per (sequence, KV head), >= 1 */
} kvpop_cache_shape;

/* Compaction: per sequence b and KV head h, the positions with keep = 1 (in
 * increasing order) fill slots 0, 1, ... of the fixed cache.
 *   k, v       device bf16 [T, n_kv_heads, head_dim], 16-byte aligned
 *   keep       device uint8 [n_kv_heads, T] (normally from kvpop_keep_mask)
 *   capacity   slots per (b, h); a row with more kept positions keeps its first
 *              `capacity` and still reports its full count
 *   k_cache, v_cache  device bf16 [batch, n_kv_heads, capacity, head_dim], 16-byte aligned;
 *              unused slots are zero-filled
 *   pos        device int32 [batch, n_kv_heads, capacity]: the source position
 *              (relative to the sequence start) of each slot, -1 when unused
 *   count      device int32 [batch, n_kv_heads]: kept positions per row
 * shape.n_q_heads is ignored; no status word (no on-chip waits).  The kernel
 * is launched as a programmatic dependent of the stream's previous kernel: it
 * may start while that kernel finishes and waits for it (griddepcontrol.wait)
 * before reading any global memory, so stream order holds as usual. */
KVPOP_API kvpop_status kvpop_compact_kv(const void* k, const void* v, const uint8_t* keep,
                                        const int32_t* cu_seqlens, kvpop_shape shape, int32_t capacity,
                                        void* k_cache, void* v_cache, int32_t* pos, int32_t* count,
                                        void* stream);

/* Device workspace (bytes) kvpop_decode_attention needs for `shape`. */
KVPOP_API size_t kvpop_decode_workspace_bytes(kvpop_cache_shape shape);

/* One decode step over the compacted cache: for sequence b and query head g
 * (KV head h = g / G),
 *   out[b, g, :] = sum_{s < n} softmax_s(scale * q[b, g, :] . k_cache[b, h, s, :]) v_cache[b, h, s, :]
 * with n = min(count[b, h], capacity); n = 0 gives out = 0 and lse = -inf.
 *   q          device bf16 [batch, n_q_heads, head_dim], 16-byte aligned
 *   k_cache, v_cache, count  as written by kvpop_compact_kv
 *   out        device fp32 [batch, n_q_heads, head_dim]
 *   lse        device fp32 [batch, n_q_heads] natural log, or NULL
 *   workspace  device, >= kvpop_decode_workspace_bytes(shape) bytes, 16-byte aligned;
 *              holds the per-split partial results (its contents on entry are ignored)
 * Split-K over the cache slots (128 per CTA, staged in shared memory), and
 * one merge kernel when a row is split over several CTAs; both launched as
 * programmatic dependents of the kernel before them in the stream (each waits
 * for it before reading global memory); no on-chip spin waits. */
KVPOP_API kvpop_status kvpop_decode_attention(const void* q, const void* k_cache, const void* v_cache,
                                              const int32_t* count, kvpop_cache_shape shape, float scale,
                                              float* out, float* lse, void* workspace, size_t workspace_bytes,
                                              void* stream);

/* kvpop_decode_attention without a workspace argument, for callers that may
 * not allocate device memory when they run a decode step: for example code
 * whose device memory is all owned by another framework's allocator or a
 * pre-reserved pool (a stray cudaMalloc would fail or fragment it), decode
 * loops where cudaMalloc's device-wide synchronisation costs too much, or
 * plugin hooks whose interface hands them no scratch buffer.  The pages have
 * no counterpart: this is a deployment variant, not part of the method.
 *
 * The split partials go to one fixed scratch array of 4 MiB that is part of
 * the library's device image, so every GPU on which the library runs holds
 * those 4 MiB until the process exits.  Shapes whose partials exceed it
 * (batch * n_q_heads * ceil(capacity / 128) * (head_dim + 2) * 4 bytes)
 * return KVPOP_ERR_UNSUPPORTED; use kvpop_decode_attention for them.
 *
 * The first call on each device looks up the array's device address
 * (cudaGetSymbolAddress, with that device current) and caches it; make that
 * first call before any stream capture.  The cache remembers which context
 * the address belongs to: the first call after that context is destroyed
 * (cudaDeviceReset, say) looks the address up again.  The call never calls cudaMalloc or cudaFree.  Every call
 * uses the same array and leaves its partials there; nothing in it needs to
 * start at zero, because each call writes every partial it later reads.
 * Calls that overlap on the GPU (for example on two streams at once) race on
 * the array, so issue them one after another, e.g. on one stream per device.
 * Each process has its own copy of the array.
 * Other arguments and results as for kvpop_decode_attention. */
KVPOP_API kvpop_status kvpop_decode_attention_noalloc(const void* q, const void* k_cache, const void* v_cache,
                                                      const int32_t* count, kvpop_cache_shape shape, float scale,
                                                      float* out, float* lse, void* stream);

/* The whole hot path on device buffers: row logsumexp, transposed pass, keep
 * mask, enqueued back to back on `stream`.  lse is written as a by-product;
 * the row-logsumexp pass also writes the transposed pass's normaliser rows
 * into `workspace` (device, >= kvpop_target_workspace_bytes(shape) bytes,
 * 16-byte aligned, contents on entry ignored), so no conversion kernel runs. */
KVPOP_API kvpop_status kvpop_future_targets(const void* q, const void* k, const int32_t* cu_seqlens,
                                  kvpop_shape shape, float scale, int32_t window, int32_t sinks,
                                  const int32_t* budgets, float* lse, float* target,
                                  uint8_t* keep, void* workspace, size_t workspace_bytes,
                                  int32_t* dev_status, void* stream);

/* Device workspace (bytes) of kvpop_future_targets_fused: one int32 readiness
 * counter per (query head, 128-row tile of each sequence) plus two, rounded
 * up to 256 bytes (the counter block), then the normaliser rows
 * (kvpop_target_workspace_bytes). */
KVPOP_API size_t kvpop_fused_workspace_bytes(const int32_t* cu_seqlens, kvpop_shape shape);

/* The same three results as kvpop_future_targets with both attention passes
 * in ONE cooperative launch (then the keep-mask launch).  Each CTA runs its
 * share of the row-logsumexp pass and then of the transposed pass; before
 * the transposed pass reads a query tile's lse it waits (at most 1 s, then a
 * KVPOP_ERR_TIMEOUT code in *dev_status) for the CTAs that write it, through
 * counters in `workspace`.  lse, target and keep are bit-identical to those
 * of kvpop_future_targets.
 *   workspace  device, >= kvpop_fused_workspace_bytes(cu_seqlens, shape) bytes,
 *              16-byte aligned; its counter block must be ZERO-FILLED before
 *              the first call, and a launch that completes leaves it
 *              zero-filled again (after a timeout or a failed launch, zero
 *              it again before reuse); the rows after it are scratch.  Calls
 *              that share one workspace must not overlap on the GPU.
 * Other arguments as for kvpop_future_targets. */
KVPOP_API kvpop_status kvpop_future_targets_fused(const void* q, const void* k, const int32_t* cu_seqlens,
                                                  kvpop_shape shape, float scale, int32_t window, int32_t sinks,
                                                  const int32_t* budgets, float* lse, float* target,
                                                  uint8_t* keep, void* workspace, size_t workspace_bytes,
                                                  int32_t* dev_status, void* stream);

/* Device workspace (bytes) that kvpop_future_targets_host needs for `shape`. */
KVPOP_API size_t kvpop_host_workspace_bytes(kvpop_shape shape);

/* The whole hot path on HOST buffers: copies q and k (host, preferably pinned)
 * into `workspace` (device, at least kvpop_host_workspace_bytes(shape) bytes,
 * 256-byte aligned), runs the three passes and copies target and keep back to
 * host memory.  The KV heads are processed in up to eight groups of nearly
 * equal size (every head's result depends only on its own K head and query
 * heads): each group's passes run on `stream` as soon as its copy in has
 * landed, while the next group is copied in.  The copies in and back run on
 * two internal streams that the library creates once per device.  The
 * copies in wait for the work already queued on `stream` (which may still
 * read the workspace), and `stream` waits for the last copy back, so the
 * results are valid once `stream` has been synchronised.  Consecutive calls
 * with two workspaces (and host outputs) on two streams overlap: the copies
 * in of one run, in order on the internal stream, while the other computes.
 * Results are identical to kvpop_future_targets on device copies of q and k. */
KVPOP_API kvpop_status kvpop_future_targets_host(const void* q_host, const void* k_host,
                                       const int32_t* cu_seqlens, kvpop_shape shape,
                                       float scale, int32_t window, int32_t sinks,
                                       const int32_t* budgets, float* target_host,
                                       uint8_t* keep_host, void* workspace,
                                       size_t workspace_bytes, int32_t* dev_status,
                                       void* stream);

/* Synchronises `stream`, reads *dev_status and maps it: 0 -> KVPOP_OK, a
 * kernel wait that ran out -> KVPOP_ERR_TIMEOUT.  The word is not cleared. */
KVPOP_API kvpop_status kvpop_check_device_status(const int32_t* dev_status, void* stream);

/* Self-test of the bounded wait: one CTA waits on an on-chip barrier that
 * nothing ever completes, gives up after `limit_ns` nanoseconds (1 .. 1e9)
 * and writes its timeout code into *dev_status.  Used by the tests to show a
 * wait that runs out ends in an error status, not a hang. */
KVPOP_API kvpop_status kvpop_selftest_bounded_wait(int32_t* dev_status, uint64_t limit_ns, void* stream);

/* Bounds checks of the debug build (libkvpop_debug.so, the same sources
 * compiled with KVPOP_DEBUG; future_attention_targets_b200/build.py builds
 * it beside libkvpop.so).  There, every kernel checks the index of each
 * data-dependent global or shared-memory access against the extent it may
 * touch before making it; a failed check skips the access (nothing traps)
 * and writes, if the word is still 0,
 *   KVPOP_ERR_BOUNDS | check site << 8 | kernel << 16
 * into the device word registered here.  One word per process, used by
 * every later launch on any device until replaced (NULL stops recording);
 * it must be device memory of the device the kernels run on, zero-filled
 * by the caller, and read after the launches finish (or passed to
 * kvpop_check_device_status).  Not part of the method: a testing aid.
 * The ordinary library returns KVPOP_ERR_UNSUPPORTED from both calls. */
KVPOP_API kvpop_status kvpop_debug_set_word(int32_t* dev_word);

/* Debug build: one kernel makes a single index check that fails by design
 * (an index one past the extent it declares; the access it guards is
 * skipped) so that a test can see the code arrive in *dev_word. */
KVPOP_API kvpop_status kvpop_debug_selftest(int32_t* dev_word, void* stream);

KVPOP_API const char* kvpop_status_string(kvpop_status status);
KVPOP_API const char* kvpop_last_error(void);
KVPOP_API int32_t kvpop_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* KVPOP_H_ */
