// Host side of the C ABI declared in include/kvpop.h: argument validation,
// TMA descriptor encoding, the longest-first work schedule, and launches.
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>
#include <nvtx3/nvToolsExt.h>
#include <stdarg.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <algorithm>
#include <atomic>
#include <mutex>
#include <string>
#include <vector>

#include "kvpop.h"
#include "kvpop_cache.h"

namespace kvpop {
cudaError_t launch_row_lse(const AttnParams& p, int head_dim, int sm_count, cudaStream_t stream);
cudaError_t launch_future_target(const AttnParams& p, int head_dim, int sm_count, cudaStream_t stream);
cudaError_t launch_keep_mask(const KeepParams& p, int n_kv_heads, int sm_count, cudaStream_t stream);
cudaError_t launch_selftest_wait(int32_t* status, uint64_t limit_ns, cudaStream_t stream);
cudaError_t launch_prefix_thresholds(const ThresholdParams& p, int n_kv_heads, int max_len, cudaStream_t stream);
cudaError_t launch_compact_kv(const CompactParams& p, cudaStream_t stream);
cudaError_t launch_decode_attention(const DecodeParams& p, int batch, cudaStream_t stream);
int decode_parts(int rows, int n_chunks, int sm_count);
cudaError_t launch_fused_targets(const FusedParams& fp, int head_dim, int grid, cudaStream_t stream);
cudaError_t launch_merge_partials(const float* part, float* target, int group, int n_kv_heads, int total_tokens,
                                  int sm_count, int32_t* dbg, cudaStream_t stream);
int target_split_groups();
cudaError_t launch_norm_rows(const float* lse, void* rows, int64_t n, float inv_scale, int sm_count, int32_t* dbg,
                             cudaStream_t stream);
size_t decode_scratch_bytes();
cudaError_t decode_scratch_address(float** out);
cudaError_t launch_debug_selftest(int32_t* word, cudaStream_t stream);
}  // namespace kvpop

using namespace kvpop;

namespace {

thread_local std::string g_last_error;

// Debug build: the device word that kernels' bounds checks write
// (kvpop_debug_set_word); every launch passes it in its parameter block.
#ifdef KVPOP_DEBUG
std::atomic<int32_t*> g_debug_word{nullptr};
int32_t* debug_word() { return g_debug_word.load(std::memory_order_relaxed); }
#else
int32_t* debug_word() { return nullptr; }
#endif

// An NVTX range named after the entry point around its host work and
// launches: Nsight tools show (and ncu can filter by) it when attached; a
// no-op otherwise.
struct TraceRange {
  explicit TraceRange(const char* name) { nvtxRangePushA(name); }
  ~TraceRange() { nvtxRangePop(); }
  TraceRange(const TraceRange&) = delete;
  TraceRange& operator=(const TraceRange&) = delete;
};
#define KVPOP_TRACE() TraceRange kvpop_trace_range_(__func__)

// Time limit of every bounded on-chip wait: KVPOP_WAIT_NS nanoseconds when
// that environment variable holds a number in [1e3, 6e10] at the call, else
// 1 s.
uint64_t wait_limit_ns() {
  const char* v = getenv("KVPOP_WAIT_NS");
  if (v != nullptr && *v != 0) {
    char* end = nullptr;
    const unsigned long long x = strtoull(v, &end, 10);
    if (end != nullptr && *end == 0 && x >= 1000ull && x <= 60000000000ull) return x;
  }
  return kDefaultWaitNs;
}

kvpop_status fail(kvpop_status st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return st;
}

kvpop_status cuda_fail(cudaError_t e, const char* what) {
  return fail(KVPOP_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

// ---------------------------------------------------------------- device info

struct DeviceInfo {
  int sm_count = 0;
  int major = 0, minor = 0;
};

kvpop_status device_info(DeviceInfo* out) {
  static std::mutex mu;
  static std::vector<DeviceInfo> cache;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  std::lock_guard<std::mutex> lock(mu);
  if (static_cast<int>(cache.size()) <= dev) cache.resize(dev + 1);
  DeviceInfo& d = cache[dev];
  if (d.sm_count == 0) {
    if ((e = cudaDeviceGetAttribute(&d.sm_count, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess ||
        (e = cudaDeviceGetAttribute(&d.major, cudaDevAttrComputeCapabilityMajor, dev)) != cudaSuccess ||
        (e = cudaDeviceGetAttribute(&d.minor, cudaDevAttrComputeCapabilityMinor, dev)) != cudaSuccess) {
      d.sm_count = 0;
      return cuda_fail(e, "cudaDeviceGetAttribute");
    }
  }
  *out = d;
  if (d.major != 10 || d.minor != 0)
    return fail(KVPOP_ERR_UNSUPPORTED, "device compute capability %d.%d; this library is built for sm_100a only",
                d.major, d.minor);
  return KVPOP_OK;
}

// ---------------------------------------------------------------- tensor maps

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                                  CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// bf16 matrix [rows, cols] (row-major, cols contiguous) read as boxes of
// 64 columns x box_rows rows with 128-byte swizzle; rows past the end read as 0.
kvpop_status make_map(CUtensorMap* m, const void* base, int64_t cols, int64_t rows, uint32_t box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (enc == nullptr) return fail(KVPOP_ERR_CUDA, "cuTensorMapEncodeTiled entry point not available");
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols) * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(KVPOP_ERR_CUDA, "cuTensorMapEncodeTiled failed (CUresult %d)", static_cast<int>(r));
  return KVPOP_OK;
}

// Normaliser rows [n_heads][T] of 16 bytes (8 bf16 values each) read as boxes
// of 128 rows of one head: rows past T read as 0 (CTA pairs, pass 2).
kvpop_status make_rows_map(CUtensorMap* m, const void* rows, int64_t T, int64_t n_heads) {
  EncodeTiledFn enc = encode_fn();
  if (enc == nullptr) return fail(KVPOP_ERR_CUDA, "cuTensorMapEncodeTiled entry point not available");
  cuuint64_t dims[3] = {8, static_cast<cuuint64_t>(T), static_cast<cuuint64_t>(n_heads)};
  cuuint64_t strides[2] = {16, static_cast<cuuint64_t>(T) * 16};
  cuuint32_t box[3] = {8, static_cast<cuuint32_t>(kTileRows), 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(rows), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS)
    return fail(KVPOP_ERR_CUDA, "cuTensorMapEncodeTiled (normaliser rows) failed (CUresult %d)", static_cast<int>(r));
  return KVPOP_OK;
}

// ---------------------------------------------------------------- validation

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

kvpop_status check_shape(const int32_t* cu, const kvpop_shape& sh, bool need_heads) {
  if (cu == nullptr) return fail(KVPOP_ERR_INVALID_ARG, "cu_seqlens is NULL");
  if (sh.batch < 1) return fail(KVPOP_ERR_INVALID_ARG, "batch must be >= 1 (got %d)", sh.batch);
  if (sh.batch > kMaxSeqs) return fail(KVPOP_ERR_UNSUPPORTED, "batch %d exceeds the %d-sequence limit", sh.batch, kMaxSeqs);
  if (sh.total_tokens < 0) return fail(KVPOP_ERR_INVALID_ARG, "total_tokens must be >= 0");
  if (sh.n_kv_heads < 1) return fail(KVPOP_ERR_INVALID_ARG, "n_kv_heads must be >= 1");
  if (need_heads) {
    if (sh.n_q_heads < 1) return fail(KVPOP_ERR_INVALID_ARG, "n_q_heads must be >= 1");
    if (sh.n_q_heads % sh.n_kv_heads != 0)
      return fail(KVPOP_ERR_INVALID_ARG, "n_q_heads (%d) is not a multiple of n_kv_heads (%d)", sh.n_q_heads,
                  sh.n_kv_heads);
    if (sh.head_dim != 64 && sh.head_dim != 128)
      return fail(KVPOP_ERR_UNSUPPORTED, "head_dim %d not supported (64 or 128)", sh.head_dim);
    if (static_cast<int64_t>(sh.n_q_heads) * sh.head_dim > (1 << 24))
      return fail(KVPOP_ERR_UNSUPPORTED, "n_q_heads * head_dim too large");
  }
  if (cu[0] != 0) return fail(KVPOP_ERR_INVALID_ARG, "cu_seqlens[0] must be 0 (got %d)", cu[0]);
  for (int b = 0; b < sh.batch; ++b) {
    const int64_t L = static_cast<int64_t>(cu[b + 1]) - cu[b];
    if (L < 0) return fail(KVPOP_ERR_INVALID_ARG, "cu_seqlens decreases at %d", b);
    if (L > static_cast<int64_t>(kMaxLevels) * kTileRows)
      return fail(KVPOP_ERR_UNSUPPORTED, "sequence %d has %lld tokens (limit %d)", b, static_cast<long long>(L),
                  kMaxLevels * kTileRows);
  }
  if (cu[sh.batch] != sh.total_tokens)
    return fail(KVPOP_ERR_INVALID_ARG, "cu_seqlens[batch] (%d) != total_tokens (%d)", cu[sh.batch],
                sh.total_tokens);
  return KVPOP_OK;
}

kvpop_status check_qk(const void* q, const void* k, float scale) {
  if (q == nullptr || k == nullptr) return fail(KVPOP_ERR_INVALID_ARG, "q or k is NULL");
  if (!aligned16(q) || !aligned16(k)) return fail(KVPOP_ERR_INVALID_ARG, "q and k must be 16-byte aligned");
  if (!isfinite(scale) || !(scale > 0.f)) return fail(KVPOP_ERR_INVALID_ARG, "scale must be finite and > 0");
  return KVPOP_OK;
}

// ---------------------------------------------------------------- schedule

// Items (level, sequence, head), heaviest level first.  Sequences with t
// blocks of block_rows rows take part in levels 0 .. t-1.
// order (optional) receives the original index of each scheduled sequence.
void build_schedule(const int32_t* cu, int batch, int n_heads, LevelSchedule* s, std::vector<int>* order = nullptr,
                    int block_rows = kTileRows) {
  std::vector<std::pair<int, int>> seqs;  // (tiles, index)
  for (int b = 0; b < batch; ++b) {
    const int L = cu[b + 1] - cu[b];
    const int t = (L + block_rows - 1) / block_rows;
    if (t > 0) seqs.emplace_back(t, b);
  }
  std::stable_sort(seqs.begin(), seqs.end(), [](const std::pair<int, int>& a, const std::pair<int, int>& b) {
    return a.first > b.first;
  });
  memset(s, 0, sizeof(*s));
  s->n_seqs = static_cast<int32_t>(seqs.size());
  s->n_heads = n_heads;
  s->n_levels = seqs.empty() ? 0 : seqs[0].first;
  for (size_t r = 0; r < seqs.size(); ++r) {
    s->seq_start[r] = cu[seqs[r].second];
    s->seq_len[r] = cu[seqs[r].second + 1] - cu[seqs[r].second];
  }
  if (order != nullptr) {
    order->clear();
    for (const auto& e : seqs) order->push_back(e.second);
  }
  int32_t running = 0;
  size_t active = 0;  // sequences with a tile at this level form a prefix of the sorted list
  for (int k = 0; k < s->n_levels; ++k) {
    const int level = s->n_levels - 1 - k;
    while (active < seqs.size() && seqs[active].first > level) ++active;
    s->level_base[k] = running;
    running += static_cast<int32_t>(active) * n_heads;
  }
  s->level_base[s->n_levels] = running;
  s->total_items = running;
}

int grid_for(int items, int sm_count) { return std::max(1, std::min(items, sm_count)); }

// cta = 1: one CTA per work item, resident (A) tiles of 128 rows and
// streamed (B) tiles of 256; cta = 2: a CTA pair per item of 256 rows, each
// CTA loading 128 rows of A and 128 rows of every B tile.
kvpop_status fill_attn_common(AttnParams* p, const void* q, const void* k, const int32_t* cu,
                              const kvpop_shape& sh, float scale, bool target_pass,
                              std::vector<int>* order = nullptr, int cta = 1) {
  memset(p, 0, sizeof(*p));
  p->dbg = debug_word();
  const int64_t T = sh.total_tokens;
  kvpop_status st;
  const uint32_t a_rows = kTileRows, b_rows = kStreamRows / cta;
  if ((st = make_map(&p->tmap_q, q, static_cast<int64_t>(sh.n_q_heads) * sh.head_dim, T,
                     target_pass ? b_rows : a_rows)) != KVPOP_OK)
    return st;
  if ((st = make_map(&p->tmap_k, k, static_cast<int64_t>(sh.n_kv_heads) * sh.head_dim, T,
                     target_pass ? a_rows : b_rows)) != KVPOP_OK)
    return st;
  p->cta = cta;
  p->q = static_cast<const uint16_t*>(q);
  p->k = static_cast<const uint16_t*>(k);
  p->wait_ns = wait_limit_ns();
  p->total_tokens = sh.total_tokens;
  p->n_q_heads = sh.n_q_heads;
  p->n_kv_heads = sh.n_kv_heads;
  p->group = sh.n_q_heads / sh.n_kv_heads;
  p->scale_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
  p->inv_scale = static_cast<float>(1.0 / static_cast<double>(scale));
  p->g_split = 1;
  build_schedule(cu, sh.batch, target_pass ? sh.n_kv_heads : sh.n_q_heads, &p->sched, order, kTileRows * cta);
  return KVPOP_OK;
}

// The standalone passes run on CTA pairs (cta = 2): each M = 256 MMA is
// shared by two SMs, which halves the B tiles every SM reads from L2 and
// feeds to its tensor core.  The single-launch variant keeps one CTA per SM.
#ifndef KVPOP_PAIR_CTAS
#define KVPOP_PAIR_CTAS 1
#endif
constexpr int kPassCtas = KVPOP_PAIR_CTAS ? 2 : 1;

// 128-row tiles of every sequence (the lse readiness flags of the single
// launch are one per query head and tile), -1 for a malformed cu_seqlens.
int64_t flag_tiles(const int32_t* cu, int batch) {
  int64_t t = 0;
  for (int b = 0; b < batch; ++b) {
    const int64_t L = static_cast<int64_t>(cu[b + 1]) - cu[b];
    if (L < 0) return -1;
    t += (L + kTileRows - 1) / kTileRows;
  }
  return t;
}

static_assert(sizeof(FusedParams) <= 32764, "kernel parameter space");

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// KV-head groups of the host-buffer pipeline (copy of group c+1 overlaps the
// compute of group c).
constexpr int kHostGroups = 8;

// Two internal streams per device for the host-buffer pipeline's copies in
// and out, created on first use and kept for the life of the process.
struct HostStreams {
  cudaStream_t in = nullptr;
  cudaStream_t out = nullptr;
};

kvpop_status host_streams(HostStreams* out) {
  static std::mutex mu;
  static std::vector<HostStreams> cache;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  std::lock_guard<std::mutex> lock(mu);
  if (static_cast<int>(cache.size()) <= dev) cache.resize(dev + 1);
  HostStreams& h = cache[dev];
  if (h.in == nullptr) {
    HostStreams n;
    if ((e = cudaStreamCreateWithFlags(&n.in, cudaStreamNonBlocking)) == cudaSuccess &&
        (e = cudaStreamCreateWithFlags(&n.out, cudaStreamNonBlocking)) == cudaSuccess) {
      h = n;
    } else {
      if (n.in != nullptr) cudaStreamDestroy(n.in);
      return cuda_fail(e, "cudaStreamCreate");
    }
  }
  *out = h;
  return KVPOP_OK;
}

// Events of one call, destroyed when the call returns (an event still pending
// on the GPU is released once it completes).
struct EventSet {
  std::vector<cudaEvent_t> ev;
  cudaError_t make(cudaEvent_t* out) {
    cudaError_t e = cudaEventCreateWithFlags(out, cudaEventDisableTiming);
    if (e == cudaSuccess) ev.push_back(*out);
    return e;
  }
  ~EventSet() {
    for (cudaEvent_t x : ev) cudaEventDestroy(x);
  }
};

}  // namespace

extern "C" {

int32_t kvpop_abi_version(void) { return KVPOP_ABI_VERSION; }

const char* kvpop_last_error(void) { return g_last_error.c_str(); }

const char* kvpop_status_string(kvpop_status s) {
  switch (s) {
    case KVPOP_OK: return "ok";
    case KVPOP_ERR_INVALID_ARG: return "invalid argument";
    case KVPOP_ERR_UNSUPPORTED: return "unsupported";
    case KVPOP_ERR_CUDA: return "CUDA error";
    case KVPOP_ERR_TIMEOUT: return "device wait timed out";
    case KVPOP_ERR_BOUNDS: return "a bounds check of the debug build failed";
  }
  return "unknown status";
}

// Bytes of the normaliser rows that the transposed pass streams beside its
// query tiles: 16 per (query head, token).
static size_t norm_rows_bytes(const kvpop_shape& shape) {
  return static_cast<size_t>(shape.n_q_heads) * static_cast<size_t>(shape.total_tokens) * 16;
}

// Pass 1 on validated device arguments; rows (nullable) also receives the
// normaliser rows of pass 2.
static kvpop_status run_row_lse(const void* q, const void* k, const int32_t* cu_seqlens, const kvpop_shape& shape,
                                float scale, float* lse, void* rows, int32_t* dev_status, cudaStream_t stream,
                                const DeviceInfo& dev) {
  AttnParams p;
  kvpop_status st;
  if ((st = fill_attn_common(&p, q, k, cu_seqlens, shape, scale, false, nullptr, kPassCtas)) != KVPOP_OK) return st;
  p.out = lse;
  p.nrm_rows = rows;
  p.status = dev_status;
  if (p.sched.total_items == 0) return KVPOP_OK;
  cudaError_t e = launch_row_lse(p, shape.head_dim, dev.sm_count, stream);
  return e == cudaSuccess ? KVPOP_OK : cuda_fail(e, "row_lse launch");
}

// Pass 2 on validated device arguments, from normaliser rows.  partials
// non-null: one item per (key tile, query head), then the ordered merge.
static kvpop_status run_target(const void* q, const void* k, const int32_t* cu_seqlens, const kvpop_shape& shape,
                               float scale, int32_t window, const void* rows, float* target, float* partials,
                               int32_t* dev_status, cudaStream_t stream, const DeviceInfo& dev) {
  AttnParams p;
  kvpop_status st;
  if ((st = fill_attn_common(&p, q, k, cu_seqlens, shape, scale, true, nullptr, kPassCtas)) != KVPOP_OK) return st;
  if (kPassCtas == 2 &&
      (st = make_rows_map(&p.tmap_rows, rows, shape.total_tokens, shape.n_q_heads)) != KVPOP_OK)
    return st;
  const int G = shape.n_q_heads / shape.n_kv_heads;
  if (partials != nullptr) {
    build_schedule(cu_seqlens, shape.batch, shape.n_kv_heads * G, &p.sched, nullptr, kTileRows * kPassCtas);
    p.g_split = G;
  }
  // A window longer than any sequence leaves every target at zero; clamp it
  // so the tile arithmetic stays in range.
  p.window = std::min<int32_t>(window, kMaxLevels * kTileRows + 1);
  p.nrm_rows = const_cast<void*>(rows);
  p.out = partials != nullptr ? partials : target;
  p.status = dev_status;
  if (p.sched.total_items == 0) return KVPOP_OK;
  cudaError_t e = launch_future_target(p, shape.head_dim, dev.sm_count, stream);
  if (e != cudaSuccess) return cuda_fail(e, "future_target launch");
  if (partials == nullptr) return KVPOP_OK;
  e = launch_merge_partials(partials, target, G, shape.n_kv_heads, shape.total_tokens, dev.sm_count, debug_word(),
                            stream);
  return e == cudaSuccess ? KVPOP_OK : cuda_fail(e, "merge of the split partials");
}

// Every sequence's budget covers its sinks and window (budgets: host [batch]).
static kvpop_status check_budgets(const int32_t* budgets, int batch, int32_t sinks, int32_t window) {
  if (budgets == nullptr) return fail(KVPOP_ERR_INVALID_ARG, "budgets is NULL");
  for (int b = 0; b < batch; ++b)
    if (static_cast<int64_t>(budgets[b]) < static_cast<int64_t>(sinks) + window)
      return fail(KVPOP_ERR_INVALID_ARG, "budget[%d] = %d is below sinks + window = %lld", b, budgets[b],
                  static_cast<long long>(sinks) + window);
  return KVPOP_OK;
}

static kvpop_status check_workspace(const void* ws, size_t bytes, size_t need, size_t align) {
  if (ws == nullptr || bytes < need)
    return fail(KVPOP_ERR_INVALID_ARG, "workspace of %zu bytes is smaller than the %zu required", bytes, need);
  if ((reinterpret_cast<uintptr_t>(ws) & (align - 1)) != 0)
    return fail(KVPOP_ERR_INVALID_ARG, "workspace must be %zu-byte aligned", align);
  return KVPOP_OK;
}

kvpop_status kvpop_row_lse(const void* q, const void* k, const int32_t* cu_seqlens, kvpop_shape shape, float scale,
                           float* lse, int32_t* dev_status, void* stream) {
  KVPOP_TRACE();
  kvpop_status st;
  if ((st = check_qk(q, k, scale)) != KVPOP_OK) return st;
  if (lse == nullptr) return fail(KVPOP_ERR_INVALID_ARG, "lse is NULL");
  if ((st = check_shape(cu_seqlens, shape, true)) != KVPOP_OK) return st;
  if (shape.total_tokens == 0) return KVPOP_OK;
  DeviceInfo dev;
  if ((st = device_info(&dev)) != KVPOP_OK) return st;
  return run_row_lse(q, k, cu_seqlens, shape, scale, lse, nullptr, dev_status, static_cast<cudaStream_t>(stream),
                     dev);
}

size_t kvpop_target_workspace_bytes(kvpop_shape shape) {
  if (shape.total_tokens <= 0 || shape.n_q_heads <= 0) return 0;
  return align256(norm_rows_bytes(shape));
}

kvpop_status kvpop_future_target(const void* q, const void* k, const int32_t* cu_seqlens, kvpop_shape shape,
                                 float scale, int32_t window, const float* lse, float* target, void* workspace,
                                 size_t workspace_bytes, int32_t* dev_status, void* stream) {
  KVPOP_TRACE();
  kvpop_status st;
  if ((st = check_qk(q, k, scale)) != KVPOP_OK) return st;
  if (lse == nullptr || target == nullptr) return fail(KVPOP_ERR_INVALID_ARG, "lse or target is NULL");
  if (window < 0) return fail(KVPOP_ERR_INVALID_ARG, "window must be >= 0 (got %d)", window);
  if ((st = check_shape(cu_seqlens, shape, true)) != KVPOP_OK) return st;
  if (shape.total_tokens == 0) return KVPOP_OK;
  if ((st = check_workspace(workspace, workspace_bytes, kvpop_target_workspace_bytes(shape), 16)) != KVPOP_OK)
    return st;
  DeviceInfo dev;
  if ((st = device_info(&dev)) != KVPOP_OK) return st;
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  const float inv_scale = static_cast<float>(1.0 / static_cast<double>(scale));
  cudaError_t e = launch_norm_rows(lse, workspace, static_cast<int64_t>(shape.n_q_heads) * shape.total_tokens,
                                   inv_scale, dev.sm_count, debug_word(), s);
  if (e != cudaSuccess) return cuda_fail(e, "normaliser rows launch");
  return run_target(q, k, cu_seqlens, shape, scale, window, workspace, target, nullptr, dev_status, s, dev);
}

size_t kvpop_target_split_workspace_bytes(kvpop_shape shape) {
  if (shape.total_tokens <= 0 || shape.n_kv_heads <= 0 || shape.n_q_heads <= 0 ||
      shape.n_q_heads % shape.n_kv_heads != 0)
    return 0;
  return kvpop_target_workspace_bytes(shape) + static_cast<size_t>(shape.n_q_heads) * target_split_groups() *
                                                   static_cast<size_t>(shape.total_tokens) * sizeof(float);
}

kvpop_status kvpop_future_target_split(const void* q, const void* k, const int32_t* cu_seqlens, kvpop_shape shape,
                                       float scale, int32_t window, const float* lse, float* target, void* workspace,
                                       size_t workspace_bytes, int32_t* dev_status, void* stream) {
  KVPOP_TRACE();
  kvpop_status st;
  if ((st = check_qk(q, k, scale)) != KVPOP_OK) return st;
  if (lse == nullptr || target == nullptr) return fail(KVPOP_ERR_INVALID_ARG, "lse or target is NULL");
  if (window < 0) return fail(KVPOP_ERR_INVALID_ARG, "window must be >= 0 (got %d)", window);
  if ((st = check_shape(cu_seqlens, shape, true)) != KVPOP_OK) return st;
  if (shape.total_tokens == 0) return KVPOP_OK;
  if ((st = check_workspace(workspace, workspace_bytes, kvpop_target_split_workspace_bytes(shape), 16)) != KVPOP_OK)
    return st;
  const int G = shape.n_q_heads / shape.n_kv_heads;
  if (G == 1)   // one query head per KV head: the split is the plain pass
    return kvpop_future_target(q, k, cu_seqlens, shape, scale, window, lse, target, workspace, workspace_bytes,
                               dev_status, stream);
  DeviceInfo dev;
  if ((st = device_info(&dev)) != KVPOP_OK) return st;
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  const float inv_scale = static_cast<float>(1.0 / static_cast<double>(scale));
  cudaError_t e = launch_norm_rows(lse, workspace, static_cast<int64_t>(shape.n_q_heads) * shape.total_tokens,
                                   inv_scale, dev.sm_count, debug_word(), s);
  if (e != cudaSuccess) return cuda_fail(e, "normaliser rows launch");
  float* partials = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + kvpop_target_workspace_bytes(shape));
  return run_target(q, k, cu_seqlens, shape, scale, window, workspace, target, partials, dev_status, s, dev);
}

kvpop_status kvpop_keep_mask(const float* score, const int32_t* cu_seqlens, kvpop_shape shape, int32_t window,
                             int32_t sinks, const int32_t* budgets, uint8_t* keep, void* stream) {
  KVPOP_TRACE();
  kvpop_status st;
  if (score == nullptr || keep == nullptr) return fail(KVPOP_ERR_INVALID_ARG, "score or keep is NULL");
  if (budgets == nullptr) return fail(KVPOP_ERR_INVALID_ARG, "budgets is NULL");
  if (window < 0 || sinks < 0) return fail(KVPOP_ERR_INVALID_ARG, "window and sinks must be >= 0");
  if ((st = check_shape(cu_seqlens, shape, false)) != KVPOP_OK) return st;
  if ((st = check_budgets(budgets, shape.batch, sinks, window)) != KVPOP_OK) return st;
  if (shape.total_tokens == 0) return KVPOP_OK;
  DeviceInfo dev;
  if ((st = device_info(&dev)) != KVPOP_OK) return st;
  KeepParams p;
  memset(&p, 0, sizeof(p));
  p.dbg = debug_word();
  p.score = score;
  p.keep = keep;
  p.total_tokens = shape.total_tokens;
  p.window = window;
  p.sinks = sinks;
  p.n_seqs = shape.batch;
  for (int b = 0; b < shape.batch; ++b) {
    p.seq_start[b] = cu_seqlens[b];
    p.seq_len[b] = cu_seqlens[b + 1] - cu_seqlens[b];
    p.budget[b] = budgets[b];
  }
  cudaError_t e = launch_keep_mask(p, shape.n_kv_heads, dev.sm_count, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? KVPOP_OK : cuda_fail(e, "keep_mask launch");
}

kvpop_status kvpop_prefix_topk_thresholds(const float* score, const int32_t* cu_seqlens, kvpop_shape shape,
                                          int32_t window, int32_t sinks, const int32_t* budgets, float* thr_score,
                                          int32_t* thr_pos, void* stream) {
  KVPOP_TRACE();
  kvpop_status st;
  if (score == nullptr || thr_score == nullptr || thr_pos == nullptr)
    return fail(KVPOP_ERR_INVALID_ARG, "score, thr_score or thr_pos is NULL");
  if (budgets == nullptr) return fail(KVPOP_ERR_INVALID_ARG, "budgets is NULL");
  if (window < 0 || sinks < 0) return fail(KVPOP_ERR_INVALID_ARG, "window and sinks must be >= 0");
  if ((st = check_shape(cu_seqlens, shape, false)) != KVPOP_OK) return st;
  if ((st = check_budgets(budgets, shape.batch, sinks, window)) != KVPOP_OK) return st;
  if (shape.total_tokens == 0) return KVPOP_OK;
  DeviceInfo dev;
  if ((st = device_info(&dev)) != KVPOP_OK) return st;
  ThresholdParams p;
  memset(&p, 0, sizeof(p));
  p.dbg = debug_word();
  p.score = score;
  p.thr_score = thr_score;
  p.thr_pos = thr_pos;
  p.total_tokens = shape.total_tokens;
  p.window = window;
  p.sinks = sinks;
  p.n_seqs = shape.batch;
  int max_len = 0;
  for (int b = 0; b < shape.batch; ++b) {
    p.seq_start[b] = cu_seqlens[b];
    p.seq_len[b] = cu_seqlens[b + 1] - cu_seqlens[b];
    p.budget[b] = budgets[b];
    max_len = std::max(max_len, p.seq_len[b]);
  }
  cudaError_t e = launch_prefix_thresholds(p, shape.n_kv_heads, max_len, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? KVPOP_OK : cuda_fail(e, "prefix thresholds launch");
}

kvpop_status kvpop_compact_kv(const void* k, const void* v, const uint8_t* keep, const int32_t* cu_seqlens,
                              kvpop_shape shape, int32_t capacity, void* k_cache, void* v_cache, int32_t* pos,
                              int32_t* count, void* stream) {
  KVPOP_TRACE();
  kvpop_status st;
  if (k == nullptr || v == nullptr || keep == nullptr || k_cache == nullptr || v_cache == nullptr ||
      pos == nullptr || count == nullptr)
    return fail(KVPOP_ERR_INVALID_ARG, "a pointer argument is NULL");
  if (!aligned16(k) || !aligned16(v) || !aligned16(k_cache) || !aligned16(v_cache))
    return fail(KVPOP_ERR_INVALID_ARG, "k, v, k_cache and v_cache must be 16-byte aligned");
  if (capacity < 1) return fail(KVPOP_ERR_INVALID_ARG, "capacity must be >= 1");
  if (shape.head_dim != 64 && shape.head_dim != 128)
    return fail(KVPOP_ERR_UNSUPPORTED, "head_dim %d not supported (64 or 128)", shape.head_dim);
  if ((st = check_shape(cu_seqlens, shape, false)) != KVPOP_OK) return st;
  DeviceInfo dev;
  if ((st = device_info(&dev)) != KVPOP_OK) return st;
  CompactParams p;
  memset(&p, 0, sizeof(p));
  p.dbg = debug_word();
  p.k = static_cast<const uint16_t*>(k);
  p.v = static_cast<const uint16_t*>(v);
  p.keep = keep;
  p.k_cache = static_cast<uint16_t*>(k_cache);
  p.v_cache = static_cast<uint16_t*>(v_cache);
  p.pos = pos;
  p.count = count;
  p.total_tokens = shape.total_tokens;
  p.n_kv_heads = shape.n_kv_heads;
  p.head_dim = shape.head_dim;
  p.capacity = capacity;
  p.n_seqs = shape.batch;
  for (int b = 0; b < shape.batch; ++b) {
    p.seq_start[b] = cu_seqlens[b];
    p.seq_len[b] = cu_seqlens[b + 1] - cu_seqlens[b];
  }
  cudaError_t e = launch_compact_kv(p, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? KVPOP_OK : cuda_fail(e, "compact_kv launch");
}

static bool check_cache_shape(const kvpop_cache_shape& sh) {
  if (sh.batch < 1 || sh.batch > kMaxSeqs || sh.n_kv_heads < 1 || sh.n_q_heads < 1 || sh.capacity < 1) return false;
  if (sh.n_q_heads % sh.n_kv_heads != 0) return false;
  const int G = sh.n_q_heads / sh.n_kv_heads;
  if (G > 16 || (G & (G - 1)) != 0) return false;
  return sh.head_dim == 64 || sh.head_dim == 128;
}

size_t kvpop_decode_workspace_bytes(kvpop_cache_shape shape) {
  if (!check_cache_shape(shape)) return 0;
  const size_t n_split = (static_cast<size_t>(shape.capacity) + kDecSplit - 1) / kDecSplit;
  return static_cast<size_t>(shape.batch) * shape.n_q_heads * n_split * (shape.head_dim + 2) * sizeof(float);
}

kvpop_status kvpop_decode_attention(const void* q, const void* k_cache, const void* v_cache, const int32_t* count,
                                    kvpop_cache_shape shape, float scale, float* out, float* lse, void* workspace,
                                    size_t workspace_bytes, void* stream) {
  KVPOP_TRACE();
  kvpop_status st;
  if (q == nullptr || k_cache == nullptr || v_cache == nullptr || count == nullptr || out == nullptr)
    return fail(KVPOP_ERR_INVALID_ARG, "a pointer argument is NULL");
  if (!aligned16(k_cache) || !aligned16(v_cache) || !aligned16(workspace))
    return fail(KVPOP_ERR_INVALID_ARG, "k_cache, v_cache and workspace must be 16-byte aligned");
  if (!aligned16(q)) return fail(KVPOP_ERR_INVALID_ARG, "q must be 16-byte aligned");
  if (!isfinite(scale) || !(scale > 0.f)) return fail(KVPOP_ERR_INVALID_ARG, "scale must be finite and > 0");
  if (!check_cache_shape(shape))
    return fail(KVPOP_ERR_UNSUPPORTED,
                "cache shape not supported (head_dim 64/128, group size a power of two <= 16, 1..512 sequences)");
  const size_t need = kvpop_decode_workspace_bytes(shape);
  if (workspace == nullptr || workspace_bytes < need)
    return fail(KVPOP_ERR_INVALID_ARG, "workspace of %zu bytes is smaller than the %zu required", workspace_bytes,
                need);
  DeviceInfo dev;
  if ((st = device_info(&dev)) != KVPOP_OK) return st;
  DecodeParams p;
  memset(&p, 0, sizeof(p));
  p.dbg = debug_word();
  p.q = static_cast<const uint16_t*>(q);
  p.k_cache = static_cast<const uint16_t*>(k_cache);
  p.v_cache = static_cast<const uint16_t*>(v_cache);
  p.count = count;
  p.partial = static_cast<float*>(workspace);
  p.out = out;
  p.lse = lse;
  p.n_q_heads = shape.n_q_heads;
  p.n_kv_heads = shape.n_kv_heads;
  p.head_dim = shape.head_dim;
  p.capacity = shape.capacity;
  p.n_split = decode_parts(shape.batch * shape.n_kv_heads, (shape.capacity + kDecSplit - 1) / kDecSplit, dev.sm_count);
  p.scale_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
  cudaError_t e = launch_decode_attention(p, shape.batch, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? KVPOP_OK : cuda_fail(e, "decode attention launch");
}

kvpop_status kvpop_decode_attention_noalloc(const void* q, const void* k_cache, const void* v_cache,
                                            const int32_t* count, kvpop_cache_shape shape, float scale, float* out,
                                            float* lse, void* stream) {
  KVPOP_TRACE();
  kvpop_status st;
  if (q == nullptr || k_cache == nullptr || v_cache == nullptr || count == nullptr || out == nullptr)
    return fail(KVPOP_ERR_INVALID_ARG, "a pointer argument is NULL");
  if (!aligned16(k_cache) || !aligned16(v_cache))
    return fail(KVPOP_ERR_INVALID_ARG, "k_cache and v_cache must be 16-byte aligned");
  if (!aligned16(q)) return fail(KVPOP_ERR_INVALID_ARG, "q must be 16-byte aligned");
  if (!isfinite(scale) || !(scale > 0.f)) return fail(KVPOP_ERR_INVALID_ARG, "scale must be finite and > 0");
  if (!check_cache_shape(shape))
    return fail(KVPOP_ERR_UNSUPPORTED,
                "cache shape not supported (head_dim 64/128, group size a power of two <= 16, 1..512 sequences)");
  const size_t need = kvpop_decode_workspace_bytes(shape);
  if (need > decode_scratch_bytes())
    return fail(KVPOP_ERR_UNSUPPORTED,
                "this shape needs %zu bytes of split partials, more than the %zu-byte fixed scratch; "
                "use kvpop_decode_attention with a workspace",
                need, decode_scratch_bytes());
  DeviceInfo dev;
  if ((st = device_info(&dev)) != KVPOP_OK) return st;
  float* scratch = nullptr;
  cudaError_t e = decode_scratch_address(&scratch);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress of the decode scratch");
  DecodeParams p;
  memset(&p, 0, sizeof(p));
  p.dbg = debug_word();
  p.q = static_cast<const uint16_t*>(q);
  p.k_cache = static_cast<const uint16_t*>(k_cache);
  p.v_cache = static_cast<const uint16_t*>(v_cache);
  p.count = count;
  p.partial = scratch;
  p.out = out;
  p.lse = lse;
  p.n_q_heads = shape.n_q_heads;
  p.n_kv_heads = shape.n_kv_heads;
  p.head_dim = shape.head_dim;
  p.capacity = shape.capacity;
  p.n_split = decode_parts(shape.batch * shape.n_kv_heads, (shape.capacity + kDecSplit - 1) / kDecSplit, dev.sm_count);
  p.scale_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
  e = launch_decode_attention(p, shape.batch, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? KVPOP_OK : cuda_fail(e, "decode attention launch");
}

kvpop_status kvpop_future_targets(const void* q, const void* k, const int32_t* cu_seqlens, kvpop_shape shape,
                                  float scale, int32_t window, int32_t sinks, const int32_t* budgets, float* lse,
                                  float* target, uint8_t* keep, void* workspace, size_t workspace_bytes,
                                  int32_t* dev_status, void* stream) {
  KVPOP_TRACE();
  kvpop_status st;
  // Validate everything before the first launch.
  if ((st = check_qk(q, k, scale)) != KVPOP_OK) return st;
  if (lse == nullptr || target == nullptr || keep == nullptr || budgets == nullptr)
    return fail(KVPOP_ERR_INVALID_ARG, "lse, target, keep or budgets is NULL");
  if (window < 0 || sinks < 0) return fail(KVPOP_ERR_INVALID_ARG, "window and sinks must be >= 0");
  if ((st = check_shape(cu_seqlens, shape, true)) != KVPOP_OK) return st;
  if ((st = check_budgets(budgets, shape.batch, sinks, window)) != KVPOP_OK) return st;
  if (shape.total_tokens == 0) return KVPOP_OK;
  if ((st = check_workspace(workspace, workspace_bytes, kvpop_target_workspace_bytes(shape), 16)) != KVPOP_OK)
    return st;
  DeviceInfo dev;
  if ((st = device_info(&dev)) != KVPOP_OK) return st;
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  // Pass 1 writes the normaliser rows next to lse; pass 2 streams them.
  if ((st = run_row_lse(q, k, cu_seqlens, shape, scale, lse, workspace, dev_status, s, dev)) != KVPOP_OK ||
      (st = run_target(q, k, cu_seqlens, shape, scale, window, workspace, target, nullptr, dev_status, s, dev)) !=
          KVPOP_OK)
    return st;
  return kvpop_keep_mask(target, cu_seqlens, shape, window, sinks, budgets, keep, stream);
}

size_t kvpop_fused_workspace_bytes(const int32_t* cu_seqlens, kvpop_shape shape) {
  if (cu_seqlens == nullptr || shape.batch < 1 || shape.batch > kMaxSeqs || shape.n_q_heads < 1) return 0;
  const int64_t tiles = flag_tiles(cu_seqlens, shape.batch);
  if (tiles < 0) return 0;
  return align256(static_cast<size_t>(shape.n_q_heads * tiles + 2) * sizeof(int32_t)) +
         align256(norm_rows_bytes(shape));
}

kvpop_status kvpop_future_targets_fused(const void* q, const void* k, const int32_t* cu_seqlens, kvpop_shape shape,
                                        float scale, int32_t window, int32_t sinks, const int32_t* budgets,
                                        float* lse, float* target, uint8_t* keep, void* workspace,
                                        size_t workspace_bytes, int32_t* dev_status, void* stream) {
  KVPOP_TRACE();
  kvpop_status st;
  if ((st = check_qk(q, k, scale)) != KVPOP_OK) return st;
  if (lse == nullptr || target == nullptr || keep == nullptr || budgets == nullptr)
    return fail(KVPOP_ERR_INVALID_ARG, "lse, target, keep or budgets is NULL");
  if (window < 0 || sinks < 0) return fail(KVPOP_ERR_INVALID_ARG, "window and sinks must be >= 0");
  if ((st = check_shape(cu_seqlens, shape, true)) != KVPOP_OK) return st;
  if ((st = check_budgets(budgets, shape.batch, sinks, window)) != KVPOP_OK) return st;
  if ((st = check_workspace(workspace, workspace_bytes, kvpop_fused_workspace_bytes(cu_seqlens, shape), 16)) !=
      KVPOP_OK)
    return st;
  if (static_cast<int64_t>(shape.n_q_heads) * flag_tiles(cu_seqlens, shape.batch) >= (int64_t(1) << 31))
    return fail(KVPOP_ERR_UNSUPPORTED, "too many (query head, tile) flags for one launch");
  if (shape.total_tokens == 0) return KVPOP_OK;
  DeviceInfo dev;
  if ((st = device_info(&dev)) != KVPOP_OK) return st;

  std::vector<FusedParams> holder(1);   // ~21 KB: keep it off the stack
  FusedParams& fp = holder[0];
  memset(&fp, 0, sizeof(fp));
  std::vector<int> order_lse, order_tgt;
  if ((st = fill_attn_common(&fp.attn, q, k, cu_seqlens, shape, scale, false, &order_lse)) != KVPOP_OK) return st;
  {
    std::vector<AttnParams> tgt(1);
    if ((st = fill_attn_common(&tgt[0], q, k, cu_seqlens, shape, scale, true, &order_tgt)) != KVPOP_OK) return st;
    fp.tmap_q_stream = tgt[0].tmap_q;
    fp.tmap_k_tile = tgt[0].tmap_k;
    fp.sched_target = tgt[0].sched;
  }
  fp.attn.window = std::min<int32_t>(window, kMaxLevels * kTileRows + 1);
  fp.attn.out = lse;
  fp.attn.status = dev_status;
  fp.target = target;
  std::vector<int32_t> base(shape.batch + 1, 0);
  for (int b = 0; b < shape.batch; ++b)
    base[b + 1] = base[b] + (cu_seqlens[b + 1] - cu_seqlens[b] + kTileRows - 1) / kTileRows;
  fp.n_flag_tiles = base[shape.batch];
  fp.n_flags = shape.n_q_heads * fp.n_flag_tiles;
  fp.flags = static_cast<int32_t*>(workspace);
  fp.done = fp.flags + fp.n_flags;
  fp.lse_done = fp.done + 1;
  // Pass 1 writes the normaliser rows after the counters; pass 2 reads them.
  fp.attn.nrm_rows = static_cast<uint8_t*>(workspace) + align256(static_cast<size_t>(fp.n_flags + 2) * sizeof(int32_t));
  for (size_t r = 0; r < order_lse.size(); ++r) fp.tile_base_lse[r] = base[order_lse[r]];
  for (size_t r = 0; r < order_tgt.size(); ++r) fp.tile_base_target[r] = base[order_tgt[r]];
  if (fp.attn.sched.total_items > 0) {
    const int items = std::max(fp.attn.sched.total_items, fp.sched_target.total_items);
    cudaError_t e = launch_fused_targets(fp, shape.head_dim, grid_for(items, dev.sm_count),
                                         static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "fused attention launch");
  }
  return kvpop_keep_mask(target, cu_seqlens, shape, window, sinks, budgets, keep, stream);
}

// Largest KV-head group of the host-buffer pipeline.
static int host_group_max(int n_kv_heads) {
  const int n_groups = std::min(n_kv_heads, kHostGroups);
  return (n_kv_heads + n_groups - 1) / n_groups;
}

size_t kvpop_host_workspace_bytes(kvpop_shape shape) {
  if (shape.total_tokens <= 0 || shape.n_q_heads <= 0 || shape.n_kv_heads <= 0 || shape.head_dim <= 0 ||
      shape.n_q_heads % shape.n_kv_heads != 0)
    return 0;
  const size_t T = static_cast<size_t>(shape.total_tokens);
  const size_t G = static_cast<size_t>(shape.n_q_heads / shape.n_kv_heads);
  const size_t group_q_heads = G * host_group_max(shape.n_kv_heads);
  const size_t partials = group_q_heads * target_split_groups() * T * 4;
  const size_t rows = group_q_heads * T * 16;
  return align256(T * shape.n_q_heads * shape.head_dim * 2) + align256(T * shape.n_kv_heads * shape.head_dim * 2) +
         align256(T * shape.n_q_heads * 4) + align256(T * shape.n_kv_heads * 4) + align256(T * shape.n_kv_heads) +
         align256(rows) + align256(partials);
}

kvpop_status kvpop_future_targets_host(const void* q_host, const void* k_host, const int32_t* cu_seqlens,
                                       kvpop_shape shape, float scale, int32_t window, int32_t sinks,
                                       const int32_t* budgets, float* target_host, uint8_t* keep_host,
                                       void* workspace, size_t workspace_bytes, int32_t* dev_status, void* stream) {
  KVPOP_TRACE();
  kvpop_status st;
  if (q_host == nullptr || k_host == nullptr || target_host == nullptr || keep_host == nullptr)
    return fail(KVPOP_ERR_INVALID_ARG, "a host buffer is NULL");
  if (!isfinite(scale) || !(scale > 0.f)) return fail(KVPOP_ERR_INVALID_ARG, "scale must be finite and > 0");
  if (budgets == nullptr) return fail(KVPOP_ERR_INVALID_ARG, "budgets is NULL");
  if (window < 0 || sinks < 0) return fail(KVPOP_ERR_INVALID_ARG, "window and sinks must be >= 0");
  if ((st = check_shape(cu_seqlens, shape, true)) != KVPOP_OK) return st;
  if ((st = check_budgets(budgets, shape.batch, sinks, window)) != KVPOP_OK) return st;
  if (shape.total_tokens == 0) return KVPOP_OK;
  const size_t need = kvpop_host_workspace_bytes(shape);
  if (workspace == nullptr || workspace_bytes < need)
    return fail(KVPOP_ERR_INVALID_ARG, "workspace of %zu bytes is smaller than the %zu required", workspace_bytes,
                need);
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return fail(KVPOP_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  const size_t T = static_cast<size_t>(shape.total_tokens);
  const int G = shape.n_q_heads / shape.n_kv_heads, d = shape.head_dim;
  const size_t qb = T * shape.n_q_heads * d * 2, kb = T * shape.n_kv_heads * d * 2;
  const size_t lb = T * shape.n_q_heads * 4, tb = T * shape.n_kv_heads * 4;
  uint8_t* w = static_cast<uint8_t*>(workspace);
  uint8_t* q_all = w;
  uint8_t* k_all = w + align256(qb);
  float* lse = reinterpret_cast<float*>(w + align256(qb) + align256(kb));
  float* target = reinterpret_cast<float*>(w + align256(qb) + align256(kb) + align256(lb));
  uint8_t* keep = w + align256(qb) + align256(kb) + align256(lb) + align256(tb);
  uint8_t* rows = w + align256(qb) + align256(kb) + align256(lb) + align256(tb) + align256(T * shape.n_kv_heads);
  float* partials = reinterpret_cast<float*>(rows + align256(static_cast<size_t>(G) * host_group_max(shape.n_kv_heads) *
                                                             T * 16));
  DeviceInfo dev;
  if ((st = device_info(&dev)) != KVPOP_OK) return st;
  HostStreams hs;
  if ((st = host_streams(&hs)) != KVPOP_OK) return st;
  const cudaStream_t s = static_cast<cudaStream_t>(stream);

  // KV-head groups: group c's Q and K land as a compact problem of their own
  // (strided 2-D copies), so its two passes and keep mask can run while the
  // next group is still being copied in.  Groups of (nearly) equal size; the
  // split transposed pass keeps even one-head groups balanced, and smaller
  // groups leave less compute after the last copy.
  const int n_groups = std::min(shape.n_kv_heads, kHostGroups);
  int sizes[kHostGroups] = {};
  for (int c = 0; c < n_groups; ++c) sizes[c] = shape.n_kv_heads / n_groups + (c < shape.n_kv_heads % n_groups ? 1 : 0);
  EventSet ev;
  cudaError_t e;
  cudaEvent_t start;
  if ((e = ev.make(&start)) != cudaSuccess) return cuda_fail(e, "cudaEventCreate");
  // The copies must not overwrite the workspace while earlier work on `stream` may still read it.
  if ((e = cudaEventRecord(start, s)) != cudaSuccess) return cuda_fail(e, "cudaEventRecord");
  if ((e = cudaStreamWaitEvent(hs.in, start, 0)) != cudaSuccess) return cuda_fail(e, "cudaStreamWaitEvent");
  size_t q_off = 0, k_off = 0;
  int h0 = 0;
  for (int c = 0; c < n_groups; ++c) {
    const int hn = sizes[c];
    const size_t q_row = static_cast<size_t>(hn) * G * d * 2, k_row = static_cast<size_t>(hn) * d * 2;
    uint8_t* qc = q_all + q_off;
    uint8_t* kc = k_all + k_off;
    const uint8_t* qh = static_cast<const uint8_t*>(q_host) + static_cast<size_t>(h0) * G * d * 2;
    const uint8_t* kh = static_cast<const uint8_t*>(k_host) + static_cast<size_t>(h0) * d * 2;
    cudaEvent_t copied, computed;
    if ((e = ev.make(&copied)) != cudaSuccess || (e = ev.make(&computed)) != cudaSuccess)
      return cuda_fail(e, "cudaEventCreate");
    if ((e = cudaMemcpy2DAsync(qc, q_row, qh, static_cast<size_t>(shape.n_q_heads) * d * 2, q_row, T,
                               cudaMemcpyHostToDevice, hs.in)) != cudaSuccess)
      return cuda_fail(e, "copy q");
    if ((e = cudaMemcpy2DAsync(kc, k_row, kh, static_cast<size_t>(shape.n_kv_heads) * d * 2, k_row, T,
                               cudaMemcpyHostToDevice, hs.in)) != cudaSuccess)
      return cuda_fail(e, "copy k");
    if ((e = cudaEventRecord(copied, hs.in)) != cudaSuccess) return cuda_fail(e, "cudaEventRecord");
    if ((e = cudaStreamWaitEvent(s, copied, 0)) != cudaSuccess) return cuda_fail(e, "cudaStreamWaitEvent");
    // A group holds few KV heads, so its transposed pass takes one item per
    // (key tile, query head): same result, G times as many items.
    kvpop_shape sc = shape;
    sc.n_q_heads = hn * G;
    sc.n_kv_heads = hn;
    float* lse_c = lse + static_cast<size_t>(h0) * G * T;
    float* target_c = target + static_cast<size_t>(h0) * T;
    // Groups run one after another on `stream`, so they share the rows and partials.
    if ((st = run_row_lse(qc, kc, cu_seqlens, sc, scale, lse_c, rows, dev_status, s, dev)) != KVPOP_OK ||
        (st = run_target(qc, kc, cu_seqlens, sc, scale, window, rows, target_c, G > 1 ? partials : nullptr,
                         dev_status, s, dev)) != KVPOP_OK ||
        (st = kvpop_keep_mask(target_c, cu_seqlens, sc, window, sinks, budgets, keep + static_cast<size_t>(h0) * T,
                              stream)) != KVPOP_OK)
      return st;
    if ((e = cudaEventRecord(computed, s)) != cudaSuccess) return cuda_fail(e, "cudaEventRecord");
    if ((e = cudaStreamWaitEvent(hs.out, computed, 0)) != cudaSuccess) return cuda_fail(e, "cudaStreamWaitEvent");
    if ((e = cudaMemcpyAsync(target_host + static_cast<size_t>(h0) * T, target + static_cast<size_t>(h0) * T,
                             static_cast<size_t>(hn) * T * 4, cudaMemcpyDeviceToHost, hs.out)) != cudaSuccess)
      return cuda_fail(e, "copy target");
    if ((e = cudaMemcpyAsync(keep_host + static_cast<size_t>(h0) * T, keep + static_cast<size_t>(h0) * T,
                             static_cast<size_t>(hn) * T, cudaMemcpyDeviceToHost, hs.out)) != cudaSuccess)
      return cuda_fail(e, "copy keep");
    q_off += q_row * T;
    k_off += k_row * T;
    h0 += hn;
  }
  // `stream` completes only after the last copy back.
  cudaEvent_t done;
  if ((e = ev.make(&done)) != cudaSuccess) return cuda_fail(e, "cudaEventCreate");
  if ((e = cudaEventRecord(done, hs.out)) != cudaSuccess) return cuda_fail(e, "cudaEventRecord");
  if ((e = cudaStreamWaitEvent(s, done, 0)) != cudaSuccess) return cuda_fail(e, "cudaStreamWaitEvent");
  return KVPOP_OK;
}

kvpop_status kvpop_check_device_status(const int32_t* dev_status, void* stream) {
  if (dev_status == nullptr) return fail(KVPOP_ERR_INVALID_ARG, "dev_status is NULL");
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  int32_t v = 0;
  e = cudaMemcpy(&v, dev_status, sizeof(v), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "read dev_status");
  if (v == 0) return KVPOP_OK;
  if ((v & 0xff) == KVPOP_ERR_TIMEOUT)
    return fail(KVPOP_ERR_TIMEOUT, "a kernel wait timed out (site %d)", (v >> 8) & 0xff);
  if ((v & 0xff) == KVPOP_ERR_BOUNDS)
    return fail(KVPOP_ERR_BOUNDS, "bounds check failed in kernel %d at site %d", (v >> 16) & 0xff, (v >> 8) & 0xff);
  return fail(KVPOP_ERR_CUDA, "device status word holds %d", v);
}

kvpop_status kvpop_selftest_bounded_wait(int32_t* dev_status, uint64_t limit_ns, void* stream) {
  if (dev_status == nullptr) return fail(KVPOP_ERR_INVALID_ARG, "dev_status is NULL");
  if (limit_ns < 1 || limit_ns > 1000000000ull) return fail(KVPOP_ERR_INVALID_ARG, "limit_ns out of range");
  DeviceInfo dev;
  kvpop_status st;
  if ((st = device_info(&dev)) != KVPOP_OK) return st;
  cudaError_t e = launch_selftest_wait(dev_status, limit_ns, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? KVPOP_OK : cuda_fail(e, "selftest launch");
}

kvpop_status kvpop_debug_set_word(int32_t* dev_word) {
#ifdef KVPOP_DEBUG
  g_debug_word.store(dev_word, std::memory_order_relaxed);
  return KVPOP_OK;
#else
  (void)dev_word;
  return fail(KVPOP_ERR_UNSUPPORTED, "this library was built without bounds checks (KVPOP_DEBUG)");
#endif
}

kvpop_status kvpop_debug_selftest(int32_t* dev_word, void* stream) {
#ifdef KVPOP_DEBUG
  if (dev_word == nullptr) return fail(KVPOP_ERR_INVALID_ARG, "dev_word is NULL");
  DeviceInfo dev;
  kvpop_status st;
  if ((st = device_info(&dev)) != KVPOP_OK) return st;
  cudaError_t e = launch_debug_selftest(dev_word, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? KVPOP_OK : cuda_fail(e, "debug self-test launch");
#else
  (void)dev_word;
  (void)stream;
  return fail(KVPOP_ERR_UNSUPPORTED, "this library was built without bounds checks (KVPOP_DEBUG)");
#endif
}

}  // extern "C"
