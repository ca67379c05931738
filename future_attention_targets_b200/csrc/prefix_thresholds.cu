// Prefix top-k eviction thresholds, sm_100a.
//
// For every decoding step t of a sequence, the tokens p in [S, t - W] have
// left the recent window and compete for the k = budget - S - W scored
// slots; the threshold of step t is the k-th best of them (higher score
// first, then smaller position).  Scores are compared through 64-bit keys
// (order-preserving score bits, then the inverted position), so the order is
// total and every comparison exact.
//
// The steps are cut into blocks of kBlock candidates, one CTA per
// (sequence, KV head, block), all independent.  With K = the top-min(p, k)
// of the p candidates before the block:
//   1. K's minimum by radix select over the prefix (four 8-bit digits of the
//      score key, the keys cached in shared memory; ties resolved by
//      position with one block scan of per-thread counts).
//   2. Only the block's candidates D that beat K's minimum (all of them
//      while K is not full) can matter; they are compacted and sorted.
//   3. The threshold after candidate j is the (|K| + d_j - k + 1)-th
//      smallest of K together with the first d_j entries of D (d_j = how
//      many of candidates 0..j beat K's minimum).  That rank never exceeds
//      m = |K| + |D| - k + 1, so only K's m smallest members are needed: a
//      second radix select bounds them (skipped when m = 1), they are
//      gathered and sorted, and merged with D into one sorted list tagged
//      with each entry's step.
//   4. Every thread counts its way along that list (8 tags per 16-byte load)
//      to its rank, skipping D entries that arrive after its step.
#include <cuda_runtime.h>
#include <stdint.h>

#include "kvpop_cache.h"
#include "kvpop_debug.cuh"

namespace kvpop {

constexpr int kThrThreads = 1024;
constexpr int kThrWarps = kThrThreads / 32;
constexpr int kBlock = 1024;                 // candidates (steps) per CTA
constexpr int kBandMax = kBlock + 1;         // the band of K never needs more keys than this
constexpr int kSortMax = 2 * kBlock;         // power-of-two room for sorting the band
constexpr int kMergedMax = kBandMax + kBlock + 7;   // band + D, tags padded to a multiple of 8
constexpr int kHistCopies = 8;               // per-warp-group histogram copies (fewer atomic collisions)
constexpr int kKeyCache = 16384;             // prefix score keys kept in shared memory (longer prefixes re-read L2)
constexpr int16_t kNeverTag = 0x7fff;        // padding tag: never present

// Larger float -> larger key; -0 == +0; NaN -> 0 (below -inf).
__device__ __forceinline__ uint32_t score_key(float f) {
  uint32_t u = __float_as_uint(f);
  if ((u & 0x7fffffffu) > 0x7f800000u) return 0u;
  if (u == 0x80000000u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float key_score(uint32_t k) {
  if (k == 0u) return __uint_as_float(0x7fc00000u);            // NaN
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

// Total order: score key, then smaller position first.  Never 0 for p < 2^31.
__device__ __forceinline__ uint64_t compose_key(uint32_t sk, int32_t p) {
  return (static_cast<uint64_t>(sk) << 32) | (0xffffffffu - static_cast<uint32_t>(p));
}
__device__ __forceinline__ int32_t key_pos(uint64_t k) {
  return static_cast<int32_t>(0xffffffffu - static_cast<uint32_t>(k));
}

// Number of entries of the ascending array a[0..n) that are < x.
__device__ __forceinline__ int lower_bound_u64(const uint64_t* a, int n, uint64_t x) {
  int lo = 0, hi = n;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (a[mid] < x) lo = mid + 1; else hi = mid;
  }
  return lo;
}

// Ascending bitonic sort of a[0 .. n) (n a power of two, <= 2 * kThrThreads):
// each thread does one compare-exchange per stage.
__device__ __forceinline__ void bitonic_sort(uint64_t* a, int n) {
  for (int kk = 2; kk <= n; kk <<= 1) {
    for (int jj = kk >> 1; jj > 0; jj >>= 1) {
      for (int t = threadIdx.x; t < n / 2; t += kThrThreads) {
        const int i = ((t & ~(jj - 1)) << 1) | (t & (jj - 1));   // index with bit jj clear
        const int ixj = i | jj;
        const uint64_t x = a[i], y = a[ixj];
        if ((x > y) == ((i & kk) == 0)) {
          a[i] = y;
          a[ixj] = x;
        }
      }
      __syncthreads();
    }
  }
}

// Inclusive count, over the block, of the threads whose `flag` is set, in
// thread order; *total gets the block's count.
__device__ __forceinline__ int block_rank(bool flag, int* warp_tot, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const uint32_t m = __ballot_sync(0xffffffffu, flag);
  if (lane == 0) warp_tot[warp] = __popc(m);
  __syncthreads();
  int before = 0, all = 0;
  for (int w = 0; w < kThrWarps; ++w) {
    const int c = warp_tot[w];
    before += (w < warp) ? c : 0;
    all += c;
  }
  *total = all;
  const int r = before + __popc(m & ((2u << lane) - 1u));
  __syncthreads();                          // warp_tot is reused by the next call
  return r;
}

// Exclusive prefix sum over the block of a per-thread count.
__device__ __forceinline__ int block_excl_scan(int a, int* warp_tot) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int ia = a;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, ia, o);
    if (lane >= o) ia += y;
  }
  if (lane == 31) warp_tot[warp] = ia;
  __syncthreads();
  int before = 0;
  for (int w = 0; w < warp; ++w) before += warp_tot[w];
  __syncthreads();
  return before + ia - a;
}

struct ThrShared {
  uint32_t* hist;        // [kHistCopies][256]
  uint32_t* bins;        // [256]
  uint32_t* sel;         // [2]
  int* warp_tot;         // [kThrWarps]
  int32_t* tie_pos;      // [1]
};

// The composite key of rank `need` (1-based, from the largest) among the
// prefix candidates 0..n-1, whose score keys key_at(i) returns: radix select
// on the score key, then the need'-th smallest position among its ties.
template <class KeyAt>
__device__ uint64_t select_rank(KeyAt key_at, int n, uint32_t need, int32_t pos0, const ThrShared& sh) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  uint32_t prefix = 0u, pmask = 0u;
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int i = tid; i < kHistCopies * 256; i += kThrThreads) sh.hist[i] = 0u;
    __syncthreads();
    uint32_t* hw = sh.hist + (warp % kHistCopies) * 256;
    for (int32_t i = tid; i < n; i += kThrThreads) {
      const uint32_t u = key_at(i);
      if ((u & pmask) == prefix) atomicAdd(hw + ((u >> shift) & 255u), 1u);
    }
    __syncthreads();
    if (tid < 256) {
      uint32_t c = 0;
#pragma unroll
      for (int q = 0; q < kHistCopies; ++q) c += sh.hist[q * 256 + tid];
      sh.bins[tid] = c;
    }
    __syncthreads();
    if (warp == 0) {
      // Lane l covers digits 255-8l .. 248-8l (descending); find the digit
      // holding the need-th largest key.
      uint32_t cnt[8], tot = 0;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        cnt[q] = sh.bins[255 - 8 * lane - q];
        tot += cnt[q];
      }
      uint32_t incl = tot;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
      }
      const uint32_t excl = incl - tot;
      const uint32_t hit = __ballot_sync(0xffffffffu, incl >= need && excl < need);
      if (lane == __ffs(hit) - 1) {
        uint32_t before = excl;
        int q = 0;
        while (before + cnt[q] < need) before += cnt[q++];
        sh.sel[0] = 255u - 8u * lane - q;
        sh.sel[1] = need - before;
      }
    }
    __syncthreads();
    prefix |= sh.sel[0] << shift;
    pmask |= 255u << shift;
    need = sh.sel[1];
    __syncthreads();
  }
  // Among the keys equal to prefix, the need-th largest composite has the
  // need-th smallest position: per-thread counts over contiguous runs, one
  // block scan, and the thread whose run holds it finds it.
  const int run = (n + kThrThreads - 1) / kThrThreads;
  const int r0 = min(n, tid * run), r1 = min(n, r0 + run);
  int cnt = 0;
  for (int32_t i = r0; i < r1; ++i) cnt += (key_at(i) == prefix);
  if (tid == 0) *sh.tie_pos = 0;
  const int e = block_excl_scan(cnt, sh.warp_tot);
  const int want = static_cast<int>(need);
  if (e < want && want <= e + cnt) {
    int seen = e;
    for (int32_t i = r0; i < r1; ++i)
      if (key_at(i) == prefix && ++seen == want) {
        *sh.tie_pos = pos0 + i;
        break;
      }
  }
  __syncthreads();
  const uint64_t r = compose_key(prefix, *sh.tie_pos);
  __syncthreads();
  return r;
}

__global__ void __launch_bounds__(kThrThreads, 1) prefix_thresholds_kernel(const __grid_constant__ ThresholdParams p) {
  extern __shared__ uint64_t thr_smem[];
  uint64_t* band = thr_smem;                                     // kSortMax
  uint64_t* dsort = band + kSortMax;                             // kBlock
  uint64_t* merged = dsort + kBlock;                             // kMergedMax
  int16_t* tags = reinterpret_cast<int16_t*>(merged + kMergedMax);   // kMergedMax (16-byte aligned)
  uint32_t* hist = reinterpret_cast<uint32_t*>(tags + kMergedMax);    // [kHistCopies][256]
  uint32_t* keys = hist + kHistCopies * 256;                     // kKeyCache
  __shared__ uint32_t bins[256];
  __shared__ uint32_t sel[2];
  __shared__ int warp_tot[kThrWarps];
  __shared__ int32_t tie_pos;
  __shared__ int band_n;
  const ThrShared sh{hist, bins, sel, warp_tot, &tie_pos};

  const int b = blockIdx.x, h = blockIdx.y, c = blockIdx.z;
  const int tid = threadIdx.x;
  const int32_t s0 = p.seq_start[b], L = p.seq_len[b];
  const int32_t S = p.sinks, W = p.window;
  const int32_t k = p.budget[b] - S - W;
  const float* score = p.score + static_cast<int64_t>(h) * p.total_tokens + s0;
  float* out_s = p.thr_score + static_cast<int64_t>(h) * p.total_tokens + s0;
  int32_t* out_p = p.thr_pos + static_cast<int64_t>(h) * p.total_tokens + s0;
  // Debug build: a step or position t of this row lies inside the row and the [H_kv, T] arrays.
  auto in_row = [&](int32_t t, int32_t site) {
    return KVPOP_IN(t >= 0 && t < L && s0 >= 0 && s0 + t < p.total_tokens, p.dbg, DBG_THRESHOLDS, site);
  };

  // Steps before the first candidate leaves the window: no eviction.
  if (c == 0) {
    const int32_t first = min(L, S + W);
    for (int32_t t = tid; t < first; t += kThrThreads) {
      if (!in_row(t, 1)) continue;
      out_s[t] = -INFINITY;
      out_p[t] = -1;
    }
  }
  const int32_t n = L - S - W;                  // candidates S .. L-W-1, candidate i enters at step S+W+i
  const int32_t base = c * kBlock;
  if (n <= 0 || base >= n) return;
  const int nb = min(kBlock, n - base);
  if (k == 0) {                                 // no scored slots: every candidate is evicted at once
    for (int32_t i = tid; i < nb; i += kThrThreads) {
      if (!in_row(S + W + base + i, 1)) continue;
      out_s[S + W + base + i] = INFINITY;
      out_p[S + W + base + i] = -1;
    }
    return;
  }

  const int ksz = min(base, k);                 // |K|
  const bool cached = base <= kKeyCache;
  if (cached)
    for (int32_t i = tid; i < base; i += kThrThreads)
      if (in_row(S + i, 2) && KVPOP_IN(i < kKeyCache, p.dbg, DBG_THRESHOLDS, 3)) keys[i] = score_key(__ldg(score + S + i));
  __syncthreads();
  auto key_at = [&](int32_t i) -> uint32_t {
    if (cached) return KVPOP_IN(i >= 0 && i < kKeyCache, p.dbg, DBG_THRESHOLDS, 3) ? keys[i] : 0u;
    return in_row(S + i, 2) ? score_key(__ldg(score + S + i)) : 0u;
  };

  // ---- 1. K's minimum: the ksz-th largest key of the prefix.
  const uint64_t kmin = (ksz > 0) ? select_rank(key_at, base, static_cast<uint32_t>(ksz), S, sh) : 0ull;

  // ---- 2. the block's candidates that beat K's minimum (all while K is not full)
  const uint64_t tau = (ksz >= k) ? kmin : 0ull;      // every key is > 0
  uint64_t v = 0;
  bool beats = false;
  if (tid < nb && in_row(S + base + tid, 2)) {
    v = compose_key(score_key(__ldg(score + S + base + tid)), S + base + tid);
    beats = v > tau;
  }
  int d_total = 0;
  const int d_j = block_rank(beats, warp_tot, &d_total);   // inclusive
  int np2 = 1;
  while (np2 < d_total) np2 <<= 1;
  if (beats && KVPOP_IN(d_j >= 1 && d_j <= kBlock, p.dbg, DBG_THRESHOLDS, 4)) dsort[d_j - 1] = v;
  for (int i = d_total + tid; i < np2; i += kThrThreads)
    if (KVPOP_IN(i < kBlock, p.dbg, DBG_THRESHOLDS, 4)) dsort[i] = ~0ull;
  __syncthreads();
  bitonic_sort(dsort, np2);

  // ---- 3. K's m smallest members (m = the deepest rank any step can reach)
  const int m = max(0, min(ksz, ksz + d_total - k + 1));
  if (m == 1) {
    if (tid == 0) band[0] = kmin;
  } else if (m > 1) {
    const uint64_t kmax_band = select_rank(key_at, base, static_cast<uint32_t>(ksz - m + 1), S, sh);
    if (tid == 0) band_n = 0;
    __syncthreads();
    const uint32_t s_lo = static_cast<uint32_t>(kmin >> 32), s_hi = static_cast<uint32_t>(kmax_band >> 32);
    for (int32_t i = tid; i < base; i += kThrThreads) {
      const uint32_t u = key_at(i);
      if (u < s_lo || u > s_hi) continue;      // outside the band's score range
      const uint64_t x = compose_key(u, S + i);
      if (x >= kmin && x <= kmax_band) {
        const int slot = atomicAdd(&band_n, 1);
        if (slot < kBandMax) band[slot] = x;
      }
    }
    __syncthreads();
    int bp2 = 1;
    while (bp2 < m) bp2 <<= 1;
    for (int i = m + tid; i < bp2; i += kThrThreads)
      if (KVPOP_IN(i < kSortMax, p.dbg, DBG_THRESHOLDS, 5)) band[i] = ~0ull;
    __syncthreads();
    bitonic_sort(band, bp2);
  }
  __syncthreads();

  // Merge the band (tag -1: always present) and D (tag = its step in the
  // block) into one ascending list; the keys are distinct.
  const int n_merged = m + d_total;
  const int n_padded = (n_merged + 7) & ~7;
  for (int a = tid; a < m; a += kThrThreads) {
    const int at = a + lower_bound_u64(dsort, d_total, band[a]);
    if (!KVPOP_IN(at >= 0 && at < kMergedMax, p.dbg, DBG_THRESHOLDS, 6)) continue;
    merged[at] = band[a];
    tags[at] = -1;
  }
  for (int r = tid; r < d_total; r += kThrThreads) {
    const int at = r + lower_bound_u64(band, m, dsort[r]);
    if (!KVPOP_IN(at >= 0 && at < kMergedMax, p.dbg, DBG_THRESHOLDS, 6)) continue;
    merged[at] = dsort[r];
    tags[at] = static_cast<int16_t>(key_pos(dsort[r]) - (S + base));
  }
  for (int i = n_merged + tid; i < n_padded; i += kThrThreads)
    if (KVPOP_IN(i < kMergedMax, p.dbg, DBG_THRESHOLDS, 6)) tags[i] = kNeverTag;
  __syncthreads();

  // ---- 4. threshold of this thread's step: its rank among the entries
  // present at the step (band entries, and D entries of steps <= tid).
  if (tid < nb) {
    const int t = S + W + base + tid;
    const int total = ksz + d_j;
    if (!in_row(t, 1)) {
    } else if (total < k) {
      out_s[t] = -INFINITY;
      out_p[t] = -1;
    } else {
      const int want = total - k + 1;
      const uint32_t me2 = (static_cast<uint32_t>(tid) & 0xffffu) * 0x10001u;   // this step in both halves
      int cnt = 0, i = 0;
      for (; i < n_padded && KVPOP_IN(i + 8 <= kMergedMax, p.dbg, DBG_THRESHOLDS, 7); i += 8) {
        const uint4 w = *reinterpret_cast<const uint4*>(tags + i);
        const int here = (__popc(__vcmples2(w.x, me2)) + __popc(__vcmples2(w.y, me2)) +
                          __popc(__vcmples2(w.z, me2)) + __popc(__vcmples2(w.w, me2))) >> 4;
        if (cnt + here >= want) break;
        cnt += here;
      }
      uint64_t x = 0;
      for (int q = 0; q < 8 && KVPOP_IN(i + q < kMergedMax, p.dbg, DBG_THRESHOLDS, 7); ++q) {
        if (tags[i + q] <= tid && ++cnt == want) {
          x = merged[i + q];
          break;
        }
      }
      out_s[t] = key_score(static_cast<uint32_t>(x >> 32));
      out_p[t] = key_pos(x);
    }
  }
}

static size_t threshold_smem_bytes() {
  return (kSortMax + kBlock + kMergedMax) * sizeof(uint64_t) + kMergedMax * sizeof(int16_t) +
         (kHistCopies * 256 + kKeyCache) * sizeof(uint32_t);
}

cudaError_t launch_prefix_thresholds(const ThresholdParams& p, int n_kv_heads, int max_len, cudaStream_t stream) {
  const size_t smem = threshold_smem_bytes();
  cudaError_t e = cudaFuncSetAttribute(prefix_thresholds_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const int n_max = max_len - p.sinks - p.window;
  const int blocks = n_max > 0 ? (n_max + kBlock - 1) / kBlock : 1;
  dim3 grid(p.n_seqs, n_kv_heads, blocks);
  prefix_thresholds_kernel<<<grid, kThrThreads, smem, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace kvpop
