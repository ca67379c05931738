// Prefix top-k eviction thresholds, sm_100a.
//
// For every decoding step t of a sequence, the tokens p in [S, t - W] have
// left the recent window and compete for the k = budget - S - W scored
// slots; the threshold of step t is the k-th best of them (higher score
// first, then smaller position).  One CTA per (sequence, KV head) walks the
// steps in blocks of kBlock candidates, keeping the current top-k set K
// sorted in shared memory:
//   1. a candidate matters only if it beats K's minimum (all of them while
//      K is not yet full);
//   2. those candidates D are compacted and bitonic-sorted;
//   3. the threshold after candidate j of the block is the
//      (|K| + d_j - k + 1)-th smallest of K together with the first d_j
//      entries of D (d_j = how many of candidates 0..j beat K's minimum):
//      every thread walks that merged order for its own step;
//   4. K becomes the k largest of K and D (a parallel merge by binary search).
// Scores are compared through 64-bit keys (order-preserving score bits, then
// the inverted position), so the order is total and every comparison exact.
#include <cuda_runtime.h>
#include <stdint.h>

#include "kvpop_cache.h"

namespace kvpop {

constexpr int kThrThreads = 1024;
constexpr int kBlock = 1024;                 // candidates (steps) per block

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
__device__ __forceinline__ uint64_t cand_key(float score, int32_t p) {
  return (static_cast<uint64_t>(score_key(score)) << 32) | (0xffffffffu - static_cast<uint32_t>(p));
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

__global__ void __launch_bounds__(kThrThreads, 1) prefix_thresholds_kernel(const __grid_constant__ ThresholdParams p) {
  extern __shared__ uint64_t thr_smem[];
  uint64_t* kset[2] = {thr_smem, thr_smem + kMaxScored};   // sorted ascending, double-buffered
  uint64_t* dsort = thr_smem + 2 * kMaxScored;             // kBlock slots
  __shared__ int warp_tot[kThrThreads / 32];

  const int b = blockIdx.x, h = blockIdx.y;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int32_t s0 = p.seq_start[b], L = p.seq_len[b];
  const int32_t S = p.sinks, W = p.window;
  const int32_t k = p.budget[b] - S - W;
  const float* score = p.score + static_cast<int64_t>(h) * p.total_tokens + s0;
  float* out_s = p.thr_score + static_cast<int64_t>(h) * p.total_tokens + s0;
  int32_t* out_p = p.thr_pos + static_cast<int64_t>(h) * p.total_tokens + s0;

  // Steps before the first candidate leaves the window: no eviction.
  const int32_t first = min(L, S + W);
  for (int32_t t = tid; t < first; t += kThrThreads) {
    out_s[t] = -INFINITY;
    out_p[t] = -1;
  }
  const int32_t n = L - S - W;                  // candidates S .. L-W-1, candidate i enters at step S+W+i
  if (n <= 0) return;
  if (k == 0) {                                 // no scored slots: every candidate is evicted at once
    for (int32_t i = tid; i < n; i += kThrThreads) {
      out_s[S + W + i] = INFINITY;
      out_p[S + W + i] = -1;
    }
    return;
  }

  int cur = 0, size = 0;                        // K = kset[cur][0 .. size)
  for (int32_t base = 0; base < n; base += kBlock) {
    const int nb = min(kBlock, n - base);
    const uint64_t tau = (size >= k) ? kset[cur][0] : 0ull;   // every key is > 0
    uint64_t v = 0;
    bool beats = false;
    if (tid < nb) {
      v = cand_key(__ldg(score + S + base + tid), S + base + tid);
      beats = v > tau;
    }
    // d_j = number of beating candidates among 0..j (block-wide inclusive scan)
    const uint32_t m = __ballot_sync(0xffffffffu, beats);
    if (lane == 0) warp_tot[warp] = __popc(m);
    __syncthreads();
    int before = 0, d_total = 0;
    for (int w = 0; w < kThrThreads / 32; ++w) {
      const int c = warp_tot[w];
      before += (w < warp) ? c : 0;
      d_total += c;
    }
    const int d_j = before + __popc(m & ((2u << lane) - 1u));   // inclusive
    // Compact D, pad to a power of two, bitonic sort ascending.
    int np2 = 1;
    while (np2 < d_total) np2 <<= 1;
    if (beats) dsort[d_j - 1] = v;
    for (int i = d_total + tid; i < np2; i += kThrThreads) dsort[i] = ~0ull;
    __syncthreads();
    for (int kk = 2; kk <= np2; kk <<= 1) {
      for (int jj = kk >> 1; jj > 0; jj >>= 1) {
        for (int i = tid; i < np2; i += kThrThreads) {
          const int ixj = i ^ jj;
          if (ixj > i) {
            const uint64_t a = dsort[i], c = dsort[ixj];
            const bool up = (i & kk) == 0;
            if ((a > c) == up) {
              dsort[i] = c;
              dsort[ixj] = a;
            }
          }
        }
        __syncthreads();
      }
    }
    // Threshold of this thread's step: the (size + d_j - k + 1)-th smallest
    // of K and the D entries with block index <= tid.
    if (tid < nb) {
      const int t = S + W + base + tid;
      const int total = size + d_j;
      if (total < k) {
        out_s[t] = -INFINITY;
        out_p[t] = -1;
      } else {
        const int want = total - k + 1;
        const uint64_t* K = kset[cur];
        const int32_t my_pos = S + base + tid;
        int ia = 0, ib = 0, cnt = 0;
        uint64_t x = 0;
        while (cnt < want) {
          while (ib < d_total && key_pos(dsort[ib]) > my_pos) ++ib;   // entered after this step
          const bool take_k = (ia < size) && (ib >= d_total || K[ia] < dsort[ib]);
          x = take_k ? K[ia++] : dsort[ib++];
          ++cnt;
        }
        out_s[t] = key_score(static_cast<uint32_t>(x >> 32));
        out_p[t] = key_pos(x);
      }
    }
    // K <- the k largest of K and D (merge by ranks; keys are distinct).
    const int merged = size + d_total;
    const int new_size = min(k, merged);
    const int drop = merged - new_size;
    const uint64_t* K = kset[cur];
    uint64_t* KN = kset[cur ^ 1];
    for (int i = tid; i < size; i += kThrThreads) {
      const int r = i + lower_bound_u64(dsort, d_total, K[i]) - drop;
      if (r >= 0) KN[r] = K[i];
    }
    for (int q = tid; q < d_total; q += kThrThreads) {
      const int r = q + lower_bound_u64(K, size, dsort[q]) - drop;
      if (r >= 0) KN[r] = dsort[q];
    }
    __syncthreads();
    cur ^= 1;
    size = new_size;
  }
}

static size_t threshold_smem_bytes() { return (2 * kMaxScored + kBlock) * sizeof(uint64_t); }

cudaError_t launch_prefix_thresholds(const ThresholdParams& p, int n_kv_heads, cudaStream_t stream) {
  const size_t smem = threshold_smem_bytes();
  cudaError_t e = cudaFuncSetAttribute(prefix_thresholds_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  dim3 grid(p.n_seqs, n_kv_heads);
  prefix_thresholds_kernel<<<grid, kThrThreads, smem, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace kvpop
