// Sink + top-k + recent-window keep mask, sm_100a.
//
// One CTA of 1024 threads per (sequence, KV head).  The k-th largest score
// among the candidate positions [sinks, L - window) is found by an exact
// radix select on 32-bit order-preserving keys (four 8-bit digits, one
// histogram pass over the row each, the keys cached in shared memory); then a
// single ordered pass writes the mask, keeping every candidate above the
// threshold and, of those equal to it, the ones with the smallest positions
// (a block-wide prefix count in position order).  All arithmetic is integer,
// so the result is exact.
#include <cuda_runtime.h>
#include <stdint.h>

#include "kvpop_sched.h"

namespace kvpop {

constexpr int kKeepThreads = 1024;
constexpr int kKeepWarps = kKeepThreads / 32;

// Order-preserving key: larger float -> larger key; -0 == +0; NaN -> 0,
// below every number (including -inf, which maps to 0x007fffff).
__device__ __forceinline__ uint32_t order_key(float f) {
  uint32_t u = __float_as_uint(f);
  if ((u & 0x7fffffffu) > 0x7f800000u) return 0u;
  if (u == 0x80000000u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

constexpr int kKeepCache = 16384;   // candidate keys kept in shared memory (longer rows re-read L2)

__global__ void __launch_bounds__(kKeepThreads, 1) keep_mask_kernel(const __grid_constant__ KeepParams p) {
  extern __shared__ uint32_t keys[];   // kKeepCache order keys of the candidates
  __shared__ uint32_t hist[kKeepWarps][256];
  __shared__ uint32_t bins[256];
  __shared__ uint32_t sel[2];          // chosen digit, remaining rank inside it
  __shared__ uint32_t warp_tot[kKeepWarps];
  __shared__ uint32_t warp_off[kKeepWarps + 1];

  const int b = blockIdx.x, h = blockIdx.y;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int32_t s = p.seq_start[b], L = p.seq_len[b], B = p.budget[b];
  const float* score = p.score + static_cast<int64_t>(h) * p.total_tokens + s;
  uint8_t* keep = p.keep + static_cast<int64_t>(h) * p.total_tokens + s;

  if (L <= B) {
    for (int32_t i = tid; i < L; i += kKeepThreads) keep[i] = 1;
    return;
  }
  const int32_t S = p.sinks, W = p.window;
  const int32_t lo = S, hi = L - W;    // candidates; hi > lo because L > B >= S + W
  const bool cached = (hi - lo) <= kKeepCache;
  if (cached)
    for (int32_t i = lo + tid; i < hi; i += kKeepThreads) keys[i - lo] = order_key(__ldg(score + i));
  __syncthreads();
  auto key_at = [&](int32_t i) -> uint32_t { return cached ? keys[i - lo] : order_key(__ldg(score + i)); };
  uint32_t need = static_cast<uint32_t>(B - S - W);  // rank (1-based) of the threshold among candidates
  uint32_t prefix = 0, pmask = 0;
  if (need == 0) prefix = 0xffffffffu;  // no scored slots: no key can exceed the threshold

  for (int shift = 24; shift >= 0 && need > 0; shift -= 8) {
    for (int i = tid; i < kKeepWarps * 256; i += kKeepThreads) (&hist[0][0])[i] = 0;
    __syncthreads();
    for (int32_t i = lo + tid; i < hi; i += kKeepThreads) {
      const uint32_t u = key_at(i);
      if ((u & pmask) == prefix) atomicAdd(&hist[warp][(u >> shift) & 255u], 1u);
    }
    __syncthreads();
    if (tid < 256) {
      uint32_t c = 0;
#pragma unroll 8
      for (int w = 0; w < kKeepWarps; ++w) c += hist[w][tid];
      bins[tid] = c;
    }
    __syncthreads();
    if (warp == 0) {
      // Lane l covers digits 255-8l .. 248-8l (descending); find the digit
      // holding the need-th largest key.
      uint32_t cnt[8], tot = 0;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        cnt[q] = bins[255 - 8 * lane - q];
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
        sel[0] = 255u - 8u * lane - q;
        sel[1] = need - before;
      }
    }
    __syncthreads();
    prefix |= sel[0] << shift;
    pmask |= 255u << shift;
    need = sel[1];
    __syncthreads();
  }
  // prefix = the threshold key; keep the `need` smallest positions equal to it.
  const uint32_t tau = prefix, keep_eq = need;
  uint32_t seen_eq = 0;
  for (int32_t base = 0; base < L; base += kKeepThreads) {
    const int32_t i = base + tid;
    uint32_t u = 0;
    bool cand = false;
    if (i < L) {
      cand = (i >= lo && i < hi);
      if (cand) u = key_at(i);
    }
    const bool eq = cand && u == tau;
    const uint32_t m = __ballot_sync(0xffffffffu, eq);
    if (lane == 0) warp_tot[warp] = __popc(m);
    __syncthreads();
    if (warp == 0) {   // exclusive scan of the warp counts, once for the block
      const uint32_t v = warp_tot[lane];
      uint32_t incl = v;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      warp_off[lane] = incl - v;
      if (lane == 31) warp_off[kKeepWarps] = incl;
    }
    __syncthreads();
    const uint32_t rank = seen_eq + warp_off[warp] + __popc(m & ((1u << lane) - 1u));
    if (i < L) {
      const bool k = (i < S) || (i >= hi) || (cand && (u > tau || (eq && rank < keep_eq)));
      keep[i] = k ? 1 : 0;
    }
    seen_eq += warp_off[kKeepWarps];
    __syncthreads();
  }
}

cudaError_t launch_keep_mask(const KeepParams& p, int n_kv_heads, cudaStream_t stream) {
  const int smem = kKeepCache * static_cast<int>(sizeof(uint32_t));
  cudaError_t e = cudaFuncSetAttribute(keep_mask_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  dim3 grid(p.n_seqs, n_kv_heads);
  keep_mask_kernel<<<grid, kKeepThreads, smem, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace kvpop
