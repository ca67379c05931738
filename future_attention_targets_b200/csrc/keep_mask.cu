// Sink + top-k + recent-window keep mask, sm_100a.
//
// Each (sequence, KV head) row is handled by a cluster of C CTAs (512 threads
// each; C = 1, 2, 4 or 8, chosen per call so that the clusters fill the GPU:
// 8 for a few long rows, fewer for many rows).  CTA r of the cluster owns the
// r-th of C slices of the candidate positions [sinks, L - window) and caches
// their 32-bit order-preserving keys in shared memory.  The k-th largest score
// is found by an exact radix select (four 8-bit digits): each pass every CTA
// histograms its slice, the C histograms are summed through distributed
// shared memory, and every CTA takes the same digit.  Then each CTA writes the
// mask of its slice, keeping every candidate above the threshold and, of those
// equal to it, the ones with the smallest positions: a CTA's rank among the
// equal keys starts after the equal keys of the slices before it (one count
// per CTA, read across the cluster) and continues in position order inside
// it.  All arithmetic is integer, so the result is exact.
#include <cooperative_groups.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>

#include "kvpop_debug.cuh"
#include "kvpop_sched.h"

namespace kvpop {

namespace cg = cooperative_groups;

constexpr int kKeepThreads = 512;
constexpr int kKeepWarps = kKeepThreads / 32;
constexpr int kKeepMaxCluster = 8;
constexpr int kKeepSliceMax = 16384;      // keys one CTA caches at most (64 KiB); 8 x 16384 = the longest row

// Order-preserving key: larger float -> larger key; -0 == +0; NaN -> 0,
// below every number (including -inf, which maps to 0x007fffff).
__device__ __forceinline__ uint32_t order_key(float f) {
  uint32_t u = __float_as_uint(f);
  if ((u & 0x7fffffffu) > 0x7f800000u) return 0u;
  if (u == 0x80000000u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

template <int kKeepCluster>
__global__ void __launch_bounds__(kKeepThreads, 2) keep_mask_kernel(const __grid_constant__ KeepParams p) {
  cg::cluster_group cluster = cg::this_cluster();
  extern __shared__ uint32_t keys[];        // order keys of this CTA's candidate slice
  __shared__ uint32_t hist[kKeepWarps][256];
  __shared__ uint32_t bins[2][256];         // this CTA's histogram of a pass (read by the whole cluster)
  __shared__ uint32_t gbins[256];           // the cluster's histogram
  __shared__ uint32_t sel[2];               // chosen digit, remaining rank inside it
  __shared__ uint32_t warp_tot[kKeepWarps];
  __shared__ uint32_t warp_off[kKeepWarps + 1];
  __shared__ uint32_t eq_count;             // keys of this slice equal to the threshold

  const int r = static_cast<int>(cluster.block_rank());
  const int b = blockIdx.x / kKeepCluster, h = blockIdx.y;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int32_t s = p.seq_start[b], L = p.seq_len[b], B = p.budget[b];
  const float* score = p.score + static_cast<int64_t>(h) * p.total_tokens + s;
  uint8_t* keep = p.keep + static_cast<int64_t>(h) * p.total_tokens + s;
  // Debug build: positions i of this row must lie inside [0, T) once offset by s.
  auto in_row = [&](int32_t i, int32_t site) {
    return KVPOP_IN(i >= 0 && i < L && s >= 0 && s + i < p.total_tokens, p.dbg, DBG_KEEP, site);
  };

#if KVPOP_PDL_PASSES
  // A programmatic dependent of the kernel that wrote the scores: everything
  // above overlapped its tail.
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
#endif
  // Every branch below depends only on (b, h): all CTAs of a cluster take it.
  if (L <= B) {
    for (int32_t i = r * kKeepThreads + tid; i < L; i += kKeepCluster * kKeepThreads)
      if (in_row(i, 1)) keep[i] = 1;
    return;
  }
  const int32_t S = p.sinks, W = p.window;
  const int32_t lo = S, hi = L - W;          // candidates; hi > lo because L > B >= S + W
  const int32_t chunk = (hi - lo + kKeepCluster - 1) / kKeepCluster;
  const int32_t s0 = min(hi, lo + r * chunk), s1 = min(hi, s0 + chunk);
  for (int32_t i = s0 + tid; i < s1; i += kKeepThreads)
    if (in_row(i, 2) && KVPOP_IN(i - s0 < p.key_cap, p.dbg, DBG_KEEP, 3)) keys[i - s0] = order_key(__ldg(score + i));
  if (r == 0)
    for (int32_t i = tid; i < S; i += kKeepThreads)
      if (in_row(i, 4)) keep[i] = 1;
  if (r == kKeepCluster - 1)
    for (int32_t i = hi + tid; i < L; i += kKeepThreads)
      if (in_row(i, 4)) keep[i] = 1;
  __syncthreads();

  uint32_t need = static_cast<uint32_t>(B - S - W);  // rank (1-based) of the threshold among candidates
  uint32_t prefix = 0, pmask = 0;
  if (need == 0) prefix = 0xffffffffu;  // no scored slots: no key can reach the threshold
  int pass = 0;
  for (int shift = 24; shift >= 0 && need > 0; shift -= 8, ++pass) {
    for (int i = tid; i < kKeepWarps * 256; i += kKeepThreads) (&hist[0][0])[i] = 0;
    __syncthreads();
    for (int32_t i = tid; i < s1 - s0; i += kKeepThreads) {
      if (!KVPOP_IN(i < p.key_cap, p.dbg, DBG_KEEP, 5)) break;
      const uint32_t u = keys[i];
      if ((u & pmask) == prefix) atomicAdd(&hist[warp][(u >> shift) & 255u], 1u);
    }
    __syncthreads();
    uint32_t* mine = bins[pass & 1];
    if (tid < 256) {
      uint32_t c = 0;
#pragma unroll
      for (int w = 0; w < kKeepWarps; ++w) c += hist[w][tid];
      mine[tid] = c;
    }
    // Every CTA's histogram of this pass is written.  A buffer is rewritten
    // two passes later, after every CTA has passed this barrier once more,
    // so its readers are done with it.
    cluster.sync();
    if (tid < 256) {
      uint32_t c = 0;
#pragma unroll
      for (int q = 0; q < kKeepCluster; ++q) c += cluster.map_shared_rank(mine, q)[tid];
      gbins[tid] = c;
    }
    __syncthreads();
    if (warp == 0) {
      // Lane l covers digits 255-8l .. 248-8l (descending); find the digit
      // holding the need-th largest key.
      uint32_t cnt[8], tot = 0;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        cnt[q] = gbins[255 - 8 * lane - q];
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
  {
    uint32_t c = 0;
    for (int32_t i = tid; i < s1 - s0 && KVPOP_IN(i < p.key_cap, p.dbg, DBG_KEEP, 5); i += kKeepThreads)
      c += keys[i] == tau;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
    if (lane == 0) warp_tot[warp] = c;
    __syncthreads();
    if (tid == 0) {
      uint32_t t = 0;
      for (int w = 0; w < kKeepWarps; ++w) t += warp_tot[w];
      eq_count = t;
    }
  }
  cluster.sync();
  uint32_t seen_eq = 0;                     // equal keys in the slices before this one
  for (int q = 0; q < r; ++q) seen_eq += *cluster.map_shared_rank(&eq_count, q);
  for (int32_t base = s0; base < s1; base += kKeepThreads) {
    const int32_t i = base + tid;
    const bool in = i < s1 && KVPOP_IN(i - s0 < p.key_cap, p.dbg, DBG_KEEP, 5);
    const uint32_t u = in ? keys[i - s0] : 0u;
    const bool eq = in && u == tau;
    const uint32_t m = __ballot_sync(0xffffffffu, eq);
    if (lane == 0) warp_tot[warp] = __popc(m);
    __syncthreads();
    if (warp == 0) {   // exclusive scan of the warp counts, once for the block
      const uint32_t v = lane < kKeepWarps ? warp_tot[lane] : 0u;
      uint32_t incl = v;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      if (lane < kKeepWarps) warp_off[lane] = incl - v;
      if (lane == kKeepWarps - 1) warp_off[kKeepWarps] = incl;
    }
    __syncthreads();
    const uint32_t rank = seen_eq + warp_off[warp] + __popc(m & ((1u << lane) - 1u));
    if (in && in_row(i, 6)) keep[i] = (u > tau || (eq && rank < keep_eq)) ? 1 : 0;
    seen_eq += warp_off[kKeepWarps];
    __syncthreads();
  }
  // No CTA leaves while another may still read its shared memory.
  cluster.sync();
}

template <int kC>
static cudaError_t launch_keep_cluster(const KeepParams& p, int n_kv_heads, int smem, cudaStream_t stream) {
  cudaError_t e = cudaFuncSetAttribute(keep_mask_kernel<kC>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.n_seqs * kC, n_kv_heads);
  cfg.blockDim = dim3(kKeepThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = kC;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = KVPOP_PDL_PASSES ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, keep_mask_kernel<kC>, p);
}

// Cluster size: the largest of 8, 4, 2, 1 whose rows x size still fit two
// CTAs per SM (measured on the 16k / 64k rows: 8 -> 17 / 26 us against 24 / 111
// us for one CTA per row; on 64 varlen rows 4 -> 19 us where 8 takes 32), but
// never so small that the longest slice outgrows kKeepSliceMax.
cudaError_t launch_keep_mask(const KeepParams& p, int n_kv_heads, int sm_count, cudaStream_t stream) {
  int32_t max_cand = 1;
  for (int b = 0; b < p.n_seqs; ++b) max_cand = std::max(max_cand, p.seq_len[b] - p.sinks - p.window);
  const int64_t rows = static_cast<int64_t>(p.n_seqs) * n_kv_heads;
  int c = kKeepMaxCluster;
  while (c > 1 && rows * c > 2 * static_cast<int64_t>(sm_count)) c >>= 1;
  while (c < kKeepMaxCluster && (max_cand + c - 1) / c > kKeepSliceMax) c <<= 1;
  const int slice = (max_cand + c - 1) / c;
  const int smem = ((slice + 3) / 4) * 16;
  KeepParams q = p;
  q.key_cap = smem / 4;
  switch (c) {
    case 1: return launch_keep_cluster<1>(q, n_kv_heads, smem, stream);
    case 2: return launch_keep_cluster<2>(q, n_kv_heads, smem, stream);
    case 4: return launch_keep_cluster<4>(q, n_kv_heads, smem, stream);
    default: return launch_keep_cluster<8>(q, n_kv_heads, smem, stream);
  }
}

}  // namespace kvpop
