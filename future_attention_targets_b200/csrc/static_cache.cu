// Static fixed-budget cache: compaction of the kept K/V rows, and one decode
// step of attention over the compacted cache, sm_100a.
//
// Both are memory-bound (a gather, and a GEMV with G query heads per KV
// head), so they run on CUDA cores with 16-byte vector accesses; the grid is
// split along the sequence / the cache slots so that every SM streams.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include <mutex>

#include "kvpop_sched.h"

namespace kvpop {

// ------------------------------------------------------------------ compaction

constexpr int kCompactThreads = 256;

__device__ __forceinline__ int block_sum_256(int x, int* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  __syncthreads();
  if (lane == 0) red[warp] = x;
  __syncthreads();
  int t = 0;
#pragma unroll
  for (int w = 0; w < kCompactThreads / 32; ++w) t += red[w];
  return t;
}

// Copies one row of d bf16 (d * 2 bytes, a multiple of 16) with `lanes` threads.
__device__ __forceinline__ void copy_row(uint16_t* dst, const uint16_t* src, int d, int sub) {
  const int n16 = d / 8;    // 16-byte words per row
  for (int i = sub; i < n16; i += 16)
    reinterpret_cast<uint4*>(dst)[i] = __ldg(reinterpret_cast<const uint4*>(src) + i);
}

__global__ void __launch_bounds__(kCompactThreads) compact_kv_kernel(const __grid_constant__ CompactParams p) {
  __shared__ int red[kCompactThreads / 32];
  __shared__ int32_t list_pos[kCompactRange];
  __shared__ int32_t list_slot[kCompactRange];
  __shared__ int list_n;
  const int bh = blockIdx.x, r = blockIdx.y;
  const int b = bh / p.n_kv_heads, h = bh - b * p.n_kv_heads;
  const int32_t s0 = p.seq_start[b], L = p.seq_len[b];
  const int32_t r0 = r * kCompactRange;
  const int tid = threadIdx.x;
  const uint8_t* mask = p.keep + static_cast<int64_t>(h) * p.total_tokens + s0;
  const int64_t row0 = (static_cast<int64_t>(b) * p.n_kv_heads + h) * p.capacity;   // first slot of (b, h)
  if (r0 >= L && r != p.n_ranges - 1) return;

  // Kept positions before this range.
  int before = 0;
  for (int32_t i = tid; i < min(r0, L); i += kCompactThreads) before += mask[i] ? 1 : 0;
  before = block_sum_256(before, red);

  // This range: slot of every kept position (ballot + warp offsets).
  if (tid == 0) list_n = 0;
  int mine = 0;
  __syncthreads();
  for (int32_t c = r0; c < min(r0 + kCompactRange, L); c += kCompactThreads) {
    const int32_t i = c + tid;
    const bool kept = (i < L) && mask[i] != 0;
    const uint32_t m = __ballot_sync(0xffffffffu, kept);
    const int lane = tid & 31, warp = tid >> 5;
    if (lane == 0) red[warp] = __popc(m);
    __syncthreads();
    int wbefore = 0, tot = 0;
    for (int w = 0; w < kCompactThreads / 32; ++w) {
      wbefore += (w < warp) ? red[w] : 0;
      tot += red[w];
    }
    if (kept) {
      const int k = list_n + wbefore + __popc(m & ((1u << lane) - 1u));
      list_pos[k] = i;
      list_slot[k] = before + k;
    }
    __syncthreads();
    if (tid == 0) list_n += tot;
    __syncthreads();
  }
  mine = list_n;

  // Copy the kept rows: a half-warp per row.
  const int d = p.head_dim;
  const int half = tid >> 4, sub = tid & 15;
  for (int e = half; e < mine; e += kCompactThreads / 16) {
    const int32_t slot = list_slot[e];
    if (slot >= p.capacity) continue;
    const int32_t i = list_pos[e];
    const int64_t src = (static_cast<int64_t>(s0 + i) * p.n_kv_heads + h) * d;
    const int64_t dst = (row0 + slot) * d;
    copy_row(p.k_cache + dst, p.k + src, d, sub);
    copy_row(p.v_cache + dst, p.v + src, d, sub);
    if (sub == 0) p.pos[row0 + slot] = i;
  }

  // The last range also clears the unused slots and writes the count.
  if (r == p.n_ranges - 1) {
    int after = 0;
    for (int32_t i = r0 + kCompactRange + tid; i < L; i += kCompactThreads) after += mask[i] ? 1 : 0;
    after = block_sum_256(after, red);
    const int total = before + mine + after;
    if (tid == 0) p.count[b * p.n_kv_heads + h] = total;
    const int filled = min(total, p.capacity);
    for (int slot = filled + half; slot < p.capacity; slot += kCompactThreads / 16) {
      const int64_t dst = (row0 + slot) * d;
      for (int w = sub; w < d / 8; w += 16) {
        reinterpret_cast<uint4*>(p.k_cache + dst)[w] = make_uint4(0, 0, 0, 0);
        reinterpret_cast<uint4*>(p.v_cache + dst)[w] = make_uint4(0, 0, 0, 0);
      }
      if (sub == 0) p.pos[row0 + slot] = -1;
    }
  }
}

cudaError_t launch_compact_kv(const CompactParams& p, cudaStream_t stream) {
  dim3 grid(p.n_seqs * p.n_kv_heads, p.n_ranges);
  compact_kv_kernel<<<grid, kCompactThreads, 0, stream>>>(p);
  return cudaGetLastError();
}

// ------------------------------------------------------------------ decode attention

constexpr int kDecThreads = 128;       // 4 warps

__device__ __forceinline__ float bf16_to_f32(uint16_t x) { return __uint_as_float(static_cast<uint32_t>(x) << 16); }

// One CTA: KV head h of sequence b, slots [split * kDecSplit, ...), all G query
// heads of the group.  Lane l of a warp owns head dims [l * D, l * D + D), D = d / 32.
template <int D, int G>
__global__ void __launch_bounds__(kDecThreads) decode_split_kernel(const __grid_constant__ DecodeParams p) {
  const int bh = blockIdx.x, split = blockIdx.y;
  const int b = bh / p.n_kv_heads, h = bh - b * p.n_kv_heads;
  constexpr int d = 32 * D;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int n = min(p.count[b * p.n_kv_heads + h], p.capacity);
  const int s_lo = split * kDecSplit, s_hi = min(n, s_lo + kDecSplit);

  __shared__ float sm_m[kDecThreads / 32][G];
  __shared__ float sm_l[kDecThreads / 32][G];
  __shared__ float sm_o[kDecThreads / 32][G][d];

  float qv[G][D];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    const uint16_t* qr = p.q + (static_cast<int64_t>(b) * p.n_q_heads + h * G + g) * d + lane * D;
#pragma unroll
    for (int e = 0; e < D; ++e) qv[g][e] = bf16_to_f32(qr[e]) * p.scale_log2;   // log2 units
  }
  float m[G], l[G], o[G][D];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    m[g] = -INFINITY;
    l[g] = 0.f;
#pragma unroll
    for (int e = 0; e < D; ++e) o[g][e] = 0.f;
  }
  const int64_t base = (static_cast<int64_t>(b) * p.n_kv_heads + h) * p.capacity;
  for (int s = s_lo + warp; s < s_hi; s += kDecThreads / 32) {
    const uint16_t* kr = p.k_cache + (base + s) * d + lane * D;
    const uint16_t* vr = p.v_cache + (base + s) * d + lane * D;
    float kk[D], vv[D];
    if constexpr (D == 4) {
      const uint2 kw = __ldg(reinterpret_cast<const uint2*>(kr));
      const uint2 vw = __ldg(reinterpret_cast<const uint2*>(vr));
      kk[0] = __uint_as_float(kw.x << 16); kk[1] = __uint_as_float(kw.x & 0xffff0000u);
      kk[2] = __uint_as_float(kw.y << 16); kk[3] = __uint_as_float(kw.y & 0xffff0000u);
      vv[0] = __uint_as_float(vw.x << 16); vv[1] = __uint_as_float(vw.x & 0xffff0000u);
      vv[2] = __uint_as_float(vw.y << 16); vv[3] = __uint_as_float(vw.y & 0xffff0000u);
    } else {
      const uint32_t kw = __ldg(reinterpret_cast<const uint32_t*>(kr));
      const uint32_t vw = __ldg(reinterpret_cast<const uint32_t*>(vr));
      kk[0] = __uint_as_float(kw << 16); kk[1] = __uint_as_float(kw & 0xffff0000u);
      vv[0] = __uint_as_float(vw << 16); vv[1] = __uint_as_float(vw & 0xffff0000u);
    }
#pragma unroll
    for (int g = 0; g < G; ++g) {
      float x = 0.f;
#pragma unroll
      for (int e = 0; e < D; ++e) x = fmaf(qv[g][e], kk[e], x);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
      const float mn = fmaxf(m[g], x);
      const float corr = exp2f(m[g] - mn);
      const float pr = exp2f(x - mn);
      l[g] = l[g] * corr + pr;
#pragma unroll
      for (int e = 0; e < D; ++e) o[g][e] = fmaf(pr, vv[e], o[g][e] * corr);
      m[g] = mn;
    }
  }
  // Merge the four warps, then write this split's partial.
#pragma unroll
  for (int g = 0; g < G; ++g) {
    if (lane == 0) {
      sm_m[warp][g] = m[g];
      sm_l[warp][g] = l[g];
    }
#pragma unroll
    for (int e = 0; e < D; ++e) sm_o[warp][g][lane * D + e] = o[g][e];
  }
  __syncthreads();
  for (int idx = threadIdx.x; idx < G * d; idx += kDecThreads) {
    const int g = idx / d, e = idx - g * d;
    float mm = -INFINITY;
    for (int w = 0; w < kDecThreads / 32; ++w) mm = fmaxf(mm, sm_m[w][g]);
    float ll = 0.f, oo = 0.f;
    if (mm > -INFINITY) {
      for (int w = 0; w < kDecThreads / 32; ++w) {
        const float c = exp2f(sm_m[w][g] - mm);
        ll += sm_l[w][g] * c;
        oo += sm_o[w][g][e] * c;
      }
    }
    float* dst = p.partial + ((static_cast<int64_t>(b) * p.n_q_heads + h * G + g) * p.n_split + split) * (d + 2);
    dst[e] = oo;
    if (e == 0) {
      dst[d] = mm;
      dst[d + 1] = ll;
    }
  }
}

// One CTA per (sequence, query head): merge the splits.
__global__ void __launch_bounds__(128) decode_combine_kernel(const __grid_constant__ DecodeParams p) {
  const int bg = blockIdx.x;
  const int d = p.head_dim;
  const float* part = p.partial + static_cast<int64_t>(bg) * p.n_split * (d + 2);
  float mm = -INFINITY;
  for (int s = 0; s < p.n_split; ++s) mm = fmaxf(mm, part[s * (d + 2) + d]);
  float ll = 0.f;
  for (int s = 0; s < p.n_split && mm > -INFINITY; ++s)
    ll += part[s * (d + 2) + d + 1] * exp2f(part[s * (d + 2) + d] - mm);
  for (int e = threadIdx.x; e < d; e += blockDim.x) {
    float oo = 0.f;
    for (int s = 0; s < p.n_split && mm > -INFINITY; ++s)
      oo += part[s * (d + 2) + e] * exp2f(part[s * (d + 2) + d] - mm);
    p.out[static_cast<int64_t>(bg) * d + e] = (ll > 0.f) ? oo / ll : 0.f;
  }
  if (threadIdx.x == 0 && p.lse != nullptr)
    p.lse[bg] = (ll > 0.f) ? (mm + log2f(ll)) * 0.6931471805599453f : -INFINITY;
}


template <int D>
static void launch_split(const DecodeParams& p, dim3 grid, int G, cudaStream_t stream) {
  switch (G) {
    case 1: decode_split_kernel<D, 1><<<grid, kDecThreads, 0, stream>>>(p); break;
    case 2: decode_split_kernel<D, 2><<<grid, kDecThreads, 0, stream>>>(p); break;
    case 4: decode_split_kernel<D, 4><<<grid, kDecThreads, 0, stream>>>(p); break;
    case 8: decode_split_kernel<D, 8><<<grid, kDecThreads, 0, stream>>>(p); break;
    default: decode_split_kernel<D, 16><<<grid, kDecThreads, 0, stream>>>(p); break;
  }
}

cudaError_t launch_decode_attention(const DecodeParams& p, int batch, cudaStream_t stream) {
  dim3 grid(batch * p.n_kv_heads, p.n_split);
  const int G = p.n_q_heads / p.n_kv_heads;
  if (p.head_dim == 128)
    launch_split<4>(p, grid, G, stream);
  else
    launch_split<2>(p, grid, G, stream);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  decode_combine_kernel<<<batch * p.n_q_heads, 128, 0, stream>>>(p);
  return cudaGetLastError();
}

// ------------------------------------------------------------------ fixed scratch for the allocation-free decode

// Split partials of kvpop_decode_attention_noalloc live here instead of in a
// caller workspace.  Every device on which this library's kernels run holds
// these bytes until the process exits.
constexpr size_t kDecodeScratchBytes = size_t(4) << 20;
static __device__ __align__(256) float g_decode_scratch[kDecodeScratchBytes / sizeof(float)];

size_t decode_scratch_bytes() { return kDecodeScratchBytes; }

// Device address of g_decode_scratch on the current device.  In host code the
// symbol's name is only a stand-in, so the address is looked up once per
// device (with that device current) and cached.
cudaError_t decode_scratch_address(float** out) {
  constexpr int kMaxDevices = 64;
  static std::mutex mu;
  static void* addr[kMaxDevices] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(mu);
  if (addr[dev] == nullptr) {
    void* ptr = nullptr;
    e = cudaGetSymbolAddress(&ptr, g_decode_scratch);
    if (e != cudaSuccess) return e;
    addr[dev] = ptr;
  }
  *out = static_cast<float*>(addr[dev]);
  return cudaSuccess;
}

}  // namespace kvpop
