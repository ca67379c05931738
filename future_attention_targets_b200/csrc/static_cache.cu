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

#include "kvpop_cache.h"

namespace kvpop {

// ------------------------------------------------------------------ compaction

constexpr int kCompactThreads = 256;
constexpr int kCompactUnroll = 16;     // 16-byte words each thread has in flight

// Non-zero bytes of a 32-bit word: bit 7 of ((b & 0x7f) + 0x7f) | b is set
// exactly when the byte b is non-zero, and the sum cannot carry into the next byte.
__device__ __forceinline__ uint32_t nonzero_byte_bits(uint32_t x) {
  return (((x & 0x7f7f7f7fu) + 0x7f7f7f7fu) | x) & 0x80808080u;
}
// The 16 non-zero flags of a 16-byte word as a 16-bit mask (bit i = byte i).
__device__ __forceinline__ uint32_t nonzero_mask16(uint4 w) {
  const uint32_t a = nonzero_byte_bits(w.x), b = nonzero_byte_bits(w.y);
  const uint32_t c = nonzero_byte_bits(w.z), e = nonzero_byte_bits(w.w);
  // gather bit 7 of every byte: byte j of a word -> bit j
  auto pick = [](uint32_t v) { return ((v >> 7) & 1u) | ((v >> 14) & 2u) | ((v >> 21) & 4u) | ((v >> 28) & 8u); };
  return pick(a) | (pick(b) << 4) | (pick(c) << 8) | (pick(e) << 12);
}

// Calls f(i) for every i in [lo, hi) with mask[i] != 0, in increasing order:
// scalar bytes up to the first 16-byte boundary and after the last one,
// 16-byte loads in between.  Returns how many it visited.
template <typename F>
__device__ __forceinline__ int for_each_kept(const uint8_t* mask, int lo, int hi, F&& f) {
  int n = 0;
  if (hi <= lo) return 0;
  const int head = min(hi - lo, static_cast<int>((16u - (reinterpret_cast<uintptr_t>(mask + lo) & 15u)) & 15u));
  for (int i = lo; i < lo + head; ++i)
    if (mask[i]) f(i), ++n;
  const int mid = lo + head, n16 = (hi - mid) >> 4;
  const uint4* v = reinterpret_cast<const uint4*>(mask + mid);
  for (int w = 0; w < n16; ++w) {
    uint32_t bits = nonzero_mask16(__ldg(v + w));
    while (bits) {
      const int j = __ffs(bits) - 1;
      bits &= bits - 1;
      f(mid + (w << 4) + j);
      ++n;
    }
  }
  for (int i = mid + (n16 << 4); i < hi; ++i)
    if (mask[i]) f(i), ++n;
  return n;
}

__device__ __forceinline__ int count_kept(const uint8_t* mask, int lo, int hi) {
  int n = 0;
  if (hi <= lo) return 0;
  const int head = min(hi - lo, static_cast<int>((16u - (reinterpret_cast<uintptr_t>(mask + lo) & 15u)) & 15u));
  for (int i = lo; i < lo + head; ++i) n += mask[i] != 0;
  const int mid = lo + head, n16 = (hi - mid) >> 4;
  const uint4* v = reinterpret_cast<const uint4*>(mask + mid);
  for (int w = 0; w < n16; ++w) {
    const uint4 x = __ldg(v + w);
    n += __popc(nonzero_byte_bits(x.x)) + __popc(nonzero_byte_bits(x.y)) + __popc(nonzero_byte_bits(x.z)) +
         __popc(nonzero_byte_bits(x.w));
  }
  for (int i = mid + (n16 << 4); i < hi; ++i) n += mask[i] != 0;
  return n;
}

// Exclusive prefix sum over the block's 256 threads; *total gets the sum.
__device__ __forceinline__ int block_exclusive_scan_256(int x, int* warp_sums, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = x;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) warp_sums[warp] = incl;
  __syncthreads();
  int before = 0, all = 0;
#pragma unroll
  for (int w = 0; w < kCompactThreads / 32; ++w) {
    before += (w < warp) ? warp_sums[w] : 0;
    all += warp_sums[w];
  }
  *total = all;
  return before + incl - x;
}

// One CTA: cache slots [c * kCompactSlots, (c + 1) * kCompactSlots) of
// sequence b, KV head h.  The slot of a kept position is the number of kept
// positions before it, so every CTA scans the whole mask row (one contiguous
// chunk per thread, counted with 16-byte loads, then one block scan), keeps
// the positions that land in its own slots, and copies those rows.  Splitting
// by output slots gives every CTA the same number of rows to move wherever
// the kept positions cluster.
template <int d>
__global__ void __launch_bounds__(kCompactThreads, 2) compact_kv_kernel(const __grid_constant__ CompactParams p) {
  constexpr int kWords = d / 8;              // 16-byte words per row
  constexpr int kRowWords = 2 * kWords;      // K row then V row
  __shared__ int warp_sums[kCompactThreads / 32];
  __shared__ int32_t list_pos[kCompactSlots];
  const int bh = blockIdx.x, c = blockIdx.y;
  const int b = bh / p.n_kv_heads, h = bh - b * p.n_kv_heads;
  const int32_t s0 = p.seq_start[b], L = p.seq_len[b];
  const int tid = threadIdx.x;
  const uint8_t* mask = p.keep + static_cast<int64_t>(h) * p.total_tokens + s0;
  const int64_t row0 = (static_cast<int64_t>(b) * p.n_kv_heads + h) * p.capacity;   // first slot of (b, h)
  const int S0 = c * kCompactSlots, S1 = min(S0 + kCompactSlots, p.capacity);

  const int chunk = (L + kCompactThreads - 1) / kCompactThreads;
  const int c0 = min(L, tid * chunk), c1 = min(L, c0 + chunk);
  const int mine = count_kept(mask, c0, c1);
  int total = 0;
  const int first = block_exclusive_scan_256(mine, warp_sums, &total);
  if (first < S1 && first + mine > S0) {
    int slot = first;
    for_each_kept(mask, c0, c1, [&](int i) {
      if (slot >= S0 && slot < S1) list_pos[slot - S0] = i;
      ++slot;
    });
  }
  __syncthreads();
  const int n_fill = max(0, min(S1, total) - S0);

  // Copy the rows: word idx is row idx / kRowWords, K for its first kWords
  // words and V for the rest.
  const int total_words = n_fill * kRowWords;
  for (int base = tid; base < total_words; base += kCompactThreads * kCompactUnroll) {
    uint4 buf[kCompactUnroll];
#pragma unroll
    for (int u = 0; u < kCompactUnroll; ++u) {
      const int idx = base + u * kCompactThreads;
      if (idx < total_words) {
        const int e = idx / kRowWords, rem = idx - e * kRowWords;
        const bool is_v = rem >= kWords;
        const int w = is_v ? rem - kWords : rem;
        const int64_t src = (static_cast<int64_t>(s0 + list_pos[e]) * p.n_kv_heads + h) * d + w * 8;
        buf[u] = __ldg(reinterpret_cast<const uint4*>((is_v ? p.v : p.k) + src));
      }
    }
#pragma unroll
    for (int u = 0; u < kCompactUnroll; ++u) {
      const int idx = base + u * kCompactThreads;
      if (idx < total_words) {
        const int e = idx / kRowWords, rem = idx - e * kRowWords;
        const bool is_v = rem >= kWords;
        const int w = is_v ? rem - kWords : rem;
        *reinterpret_cast<uint4*>((is_v ? p.v_cache : p.k_cache) + (row0 + S0 + e) * d + w * 8) = buf[u];
      }
    }
  }
  // Slot positions (-1 when unused) and zeros in the unused rows.
  for (int e = tid; e < S1 - S0; e += kCompactThreads) p.pos[row0 + S0 + e] = (e < n_fill) ? list_pos[e] : -1;
  const int clear_words = (S1 - S0 - n_fill) * kWords;
  uint4* kz = reinterpret_cast<uint4*>(p.k_cache + (row0 + S0 + n_fill) * d);
  uint4* vz = reinterpret_cast<uint4*>(p.v_cache + (row0 + S0 + n_fill) * d);
  for (int i = tid; i < clear_words; i += kCompactThreads) {
    kz[i] = make_uint4(0, 0, 0, 0);
    vz[i] = make_uint4(0, 0, 0, 0);
  }
  if (c == 0 && tid == 0) p.count[b * p.n_kv_heads + h] = total;
}

cudaError_t launch_compact_kv(const CompactParams& p, cudaStream_t stream) {
  dim3 grid(p.n_seqs * p.n_kv_heads, (p.capacity + kCompactSlots - 1) / kCompactSlots);
  if (p.head_dim == 128)
    compact_kv_kernel<128><<<grid, kCompactThreads, 0, stream>>>(p);
  else
    compact_kv_kernel<64><<<grid, kCompactThreads, 0, stream>>>(p);
  return cudaGetLastError();
}

// ------------------------------------------------------------------ decode attention

constexpr int kDecThreads = 128;                          // 4 warps
constexpr int kDecRowsPerWarp = kDecSplit / (kDecThreads / 32);
static_assert(kDecRowsPerWarp == 32, "each warp stages 32 cache rows");

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
  const uint32_t s = static_cast<uint32_t>(__cvta_generic_to_shared(smem));
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(s), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// Packed fp32 pairs (the f32x2 forms issue two lanes of work per instruction).
__device__ __forceinline__ uint64_t dec_pack(float a, float b) {
  uint64_t r;
  asm("mov.b64 %0, {%1,%2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ void dec_unpack(uint64_t v, float& a, float& b) {
  asm("mov.b64 {%0,%1}, %2;" : "=f"(a), "=f"(b) : "l"(v));
}
__device__ __forceinline__ uint64_t dec_fma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t r;
  asm("fma.rn.ftz.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}
__device__ __forceinline__ uint64_t dec_mul2(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("mul.rn.ftz.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
// Two bf16 in one 32-bit word -> the packed pair (low half first).
__device__ __forceinline__ uint64_t bf16x2_to_f32x2(uint32_t w) {
  return dec_pack(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
}

// D consecutive bf16 (D = 2, 4 or 8; 4, 8 or 16 aligned bytes) as D / 2 packed pairs.
template <int D>
__device__ __forceinline__ void load_pairs(const uint16_t* p, uint64_t (&x)[D / 2]) {
  if constexpr (D == 8) {
    const uint4 w = *reinterpret_cast<const uint4*>(p);
    x[0] = bf16x2_to_f32x2(w.x); x[1] = bf16x2_to_f32x2(w.y);
    x[2] = bf16x2_to_f32x2(w.z); x[3] = bf16x2_to_f32x2(w.w);
  } else if constexpr (D == 4) {
    const uint2 w = *reinterpret_cast<const uint2*>(p);
    x[0] = bf16x2_to_f32x2(w.x); x[1] = bf16x2_to_f32x2(w.y);
  } else {
    x[0] = bf16x2_to_f32x2(*reinterpret_cast<const uint32_t*>(p));
  }
}

// Sums v[i] over the N lanes of a lane group for all N indices at once and
// leaves the sum of index `sub` (the lane's index in its group) in that
// lane: at each butterfly level a lane keeps the half of its entries whose
// index bit matches its own lane bit and ships the other half to its partner
// (N - 1 shuffles for N sums).
template <int N>
__device__ __forceinline__ float transpose_reduce(float (&v)[N], int sub) {
#pragma unroll
  for (int w = N / 2; w >= 1; w >>= 1) {
    const bool upper = (sub & w) != 0;
#pragma unroll
    for (int i = 0; i < w; ++i) {
      const float send = upper ? v[i] : v[i + w];
      const float keep = upper ? v[i + w] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, w);
    }
  }
  return v[0];
}

// One CTA: KV head h of sequence b, cache slots [split * kDecSplit, ...), all
// G query heads of the group.  Each warp stages its 32 rows of K and V in
// shared memory with one burst of cp.async (two commit groups, so the first
// rows can be used while the rest arrive), then walks them in batches of
// R = 32 / G rows.  A row is owned by a group of LPR lanes (16 when G <= 4,
// else 32), each holding D = d / LPR head dims, so a warp step covers
// 32 / LPR rows.  The q.k partial sums of a batch (LPR per lane) become one
// score per lane with one transpose-reduce (lane index i * G + g of its group
// = batch row i of the group, head g); the online softmax runs on those
// lanes, then the P.V update with packed f32x2 FMAs.
template <int LPR, int D, int G>
__global__ void __launch_bounds__(kDecThreads) decode_split_kernel(const __grid_constant__ DecodeParams p) {
  constexpr int d = LPR * D;
  constexpr int RS = 32 / LPR;          // rows per warp step
  constexpr int R = 32 / G;             // rows per batch
  constexpr int NI = R / RS;            // rows of one lane group per batch
  constexpr int P = D / 2;              // packed pairs per lane
  constexpr int kWords = d / 8;
  static_assert(NI * G == LPR, "one score per lane after the transpose-reduce");
  extern __shared__ __align__(16) uint16_t dec_smem[];     // K rows [kDecSplit][d], then V rows
  __shared__ float sm_m[kDecThreads / 32][G];
  __shared__ float sm_l[kDecThreads / 32][G];

  const int bh = blockIdx.x, split = blockIdx.y;
  const int b = bh / p.n_kv_heads, h = bh - b * p.n_kv_heads;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int grp = lane / LPR, sub = lane % LPR;
  const int n = min(p.count[b * p.n_kv_heads + h], p.capacity);
  const int w_lo = split * kDecSplit + warp * kDecRowsPerWarp;
  const int rows = max(0, min(kDecRowsPerWarp, n - w_lo));
  uint16_t* sk = dec_smem + warp * kDecRowsPerWarp * d;
  uint16_t* sv = dec_smem + kDecSplit * d + warp * kDecRowsPerWarp * d;
  {
    const int64_t g0 = ((static_cast<int64_t>(b) * p.n_kv_heads + h) * p.capacity + w_lo) * d;
    const int half_words = min(rows, kDecRowsPerWarp / 2) * kWords;
    for (int idx = lane; idx < half_words; idx += 32) {
      cp_async16(sk + idx * 8, p.k_cache + g0 + idx * 8);
      cp_async16(sv + idx * 8, p.v_cache + g0 + idx * 8);
    }
    cp_async_commit();
    for (int idx = half_words + lane; idx < rows * kWords; idx += 32) {
      cp_async16(sk + idx * 8, p.k_cache + g0 + idx * 8);
      cp_async16(sv + idx * 8, p.v_cache + g0 + idx * 8);
    }
    cp_async_commit();
  }
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  uint64_t q2[G][P];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    load_pairs<D>(p.q + (static_cast<int64_t>(b) * p.n_q_heads + h * G + g) * d + sub * D, q2[g]);
    const uint64_t s2 = dec_pack(p.scale_log2, p.scale_log2);   // scores in log2 units
#pragma unroll
    for (int j = 0; j < P; ++j) q2[g][j] = dec_mul2(q2[g][j], s2);
  }
  float m = -INFINITY, l = 0.f;      // running max and sum of head sub % G (equal on all its lanes)
  uint64_t o2[G][P];
#pragma unroll
  for (int g = 0; g < G; ++g)
#pragma unroll
    for (int j = 0; j < P; ++j) o2[g][j] = 0ull;

  bool all_here = false;
  for (int r0 = 0; r0 < rows; r0 += R) {
    if (!all_here) {
      if (r0 + R <= kDecRowsPerWarp / 2) {
        cp_async_wait<1>();
      } else {
        cp_async_wait<0>();
        all_here = true;
      }
      __syncwarp();
    }
    float part[LPR];
#pragma unroll
    for (int i = 0; i < NI; ++i) {
      uint64_t k2[P];
      load_pairs<D>(sk + (r0 + i * RS + grp) * d + sub * D, k2);
#pragma unroll
      for (int g = 0; g < G; ++g) {
        uint64_t acc = dec_mul2(q2[g][0], k2[0]);
#pragma unroll
        for (int j = 1; j < P; ++j) acc = dec_fma2(q2[g][j], k2[j], acc);
        float a, c;
        dec_unpack(acc, a, c);
        part[i * G + g] = a + c;
      }
    }
    float x = transpose_reduce<LPR>(part, sub);
    if (r0 + (sub / G) * RS + grp >= rows) x = -INFINITY;   // past the filled slots (never read below)
    float bm = x;
#pragma unroll
    for (int off = G; off < 32; off <<= 1) bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, off));
    const float mn = fmaxf(m, bm);
    const bool none = (mn == -INFINITY);
    const float corr = none ? 1.f : exp2f(m - mn);
    const float pr = none ? 0.f : exp2f(x - mn);
    float bs = pr;
#pragma unroll
    for (int off = G; off < 32; off <<= 1) bs += __shfl_xor_sync(0xffffffffu, bs, off);
    l = l * corr + bs;
    m = mn;
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const float c = __shfl_sync(0xffffffffu, corr, g);
      const uint64_t c2 = dec_pack(c, c);
#pragma unroll
      for (int j = 0; j < P; ++j) o2[g][j] = dec_mul2(o2[g][j], c2);
    }
#pragma unroll
    for (int i = 0; i < NI; ++i) {
      const int row = r0 + i * RS + grp;
      uint64_t v2[P];
      if (row < rows) {
        load_pairs<D>(sv + row * d + sub * D, v2);
      } else {
#pragma unroll
        for (int j = 0; j < P; ++j) v2[j] = 0ull;
      }
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const float pg = __shfl_sync(0xffffffffu, pr, grp * LPR + i * G + g);
        const uint64_t p2 = dec_pack(pg, pg);
#pragma unroll
        for (int j = 0; j < P; ++j) o2[g][j] = dec_fma2(p2, v2[j], o2[g][j]);
      }
    }
  }
  cp_async_wait<0>();                // nothing left in flight when the staging area is reused

  // The lane groups hold the same dims for different rows: add them up.
#pragma unroll
  for (int g = 0; g < G; ++g)
#pragma unroll
    for (int j = 0; j < P; ++j)
#pragma unroll
      for (int off = LPR; off < 32; off <<= 1) {
        const uint64_t y = __shfl_xor_sync(0xffffffffu, static_cast<unsigned long long>(o2[g][j]), off);
        float a, c, ya, yc;
        dec_unpack(o2[g][j], a, c);
        dec_unpack(y, ya, yc);
        o2[g][j] = dec_pack(a + ya, c + yc);
      }

  // Merge the four warps (the K/V staging area is reused for their outputs),
  // then write this split's partial.
  if (lane < G) {
    sm_m[warp][lane] = m;
    sm_l[warp][lane] = l;
  }
  __syncthreads();
  float* so = reinterpret_cast<float*>(dec_smem);          // [4][G][d]
  if (grp == 0) {
#pragma unroll
    for (int g = 0; g < G; ++g)
#pragma unroll
      for (int j = 0; j < P; ++j) {
        float a, c;
        dec_unpack(o2[g][j], a, c);
        so[(warp * G + g) * d + sub * D + 2 * j] = a;
        so[(warp * G + g) * d + sub * D + 2 * j + 1] = c;
      }
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
        oo += so[(w * G + g) * d + e] * c;
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

// One CTA per (sequence, query head): merge the splits.  Launched as a
// programmatic dependent of the split kernel, so it waits (griddepcontrol)
// until that grid has finished and its writes are visible.  The split loops
// are strided over the threads or unrolled so that their loads overlap.
__device__ __forceinline__ float block_reduce_128(float x, float* red, bool is_max) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float y = __shfl_xor_sync(0xffffffffu, x, o);
    x = is_max ? fmaxf(x, y) : x + y;
  }
  __syncthreads();
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = x;
  __syncthreads();
  float t = red[0];
#pragma unroll
  for (int w = 1; w < 4; ++w) t = is_max ? fmaxf(t, red[w]) : t + red[w];
  return t;
}

__global__ void __launch_bounds__(128) decode_combine_kernel(const __grid_constant__ DecodeParams p) {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  __shared__ float red[4];
  const int bg = blockIdx.x, tid = threadIdx.x;
  const int d = p.head_dim, ns = p.n_split, stride = d + 2;
  const float* part = p.partial + static_cast<int64_t>(bg) * ns * stride;
  float mm = -INFINITY;
  for (int s = tid; s < ns; s += 128) mm = fmaxf(mm, part[s * stride + d]);
  mm = block_reduce_128(mm, red, true);
  float ll = 0.f;
  if (mm > -INFINITY)
    for (int s = tid; s < ns; s += 128) ll += part[s * stride + d + 1] * exp2f(part[s * stride + d] - mm);
  ll = block_reduce_128(ll, red, false);
  for (int e = tid; e < d; e += 128) {
    float oo = 0.f;
    if (mm > -INFINITY) {
#pragma unroll 8
      for (int s = 0; s < ns; ++s) oo += part[s * stride + e] * exp2f(part[s * stride + d] - mm);
    }
    p.out[static_cast<int64_t>(bg) * d + e] = (ll > 0.f) ? oo / ll : 0.f;
  }
  if (tid == 0 && p.lse != nullptr) p.lse[bg] = (ll > 0.f) ? (mm + log2f(ll)) * 0.6931471805599453f : -INFINITY;
}

template <int LPR, int D, int G>
static cudaError_t launch_split_g(const DecodeParams& p, dim3 grid, cudaStream_t stream) {
  const int smem = 2 * kDecSplit * LPR * D * static_cast<int>(sizeof(uint16_t));
  cudaError_t e =
      cudaFuncSetAttribute(decode_split_kernel<LPR, D, G>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  decode_split_kernel<LPR, D, G><<<grid, kDecThreads, smem, stream>>>(p);
  return cudaGetLastError();
}

// Lane groups of 16 for G <= 4 (16-byte slices of a row per lane), of 32
// for larger groups (whose per-lane registers grow with G).
template <int d>
static cudaError_t launch_split(const DecodeParams& p, dim3 grid, int G, cudaStream_t stream) {
  switch (G) {
    case 1: return launch_split_g<16, d / 16, 1>(p, grid, stream);
    case 2: return launch_split_g<16, d / 16, 2>(p, grid, stream);
    case 4: return launch_split_g<16, d / 16, 4>(p, grid, stream);
    case 8: return launch_split_g<32, d / 32, 8>(p, grid, stream);
    default: return launch_split_g<32, d / 32, 16>(p, grid, stream);
  }
}

cudaError_t launch_decode_attention(const DecodeParams& p, int batch, cudaStream_t stream) {
  dim3 grid(batch * p.n_kv_heads, p.n_split);
  const int G = p.n_q_heads / p.n_kv_heads;
  cudaError_t e = (p.head_dim == 128) ? launch_split<128>(p, grid, G, stream) : launch_split<64>(p, grid, G, stream);
  if (e != cudaSuccess) return e;
  // The merge overlaps its launch with the split kernel's tail.
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(batch * p.n_q_heads);
  cfg.blockDim = dim3(128);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, decode_combine_kernel, p);
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
