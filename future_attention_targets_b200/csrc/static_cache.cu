// Static fixed-budget cache: compaction of the kept K/V rows, and one decode
// step of attention over the compacted cache, sm_100a.
//
// Both are memory-bound (a gather, and a GEMV with G query heads per KV
// head), so they run on CUDA cores with 16-byte vector accesses; the grid is
// split along the sequence / the cache slots so that every SM streams.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include <algorithm>
#include <mutex>

#include "kvpop_cache.h"
#include "kvpop_debug.cuh"

namespace kvpop {

// ------------------------------------------------------------------ compaction

constexpr int kCompactThreads = 512;    // short per-thread mask runs: 32 positions at 16k
constexpr int kCompactUnroll = 8;       // 16-byte words each thread has in flight (128 rows = one round)

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

// Exclusive prefix sum over the block's threads; *total gets the sum.
__device__ __forceinline__ int block_exclusive_scan(int x, int* warp_sums, int* total) {
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
  // Launched as a programmatic dependent: everything above overlapped the
  // previous kernel's tail; its writes (the keep mask) are visible after this.
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  const int chunk = (L + kCompactThreads - 1) / kCompactThreads;
  const int c0 = min(L, tid * chunk), c1 = min(L, c0 + chunk);
  // Debug build: the mask row [s0, s0 + L) of head h lies inside [H_kv, T].
  KVPOP_CHECK(s0 >= 0 && s0 + L <= p.total_tokens && h < p.n_kv_heads, p.dbg, DBG_COMPACT, 1);
  const int mine = count_kept(mask, c0, c1);
  int total = 0;
  const int first = block_exclusive_scan(mine, warp_sums, &total);
  if (first < S1 && first + mine > S0) {
    int slot = first;
    for_each_kept(mask, c0, c1, [&](int i) {
      if (slot >= S0 && slot < S1 && KVPOP_IN(slot - S0 < kCompactSlots, p.dbg, DBG_COMPACT, 2)) list_pos[slot - S0] = i;
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
        buf[u] = KVPOP_IN(list_pos[e] >= 0 && list_pos[e] < L && s0 + list_pos[e] < p.total_tokens, p.dbg,
                          DBG_COMPACT, 3)
                     ? __ldg(reinterpret_cast<const uint4*>((is_v ? p.v : p.k) + src))
                     : make_uint4(0, 0, 0, 0);
      }
    }
#pragma unroll
    for (int u = 0; u < kCompactUnroll; ++u) {
      const int idx = base + u * kCompactThreads;
      if (idx < total_words) {
        const int e = idx / kRowWords, rem = idx - e * kRowWords;
        const bool is_v = rem >= kWords;
        const int w = is_v ? rem - kWords : rem;
        if (KVPOP_IN(S0 + e < p.capacity, p.dbg, DBG_COMPACT, 4))
          *reinterpret_cast<uint4*>((is_v ? p.v_cache : p.k_cache) + (row0 + S0 + e) * d + w * 8) = buf[u];
      }
    }
  }
  // Slot positions (-1 when unused) and zeros in the unused rows.
  for (int e = tid; e < S1 - S0; e += kCompactThreads)
    if (KVPOP_IN(S0 + e < p.capacity && e < kCompactSlots, p.dbg, DBG_COMPACT, 5))
      p.pos[row0 + S0 + e] = (e < n_fill) ? list_pos[e] : -1;
  const int clear_words = (S1 - S0 - n_fill) * kWords;
  KVPOP_CHECK(S0 + n_fill + clear_words / kWords <= p.capacity, p.dbg, DBG_COMPACT, 4);
  uint4* kz = reinterpret_cast<uint4*>(p.k_cache + (row0 + S0 + n_fill) * d);
  uint4* vz = reinterpret_cast<uint4*>(p.v_cache + (row0 + S0 + n_fill) * d);
  for (int i = tid; i < clear_words; i += kCompactThreads) {
    kz[i] = make_uint4(0, 0, 0, 0);
    vz[i] = make_uint4(0, 0, 0, 0);
  }
  if (c == 0 && tid == 0 && KVPOP_IN(b < p.n_seqs, p.dbg, DBG_COMPACT, 6)) p.count[b * p.n_kv_heads + h] = total;
}

// Launch with programmatic stream serialization: the kernel may start while
// the previous kernel in the stream finishes, and waits for it
// (griddepcontrol.wait) before its first read of global memory.
template <class Kern, class Params>
static cudaError_t launch_dependent(Kern kern, dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                                    const Params& p) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, p);
}

cudaError_t launch_compact_kv(const CompactParams& p, cudaStream_t stream) {
  dim3 grid(p.n_seqs * p.n_kv_heads, (p.capacity + kCompactSlots - 1) / kCompactSlots);
  return p.head_dim == 128 ? launch_dependent(compact_kv_kernel<128>, grid, dim3(kCompactThreads), 0, stream, p)
                           : launch_dependent(compact_kv_kernel<64>, grid, dim3(kCompactThreads), 0, stream, p);
}

// ------------------------------------------------------------------ decode attention

// A decode CTA has kDecWarps(kS) warps, each owning kDecSplit / warps slots of
// every chunk: 8 warps of 16 slots when it streams chunks through kS > 1
// buffers (one CTA per SM: two warps per scheduler hide the MMA chains), 4
// warps of 32 when it takes a single chunk (two CTAs per SM fit the registers).
template <int kS>
__host__ __device__ constexpr int kDecWarps() { return kS > 1 ? 8 : 4; }

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
  const uint32_t s = static_cast<uint32_t>(__cvta_generic_to_shared(smem));
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(s), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// Warp-level bf16 MMA (m16n8k16, fp32 accumulate) and the shared-memory
// matrix loads that feed it.  A decode step is a G x d by d x n product and
// its P.V follow-up; with the G query heads padded to the MMA's 16 rows one
// instruction does the multiply-adds that would otherwise take hundreds of
// scalar ones, which keeps this memory-bound kernel off the issue limit.
__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], const uint16_t* row) {
  const uint32_t a = static_cast<uint32_t>(__cvta_generic_to_shared(row));
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(a));
}
__device__ __forceinline__ void ldsm_x4_trans(uint32_t (&r)[4], const uint16_t* row) {
  const uint32_t a = static_cast<uint32_t>(__cvta_generic_to_shared(row));
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(a));
}
__device__ __forceinline__ void mma_bf16(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}
__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xffff0000u); }

// Shared-memory address of 16-byte chunk `c` of cache row `r` (rows of HD
// bf16): the chunks of a row are permuted by r mod 8, so the eight row
// addresses of an ldmatrix hit eight different bank groups.
template <int HD>
__device__ __forceinline__ uint16_t* swz(uint16_t* base, int r, int c) {
  return base + r * HD + ((c ^ (r & 7)) << 3);
}

// One CTA: KV head h of sequence b, all G <= 16 query heads of its group, over
// a contiguous range of the filled 128-slot chunks of its cache row (the
// whole row when there are enough rows to fill the GPU; otherwise the row is
// split over p.n_split CTAs whose partials a merge kernel combines).  Each
// warp owns its share of the slots of every chunk and streams its slices through
// a ring of kDecStages shared-memory buffers with cp.async, two chunks ahead
// of the one it computes (rows past the filled slots are zeroed so that
// 0 x garbage cannot make a NaN).  Per chunk:
//   S = Q K^T   16 (heads, padded) x the warp's keys, fp32, by MMA (q unscaled bf16,
//               the scale applied to S in fp32)
//   softmax     a running max and sum per head over the warp's keys so far
//               (rows of S live on four lanes); O is rescaled when the max grows
//   O += P V    16 x d, P split into bf16 high and low parts (two MMAs) so the
//               product keeps ~16 bits of P
// and at the end the warps' (max, sum, O) are merged in shared memory
// into the output (one CTA per row) or this CTA's partial.  kDecStages
// buffers (kDecStages - 1 chunks in flight while one is computed) when a CTA
// streams several chunks; one buffer when it has a single chunk, which leaves
// room for three CTAs per SM.
template <int HD, int kDecStages>
__global__ void __launch_bounds__(32 * kDecWarps<kDecStages>()) decode_split_kernel(const __grid_constant__ DecodeParams p) {
  constexpr int kDecThreads = 32 * kDecWarps<kDecStages>();
  constexpr int kDecRowsPerWarp = kDecSplit / kDecWarps<kDecStages>();
  constexpr int kDecKeyTiles = kDecRowsPerWarp / 8;       // 8-key tiles of S per warp
  static_assert(kDecRowsPerWarp % 16 == 0, "whole 16-key MMA steps per warp");
  constexpr int kChunks = HD / 8;      // 16-byte chunks per row
  constexpr int KS = HD / 16;          // k-steps of S = Q K^T
  constexpr int NT = HD / 8;           // 8-column tiles of O
  constexpr int kWarpStage = 2 * kDecRowsPerWarp * HD;     // bf16 elements: a warp's K then V rows of one chunk
  extern __shared__ __align__(16) uint16_t dec_smem[];     // [warp][stage] K rows, V rows (swizzled)
  __shared__ float sm_m[kDecThreads / 32][16];
  __shared__ float sm_l[kDecThreads / 32][16];

  const int bh = blockIdx.x, part = blockIdx.y;
  const int b = bh / p.n_kv_heads, h = bh - b * p.n_kv_heads;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int gid = lane >> 2, tid4 = lane & 3;
  const int G = p.n_q_heads / p.n_kv_heads;
  [[maybe_unused]] const int batch = static_cast<int>(gridDim.x) / p.n_kv_heads;
  // A programmatic dependent of the previous kernel (the compaction, or the
  // last step): its writes to the cache are visible after this.
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int n = min(p.count[b * p.n_kv_heads + h], p.capacity);
  // This CTA's chunks: its share of the chunk range, cut at the filled slots.
  const int n_chunks = (p.capacity + kDecSplit - 1) / kDecSplit;
  const int per_part = (n_chunks + p.n_split - 1) / p.n_split;
  const int c_lo = part * per_part;
  const int c_hi = min(min(c_lo + per_part, n_chunks), (n + kDecSplit - 1) / kDecSplit);
  const int nch = max(0, c_hi - c_lo);
  uint16_t* wbase = dec_smem + warp * kDecStages * kWarpStage;
  const int64_t row_base = (static_cast<int64_t>(b) * p.n_kv_heads + h) * p.capacity;

  // Issues the cp.async copies of this warp's rows of chunk c_lo + k into stage k % kDecStages.
  auto stage_in = [&](int k) {
    const int w_lo = (c_lo + k) * kDecSplit + warp * kDecRowsPerWarp;
    const int rows = max(0, min(kDecRowsPerWarp, n - w_lo));
    uint16_t* sk = wbase + (k % kDecStages) * kWarpStage;
    uint16_t* sv = sk + kDecRowsPerWarp * HD;
    const int64_t g0 = (row_base + w_lo) * HD;
    for (int idx = lane; idx < rows * kChunks; idx += 32) {
      const int r = idx / kChunks, c = idx - r * kChunks;
      // Debug build: the staged row is one of this (sequence, KV head)'s filled slots.
      if (!KVPOP_IN(w_lo + r < p.capacity && w_lo + r < n && b < batch, p.dbg, DBG_DECODE, 1)) continue;
      cp_async16(swz<HD>(sk, r, c), p.k_cache + g0 + idx * 8);
      cp_async16(swz<HD>(sv, r, c), p.v_cache + g0 + idx * 8);
    }
  };
  // Chunks in flight ahead of the one being computed (a single buffer takes its
  // one chunk here too, so its copies overlap the loads of q below).
  constexpr int kLead = kDecStages > 1 ? kDecStages - 1 : 1;
  constexpr int kWait = kDecStages > 1 ? kDecStages - 1 : 0;   // copy groups that may stay in flight
#pragma unroll
  for (int k = 0; k < kLead; ++k) {
    if (k < nch) stage_in(k);
    cp_async_commit();
  }
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  // q as the A operand: rows = query heads (>= G read as 0), cols = head dims.
  uint32_t qa[KS][4];
  {
    KVPOP_CHECK(h * G + G <= p.n_q_heads && G <= 16, p.dbg, DBG_DECODE, 2);
    const uint16_t* qb = p.q + (static_cast<int64_t>(b) * p.n_q_heads + h * G) * HD;
#pragma unroll
    for (int kk = 0; kk < KS; ++kk) {
      const int d0 = 16 * kk + 2 * tid4;
      qa[kk][0] = (gid < G) ? *reinterpret_cast<const uint32_t*>(qb + gid * HD + d0) : 0u;
      qa[kk][1] = (gid + 8 < G) ? *reinterpret_cast<const uint32_t*>(qb + (gid + 8) * HD + d0) : 0u;
      qa[kk][2] = (gid < G) ? *reinterpret_cast<const uint32_t*>(qb + gid * HD + d0 + 8) : 0u;
      qa[kk][3] = (gid + 8 < G) ? *reinterpret_cast<const uint32_t*>(qb + (gid + 8) * HD + d0 + 8) : 0u;
    }
  }

  // Running state of head rows gid (0) and gid + 8 (1): max (log2 units), sum, O.
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
  float o[NT][4];
#pragma unroll
  for (int t = 0; t < NT; ++t)
#pragma unroll
    for (int e = 0; e < 4; ++e) o[t][e] = 0.f;
  const int mi = lane >> 3, ri = lane & 7;    // this lane's ldmatrix row address: matrix mi, row ri

  for (int k = 0; k < nch; ++k) {
    if constexpr (kDecStages > 1) {
      if (k + kDecStages - 1 < nch) stage_in(k + kDecStages - 1);
    } else {
      if (k >= 1) stage_in(k);                // one buffer: the previous chunk is done with it
    }
    cp_async_commit();
    const int w_lo = (c_lo + k) * kDecSplit + warp * kDecRowsPerWarp;
    const int rows = max(0, min(kDecRowsPerWarp, n - w_lo));
    uint16_t* sk = wbase + (k % kDecStages) * kWarpStage;
    uint16_t* sv = sk + kDecRowsPerWarp * HD;
    // V rows past the filled slots (no copy lands there) are zeroed while the copies fly.
    for (int idx = rows * kChunks + lane; idx < kDecRowsPerWarp * kChunks; idx += 32) {
      const int r = idx / kChunks, c = idx - r * kChunks;
      *reinterpret_cast<uint4*>(swz<HD>(sv, r, c)) = make_uint4(0, 0, 0, 0);
    }
    cp_async_wait<kWait>();                   // chunk k's copies have landed
    __syncwarp();

    // S = Q K^T over the warp's keys: 8-key tiles.
    float s[kDecKeyTiles][4];
#pragma unroll
    for (int j = 0; j < kDecKeyTiles; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) s[j][e] = 0.f;
#pragma unroll
    for (int kk = 0; kk < KS; ++kk) {
#pragma unroll
      for (int np = 0; np < kDecKeyTiles / 2; ++np) {
        uint32_t kb[4];
        ldsm_x4(kb, swz<HD>(sk, 16 * np + (mi >> 1) * 8 + ri, 2 * kk + (mi & 1)));
        mma_bf16(s[2 * np], qa[kk], kb[0], kb[1]);
        mma_bf16(s[2 * np + 1], qa[kk], kb[2], kb[3]);
      }
    }
    // Scale to log2 units, mask keys past the filled slots, chunk max per head row.
    float cm0 = -INFINITY, cm1 = -INFINITY;
#pragma unroll
    for (int j = 0; j < kDecKeyTiles; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int key = 8 * j + 2 * tid4 + (e & 1);
        s[j][e] = (key < rows) ? s[j][e] * p.scale_log2 : -INFINITY;
        if (e < 2) cm0 = fmaxf(cm0, s[j][e]); else cm1 = fmaxf(cm1, s[j][e]);
      }
#pragma unroll
    for (int off = 1; off <= 2; off <<= 1) {
      cm0 = fmaxf(cm0, __shfl_xor_sync(0xffffffffu, cm0, off));
      cm1 = fmaxf(cm1, __shfl_xor_sync(0xffffffffu, cm1, off));
    }
    // New running max; the old sum and O are rescaled by exp2(old - new) (exactly 1 when the max
    // stays, 0 for a row that had nothing yet).
    const float nm0 = fmaxf(m0, cm0), nm1 = fmaxf(m1, cm1);
    const float sc0 = (m0 == -INFINITY) ? 0.f : exp2f(m0 - nm0);
    const float sc1 = (m1 == -INFINITY) ? 0.f : exp2f(m1 - nm1);
    m0 = nm0;
    m1 = nm1;
    float cl0 = 0.f, cl1 = 0.f;
#pragma unroll
    for (int j = 0; j < kDecKeyTiles; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float m = (e < 2) ? nm0 : nm1;
        const float pe = (m == -INFINITY) ? 0.f : exp2f(s[j][e] - m);
        s[j][e] = pe;
        if (e < 2) cl0 += pe; else cl1 += pe;
      }
#pragma unroll
    for (int off = 1; off <= 2; off <<= 1) {
      cl0 += __shfl_xor_sync(0xffffffffu, cl0, off);
      cl1 += __shfl_xor_sync(0xffffffffu, cl1, off);
    }
    l0 = l0 * sc0 + cl0;
    l1 = l1 * sc1 + cl1;
#pragma unroll
    for (int t = 0; t < NT; ++t) {
      o[t][0] *= sc0;
      o[t][1] *= sc0;
      o[t][2] *= sc1;
      o[t][3] *= sc1;
    }

    // O += P V: one k-step per 16 keys, P as the A operand straight from S's
    // registers (high and low bf16 parts), V through transposing matrix loads.
#pragma unroll
    for (int kk = 0; kk < kDecKeyTiles / 2; ++kk) {
      uint32_t ph[4], pl[4];
      const float* t0 = s[2 * kk];
      const float* t1 = s[2 * kk + 1];
      const float src[4][2] = {{t0[0], t0[1]}, {t0[2], t0[3]}, {t1[0], t1[1]}, {t1[2], t1[3]}};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        ph[i] = pack_bf16x2(src[i][0], src[i][1]);
        pl[i] = pack_bf16x2(src[i][0] - bf16_lo(ph[i]), src[i][1] - bf16_hi(ph[i]));
      }
#pragma unroll
      for (int jp = 0; jp < NT / 2; ++jp) {
        uint32_t vb[4];
        ldsm_x4_trans(vb, swz<HD>(sv, 16 * kk + (mi & 1) * 8 + ri, 2 * jp + (mi >> 1)));
        mma_bf16(o[2 * jp], ph, vb[0], vb[1]);
        mma_bf16(o[2 * jp], pl, vb[0], vb[1]);
        mma_bf16(o[2 * jp + 1], ph, vb[2], vb[3]);
        mma_bf16(o[2 * jp + 1], pl, vb[2], vb[3]);
      }
    }
    __syncwarp();    // every lane is done with this stage before a later chunk's copies overwrite it
  }
  cp_async_wait<0>();

  // Merge the warps (the staging area is reused for their outputs),
  // then write the output or this CTA's partial.
  if (tid4 == 0) {
    if (gid < G) {
      sm_m[warp][gid] = m0;
      sm_l[warp][gid] = l0;
    }
    if (gid + 8 < G) {
      sm_m[warp][gid + 8] = m1;
      sm_l[warp][gid + 8] = l1;
    }
  }
  __syncthreads();
  float* so = reinterpret_cast<float*>(dec_smem);          // [warps][G][HD]: fits in one stage's staging area
#pragma unroll
  for (int t = 0; t < NT; ++t) {
    const int d0 = 8 * t + 2 * tid4;
    if (gid < G) {
      so[(warp * G + gid) * HD + d0] = o[t][0];
      so[(warp * G + gid) * HD + d0 + 1] = o[t][1];
    }
    if (gid + 8 < G) {
      so[(warp * G + gid + 8) * HD + d0] = o[t][2];
      so[(warp * G + gid + 8) * HD + d0 + 1] = o[t][3];
    }
  }
  __syncthreads();
  for (int idx = threadIdx.x; idx < G * HD; idx += kDecThreads) {
    const int g = idx / HD, e = idx - g * HD;
    float mm = -INFINITY;
    for (int w = 0; w < kDecThreads / 32; ++w) mm = fmaxf(mm, sm_m[w][g]);
    float ll = 0.f, oo = 0.f;
    if (mm > -INFINITY) {
      for (int w = 0; w < kDecThreads / 32; ++w) {
        const float c = (sm_m[w][g] > -INFINITY) ? exp2f(sm_m[w][g] - mm) : 0.f;
        ll += sm_l[w][g] * c;
        oo += so[(w * G + g) * HD + e] * c;
      }
    }
    const int64_t bg = static_cast<int64_t>(b) * p.n_q_heads + h * G + g;
    if (p.n_split == 1) {
      // The whole row in this CTA: the final output.
      if (!KVPOP_IN(bg < static_cast<int64_t>(batch) * p.n_q_heads, p.dbg, DBG_DECODE, 3)) continue;
      p.out[bg * HD + e] = (ll > 0.f) ? oo / ll : 0.f;
      if (e == 0 && p.lse != nullptr) p.lse[bg] = (ll > 0.f) ? (mm + log2f(ll)) * 0.6931471805599453f : -INFINITY;
      continue;
    }
    const int64_t at = (bg * p.n_split + part) * (HD + 2);
    if (!KVPOP_IN(part < p.n_split && at + HD + 2 <= static_cast<int64_t>(batch) * p.n_q_heads * p.n_split * (HD + 2),
                  p.dbg, DBG_DECODE, 3))
      continue;
    float* dst = p.partial + at;
    dst[e] = oo;
    if (e == 0) {
      dst[HD] = mm;
      dst[HD + 1] = ll;
    }
  }
}

// One CTA per (sequence, query head): merge the splits.  Launched as a
// programmatic dependent of the split kernel, so it waits (griddepcontrol)
// until that grid has finished and its writes are visible.  Up to 64 splits
// the whole partial block is staged in shared memory with every load issued
// at once (one round trip instead of three dependent ones); beyond that the
// split loops are strided over the threads or unrolled so that their loads
// overlap.
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

// Splits whose partials are staged whole in shared memory (one round of
// loads); more splits take the streaming path below.
constexpr int kCombineStagedSplits = 64;

__global__ void __launch_bounds__(128) decode_combine_kernel(const __grid_constant__ DecodeParams p) {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  __shared__ float2 staged[kCombineStagedSplits * 65];       // ns x (d + 2) floats, d <= 128
  __shared__ float wsm[kCombineStagedSplits];
  __shared__ float red2[2];
  if (p.n_split <= kCombineStagedSplits) {
    const int bg = blockIdx.x, tid = threadIdx.x;
    const int d = p.head_dim, ns = p.n_split, stride = d + 2, half = stride / 2;
    const float2* part = reinterpret_cast<const float2*>(p.partial + static_cast<int64_t>(bg) * ns * stride);
    for (int i = tid; i < ns * half; i += 128)                          // every load issued before any use
      if (KVPOP_IN(i < kCombineStagedSplits * 65 && (stride & 1) == 0, p.dbg, DBG_COMBINE, 1)) staged[i] = part[i];
    __syncthreads();
    const float* st = reinterpret_cast<const float*>(staged);
    if (tid < 32) {
      float m = -INFINITY;
      for (int s2 = tid; s2 < ns; s2 += 32) m = fmaxf(m, st[s2 * stride + d]);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      float l = 0.f;
      for (int s2 = tid; s2 < ns; s2 += 32) {
        const float ms = st[s2 * stride + d];
        const float w = (m > -INFINITY && ms > -INFINITY) ? exp2f(ms - m) : 0.f;
        wsm[s2] = w;
        l += st[s2 * stride + d + 1] * w;
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
      if (tid == 0) {
        red2[0] = m;
        red2[1] = l;
      }
    }
    __syncthreads();
    const float mm = red2[0], ll = red2[1];
    for (int e = tid; e < d; e += 128) {
      float oo = 0.f;
      for (int s2 = 0; s2 < ns; ++s2) oo = fmaf(st[s2 * stride + e], wsm[s2], oo);
      if (KVPOP_IN(bg < static_cast<int>(gridDim.x) && e < d, p.dbg, DBG_COMBINE, 2))
        p.out[static_cast<int64_t>(bg) * d + e] = (ll > 0.f) ? oo / ll : 0.f;
    }
    if (tid == 0 && p.lse != nullptr) p.lse[bg] = (ll > 0.f) ? (mm + log2f(ll)) * 0.6931471805599453f : -INFINITY;
    return;
  }
  constexpr int kMaxSplitsInSmem = 1024;      // split weights kept in shared memory (more splits: recomputed)
  __shared__ float red[4];
  __shared__ float wsplit[kMaxSplitsInSmem];
  const int bg = blockIdx.x, tid = threadIdx.x;
  const int d = p.head_dim, ns = p.n_split, stride = d + 2;
  const float* part = p.partial + static_cast<int64_t>(bg) * ns * stride;
  KVPOP_CHECK(ns > kCombineStagedSplits && d <= 128, p.dbg, DBG_COMBINE, 3);
  // Split maxima, their maximum, then each split's weight exp2(m_s - m) and the total sum.
  float mm = -INFINITY;
  for (int s = tid; s < ns; s += 128) mm = fmaxf(mm, part[s * stride + d]);
  mm = block_reduce_128(mm, red, true);
  float ll = 0.f;
  for (int s = tid; s < ns; s += 128) {
    const float m_s = part[s * stride + d];
    const float w = (mm > -INFINITY && m_s > -INFINITY) ? exp2f(m_s - mm) : 0.f;
    if (s < kMaxSplitsInSmem) wsplit[s] = w;
    ll += part[s * stride + d + 1] * w;
  }
  ll = block_reduce_128(ll, red, false);   // its barriers also publish wsplit
  // Output: 16 independent loads in flight per thread before their sums.
  for (int e = tid; e < d; e += 128) {
    float oo = 0.f;
    int s = 0;
    for (; s + 16 <= ns && s + 16 <= kMaxSplitsInSmem; s += 16) {
      float v[16];
#pragma unroll
      for (int u = 0; u < 16; ++u) v[u] = part[(s + u) * stride + e];
#pragma unroll
      for (int u = 0; u < 16; ++u) oo = fmaf(v[u], wsplit[s + u], oo);
    }
    for (; s < ns; ++s) {
      const float m_s = part[s * stride + d];
      const float w = (s < kMaxSplitsInSmem) ? wsplit[s]
                                             : ((mm > -INFINITY && m_s > -INFINITY) ? exp2f(m_s - mm) : 0.f);
      oo = fmaf(part[s * stride + e], w, oo);
    }
    p.out[static_cast<int64_t>(bg) * d + e] = (ll > 0.f) ? oo / ll : 0.f;
  }
  if (tid == 0 && p.lse != nullptr) p.lse[bg] = (ll > 0.f) ? (mm + log2f(ll)) * 0.6931471805599453f : -INFINITY;
}

template <int HD, int kS>
static cudaError_t launch_split(const DecodeParams& p, dim3 grid, cudaStream_t stream) {
  const int smem = kS * 2 * kDecSplit * HD * static_cast<int>(sizeof(uint16_t));   // every warp's K and V rows
  cudaError_t e = cudaFuncSetAttribute(decode_split_kernel<HD, kS>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  return launch_dependent(decode_split_kernel<HD, kS>, grid, dim3(32 * kDecWarps<kS>()), smem, stream, p);
}

// Parts each cache row is split into.  One chunk per CTA (single-buffered,
// three CTAs per SM) when that gives at most about one wave of CTAs; else one
// CTA per row when the rows alone fill the GPU (no partials, no merge), or
// enough parts for about one streaming CTA per SM.
int decode_parts(int rows, int n_chunks, int sm_count) {
  if (static_cast<int64_t>(rows) * n_chunks <= 3 * static_cast<int64_t>(sm_count)) return n_chunks;
  return std::max(1, std::min(n_chunks, sm_count / std::max(1, rows)));
}

cudaError_t launch_decode_attention(const DecodeParams& p, int batch, cudaStream_t stream) {
  dim3 grid(batch * p.n_kv_heads, p.n_split);
  const int n_chunks = (p.capacity + kDecSplit - 1) / kDecSplit;
  const bool single = (n_chunks + p.n_split - 1) / p.n_split == 1;   // one chunk per CTA
  cudaError_t e = (p.head_dim == 128) ? (single ? launch_split<128, 1>(p, grid, stream) : launch_split<128, 3>(p, grid, stream))
                                      : (single ? launch_split<64, 1>(p, grid, stream) : launch_split<64, 3>(p, grid, stream));
  if (e != cudaSuccess) return e;
  if (p.n_split == 1) return cudaSuccess;   // the split kernel wrote the output
  // The merge overlaps its launch with the split kernel's tail.
  return launch_dependent(decode_combine_kernel, dim3(batch * p.n_q_heads), dim3(128), 0, stream, p);
}

// ------------------------------------------------------------------ fixed scratch for the allocation-free decode

// Split partials of kvpop_decode_attention_noalloc live here instead of in a
// caller workspace.  Every device on which this library's kernels run holds
// these bytes until the process exits.
constexpr size_t kDecodeScratchBytes = size_t(4) << 20;
static __device__ __align__(256) float g_decode_scratch[kDecodeScratchBytes / sizeof(float)];

size_t decode_scratch_bytes() { return kDecodeScratchBytes; }

// Unique id of the calling thread's current CUDA context, or 0 when no
// context is current or the driver cannot say.  Ids are never reused, so a
// context created after cudaDeviceReset has a new one.
static unsigned long long current_context_id() {
  using GetCurrent = CUresult (*)(CUcontext*);
  using GetId = CUresult (*)(CUcontext, unsigned long long*);
  static GetCurrent get_current = nullptr;
  static GetId get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<GetCurrent>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<GetId>(p);
  });
  if (get_current == nullptr || get_id == nullptr) return 0;
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr || get_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return id;
}

// Device address of g_decode_scratch on the current device.  In host code the
// symbol's name is only a stand-in, so the address is looked up with the
// device current, once per device, and cached together with the id of the
// context it belongs to.  If that context has since been destroyed (by
// cudaDeviceReset, say), the module is loaded anew at a possibly different
// address, so a changed context id triggers a fresh lookup.
cudaError_t decode_scratch_address(float** out) {
  constexpr int kMaxDevices = 64;
  static std::mutex mu;
  static void* addr[kMaxDevices] = {};
  static unsigned long long ctx_of[kMaxDevices] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(mu);
  const unsigned long long ctx = current_context_id();
  if (addr[dev] == nullptr || ctx == 0 || ctx != ctx_of[dev]) {
    void* ptr = nullptr;
    e = cudaGetSymbolAddress(&ptr, g_decode_scratch);
    if (e != cudaSuccess) return e;
    addr[dev] = ptr;
    ctx_of[dev] = current_context_id();   // the lookup makes the device's primary context current
  }
  *out = static_cast<float*>(addr[dev]);
  return cudaSuccess;
}

}  // namespace kvpop
