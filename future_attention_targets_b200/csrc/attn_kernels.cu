// The two attention passes of the future-attention target, sm_100a.
//
// Pass 1 (row logsumexp): a CTA owns 128 query rows of one query head (the
// resident A operand) and streams 256-key tiles of its KV head (B) up to the
// causal diagonal.  S = Q K^T lands in TMEM (lane = query, column = key); the
// softmax warps turn each row into a running (offset, sum) pair and write
// lse = ln sum_j exp(s q.k_j).
//
// Pass 2 (transposed pass): a CTA owns 128 keys of one KV head (A) and
// streams 256-query tiles (B) of all G query heads of its group, starting at
// i = j0 + W, where the first key of the tile has left the recent window.
// S^T = K Q^T lands in TMEM with lane = key and column = query, so each
// softmax thread owns one key and adds exp2(s log2e q.k - lse_i log2e) over
// all its queries and heads without any cross-thread reduction.
//
// Warp roles (320 threads, one CTA per SM):
//   warp 0      TMA producer: A tile once per item, B tiles into a 2-stage ring
//   warp 1      TMEM allocator + single-thread tcgen05.mma issuer
//   warps 2..9  softmax: two groups of four warps split the 256 accumulator
//               columns (each warp reads its TMEM lane quadrant, warp % 4)
// Two TMEM accumulators of 256 fp32 columns (all 512 columns) let the MMA of
// tile t+1 run while the softmax warps read tile t.
#include <math.h>

#include <type_traits>

#include "kvpop_device.cuh"

namespace kvpop {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr int kStages = 2;
constexpr int kSoftmaxWarps = 8;

template <int HD>
struct SmemLayout {
  static constexpr int A_HALF = kTileRows * 128;                 // one 64-element column slab of A
  static constexpr int B_HALF = kStreamRows * 128;
  static constexpr int A_BYTES = A_HALF * (HD / 64);
  static constexpr int B_BYTES = B_HALF * (HD / 64);
  static constexpr int OFF_A = 0;                                // 2 buffers
  static constexpr int OFF_B = OFF_A + 2 * A_BYTES;              // kStages buffers
  static constexpr int OFF_LSE = OFF_B + kStages * B_BYTES;      // float [8 warps][2][128]
  static constexpr int OFF_COMB = OFF_LSE + kSoftmaxWarps * 2 * 128 * 4;  // float [2][128]
  static constexpr int OFF_BAR = OFF_COMB + 2 * 128 * 4;
  // a_full[2] a_empty[2] b_full[S] b_empty[S] acc_full[2] acc_empty[2] comb_full comb_empty mma_done
  static constexpr int N_BARS = 4 + 2 * kStages + 4 + 3;
  static constexpr int OFF_MISC = OFF_BAR + N_BARS * 8;
  static constexpr int BYTES = OFF_MISC + 16;
  static constexpr int ALLOC = BYTES + 1024;                     // room to align the base to 1 KiB
};

struct Bars {
  uint64_t* a_full;
  uint64_t* a_empty;
  uint64_t* b_full;
  uint64_t* b_empty;
  uint64_t* acc_full;
  uint64_t* acc_empty;
  uint64_t* comb_full;
  uint64_t* comb_empty;
  uint64_t* mma_done;
};

__device__ __forceinline__ Bars carve_bars(uint64_t* b) {
  Bars r;
  r.a_full = b;
  r.a_empty = b + 2;
  r.b_full = b + 4;
  r.b_empty = b + 4 + kStages;
  r.acc_full = b + 4 + 2 * kStages;
  r.acc_empty = r.acc_full + 2;
  r.comb_full = r.acc_empty + 2;
  r.comb_empty = r.comb_full + 1;
  r.mma_done = r.comb_empty + 1;
  return r;
}

// ------------------------------------------------------------------ policies

// Pass 1: item = (sequence, query tile = level, query head).
struct LsePass {
  struct Item {
    int32_t s, L, g, h, i0, ntiles;
  };
  static __device__ __forceinline__ Item item(const AttnParams& p, int32_t n) {
    const WorkItem w = decode_item(p.sched, n);
    Item it;
    it.s = w.seq_start;
    it.L = w.seq_len;
    it.g = w.head;
    it.h = w.head / p.group;
    it.i0 = w.level * kTileRows;
    it.ntiles = it.i0 / kStreamRows + 1;  // key tiles [0,256), [256,512), ... up to the diagonal
    return it;
  }
  template <int HD>
  static __device__ __forceinline__ void load_a(const AttnParams& p, const Item& it, uint8_t* dst,
                                                uint64_t* bar) {
#pragma unroll
    for (int kh = 0; kh < HD / 64; ++kh)
      tma_load_2d(dst + kh * SmemLayout<HD>::A_HALF, &p.tmap_q, bar, it.g * HD + kh * 64, it.s + it.i0);
  }
  template <int HD>
  static __device__ __forceinline__ void load_b(const AttnParams& p, const Item& it, int32_t t, uint8_t* dst,
                                                uint64_t* bar) {
#pragma unroll
    for (int kh = 0; kh < HD / 64; ++kh)
      tma_load_2d(dst + kh * SmemLayout<HD>::B_HALF, &p.tmap_k, bar, it.h * HD + kh * 64,
                  it.s + t * kStreamRows);
  }
  // The last key tile holds the diagonal; when the query tile starts on a
  // 256-key boundary only its first 128 columns can be unmasked.
  static __device__ __forceinline__ bool half_tile(const Item& it, int32_t t) {
    return t == it.ntiles - 1 && it.i0 == t * kStreamRows;
  }
};

// Pass 2: item = (sequence, key tile, KV head); level = key tiles after this one.
struct TargetPass {
  struct Item {
    int32_t s, L, h, j0, i0, nq, ntiles;
  };
  static __device__ __forceinline__ Item item(const AttnParams& p, int32_t n) {
    const WorkItem w = decode_item(p.sched, n);
    Item it;
    it.s = w.seq_start;
    it.L = w.seq_len;
    it.h = w.head;
    const int32_t nkt = (w.seq_len + kTileRows - 1) / kTileRows;
    it.j0 = (nkt - 1 - w.level) * kTileRows;
    it.i0 = it.j0 + p.window;
    it.nq = it.i0 < it.L ? (it.L - it.i0 + kStreamRows - 1) / kStreamRows : 0;
    it.ntiles = it.nq * p.group;
    return it;
  }
  template <int HD>
  static __device__ __forceinline__ void load_a(const AttnParams& p, const Item& it, uint8_t* dst,
                                                uint64_t* bar) {
#pragma unroll
    for (int kh = 0; kh < HD / 64; ++kh)
      tma_load_2d(dst + kh * SmemLayout<HD>::A_HALF, &p.tmap_k, bar, it.h * HD + kh * 64, it.s + it.j0);
  }
  template <int HD>
  static __device__ __forceinline__ void load_b(const AttnParams& p, const Item& it, int32_t t, uint8_t* dst,
                                                uint64_t* bar) {
    const int32_t g = t / it.nq, qt = t - g * it.nq;
    const int32_t qh = it.h * p.group + g;
#pragma unroll
    for (int kh = 0; kh < HD / 64; ++kh)
      tma_load_2d(dst + kh * SmemLayout<HD>::B_HALF, &p.tmap_q, bar, qh * HD + kh * 64,
                  it.s + it.i0 + qt * kStreamRows);
  }
  static __device__ __forceinline__ bool half_tile(const Item&, int32_t) { return false; }
};

// ------------------------------------------------------------------ roles

// Waits that must end even while the CTA is aborting (teardown drains).
__device__ __forceinline__ bool wait_drain(uint64_t* bar, uint32_t parity, const WaitCtl& ctl) {
  int dummy = 0;
  WaitCtl c2{&dummy, ctl.status, ctl.limit_ns};
  return wait_bounded(bar, parity, c2, SITE_TEARDOWN);
}

template <class Pass, int HD>
__device__ void producer_role(const AttnParams& p, uint8_t* smem, const Bars& bars, const WaitCtl& ctl) {
  using L = SmemLayout<HD>;
  uint32_t a_cnt = 0, b_cnt = 0;
  bool ok = true;
  const int32_t total = p.sched.total_items;
  for (int32_t k = 0; ok; ++k) {
    const int32_t n = cta_item(k, blockIdx.x, gridDim.x);
    if (n >= total) break;
    const typename Pass::Item it = Pass::item(p, n);
    if (it.ntiles == 0) continue;
    const uint32_t ab = a_cnt & 1u;
    if (!wait_bounded(&bars.a_empty[ab], ((a_cnt >> 1) & 1u) ^ 1u, ctl, SITE_PRODUCER_A_EMPTY)) {
      ok = false;
      break;
    }
    mbar_arrive_expect_tx(&bars.a_full[ab], L::A_BYTES);
    Pass::template load_a<HD>(p, it, smem + L::OFF_A + ab * L::A_BYTES, &bars.a_full[ab]);
    ++a_cnt;
    for (int32_t t = 0; t < it.ntiles; ++t) {
      const uint32_t st = b_cnt % kStages;
      if (!wait_bounded(&bars.b_empty[st], ((b_cnt / kStages) & 1u) ^ 1u, ctl, SITE_PRODUCER_B_EMPTY)) {
        ok = false;
        break;
      }
      mbar_arrive_expect_tx(&bars.b_full[st], L::B_BYTES);
      Pass::template load_b<HD>(p, it, t, smem + L::OFF_B + st * L::B_BYTES, &bars.b_full[st]);
      ++b_cnt;
    }
  }
  if (!ok) {
    // Let every load issued by this thread land before the CTA exits.
    for (uint32_t ab = 0; ab < 2; ++ab) {
      if (a_cnt > ab) {
        const uint32_t fills = (a_cnt - ab + 1) / 2;
        wait_drain(&bars.a_full[ab], (fills - 1) & 1u, ctl);
      }
    }
    for (uint32_t st = 0; st < kStages; ++st) {
      if (b_cnt > st) {
        const uint32_t fills = (b_cnt - st + kStages - 1) / kStages;
        wait_drain(&bars.b_full[st], (fills - 1) & 1u, ctl);
      }
    }
  }
}

template <class Pass, int HD>
__device__ void mma_role(const AttnParams& p, uint8_t* smem, const Bars& bars, const WaitCtl& ctl,
                         uint32_t tmem_base) {
  using L = SmemLayout<HD>;
  uint32_t a_cnt = 0, b_cnt = 0, acc_cnt = 0;
  bool ok = true, issued = false;
  const int32_t total = p.sched.total_items;
  const uint32_t idesc_full = umma_idesc_bf16(kTileRows, kStreamRows);
  const uint32_t idesc_half = umma_idesc_bf16(kTileRows, kStreamRows / 2);
  for (int32_t k = 0; ok; ++k) {
    const int32_t n = cta_item(k, blockIdx.x, gridDim.x);
    if (n >= total) break;
    const typename Pass::Item it = Pass::item(p, n);
    if (it.ntiles == 0) continue;
    const uint32_t ab = a_cnt & 1u;
    if (!wait_bounded(&bars.a_full[ab], (a_cnt >> 1) & 1u, ctl, SITE_MMA_A_FULL)) {
      ok = false;
      break;
    }
    tc_fence_after_sync();
    const uint32_t a_addr = smem_u32(smem + L::OFF_A + ab * L::A_BYTES);
    for (int32_t t = 0; t < it.ntiles; ++t) {
      const uint32_t st = b_cnt % kStages;
      const uint32_t acc = acc_cnt & 1u;
      if (!wait_bounded(&bars.b_full[st], (b_cnt / kStages) & 1u, ctl, SITE_MMA_B_FULL) ||
          !wait_bounded(&bars.acc_empty[acc], ((acc_cnt >> 1) & 1u) ^ 1u, ctl, SITE_MMA_ACC_EMPTY)) {
        ok = false;
        break;
      }
      tc_fence_after_sync();
      const uint32_t b_addr = smem_u32(smem + L::OFF_B + st * L::B_BYTES);
      const uint32_t d_tmem = tmem_base + acc * kStreamRows;
      const uint32_t idesc = Pass::half_tile(it, t) ? idesc_half : idesc_full;
#pragma unroll
      for (int kk = 0; kk < HD / 16; ++kk) {
        const int kh = kk / 4, kw = kk % 4;  // 64-element slab, 16-element step inside its 128-byte rows
        const uint64_t ad = umma_desc_sw128(a_addr + kh * L::A_HALF + kw * 32);
        const uint64_t bd = umma_desc_sw128(b_addr + kh * L::B_HALF + kw * 32);
        umma_bf16(d_tmem, ad, bd, idesc, kk > 0 ? 1u : 0u);
      }
      issued = true;
      umma_commit(&bars.b_empty[st]);
      umma_commit(&bars.acc_full[acc]);
      ++b_cnt;
      ++acc_cnt;
    }
    if (!ok) break;
    umma_commit(&bars.a_empty[ab]);
    ++a_cnt;
  }
  if (issued) {
    // Every MMA issued here must be finished before TMEM is released.
    umma_commit(bars.mma_done);
    wait_drain(bars.mma_done, 0, ctl);
  }
}

// ------------------------------------------------------------------ softmax: pass 1

// Every lane waits; the outcome is made warp-uniform so that the
// warp-collective TMEM loads that follow never run in a partial warp.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, const WaitCtl& ctl, int32_t site) {
  const bool ok = wait_bounded(bar, parity, ctl, site);
  return __all_sync(0xffffffffu, ok);
}

// Sum of exp2(x * c - off) over 32 columns, with columns >= lim masked out.
template <bool kMasked>
__device__ __forceinline__ float exp_sum32(const uint32_t (&r)[32], float c, float off, int lim) {
  float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
#pragma unroll
  for (int e = 0; e < 32; e += 4) {
    float y0 = fmaf(__uint_as_float(r[e + 0]), c, -off);
    float y1 = fmaf(__uint_as_float(r[e + 1]), c, -off);
    float y2 = fmaf(__uint_as_float(r[e + 2]), c, -off);
    float y3 = fmaf(__uint_as_float(r[e + 3]), c, -off);
    if (kMasked) {
      y0 = (e + 0 < lim) ? y0 : -INFINITY;
      y1 = (e + 1 < lim) ? y1 : -INFINITY;
      y2 = (e + 2 < lim) ? y2 : -INFINITY;
      y3 = (e + 3 < lim) ? y3 : -INFINITY;
    }
    s0 += ex2_approx(y0);
    s1 += ex2_approx(y1);
    s2 += ex2_approx(y2);
    s3 += ex2_approx(y3);
  }
  return (s0 + s1) + (s2 + s3);
}

template <bool kMasked>
__device__ __forceinline__ float max32(const uint32_t (&r)[32], float c, int lim) {
  float m = -INFINITY;
#pragma unroll
  for (int e = 0; e < 32; ++e) {
    const float y = __uint_as_float(r[e]) * c;
    if (!kMasked || e < lim) m = fmaxf(m, y);
  }
  return m;
}

// One 128-column half of a tile for one query row: returns sum exp2(y - off)
// (columns c with c > diag_lim masked when masked is set).
template <bool kMasked>
__device__ __forceinline__ float lse_tile_sum(uint32_t taddr, float c, float off, int row) {
  float s = 0.f;
#pragma unroll 1
  for (int ch = 0; ch < 4; ++ch) {
    uint32_t r[32];
    tmem_load32(taddr + ch * 32, r);
    tmem_load_wait(r);
    s += exp_sum32<kMasked>(r, c, off, row + 1 - ch * 32);
  }
  return s;
}

template <bool kMasked>
__device__ __forceinline__ float lse_tile_max(uint32_t taddr, float c, int row) {
  float m = -INFINITY;
#pragma unroll 1
  for (int ch = 0; ch < 4; ++ch) {
    uint32_t r[32];
    tmem_load32(taddr + ch * 32, r);
    tmem_load_wait(r);
    m = fmaxf(m, max32<kMasked>(r, c, row + 1 - ch * 32));
  }
  return m;
}

template <int HD>
__device__ void lse_softmax_role(const AttnParams& p, uint8_t* smem, const Bars& bars, const WaitCtl& ctl,
                                 uint32_t tmem_base) {
  using L = SmemLayout<HD>;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int sw = warp - 2;                 // softmax warp 0..7
  const int wg = sw >> 2;                  // column half
  const int quad = warp & 3;               // TMEM lane quadrant this warp may access
  const int row = quad * 32 + lane;        // query row within the tile
  const uint32_t lane_addr = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + wg * 128;
  float* comb = reinterpret_cast<float*>(smem + L::OFF_COMB);
  const float c = p.scale_log2;
  const float kBig = 18446744073709551616.0f;   // 2^64: larger tile sums force an exact rescale
  const float kRebase = 4294967296.0f;          // 2^32: keep the running sum moderate
  uint32_t acc_cnt = 0, item_cnt = 0;
  bool ok = true;
  const int32_t total = p.sched.total_items;
  for (int32_t k = 0; ok; ++k) {
    const int32_t n = cta_item(k, blockIdx.x, gridDim.x);
    if (n >= total) break;
    const LsePass::Item it = LsePass::item(p, n);
    float off = -INFINITY, sum = 0.f;      // running offset (log2 units) and sum of exp2(y - off)
    for (int32_t t = 0; t < it.ntiles; ++t) {
      const uint32_t acc = acc_cnt & 1u;
      if (!warp_wait(&bars.acc_full[acc], (acc_cnt >> 1) & 1u, ctl, SITE_SOFTMAX_ACC_FULL)) {
        ok = false;
        break;
      }
      tc_fence_after_sync();
      const bool last = (t == it.ntiles - 1);
      const bool half = LsePass::half_tile(it, t);
      const bool skip = half && wg == 1;                  // columns 128..255 not computed
      const bool masked = last && (half ? wg == 0 : wg == 1);
      if (!skip) {
        const uint32_t taddr = lane_addr + acc * kStreamRows;
        float ts = masked ? lse_tile_sum<true>(taddr, c, off, row) : lse_tile_sum<false>(taddr, c, off, row);
        // Warp-uniform: the rescale path issues warp-collective TMEM loads.
        if (__any_sync(0xffffffffu, !(ts < kBig))) {
          // The stale offset is too small (or unset): rescale to the exact tile max.
          const float tm = masked ? lse_tile_max<true>(taddr, c, row) : lse_tile_max<false>(taddr, c, row);
          const float noff = fmaxf(off, tm);
          if (noff > -INFINITY) {
            sum = sum * ex2_approx(off - noff);
            off = noff;
            ts = masked ? lse_tile_sum<true>(taddr, c, off, row) : lse_tile_sum<false>(taddr, c, off, row);
          } else {
            ts = 0.f;
          }
        }
        sum += ts;
        if (sum > kRebase) {
          const int e = static_cast<int>(floorf(__log2f(sum)));
          sum = sum * __int_as_float((127 - e) << 23);   // exact 2^-e
          off = off + static_cast<float>(e);
        }
      }
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.acc_empty[acc]);
      ++acc_cnt;
    }
    if (!ok) break;
    // Combine the two column halves of each row.
    if (wg == 1) {
      if (!warp_wait(bars.comb_empty, (item_cnt & 1u) ^ 1u, ctl, SITE_SOFTMAX_ACC_FULL)) break;
      comb[row] = off;
      comb[128 + row] = sum;
      __syncwarp();
      if (lane == 0) mbar_arrive(bars.comb_full);
    } else {
      if (!warp_wait(bars.comb_full, item_cnt & 1u, ctl, SITE_SOFTMAX_ACC_FULL)) break;
      const float off1 = comb[row], sum1 = comb[128 + row];
      __syncwarp();
      if (lane == 0) mbar_arrive(bars.comb_empty);
      const float m = fmaxf(off, off1);
      const float s = sum * ex2_approx(off - m) + (off1 > -INFINITY ? sum1 * ex2_approx(off1 - m) : 0.f);
      const int32_t i = it.i0 + row;
      if (i < it.L) p.out[static_cast<int64_t>(it.g) * p.total_tokens + it.s + i] = (m + log2f(s)) * kLn2;
    }
    ++item_cnt;
  }
}

// ------------------------------------------------------------------ softmax: pass 2

struct TileCursor {  // walks this CTA's pass-2 tiles (items without tiles are skipped)
  int32_t k;
  TargetPass::Item it;
  int32_t t;
  bool have;
  __device__ __forceinline__ void next_item(const AttnParams& p) {
    have = false;
    for (;;) {
      const int32_t n = cta_item(k++, blockIdx.x, gridDim.x);
      if (n >= p.sched.total_items) return;
      it = TargetPass::item(p, n);
      if (it.ntiles > 0) {
        t = 0;
        have = true;
        return;
      }
    }
  }
  __device__ __forceinline__ void start(const AttnParams& p) {
    k = 0;
    next_item(p);
  }
  __device__ __forceinline__ void advance(const AttnParams& p) {
    if (++t == it.ntiles) next_item(p);
  }
};

// lse (log2 units) of query column `col` of the cursor's tile; +inf past the sequence end.
__device__ __forceinline__ float tile_lse2(const AttnParams& p, const TileCursor& cur, int col) {
  const int32_t g = cur.t / cur.it.nq, qt = cur.t - g * cur.it.nq;
  const int32_t i = cur.it.i0 + qt * kStreamRows + col;
  if (i >= cur.it.L) return INFINITY;
  const int32_t qh = cur.it.h * p.group + g;
  return __ldg(p.lse_in + static_cast<int64_t>(qh) * p.total_tokens + cur.it.s + i) * kLog2e;
}

template <int HD>
__device__ void target_softmax_role(const AttnParams& p, uint8_t* smem, const Bars& bars, const WaitCtl& ctl,
                                    uint32_t tmem_base) {
  using L = SmemLayout<HD>;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int sw = warp - 2;
  const int wg = sw >> 2;
  const int quad = warp & 3;
  const int row = quad * 32 + lane;        // key row within the tile
  const uint32_t lane_addr = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + wg * 128;
  float* lse_w = reinterpret_cast<float*>(smem + L::OFF_LSE) + sw * 256;   // this warp's 2 x 128 slots
  float* comb = reinterpret_cast<float*>(smem + L::OFF_COMB);
  const float c = p.scale_log2;
  const int32_t total = p.sched.total_items;

  // Prefetch cursor: the lse values of the next tile are loaded one tile ahead.
  TileCursor ahead;
  ahead.start(p);
  float pre[4];
#pragma unroll
  for (int m = 0; m < 4; ++m) pre[m] = ahead.have ? tile_lse2(p, ahead, wg * 128 + lane + 32 * m) : 0.f;

  uint32_t acc_cnt = 0, item_cnt = 0;
  bool ok = true;
  for (int32_t k = 0; ok; ++k) {
    const int32_t n = cta_item(k, blockIdx.x, gridDim.x);
    if (n >= total) break;
    const TargetPass::Item it = TargetPass::item(p, n);
    float run = 0.f, comp = 0.f;           // Kahan-compensated running sum over tiles
    for (int32_t t = 0; t < it.ntiles; ++t) {
      // Stage this tile's lse values (loaded during the previous tile).
      float* ls = lse_w + (acc_cnt & 1u) * 128;
#pragma unroll
      for (int m = 0; m < 4; ++m) ls[lane + 32 * m] = pre[m];
      __syncwarp();
      ahead.advance(p);
#pragma unroll
      for (int m = 0; m < 4; ++m) pre[m] = ahead.have ? tile_lse2(p, ahead, wg * 128 + lane + 32 * m) : 0.f;

      const uint32_t acc = acc_cnt & 1u;
      if (!warp_wait(&bars.acc_full[acc], (acc_cnt >> 1) & 1u, ctl, SITE_SOFTMAX_ACC_FULL)) {
        ok = false;
        break;
      }
      tc_fence_after_sync();
      const int32_t qt = t % it.nq;
      const bool diag = (qt == 0) && (wg == 0);   // first query tile: column c valid iff c >= row
      const uint32_t taddr = lane_addr + acc * kStreamRows;
      float ts = 0.f;
#pragma unroll 1
      for (int ch = 0; ch < 4; ++ch) {
        uint32_t r[32];
        tmem_load32(taddr + ch * 32, r);
        tmem_load_wait(r);
        const float4* l4 = reinterpret_cast<const float4*>(ls + ch * 32);
        float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
#pragma unroll
        for (int e = 0; e < 32; e += 4) {
          const float4 lv = l4[e / 4];
          float y0 = fmaf(__uint_as_float(r[e + 0]), c, -lv.x);
          float y1 = fmaf(__uint_as_float(r[e + 1]), c, -lv.y);
          float y2 = fmaf(__uint_as_float(r[e + 2]), c, -lv.z);
          float y3 = fmaf(__uint_as_float(r[e + 3]), c, -lv.w);
          if (diag) {
            const int col = ch * 32 + e;
            y0 = (col + 0 >= row) ? y0 : -INFINITY;
            y1 = (col + 1 >= row) ? y1 : -INFINITY;
            y2 = (col + 2 >= row) ? y2 : -INFINITY;
            y3 = (col + 3 >= row) ? y3 : -INFINITY;
          }
          s0 += ex2_approx(y0);
          s1 += ex2_approx(y1);
          s2 += ex2_approx(y2);
          s3 += ex2_approx(y3);
        }
        ts += (s0 + s1) + (s2 + s3);
      }
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.acc_empty[acc]);
      ++acc_cnt;
      const float yk = ts - comp;
      const float tk = run + yk;
      comp = (tk - run) - yk;
      run = tk;
    }
    if (!ok) break;
    if (wg == 1) {
      if (!warp_wait(bars.comb_empty, (item_cnt & 1u) ^ 1u, ctl, SITE_SOFTMAX_ACC_FULL)) break;
      comb[row] = run;
      __syncwarp();
      if (lane == 0) mbar_arrive(bars.comb_full);
    } else {
      if (!warp_wait(bars.comb_full, item_cnt & 1u, ctl, SITE_SOFTMAX_ACC_FULL)) break;
      const float other = comb[row];
      __syncwarp();
      if (lane == 0) mbar_arrive(bars.comb_empty);
      const int32_t j = it.j0 + row;
      if (j < it.L) p.out[static_cast<int64_t>(it.h) * p.total_tokens + it.s + j] = run + other;
    }
    ++item_cnt;
  }
}

// ------------------------------------------------------------------ kernels

template <int HD>
__device__ __forceinline__ uint8_t* aligned_smem(uint8_t* raw) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(raw) + 1023) & ~static_cast<uintptr_t>(1023));
}

template <class Pass, int HD>
__device__ __forceinline__ void attn_kernel_body(const AttnParams& p, uint8_t* smem_raw) {
  using L = SmemLayout<HD>;
  uint8_t* smem = aligned_smem<HD>(smem_raw);
  const Bars bars = carve_bars(reinterpret_cast<uint64_t*>(smem + L::OFF_BAR));
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::OFF_MISC + 4);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars.a_full[i], 1);
      mbar_init(&bars.a_empty[i], 1);
      mbar_init(&bars.acc_full[i], 1);
      mbar_init(&bars.acc_empty[i], kSoftmaxWarps);
    }
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&bars.b_full[i], 1);
      mbar_init(&bars.b_empty[i], 1);
    }
    mbar_init(bars.comb_full, 4);
    mbar_init(bars.comb_empty, 4);
    mbar_init(bars.mma_done, 1);
    *abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_map(&p.tmap_q);
    tma_prefetch_map(&p.tmap_k);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
    tc_fence_before_sync();
  }
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem_base = *tmem_slot;
  const WaitCtl ctl{abort_flag, p.status, p.wait_ns};

  if (warp == 0) {
    if (lane == 0) producer_role<Pass, HD>(p, smem, bars, ctl);
  } else if (warp == 1) {
    if (lane == 0) mma_role<Pass, HD>(p, smem, bars, ctl, tmem_base);
  } else {
    if constexpr (std::is_same<Pass, LsePass>::value) {
      lse_softmax_role<HD>(p, smem, bars, ctl, tmem_base);
    } else {
      target_softmax_role<HD>(p, smem, bars, ctl, tmem_base);
    }
  }

  tc_fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after_sync();
    tmem_dealloc(tmem_base, 512);
  }
}

template <int HD>
__global__ void __launch_bounds__(kThreads, 1) row_lse_kernel(const __grid_constant__ AttnParams p) {
  extern __shared__ uint8_t smem_raw[];
  attn_kernel_body<LsePass, HD>(p, smem_raw);
}

template <int HD>
__global__ void __launch_bounds__(kThreads, 1) future_target_kernel(const __grid_constant__ AttnParams p) {
  extern __shared__ uint8_t smem_raw[];
  attn_kernel_body<TargetPass, HD>(p, smem_raw);
}

// ------------------------------------------------------------------ launchers

template <int HD>
static cudaError_t launch_attn(bool target_pass, const AttnParams& p, int grid, cudaStream_t stream) {
  using L = SmemLayout<HD>;
  auto kern = target_pass ? future_target_kernel<HD> : row_lse_kernel<HD>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::ALLOC);
  if (e != cudaSuccess) return e;
  kern<<<grid, kThreads, L::ALLOC, stream>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_row_lse(const AttnParams& p, int head_dim, int grid, cudaStream_t stream) {
  return head_dim == 64 ? launch_attn<64>(false, p, grid, stream) : launch_attn<128>(false, p, grid, stream);
}

cudaError_t launch_future_target(const AttnParams& p, int head_dim, int grid, cudaStream_t stream) {
  return head_dim == 64 ? launch_attn<64>(true, p, grid, stream) : launch_attn<128>(true, p, grid, stream);
}

// ------------------------------------------------------------------ bounded-wait self-test

__global__ void selftest_wait_kernel(int32_t* status, uint64_t limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);  // nothing ever arrives
    abort_flag = 0;
    fence_mbarrier_init();
  }
  __syncthreads();
  const WaitCtl ctl{&abort_flag, status, limit_ns};
  if (threadIdx.x == 0) wait_bounded(&bar, 0, ctl, SITE_SELFTEST);
  __syncthreads();
}

cudaError_t launch_selftest_wait(int32_t* status, uint64_t limit_ns, cudaStream_t stream) {
  selftest_wait_kernel<<<1, 32, 0, stream>>>(status, limit_ns);
  return cudaGetLastError();
}

}  // namespace kvpop
