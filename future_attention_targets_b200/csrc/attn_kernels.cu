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
// The normaliser of every query column rides along in the contraction: the
// K tile gets 16 extra K-columns (1, 1, 1, 0, ...) and each Q tile gets
// (-hi, -mid, -lo, 0, ...) with hi + mid + lo = lse_i / s split exactly into
// three bf16 parts, so the accumulator holds q.k - lse_i / s and the softmax
// warps only evaluate exp2(s log2e * acc).  TMEM lanes are keys and columns
// queries, so each thread owns one key and sums over all its queries and all
// G heads without any cross-thread reduction.
//
// Warp roles (320 threads, one CTA per SM):
//   warp 0      TMA producer: A tile once per item, B tiles into a 2-stage
//               ring (pass 2: the warp also writes the normaliser slab)
//   warp 1      TMEM allocator + single-thread tcgen05.mma issuer
//   warps 2..9  softmax: two groups of four warps split the 256 accumulator
//               columns (each warp reads its TMEM lane quadrant, warp % 4)
// Two TMEM accumulators of 256 fp32 columns (all 512 columns) let the MMA of
// tile t+1 run while the softmax warps read tile t.
#include <cuda_bf16.h>
#include <math.h>

#include <type_traits>

#include "kvpop_device.cuh"

namespace kvpop {

constexpr float kLn2 = 0.6931471805599453f;
constexpr int kStages = 2;
constexpr int kSoftmaxWarps = 8;
// Extra K=16 slab (no swizzle, K-major): 8-row groups of two 8x16-byte core
// matrices; element (r, e) sits at (r/8)*256 + (e/8)*128 + (r%8)*16 + (e%8)*2.
constexpr int kSlabLBO = 128;   // between the two core matrices along K
constexpr int kSlabSBO = 256;   // between 8-row groups
constexpr float kPastEnd = 1e30f;  // normaliser of query columns past the sequence: exp2 -> 0

template <int HD, bool kSlab>
struct SmemLayout {
  static constexpr int A_HALF = kTileRows * 128;                 // one 64-element column slab of A
  static constexpr int B_HALF = kStreamRows * 128;
  static constexpr int A_BYTES = A_HALF * (HD / 64);
  static constexpr int B_TILE = B_HALF * (HD / 64);              // TMA bytes per B stage
  static constexpr int A_SLAB = kSlab ? kTileRows * 32 : 0;      // ones column block for A
  static constexpr int B_SLAB = kSlab ? kStreamRows * 32 : 0;    // normaliser block per B stage
  static constexpr int B_STAGE = B_TILE + B_SLAB;
  static constexpr int OFF_A = 0;                                // 2 buffers
  static constexpr int OFF_B = OFF_A + 2 * A_BYTES;              // kStages stages
  static constexpr int OFF_ASLAB = OFF_B + kStages * B_STAGE;
  static constexpr int OFF_COMB = OFF_ASLAB + A_SLAB;            // float [2][128]
  static constexpr int OFF_BAR = OFF_COMB + 2 * 128 * 4;
  // a_full[2] a_empty[2] b_full[S] b_empty[S] acc_full[2] acc_empty[2] comb_full comb_empty mma_done
  static constexpr int N_BARS = 4 + 2 * kStages + 4 + 3;
  static constexpr int OFF_MISC = OFF_BAR + N_BARS * 8;
  static constexpr int BYTES = OFF_MISC + 16;
  static constexpr int ALLOC = BYTES + 1024;                     // room to align the base to 1 KiB
  static_assert(ALLOC <= 232448, "shared memory budget");
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

__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.expect_tx.relaxed.cta.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Descriptor of a K=16 slab in the no-swizzle K-major layout above.
__device__ __forceinline__ uint64_t umma_desc_slab(uint32_t saddr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>(kSlabLBO >> 4) << 16;
  d |= static_cast<uint64_t>(kSlabSBO >> 4) << 32;
  d |= static_cast<uint64_t>(1u) << 46;          // version 1, layout type 0 (no swizzle)
  return d;
}

__device__ __forceinline__ uint32_t slab_row_offset(int r) { return (r >> 3) * kSlabSBO + (r & 7) * 16; }

// ------------------------------------------------------------------ policies

// Pass 1: item = (sequence, query tile = level, query head).
struct LsePass {
  static constexpr bool kSlab = false;
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
      tma_load_2d(dst + kh * kTileRows * 128, &p.tmap_q, bar, it.g * HD + kh * 64, it.s + it.i0);
  }
  template <int HD>
  static __device__ __forceinline__ void load_b(const AttnParams& p, const Item& it, int32_t t, uint8_t* dst,
                                                uint64_t* bar) {
#pragma unroll
    for (int kh = 0; kh < HD / 64; ++kh)
      tma_load_2d(dst + kh * kStreamRows * 128, &p.tmap_k, bar, it.h * HD + kh * 64, it.s + t * kStreamRows);
  }
  // The last key tile holds the diagonal; when the query tile starts on a
  // 256-key boundary only its first 128 columns can be unmasked.
  static __device__ __forceinline__ bool half_tile(const Item& it, int32_t t) {
    return t == it.ntiles - 1 && it.i0 == t * kStreamRows;
  }
};

// Pass 2: item = (sequence, key tile, KV head); level = key tiles after this one.
struct TargetPass {
  static constexpr bool kSlab = true;
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
      tma_load_2d(dst + kh * kTileRows * 128, &p.tmap_k, bar, it.h * HD + kh * 64, it.s + it.j0);
  }
  template <int HD>
  static __device__ __forceinline__ void load_b(const AttnParams& p, const Item& it, int32_t g, int32_t qt,
                                                uint8_t* dst, uint64_t* bar) {
    const int32_t qh = it.h * p.group + g;
#pragma unroll
    for (int kh = 0; kh < HD / 64; ++kh)
      tma_load_2d(dst + kh * kStreamRows * 128, &p.tmap_q, bar, qh * HD + kh * 64,
                  it.s + it.i0 + qt * kStreamRows);
  }
  static __device__ __forceinline__ bool half_tile(const Item&, int32_t) { return false; }
};

// Walks this CTA's pass-2 tiles in issue order (items without tiles skipped).
struct TileCursor {
  int32_t k;
  TargetPass::Item it;
  int32_t g, qt;
  bool have;
  __device__ __forceinline__ void next_item(const AttnParams& p) {
    have = false;
    for (;;) {
      const int32_t n = cta_item(k++, blockIdx.x, gridDim.x);
      if (n >= p.sched.total_items) return;
      it = TargetPass::item(p, n);
      if (it.ntiles > 0) {
        g = 0;
        qt = 0;
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
    if (++qt == it.nq) {
      qt = 0;
      if (++g == p.group) next_item(p);
    }
  }
};

// ------------------------------------------------------------------ roles

// Every lane waits; the outcome is made warp-uniform so that warp-collective
// instructions that follow never run in a partial warp.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, const WaitCtl& ctl, int32_t site) {
  const bool ok = mbar_try_wait(bar, parity) || wait_bounded(bar, parity, ctl, site);
  return __all_sync(0xffffffffu, ok);
}

// Waits that must end even while the CTA is aborting (teardown drains).
__device__ __forceinline__ bool wait_drain(uint64_t* bar, uint32_t parity, const WaitCtl& ctl) {
  int dummy = 0;
  WaitCtl c2{&dummy, ctl.status, ctl.limit_ns};
  return wait_bounded(bar, parity, c2, SITE_TEARDOWN);
}

// Normaliser rows of one pass-2 B tile, this lane's 8 rows (lane + 32 m):
// lse_i / s, or kPastEnd past the sequence end.
__device__ __forceinline__ void load_norm_rows(const AttnParams& p, const TileCursor& cur, int lane,
                                               float (&v)[8]) {
  const int32_t qh = cur.it.h * p.group + cur.g;
  const float* src = p.lse_in + static_cast<int64_t>(qh) * p.total_tokens + cur.it.s;
#pragma unroll
  for (int m = 0; m < 8; ++m) {
    const int32_t i = cur.it.i0 + cur.qt * kStreamRows + lane + 32 * m;
    v[m] = (i < cur.it.L) ? __ldg(src + i) * p.inv_scale : kPastEnd;
  }
}

// Writes (-hi, -mid, -lo, 0) with hi + mid + lo = v (three bf16 parts) into
// the slab rows of this lane.
__device__ __forceinline__ void store_norm_rows(uint8_t* slab, int lane, const float (&v)[8]) {
#pragma unroll
  for (int m = 0; m < 8; ++m) {
    const float x = v[m];
    const __nv_bfloat16 hi = __float2bfloat16_rn(x);
    const float r1 = x - __bfloat162float(hi);
    const __nv_bfloat16 mid = __float2bfloat16_rn(r1);
    const __nv_bfloat16 lo = __float2bfloat16_rn(r1 - __bfloat162float(mid));
    const uint32_t w0 = static_cast<uint32_t>(__bfloat16_as_ushort(__hneg(hi))) |
                        (static_cast<uint32_t>(__bfloat16_as_ushort(__hneg(mid))) << 16);
    const uint32_t w1 = static_cast<uint32_t>(__bfloat16_as_ushort(__hneg(lo)));
    const uint32_t addr = smem_u32(slab + slab_row_offset(lane + 32 * m));
    asm volatile("st.shared.v2.b32 [%0], {%1, %2};" ::"r"(addr), "r"(w0), "r"(w1) : "memory");
  }
}

template <class Pass, int HD>
__device__ void producer_role(const AttnParams& p, uint8_t* smem, const Bars& bars, const WaitCtl& ctl) {
  using L = SmemLayout<HD, Pass::kSlab>;
  const int lane = threadIdx.x & 31;
  uint32_t a_cnt = 0, b_cnt = 0;
  bool ok = true;
  const int32_t total = p.sched.total_items;
  // Pass 2: normaliser values of the next tile, loaded one tile ahead.
  TileCursor nxt;
  float norm[8];
  if constexpr (Pass::kSlab) {
    nxt.start(p);
    if (nxt.have) load_norm_rows(p, nxt, lane, norm);
  }
  for (int32_t k = 0; ok; ++k) {
    const int32_t n = cta_item(k, blockIdx.x, gridDim.x);
    if (n >= total) break;
    const typename Pass::Item it = Pass::item(p, n);
    if (it.ntiles == 0) continue;
    const uint32_t ab = a_cnt & 1u;
    if (!warp_wait(&bars.a_empty[ab], ((a_cnt >> 1) & 1u) ^ 1u, ctl, SITE_PRODUCER_A_EMPTY)) {
      ok = false;
      break;
    }
    if (lane == 0) {
      mbar_arrive_expect_tx(&bars.a_full[ab], L::A_BYTES);
      Pass::template load_a<HD>(p, it, smem + L::OFF_A + ab * L::A_BYTES, &bars.a_full[ab]);
    }
    ++a_cnt;
    for (int32_t t = 0; t < it.ntiles; ++t) {
      const uint32_t st = b_cnt % kStages;
      if (!warp_wait(&bars.b_empty[st], ((b_cnt / kStages) & 1u) ^ 1u, ctl, SITE_PRODUCER_B_EMPTY)) {
        ok = false;
        break;
      }
      uint8_t* stage = smem + L::OFF_B + st * L::B_STAGE;
      if constexpr (Pass::kSlab) {
        // Tile bytes are expected before the loads are issued; the 32 lane
        // arrivals below (after their slab rows are written) complete the phase.
        const int32_t g = t / it.nq, qt = t - g * it.nq;
        if (lane == 0) {
          mbar_expect_tx(&bars.b_full[st], L::B_TILE);
          Pass::template load_b<HD>(p, it, g, qt, stage, &bars.b_full[st]);
        }
        float cur[8];
#pragma unroll
        for (int m = 0; m < 8; ++m) cur[m] = norm[m];
        nxt.advance(p);
        if (nxt.have) load_norm_rows(p, nxt, lane, norm);
        store_norm_rows(stage + L::B_TILE, lane, cur);
        fence_proxy_async_smem();
        mbar_arrive(&bars.b_full[st]);
      } else {
        if (lane == 0) {
          mbar_arrive_expect_tx(&bars.b_full[st], L::B_TILE);
          Pass::template load_b<HD>(p, it, t, stage, &bars.b_full[st]);
        }
      }
      ++b_cnt;
    }
  }
  if (!ok && lane == 0) {
    // Let every TMA load issued by this warp land before the CTA exits.
    for (uint32_t ab = 0; ab < 2; ++ab) {
      if (a_cnt > ab) wait_drain(&bars.a_full[ab], (((a_cnt - ab + 1) / 2) - 1) & 1u, ctl);
    }
    for (uint32_t st = 0; st < kStages; ++st) {
      if (b_cnt > st) wait_drain(&bars.b_full[st], (((b_cnt - st + kStages - 1) / kStages) - 1) & 1u, ctl);
    }
  }
}

template <class Pass, int HD>
__device__ void mma_role(const AttnParams& p, uint8_t* smem, const Bars& bars, const WaitCtl& ctl,
                         uint32_t tmem_base) {
  using L = SmemLayout<HD, Pass::kSlab>;
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
      const uint32_t b_addr = smem_u32(smem + L::OFF_B + st * L::B_STAGE);
      const uint32_t d_tmem = tmem_base + acc * kStreamRows;
      const uint32_t idesc = Pass::half_tile(it, t) ? idesc_half : idesc_full;
#pragma unroll
      for (int kk = 0; kk < HD / 16; ++kk) {
        const int kh = kk / 4, kw = kk % 4;  // 64-element slab, 16-element step inside its 128-byte rows
        const uint64_t ad = umma_desc_sw128(a_addr + kh * kTileRows * 128 + kw * 32);
        const uint64_t bd = umma_desc_sw128(b_addr + kh * kStreamRows * 128 + kw * 32);
        umma_bf16(d_tmem, ad, bd, idesc, kk > 0 ? 1u : 0u);
      }
      if constexpr (Pass::kSlab) {
        // acc += (1, 1, 1) . (-hi, -mid, -lo): subtract lse_i / s from every column.
        umma_bf16(d_tmem, umma_desc_slab(smem_u32(smem + L::OFF_ASLAB)), umma_desc_slab(b_addr + L::B_TILE),
                  idesc, 1u);
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

// ------------------------------------------------------------------ exp2 on two pipes

// Packed fp32 pairs (one 64-bit register pair) for the f32x2 FMA/ADD forms.
__device__ __forceinline__ uint64_t f2_pack(float a, float b) {
  uint64_t r;
  asm("mov.b64 %0, {%1,%2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ void f2_unpack(uint64_t v, float& a, float& b) {
  asm("mov.b64 {%0,%1}, %2;" : "=f"(a), "=f"(b) : "l"(v));
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.ftz.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.ftz.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t f2_add_rm(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rm.ftz.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

// 2^y for a pair, on the FMA pipe: Cody-Waite reduction y = n + f with
// n = floor(y) (adding 1.5 * 2^23 rounded toward -inf leaves n in the low
// mantissa bits), 2^f from a degree-4 minimax polynomial with p(0) = 1
// (coefficients from fit_exp2_poly.py, max relative error 3.0e-6 in fp32),
// and 2^n applied by adding n to the exponent field.  Inputs are clamped to
// >= -126 so the exponent arithmetic cannot wrap; results below 2^-126 are
// therefore at most 2^-125 instead of 0, far below any tolerance.
constexpr float kRoundMagic = 12582912.0f;  // 1.5 * 2^23
constexpr float kP1 = 0x1.62d6c6p-1f, kP2 = 0x1.ee2450p-3f, kP3 = 0x1.abf868p-5f, kP4 = 0x1.b7f730p-7f;

__device__ __forceinline__ uint64_t exp2_poly_pair(uint64_t y) {
  float y0, y1;
  f2_unpack(y, y0, y1);
  const uint64_t yc = f2_pack(fmaxf(y0, -126.f), fmaxf(y1, -126.f));
  const uint64_t t = f2_add_rm(yc, f2_pack(kRoundMagic, kRoundMagic));
  const uint64_t n = f2_add(t, f2_pack(-kRoundMagic, -kRoundMagic));
  const uint64_t f = f2_fma(n, f2_pack(-1.f, -1.f), yc);
  uint64_t q = f2_fma(f, f2_pack(kP4, kP4), f2_pack(kP3, kP3));
  q = f2_fma(q, f, f2_pack(kP2, kP2));
  q = f2_fma(q, f, f2_pack(kP1, kP1));
  q = f2_fma(q, f, f2_pack(1.f, 1.f));
  float t0, t1, q0, q1;
  f2_unpack(t, t0, t1);
  f2_unpack(q, q0, q1);
  const uint32_t b0 = __float_as_uint(q0) + __float_as_uint(t0) * (1u << 23);
  const uint32_t b1 = __float_as_uint(q1) + __float_as_uint(t1) * (1u << 23);
  return f2_pack(__uint_as_float(b0), __uint_as_float(b1));
}

// 2^(c x) for a pair with the scale folded into the range reduction:
// x is clamped so that c x >= -126, then t = rm(c x + 1.5 * 2^23) in one
// fused multiply-add, n = t - 1.5 * 2^23 = floor(c x), f = c x - n (exact).
__device__ __forceinline__ uint64_t exp2_poly_pair_scaled(uint64_t x, uint64_t c2, float xmin) {
  float x0, x1;
  f2_unpack(x, x0, x1);
  const uint64_t xc = f2_pack(fmaxf(x0, xmin), fmaxf(x1, xmin));
  uint64_t t;
  asm("fma.rm.ftz.f32x2 %0, %1, %2, %3;" : "=l"(t) : "l"(xc), "l"(c2), "l"(f2_pack(kRoundMagic, kRoundMagic)));
  const uint64_t n = f2_add(t, f2_pack(-kRoundMagic, -kRoundMagic));
  float n0, n1;
  f2_unpack(n, n0, n1);
  const uint64_t f = f2_fma(xc, c2, f2_pack(-n0, -n1));
  uint64_t q = f2_fma(f, f2_pack(kP4, kP4), f2_pack(kP3, kP3));
  q = f2_fma(q, f, f2_pack(kP2, kP2));
  q = f2_fma(q, f, f2_pack(kP1, kP1));
  q = f2_fma(q, f, f2_pack(1.f, 1.f));
  float t0, t1, q0, q1;
  f2_unpack(t, t0, t1);
  f2_unpack(q, q0, q1);
  const uint32_t b0 = __float_as_uint(q0) + __float_as_uint(t0) * (1u << 23);
  const uint32_t b1 = __float_as_uint(q1) + __float_as_uint(t1) * (1u << 23);
  return f2_pack(__uint_as_float(b0), __uint_as_float(b1));
}

__device__ __forceinline__ uint64_t exp2_mufu_pair(uint64_t y) {
  float y0, y1;
  f2_unpack(y, y0, y1);
  return f2_pack(ex2_approx(y0), ex2_approx(y1));
}

// Split between the exponent paths: pairs (of the 16 in a 32-column chunk)
// evaluated by the polynomial, spread evenly over the chunk (measured on
// B200 for each pass at the Qwen3-8B 16k shape).
#ifndef KVPOP_POLY16_LSE
#define KVPOP_POLY16_LSE 4
#endif
#ifndef KVPOP_POLY16_TARGET
#define KVPOP_POLY16_TARGET 4
#endif

template <int kPoly>
__device__ __forceinline__ constexpr bool poly_pair(int q) {
  return ((q * kPoly) & 15) < kPoly;
}

// acc += exp2(x * c + nb) over one 32-column chunk (nb: one negated offset
// for the whole chunk); kPoly of the 16 pairs go through the polynomial, the
// rest through MUFU.  kBiasFree: nb is zero (pass 2), the scale is folded
// into the polynomial's range reduction and x >= xmin keeps c x >= -126.
template <int kPoly, bool kBiasFree>
__device__ __forceinline__ void chunk_exp_sum(const uint32_t (&r)[32], uint64_t c2, uint64_t nb, float xmin,
                                              uint64_t (&acc)[4]) {
#pragma unroll
  for (int q = 0; q < 16; ++q) {
    const uint64_t x = f2_pack(__uint_as_float(r[2 * q]), __uint_as_float(r[2 * q + 1]));
    uint64_t e;
    if (poly_pair<kPoly>(q)) {
      e = kBiasFree ? exp2_poly_pair_scaled(x, c2, xmin) : exp2_poly_pair(f2_fma(x, c2, nb));
    } else {
      e = exp2_mufu_pair(f2_fma(x, c2, nb));
    }
    acc[q & 3] = f2_add(acc[q & 3], e);
  }
}

// Same with only columns lo <= e < hi of the chunk counted (MUFU only, so
// huge negative arguments give exact zeros).
__device__ __forceinline__ void chunk_exp_sum_masked(const uint32_t (&r)[32], uint64_t c2, uint64_t nb, int lo,
                                                     int hi, uint64_t (&acc)[4]) {
#pragma unroll
  for (int q = 0; q < 16; ++q) {
    const uint64_t x = f2_pack(__uint_as_float(r[2 * q]), __uint_as_float(r[2 * q + 1]));
    float y0, y1;
    f2_unpack(f2_fma(x, c2, nb), y0, y1);
    const int e0 = 2 * q, e1 = 2 * q + 1;
    y0 = (e0 >= lo && e0 < hi) ? y0 : -INFINITY;
    y1 = (e1 >= lo && e1 < hi) ? y1 : -INFINITY;
    acc[q & 3] = f2_add(acc[q & 3], f2_pack(ex2_approx(y0), ex2_approx(y1)));
  }
}

__device__ __forceinline__ float acc_total(uint64_t (&acc)[4]) {
  const uint64_t s = f2_add(f2_add(acc[0], acc[1]), f2_add(acc[2], acc[3]));
  float a, b;
  f2_unpack(s, a, b);
  return a + b;
}

// Sum of exp2(x * c - off) over the 128 columns of this thread's TMEM lane
// starting at taddr: four chunks of 32, the load of chunk c+1 in flight
// while chunk c is summed.  kMasked: column m counts iff lo <= m < hi.
template <bool kMasked, int kPoly, bool kBiasFree = false>
__device__ __forceinline__ float half_tile_exp_sum(uint32_t taddr, uint64_t c2, uint64_t nb, int lo, int hi,
                                                   float xmin = 0.f) {
  uint32_t ra[32], rb[32];
  uint64_t acc[4] = {0, 0, 0, 0};
  auto run = [&](const uint32_t (&r)[32], int ch) {
    if constexpr (kMasked)
      chunk_exp_sum_masked(r, c2, nb, lo - 32 * ch, hi - 32 * ch, acc);
    else
      chunk_exp_sum<kPoly, kBiasFree>(r, c2, nb, xmin, acc);
  };
  tmem_load<32>(taddr, ra);
  tmem_load_wait<32>(ra);
  tmem_load<32>(taddr + 32, rb);
  run(ra, 0);
  tmem_load_wait<32>(rb);
  tmem_load<32>(taddr + 64, ra);
  run(rb, 1);
  tmem_load_wait<32>(ra);
  tmem_load<32>(taddr + 96, rb);
  run(ra, 2);
  tmem_load_wait<32>(rb);
  run(rb, 3);
  return acc_total(acc);
}

// Max of x * c over columns lo <= m < hi of the 128 (pass-1 rescale path).
__device__ __forceinline__ float half_tile_max(uint32_t taddr, float c, int lo, int hi) {
  float m = -INFINITY;
#pragma unroll 1
  for (int ch = 0; ch < 4; ++ch) {
    uint32_t r[32];
    tmem_load<32>(taddr + 32 * ch, r);
    tmem_load_wait<32>(r);
#pragma unroll
    for (int e = 0; e < 32; ++e) {
      const int col = 32 * ch + e;
      if (col >= lo && col < hi) m = fmaxf(m, __uint_as_float(r[e]) * c);
    }
  }
  return m;
}

// ------------------------------------------------------------------ softmax: pass 1

template <int HD>
__device__ void lse_softmax_role(const AttnParams& p, uint8_t* smem, const Bars& bars, const WaitCtl& ctl,
                                 uint32_t tmem_base) {
  using L = SmemLayout<HD, false>;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int sw = warp - 2;                 // softmax warp 0..7
  const int wg = sw >> 2;                  // column half
  const int quad = warp & 3;               // TMEM lane quadrant this warp may access
  const int row = quad * 32 + lane;        // query row within the tile
  const uint32_t lane_addr = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + wg * 128;
  float* comb = reinterpret_cast<float*>(smem + L::OFF_COMB);
  const float c = p.scale_log2;
  const uint64_t c2 = f2_pack(c, c);
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
      const int hi = masked ? row + 1 : 128;              // on the diagonal: key column m <= query row
      if (!skip) {
        const uint32_t taddr = lane_addr + acc * kStreamRows;
        float ts = 0.f;
        bool rescale = (off == -INFINITY);                 // first tile of the row: no offset yet
        if (!rescale) {
          const uint64_t nb = f2_pack(-off, -off);
          ts = masked ? half_tile_exp_sum<true, 0>(taddr, c2, nb, 0, hi)
                      : half_tile_exp_sum<false, KVPOP_POLY16_LSE>(taddr, c2, nb, 0, 128);
          rescale = !(ts < kBig);
        }
        // Warp-uniform: the rescale path issues warp-collective TMEM loads.
        if (__any_sync(0xffffffffu, rescale)) {
          const float tm = half_tile_max(taddr, c, 0, hi);
          const float noff = fmaxf(off, tm);
          if (noff > -INFINITY) {
            sum = (off > -INFINITY) ? sum * ex2_approx(off - noff) : 0.f;
            off = noff;
          }
          const uint64_t nb = f2_pack(-off, -off);
          ts = masked ? half_tile_exp_sum<true, 0>(taddr, c2, nb, 0, hi)
                      : half_tile_exp_sum<false, KVPOP_POLY16_LSE>(taddr, c2, nb, 0, 128);
          if (!(off > -INFINITY)) ts = 0.f;
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

template <int HD>
__device__ void target_softmax_role(const AttnParams& p, uint8_t* smem, const Bars& bars, const WaitCtl& ctl,
                                    uint32_t tmem_base) {
  using L = SmemLayout<HD, true>;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int sw = warp - 2;
  const int wg = sw >> 2;
  const int quad = warp & 3;
  const int row = quad * 32 + lane;        // key row within the tile
  const uint32_t lane_addr = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + wg * 128;
  float* comb = reinterpret_cast<float*>(smem + L::OFF_COMB);
  const uint64_t c2 = f2_pack(p.scale_log2, p.scale_log2);
  const uint64_t zero2 = f2_pack(0.f, 0.f);
  const float xmin = -126.f / p.scale_log2;   // below it exp2(c x) < 2^-126: clamp for the polynomial
  const int32_t total = p.sched.total_items;
  uint32_t acc_cnt = 0, item_cnt = 0;
  bool ok = true;
  for (int32_t k = 0; ok; ++k) {
    const int32_t n = cta_item(k, blockIdx.x, gridDim.x);
    if (n >= total) break;
    const TargetPass::Item it = TargetPass::item(p, n);
    float run = 0.f, comp = 0.f;           // Kahan-compensated running sum over tiles
    const bool ragged_end = it.i0 + it.nq * kStreamRows > it.L;
    for (int32_t g = 0; g < (it.nq > 0 ? p.group : 0) && ok; ++g) {
      for (int32_t qt = 0; qt < it.nq; ++qt) {
        const uint32_t acc = acc_cnt & 1u;
        if (!warp_wait(&bars.acc_full[acc], (acc_cnt >> 1) & 1u, ctl, SITE_SOFTMAX_ACC_FULL)) {
          ok = false;
          break;
        }
        tc_fence_after_sync();
        const uint32_t taddr = lane_addr + acc * kStreamRows;
        // First query tile: column m of the first half is valid iff m >= row.
        // Last query tile: columns past the sequence hold -1e30 (exp2 -> 0 on MUFU).
        const bool diag = (qt == 0) && (wg == 0);
        const bool ragged = (qt == it.nq - 1) && ragged_end;
        const float ts = (diag || ragged)
                             ? half_tile_exp_sum<true, 0>(taddr, c2, zero2, diag ? row : 0, 128)
                             : half_tile_exp_sum<false, KVPOP_POLY16_TARGET, true>(taddr, c2, zero2, 0, 128,
                                                                                      xmin);
        tc_fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars.acc_empty[acc]);
        ++acc_cnt;
        const float yk = ts - comp;
        const float tk = run + yk;
        comp = (tk - run) - yk;
        run = tk;
      }
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

__device__ __forceinline__ uint8_t* aligned_smem(uint8_t* raw) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(raw) + 1023) & ~static_cast<uintptr_t>(1023));
}

template <class Pass, int HD>
__device__ __forceinline__ void attn_kernel_body(const AttnParams& p, uint8_t* smem_raw) {
  using L = SmemLayout<HD, Pass::kSlab>;
  uint8_t* smem = aligned_smem(smem_raw);
  const Bars bars = carve_bars(reinterpret_cast<uint64_t*>(smem + L::OFF_BAR));
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::OFF_MISC + 4);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if constexpr (Pass::kSlab) {
    // Zero the extra K-columns of A and of every B stage, then put the ones in A.
    for (int s = 0; s < kStages; ++s) {
      uint32_t* z = reinterpret_cast<uint32_t*>(smem + L::OFF_B + s * L::B_STAGE + L::B_TILE);
      for (int i = threadIdx.x; i < L::B_SLAB / 4; i += blockDim.x) z[i] = 0u;
    }
    uint32_t* za = reinterpret_cast<uint32_t*>(smem + L::OFF_ASLAB);
    for (int i = threadIdx.x; i < L::A_SLAB / 4; i += blockDim.x) za[i] = 0u;
    __syncthreads();
    if (threadIdx.x < kTileRows) {
      uint32_t* r = reinterpret_cast<uint32_t*>(smem + L::OFF_ASLAB + slab_row_offset(threadIdx.x));
      r[0] = 0x3F803F80u;   // e = 0, 1: bf16 1.0, 1.0
      r[1] = 0x00003F80u;   // e = 2: 1.0; e = 3: 0
    }
    fence_proxy_async_smem();
  }
  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars.a_full[i], 1);
      mbar_init(&bars.a_empty[i], 1);
      mbar_init(&bars.acc_full[i], 1);
      mbar_init(&bars.acc_empty[i], kSoftmaxWarps);
    }
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&bars.b_full[i], Pass::kSlab ? 32 : 1);
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
    producer_role<Pass, HD>(p, smem, bars, ctl);
  } else if (warp == 1) {
    if (lane == 0) mma_role<Pass, HD>(p, smem, bars, ctl, tmem_base);
  } else {
    if constexpr (std::is_same<Pass, LsePass>::value)
      lse_softmax_role<HD>(p, smem, bars, ctl, tmem_base);
    else
      target_softmax_role<HD>(p, smem, bars, ctl, tmem_base);
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

template <int HD, bool kTarget>
static cudaError_t launch_attn(const AttnParams& p, int grid, cudaStream_t stream) {
  using L = SmemLayout<HD, kTarget>;
  auto kern = kTarget ? future_target_kernel<HD> : row_lse_kernel<HD>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::ALLOC);
  if (e != cudaSuccess) return e;
  kern<<<grid, kThreads, L::ALLOC, stream>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_row_lse(const AttnParams& p, int head_dim, int grid, cudaStream_t stream) {
  return head_dim == 64 ? launch_attn<64, false>(p, grid, stream) : launch_attn<128, false>(p, grid, stream);
}

cudaError_t launch_future_target(const AttnParams& p, int head_dim, int grid, cudaStream_t stream) {
  return head_dim == 64 ? launch_attn<64, true>(p, grid, stream) : launch_attn<128, true>(p, grid, stream);
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
