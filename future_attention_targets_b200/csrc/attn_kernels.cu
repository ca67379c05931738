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
// Warp roles (576 threads, one CTA per SM):
//   warp 0      TMA producer: A tile once per item, B tiles into a 2-stage
//               ring (pass 2: the warp also writes the normaliser slab)
//   warp 1      TMEM allocator + single-thread tcgen05.mma issuer
//   warps 2..17 softmax: four groups of four warps split the 256 accumulator
//               columns, 64 each (each warp reads its TMEM lane quadrant,
//               warp % 4); four warps per scheduler hide the exponential
//               chains' latency
// Two TMEM accumulators of 256 fp32 columns (all 512 columns) let the MMA of
// tile t+1 run while the softmax warps read tile t.
//
// The single-launch variant runs both passes in one persistent cooperative
// grid: every CTA walks its pass-1 items, then its pass-2 items, with the
// pipeline state carried across.  Pass-1 writers publish each (query head,
// 128-row tile) of lse with a release increment on a flag in global memory;
// the pass-2 producer acquires the flags of a query tile before it reads that
// tile's lse (through L2), with the same 1 s bound as every other wait.  The
// last CTA to finish clears the flags for the next launch.
#include <cuda_bf16.h>
#include <math.h>

#include <algorithm>
#include <mutex>
#include <utility>
#include <vector>

#include <type_traits>

#include "kvpop_device.cuh"

namespace kvpop {

constexpr float kLn2 = 0.6931471805599453f;
constexpr int kStages = 2;          // B stages of a single-CTA pass
constexpr int kPairStages = 4;      // B stages per CTA of a CTA pair (half tiles: twice the depth in the same room)
constexpr int kColGroups = 4;                          // softmax warp groups per CTA
constexpr int kGroupCols = kStreamRows / kColGroups;   // accumulator columns per group
constexpr int kSoftmaxWarps = 4 * kColGroups;          // one warp per TMEM lane quadrant per group
static_assert(kThreads == 32 * (2 + kSoftmaxWarps), "producer warp + MMA warp + softmax warps");
static_assert(kGroupCols == 64, "group_exp_sum walks four 16-column chunks");
// Extra K=16 slabs (no swizzle, K-major) that subtract lse_i / s from every
// pass-2 score.  A (ones, 128 rows): 8-row groups of two 8x16-byte core
// matrices, element (r, e) at (r/8)*256 + (e/8)*128 + (r%8)*16 + (e%8)*2.
// B (normaliser rows, 256 rows): row r's 16 bytes (e = 0..7) at r * 16, so
// that one bulk copy of consecutive rows fills it; the e = 8..15 half is a
// zero block kSlabRowBytes further on.
constexpr int kSlabLBO = 128;   // A: between the two core matrices along K
constexpr int kSlabSBO = 256;   // A: between 8-row groups

// Shared memory of one CTA.  kCta = 2 (a CTA pair): each CTA holds 128 rows
// of the 256-row B tile, and the B slab's upper (zero) half sits
// kBRows * 16 bytes after its rows.
template <int HD, bool kSlab, int kCta = 1>
struct SmemLayout {
  static constexpr int kBRows = kStreamRows / kCta;              // B rows held by this CTA
  static constexpr int kNStages = kCta == 1 ? kStages : kPairStages;
  static constexpr int kSlabRowBytes = kBRows * 16;              // B slab: rows of one stage; also its LBO
  static constexpr int A_HALF = kTileRows * 128;                 // one 64-element column slab of A
  static constexpr int B_HALF = kBRows * 128;
  static constexpr int A_BYTES = A_HALF * (HD / 64);
  static constexpr int B_TILE = B_HALF * (HD / 64);              // TMA bytes per B stage
  static constexpr int A_SLAB = kSlab ? kTileRows * 32 : 0;      // ones column block for A
  static constexpr int B_SLAB = kSlab ? kBRows * 32 : 0;         // normaliser block per B stage
  static constexpr int B_STAGE = B_TILE + B_SLAB;
  static constexpr int OFF_A = 0;                                // 2 buffers
  static constexpr int OFF_B = OFF_A + 2 * A_BYTES;              // kNStages stages
  static constexpr int OFF_ASLAB = OFF_B + kNStages * B_STAGE;
  static constexpr int OFF_COMB = OFF_ASLAB + A_SLAB;            // float [kColGroups - 1][2][128]
  static constexpr int OFF_BAR = OFF_COMB + (kColGroups - 1) * 2 * 128 * 4;
  // a_full[2] a_empty[2] b_full[S] b_empty[S] acc_full[2] acc_empty[2] comb_full comb_empty mma_done
  static constexpr int N_BARS = 4 + 2 * kNStages + 4 + 3;
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

template <int kNStages = kStages>
__device__ __forceinline__ Bars carve_bars(uint64_t* b) {
  Bars r;
  r.a_full = b;
  r.a_empty = b + 2;
  r.b_full = b + 4;
  r.b_empty = b + 4 + kNStages;
  r.acc_full = b + 4 + 2 * kNStages;
  r.acc_empty = r.acc_full + 2;
  r.comb_full = r.acc_empty + 2;
  r.comb_empty = r.comb_full + 1;
  r.mma_done = r.comb_empty + 1;
  return r;
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Orders this thread's generic-proxy view of global memory with its later
// (or, on the writing side, earlier) async-proxy bulk copies.
__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
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

// Descriptor of the B normaliser slab (LBO = the stage's row bytes, SBO one 8-row group).
__device__ __forceinline__ uint64_t umma_desc_slab_rows(uint32_t saddr, uint32_t row_bytes) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>(row_bytes >> 4) << 16;
  d |= static_cast<uint64_t>(128 >> 4) << 32;
  d |= static_cast<uint64_t>(1u) << 46;
  return d;
}

__device__ __forceinline__ uint32_t slab_row_offset(int r) { return (r >> 3) * kSlabSBO + (r & 7) * 16; }

// Normaliser row of one query row: (-hi, -mid, -lo, 0, 0, 0, 0, 0) in bf16
// with hi + mid + lo = lse * inv_scale (each part the bf16 rounding of what
// the parts before it leave), so that (1, 1, 1) . row = -lse / s to within
// fp32 rounding of the three-term sum.
__device__ __forceinline__ uint4 norm_row(float lse, float inv_scale) {
  const float x = lse * inv_scale;
  const __nv_bfloat16 hi = __float2bfloat16_rn(x);
  const float r1 = x - __bfloat162float(hi);
  const __nv_bfloat16 mid = __float2bfloat16_rn(r1);
  const __nv_bfloat16 lo = __float2bfloat16_rn(r1 - __bfloat162float(mid));
  uint4 v;
  v.x = static_cast<uint32_t>(__bfloat16_as_ushort(__hneg(hi))) |
        (static_cast<uint32_t>(__bfloat16_as_ushort(__hneg(mid))) << 16);
  v.y = static_cast<uint32_t>(__bfloat16_as_ushort(__hneg(lo)));
  v.z = 0u;
  v.w = 0u;
  return v;
}

// ------------------------------------------------------------------ policies

// What a pass needs besides the common parameters: its schedule, tensor maps
// (A tiles are 128 rows, B tiles 256, so each pass has its own boxes), its
// output and, in the single-launch variant, the lse readiness flags.
struct Phase {
  const LevelSchedule* sched;
  const CUtensorMap* tmap_q;
  const CUtensorMap* tmap_k;
  float* out;                  // pass 1: lse [H_q, T]; pass 2: target [H_kv, T]
  int32_t* flags;              // single launch: [H_q, n_flag_tiles] counters (else unused)
  const int32_t* tile_base;    // single launch: first flag tile of each scheduled sequence
  int32_t n_flag_tiles;
  int32_t* lse_done;           // single launch: softmax warps that have finished pass 1
};

// Pass-1 warps that write one item's lse rows; each adds 1 to the tile's flag.
constexpr int32_t kLseFlagWriters = 4;

// Rank of this CTA in its pair (0 for a single CTA): rank 1 holds rows
// 128 .. 255 of every 256-row A block and of every B tile.
template <int kCta>
__device__ __forceinline__ int cta_rank() {
  if constexpr (kCta == 1) return 0;
  else return static_cast<int>(blockIdx.x & 1u);
}

// This CTA's rows of the 256-row B tile starting at row y0 (columns x0 ..
// x0 + HD of the map): all of them for one CTA, rows 128 * rank .. + 127 of
// the tile for a CTA of a pair.
template <int HD, int kCta>
__device__ __forceinline__ void load_b_rows(const CUtensorMap* map, int32_t x0, int32_t y0, uint8_t* dst,
                                            uint64_t* bar) {
  constexpr int kBRows = kStreamRows / kCta;
#pragma unroll
  for (int kh = 0; kh < HD / 64; ++kh) {
    if constexpr (kCta == 1) {
      tma_load_2d(dst + kh * kBRows * 128, map, bar, x0 + kh * 64, y0);
    } else {
      tma_load_2d_pair(dst + kh * kBRows * 128, map, bar, x0 + kh * 64, y0 + kBRows * cta_rank<kCta>());
    }
  }
}

// Pass 1: item = (sequence, query block = level, query head); a query block
// is 128 rows for a single CTA and 256 rows (128 per CTA) for a pair.
template <int kCta>
struct LsePassT {
  static constexpr bool kSlab = false;
  struct Item {
    int32_t s, L, g, h, i0, ntiles, seq;
  };
  static __device__ __forceinline__ Item item(const AttnParams& p, const LevelSchedule& sched, int32_t n) {
    const WorkItem w = decode_item(sched, n);
    Item it;
    it.s = w.seq_start;
    it.L = w.seq_len;
    it.g = w.head;
    it.h = w.head / p.group;
    it.i0 = w.level * kTileRows * kCta;
    it.ntiles = it.i0 / kStreamRows + 1;  // key tiles [0,256), [256,512), ... up to the diagonal
    it.seq = w.seq;
    return it;
  }
  template <int HD>
  static __device__ __forceinline__ void load_a(const Phase& ph, const Item& it, uint8_t* dst, uint64_t* bar) {
    const int32_t y = it.s + it.i0 + kTileRows * cta_rank<kCta>();
#pragma unroll
    for (int kh = 0; kh < HD / 64; ++kh) {
      if constexpr (kCta == 1) tma_load_2d(dst + kh * kTileRows * 128, ph.tmap_q, bar, it.g * HD + kh * 64, y);
      else tma_load_2d_pair(dst + kh * kTileRows * 128, ph.tmap_q, bar, it.g * HD + kh * 64, y);
    }
  }
  template <int HD>
  static __device__ __forceinline__ void load_b(const Phase& ph, const Item& it, int32_t t, uint8_t* dst,
                                                uint64_t* bar) {
    load_b_rows<HD, kCta>(ph.tmap_k, it.h * HD, it.s + t * kStreamRows, dst, bar);
  }
  // Single CTA: the last key tile holds the diagonal; when the query tile
  // starts on a 256-key boundary only its first 128 columns can be unmasked.
  // A pair's 256-row query blocks always start on that boundary and use the
  // whole tile (the first CTA's rows end at column 127 of it).
  static __device__ __forceinline__ bool half_tile(const Item& it, int32_t t) {
    if constexpr (kCta == 2) return false;
    else return t == it.ntiles - 1 && it.i0 == t * kStreamRows;
  }
  // Column of the last key tile at which row 0 of this CTA meets the diagonal.
  static __device__ __forceinline__ int diag_col(const Item& it, int32_t t) {
    if constexpr (kCta == 2) return kTileRows * cta_rank<kCta>();
    else return half_tile(it, t) ? 0 : kStreamRows / 2;
  }
};
using LsePass = LsePassT<1>;

// Pass 2: item = (sequence, key block, KV head) with all G query heads of
// the group, or, when p.g_split = G, (sequence, key block, KV head, one
// query head) so that few KV heads still give enough items; level = key
// blocks after this one.  A key block is 128 keys for a single CTA and 256
// (128 per CTA) for a pair.
template <int kCta>
struct TargetPassT {
  static constexpr bool kSlab = true;
  struct Item {
    int32_t s, L, h, g0, ng, j0, i0, nq, ntiles, seq;
  };
  static __device__ __forceinline__ Item item(const AttnParams& p, const LevelSchedule& sched, int32_t n) {
    const WorkItem w = decode_item(sched, n);
    Item it;
    it.s = w.seq_start;
    it.L = w.seq_len;
    it.h = w.head / p.g_split;
    it.ng = p.group / p.g_split;                 // query heads of this item
    it.g0 = (w.head % p.g_split) * it.ng;        // the first of them, within the group
    constexpr int32_t kRows = kTileRows * kCta;
    const int32_t nkt = (w.seq_len + kRows - 1) / kRows;
    it.j0 = (nkt - 1 - w.level) * kRows;
    it.i0 = it.j0 + p.window;
    it.nq = it.i0 < it.L ? (it.L - it.i0 + kStreamRows - 1) / kStreamRows : 0;
    it.ntiles = it.nq * it.ng;
    it.seq = w.seq;
    return it;
  }
  template <int HD>
  static __device__ __forceinline__ void load_a(const Phase& ph, const Item& it, uint8_t* dst, uint64_t* bar) {
    const int32_t y = it.s + it.j0 + kTileRows * cta_rank<kCta>();
#pragma unroll
    for (int kh = 0; kh < HD / 64; ++kh) {
      if constexpr (kCta == 1) tma_load_2d(dst + kh * kTileRows * 128, ph.tmap_k, bar, it.h * HD + kh * 64, y);
      else tma_load_2d_pair(dst + kh * kTileRows * 128, ph.tmap_k, bar, it.h * HD + kh * 64, y);
    }
  }
  template <int HD>
  static __device__ __forceinline__ void load_b(const Phase& ph, const Item& it, int32_t qh, int32_t qt,
                                                uint8_t* dst, uint64_t* bar) {
    load_b_rows<HD, kCta>(ph.tmap_q, qh * HD, it.s + it.i0 + qt * kStreamRows, dst, bar);
  }
  static __device__ __forceinline__ bool half_tile(const Item&, int32_t) { return false; }
};
using TargetPass = TargetPassT<1>;


// Pipeline counters of each role, carried from one phase to the next.
struct ProducerState {
  uint32_t a_cnt = 0, b_cnt = 0;
  bool ok = true;
};
struct MmaState {
  uint32_t a_cnt = 0, b_cnt = 0, acc_cnt = 0;
  bool ok = true, issued = false;
};
struct SoftmaxState {
  uint32_t acc_cnt = 0, item_cnt = 0;
  bool ok = true;
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

// Single launch: waits until every 128-row lse tile under query rows
// [a, a + 256) of query head qh (a = i0 + qt * 256) has been published.
// Lanes 0..2 poll the (at most three) tile flags and lane 31 the count of
// softmax warps that finished pass 1, all in one round trip; once every CTA's
// pass 1 is done (*all_lse) no flag is read again.  Bounded like every other
// wait; warp-uniform result.  The warp barrier on success passes every
// lane's acquire on to the whole warp.
template <bool kFused>
__device__ __forceinline__ bool norm_ready(const AttnParams& p, const Phase& ph, const TargetPass::Item& it,
                                           int32_t qh, int32_t qt, int lane, const WaitCtl& ctl, bool& all_lse) {
  if constexpr (!kFused) {
    return true;
  } else {
    if (all_lse) return true;
    const int32_t a = it.i0 + qt * kStreamRows;
    const int32_t b = min(a + kStreamRows, it.L);
    const int32_t t0 = a / kTileRows, nt = (b - 1) / kTileRows - t0 + 1;
    const int32_t* f = ph.flags + static_cast<int64_t>(qh) * ph.n_flag_tiles + ph.tile_base[it.seq] + t0;
    const int32_t all_warps = kSoftmaxWarps * static_cast<int32_t>(gridDim.x);
    uint64_t t_start = 0;
    for (uint32_t k = 0;; ++k) {
      bool mine = true;
      if (lane < nt) mine = flag_acquire_load(f + lane) >= kLseFlagWriters;
      const bool done_all = (lane == 31) && flag_acquire_load(ph.lse_done) >= all_warps;
      if (__any_sync(0xffffffffu, done_all)) {
        all_lse = true;
        __syncwarp();
        return true;
      }
      if (__all_sync(0xffffffffu, mine)) {
        __syncwarp();
        return true;
      }
      int give_up = 0;
      if (lane == 0 && (k & 15u) == 0u) {
        const uint64_t now = global_timer_ns();
        if (k == 0) t_start = now;
        if (*ctl.abort_flag) {
          give_up = 1;
        } else if (now - t_start > ctl.limit_ns) {
          raise_abort(ctl);
          if (ctl.status != nullptr) atomicCAS(ctl.status, 0, 4 | (SITE_LSE_FLAG << 8));
          give_up = 1;
        }
      }
      if (__shfl_sync(0xffffffffu, give_up, 0)) return false;
      __nanosleep(64);
    }
  }
}

// One pass of the TMA producer warp.  Pass 2 also copies, per B stage, the
// normaliser rows of its query tile (p.nrm_rows, 16 bytes per row; columns
// past the sequence end are masked by the softmax): a single CTA with one
// bulk copy of its 256 rows that stops at row T, each CTA of a pair with one
// tiled load of its 128 rows through p.tmap_rows (rows past the query head's
// last token read as zero).  kFused: the single launch, whose normaliser rows
// are written by pass 1 during the launch; the query tile is requested
// first, the rows only once their lse flags are set.
//
// CTA pairs: both CTAs load their own halves of every A and B tile into
// their own shared memory; the completion bytes of both count on the first
// CTA's barriers, which only the first CTA's producer arms (expect_tx) and
// only its MMA issuer waits on.  Each CTA reuses a buffer once its own empty
// barrier (signalled to both CTAs by the first CTA's MMA commits) says so.
template <class Pass, int HD, bool kFused, int kCta = 1>
__device__ void producer_phase(const AttnParams& p, const Phase& ph, uint8_t* smem, const Bars& bars,
                               const WaitCtl& ctl, ProducerState& st) {
  using L = SmemLayout<HD, Pass::kSlab || kFused, kCta>;
  const int lane = threadIdx.x & 31;
  const bool arms = cta_rank<kCta>() == 0;   // this CTA's producer sets the expected bytes
  const LevelSchedule& sched = *ph.sched;
  const int32_t total = sched.total_items;
  bool all_lse = false;
  for (int32_t k = 0; st.ok; ++k) {
    const int32_t n = cta_item(k, blockIdx.x / kCta, gridDim.x / kCta);
    if (n >= total) break;
    const typename Pass::Item it = Pass::item(p, sched, n);
    if (it.ntiles == 0) continue;
    // Debug build: the item lies inside the tensors (the tiled loads below
    // clip at the tensor edges in hardware, so these checks only record).
    [[maybe_unused]] constexpr int32_t kDbg = Pass::kSlab ? DBG_TARGET : DBG_ROW_LSE;
    if (lane == 0) {
      KVPOP_CHECK(it.s >= 0 && it.L > 0 && it.s + it.L <= p.total_tokens, p.dbg, kDbg, 1);
      if constexpr (Pass::kSlab)
        KVPOP_CHECK(it.h >= 0 && it.h < p.n_kv_heads && it.g0 + it.ng <= p.group && it.j0 >= 0 && it.j0 < it.L, p.dbg,
                 kDbg, 2);
      else
        KVPOP_CHECK(it.g >= 0 && it.g < p.n_q_heads && it.i0 >= 0 && it.i0 < it.L, p.dbg, kDbg, 2);
    }
    const uint32_t ab = st.a_cnt & 1u;
    if (!warp_wait(&bars.a_empty[ab], ((st.a_cnt >> 1) & 1u) ^ 1u, ctl, SITE_PRODUCER_A_EMPTY)) {
      st.ok = false;
      break;
    }
    if (lane == 0) {
      if (arms) mbar_arrive_expect_tx(&bars.a_full[ab], kCta * L::A_BYTES);
      Pass::template load_a<HD>(ph, it, smem + L::OFF_A + ab * L::A_BYTES, &bars.a_full[ab]);
    }
    ++st.a_cnt;
    for (int32_t t = 0; t < it.ntiles; ++t) {
      const uint32_t sg = st.b_cnt % L::kNStages;
      if (!warp_wait(&bars.b_empty[sg], ((st.b_cnt / L::kNStages) & 1u) ^ 1u, ctl, SITE_PRODUCER_B_EMPTY)) {
        st.ok = false;
        break;
      }
      uint8_t* stage = smem + L::OFF_B + sg * L::B_STAGE;
      if constexpr (Pass::kSlab) {
        const int32_t g = t / it.nq, qt = t - g * it.nq;
        const int32_t qh = it.h * p.group + it.g0 + g;
        const int32_t row0 = it.s + it.i0 + qt * kStreamRows;   // < T: qt < nq
        if (lane == 0) KVPOP_CHECK(qh < p.n_q_heads && row0 >= it.s && row0 < it.s + it.L, p.dbg, kDbg, 3);
        if constexpr (kCta == 2) {
          if (lane == 0) {
            if (arms) mbar_arrive_expect_tx(&bars.b_full[sg], 2 * (L::B_TILE + L::kSlabRowBytes));
            Pass::template load_b<HD>(ph, it, qh, qt, stage, &bars.b_full[sg]);
            tma_load_3d_pair(stage + L::B_TILE, &p.tmap_rows, &bars.b_full[sg], 0,
                             row0 + L::kBRows * cta_rank<kCta>(), qh);
          }
          ++st.b_cnt;
        } else {
          const uint32_t rows_bytes = static_cast<uint32_t>(min(kStreamRows, p.total_tokens - row0)) * 16u;
          if (lane == 0) {
            mbar_arrive_expect_tx(&bars.b_full[sg], L::B_TILE + rows_bytes);
            Pass::template load_b<HD>(ph, it, qh, qt, stage, &bars.b_full[sg]);
          }
          // After a failed wait the rows are still copied (in bounds, unused)
          // so that the stage completes and the drain below ends.
          const bool ready = norm_ready<kFused>(p, ph, it, qh, qt, lane, ctl, all_lse);
          if (lane == 0) {
            if constexpr (kFused) fence_proxy_async_global();
            // The rows read lie inside the [H_q, T] normaliser rows (a failed
            // check skips the copy; the stage then never completes and the
            // launch ends through its bounded waits).
            if (KVPOP_IN(qh < p.n_q_heads && row0 >= 0 && row0 * 16 + rows_bytes <= p.total_tokens * 16u, p.dbg,
                         kDbg, 4))
              bulk_load_1d(stage + L::B_TILE,
                           static_cast<const uint8_t*>(p.nrm_rows) + (static_cast<int64_t>(qh) * p.total_tokens + row0) * 16,
                           rows_bytes, &bars.b_full[sg]);
          }
          ++st.b_cnt;
          if (!ready) {
            st.ok = false;
            break;
          }
        }
      } else {
        if (lane == 0) {
          KVPOP_CHECK(t * kStreamRows < it.L, p.dbg, kDbg, 3);
          if (arms) mbar_arrive_expect_tx(&bars.b_full[sg], kCta * L::B_TILE);
          Pass::template load_b<HD>(ph, it, t, stage, &bars.b_full[sg]);
        }
        ++st.b_cnt;
      }
    }
  }
}

// After an abort: let every TMA load issued by the producer land before the
// CTA exits.  A pair's loads complete on the first CTA's barriers, which only
// that CTA can wait on; the second CTA's loads are covered by the grace
// period in the pair teardown.
template <int kNStages = kStages>
__device__ void producer_drain(const Bars& bars, const WaitCtl& ctl, const ProducerState& st, bool waits = true) {
  if (st.ok || !waits || (threadIdx.x & 31) != 0) return;
  for (uint32_t ab = 0; ab < 2; ++ab) {
    if (st.a_cnt > ab) wait_drain(&bars.a_full[ab], (((st.a_cnt - ab + 1) / 2) - 1) & 1u, ctl);
  }
  for (uint32_t sg = 0; sg < kNStages; ++sg) {
    if (st.b_cnt > sg)
      wait_drain(&bars.b_full[sg], (((st.b_cnt - sg + kNStages - 1) / kNStages) - 1) & 1u, ctl);
  }
}

// One pass of the single-thread MMA issuer.  CTA pairs: only the first CTA
// issues (M = 256 across both CTAs, each CTA's half of B from its own shared
// memory), and its commits arrive on the barriers of both CTAs.
template <class Pass, int HD, bool kFused, int kCta = 1>
__device__ void mma_phase(const AttnParams& p, const Phase& ph, uint8_t* smem, const Bars& bars, const WaitCtl& ctl,
                          uint32_t tmem_base, MmaState& st) {
  using L = SmemLayout<HD, Pass::kSlab || kFused, kCta>;
  const LevelSchedule& sched = *ph.sched;
  const int32_t total = sched.total_items;
  const uint32_t idesc_full = umma_idesc_bf16(kTileRows * kCta, kStreamRows);
  const uint32_t idesc_half = umma_idesc_bf16(kTileRows * kCta, kStreamRows / 2);
  auto commit = [](uint64_t* bar) {
    if constexpr (kCta == 1) umma_commit(bar);
    else umma_commit_pair(bar);
  };
  for (int32_t k = 0; st.ok; ++k) {
    const int32_t n = cta_item(k, blockIdx.x / kCta, gridDim.x / kCta);
    if (n >= total) break;
    const typename Pass::Item it = Pass::item(p, sched, n);
    if (it.ntiles == 0) continue;
    const uint32_t ab = st.a_cnt & 1u;
    if (!wait_bounded(&bars.a_full[ab], (st.a_cnt >> 1) & 1u, ctl, SITE_MMA_A_FULL)) {
      st.ok = false;
      break;
    }
    tc_fence_after_sync();
    const uint32_t a_addr = smem_u32(smem + L::OFF_A + ab * L::A_BYTES);
    for (int32_t t = 0; t < it.ntiles; ++t) {
      const uint32_t sg = st.b_cnt % L::kNStages;
      const uint32_t acc = st.acc_cnt & 1u;
      if (!wait_bounded(&bars.b_full[sg], (st.b_cnt / L::kNStages) & 1u, ctl, SITE_MMA_B_FULL) ||
          !wait_bounded(&bars.acc_empty[acc], ((st.acc_cnt >> 1) & 1u) ^ 1u, ctl, SITE_MMA_ACC_EMPTY)) {
        st.ok = false;
        break;
      }
      tc_fence_after_sync();
      const uint32_t b_addr = smem_u32(smem + L::OFF_B + sg * L::B_STAGE);
      const uint32_t d_tmem = tmem_base + acc * kStreamRows;
      const uint32_t idesc = Pass::half_tile(it, t) ? idesc_half : idesc_full;
#pragma unroll
      for (int kk = 0; kk < HD / 16; ++kk) {
        const int kh = kk / 4, kw = kk % 4;  // 64-element slab, 16-element step inside its 128-byte rows
        const uint64_t ad = umma_desc_sw128(a_addr + kh * kTileRows * 128 + kw * 32);
        const uint64_t bd = umma_desc_sw128(b_addr + kh * L::kBRows * 128 + kw * 32);
        if constexpr (kCta == 1) umma_bf16(d_tmem, ad, bd, idesc, kk > 0 ? 1u : 0u);
        else umma_bf16_pair(d_tmem, ad, bd, idesc, kk > 0 ? 1u : 0u);
      }
      if constexpr (Pass::kSlab) {
        // acc += (1, 1, 1) . (-hi, -mid, -lo): subtract lse_i / s from every column.
        const uint64_t ad = umma_desc_slab(smem_u32(smem + L::OFF_ASLAB));
        const uint64_t bd = umma_desc_slab_rows(b_addr + L::B_TILE, L::kSlabRowBytes);
        if constexpr (kCta == 1) umma_bf16(d_tmem, ad, bd, idesc, 1u);
        else umma_bf16_pair(d_tmem, ad, bd, idesc, 1u);
      }
      st.issued = true;
      commit(&bars.b_empty[sg]);
      commit(&bars.acc_full[acc]);
      ++st.b_cnt;
      ++st.acc_cnt;
    }
    if (!st.ok) break;
    commit(&bars.a_empty[ab]);
    ++st.a_cnt;
  }
}

// Every MMA issued must be finished before TMEM is released (a pair's commit
// also arrives on the second CTA's barrier, which nothing waits on).
template <int kCta = 1>
__device__ void mma_finish(const Bars& bars, const WaitCtl& ctl, const MmaState& st) {
  if (st.issued) {
    if constexpr (kCta == 1) umma_commit(bars.mma_done);
    else umma_commit_pair(bars.mma_done);
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
// mantissa bits), 2^f from a minimax polynomial with p(0) = 1 (coefficients
// from fit_exp2_poly.py: degree 3, max relative error 8.6e-5 in fp32, on
// 3 (row logsumexp) or 5 (transposed pass) of every 16 pairs: a row's lse moves by at most that
// relative error of its polynomial terms' share, and a target by about the
// same relative amount, against 2e-3; degree 4, 3.0e-6, is kept for the
// KVPOP_LSE_DEG3 = 0 build of the row logsumexp),
// and 2^n applied by adding n to the exponent field.  Inputs are clamped to
// >= -126 so the exponent arithmetic cannot wrap below; results below 2^-126
// are therefore at most 2^-125 instead of 0, far below any tolerance.  Where
// an argument can be large (the row logsumexp, whose scores may lie far above
// the running offset), it is also clamped to <= 127: the result is then at
// least 2^127, so the tile's sum reaches the overflow check (>= 2^64) that
// sends the row to its exact path, as MUFU's +inf does, instead of the
// exponent field wrapping to a tiny value that would drop the term.
constexpr float kRoundMagic = 12582912.0f;  // 1.5 * 2^23
constexpr float kP1 = 0x1.62d6c6p-1f, kP2 = 0x1.ee2450p-3f, kP3 = 0x1.abf868p-5f, kP4 = 0x1.b7f730p-7f;
constexpr float kT1 = 0x1.63e658p-1f, kT2 = 0x1.d2378ap-3f, kT3 = 0x1.3baaa6p-4f;

template <bool kDeg3 = false>
__device__ __forceinline__ uint64_t exp2_poly_pair(uint64_t y) {
  float y0, y1;
  f2_unpack(y, y0, y1);
  // The row logsumexp's path (the only user): both clamps.
  const uint64_t yc = f2_pack(fminf(fmaxf(y0, -126.f), 127.f), fminf(fmaxf(y1, -126.f), 127.f));
  const uint64_t t = f2_add_rm(yc, f2_pack(kRoundMagic, kRoundMagic));
  const uint64_t n = f2_add(t, f2_pack(-kRoundMagic, -kRoundMagic));
  const uint64_t f = f2_fma(n, f2_pack(-1.f, -1.f), yc);
  uint64_t q;
  if constexpr (kDeg3) {
    q = f2_fma(f, f2_pack(kT3, kT3), f2_pack(kT2, kT2));
    q = f2_fma(q, f, f2_pack(kT1, kT1));
  } else {
    q = f2_fma(f, f2_pack(kP4, kP4), f2_pack(kP3, kP3));
    q = f2_fma(q, f, f2_pack(kP2, kP2));
    q = f2_fma(q, f, f2_pack(kP1, kP1));
  }
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
// fused multiply-add, n = t - 1.5 * 2^23 = floor(c x) (taken negated, in one
// packed FMA), f = c x - n (exact).  kClampHigh: x is also clamped to
// <= xmax (c xmax = 127; the row logsumexp at offset 0); the transposed pass
// needs no upper clamp, its arguments are <= 0 up to rounding.
template <bool kClampHigh>
__device__ __forceinline__ uint64_t exp2_poly_pair_scaled(uint64_t x, uint64_t c2, float xmin, float xmax) {
  float x0, x1;
  f2_unpack(x, x0, x1);
  x0 = fmaxf(x0, xmin);
  x1 = fmaxf(x1, xmin);
  if constexpr (kClampHigh) {
    x0 = fminf(x0, xmax);
    x1 = fminf(x1, xmax);
  }
  const uint64_t xc = f2_pack(x0, x1);
  uint64_t t;
  asm("fma.rm.ftz.f32x2 %0, %1, %2, %3;" : "=l"(t) : "l"(xc), "l"(c2), "l"(f2_pack(kRoundMagic, kRoundMagic)));
  const uint64_t neg_n = f2_fma(t, f2_pack(-1.f, -1.f), f2_pack(kRoundMagic, kRoundMagic));   // -n, exact
  const uint64_t f = f2_fma(xc, c2, neg_n);
  uint64_t q = f2_fma(f, f2_pack(kT3, kT3), f2_pack(kT2, kT2));
  q = f2_fma(q, f, f2_pack(kT1, kT1));
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
// evaluated by the polynomial, spread evenly over the chunk, and the row
// logsumexp's polynomial degree (measured on B200 for each pass at the
// Qwen3-8B 16k shape: degree 3 beat degree 4; pass 1, whose polynomial also
// clamps from above, is fastest at 3 of 16 pairs (2 to 6 measured), pass 2
// at 5).
#ifndef KVPOP_LSE_DEG3
#define KVPOP_LSE_DEG3 1
#endif
#ifndef KVPOP_POLY16_LSE
#define KVPOP_POLY16_LSE 3
#endif
#ifndef KVPOP_POLY16_TARGET
#define KVPOP_POLY16_TARGET 5
#endif

template <int kPoly>
__device__ __forceinline__ constexpr bool poly_pair(int q) {
  return ((q * kPoly) & 15) < kPoly;
}

// acc += exp2(x * c + nb) over one 16-column chunk (nb: one negated offset
// for the whole chunk); of every 16 pairs kPoly go through the polynomial
// (pairs kQ0 .. kQ0+7 of that pattern are this chunk's), the rest through
// MUFU.  kBiasFree: nb is zero, the scale is folded into the polynomial's
// range reduction and xmin <= x (<= xmax with kClampHigh) keeps c x in
// [-126, 127].
template <int kPoly, bool kBiasFree, int kQ0, bool kDeg3 = kBiasFree, bool kClampHigh = false>
__device__ __forceinline__ void chunk_exp_sum(const uint32_t (&r)[16], uint64_t c2, uint64_t nb, float xmin,
                                              float xmax, uint64_t (&acc)[4]) {
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    const uint64_t x = f2_pack(__uint_as_float(r[2 * q]), __uint_as_float(r[2 * q + 1]));
    uint64_t e;
    if (poly_pair<kPoly>(kQ0 + q)) {
      e = kBiasFree ? exp2_poly_pair_scaled<kClampHigh>(x, c2, xmin, xmax)
                    : exp2_poly_pair<kDeg3>(f2_fma(x, c2, nb));
    } else {
      e = exp2_mufu_pair(f2_fma(x, c2, nb));
    }
    acc[q & 3] = f2_add(acc[q & 3], e);
  }
}

// Same with only columns lo <= e < hi of the chunk counted (MUFU only, so
// huge negative arguments give exact zeros).
__device__ __forceinline__ void chunk_exp_sum_masked(const uint32_t (&r)[16], uint64_t c2, uint64_t nb, int lo,
                                                     int hi, uint64_t (&acc)[4]) {
#pragma unroll
  for (int q = 0; q < 8; ++q) {
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

// Sum of exp2(x * c - off) over the kGroupCols = 64 columns of this thread's
// TMEM lane starting at taddr: four chunks of 16, each load in flight while
// the chunk before it is summed (small chunks shorten the load every warp of
// the CTA waits for at the start of a tile).  `release` runs (warp-converged)
// once the last chunk's load has landed, before its exponentials: the
// accumulator is free for the next MMA from then on.  kMasked: column m
// counts iff lo <= m < hi.
template <bool kMasked, int kPoly, bool kBiasFree = false, bool kDeg3 = kBiasFree, bool kClampHigh = false,
          class Release>
__device__ __forceinline__ float group_exp_sum(uint32_t taddr, uint64_t c2, uint64_t nb, int lo, int hi, float xmin,
                                               float xmax, Release&& release) {
  uint32_t ra[16], rb[16];
  uint64_t acc[4] = {0, 0, 0, 0};
  tmem_load<16>(taddr, ra);
  tmem_load_wait<16>(ra);
  tmem_load<16>(taddr + 16, rb);
  if constexpr (kMasked) chunk_exp_sum_masked(ra, c2, nb, lo, hi, acc);
  else chunk_exp_sum<kPoly, kBiasFree, 0, kDeg3, kClampHigh>(ra, c2, nb, xmin, xmax, acc);
  tmem_load_wait<16>(rb);
  tmem_load<16>(taddr + 32, ra);
  if constexpr (kMasked) chunk_exp_sum_masked(rb, c2, nb, lo - 16, hi - 16, acc);
  else chunk_exp_sum<kPoly, kBiasFree, 8, kDeg3, kClampHigh>(rb, c2, nb, xmin, xmax, acc);
  tmem_load_wait<16>(ra);
  tmem_load<16>(taddr + 48, rb);
  if constexpr (kMasked) chunk_exp_sum_masked(ra, c2, nb, lo - 32, hi - 32, acc);
  else chunk_exp_sum<kPoly, kBiasFree, 0, kDeg3, kClampHigh>(ra, c2, nb, xmin, xmax, acc);
  tmem_load_wait<16>(rb);
  release();
  if constexpr (kMasked) chunk_exp_sum_masked(rb, c2, nb, lo - 48, hi - 48, acc);
  else chunk_exp_sum<kPoly, kBiasFree, 8, kDeg3, kClampHigh>(rb, c2, nb, xmin, xmax, acc);
  return acc_total(acc);
}

// q . k of one bf16 row pair of HD elements, in fp32, on CUDA cores.
template <int HD>
__device__ __forceinline__ float dot_bf16_row(const uint16_t* a, const uint16_t* b) {
  float s0 = 0.f, s1 = 0.f;
#pragma unroll 4
  for (int d = 0; d < HD; d += 8) {
    const uint4 x = __ldg(reinterpret_cast<const uint4*>(a + d));
    const uint4 y = __ldg(reinterpret_cast<const uint4*>(b + d));
    const uint32_t xs[4] = {x.x, x.y, x.z, x.w}, ys[4] = {y.x, y.y, y.z, y.w};
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      s0 = fmaf(__uint_as_float(xs[w] << 16), __uint_as_float(ys[w] << 16), s0);
      s1 = fmaf(__uint_as_float(xs[w] & 0xffff0000u), __uint_as_float(ys[w] & 0xffff0000u), s1);
    }
  }
  return s0 + s1;
}

// Pass 1's exact path for one lane whose tile sum left the safe range (a
// row's first tile outside [2^-64, 2^64), any later tile past 2^64): the
// scores of its row over the group's columns 0 .. hi-1 are computed again on
// CUDA cores from Q and K in global memory (qrow: the query row; k0: the key
// of column 0, the next column kstride elements further on), because the
// accumulator has already gone back to the MMA.  Their exact max, if above
// the running offset, becomes the new offset (the running sum rescaled), and
// the tile's sum is returned at that offset.  Rare: ordinary inputs never
// reach it; scores (in log2 units) beyond about +-64 in a row's first tile,
// or more than about 58 above the running offset later, do.
template <int HD>
__device__ __noinline__ float lse_tile_exact(const uint16_t* qrow, const uint16_t* k0, int64_t kstride, int hi,
                                             float c, float& off, float& sum) {
  float m = -INFINITY;
  for (int e = 0; e < hi; ++e) m = fmaxf(m, dot_bf16_row<HD>(qrow, k0 + e * kstride) * c);
  const float noff = fmaxf(off, m);
  if (!(noff > -INFINITY)) return 0.f;   // no column counts
  sum = (off > -INFINITY) ? sum * ex2_approx(off - noff) : 0.f;
  off = noff;
  float ts = 0.f;
  for (int e = 0; e < hi; ++e) ts += ex2_approx(dot_bf16_row<HD>(qrow, k0 + e * kstride) * c - off);
  return ts;
}

// ------------------------------------------------------------------ softmax: pass 1

// Releases an accumulator: a single CTA's own barrier, or (CTA pairs) the
// first CTA's, which counts the softmax warps of both CTAs.
template <int kCta>
__device__ __forceinline__ void release_acc(uint64_t* bar) {
  if constexpr (kCta == 1) mbar_arrive(bar);
  else mbar_arrive_leader(bar);
}

template <int HD, bool kFused, int kCta = 1>
__device__ void lse_softmax_phase(const AttnParams& p, const Phase& ph, uint8_t* smem, const Bars& bars,
                                  const WaitCtl& ctl, uint32_t tmem_base, SoftmaxState& st) {
  using L = SmemLayout<HD, kFused, kCta>;
  using Pass = LsePassT<kCta>;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int sw = warp - 2;                 // softmax warp 0 .. kSoftmaxWarps-1
  const int wg = sw >> 2;                  // column group
  const int c0 = wg * kGroupCols;          // its first accumulator column
  const int quad = warp & 3;               // TMEM lane quadrant this warp may access
  const int row = quad * 32 + lane;        // query row within the tile
  const uint32_t lane_addr = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + c0;
  float* comb = reinterpret_cast<float*>(smem + L::OFF_COMB);
  const float c = p.scale_log2;
  const uint64_t c2 = f2_pack(c, c);
  const float kBig = 18446744073709551616.0f;   // 2^64: larger tile sums force an exact rescale
  const float kRebase = 4294967296.0f;          // 2^32: keep the running sum moderate
  const float kTiny = 5.421010862427522e-20f;   // 2^-64: smaller first-tile sums take the exact max
  const float xmin = -126.f / p.scale_log2;     // below it exp2(c x) < 2^-126: clamp for the polynomial
  const float xmax = 127.f / p.scale_log2;      // above it the exponent field would wrap: clamp
  const LevelSchedule& sched = *ph.sched;
  const int32_t total = sched.total_items;
  for (int32_t k = 0; st.ok; ++k) {
    const int32_t n = cta_item(k, blockIdx.x / kCta, gridDim.x / kCta);
    if (n >= total) break;
    const typename Pass::Item it = Pass::item(p, sched, n);
    float off = -INFINITY, sum = 0.f;      // running offset (log2 units) and sum of exp2(y - off)
    for (int32_t t = 0; t < it.ntiles; ++t) {
      const uint32_t acc = st.acc_cnt & 1u;
      if (!warp_wait(&bars.acc_full[acc], (st.acc_cnt >> 1) & 1u, ctl, SITE_SOFTMAX_ACC_FULL)) {
        st.ok = false;
        break;
      }
      tc_fence_after_sync();
      // The last key tile holds the diagonal: row r of this CTA may see
      // columns up to dcol + r, with dcol = 0 when a single CTA's query tile
      // starts on a 256-key boundary (then only columns 0..127 were
      // computed), 128 otherwise, and 128 * rank in a CTA pair.  A column
      // group wholly right of every row's diagonal is skipped; one wholly
      // left of it takes the unmasked path.
      const bool last = (t == it.ntiles - 1);
      const int dcol = Pass::diag_col(it, t);
      const bool skip = last && (kCta == 1 ? (Pass::half_tile(it, t) && c0 >= kStreamRows / 2)
                                           : c0 > dcol + kTileRows - 1);
      const bool masked = last && !skip && c0 + kGroupCols - 1 > dcol;
      const int hi = masked ? min(kGroupCols, max(0, row - (c0 - dcol) + 1)) : kGroupCols;
      // The accumulator goes back to the MMA once the group's last chunk is
      // in registers (at once for a skipped group): the rare exact path
      // below recomputes scores on CUDA cores instead of re-reading it.
      auto release = [&]() {
        tc_fence_before_sync();
        __syncwarp();
        if (lane == 0) release_acc<kCta>(&bars.acc_empty[acc]);
      };
      if (skip) {
        release();
      } else {
        const uint32_t taddr = lane_addr + acc * kStreamRows;
        float ts = 0.f;
        // A row's first tile is summed with offset 0 instead of its exact max
        // (one TMEM pass instead of two) and kept when the sum lands in
        // [2^-64, 2^64): no overflow, and far from the fp32 underflow.
        // Otherwise, as for any later tile past 2^64, the exact max is taken.
        const bool first = (off == -INFINITY);
        if (first) off = 0.f;
        {
          const uint64_t nb = f2_pack(-off, -off);
#if KVPOP_LSE_DEG3
          // Rows whose running offset is still 0 (the common case) take the
          // transposed pass's scale-folded polynomial; chosen per warp.
          if (masked)
            ts = group_exp_sum<true, 0>(taddr, c2, nb, 0, hi, 0.f, 0.f, release);
          else if (__all_sync(0xffffffffu, off == 0.f))
            ts = group_exp_sum<false, KVPOP_POLY16_LSE, true, true, true>(taddr, c2, nb, 0, kGroupCols, xmin, xmax,
                                                                         release);
          else
            ts = group_exp_sum<false, KVPOP_POLY16_LSE, false, true>(taddr, c2, nb, 0, kGroupCols, 0.f, 0.f,
                                                                    release);
#else
          ts = masked ? group_exp_sum<true, 0>(taddr, c2, nb, 0, hi, 0.f, 0.f, release)
                      : group_exp_sum<false, KVPOP_POLY16_LSE>(taddr, c2, nb, 0, kGroupCols, 0.f, 0.f, release);
#endif
        }
        const bool rescale = !(ts < kBig) || (first && !(ts >= kTiny));
        if (rescale) {
          if (first) off = -INFINITY;
          // Per lane (no TMEM access): rows past the sequence end are not
          // written, and their keys may lie past T, so they only reset.
          const int32_t i = it.i0 + kTileRows * cta_rank<kCta>() + row;   // query row within the sequence
          const int32_t j = t * kStreamRows + c0;                          // key of the group's column 0
          if (i < it.L &&
              KVPOP_IN(it.s + i < p.total_tokens && (hi <= 0 || it.s + j + hi <= p.total_tokens) &&
                           it.g < p.n_q_heads,
                       p.dbg, DBG_ROW_LSE, 7)) {
            const uint16_t* qrow = p.q + (static_cast<int64_t>(it.s + i) * p.n_q_heads + it.g) * HD;
            const uint16_t* k0 = p.k + (static_cast<int64_t>(it.s + j) * p.n_kv_heads + it.h) * HD;
            ts = lse_tile_exact<HD>(qrow, k0, static_cast<int64_t>(p.n_kv_heads) * HD, hi, c, off, sum);
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
      ++st.acc_cnt;
    }
    if (!st.ok) break;
    // Combine the column groups of each row: groups 1.. hand (offset, sum)
    // to group 0 through shared memory.
    if (wg != 0) {
      if (!warp_wait(bars.comb_empty, (st.item_cnt & 1u) ^ 1u, ctl, SITE_SOFTMAX_ACC_FULL)) {
        st.ok = false;
        break;
      }
      comb[(2 * (wg - 1)) * 128 + row] = off;
      comb[(2 * (wg - 1) + 1) * 128 + row] = sum;
      __syncwarp();
      if (lane == 0) mbar_arrive(bars.comb_full);
    } else {
      if (!warp_wait(bars.comb_full, st.item_cnt & 1u, ctl, SITE_SOFTMAX_ACC_FULL)) {
        st.ok = false;
        break;
      }
      float offs[kColGroups], sums[kColGroups];
      offs[0] = off;
      sums[0] = sum;
#pragma unroll
      for (int g = 1; g < kColGroups; ++g) {
        offs[g] = comb[(2 * (g - 1)) * 128 + row];
        sums[g] = comb[(2 * (g - 1) + 1) * 128 + row];
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(bars.comb_empty);
      float m = offs[0];
#pragma unroll
      for (int g = 1; g < kColGroups; ++g) m = fmaxf(m, offs[g]);
      float s = 0.f;
#pragma unroll
      for (int g = 0; g < kColGroups; ++g) s += (offs[g] > -INFINITY) ? sums[g] * ex2_approx(offs[g] - m) : 0.f;
      const int32_t i = it.i0 + kTileRows * cta_rank<kCta>() + row;
      if (i < it.L) {
        const float lse = (m + log2f(s)) * kLn2;
        const int64_t at = static_cast<int64_t>(it.g) * p.total_tokens + it.s + i;
        if (KVPOP_IN(at >= 0 && at < static_cast<int64_t>(p.n_q_heads) * p.total_tokens, p.dbg, DBG_ROW_LSE, 5)) {
          ph.out[at] = lse;
          if (p.nrm_rows != nullptr) static_cast<uint4*>(p.nrm_rows)[at] = norm_row(lse, p.inv_scale);
        }
      }
      if constexpr (kFused) {
        // Publish this warp's 32 rows: the proxy fence and the warp barrier
        // order every lane's stores (read by other CTAs' bulk copies) before
        // lane 0's gpu-scope release.
        fence_proxy_async_global();
        __syncwarp();
        const int64_t fi = static_cast<int64_t>(it.g) * ph.n_flag_tiles + ph.tile_base[it.seq] + it.i0 / kTileRows;
        if (lane == 0 && KVPOP_IN(fi >= 0 && fi < static_cast<int64_t>(p.n_q_heads) * ph.n_flag_tiles, p.dbg,
                                  DBG_ROW_LSE, 6))
          flag_release_add(ph.flags + fi, 1);
      }
    }
    ++st.item_cnt;
  }
}

// ------------------------------------------------------------------ softmax: pass 2

template <int HD, int kCta = 1>
__device__ void target_softmax_phase(const AttnParams& p, const Phase& ph, uint8_t* smem, const Bars& bars,
                                     const WaitCtl& ctl, uint32_t tmem_base, SoftmaxState& st) {
  using L = SmemLayout<HD, true, kCta>;
  using Pass = TargetPassT<kCta>;
  const int rk = kTileRows * cta_rank<kCta>();   // this CTA's first key within the item
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int sw = warp - 2;
  const int wg = sw >> 2;                  // column group
  const int c0 = wg * kGroupCols;          // its first accumulator column
  const int quad = warp & 3;
  const int row = quad * 32 + lane;        // key row within the tile
  const uint32_t lane_addr = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + c0;
  float* comb = reinterpret_cast<float*>(smem + L::OFF_COMB);
  const uint64_t c2 = f2_pack(p.scale_log2, p.scale_log2);
  const uint64_t zero2 = f2_pack(0.f, 0.f);
  const float xmin = -126.f / p.scale_log2;   // below it exp2(c x) < 2^-126: clamp for the polynomial
  const LevelSchedule& sched = *ph.sched;
  const int32_t total = sched.total_items;
  for (int32_t k = 0; st.ok; ++k) {
    const int32_t n = cta_item(k, blockIdx.x / kCta, gridDim.x / kCta);
    if (n >= total) break;
    const typename Pass::Item it = Pass::item(p, sched, n);
    // Each query head's tiles are summed on their own (Kahan-compensated),
    // then the heads are added in order: the same sums, in the same order,
    // whether an item covers all G heads or one of them.
    float heads = 0.f;
    const bool ragged_end = it.i0 + it.nq * kStreamRows > it.L;
    for (int32_t g = 0; g < (it.nq > 0 ? it.ng : 0) && st.ok; ++g) {
      float run = 0.f, comp = 0.f;
      for (int32_t qt = 0; qt < it.nq; ++qt) {
        const uint32_t acc = st.acc_cnt & 1u;
        if (!warp_wait(&bars.acc_full[acc], (st.acc_cnt >> 1) & 1u, ctl, SITE_SOFTMAX_ACC_FULL)) {
          st.ok = false;
          break;
        }
        tc_fence_after_sync();
        const uint32_t taddr = lane_addr + acc * kStreamRows;
        // First query tile: query column m is valid for key row r (of this
        // CTA; rk + r within the item) iff m >= rk + r, which can mask
        // columns of the groups below column rk + 128 (per-lane bound lo); a
        // pair's second CTA skips the groups wholly below column 128.  Last
        // query tile: columns past the sequence end (their normaliser rows
        // belong to another sequence, or are stale) are cut by hi.  The path
        // is chosen per warp: its TMEM loads are warp-collective.
        const bool skip = (qt == 0) && (c0 + kGroupCols <= rk);
        const bool diag = (qt == 0) && (c0 < rk + kTileRows);
        const bool ragged = (qt == it.nq - 1) && ragged_end;
        const int lo = diag ? max(0, rk + row - c0) : 0;
        const int hi = ragged ? min(kGroupCols, it.L - it.i0 - qt * kStreamRows - c0) : kGroupCols;
        auto release = [&]() {
          tc_fence_before_sync();
          __syncwarp();
          if (lane == 0) release_acc<kCta>(&bars.acc_empty[acc]);
        };
        float ts = 0.f;
        if (skip)
          release();
        else if (diag || ragged)
          ts = group_exp_sum<true, 0>(taddr, c2, zero2, lo, hi, 0.f, 0.f, release);
        else
          ts = group_exp_sum<false, KVPOP_POLY16_TARGET, true>(taddr, c2, zero2, 0, kGroupCols, xmin, 0.f, release);
        ++st.acc_cnt;
        const float yk = ts - comp;
        const float tk = run + yk;
        comp = (tk - run) - yk;
        run = tk;
      }
      heads += run;
    }
    if (!st.ok) break;
    if (p.g_split > 1) {
      // One query head per item: every column group writes its own partial
      // [g, column group, h, T]; a merge kernel adds them in the order below.
      const int32_t j = it.j0 + rk + row;
      const int64_t at = (static_cast<int64_t>(it.g0 * kColGroups + wg) * p.n_kv_heads + it.h) * p.total_tokens + it.s + j;
      if (j < it.L &&
          KVPOP_IN(at >= 0 && at < static_cast<int64_t>(p.n_q_heads) * kColGroups * p.total_tokens, p.dbg, DBG_TARGET, 7))
        ph.out[at] = heads;
    } else if (wg != 0) {
      if (!warp_wait(bars.comb_empty, (st.item_cnt & 1u) ^ 1u, ctl, SITE_SOFTMAX_ACC_FULL)) {
        st.ok = false;
        break;
      }
      comb[(wg - 1) * 128 + row] = heads;
      __syncwarp();
      if (lane == 0) mbar_arrive(bars.comb_full);
    } else {
      if (!warp_wait(bars.comb_full, st.item_cnt & 1u, ctl, SITE_SOFTMAX_ACC_FULL)) {
        st.ok = false;
        break;
      }
      float sum = heads;
#pragma unroll
      for (int g = 1; g < kColGroups; ++g) sum += comb[(g - 1) * 128 + row];
      __syncwarp();
      if (lane == 0) mbar_arrive(bars.comb_empty);
      const int32_t j = it.j0 + rk + row;
      const int64_t at = static_cast<int64_t>(it.h) * p.total_tokens + it.s + j;
      if (j < it.L && KVPOP_IN(at >= 0 && at < static_cast<int64_t>(p.n_kv_heads) * p.total_tokens, p.dbg, DBG_TARGET, 8))
        ph.out[at] = sum;
    }
    ++st.item_cnt;
  }
}

// ------------------------------------------------------------------ kernels

__device__ __forceinline__ uint8_t* aligned_smem(uint8_t* raw) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(raw) + 1023) & ~static_cast<uintptr_t>(1023));
}

// Barriers, slab constants and TMEM of one CTA.  kSlab: the pass-2 layout
// (the ones block of A; the normaliser block of every B stage zeroed, so
// that its upper half stays zero under the loads of the lower half).  CTA
// pairs: the accumulator-empty barrier of the first CTA counts the softmax
// warps of both CTAs; TMEM is allocated in both CTAs by the same warp, and
// the pair synchronises once its barriers are initialised, before any
// cross-CTA arrival.
template <int HD, bool kSlab, int kCta = 1>
__device__ __forceinline__ void cta_setup(uint8_t* smem, const Bars& bars, uint32_t* tmem_slot,
                                          volatile int* abort_flag) {
  using L = SmemLayout<HD, kSlab, kCta>;
  if constexpr (kSlab) {
    // Zero the extra K-columns of A and of every B stage, then put the ones in A.
    for (int s = 0; s < L::kNStages; ++s) {
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
      mbar_init(&bars.acc_empty[i], kSoftmaxWarps * kCta);
    }
    for (int i = 0; i < L::kNStages; ++i) {
      mbar_init(&bars.b_full[i], 1);
      mbar_init(&bars.b_empty[i], 1);
    }
    mbar_init(bars.comb_full, 4 * (kColGroups - 1));
    mbar_init(bars.comb_empty, 4);
    mbar_init(bars.mma_done, 1);
    *abort_flag = 0;
    fence_mbarrier_init();
  }
  if ((threadIdx.x >> 5) == 1) {
    tmem_alloc<kCta>(tmem_slot, 512);
    tmem_relinquish<kCta>();
    tc_fence_before_sync();
  }
  __syncthreads();
  if constexpr (kCta == 2) cluster_sync_all();
  tc_fence_after_sync();
}

// CTA pairs: after an abort, how long the CTAs wait before leaving, so that
// tiled loads already issued (whose completion the second CTA cannot wait
// for) land while both CTAs are still resident.
constexpr uint64_t kPairAbortGraceNs = 100000;

template <int kCta = 1>
__device__ __forceinline__ void cta_teardown(uint32_t tmem_base, volatile int* abort_flag) {
  tc_fence_before_sync();
  __syncthreads();
  if constexpr (kCta == 2) {
    if (threadIdx.x == 0 && *abort_flag) {
      const uint64_t t0 = global_timer_ns();
      while (global_timer_ns() - t0 < kPairAbortGraceNs) __nanosleep(1000);
    }
    __syncthreads();
    cluster_sync_all();   // neither CTA leaves while the other may still arrive on its barriers
  }
  if ((threadIdx.x >> 5) == 1) {
    __syncwarp();
    tc_fence_after_sync();
    tmem_dealloc<kCta>(tmem_base, 512);
  }
}

template <class Pass, int HD, int kCta>
__device__ __forceinline__ void attn_kernel_body(const AttnParams& p, uint8_t* smem_raw) {
  using L = SmemLayout<HD, Pass::kSlab, kCta>;
  uint8_t* smem = aligned_smem(smem_raw);
  const Bars bars = carve_bars<L::kNStages>(reinterpret_cast<uint64_t*>(smem + L::OFF_BAR));
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::OFF_MISC + 4);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (warp == 0 && lane == 0) {
    tma_prefetch_map(&p.tmap_q);
    tma_prefetch_map(&p.tmap_k);
    if constexpr (kCta == 2 && Pass::kSlab) tma_prefetch_map(&p.tmap_rows);
  }
  cta_setup<HD, Pass::kSlab, kCta>(smem, bars, tmem_slot, abort_flag);
  const uint32_t tmem_base = *tmem_slot;
  WaitCtl ctl{abort_flag, p.status, p.wait_ns};
  if constexpr (kCta == 2)
    ctl.peer_abort = cluster_map(const_cast<int*>(reinterpret_cast<volatile int*>(abort_flag)),
                                 static_cast<uint32_t>(cta_rank<kCta>() ^ 1));
  const Phase ph{&p.sched, &p.tmap_q, &p.tmap_k, p.out, nullptr, nullptr, 0, nullptr};
#if KVPOP_PDL_PASSES
  // Launched as a programmatic dependent: the setup above (barriers, TMEM,
  // tensor-map prefetch) overlapped the previous kernel's tail; every global
  // read and write of the roles comes after this wait.
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
#endif

  if (warp == 0) {
    ProducerState st;
    producer_phase<Pass, HD, false, kCta>(p, ph, smem, bars, ctl, st);
    producer_drain<L::kNStages>(bars, ctl, st, cta_rank<kCta>() == 0);
  } else if (warp == 1) {
    if (lane == 0 && cta_rank<kCta>() == 0) {
      MmaState st;
      mma_phase<Pass, HD, false, kCta>(p, ph, smem, bars, ctl, tmem_base, st);
      mma_finish<kCta>(bars, ctl, st);
    }
  } else {
    SoftmaxState st;
    if constexpr (Pass::kSlab)
      target_softmax_phase<HD, kCta>(p, ph, smem, bars, ctl, tmem_base, st);
    else
      lse_softmax_phase<HD, false, kCta>(p, ph, smem, bars, ctl, tmem_base, st);
  }
  cta_teardown<kCta>(tmem_base, abort_flag);
}

// One CTA per SM (kCta = 1), or one CTA pair per two SMs (kCta = 2, a
// cluster of two that shares each M = 256 MMA).
template <int HD, int kCta>
__global__ void __launch_bounds__(kThreads, 1) row_lse_kernel(const __grid_constant__ AttnParams p) {
  extern __shared__ uint8_t smem_raw[];
  attn_kernel_body<LsePassT<kCta>, HD, kCta>(p, smem_raw);
}

template <int HD, int kCta>
__global__ void __launch_bounds__(kThreads, 1) future_target_kernel(const __grid_constant__ AttnParams p) {
  extern __shared__ uint8_t smem_raw[];
  attn_kernel_body<TargetPassT<kCta>, HD, kCta>(p, smem_raw);
}

// Both passes in one cooperative launch (one CTA per SM, all co-resident, so
// a CTA waiting for another CTA's lse tile always has that CTA running).
// Each role runs pass 1, then pass 2 with its pipeline counters carried over;
// a role whose pass 1 gave up skips pass 2.
template <int HD>
__global__ void __launch_bounds__(kThreads, 1) fused_targets_kernel(const __grid_constant__ FusedParams fp) {
  extern __shared__ uint8_t smem_raw[];
  using L = SmemLayout<HD, true>;
  const AttnParams& p = fp.attn;
  uint8_t* smem = aligned_smem(smem_raw);
  const Bars bars = carve_bars(reinterpret_cast<uint64_t*>(smem + L::OFF_BAR));
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::OFF_MISC + 4);
  volatile int* last_cta = reinterpret_cast<volatile int*>(smem + L::OFF_MISC + 8);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (warp == 0 && lane == 0) {
    tma_prefetch_map(&p.tmap_q);
    tma_prefetch_map(&p.tmap_k);
    tma_prefetch_map(&fp.tmap_q_stream);
    tma_prefetch_map(&fp.tmap_k_tile);
  }
  cta_setup<HD, true>(smem, bars, tmem_slot, abort_flag);
  const uint32_t tmem_base = *tmem_slot;
  const WaitCtl ctl{abort_flag, p.status, p.wait_ns};
  const Phase ph1{&p.sched, &p.tmap_q, &p.tmap_k, p.out, fp.flags, fp.tile_base_lse, fp.n_flag_tiles, fp.lse_done};
  const Phase ph2{&fp.sched_target, &fp.tmap_q_stream, &fp.tmap_k_tile, fp.target, fp.flags,
                  fp.tile_base_target, fp.n_flag_tiles, fp.lse_done};

  if (warp == 0) {
    ProducerState st;
    producer_phase<LsePass, HD, true>(p, ph1, smem, bars, ctl, st);
    if (st.ok) producer_phase<TargetPass, HD, true>(p, ph2, smem, bars, ctl, st);
    producer_drain(bars, ctl, st);
  } else if (warp == 1) {
    if (lane == 0) {
      MmaState st;
      mma_phase<LsePass, HD, true>(p, ph1, smem, bars, ctl, tmem_base, st);
      if (st.ok) mma_phase<TargetPass, HD, true>(p, ph2, smem, bars, ctl, tmem_base, st);
      mma_finish(bars, ctl, st);
    }
  } else {
    SoftmaxState st;
    lse_softmax_phase<HD, true>(p, ph1, smem, bars, ctl, tmem_base, st);
    if (st.ok) {
      // This warp's pass-1 rows are all written (and published tile by tile).
      __syncwarp();
      if (lane == 0) flag_release_add(fp.lse_done, 1);
      target_softmax_phase<HD>(p, ph2, smem, bars, ctl, tmem_base, st);
    }
  }
  cta_teardown(tmem_base, abort_flag);

  // The last CTA out (every other CTA has finished all its flag traffic)
  // clears the flags and the counter, leaving the workspace zeroed.
  if (threadIdx.x == 0) *last_cta = (flag_arrive_count(fp.done) == static_cast<int32_t>(gridDim.x) - 1) ? 1 : 0;
  __syncthreads();
  if (*last_cta) {
    for (int32_t i = threadIdx.x; i < fp.n_flags; i += blockDim.x) fp.flags[i] = 0;
    if (threadIdx.x == 0) {
      *fp.done = 0;
      *fp.lse_done = 0;
    }
  }
}

// ------------------------------------------------------------------ launchers

// Most clusters of two CTAs of `kern` that can be resident at once (cached
// per device and kernel): GPCs with an odd number of free SMs leave one idle.
template <class Kern>
static int max_pair_clusters(Kern kern, int smem, int sm_count) {
  static std::mutex mu;
  static std::vector<std::pair<std::pair<int, const void*>, int>> cache;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return sm_count / 2;
  const void* key = reinterpret_cast<const void*>(kern);
  std::lock_guard<std::mutex> lock(mu);
  for (const auto& e : cache)
    if (e.first.first == dev && e.first.second == key) return e.second;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * (sm_count / 2));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess || n < 1) {
    cudaGetLastError();
    n = sm_count / 2;
  }
  cache.push_back({{dev, key}, n});
  return n;
}

template <int HD, bool kTarget, int kCta>
static cudaError_t launch_attn(const AttnParams& p, int sm_count, cudaStream_t stream) {
  using L = SmemLayout<HD, kTarget, kCta>;
  auto kern = kTarget ? future_target_kernel<HD, kCta> : row_lse_kernel<HD, kCta>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::ALLOC);
  if (e != cudaSuccess) return e;
  const int items = std::max(1, p.sched.total_items);
  if constexpr (kCta == 1) {
    kern<<<std::min(items, sm_count), kThreads, L::ALLOC, stream>>>(p);
    return cudaGetLastError();
  } else {
    const int pairs = std::min(items, std::max(1, max_pair_clusters(kern, L::ALLOC, sm_count)));
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * pairs);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = L::ALLOC;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = KVPOP_PDL_PASSES ? 2 : 1;
    return cudaLaunchKernelEx(&cfg, kern, p);
  }
}

// The standalone passes: p.cta = 2 (parameters built for CTA pairs) or 1.
cudaError_t launch_row_lse(const AttnParams& p, int head_dim, int sm_count, cudaStream_t stream) {
  if (p.cta == 2)
    return head_dim == 64 ? launch_attn<64, false, 2>(p, sm_count, stream)
                          : launch_attn<128, false, 2>(p, sm_count, stream);
  return head_dim == 64 ? launch_attn<64, false, 1>(p, sm_count, stream) : launch_attn<128, false, 1>(p, sm_count, stream);
}

cudaError_t launch_future_target(const AttnParams& p, int head_dim, int sm_count, cudaStream_t stream) {
  if (p.cta == 2)
    return head_dim == 64 ? launch_attn<64, true, 2>(p, sm_count, stream)
                          : launch_attn<128, true, 2>(p, sm_count, stream);
  return head_dim == 64 ? launch_attn<64, true, 1>(p, sm_count, stream) : launch_attn<128, true, 1>(p, sm_count, stream);
}

template <int HD>
static cudaError_t launch_fused_hd(const FusedParams& fp, int grid, cudaStream_t stream) {
  using L = SmemLayout<HD, true>;
  cudaError_t e =
      cudaFuncSetAttribute(fused_targets_kernel<HD>, cudaFuncAttributeMaxDynamicSharedMemorySize, L::ALLOC);
  if (e != cudaSuccess) return e;
  void* args[] = {const_cast<FusedParams*>(&fp)};
  return cudaLaunchCooperativeKernel(reinterpret_cast<const void*>(fused_targets_kernel<HD>), dim3(grid),
                                     dim3(kThreads), args, L::ALLOC, stream);
}

cudaError_t launch_fused_targets(const FusedParams& fp, int head_dim, int grid, cudaStream_t stream) {
  return head_dim == 64 ? launch_fused_hd<64>(fp, grid, stream) : launch_fused_hd<128>(fp, grid, stream);
}

// Sum of the split pass's partials [G][kColGroups][H_kv][T] into the target
// [H_kv][T], in the order the unsplit pass adds them: per column group the
// query heads in order, then the column groups in order.
__global__ void __launch_bounds__(256) merge_partials_kernel(const float* __restrict__ part, float* __restrict__ target,
                                                             int32_t group, int32_t n_kv_heads, int32_t total_tokens,
                                                             int32_t* dbg) {
  const int64_t n = static_cast<int64_t>(n_kv_heads) * total_tokens;
  const int64_t plane = n;   // one (g, column group) slice
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    float sum = 0.f;
#pragma unroll
    for (int c = 0; c < kColGroups; ++c) {
      float heads = 0.f;
      for (int32_t g = 0; g < group; ++g) {
        const int64_t at = (static_cast<int64_t>(g) * kColGroups + c) * plane + i;
        if (KVPOP_IN(at < static_cast<int64_t>(group) * kColGroups * plane, dbg, DBG_MERGE, 1)) heads += part[at];
      }
      sum = (c == 0) ? heads : sum + heads;
    }
    target[i] = sum;
  }
}

cudaError_t launch_merge_partials(const float* part, float* target, int group, int n_kv_heads, int total_tokens,
                                  int sm_count, int32_t* dbg, cudaStream_t stream) {
  const int64_t n = static_cast<int64_t>(n_kv_heads) * total_tokens;
  const int blocks = static_cast<int>(std::min<int64_t>((n + 255) / 256, static_cast<int64_t>(sm_count) * 8));
  merge_partials_kernel<<<std::max(blocks, 1), 256, 0, stream>>>(part, target, group, n_kv_heads, total_tokens, dbg);
  return cudaGetLastError();
}

int target_split_groups() { return kColGroups; }

// Normaliser rows [H_q, T] of pass 2 from a given lse [H_q, T] (the
// standalone pass; the pipelines have pass 1 write them next to lse).
__global__ void __launch_bounds__(256) norm_rows_kernel(const float* __restrict__ lse, uint4* __restrict__ rows,
                                                        int64_t n, float inv_scale, int32_t* dbg) {
#if KVPOP_PDL_PASSES
  asm volatile("griddepcontrol.wait;" ::: "memory");   // lse comes from the kernel before
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
#endif
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    if (KVPOP_IN(i >= 0 && i < n, dbg, DBG_NORM_ROWS, 1)) rows[i] = norm_row(__ldg(lse + i), inv_scale);
}

cudaError_t launch_norm_rows(const float* lse, void* rows, int64_t n, float inv_scale, int sm_count, int32_t* dbg,
                             cudaStream_t stream) {
  const int blocks = static_cast<int>(std::min<int64_t>((n + 255) / 256, static_cast<int64_t>(sm_count) * 8));
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(std::max(blocks, 1));
  cfg.blockDim = dim3(256);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = KVPOP_PDL_PASSES ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, norm_rows_kernel, lse, static_cast<uint4*>(rows), n, inv_scale, dbg);
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

// ------------------------------------------------------------------ debug-build self-test

// One index check that fails by design: the array declares n_valid = 1
// usable cells and the index is 1.  The array has 4 cells, so the guarded
// store would stay inside it even without the check; with the check (debug
// build) it is skipped and the code lands in *word.
__global__ void debug_selftest_kernel(int32_t* word, int32_t n_valid) {
  __shared__ int32_t cells[4];
  const int32_t idx = n_valid;
  if (threadIdx.x == 0) {
    cells[0] = 0;
    if (KVPOP_IN(idx >= 0 && idx < n_valid, word, DBG_SELFTEST, 1)) cells[idx & 3] = 1;
    if (cells[0] != 0) *word = -1;   // keeps the array live; never taken
  }
}

cudaError_t launch_debug_selftest(int32_t* word, cudaStream_t stream) {
  debug_selftest_kernel<<<1, 32, 0, stream>>>(word, 1);
  return cudaGetLastError();
}

}  // namespace kvpop
