// Device building blocks for the sm_100a kernels: mbarriers with bounded
// waits, TMA tile loads, tcgen05 (TMEM allocation, UMMA, TMEM loads), and the
// longest-first work schedule shared by both attention passes.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "kvpop_debug.cuh"
#include "kvpop_sched.h"

namespace kvpop {

// ------------------------------------------------------------------ basics

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// ------------------------------------------------------------------ mbarrier

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbarrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ uint32_t mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(done)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return done;
}

// Status word codes written by kernels (low byte = kvpop_status, next byte = wait site).
enum WaitSite : int32_t {
  SITE_PRODUCER_A_EMPTY = 1,
  SITE_PRODUCER_B_EMPTY = 2,
  SITE_MMA_A_FULL = 3,
  SITE_MMA_B_FULL = 4,
  SITE_MMA_ACC_EMPTY = 5,
  SITE_SOFTMAX_ACC_FULL = 6,
  SITE_TEARDOWN = 7,
  SITE_SELFTEST = 8,
  SITE_LSE_FLAG = 9,
};

struct WaitCtl {
  volatile int* abort_flag;  // shared memory; set by the first wait that gives up
  int32_t* status;           // device status word (may be null)
  uint64_t limit_ns;         // per-wait time limit
  volatile int* peer_abort = nullptr;  // CTA pairs: the other CTA's abort flag (distributed shared memory)
};

__device__ __forceinline__ void raise_abort(const WaitCtl& ctl) {
  *ctl.abort_flag = 1;
  if (ctl.peer_abort != nullptr) *ctl.peer_abort = 1;
}

// Waits for the phase of `bar` with parity `parity` to complete.  Returns
// false when the CTA is aborting or the wait ran past its limit (then the
// abort flag is raised and a timeout code is recorded).
__device__ __noinline__ bool wait_bounded(uint64_t* bar, uint32_t parity, const WaitCtl& ctl,
                                          int32_t site) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 15u) == 0u) {
      if (*ctl.abort_flag) return false;
      if (global_timer_ns() - t0 > ctl.limit_ns) {
        raise_abort(ctl);
        if (ctl.status != nullptr) atomicCAS(ctl.status, 0, 4 | (site << 8));
        return false;
      }
    }
  }
}

// ------------------------------------------------------------------ cross-CTA flags

// Adds v to a counter in global memory with gpu-scope release semantics: the
// calling thread's earlier writes (and those ordered before it by a barrier)
// are visible to any thread that later acquires the new value.
__device__ __forceinline__ void flag_release_add(int32_t* f, int32_t v) {
  asm volatile("red.release.gpu.global.add.s32 [%0], %1;" ::"l"(f), "r"(v) : "memory");
}

__device__ __forceinline__ int32_t flag_acquire_load(const int32_t* f) {
  int32_t v;
  asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(f) : "memory");
  return v;
}

// Returns the old value of *f and adds 1, acquire + release at gpu scope.
__device__ __forceinline__ int32_t flag_arrive_count(int32_t* f) {
  int32_t old;
  asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], 1;" : "=r"(old) : "l"(f) : "memory");
  return old;
}

// ------------------------------------------------------------------ TMA

__device__ __forceinline__ void tma_prefetch_map(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// 2-D tiled bulk load global -> shared, completion counted in bytes on `bar`.
// x is the element coordinate of the innermost dimension (must keep x * 2
// bytes a multiple of 16), y the row.
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar, int32_t x,
                                            int32_t y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y)
      : "memory");
}

// CTA pairs (a cluster of two CTAs sharing one tcgen05 MMA): the same
// shared-memory offset in the pair's first CTA.  A shared::cta address of
// this CTA, used as a shared::cluster address, names this CTA's own memory;
// clearing bit 24 names the first CTA's.
constexpr uint32_t kPairLeaderMask = 0xFEFFFFFFu;
__device__ __forceinline__ uint32_t leader_addr(const void* p) { return smem_u32(p) & kPairLeaderMask; }

// 2-D tiled load into this CTA's shared memory whose completion bytes count
// on the mbarrier at `bar`'s offset in the pair's first CTA (`.cta_group::2`).
__device__ __forceinline__ void tma_load_2d_pair(void* dst, const CUtensorMap* map, const uint64_t* bar, int32_t x,
                                                 int32_t y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(leader_addr(bar)), "r"(x), "r"(y)
      : "memory");
}

// The same for a 3-D map (coordinates x, y, z).
__device__ __forceinline__ void tma_load_3d_pair(void* dst, const CUtensorMap* map, const uint64_t* bar, int32_t x,
                                                 int32_t y, int32_t z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(leader_addr(bar)), "r"(x), "r"(y), "r"(z)
      : "memory");
}

// Arrive on the mbarrier at `bar`'s offset in the pair's first CTA.  Used to
// hand an accumulator back after this warp's TMEM reads, which
// tcgen05.wait::ld and tcgen05.fence::before_thread_sync already order; no
// generic memory write needs releasing, so the arrive keeps its default
// (CTA-scope) semantics: a cluster-scope release costs a memory barrier per
// warp and tile.
__device__ __forceinline__ void mbar_arrive_leader(const uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(leader_addr(bar)) : "memory");
}

// All threads of both CTAs of the cluster.
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Generic pointer to the same shared-memory object in CTA `rank` of the cluster.
template <class T>
__device__ __forceinline__ T* cluster_map(T* p, uint32_t rank) {
  uint64_t out;
  asm volatile("mapa.u64 %0, %1, %2;" : "=l"(out) : "l"(reinterpret_cast<uint64_t>(p)), "r"(rank));
  return reinterpret_cast<T*>(out);
}

// Contiguous bulk copy global -> shared: both addresses 16-byte aligned,
// bytes a multiple of 16; completion counted in bytes on `bar`.
__device__ __forceinline__ void bulk_load_1d(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
               ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}

// ------------------------------------------------------------------ tcgen05

// kCta = 1: this CTA's TMEM; kCta = 2: the same columns in both CTAs of a
// pair (issued by the same warp in each).
template <int kCta = 1>
__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
  if constexpr (kCta == 1)
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
                 "r"(ncols)
                 : "memory");
  else
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
                 "r"(ncols)
                 : "memory");
}
template <int kCta = 1>
__device__ __forceinline__ void tmem_relinquish() {
  if constexpr (kCta == 1)
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  else
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
template <int kCta = 1>
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  if constexpr (kCta == 1)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
  else
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before_sync() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after_sync() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Shared-memory matrix descriptor for a K-major bf16 tile written by TMA with
// 128-byte swizzle: rows of 128 bytes (64 elements), 8-row atoms of 1024 bytes.
// Leading byte offset is unused for swizzled K-major layouts (set to 16 B);
// stride byte offset = 1024 B between 8-row groups; descriptor version 1;
// layout type 2 = 128-byte swizzle.
__device__ __forceinline__ uint64_t umma_desc_sw128(uint32_t saddr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>(1u) << 16;
  d |= static_cast<uint64_t>(1024u >> 4) << 32;
  d |= static_cast<uint64_t>(1u) << 46;
  d |= static_cast<uint64_t>(2u) << 61;
  return d;
}

// Instruction descriptor, kind::f16: bf16 A and B (both K-major), fp32 accumulator.
__host__ __device__ constexpr uint32_t umma_idesc_bf16(int M, int N) {
  return (1u << 4)                                   // D format: f32
         | (1u << 7)                                 // A format: bf16
         | (1u << 10)                                // B format: bf16
         | (static_cast<uint32_t>(N >> 3) << 17)     // N / 8
         | (static_cast<uint32_t>(M >> 4) << 24);    // M / 16
}

// D[tmem] (+)= A[smem] * B[smem]^T, issued by one thread.
__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive on `bar` once every tcgen05 operation issued so far by this thread has completed.
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}

// CTA pairs: D[tmem] (+)= A * B^T with M = 256 (128 rows of A from each CTA's
// shared memory), B's N rows split in halves between the two CTAs, and the
// accumulator rows of each CTA in its own TMEM; issued by one thread of the
// first CTA.
__device__ __forceinline__ void umma_bf16_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                               uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// CTA pairs: arrive on the mbarrier at `bar`'s offset in both CTAs once every
// tcgen05 operation issued so far by this thread has completed.
__device__ __forceinline__ void umma_commit_pair(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
          smem_u32(bar)),
      "h"(static_cast<uint16_t>(3))
      : "memory");
}

// kW (16 or 32) consecutive fp32 columns of this thread's TMEM lane
// (warp-collective: every lane reads its own lane of the warp's quadrant).
template <int kW>
__device__ __forceinline__ void tmem_load(uint32_t taddr, uint32_t (&r)[kW]);

template <>
__device__ __forceinline__ void tmem_load<32>(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
        "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),
        "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]),
        "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}

template <>
__device__ __forceinline__ void tmem_load<16>(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
        "=r"(r[15])
      : "r"(taddr));
}

// Waits for this thread's outstanding TMEM loads.  The registers are passed
// through so that no use of them can be scheduled before the wait.
template <int kW>
__device__ __forceinline__ void tmem_load_wait(uint32_t (&r)[kW]);

template <>
__device__ __forceinline__ void tmem_load_wait<32>(uint32_t (&r)[32]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]),
                 "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]),
                 "+r"(r[14]), "+r"(r[15]), "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]),
                 "+r"(r[20]), "+r"(r[21]), "+r"(r[22]), "+r"(r[23]), "+r"(r[24]), "+r"(r[25]),
                 "+r"(r[26]), "+r"(r[27]), "+r"(r[28]), "+r"(r[29]), "+r"(r[30]), "+r"(r[31])
               :
               : "memory");
}

template <>
__device__ __forceinline__ void tmem_load_wait<16>(uint32_t (&r)[16]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]),
                 "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]),
                 "+r"(r[14]), "+r"(r[15])
               :
               : "memory");
}

// ------------------------------------------------------------------ schedule

struct WorkItem {
  int32_t seq_start;  // global row of the sequence's first token
  int32_t seq_len;
  int32_t level;      // pass 1: query tile index; pass 2: key tiles remaining after this one
  int32_t head;       // pass 1: query head; pass 2: KV head
  int32_t seq;        // position of the sequence in the schedule's sorted list
};

// Item n of the longest-first order: levels from the top down, then the
// sequences active at that level (longest first), then the heads.
__device__ __forceinline__ WorkItem decode_item(const LevelSchedule& s, int32_t n) {
  int32_t lo = 0, hi = s.n_levels - 1;
  while (lo < hi) {
    const int32_t mid = (lo + hi + 1) >> 1;
    if (s.level_base[mid] <= n) lo = mid; else hi = mid - 1;
  }
  const int32_t off = n - s.level_base[lo];
  const int32_t r = off / s.n_heads;
  WorkItem w;
  w.seq_start = s.seq_start[r];
  w.seq_len = s.seq_len[r];
  w.level = s.n_levels - 1 - lo;
  w.head = off - r * s.n_heads;
  w.seq = r;
  return w;
}

// k-th item of this CTA: a snake over the sorted list, so consecutive rounds
// pair the heaviest remaining items with the lightest.
__device__ __forceinline__ int32_t cta_item(int32_t k, int32_t cta, int32_t nctas) {
  return k * nctas + ((k & 1) ? (nctas - 1 - cta) : cta);
}

}  // namespace kvpop
