// Kernel parameter blocks shared by the host launchers and the kernels.
#pragma once

#include <cuda.h>
#include <stdint.h>

namespace kvpop {

constexpr int kMaxSeqs = 512;        // sequences per call
constexpr int kTileRows = 128;       // rows of the resident (A) tile = MMA M
constexpr int kMaxLevels = 1024;     // longest sequence = kMaxLevels * kTileRows tokens
constexpr int kStreamRows = 256;     // rows of a streamed (B) tile = MMA N
constexpr int kThreads = 576;        // producer warp + MMA warp + 16 softmax warps
constexpr uint64_t kDefaultWaitNs = 1000000000ull;  // 1 s per on-chip wait

// The standalone attention passes (CTA pairs) and the keep mask launch as
// programmatic dependents of the kernel before them in the stream.
#ifndef KVPOP_PDL_PASSES
#define KVPOP_PDL_PASSES 1
#endif

// Work items ordered longest first.  An item is (level, sequence, head); all
// items of one level cost (nearly) the same, so walking the levels from the
// top gives a sorted list without sorting on the device.
//   level_base[k] = index of the first item of level n_levels-1-k
//   seq_start/seq_len: sequences sorted by tile count, descending (those
//   active at level l form a prefix of this list).
struct LevelSchedule {
  int32_t n_levels;
  int32_t n_seqs;
  int32_t n_heads;
  int32_t total_items;
  int32_t level_base[kMaxLevels + 1];
  int32_t seq_start[kMaxSeqs];
  int32_t seq_len[kMaxSeqs];
};

struct AttnParams {
  CUtensorMap tmap_q;     // bf16 [T, H_q * d], box {64, rows}
  CUtensorMap tmap_k;     // bf16 [T, H_kv * d], box {64, rows}
  CUtensorMap tmap_rows;  // CTA pairs, pass 2: normaliser rows [H_q][T][8 x bf16], box {8, 128, 1}
  const uint16_t* q;      // bf16 [T, H_q, d] (pass 1's exact-max fallback reads scores from it)
  const uint16_t* k;      // bf16 [T, H_kv, d]
  void* nrm_rows;         // normaliser rows [H_q, T] x 16 bytes: pass 2 reads them, pass 1
                          // writes them when non-null (next to lse)
  float* out;             // pass 1: lse [H_q, T]; pass 2: target [H_kv, T]
  int32_t* status;
  uint64_t wait_ns;
  int32_t total_tokens;
  int32_t n_q_heads;
  int32_t n_kv_heads;
  int32_t group;
  int32_t window;
  float scale_log2;       // softmax scale * log2(e)
  float inv_scale;        // 1 / softmax scale (pass 2 normaliser slab)
  int32_t g_split;        // pass 2: 1 = an item covers the G query heads; G = one query head per item
  int32_t cta;            // 1: one CTA per item (128-row blocks); 2: a CTA pair per item (256-row blocks)
  int32_t* dbg;           // debug build: bounds-check word (kvpop_debug_set_word), else unused
  LevelSchedule sched;
};

// Both attention passes in one launch.  attn holds pass 1 (its tensor maps,
// schedule, lse output and the normaliser rows it writes, which pass 2
// reads); pass 2 has its own maps (A = 128 key rows, B = 256 query rows)
// and schedule.  flags counts, per (query head, 128-row tile of a sequence),
// the pass-1 warps that have written that tile's lse and rows; it, done and
// lse_done are zero on entry and zero again when the launch completes.
struct FusedParams {
  AttnParams attn;
  CUtensorMap tmap_q_stream;   // pass 2 B operand: Q, box {64, 256}
  CUtensorMap tmap_k_tile;     // pass 2 A operand: K, box {64, 128}
  LevelSchedule sched_target;
  float* target;               // [H_kv, T]
  int32_t* flags;              // [H_q, n_flag_tiles]
  int32_t* done;               // CTAs that have finished
  int32_t* lse_done;           // softmax warps that have finished pass 1
  int32_t n_flag_tiles;        // sum over sequences of ceil(L / 128)
  int32_t n_flags;             // H_q * n_flag_tiles
  int32_t tile_base_lse[kMaxSeqs];     // first flag tile of each sequence, in pass-1 schedule order
  int32_t tile_base_target[kMaxSeqs];  // the same in pass-2 schedule order
};

struct KeepParams {
  const float* score;     // [H_kv, T]
  uint8_t* keep;          // [H_kv, T]
  int32_t* dbg;           // debug build: bounds-check word, else unused
  int32_t key_cap;        // keys of one slice the shared-memory cache holds (set by the launcher)
  int32_t total_tokens;
  int32_t window;
  int32_t sinks;
  int32_t n_seqs;
  int32_t seq_start[kMaxSeqs];
  int32_t seq_len[kMaxSeqs];
  int32_t budget[kMaxSeqs];
};

}  // namespace kvpop
