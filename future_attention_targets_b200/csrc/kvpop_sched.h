// Kernel parameter blocks shared by the host launchers and the kernels.
#pragma once

#include <cuda.h>
#include <stdint.h>

namespace kvpop {

constexpr int kMaxSeqs = 512;        // sequences per call
constexpr int kTileRows = 128;       // rows of the resident (A) tile = MMA M
constexpr int kMaxLevels = 1024;     // longest sequence = kMaxLevels * kTileRows tokens
constexpr int kStreamRows = 256;     // rows of a streamed (B) tile = MMA N
constexpr int kThreads = 320;        // producer warp + MMA warp + 8 softmax warps
constexpr uint64_t kDefaultWaitNs = 1000000000ull;  // 1 s per on-chip wait

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
  const float* lse_in;    // pass 2: [H_q, T]
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
  LevelSchedule sched;
};

struct KeepParams {
  const float* score;     // [H_kv, T]
  uint8_t* keep;          // [H_kv, T]
  int32_t total_tokens;
  int32_t window;
  int32_t sinks;
  int32_t n_seqs;
  int32_t seq_start[kMaxSeqs];
  int32_t seq_len[kMaxSeqs];
  int32_t budget[kMaxSeqs];
};

}  // namespace kvpop
