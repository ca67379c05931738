// Parameter blocks of the kernels downstream of the keep mask: prefix top-k
// thresholds, static-cache compaction and decode attention.  Passed by value
// as __grid_constant__ kernel parameters, like those in kvpop_sched.h.
#pragma once
#include <stdint.h>

#include "kvpop_sched.h"

namespace kvpop {

struct ThresholdParams {
  const float* score;     // [H_kv, T]
  float* thr_score;       // [H_kv, T]
  int32_t* thr_pos;       // [H_kv, T]
  int32_t* dbg;           // debug build: bounds-check word, else unused
  int32_t total_tokens;
  int32_t window;
  int32_t sinks;
  int32_t n_seqs;
  int32_t seq_start[kMaxSeqs];
  int32_t seq_len[kMaxSeqs];
  int32_t budget[kMaxSeqs];
};

struct CompactParams {
  const uint16_t* k;        // bf16 [T, H_kv, d]
  const uint16_t* v;
  const uint8_t* keep;      // [H_kv, T]
  uint16_t* k_cache;        // bf16 [B, H_kv, C, d]
  uint16_t* v_cache;
  int32_t* pos;             // [B, H_kv, C]
  int32_t* count;           // [B, H_kv]
  int32_t* dbg;             // debug build: bounds-check word, else unused
  int32_t total_tokens, n_kv_heads, head_dim, capacity;
  int32_t n_seqs;
  int32_t seq_start[kMaxSeqs];
  int32_t seq_len[kMaxSeqs];
};

struct DecodeParams {
  const uint16_t* q;        // bf16 [B, H_q, d]
  const uint16_t* k_cache;  // bf16 [B, H_kv, C, d]
  const uint16_t* v_cache;
  const int32_t* count;     // [B, H_kv]
  float* partial;           // workspace [B, H_q, n_split, d + 2]: o[d], m, l
  float* out;               // [B, H_q, d]
  float* lse;               // [B, H_q] (may be null)
  int32_t* dbg;             // debug build: bounds-check word, else unused
  int32_t n_q_heads, n_kv_heads, head_dim, capacity, n_split;
  float scale_log2;
};

constexpr int kCompactSlots = 128;     // cache slots per compaction CTA
constexpr int kDecSplit = 128;         // cache slots per decode CTA (32 per warp)

}  // namespace kvpop
