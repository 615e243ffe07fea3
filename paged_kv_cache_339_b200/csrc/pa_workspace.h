// Layout of the caller-provided decode workspace (shared by host and device
// code). All offsets are multiples of 256 bytes from the workspace start.
//
//   [header 256 B][work pairs][splits per sequence][split sequences]
//   [merge counters][group list][partial (m, l)][partial o]
//
// The header holds the device status word (first 4 bytes), the work counter
// the persistent decode kernels claim items from, and the plan the planning
// kernel chose (split size, number of items). A merge counter per
// (sequence, KV head) counts the finished pieces of a split sequence: the
// CUDA-core kernel's last piece to finish merges them, the tensor-core
// kernel's merge tasks wait for the count. Partial results are indexed
// [sequence][query head][split].
#pragma once

#include <stddef.h>
#include <stdint.h>

namespace pa {

struct WsHeader {
  int32_t status;        // 0 = ok, else a pa_status code raised on the device
  int32_t work_counter;  // next unclaimed work item (reset by the plan kernel)
  int32_t num_items;     // work pairs x KV heads
  int32_t num_pairs;     // (sequence, split) pairs
  int32_t split_tokens;  // tokens per split chosen for this call
  int32_t max_splits;    // split capacity per sequence in this workspace
  int32_t num_split_seqs;  // sequences cut into more than one piece
  int32_t merge_counter;   // next unclaimed merge task (tensor-core kernel)
  int32_t num_group_items;     // group list entries x KV heads (shared prefixes)
  int32_t group_work_counter;  // next unclaimed group item
  int32_t reserved[54];
};
static_assert(sizeof(WsHeader) == 256, "header is 256 bytes");

// Hard cap on splits per sequence for an explicit split size.
constexpr int32_t kMaxSplits = 256;
// With an automatic split, at most this many splits per sequence ...
constexpr int32_t kAutoMaxSplits = 64;
// ... and never fewer than this many tokens per split.
constexpr int32_t kAutoMinSplit = 256;
// Automatic split sizes are multiples of this (one tensor-core chunk).
constexpr int32_t kAutoSplitQuantum = 128;

inline size_t align256(size_t x) { return (x + 255) / 256 * 256; }

inline int32_t ceil_div(int64_t a, int64_t b) {
  return static_cast<int32_t>((a + b - 1) / b);
}

// Smallest split the automatic choice may pick for this maximum context.
inline int32_t auto_min_split(int32_t max_ctx) {
  int64_t s = (static_cast<int64_t>(max_ctx) + kAutoMaxSplits - 1) / kAutoMaxSplits;
  s = (s + kAutoSplitQuantum - 1) / kAutoSplitQuantum * kAutoSplitQuantum;
  return static_cast<int32_t>(s < kAutoMinSplit ? kAutoMinSplit : s);
}

struct WsLayout {
  int32_t max_splits;
  size_t pairs_off, nsplit_off, split_off, cnt_off, gpairs_off, ml_off, o_off, total;
};

inline WsLayout ws_layout(int32_t num_seqs, int32_t num_q_heads,
                          int32_t head_dim, int32_t max_ctx,
                          int32_t split_tokens) {
  WsLayout w;
  const int32_t s = split_tokens > 0 ? split_tokens : auto_min_split(max_ctx);
  int32_t ms = max_ctx > 0 ? ceil_div(max_ctx, s) : 1;
  if (ms < 1) ms = 1;
  w.max_splits = ms;
  const size_t B = static_cast<size_t>(num_seqs > 0 ? num_seqs : 0);
  const size_t H = static_cast<size_t>(num_q_heads > 0 ? num_q_heads : 0);
  const size_t D = static_cast<size_t>(head_dim > 0 ? head_dim : 0);
  size_t off = 256;
  w.pairs_off = off;
  off += align256(B * ms * 16);
  w.nsplit_off = off;
  off += align256(B * 4);
  w.split_off = off;   // the sequences cut into more than one piece
  off += align256(B * 4);
  w.cnt_off = off;   // merge counters [sequence][KV head] (KV heads <= query heads)
  off += align256(B * H * 4);
  w.gpairs_off = off;   // the group list: at most one entry per (sequence, piece)
  off += align256(B * ms * 16);
  w.ml_off = off;
  off += align256(B * H * ms * 8);
  w.o_off = off;
  off += align256(B * H * ms * D * 4);
  w.total = off;
  return w;
}

}  // namespace pa
