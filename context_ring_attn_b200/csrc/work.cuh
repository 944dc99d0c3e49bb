// Work description shared by the two partial-attention kernels.
//
// One launch computes several ring blocks (method page, section 3: at ring
// step t every rank computes one block of its query shard against the KV
// shard it holds). A block's query shard is a list of ranges; each
// (block, query range) pair becomes a "segment" of query tiles, and each CTA
// computes one query tile of one KV head against every visible KV tile of the
// block's KV ranges. The table travels as a kernel parameter, so the launch
// needs no device-side setup and no allocation.
#pragma once

#include <stdint.h>

#include "cp_attn.h"

namespace cpk {

constexpr int kMaxRanges = 384;
constexpr int kMaxSegs = 320;

struct WorkSeg {
  int32_t q_range;   // index into WorkTable::ranges
  int32_t kv_begin;  // first KV range (index into WorkTable::ranges)
  int32_t kv_count;
  int32_t n_tiles;   // query tiles in the range
  int64_t out_row0;  // output row = out_row0 + Q buffer row
};

struct WorkTable {
  int32_t n_segs;
  int32_t total_tiles;
  int32_t tile_prefix[kMaxSegs + 1];
  WorkSeg segs[kMaxSegs];
  cp_range ranges[kMaxRanges];
};

// The KV tiles a query tile visits, in order: KV ranges of the block in
// order, then 128-key tiles within each range. Tiles past the last visible key
// are never visited.
struct KvTile {
  int64_t key_row0;  // first K/V buffer row of the tile
  int64_t key_pos0;  // its position
  int32_t n_valid;   // keys of the tile that exist and may be visible
  int32_t need_mask; // 1: some (row, key) pair of the tile is hidden
};

// Visible keys of range `kr` for a query tile whose token positions are
// q_pos_lo..q_pos_hi (same sequence assumed checked by the caller).
__host__ __device__ inline int64_t visible_keys(const cp_range& kr, int64_t q_pos_hi, int causal) {
  if (!causal) return kr.len;
  int64_t n = q_pos_hi - kr.pos0 + 1;
  if (n < 0) n = 0;
  if (n > kr.len) n = kr.len;
  return n;
}

// Locate blockIdx.x in the table: segment index and tile index in the segment.
// Tiles of a segment run from the last (most keys under a causal mask) to the
// first.
__device__ inline void locate_tile(const WorkTable& wt, int32_t cta, int32_t& seg, int32_t& tile) {
  int lo = 0, hi = wt.n_segs - 1;
  while (lo < hi) {  // last segment with tile_prefix[s] <= cta
    const int mid = (lo + hi + 1) >> 1;
    if (wt.tile_prefix[mid] <= cta) lo = mid; else hi = mid - 1;
  }
  seg = lo;
  tile = wt.segs[lo].n_tiles - 1 - (cta - wt.tile_prefix[lo]);
}

}  // namespace cpk
