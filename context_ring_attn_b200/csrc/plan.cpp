// Host planning for context-parallel ring attention: the load-balanced shard
// plan, the pass-KV / pass-Q ring schedules, mask classes of range pairs and
// the communication a real ring would need.
//
// Method: "Context Parallelism for Scalable Million-Token Inference", section 3
// (ring pass-KV / pass-Q, communication model) and section 4 (load-balanced
// sharding: 2N chunks, rank i holds chunks i and 2N-1-i).
#include <cstdint>
#include <cstring>
#include <vector>

#include "cp_attn.h"

namespace {

bool segs_ok(const cp_segment* segs, int32_t n_seg) {
  if (n_seg < 0 || (n_seg > 0 && !segs)) return false;
  for (int32_t i = 0; i < n_seg; ++i) {
    const cp_segment& s = segs[i];
    if (s.len < 0 || s.row0 < 0 || s.pos0 < 0 || s.reserved != 0) return false;
  }
  return true;
}

// Boundary c of a segment of length len cut into n_chunks pieces.
inline int64_t chunk_edge(int64_t len, int64_t c, int64_t n_chunks) {
  // c*len fits easily in int64 for any realistic length (< 2^40 tokens).
  return (c * len) / n_chunks;
}

void rank_chunk_ids(int32_t rank, int32_t n_ranks, cp_shard_mode mode, int32_t out[2]) {
  if (mode == CP_SHARD_LOAD_BALANCED) {
    out[0] = rank;
    out[1] = 2 * n_ranks - 1 - rank;
  } else {
    out[0] = 2 * rank;
    out[1] = 2 * rank + 1;
  }
}

void ranges_of_rank(const cp_segment* segs, int32_t n_seg, int32_t n_ranks, cp_shard_mode mode,
                    int32_t rank, std::vector<cp_range>& out) {
  int32_t ids[2];
  rank_chunk_ids(rank, n_ranks, mode, ids);  // already ascending in both modes
  const int64_t n_chunks = 2 * static_cast<int64_t>(n_ranks);
  for (int32_t s = 0; s < n_seg; ++s) {
    for (int c : ids) {
      const int64_t a = chunk_edge(segs[s].len, c, n_chunks);
      const int64_t b = chunk_edge(segs[s].len, c + 1, n_chunks);
      if (b > a) {
        cp_range r;
        r.row0 = segs[s].row0 + a;
        r.pos0 = segs[s].pos0 + a;
        r.len = b - a;
        r.seq = segs[s].seq;
        r.reserved = 0;
        out.push_back(r);
      }
    }
  }
}

// Visible (query, key) pairs of two ranges under the causal rule key <= query.
int64_t pair_count(const cp_range& q, const cp_range& k, bool causal) {
  if (q.seq != k.seq || q.len <= 0 || k.len <= 0) return 0;
  if (!causal) return q.len * k.len;
  const int64_t q_lo = q.pos0, q_hi = q.pos0 + q.len - 1;
  const int64_t k_lo = k.pos0, k_hi = k.pos0 + k.len - 1;
  int64_t total = 0;
  // queries inside the key span see (p - k_lo + 1) keys
  const int64_t a = q_lo > k_lo ? q_lo : k_lo;
  const int64_t b = q_hi < k_hi ? q_hi : k_hi;
  if (a <= b) total += (b - a + 1) * (a + b - 2 * k_lo + 2) / 2;
  // queries past the key span see all of it
  const int64_t c = q_lo > k_hi + 1 ? q_lo : k_hi + 1;
  if (c <= q_hi) total += (q_hi - c + 1) * k.len;
  return total;
}

}  // namespace

extern "C" {

const char* cp_status_string(cp_status s) {
  switch (s) {
    case CP_OK: return "ok";
    case CP_ERR_INVALID_ARG: return "invalid argument";
    case CP_ERR_UNSUPPORTED: return "unsupported configuration";
    case CP_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case CP_ERR_CUDA: return "CUDA call failed";
    case CP_ERR_TIMEOUT: return "device-side wait timed out";
    case CP_ERR_INTERNAL: return "device-side consistency check failed";
  }
  return "unknown status";
}

int32_t cp_abi_version(void) { return CP_ABI_VERSION; }

cp_status cp_shard_plan(const cp_segment* segs, int32_t n_seg, int32_t n_ranks,
                        cp_shard_mode mode, int64_t* chunk_bounds, int64_t* rank_rows,
                        int64_t* token_index, int64_t* sizes_out) {
  if (n_ranks < 1 || !segs_ok(segs, n_seg)) return CP_ERR_INVALID_ARG;
  if (mode != CP_SHARD_LOAD_BALANCED && mode != CP_SHARD_CONTIGUOUS) return CP_ERR_INVALID_ARG;
  const int64_t n_chunks = 2 * static_cast<int64_t>(n_ranks);
  if (sizes_out) {
    int64_t tokens = 0;
    for (int32_t s = 0; s < n_seg; ++s) tokens += segs[s].len;
    sizes_out[0] = static_cast<int64_t>(n_seg) * (n_chunks + 1);
    sizes_out[1] = static_cast<int64_t>(n_ranks) + 1;
    sizes_out[2] = tokens;
  }
  if (chunk_bounds) {
    for (int32_t s = 0; s < n_seg; ++s)
      for (int64_t c = 0; c <= n_chunks; ++c)
        chunk_bounds[s * (n_chunks + 1) + c] = chunk_edge(segs[s].len, c, n_chunks);
  }
  int64_t cursor = 0;
  if (rank_rows) rank_rows[0] = 0;
  std::vector<cp_range> mine;
  for (int32_t r = 0; r < n_ranks; ++r) {
    mine.clear();
    ranges_of_rank(segs, n_seg, n_ranks, mode, r, mine);
    for (const cp_range& rg : mine) {
      if (token_index)
        for (int64_t i = 0; i < rg.len; ++i) token_index[cursor + i] = rg.row0 + i;
      cursor += rg.len;
    }
    if (rank_rows) rank_rows[r + 1] = cursor;
  }
  return CP_OK;
}

cp_status cp_rank_ranges(const cp_segment* segs, int32_t n_seg, int32_t n_ranks,
                         cp_shard_mode mode, int32_t rank, cp_range* out, int32_t* n_out) {
  if (n_ranks < 1 || rank < 0 || rank >= n_ranks || !segs_ok(segs, n_seg) || !n_out)
    return CP_ERR_INVALID_ARG;
  if (mode != CP_SHARD_LOAD_BALANCED && mode != CP_SHARD_CONTIGUOUS) return CP_ERR_INVALID_ARG;
  std::vector<cp_range> mine;
  ranges_of_rank(segs, n_seg, n_ranks, mode, rank, mine);
  *n_out = static_cast<int32_t>(mine.size());
  if (out && !mine.empty()) std::memcpy(out, mine.data(), mine.size() * sizeof(cp_range));
  return CP_OK;
}

cp_status cp_ring_schedule(const cp_segment* q_segs, int32_t n_q_seg,
                           const cp_segment* kv_segs, int32_t n_kv_seg, int32_t n_ranks,
                           cp_shard_mode mode, cp_ring_variant variant, cp_range* ranges,
                           int32_t ranges_cap, int32_t* n_ranges, cp_block* blocks,
                           int32_t* block_part) {
  if (n_ranks < 1 || !segs_ok(q_segs, n_q_seg) || !segs_ok(kv_segs, n_kv_seg)) return CP_ERR_INVALID_ARG;
  if (mode != CP_SHARD_LOAD_BALANCED && mode != CP_SHARD_CONTIGUOUS) return CP_ERR_INVALID_ARG;
  if (variant != CP_PASS_KV && variant != CP_PASS_Q) return CP_ERR_INVALID_ARG;
  if (!ranges || !n_ranges || !blocks || ranges_cap < 0) return CP_ERR_INVALID_ARG;
  std::vector<cp_range> all;
  std::vector<int32_t> q_off(n_ranks + 1), kv_off(n_ranks + 1);
  for (int32_t r = 0; r < n_ranks; ++r) {
    q_off[r] = static_cast<int32_t>(all.size());
    ranges_of_rank(q_segs, n_q_seg, n_ranks, mode, r, all);
  }
  q_off[n_ranks] = static_cast<int32_t>(all.size());
  for (int32_t r = 0; r < n_ranks; ++r) {
    kv_off[r] = static_cast<int32_t>(all.size());
    ranges_of_rank(kv_segs, n_kv_seg, n_ranks, mode, r, all);
  }
  kv_off[n_ranks] = static_cast<int32_t>(all.size());
  if (static_cast<int64_t>(all.size()) > ranges_cap) return CP_ERR_INVALID_ARG;
  std::memcpy(ranges, all.data(), all.size() * sizeof(cp_range));
  *n_ranges = static_cast<int32_t>(all.size());
  for (int32_t t = 0; t < n_ranks; ++t) {
    for (int32_t i = 0; i < n_ranks; ++i) {
      const int32_t other = ((i - t) % n_ranks + n_ranks) % n_ranks;
      int32_t qr, kr, part;
      if (variant == CP_PASS_KV) {
        qr = i; kr = other; part = t;
      } else {
        kr = i; qr = other; part = i;
      }
      cp_block& b = blocks[t * n_ranks + i];
      b.q_begin = q_off[qr];
      b.q_count = q_off[qr + 1] - q_off[qr];
      b.kv_begin = kv_off[kr];
      b.kv_count = kv_off[kr + 1] - kv_off[kr];
      b.out_row0 = 0;
      if (block_part) block_part[t * n_ranks + i] = part;
    }
  }
  return CP_OK;
}

cp_pair_class cp_classify_pair(const cp_range* q, const cp_range* kv, int32_t causal) {
  if (!q || !kv || q->seq != kv->seq || q->len <= 0 || kv->len <= 0) return CP_PAIR_SKIP;
  if (!causal) return CP_PAIR_FULL;
  const int64_t q_lo = q->pos0, q_hi = q->pos0 + q->len - 1;
  const int64_t k_lo = kv->pos0, k_hi = kv->pos0 + kv->len - 1;
  if (k_lo > q_hi) return CP_PAIR_SKIP;
  if (k_hi <= q_lo) return CP_PAIR_FULL;
  return CP_PAIR_PARTIAL;
}

int64_t cp_block_pairs(const cp_range* ranges, const cp_block* block, int32_t causal) {
  if (!ranges || !block) return -1;
  int64_t total = 0;
  for (int32_t a = 0; a < block->q_count; ++a)
    for (int32_t b = 0; b < block->kv_count; ++b)
      total += pair_count(ranges[block->q_begin + a], ranges[block->kv_begin + b], causal != 0);
  return total;
}

cp_status cp_ring_comm_volume(const cp_range* ranges, const cp_block* blocks, int32_t n_ranks,
                              cp_ring_variant variant, int32_t n_h, int32_t n_kv, int32_t d,
                              int64_t* hop_elems, int64_t* total, int64_t* all_to_all) {
  if (!ranges || !blocks || n_ranks < 1 || n_h < 1 || n_kv < 1 || d < 1) return CP_ERR_INVALID_ARG;
  if (variant != CP_PASS_KV && variant != CP_PASS_Q) return CP_ERR_INVALID_ARG;
  int64_t sum = 0, a2a = 0;
  for (int32_t t = 1; t < n_ranks; ++t) {
    for (int32_t i = 0; i < n_ranks; ++i) {
      const cp_block& b = blocks[t * n_ranks + i];
      int64_t q_rows = 0, kv_rows = 0;
      for (int32_t j = 0; j < b.q_count; ++j) q_rows += ranges[b.q_begin + j].len;
      for (int32_t j = 0; j < b.kv_count; ++j) kv_rows += ranges[b.kv_begin + j].len;
      const int64_t e = (variant == CP_PASS_KV) ? kv_rows * n_kv * d : q_rows * n_h * d;
      if (hop_elems) hop_elems[(t - 1) * n_ranks + i] = e;
      sum += e;
      if (variant == CP_PASS_Q) a2a += q_rows * n_h * (static_cast<int64_t>(d) + 1);
    }
  }
  if (total) *total = sum;
  if (all_to_all) *all_to_all = a2a;
  return CP_OK;
}

// Algorithm 1 of the method page (section 3): pass-KV when the KV-cache miss
// rate T/(T+P) is above 2*N_KV/N_H, or when one ring hop's SendRecv of a KV
// shard ((T+P)/N tokens of K and V) hides under one ring step of attention;
// pass-Q otherwise.
cp_status cp_select_ring_variant(int64_t t, int64_t p, int32_t n_h, int32_t n_kv, int32_t d, int32_t n_ranks,
                                 int32_t elem_bytes, double link_bytes_per_s, double step_attn_s,
                                 cp_ring_variant* variant, int32_t* reason) {
  if (!variant || t < 0 || p < 0 || t + p == 0 || n_h < 1 || n_kv < 1 || n_h % n_kv || d < 1 || n_ranks < 1 ||
      elem_bytes < 1 || !(link_bytes_per_s > 0.0) || !(step_attn_s >= 0.0))
    return CP_ERR_INVALID_ARG;
  const double miss = static_cast<double>(t) / static_cast<double>(t + p);
  const double threshold = 2.0 * static_cast<double>(n_kv) / static_cast<double>(n_h);
  int32_t why = 0;
  if (miss > threshold) {
    why = 1;
  } else {
    const double hop_bytes = static_cast<double>(t + p) / n_ranks * n_kv * d * 2.0 * elem_bytes;
    if (hop_bytes / link_bytes_per_s <= step_attn_s) why = 2;
  }
  *variant = why ? CP_PASS_KV : CP_PASS_Q;
  if (reason) *reason = why;
  return CP_OK;
}

}  // extern "C"
