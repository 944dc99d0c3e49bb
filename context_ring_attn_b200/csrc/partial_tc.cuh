// Partial attention of ring blocks on the 5th-generation tensor cores
// (tcgen05 MMA with TMEM accumulators, TMA-staged bf16 operands).
//
// Method: "Context Parallelism for Scalable Million-Token Inference",
// section 3 (ring pass-KV / pass-Q: each rank computes the attention of a
// query shard against one KV shard; the results are later merged by LSE).
// Within a block the softmax is taken online over 128-key tiles (blockwise
// exact attention, "Context Parallelism과 Expert Parallelism" section 4.1), so
// the block yields O normalised within the block plus its log-sum-exp.
//
// One CTA = two 128-row query tiles (a, b) of one KV head. GQA packing: each
// tile's rows are (token, head-in-group) pairs, 128/G tokens x G query heads
// that share the KV head (section 8.2 of the GQA page), so every K/V tile is
// loaded once for 2 x 128 rows. Warp roles (576 threads):
//   warps 0-7  softmax of tile a, warps 8-15 softmax of tile b. Two threads
//              per row: warps w and w+4 read the same TMEM lane quarter, one
//              the 64 columns 0-63 of the row, the other 64-127. Per KV tile
//              each reads its half of the S row from TMEM, masks by global
//              position, exchanges its half-row max with its partner through
//              shared memory (a 64-thread named barrier), writes its P half
//              (bf16 pairs) over the S row in TMEM, keeps its own part of the
//              row sum, and rescales its half of the O row when the running
//              max grows by more than 2^8; at the end the two sums are added
//              and each thread writes half of the normalised O row;
//   warp 16    TMA producers: lane 0 loads Q, then K tiles into a 3-stage
//              ring; lane 1 loads V tiles into a 2-stage ring;
//   warp 17    MMA issuer (one thread) and TMEM owner. Per KV tile j it issues
//              O_a += P_a(j) V_j, S_a(j+1) = Q_a K_{j+1}^T, O_b += P_b(j) V_j,
//              S_b(j+1) = Q_b K_{j+1}^T, so that one tile's softmax always
//              overlaps the other tile's MMAs (ping-pong).
// Two threads per row halve the latency of a softmax step, which otherwise
// exceeds the MMA time of one tile and stalls the ping-pong.
// Head dims 64 and 128 are two instantiations (a row is HD/64 swizzle columns
// of 64 bf16; S = Q K^T takes HD/16 MMA steps and O has HD columns).
// TMEM (512 columns): S_a 0, S_b 128, O_a 256, O_b 384. Each half row's P
// (bf16 pairs) goes over the first 32 of its own 64 S columns. tcgen05 operations of one thread complete in issue order, so the
// completion of S_x(j+1) also means O_x += P_x(j) V_j has completed.
#pragma once

#include "common.cuh"
#include "work.cuh"

namespace cpk {
namespace tc {

constexpr int BM = 128;                      // packed query rows per tile
constexpr int BN = 128;                      // keys per KV tile
constexpr int kQTiles = 2;                   // query tiles per CTA
constexpr int kHalfBytes = 128 * 128;        // 128 rows x 64 bf16 (one 128-byte swizzle column)
constexpr int kSoftmaxWarps = 16;
constexpr int kProducerWarp = 16;
constexpr int kMmaWarp = 17;
constexpr int kThreads = 576;
constexpr int kNumBars = 24;
constexpr int kSmemMax = 232448;                     // 227 KB per block on sm_100
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0;     // + tile * 128
constexpr uint32_t kColO = 256;   // + tile * 128 (HD columns used)
constexpr float kRescaleThreshold = 8.0f;  // log2 units: O is rescaled when the max grows by > 2^8
constexpr int kPolyPairsPer8 = 1;          // of every 8 column pairs, this many take the polynomial exp2

// Shared-memory plan of a head dim HD (64 or 128): a Q, K or V tile of 128
// rows is HD/64 swizzle columns of 16 KB each.
template <int HD>
struct Cfg {
  static constexpr int kHalves = HD / 64;
  static constexpr int kTileBytes = kHalves * kHalfBytes;   // 128 rows x HD bf16
  static constexpr int kKStages = 3;
  static constexpr int kVStages = HD == 128 ? 2 : 3;
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kOffQ + kQTiles * kTileBytes;
  static constexpr int kOffV = kOffK + kKStages * kTileBytes;
  static constexpr int kOffBar = kOffV + kVStages * kTileBytes;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kOffXch = kOffMisc + 16;           // [tile][half][row] f32: half-row max, then sum
  static constexpr int kSmemNeeded = kOffXch + kQTiles * 2 * BM * 4;
  // The dynamic shared window starts 1024-aligned in practice; whatever slack is
  // left covers a smaller alignment, and the kernel checks it at run time.
  static constexpr int kSmemBytes = kSmemNeeded + 1024 <= kSmemMax ? kSmemNeeded + 1024 : kSmemMax;
  static_assert(kSmemNeeded <= kSmemMax, "shared memory plan exceeds 227 KB");
  static_assert(kKStages <= 3 && kVStages <= 3, "barrier slots hold at most 3 stages");
  // Epilogue staging of a tile's output rows (fp32, rows padded by 16 bytes so
  // that the per-row writes of a quarter warp hit distinct bank groups), over
  // the Q and K regions, which no MMA or load touches any more by then.
  static constexpr int kStageRow = HD * 4 + 16;
  static constexpr int kStageTile = BM * kStageRow;
  static_assert(kQTiles * kStageTile <= kOffV, "epilogue staging must stay clear of the V stages");
};

// barrier slots
enum {
  B_Q_FULL = 0,
  B_K_FULL = 1,     // +stage (3)
  B_K_EMPTY = 4,    // +stage (3)
  B_V_FULL = 7,     // +stage (3)
  B_V_EMPTY = 10,   // +stage (3)
  B_S_FULL = 13,    // +tile: S_x(j) is in TMEM (and O_x += P_x(j-1) V is done)
  B_P_FULL = 15,    // +tile (8 arrivals): P_x(j) is in TMEM
  B_O_DONE = 17,    // +tile: O_x += P_x(j) V_j has completed
  B_DRAIN = 19
};

struct Params {
  CUtensorMap tm_q;  // [q_rows][N_KV][G][HD] bf16, box {64, G, 1, 128/G}
  CUtensorMap tm_k;  // [kv_rows][N_KV][HD] bf16, box {64, 1, 128}
  CUtensorMap tm_v;
  float* o_part;
  float* lse_part;
  __nv_bfloat16* out_final;   // not null: write the merged, normalised row here (bf16) instead of o_part
  int32_t accumulate;         // merge each row into the (O, LSE) already at its place in o_part / lse_part
  uint32_t* status;
  int32_t n_h;
  int32_t log2_group;
  int32_t causal;
  float scale_log2;  // softmax scale * log2(e)
  WorkTable wt;      // tiles here are 256-row CTA tiles (two query tiles)
};

// Wait on a barrier with every lane of the warp; the outcome is made
// warp-uniform so warp-collective tcgen05 instructions stay converged.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile uint32_t* abort_flag,
                                          uint32_t* status) {
  const bool ok = mbar_wait(bar, parity, abort_flag, status);
  return __all_sync(0xffffffffu, ok);
}

// Wait used only while draining at exit: bounded by time alone.
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity, uint32_t* status) {
  const uint64_t t0 = globaltimer();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer() - t0 > kWaitBudgetNs) {
      if (status) atomicOr(status, kStatusTimeout);
      return;
    }
  }
}

// Exponentials of one half row (64 keys) for one KV tile: P = 2^(S*scale*log2e
// - m_use) as 32 bf16 pairs in registers (pk), returning the sum of the fp32
// values; nothing is written, so S stays in TMEM for a redo. S is read from
// TMEM 8 columns at a time, the next chunk in flight while this one is
// exponentiated. kPolyPairsPer8 of every 8 pairs take the polynomial on the
// FMA pipe, the rest the special function unit. kMasked: keys past `lim` are
// hidden and get exactly 0 (the polynomial or a large unmasked S would leave a
// value there); a separate instantiation keeps the compares out of the
// unmasked tiles. x_max receives the largest exponent S*scale*log2e - m_use
// over the visible keys.
template <bool kMasked>
__device__ __forceinline__ float half_row_exps(uint32_t s_col, float sl2, float m_use, int lim, uint32_t (&pk)[32],
                                               float& x_max) {
  float xm0 = -INFINITY, xm1 = -INFINITY;
  const uint64_t sl2_2 = f2_pack(sl2, sl2);
  const uint64_t negm_2 = f2_pack(-m_use, -m_use);
  uint64_t acc[2] = {0ull, 0ull};
  uint32_t sc[2][8];
  tmem_ld8(s_col, sc[0]);
  tmem_ld_wait();
#pragma unroll
  for (int h4 = 0; h4 < 8; ++h4) {
    if (h4 < 7) tmem_ld8(s_col + (h4 + 1) * 8, sc[(h4 + 1) & 1]);
    const uint32_t (&sv)[8] = sc[h4 & 1];
#pragma unroll
    for (int cc = 0; cc < 8; cc += 2) {
      const int c = h4 * 8 + cc;
      const uint64_t x2 = f2_fma(f2_pack(__uint_as_float(sv[cc]), __uint_as_float(sv[cc + 1])), sl2_2, negm_2);
      float x0, x1;
      f2_unpack(x2, x0, x1);
      if (kMasked) {
        const float v0 = (c > lim) ? -INFINITY : x0;
        const float v1 = (c + 1 > lim) ? -INFINITY : x1;
        if ((c >> 1) & 1) xm1 = fmax3(xm1, v0, v1);
        else xm0 = fmax3(xm0, v0, v1);
      } else {
        if ((c >> 1) & 1) xm1 = fmax3(xm1, x0, x1);
        else xm0 = fmax3(xm0, x0, x1);
      }
      uint64_t p2;
      if (((c >> 1) & 7) < kPolyPairsPer8) {
        p2 = exp2_poly_x2(x2);
      } else {
        p2 = f2_pack(ex2(x0), ex2(x1));
      }
      if (kMasked) {
        float p0, p1;
        f2_unpack(p2, p0, p1);
        if (c > lim) p0 = 0.0f;
        if (c + 1 > lim) p1 = 0.0f;
        p2 = f2_pack(p0, p1);
      }
      float p0, p1;
      f2_unpack(p2, p0, p1);
      pk[c >> 1] = pack_bf16x2(p0, p1);
      acc[(c >> 1) & 1] = f2_add(acc[(c >> 1) & 1], p2);
    }
    if (h4 < 7) tmem_ld_wait();
  }
  const uint64_t t = f2_add(acc[0], acc[1]);
  float lo, hi;
  f2_unpack(t, lo, hi);
  x_max = fmaxf(xm0, xm1);
  return lo + hi;
}

// 18 warps put five on two of the four schedulers, whose register files hold
// 16K registers each: at most 102 per thread, so 96.
template <int HD>
__global__ void __maxnreg__(96) partial_bf16_kernel(const __grid_constant__ Params p) {
  using C = Cfg<HD>;
  constexpr int kTileBytes = C::kTileBytes;
  constexpr int kKStages = C::kKStages;
  constexpr int kVStages = C::kVStages;
  constexpr int kOffQ = C::kOffQ, kOffK = C::kOffK, kOffV = C::kOffV, kOffBar = C::kOffBar;
  constexpr int kOffMisc = C::kOffMisc, kOffXch = C::kOffXch;
  constexpr int kSmemNeeded = C::kSmemNeeded, kSmemBytes = C::kSmemBytes;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  uint8_t* smem = smem_raw + pad;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffMisc);
  volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(smem + kOffMisc + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  if (pad + kSmemNeeded > kSmemBytes) {  // uniform across the CTA: nothing has started yet
    if (threadIdx.x == 0) atomicOr(p.status, kStatusInternal);
    return;
  }

  int32_t seg, tile;
  locate_tile(p.wt, blockIdx.x, seg, tile);
  const WorkSeg ws = p.wt.segs[seg];
  const cp_range qr = p.wt.ranges[ws.q_range];
  const int kvh = blockIdx.y;
  const int group = 1 << p.log2_group;
  const int tok_per_tile = BM >> p.log2_group;            // tokens per 128-row query tile
  const int64_t tok0 = static_cast<int64_t>(tile) * (kQTiles * tok_per_tile);
  const int n_tok = static_cast<int>(min(static_cast<int64_t>(kQTiles * tok_per_tile), qr.len - tok0));
  const int64_t q_row0 = qr.row0 + tok0;
  const int64_t q_pos_lo = qr.pos0 + tok0;
  const int64_t q_pos_hi = q_pos_lo + n_tok - 1;
  const int causal = p.causal;

  // KV tiles the CTA visits (enough for its last valid token)
  int n_iter = 0;
  for (int r = 0; r < ws.kv_count; ++r) {
    const cp_range kr = p.wt.ranges[ws.kv_begin + r];
    if (kr.seq != qr.seq) continue;
    n_iter += static_cast<int>((visible_keys(kr, q_pos_hi, causal) + BN - 1) / BN);
  }

  if (threadIdx.x == 0) {
    for (int i = 0; i < kNumBars; ++i) mbar_init(&bars[i], (i == B_P_FULL || i == B_P_FULL + 1) ? 8u : 1u);
    *abort_flag = 0u;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  if (warp == kProducerWarp && lane == 0) {
    prefetch_tensormap(&p.tm_q);
    prefetch_tensormap(&p.tm_k);
    prefetch_tensormap(&p.tm_v);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  uint8_t* sQ = smem + kOffQ;
  uint8_t* sK = smem + kOffK;
  uint8_t* sV = smem + kOffV;

  if (warp == kProducerWarp) {
    // ------------------------------------------------------------------ TMA producers
    if (lane < 2 && n_iter > 0) {
      const bool is_k = lane == 0;
      const int n_st = is_k ? kKStages : kVStages;
      uint8_t* base = is_k ? sK : sV;
      const CUtensorMap* map = is_k ? &p.tm_k : &p.tm_v;
      uint64_t* full = &bars[is_k ? B_K_FULL : B_V_FULL];
      uint64_t* empty = &bars[is_k ? B_K_EMPTY : B_V_EMPTY];
      uint32_t issued[3] = {0u, 0u, 0u};
      if (is_k) {
        mbar_arrive_expect_tx(&bars[B_Q_FULL], kQTiles * kTileBytes);
        for (int t = 0; t < kQTiles; ++t) {
          const int row = static_cast<int>(q_row0) + t * tok_per_tile;
#pragma unroll
          for (int h = 0; h < C::kHalves; ++h)
            tma_load_4d(sQ + t * kTileBytes + h * kHalfBytes, &p.tm_q, &bars[B_Q_FULL], h * 64, 0, kvh, row);
        }
      }
      int it = 0;
      bool ok = true;
      for (int r = 0; r < ws.kv_count && ok; ++r) {
        const cp_range kr = p.wt.ranges[ws.kv_begin + r];
        if (kr.seq != qr.seq) continue;
        const int64_t nv = visible_keys(kr, q_pos_hi, causal);
        for (int64_t k0 = 0; k0 < nv; k0 += BN, ++it) {
          const int st = it % n_st;
          const uint32_t ph = (it / n_st) & 1;
          const int key_row = static_cast<int>(kr.row0 + k0);
          if (it >= n_st && !mbar_wait(&empty[st], ph ^ 1u, abort_flag, p.status)) { ok = false; break; }
          mbar_arrive_expect_tx(&full[st], kTileBytes);
#pragma unroll
          for (int h = 0; h < C::kHalves; ++h)
            tma_load_3d(base + st * kTileBytes + h * kHalfBytes, map, &full[st], h * 64, kvh, key_row);
          issued[st] += 1;
        }
      }
      // Drain: every load issued has landed before the CTA may exit.
      if (is_k) drain_wait(&bars[B_Q_FULL], 0u, p.status);
      for (int st = 0; st < n_st; ++st)
        if (issued[st] > 0) drain_wait(&full[st], (issued[st] - 1u) & 1u, p.status);
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0 && n_iter > 0) {
      constexpr uint32_t idesc_s = umma_idesc_bf16(BM, BN, 0);   // Q, K both K-major
      constexpr uint32_t idesc_o = umma_idesc_bf16(BM, HD, 1);   // P (TMEM) K-major, V MN-major
      // Descriptors of the tile bases; an operand at byte offset `off` from a
      // base is base + off/16 (the 14-bit address field does not carry: every
      // shared address is below 256 KB).
      const uint64_t q_desc = umma_sdesc_sw128(smem_u32(sQ), 16, 1024);
      const uint64_t k_desc = umma_sdesc_sw128(smem_u32(sK), 16, 1024);
      const uint64_t v_desc = umma_sdesc_sw128(smem_u32(sV), kHalfBytes, 1024);
      auto issue_s = [&](int x, int i) {   // S_x(i) = Q_x K_i^T
        const uint64_t qd = q_desc + static_cast<uint64_t>((x * kTileBytes) >> 4);
        const uint64_t kd = k_desc + static_cast<uint64_t>(((i % kKStages) * kTileBytes) >> 4);
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) {
          const uint64_t off = static_cast<uint64_t>(((kk >> 2) * kHalfBytes + (kk & 3) * 32) >> 4);
          umma_bf16_ss(tmem + kColS + x * BN, qd + off, kd + off, idesc_s, kk > 0 ? 1u : 0u);
        }
        umma_commit(&bars[B_S_FULL + x]);
      };
      auto issue_pv = [&](int x, int j) {  // O_x += P_x(j) V_j
        const uint64_t vd = v_desc + static_cast<uint64_t>(((j % kVStages) * kTileBytes) >> 4);
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk) {
          // keys 16kk..16kk+15 as bf16 pairs: the P of each half sits in its own first 32 S columns
          const uint32_t p_addr = tmem + kColS + x * BN + (kk >> 2) * 64 + (kk & 3) * 8;
          umma_bf16_ts(tmem + kColO + x * 128, p_addr, vd + static_cast<uint64_t>((kk * 2048) >> 4), idesc_o,
                       (j > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit(&bars[B_O_DONE + x]);
      };
      bool ok = mbar_wait(&bars[B_Q_FULL], 0u, abort_flag, p.status) &&
                mbar_wait(&bars[B_K_FULL], 0u, abort_flag, p.status);
      if (ok) {
        tc_fence_after();
        issue_s(0, 0);
        issue_s(1, 0);
        umma_commit(&bars[B_K_EMPTY]);
      }
      for (int j = 0; j < n_iter && ok; ++j) {
        const bool more = j + 1 < n_iter;
        const int kn = (j + 1) % kKStages;
        if (!mbar_wait(&bars[B_V_FULL + j % kVStages], (j / kVStages) & 1, abort_flag, p.status)) { ok = false; break; }
        if (more && !mbar_wait(&bars[B_K_FULL + kn], ((j + 1) / kKStages) & 1, abort_flag, p.status)) { ok = false; break; }
        for (int x = 0; x < kQTiles; ++x) {
          if (!mbar_wait(&bars[B_P_FULL + x], j & 1, abort_flag, p.status)) { ok = false; break; }
          tc_fence_after();
          issue_pv(x, j);
          if (more) issue_s(x, j + 1);
        }
        if (!ok) break;
        umma_commit(&bars[B_V_EMPTY + j % kVStages]);
        if (more) umma_commit(&bars[B_K_EMPTY + kn]);
      }
      // Everything this thread issued completes before TMEM is released.
      umma_commit(&bars[B_DRAIN]);
      drain_wait(&bars[B_DRAIN], 0u, p.status);
    }
  } else {
    // ------------------------------------------------------------------ softmax warps 0..15
    const int x = warp >> 3;                // query tile of this warp
    const int hf = (warp >> 2) & 1;         // half of the row: columns hf*64 .. hf*64+63
    const int quarter = warp & 3;           // TMEM lane quarter
    const int row = quarter * 32 + lane;    // packed row within the tile
    const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t s_col = tmem + lane_base + kColS + x * BN + hf * 64;   // this thread's S columns
    const uint32_t o_col = tmem + lane_base + kColO + x * 128 + hf * (HD / 2);   // its O columns
    float* xch_mine = reinterpret_cast<float*>(smem + kOffXch) + (x * 2 + hf) * BM + row;
    const float* xch_peer = reinterpret_cast<const float*>(smem + kOffXch) + (x * 2 + (hf ^ 1)) * BM + row;
    const uint32_t pair_bar = 1 + x * 4 + quarter;   // named barrier of the two warps sharing these rows
    const int tok = x * tok_per_tile + (row >> p.log2_group);   // token within the CTA
    const bool row_valid = tok < n_tok;
    const int64_t qpos = q_pos_lo + tok;
    const float sl2 = p.scale_log2;
    float m_run = -INFINITY;
    float l_run = 0.0f;   // this thread's part of the row sum
    bool ok = true;
    int it = 0;

    for (int r = 0; r < ws.kv_count && ok; ++r) {
      const cp_range kr = p.wt.ranges[ws.kv_begin + r];
      if (kr.seq != qr.seq) continue;
      const int64_t nv = visible_keys(kr, q_pos_hi, causal);
      for (int64_t k0 = 0; k0 < nv; k0 += BN, ++it) {
        const int64_t kp0 = kr.pos0 + k0;
        const int n_valid = static_cast<int>(min(static_cast<int64_t>(BN), nv - k0));
        // S_x(it) is in TMEM; this also means O_x += P_x(it-1) V has completed
        const bool got = warp_wait(&bars[B_S_FULL + x], it & 1, abort_flag, p.status);
        // key hf*64 + c of the tile is visible iff c <= lim
        int lim = 63;
        if ((n_valid < BN) || (causal && kp0 + BN - 1 > qpos)) {
          int64_t l64 = n_valid - 1;
          if (causal && qpos - kp0 < l64) l64 = qpos - kp0;
          l64 -= hf * 64;
          lim = static_cast<int>(max(min(l64, static_cast<int64_t>(63)), static_cast<int64_t>(-1)));
        }
        const bool tile_masked = __any_sync(0xffffffffu, lim < 63);
        // Optimistic step: exponentiate against the running max m_run and track
        // the tile's largest exponent. The P written is final unless a row of
        // either half grew its max by more than 2^kRescaleThreshold, or has no
        // running max yet (a first visible tile), which both halves detect
        // alike (the two threads of a row hold the same m_run); then both take
        // the exact step below. The partners' row maxima (raw, log2 units) are
        // exchanged through shared memory before the vote.
        const bool first = __any_sync(0xffffffffu, m_run == -INFINITY);
        float raw_max = -INFINITY;   // max over visible keys of S*scale*log2e in this half row
        float sum = 0.0f;
        bool fine = false;
        uint32_t pk[32];             // P of this half row, bf16 pairs
        if (got) {
          tc_fence_after();
          if (first) {
            float a0 = -INFINITY, a1 = -INFINITY;
#pragma unroll
            for (int h16 = 0; h16 < 4; ++h16) {
              uint32_t sv[16];
              tmem_ld16(s_col + h16 * 16, sv);
              tmem_ld_wait();
#pragma unroll
              for (int cc = 0; cc < 16; cc += 4) {
                const int c = h16 * 16 + cc;
                const float v0 = (c > lim) ? -INFINITY : __uint_as_float(sv[cc]);
                const float v1 = (c + 1 > lim) ? -INFINITY : __uint_as_float(sv[cc + 1]);
                const float v2 = (c + 2 > lim) ? -INFINITY : __uint_as_float(sv[cc + 2]);
                const float v3 = (c + 3 > lim) ? -INFINITY : __uint_as_float(sv[cc + 3]);
                a0 = fmax3(a0, v0, v1);
                a1 = fmax3(a1, v2, v3);
              }
            }
            raw_max = fmaxf(a0, a1) * sl2;
          } else {
            float x_max;
            sum = tile_masked ? half_row_exps<true>(s_col, sl2, m_run, lim, pk, x_max)
                              : half_row_exps<false>(s_col, sl2, m_run, lim, pk, x_max);
            raw_max = x_max + m_run;
            fine = !(x_max > kRescaleThreshold);
          }
        }
        // Both warps of the pair always meet here once per KV tile and agree on
        // the outcome, so neither can wait alone. The peer reads this slot
        // before it arrives on P_FULL, and the next write comes after S_FULL,
        // which needs that arrival: no overwrite race.
        *xch_mine = raw_max;
        tc_fence_before();
        const bool all_fine = named_bar_and(pair_bar, 64, got && fine);
        tc_fence_after();
        float alpha = 1.0f;
        bool resc = false;
        if (!all_fine) {
          if (!named_bar_and(pair_bar, 64, got)) { ok = false; break; }
          // exact step: the row max over both halves; rescale if it grew past the threshold
          const float m_new = fmaxf(m_run, fmaxf(raw_max, *xch_peer));
          if (m_new > m_run + kRescaleThreshold) {
            alpha = ex2(m_run - m_new);
            m_run = m_new;
            resc = true;
          }
          const float m_use = (m_run == -INFINITY) ? 0.0f : m_run;
          float unused;
          sum = tile_masked ? half_row_exps<true>(s_col, sl2, m_use, lim, pk, unused)
                            : half_row_exps<false>(s_col, sl2, m_use, lim, pk, unused);
        }
        // P over the first 32 columns of this half row's S (read by the PV MMA)
        tmem_st32(s_col, pk);
        l_run = l_run * alpha + sum;
        // O_x holds every earlier PV (see S_FULL above): rescale this half in place if needed
        if (it > 0 && __any_sync(0xffffffffu, resc)) {
#pragma unroll 1
          for (int c = 0; c < HD / 32; ++c) {
            uint32_t o[16];
            tmem_ld16(o_col + c * 16, o);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 16; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
            tmem_st16(o_col + c * 16, o);
          }
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars[B_P_FULL + x]);
      }
    }

    // ---------------------------------------------------------------- epilogue
    // This block's row: O_blk = O / l and LSE_blk = m + ln l. Written as is, or
    // (accumulate) merged into the row's earlier (O, LSE) by LSE weighting
    // ("merge attention", method page section 5): M = max(LSE_prev, LSE_blk),
    // w = exp(LSE - M), O = (w_prev O_prev + w_blk O_blk) / (w_prev + w_blk),
    // LSE = M + ln(w_prev + w_blk); a part at -inf weighs 0.
    const int64_t out_row = ws.out_row0 + q_row0 + tok;
    const int head = kvh * group + (row & (group - 1));
    const int64_t out_idx = out_row * p.n_h + head;
    bool done_ok = __all_sync(0xffffffffu, ok);
    if (done_ok && n_iter > 0) done_ok = warp_wait(&bars[B_O_DONE + x], (n_iter - 1) & 1, abort_flag, p.status);
    // both halves read the earlier LSE before either may overwrite it (after the barrier)
    const float lse_prev = (p.accumulate && row_valid) ? p.lse_part[out_idx] : -INFINITY;
    // Whole row sum from the two halves. The partner warps agree on the
    // outcome here as in the loop (both reach this barrier exactly once).
    *xch_mine = l_run;
    done_ok = named_bar_and(pair_bar, 64, done_ok);
    const float l_tot = l_run + *xch_peer;
    const float inv_l = (l_tot > 0.0f) ? 1.0f / l_tot : 0.0f;
    const float lse_blk = (n_iter > 0 && l_tot > 0.0f) ? (m_run + log2f(l_tot)) * 0.69314718055994531f : -INFINITY;
    float wa = 0.0f, wb = inv_l, lse_new = lse_blk;   // row = wa * O_prev + wb * O (TMEM)
    if (p.accumulate) {
      const float mx = fmaxf(lse_prev, lse_blk);
      if (mx == -INFINITY) {
        wb = 0.0f;
      } else {
        const float ep = expf(lse_prev - mx), eb = expf(lse_blk - mx);
        const float sum = ep + eb;
        wa = ep / sum;
        wb = eb / sum * inv_l;
        lse_new = mx + logf(sum);
      }
    }
    // The tile's rows go through shared memory so that global memory is read
    // and written a whole row per warp instruction (a thread owns half a row;
    // written straight from registers, every 32-byte sector would be touched
    // half at a time by two instructions).
    float* stage = reinterpret_cast<float*>(smem + x * C::kStageTile);   // [row][HD] + padding
    const int wi = warp & 7;                       // warp within the tile's eight
    const uint32_t tile_bar = 9 + x;               // named barrier of the tile's 256 softmax threads
    done_ok = named_bar_and(tile_bar, 256, done_ok);
    // global row of packed row r of this tile (for the copies; r's token must exist)
    auto row_idx = [&](int r) -> int64_t {
      const int tk = x * tok_per_tile + (r >> p.log2_group);
      return (ws.out_row0 + q_row0 + tk) * p.n_h + kvh * group + (r & (group - 1));
    };
    constexpr int kRowsPerIns = 128 / HD;          // rows one warp instruction covers (float4 per lane)
    constexpr int kLanesPerRow = 32 / kRowsPerIns;
    if (done_ok && p.accumulate) {
      // the earlier rows, a whole row per instruction, into the staging rows
      for (int r0 = wi * 16; r0 < wi * 16 + 16; r0 += kRowsPerIns) {
        const int r = r0 + lane / kLanesPerRow;
        const int c4 = lane % kLanesPerRow;
        if (x * tok_per_tile + (r >> p.log2_group) < n_tok)
          *reinterpret_cast<float4*>(stage + r * (C::kStageRow / 4) + c4 * 4) =
              *reinterpret_cast<const float4*>(p.o_part + row_idx(r) * HD + c4 * 4);
      }
    }
    named_bar_sync(tile_bar, 256);
    float* srow = stage + row * (C::kStageRow / 4) + hf * (HD / 2);   // this thread's half row
    if (done_ok) {
      if (n_iter > 0) tc_fence_after();
#pragma unroll
      for (int c = 0; c < HD / 64; ++c) {
        uint32_t o[32];
        if (n_iter > 0) {
          tmem_ld32(o_col + c * 32, o);
          tmem_ld_wait();
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = 0u;
        }
        if (row_valid) {
          float r[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) r[i] = __uint_as_float(o[i]) * wb;
          if (p.accumulate && wa != 0.0f) {   // an earlier row at -inf weighs 0 and is not read
#pragma unroll
            for (int i = 0; i < 32; i += 4) {
              const float4 pv = *reinterpret_cast<const float4*>(srow + c * 32 + i);
              r[i] = fmaf(wa, pv.x, r[i]);
              r[i + 1] = fmaf(wa, pv.y, r[i + 1]);
              r[i + 2] = fmaf(wa, pv.z, r[i + 2]);
              r[i + 3] = fmaf(wa, pv.w, r[i + 3]);
            }
          }
#pragma unroll
          for (int i = 0; i < 32; i += 4)
            *reinterpret_cast<float4*>(srow + c * 32 + i) = make_float4(r[i], r[i + 1], r[i + 2], r[i + 3]);
        }
      }
    }
    named_bar_sync(tile_bar, 256);
    if (done_ok) {
      // the tile's rows to global memory, a whole row per instruction
      for (int r0 = wi * 16; r0 < wi * 16 + 16; r0 += kRowsPerIns) {
        const int r = r0 + lane / kLanesPerRow;
        const int c4 = lane % kLanesPerRow;
        if (x * tok_per_tile + (r >> p.log2_group) >= n_tok) continue;
        const float4 vv = *reinterpret_cast<const float4*>(stage + r * (C::kStageRow / 4) + c4 * 4);
        if (p.out_final)
          *reinterpret_cast<uint2*>(p.out_final + row_idx(r) * HD + c4 * 4) =
              make_uint2(pack_bf16x2(vv.x, vv.y), pack_bf16x2(vv.z, vv.w));
        else
          *reinterpret_cast<float4*>(p.o_part + row_idx(r) * HD + c4 * 4) = vv;
      }
    }
    if (done_ok && row_valid && hf == 0) p.lse_part[out_idx] = lse_new;
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace tc
}  // namespace cpk
