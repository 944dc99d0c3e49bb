// Partial attention of ring blocks on pairs of SMs (tcgen05 cta_group::2).
//
// Method: "Context Parallelism for Scalable Million-Token Inference",
// section 3 (each rank computes the attention of a query shard against one
// KV shard; the partial results are merged by LSE later). Within a block the
// softmax is taken online over 128-key tiles (blockwise exact attention,
// "Context Parallelism과 Expert Parallelism" section 4.1), so the block yields
// O normalised within the block plus its log-sum-exp.
//
// A cluster of two CTAs (one per SM) computes one 256-row query tile of one KV
// head: CTA r holds query rows 128r..128r+127 (GQA packing: rows are (token,
// head-in-group) pairs, 128/G tokens x G heads that share the KV head,
// section 8.2 of the GQA page). Every MMA is one cta_group::2 instruction of
// M = 256 issued by CTA 0 for both SMs:
//   S = Q K^T   A = Q (each CTA its own 128 rows), B = K tile split by key:
//               CTA r holds keys 64r..64r+63;
//   O += P V    A = P from TMEM (each CTA its own rows), B = V tile split by
//               column: CTA r holds columns 64r..64r+63 of all 128 keys.
// So each SM loads half of every K/V tile (32 KB per 128 keys) while the pair
// does the work of two 128-row tiles, and the shared-memory operand traffic of
// S = Q K^T drops by a quarter.
//
// TMEM (512 columns per SM): three S buffers (0, 128, 256) and O (384). With
// three S buffers the MMA issuer computes S(j+1) and S(j+2) while the softmax
// works on S(j), so a softmax step never waits for the PV and S MMAs of the
// step before it: per KV tile the issuer waits for P(j), issues O += P(j) V_j,
// then S(j+3) into the buffer P(j) occupied (tcgen05 operations of one thread
// complete in issue order, so the PV has read P before S overwrites it).
//
// Warp roles per CTA (352 threads):
//   warps 0-7   softmax: two threads per row; warp w reads TMEM lane quarter
//               w&3 and the 64 key columns 64(w>>2)..+63 of each S row. Per
//               step each thread exponentiates its 64 scores against the
//               running max, then the two threads of the row vote (one
//               64-thread bar.red.and per lane quarter): if no row grew its
//               max by more than 2^8 and none meets its first visible tile,
//               P is final; otherwise both take the exact step (row max
//               through shared memory, O rescaled after the previous PV is
//               complete, exponentials recomputed from the intact S);
//   warp 8      TMA producers of this CTA's halves: lane 0 Q and K, lane 1 V,
//               signalling CTA 0's barriers;
//   warp 9      TMEM owner (both CTAs) and, in CTA 0, the MMA issuer;
//   warp 10     in CTA 1, the relay of P (below).
// Cross-SM signals are few, since each costs: a commit multicast to both CTAs
// holds the tensor pipe about 80 cycles, and a remote mbarrier arrive holds
// the arriving thread about a thousand. So K and V use three stages, the
// stage of KV tile j being j mod 3 like its S buffer: the S(j) completion
// (S_FULL, multicast to both CTAs) frees K stage j mod 3 and the PV(j)
// completion (O_DONE, likewise) frees V stage j mod 3, so those two commits
// per tile are the only ones. Softmax warps arrive on their own CTA's P
// barrier; in CTA 1 one relay thread passes each completed step on to CTA 0
// with a single remote arrive, off the softmax warps' path. Barriers that
// collect both CTAs' loads (Q/K/V full) live in CTA 0.
//
// Launched only in a library built with CPK_PAIR_KERNEL=1. Measured on the
// 128K causal prefill it is slower than the single-SM kernel (partial_tc.cuh):
// the relayed arrive reaches CTA 0 thousands of cycles after the step, and the
// issuer waits for it.
#pragma once

#include "common.cuh"
#include "work.cuh"

namespace cpk {
namespace tc2 {

constexpr int BM = 128;                      // query rows per CTA (256 per pair)
constexpr int BN = 128;                      // keys per KV tile
constexpr int HD = 128;                      // head dim
constexpr int kQHalf = 128 * 128;            // 128 rows x 64 bf16 (one 128-byte swizzle column)
constexpr int kQBytes = 2 * kQHalf;          // this CTA's 128 query rows
constexpr int kKHalf = 64 * 128;             // 64 keys x 64 bf16
constexpr int kKBytes = 2 * kKHalf;          // this CTA's 64 keys of a K tile
constexpr int kVBytes = 128 * 128;           // 128 keys x this CTA's 64 columns of V
constexpr int kSBufs = 3;                    // S buffers, and K and V stages
constexpr int kKStages = kSBufs;
constexpr int kVStages = kSBufs;
constexpr int kSoftmaxWarps = 8;
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;
constexpr int kRelayWarp = 10;
constexpr int kThreads = 352;
constexpr int kOffQ = 0;
constexpr int kOffK = kOffQ + kQBytes;
constexpr int kOffV = kOffK + kKStages * kKBytes;
constexpr int kOffBar = kOffV + kVStages * kVBytes;
constexpr int kNumBars = 32;
constexpr int kOffMisc = kOffBar + kNumBars * 8;
constexpr int kOffXch = kOffMisc + 16;       // [step parity][column half][row] f32
constexpr int kSmemNeeded = kOffXch + 2 * 2 * BM * 4;
constexpr int kSmemMax = 232448;
constexpr int kSmemBytes = kSmemNeeded + 1024;
static_assert(kSmemBytes <= kSmemMax, "shared memory plan exceeds 227 KB");
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColO = 384;
constexpr uint32_t kPLocalArrivals = kSoftmaxWarps;
constexpr float kRescaleThreshold = 8.0f;  // log2 units: O is rescaled when the max grows by > 2^8
constexpr int kPolyPairsPer8 = 1;          // of every 8 column pairs, this many take the polynomial exp2

enum {
  B_Q_FULL = 0,     // CTA 0: both CTAs' Q halves have landed
  B_K_FULL = 1,     // +stage (3), CTA 0
  B_V_FULL = 4,     // +stage (3), CTA 0
  B_S_FULL = 7,     // +(j mod 3), both: S(j) is in TMEM, K stage j mod 3 is free
  B_O_DONE = 10,    // +(j mod 3), both: O += P(j) V_j has completed, V stage j mod 3 is free
  B_P_LOCAL = 13,   // +(j mod 3), both: this CTA's 8 softmax warps wrote P(j)
  B_P_PEER = 16,    // +(j mod 3), CTA 0: CTA 1's P(j) is written (relayed)
  B_DRAIN = 19      // CTA 0: every MMA issued has completed
};

struct Params {
  CUtensorMap tm_q;  // [q_rows][N_KV][G][128] bf16, box {64, G, 1, 128/G}
  CUtensorMap tm_k;  // [kv_rows][N_KV][128] bf16, box {64, 1, 64}
  CUtensorMap tm_v;  // [kv_rows][N_KV][128] bf16, box {64, 1, 128}
  float* o_part;
  float* lse_part;
  __nv_bfloat16* out_final;   // not null: write the merged, normalised row here (bf16) instead of o_part
  int32_t accumulate;         // merge each row into the (O, LSE) already at its place in o_part / lse_part
  uint32_t* status;
  int32_t n_h;
  int32_t log2_group;
  int32_t causal;
  float scale_log2;  // softmax scale * log2(e)
  WorkTable wt;      // tiles are 256-row pair tiles
};

// ---------------------------------------------------------------- cluster / pair helpers
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

// Address of the same shared-memory location in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t cluster_addr(const void* p, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_u32(p)), "r"(rank));
  return r;
}

// Every thread of both CTAs.
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release;\n\tbarrier.cluster.wait.acquire;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_remote(uint32_t cl_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cl_addr) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait_cl(uint64_t* bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(done)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return done != 0;
}

// Bounded wait with cluster-scope acquire (arrivals from the other CTA).
__device__ __forceinline__ bool mbar_wait_cl(uint64_t* bar, uint32_t parity, volatile uint32_t* abort_flag,
                                             uint32_t* status) {
  const uint64_t t0 = globaltimer();
  while (!mbar_try_wait_cl(bar, parity)) {
    if (*abort_flag) return false;
    if (globaltimer() - t0 > kWaitBudgetNs) {
      *abort_flag = 1u;
      if (status) atomicOr(status, kStatusTimeout);
      return false;
    }
  }
  return true;
}

__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile uint32_t* abort_flag,
                                          uint32_t* status) {
  const bool ok = mbar_wait(bar, parity, abort_flag, status);
  return __all_sync(0xffffffffu, ok);
}

__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity, uint32_t* status) {
  const uint64_t t0 = globaltimer();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer() - t0 > kWaitBudgetNs) {
      if (status) atomicOr(status, kStatusTimeout);
      return;
    }
  }
}

// TMA tile loads into this CTA's shared memory whose completion is counted on
// a barrier of CTA 0 (`bar_cl`, a cluster address). No multicast.
__device__ __forceinline__ void tma_load_3d_pair(void* dst, const CUtensorMap* map, uint32_t bar_cl, int c0, int c1,
                                                 int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_u32(dst)),
      "l"(map), "r"(c0), "r"(c1), "r"(c2), "r"(bar_cl)
      : "memory");
}

__device__ __forceinline__ void tma_load_4d_pair(void* dst, const CUtensorMap* map, uint32_t bar_cl, int c0, int c1,
                                                 int c2, int c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4, %5}], [%6];" ::"r"(smem_u32(dst)),
      "l"(map), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(bar_cl)
      : "memory");
}

// TMEM allocation of the pair: the same warp of both CTAs issues it.
__device__ __forceinline__ void tmem_alloc_pair(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}

__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// D (+)= A * B over the pair, M = 256: A, B from shared memory.
__device__ __forceinline__ void umma_pair_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                             uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// D (+)= A * B over the pair, M = 256: A from TMEM (row m of each CTA in its lane m), B from shared memory.
__device__ __forceinline__ void umma_pair_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                             uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive once on `bar` in both CTAs when every MMA issued so far has completed.
__device__ __forceinline__ void umma_commit_both(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
          smem_u32(bar)),
      "h"(static_cast<uint16_t>(3))
      : "memory");
}

// Arrive once on `bar` of this CTA when every MMA issued so far has completed.
__device__ __forceinline__ void umma_commit_own(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

// Exponentials of one thread's 64 keys of a KV tile: P = 2^(S*scale*log2e -
// m_use) as 32 bf16 pairs in registers (pk), returning the sum of the fp32
// values; nothing is written, so S stays in TMEM for a redo. S is read from
// TMEM 8 columns at a time, the next chunk in flight. kPolyPairsPer8 of every
// 8 pairs take the polynomial on the FMA pipe, the rest the special function
// unit. kMasked: keys past `lim` are hidden and get exactly 0. x_max receives
// the largest exponent over the visible keys.
template <bool kMasked>
__device__ __forceinline__ float seg_exps(uint32_t s_col, float sl2, float m_use, int lim, uint32_t (&pk)[32],
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

// 11 warps put three on three of the four schedulers, whose register files
// hold 16K registers each: at most 170 per thread, so 168.
__global__ void __cluster_dims__(2, 1, 1) __maxnreg__(168) partial_bf16_pair_kernel(const __grid_constant__ Params p) {
  extern __shared__ uint8_t smem_raw[];
  // the same offset in both CTAs: the MMA descriptors address both
  const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  uint8_t* smem = smem_raw + pad;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffMisc);
  volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(smem + kOffMisc + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  if (pad + kSmemNeeded > kSmemBytes) {  // the same in both CTAs: nothing has started yet
    if (threadIdx.x == 0) atomicOr(p.status, kStatusInternal);
    return;
  }
  const uint32_t rank = cluster_rank();

  int32_t seg, tile;
  locate_tile(p.wt, static_cast<int32_t>(blockIdx.x >> 1), seg, tile);
  const WorkSeg ws = p.wt.segs[seg];
  const cp_range qr = p.wt.ranges[ws.q_range];
  const int kvh = blockIdx.y;
  const int group = 1 << p.log2_group;
  const int tok_per_tile = BM >> p.log2_group;            // tokens per CTA
  const int64_t tok0 = static_cast<int64_t>(tile) * (2 * tok_per_tile);
  const int n_tok = static_cast<int>(min(static_cast<int64_t>(2 * tok_per_tile), qr.len - tok0));   // of the pair
  const int64_t q_row0 = qr.row0 + tok0;
  const int64_t q_pos_lo = qr.pos0 + tok0;
  const int64_t q_pos_hi = q_pos_lo + n_tok - 1;
  const int causal = p.causal;

  // KV tiles the pair visits (both CTAs count alike: enough for the pair's last token)
  int n_iter = 0;
  for (int r = 0; r < ws.kv_count; ++r) {
    const cp_range kr = p.wt.ranges[ws.kv_begin + r];
    if (kr.seq != qr.seq) continue;
    n_iter += static_cast<int>((visible_keys(kr, q_pos_hi, causal) + BN - 1) / BN);
  }

  if (threadIdx.x == 0) {
    for (int i = 0; i < kNumBars; ++i)
      mbar_init(&bars[i], (i >= B_P_LOCAL && i < B_P_LOCAL + kSBufs) ? kPLocalArrivals : 1u);
    *abort_flag = 0u;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc_pair(tmem_slot, kTmemCols);
    tmem_relinquish_pair();
  }
  if (warp == kProducerWarp && lane == 0) {
    prefetch_tensormap(&p.tm_q);
    prefetch_tensormap(&p.tm_k);
    prefetch_tensormap(&p.tm_v);
  }
  tc_fence_before();
  __syncwarp();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  uint8_t* sQ = smem + kOffQ;
  uint8_t* sK = smem + kOffK;
  uint8_t* sV = smem + kOffV;

  if (warp == kProducerWarp) {
    // ------------------------------------------------------------------ TMA producers (this CTA's halves)
    if (lane < 2 && n_iter > 0) {
      const bool is_k = lane == 0;
      uint8_t* base = is_k ? sK : sV;
      const int st_bytes = is_k ? kKBytes : kVBytes;
      uint64_t* full = &bars[is_k ? B_K_FULL : B_V_FULL];
      uint64_t* empty = &bars[is_k ? B_S_FULL : B_O_DONE];   // completion of the MMA that read the stage
      uint32_t issued[kSBufs] = {0u, 0u, 0u};
      if (is_k) {
        if (rank == 0) mbar_arrive_expect_tx(&bars[B_Q_FULL], 2 * kQBytes);
        const uint32_t qbar = cluster_addr(&bars[B_Q_FULL], 0);
        const int row = static_cast<int>(q_row0) + static_cast<int>(rank) * tok_per_tile;
        tma_load_4d_pair(sQ, &p.tm_q, qbar, 0, 0, kvh, row);
        tma_load_4d_pair(sQ + kQHalf, &p.tm_q, qbar, 64, 0, kvh, row);
      }
      int it = 0;
      bool ok = true;
      for (int r = 0; r < ws.kv_count && ok; ++r) {
        const cp_range kr = p.wt.ranges[ws.kv_begin + r];
        if (kr.seq != qr.seq) continue;
        const int64_t nv = visible_keys(kr, q_pos_hi, causal);
        for (int64_t k0 = 0; k0 < nv; k0 += BN, ++it) {
          // stage it mod 3 held KV tile it-3; its MMA completing is phase (it-3)/3 of
          // that barrier, and the next phase needs this load
          const int st = it % kSBufs;
          if (it >= kSBufs && !mbar_wait(&empty[st], ((it - kSBufs) / kSBufs) & 1, abort_flag, p.status)) {
            ok = false;
            break;
          }
          if (rank == 0) mbar_arrive_expect_tx(&full[st], 2 * st_bytes);
          const uint32_t fbar = cluster_addr(&full[st], 0);
          const int key_row = static_cast<int>(kr.row0 + k0);
          uint8_t* dst = base + st * st_bytes;
          if (is_k) {
            const int kr0 = key_row + static_cast<int>(rank) * 64;
            tma_load_3d_pair(dst, &p.tm_k, fbar, 0, kvh, kr0);
            tma_load_3d_pair(dst + kKHalf, &p.tm_k, fbar, 64, kvh, kr0);
          } else {
            tma_load_3d_pair(dst, &p.tm_v, fbar, static_cast<int>(rank) * 64, kvh, key_row);
          }
          issued[st] += 1;
        }
      }
      // Drain: CTA 0's full barriers count both CTAs' bytes, so once they
      // complete every load of the pair has landed.
      if (rank == 0) {
        if (is_k) drain_wait(&bars[B_Q_FULL], 0u, p.status);
        for (int st = 0; st < kSBufs; ++st)
          if (issued[st] > 0) drain_wait(&full[st], (issued[st] - 1u) & 1u, p.status);
      }
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------------ MMA issuer (CTA 0)
    if (rank == 0 && lane == 0 && n_iter > 0) {
      constexpr uint32_t idesc_s = umma_idesc_bf16(2 * BM, BN, 0);   // Q, K both K-major
      constexpr uint32_t idesc_o = umma_idesc_bf16(2 * BM, HD, 1);   // P (TMEM) K-major, V MN-major
      // An operand at byte offset `off` from a base is base + off/16 (every
      // shared address is below 256 KB, so the 14-bit field does not carry).
      const uint64_t q_desc = umma_sdesc_sw128(smem_u32(sQ), 16, 1024);
      const uint64_t k_desc = umma_sdesc_sw128(smem_u32(sK), 16, 1024);
      const uint64_t v_desc = umma_sdesc_sw128(smem_u32(sV), kVBytes, 1024);   // one 64-column block per CTA
      auto issue_s = [&](int i) {   // S(i) = Q K_i^T into buffer i % 3
        const uint64_t kd = k_desc + static_cast<uint64_t>(((i % kSBufs) * kKBytes) >> 4);
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) {
          const uint64_t qo = static_cast<uint64_t>(((kk >> 2) * kQHalf + (kk & 3) * 32) >> 4);
          const uint64_t ko = static_cast<uint64_t>(((kk >> 2) * kKHalf + (kk & 3) * 32) >> 4);
          umma_pair_ss(tmem + (i % kSBufs) * BN, q_desc + qo, kd + ko, idesc_s, kk > 0 ? 1u : 0u);
        }
        umma_commit_both(&bars[B_S_FULL + i % kSBufs]);
      };
      auto issue_pv = [&](int j) {  // O += P(j) V_j
        const uint64_t vd = v_desc + static_cast<uint64_t>(((j % kSBufs) * kVBytes) >> 4);
        const uint32_t pb = tmem + (j % kSBufs) * BN;
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk) {
          // keys 16kk..16kk+15 as bf16 pairs: each thread's P sits in the first 32 of its 64 S columns
          const uint32_t p_addr = pb + (kk >> 2) * 64 + (kk & 3) * 8;
          umma_pair_ts(tmem + kColO, p_addr, vd + static_cast<uint64_t>((kk * 2048) >> 4), idesc_o,
                       (j > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit_both(&bars[B_O_DONE + j % kSBufs]);
      };
      bool ok = mbar_wait(&bars[B_Q_FULL], 0u, abort_flag, p.status);
      const int pre = n_iter < kSBufs ? n_iter : kSBufs;
      for (int i = 0; i < pre && ok; ++i) {
        ok = mbar_wait(&bars[B_K_FULL + i % kSBufs], (i / kSBufs) & 1, abort_flag, p.status);
        if (ok) {
          tc_fence_after();
          issue_s(i);
        }
      }
      for (int j = 0; j < n_iter && ok; ++j) {
        const uint32_t ph = (j / kSBufs) & 1;
        if (!mbar_wait(&bars[B_V_FULL + j % kSBufs], ph, abort_flag, p.status)) break;
        if (!mbar_wait(&bars[B_P_LOCAL + j % kSBufs], ph, abort_flag, p.status)) break;
        if (!mbar_wait_cl(&bars[B_P_PEER + j % kSBufs], ph, abort_flag, p.status)) break;
        tc_fence_after();
        issue_pv(j);
        const int i = j + kSBufs;
        if (i < n_iter) {
          if (!mbar_wait(&bars[B_K_FULL + i % kSBufs], (i / kSBufs) & 1, abort_flag, p.status)) break;
          tc_fence_after();
          issue_s(i);
        }
      }
      // Everything issued completes before TMEM is released.
      umma_commit_own(&bars[B_DRAIN]);
      drain_wait(&bars[B_DRAIN], 0u, p.status);
    }
  } else if (warp == kRelayWarp) {
    // ------------------------------------------------------------------ P relay (CTA 1)
    // Step j's local barrier cannot complete its next phase (step j+3) before
    // this thread relays step j: S(j+3) is issued only after PV(j).
    if (rank == 1 && lane == 0) {
      const uint32_t peer0 = cluster_addr(&bars[B_P_PEER], 0);
      for (int j = 0; j < n_iter; ++j) {
        if (!mbar_wait(&bars[B_P_LOCAL + j % kSBufs], (j / kSBufs) & 1, abort_flag, p.status)) break;
        tc_fence_after();
        tc_fence_before();
        mbar_arrive_remote(peer0 + 8u * static_cast<uint32_t>(j % kSBufs));
      }
    }
  } else {
    // ------------------------------------------------------------------ softmax warps 0..7
    const int cg = warp >> 2;                // column half: keys 64cg .. 64cg+63 of every tile
    const int quarter = warp & 3;            // TMEM lane quarter
    const int row = quarter * 32 + lane;     // packed row within this CTA's 128
    const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t s_base = tmem + lane_base + cg * 64;          // + buffer * 128
    const uint32_t o_col = tmem + lane_base + kColO + cg * 64;   // this thread's O columns
    float* xch = reinterpret_cast<float*>(smem + kOffXch);
    const uint32_t grp_bar = 1 + quarter;    // named barrier of the two warps sharing these rows
    const int tok = static_cast<int>(rank) * tok_per_tile + (row >> p.log2_group);   // token within the pair
    const bool row_valid = tok < n_tok;
    const int64_t qpos = q_pos_lo + tok;
    const float sl2 = p.scale_log2;
    float m_run = -INFINITY;
    float l_run = 0.0f;   // this thread's part of the row sum
    bool ok = true;
    bool carry_ok = true; // a wait inside the previous step failed: the next vote ends the loop
    int it = 0;

    for (int r = 0; r < ws.kv_count && ok; ++r) {
      const cp_range kr = p.wt.ranges[ws.kv_begin + r];
      if (kr.seq != qr.seq) continue;
      const int64_t nv = visible_keys(kr, q_pos_hi, causal);
      for (int64_t k0 = 0; k0 < nv; k0 += BN, ++it) {
        const int64_t kp0 = kr.pos0 + k0;
        const int n_valid = static_cast<int>(min(static_cast<int64_t>(BN), nv - k0));
        const int b = it % kSBufs;
        const uint32_t s_col = s_base + b * BN;
        const bool got = warp_wait(&bars[B_S_FULL + b], (it / kSBufs) & 1, abort_flag, p.status) && carry_ok;
        // key 64cg + c of the tile is visible iff c <= lim
        int lim = 63;
        if ((n_valid < BN) || (causal && kp0 + BN - 1 > qpos)) {
          int64_t l64 = n_valid - 1;
          if (causal && qpos - kp0 < l64) l64 = qpos - kp0;
          l64 -= cg * 64;
          lim = static_cast<int>(max(min(l64, static_cast<int64_t>(63)), static_cast<int64_t>(-1)));
        }
        const bool tile_masked = __any_sync(0xffffffffu, lim < 63);
        // Optimistic step against the running max; the two threads of a row
        // hold the same m_run, so they agree on `first`.
        const bool first = __any_sync(0xffffffffu, m_run == -INFINITY);
        float raw_max = -INFINITY;   // max over visible keys of S*scale*log2e in this thread's columns
        float sum = 0.0f;
        bool fine = false;
        uint32_t pk[32];
        if (got) {
          tc_fence_after();
          if (first) {
            uint32_t sv[4][16];
#pragma unroll
            for (int h = 0; h < 4; ++h) tmem_ld16(s_col + h * 16, sv[h]);
            tmem_ld_wait();
            float a0 = -INFINITY, a1 = -INFINITY;
#pragma unroll
            for (int h = 0; h < 4; ++h)
#pragma unroll
              for (int cc = 0; cc < 16; cc += 4) {
                const int c = h * 16 + cc;
                const float v0 = (c > lim) ? -INFINITY : __uint_as_float(sv[h][cc]);
                const float v1 = (c + 1 > lim) ? -INFINITY : __uint_as_float(sv[h][cc + 1]);
                const float v2 = (c + 2 > lim) ? -INFINITY : __uint_as_float(sv[h][cc + 2]);
                const float v3 = (c + 3 > lim) ? -INFINITY : __uint_as_float(sv[h][cc + 3]);
                a0 = fmax3(a0, v0, v1);
                a1 = fmax3(a1, v2, v3);
              }
            raw_max = fmaxf(a0, a1) * sl2;
          } else {
            float x_max;
            sum = tile_masked ? seg_exps<true>(s_col, sl2, m_run, lim, pk, x_max)
                              : seg_exps<false>(s_col, sl2, m_run, lim, pk, x_max);
            raw_max = x_max + m_run;
            fine = !(x_max > kRescaleThreshold);
          }
        }
        // The two warps of the lane quarter meet here once per KV tile and
        // agree on the outcome. The exchange slots alternate by step: a slot
        // is written again only two steps later, after every partner has
        // passed the next step's vote, hence after its reads.
        float* slots = xch + (it & 1) * 2 * BM + row;
        slots[cg * BM] = raw_max;
        tc_fence_before();
        const bool all_fine = named_bar_and(grp_bar, 64, got && fine);
        tc_fence_after();
        float alpha = 1.0f;
        bool resc = false;
        if (!all_fine) {
          if (!named_bar_and(grp_bar, 64, got)) { ok = false; break; }
          const float m_new = fmaxf(m_run, fmaxf(slots[0], slots[BM]));
          if (m_new > m_run + kRescaleThreshold) {
            alpha = ex2(m_run - m_new);
            m_run = m_new;
            resc = true;
          }
          const float m_use = (m_run == -INFINITY) ? 0.0f : m_run;
          float unused;
          sum = tile_masked ? seg_exps<true>(s_col, sl2, m_use, lim, pk, unused)
                            : seg_exps<false>(s_col, sl2, m_use, lim, pk, unused);
        }
        // P over the first 32 of this thread's 64 S columns (read by the PV MMA)
        tmem_st32(s_col, pk);
        l_run = l_run * alpha + sum;
        // Rescale this thread's O columns once O += P(it-1) V has completed
        // (S(it) being ready implies only that PV(it-3) has).
        if (it > 0 && __any_sync(0xffffffffu, resc)) {
          const int pj = it - 1;
          const bool od = warp_wait(&bars[B_O_DONE + pj % kSBufs], (pj / kSBufs) & 1, abort_flag, p.status);
          if (od) {
            tc_fence_after();
#pragma unroll 1
            for (int c = 0; c < 4; ++c) {
              uint32_t o[16];
              tmem_ld16(o_col + c * 16, o);
              tmem_ld_wait();
#pragma unroll
              for (int i = 0; i < 16; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
              tmem_st16(o_col + c * 16, o);
            }
          }
          carry_ok = od;
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars[B_P_LOCAL + b]);
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
    bool done_ok = __all_sync(0xffffffffu, ok && carry_ok);
    if (done_ok && n_iter > 0) {
      const int lj = n_iter - 1;
      done_ok = warp_wait(&bars[B_O_DONE + lj % kSBufs], (lj / kSBufs) & 1, abort_flag, p.status);
    }
    // both threads read the earlier LSE before either may overwrite it (after the barrier)
    const float lse_prev = (p.accumulate && row_valid) ? p.lse_part[out_idx] : -INFINITY;
    float* slots = xch + (it & 1) * 2 * BM + row;
    slots[cg * BM] = l_run;
    done_ok = named_bar_and(grp_bar, 64, done_ok);
    const float l_tot = slots[0] + slots[BM];
    const float inv_l = (l_tot > 0.0f) ? 1.0f / l_tot : 0.0f;
    const float lse_blk = (n_iter > 0 && l_tot > 0.0f) ? (m_run + log2f(l_tot)) * 0.69314718055994531f : -INFINITY;
    float wa = 0.0f, wb = inv_l, lse_new = lse_blk;   // row = wa * O_prev + wb * O (TMEM)
    if (p.accumulate) {
      const float mx = fmaxf(lse_prev, lse_blk);
      if (mx == -INFINITY) {
        wb = 0.0f;
      } else {
        const float ep = expf(lse_prev - mx), eb = expf(lse_blk - mx);
        const float s2 = ep + eb;
        wa = ep / s2;
        wb = eb / s2 * inv_l;
        lse_new = mx + logf(s2);
      }
    }
    if (done_ok && n_iter > 0) tc_fence_after();
#pragma unroll 1
    for (int hc = 0; hc < 2 && done_ok; ++hc) {
      uint32_t o[32];
      if (n_iter > 0) {
        tmem_ld32(o_col + hc * 32, o);
        tmem_ld_wait();
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) o[i] = 0u;
      }
      if (row_valid) {
        float* dst = p.o_part + out_idx * HD + cg * 64 + hc * 32;
        float rr[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) rr[i] = __uint_as_float(o[i]) * wb;
        if (p.accumulate) {
#pragma unroll
          for (int i = 0; i < 32; i += 4) {
            const float4 pv = *reinterpret_cast<const float4*>(dst + i);
            rr[i] = fmaf(wa, pv.x, rr[i]);
            rr[i + 1] = fmaf(wa, pv.y, rr[i + 1]);
            rr[i + 2] = fmaf(wa, pv.z, rr[i + 2]);
            rr[i + 3] = fmaf(wa, pv.w, rr[i + 3]);
          }
        }
        if (p.out_final) {
          uint4* fo = reinterpret_cast<uint4*>(p.out_final + out_idx * HD + cg * 64 + hc * 32);
#pragma unroll
          for (int i = 0; i < 32; i += 8)
            fo[i >> 3] = make_uint4(pack_bf16x2(rr[i], rr[i + 1]), pack_bf16x2(rr[i + 2], rr[i + 3]),
                                    pack_bf16x2(rr[i + 4], rr[i + 5]), pack_bf16x2(rr[i + 6], rr[i + 7]));
        } else {
#pragma unroll
          for (int i = 0; i < 32; i += 4)
            *reinterpret_cast<float4*>(dst + i) = make_float4(rr[i], rr[i + 1], rr[i + 2], rr[i + 3]);
        }
      }
    }
    if (done_ok && row_valid && cg == 0) p.lse_part[out_idx] = lse_new;
  }

  // Both CTAs are done with TMEM (CTA 0 drained its MMAs, every TMEM load and
  // store has been waited for) and no barrier of either CTA is used again.
  tc_fence_before();
  __syncwarp();
  cluster_sync();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, kTmemCols);
  }
}

}  // namespace tc2
}  // namespace cpk
