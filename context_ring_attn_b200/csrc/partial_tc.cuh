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
// One CTA = one 128-row query tile of one KV head. GQA packing: the 128 rows
// are (token, head-in-group) pairs, 128/G tokens x G query heads that share
// the KV head (section 8.2 of the GQA page), so every K/V tile is loaded once
// for all G heads. Warp roles (192 threads):
//   warps 0-3  softmax: thread = query row; reads S rows from TMEM, masks by
//              global position, online max/sum, writes P (bf16) to shared
//              memory, rescales O in TMEM when the running max moves by more
//              than 2^8, and writes the normalised O and LSE at the end;
//   warp 4     TMA producer: Q once, then K and V tiles into a 2-stage ring;
//   warp 5     MMA issuer (one thread): S = Q K^T into a double-buffered TMEM
//              slot, O += P V into the TMEM accumulator; owns TMEM alloc.
// TMEM (512 columns): S buffers at columns 0 and 128, O at 256.
#pragma once

#include "common.cuh"
#include "work.cuh"

namespace cpk {
namespace tc {

constexpr int BM = 128;                      // packed query rows per tile
constexpr int BN = 128;                      // keys per KV tile
constexpr int HD = 128;                      // head dim
constexpr int kHalfBytes = 128 * 128;        // 128 rows x 64 bf16 (one 128-byte swizzle column)
constexpr int kTileBytes = 2 * kHalfBytes;   // 128 rows x 128 bf16
constexpr int kStages = 2;
constexpr int kThreads = 192;
constexpr int kOffQ = 0;
constexpr int kOffK = kOffQ + kTileBytes;
constexpr int kOffV = kOffK + kStages * kTileBytes;
constexpr int kOffP = kOffV + kStages * kTileBytes;
constexpr int kOffBar = kOffP + kTileBytes;
constexpr int kNumBars = 16;
constexpr int kOffMisc = kOffBar + kNumBars * 8;
constexpr int kSmemBytes = kOffMisc + 64 + 1024;  // + slack to align the base to 1024
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0;
constexpr uint32_t kColO = 256;
constexpr float kRescaleThreshold = 8.0f;  // log2 units: O is rescaled when the max grows by > 2^8

// barrier slots
enum {
  B_Q_FULL = 0,
  B_K_FULL = 1,   // +stage
  B_V_FULL = 3,   // +stage
  B_K_EMPTY = 5,  // +stage
  B_V_EMPTY = 7,  // +stage
  B_S_FULL = 9,   // +buffer
  B_S_FREE = 11,  // +buffer
  B_P_FULL = 13,
  B_PV_DONE = 14,
  B_DRAIN = 15
};

struct Params {
  CUtensorMap tm_q;  // [q_rows][N_KV][G][128] bf16, box {64, G, 1, 128/G}
  CUtensorMap tm_k;  // [kv_rows][N_KV][128] bf16, box {64, 1, 128}
  CUtensorMap tm_v;
  float* o_part;
  float* lse_part;
  uint32_t* status;
  int32_t n_h;
  int32_t log2_group;
  int32_t causal;
  float scale_log2;  // softmax scale * log2(e)
  WorkTable wt;
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

__global__ void __launch_bounds__(kThreads, 1) partial_bf16_kernel(const __grid_constant__ Params p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  uint8_t* smem = smem_raw + pad;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffMisc);
  volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(smem + kOffMisc + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  int32_t seg, tile;
  locate_tile(p.wt, blockIdx.x, seg, tile);
  const WorkSeg ws = p.wt.segs[seg];
  const cp_range qr = p.wt.ranges[ws.q_range];
  const int kvh = blockIdx.y;
  const int group = 1 << p.log2_group;
  const int tok_per_tile = BM >> p.log2_group;
  const int64_t tok0 = static_cast<int64_t>(tile) * tok_per_tile;
  const int n_tok = static_cast<int>(min(static_cast<int64_t>(tok_per_tile), qr.len - tok0));
  const int64_t q_row0 = qr.row0 + tok0;
  const int64_t q_pos_lo = qr.pos0 + tok0;
  const int64_t q_pos_hi = q_pos_lo + n_tok - 1;
  const int causal = p.causal;

  // number of KV tiles this query tile visits
  int n_iter = 0;
  for (int r = 0; r < ws.kv_count; ++r) {
    const cp_range kr = p.wt.ranges[ws.kv_begin + r];
    if (kr.seq != qr.seq) continue;
    n_iter += static_cast<int>((visible_keys(kr, q_pos_hi, causal) + BN - 1) / BN);
  }

  if (threadIdx.x == 0) {
    for (int i = 0; i < kNumBars; ++i) {
      uint32_t count = 1;
      if (i == B_S_FREE || i == B_S_FREE + 1 || i == B_P_FULL) count = 4;  // one arrive per softmax warp
      mbar_init(&bars[i], count);
    }
    *abort_flag = 0u;
    fence_mbar_init();
  }
  if (warp == 5) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  if (warp == 4 && lane == 0) {
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
  uint8_t* sP = smem + kOffP;

  if (warp == 4) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0 && n_iter > 0) {
      uint32_t issued_k[kStages] = {0u, 0u};
      uint32_t issued_v[kStages] = {0u, 0u};
      mbar_arrive_expect_tx(&bars[B_Q_FULL], kTileBytes);
      tma_load_4d(sQ, &p.tm_q, &bars[B_Q_FULL], 0, 0, kvh, static_cast<int>(q_row0));
      tma_load_4d(sQ + kHalfBytes, &p.tm_q, &bars[B_Q_FULL], 64, 0, kvh, static_cast<int>(q_row0));
      int it = 0;
      bool ok = true;
      for (int r = 0; r < ws.kv_count && ok; ++r) {
        const cp_range kr = p.wt.ranges[ws.kv_begin + r];
        if (kr.seq != qr.seq) continue;
        const int64_t nv = visible_keys(kr, q_pos_hi, causal);
        for (int64_t k0 = 0; k0 < nv; k0 += BN, ++it) {
          const int st = it & 1;
          const uint32_t ph = (it >> 1) & 1;
          const int key_row = static_cast<int>(kr.row0 + k0);
          if (it >= 2 && !mbar_wait(&bars[B_K_EMPTY + st], ph ^ 1u, abort_flag, p.status)) { ok = false; break; }
          mbar_arrive_expect_tx(&bars[B_K_FULL + st], kTileBytes);
          tma_load_3d(sK + st * kTileBytes, &p.tm_k, &bars[B_K_FULL + st], 0, kvh, key_row);
          tma_load_3d(sK + st * kTileBytes + kHalfBytes, &p.tm_k, &bars[B_K_FULL + st], 64, kvh, key_row);
          issued_k[st] += 1;
          if (it >= 2 && !mbar_wait(&bars[B_V_EMPTY + st], ph ^ 1u, abort_flag, p.status)) { ok = false; break; }
          mbar_arrive_expect_tx(&bars[B_V_FULL + st], kTileBytes);
          tma_load_3d(sV + st * kTileBytes, &p.tm_v, &bars[B_V_FULL + st], 0, kvh, key_row);
          tma_load_3d(sV + st * kTileBytes + kHalfBytes, &p.tm_v, &bars[B_V_FULL + st], 64, kvh, key_row);
          issued_v[st] += 1;
        }
      }
      // Drain: every load issued has landed before the CTA may exit.
      drain_wait(&bars[B_Q_FULL], 0u, p.status);
      for (int st = 0; st < kStages; ++st) {
        if (issued_k[st] > 0) drain_wait(&bars[B_K_FULL + st], (issued_k[st] - 1u) & 1u, p.status);
        if (issued_v[st] > 0) drain_wait(&bars[B_V_FULL + st], (issued_v[st] - 1u) & 1u, p.status);
      }
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0 && n_iter > 0) {
      constexpr uint32_t idesc_s = umma_idesc_bf16(BM, BN, 0);   // Q, K both K-major
      constexpr uint32_t idesc_o = umma_idesc_bf16(BM, HD, 1);   // P K-major, V MN-major
      const uint32_t q_addr = smem_u32(sQ);
      const uint32_t k_addr = smem_u32(sK);
      const uint32_t v_addr = smem_u32(sV);
      const uint32_t p_addr = smem_u32(sP);
      auto issue_pv = [&](int j) -> bool {
        if (!mbar_wait(&bars[B_P_FULL], j & 1, abort_flag, p.status)) return false;
        if (!mbar_wait(&bars[B_V_FULL + (j & 1)], (j >> 1) & 1, abort_flag, p.status)) return false;
        tc_fence_after();
        const uint32_t vb = v_addr + (j & 1) * kTileBytes;
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) {
          const uint64_t a = umma_sdesc_sw128(p_addr + (kk >> 2) * kHalfBytes + (kk & 3) * 32, 16, 1024);
          const uint64_t b = umma_sdesc_sw128(vb + kk * 2048, kHalfBytes, 1024);
          umma_bf16_ss(tmem + kColO, a, b, idesc_o, (j > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit(&bars[B_PV_DONE]);
        umma_commit(&bars[B_V_EMPTY + (j & 1)]);
        return true;
      };
      bool ok = mbar_wait(&bars[B_Q_FULL], 0u, abort_flag, p.status);
      for (int it = 0; it < n_iter && ok; ++it) {
        const int st = it & 1;
        const uint32_t ph = (it >> 1) & 1;
        if (!mbar_wait(&bars[B_K_FULL + st], ph, abort_flag, p.status)) { ok = false; break; }
        if (it >= 2 && !mbar_wait(&bars[B_S_FREE + st], ph ^ 1u, abort_flag, p.status)) { ok = false; break; }
        tc_fence_after();
        const uint32_t kb = k_addr + st * kTileBytes;
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) {
          const uint32_t off = (kk >> 2) * kHalfBytes + (kk & 3) * 32;
          const uint64_t a = umma_sdesc_sw128(q_addr + off, 16, 1024);
          const uint64_t b = umma_sdesc_sw128(kb + off, 16, 1024);
          umma_bf16_ss(tmem + kColS + st * BN, a, b, idesc_s, kk > 0 ? 1u : 0u);
        }
        umma_commit(&bars[B_S_FULL + st]);
        umma_commit(&bars[B_K_EMPTY + st]);
        if (it >= 1 && !issue_pv(it - 1)) { ok = false; break; }
      }
      if (ok) issue_pv(n_iter - 1);
      // Everything this thread issued completes before TMEM is released.
      umma_commit(&bars[B_DRAIN]);
      drain_wait(&bars[B_DRAIN], 0u, p.status);
    }
  } else {
    // ------------------------------------------------------------------ softmax warps 0..3
    const int row = threadIdx.x;  // TMEM lane == packed query row
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
    const int tok = row >> p.log2_group;
    const bool row_valid = tok < n_tok;
    const int64_t qpos = q_pos_lo + tok;
    const float sl2 = p.scale_log2;
    float m_run = -INFINITY;
    float l_run = 0.0f;
    bool ok = true;
    int it = 0;

    for (int r = 0; r < ws.kv_count && ok; ++r) {
      const cp_range kr = p.wt.ranges[ws.kv_begin + r];
      if (kr.seq != qr.seq) continue;
      const int64_t nv = visible_keys(kr, q_pos_hi, causal);
      for (int64_t k0 = 0; k0 < nv; k0 += BN, ++it) {
        const int sb = it & 1;
        const int64_t kp0 = kr.pos0 + k0;
        const int n_valid = static_cast<int>(min(static_cast<int64_t>(BN), nv - k0));
        const bool need_mask = (n_valid < BN) || (causal && kp0 + BN - 1 > q_pos_lo);

        if (!warp_wait(&bars[B_S_FULL + sb], (it >> 1) & 1, abort_flag, p.status)) { ok = false; break; }
        tc_fence_after();
        uint32_t s[4][32];
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld32(tmem + lane_base + kColS + sb * BN + c * 32, s[c]);
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars[B_S_FREE + sb]);

        if (need_mask) {
          // key c is visible iff c < n_valid and (not causal or kp0 + c <= qpos)
          int64_t lim = n_valid - 1;
          if (causal) {
            const int64_t c_lim = qpos - kp0;
            if (c_lim < lim) lim = c_lim;
          }
#pragma unroll
          for (int c = 0; c < BN; ++c)
            if (c > lim) s[c >> 5][c & 31] = __float_as_uint(-INFINITY);
        }
        float mx = -INFINITY;
#pragma unroll
        for (int c = 0; c < BN; ++c) mx = fmaxf(mx, __uint_as_float(s[c >> 5][c & 31]));
        const float m_new = fmaxf(m_run, mx * sl2);
        float alpha = 1.0f;
        bool resc = false;
        if (m_new > m_run + kRescaleThreshold) {
          alpha = ex2(m_run - m_new);
          m_run = m_new;
          resc = true;
        }
        const float m_use = (m_run == -INFINITY) ? 0.0f : m_run;
        float sum = 0.0f;
#pragma unroll
        for (int c = 0; c < BN; ++c) {
          const float pv = ex2(fmaf(__uint_as_float(s[c >> 5][c & 31]), sl2, -m_use));
          s[c >> 5][c & 31] = __float_as_uint(pv);
          sum += pv;
        }
        l_run = l_run * alpha + sum;

        if (it > 0) {
          // PV of the previous tile must be done: it reads P and writes O.
          if (!warp_wait(&bars[B_PV_DONE], (it - 1) & 1, abort_flag, p.status)) { ok = false; break; }
          if (__any_sync(0xffffffffu, resc)) {
            tc_fence_after();
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              uint32_t o[32];
              tmem_ld32(tmem + lane_base + kColO + c * 32, o);
              tmem_ld_wait();
#pragma unroll
              for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
              tmem_st32(tmem + lane_base + kColO + c * 32, o);
            }
            tmem_st_wait();
          }
        }
        // P row -> shared memory, bf16, 128-byte swizzled K-major layout
#pragma unroll
        for (int ch = 0; ch < 16; ++ch) {
          const int c0 = ch * 8;
          uint4 v4;
          v4.x = pack_bf16x2(__uint_as_float(s[c0 >> 5][(c0 + 0) & 31]), __uint_as_float(s[c0 >> 5][(c0 + 1) & 31]));
          v4.y = pack_bf16x2(__uint_as_float(s[c0 >> 5][(c0 + 2) & 31]), __uint_as_float(s[c0 >> 5][(c0 + 3) & 31]));
          v4.z = pack_bf16x2(__uint_as_float(s[c0 >> 5][(c0 + 4) & 31]), __uint_as_float(s[c0 >> 5][(c0 + 5) & 31]));
          v4.w = pack_bf16x2(__uint_as_float(s[c0 >> 5][(c0 + 6) & 31]), __uint_as_float(s[c0 >> 5][(c0 + 7) & 31]));
          const int half = ch >> 3;
          const int cc = ch & 7;
          const uint32_t off = half * kHalfBytes + row * 128 + ((cc ^ (row & 7)) << 4);
          *reinterpret_cast<uint4*>(sP + off) = v4;
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars[B_P_FULL]);
      }
    }

    // ---------------------------------------------------------------- epilogue
    const int64_t out_row = ws.out_row0 + q_row0 + tok;
    const int head = kvh * group + (row & (group - 1));
    if (ok && n_iter > 0) {
      ok = warp_wait(&bars[B_PV_DONE], (n_iter - 1) & 1, abort_flag, p.status);
      if (ok) {
        tc_fence_after();
        const float inv_l = (l_run > 0.0f) ? 1.0f / l_run : 0.0f;
        float* dst = p.o_part + (out_row * p.n_h + head) * HD;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t o[32];
          tmem_ld32(tmem + lane_base + kColO + c * 32, o);
          tmem_ld_wait();
          if (row_valid) {
#pragma unroll
            for (int i = 0; i < 32; i += 4) {
              float4 v4 = make_float4(__uint_as_float(o[i]) * inv_l, __uint_as_float(o[i + 1]) * inv_l,
                                      __uint_as_float(o[i + 2]) * inv_l, __uint_as_float(o[i + 3]) * inv_l);
              *reinterpret_cast<float4*>(dst + c * 32 + i) = v4;
            }
          }
        }
      }
    } else if (n_iter == 0 && row_valid) {
      float* dst = p.o_part + (out_row * p.n_h + head) * HD;
#pragma unroll
      for (int i = 0; i < HD; i += 4) *reinterpret_cast<float4*>(dst + i) = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    if (ok && row_valid) {
      const float lse = (l_run > 0.0f) ? (m_run + log2f(l_run)) * 0.69314718055994531f : -INFINITY;
      p.lse_part[out_row * p.n_h + head] = lse;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace tc
}  // namespace cpk
