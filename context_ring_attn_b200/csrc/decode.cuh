// Split-KV decode: one query token per request against its whole KV cache,
// the keys cut into n_splits splits, one partial (O, LSE) per split, then the
// LSE merge ("Context Parallelism for Scalable Million-Token Inference",
// section 5 software stack: Flash Decoding with 256 splits; decode itself per
// "Context Parallelism과 Expert Parallelism" section 5.2).
//
// The work is HBM-bound (every K/V byte is read once; 16 flop per byte with
// 16 query heads per KV head), so the design goal is streaming K/V at full
// bandwidth: each CTA (4 warps) owns one (split, request, KV head), streams
// 64-key chunks of K and V with 16-byte cp.async copies (fully coalesced rows
// of 256 bytes) into a 3-stage shared-memory ring with a 16-byte-chunk XOR
// swizzle, and each warp takes 16 keys of every chunk. All G <= 16 query
// heads of the KV head share each K/V load: they form the 16 rows of
// m16n8k16 bf16 MMAs (S = q K^T and O += P V with P kept in registers).
// At the end the four warps' (max, sum, O) are combined in shared memory.
#pragma once

#include "common.cuh"

namespace cpk {
namespace dec {

constexpr int kThreads = 128;
constexpr int kChunk = 64;       // keys per pipeline stage
constexpr int kStages = 3;
constexpr int kRowBytes = 256;   // 128 bf16
constexpr int kStageBytes = 2 * kChunk * kRowBytes;  // K + V
constexpr int kSmemBytes = kStages * kStageBytes;    // 96 KB
constexpr int kMaxSplits = 1024;

struct Params {
  const __nv_bfloat16* q;
  const __nv_bfloat16* k;
  const __nv_bfloat16* v;
  const int64_t* offsets;
  int64_t kv_rows;
  float* o_part;   // [n_splits][batch][n_h][128]
  float* lse_part; // [n_splits][batch][n_h]
  uint32_t* status;
  int32_t batch;
  int32_t n_h;
  int32_t n_kv;
  int32_t group;
  int32_t n_splits;
  float scale_log2;
};

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

// D = A(16x16 bf16, row) * B(16x8 bf16, col) + D, fp32
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// byte offset of 16-byte chunk c of key row r inside a K or V stage
__device__ __forceinline__ uint32_t swz(int r, int c) { return r * kRowBytes + ((c ^ (r & 7)) << 4); }

__global__ void __launch_bounds__(kThreads, 2) decode_split_kernel(const __grid_constant__ Params p) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int split = blockIdx.x;
  const int b = blockIdx.y / p.n_kv;
  const int g = blockIdx.y - b * p.n_kv;

  const int64_t base = p.offsets[b];
  const int64_t end = p.offsets[b + 1];
  const bool offsets_ok = base >= 0 && end >= base && end <= p.kv_rows;
  if (!offsets_ok && threadIdx.x == 0) atomicOr(p.status, kStatusInternal);
  const int64_t len = offsets_ok ? end - base : 0;
  const int64_t lo = (static_cast<int64_t>(split) * len) / p.n_splits;
  const int64_t hi = (static_cast<int64_t>(split + 1) * len) / p.n_splits;
  const int n_keys = static_cast<int>(hi - lo);
  const int n_chunks = (n_keys + kChunk - 1) / kChunk;
  const int64_t key0 = base + lo;

  const uint32_t s_base = smem_u32(smem);
  const int row_stride = p.n_kv * 128;  // elements between consecutive keys

  auto load_chunk = [&](int c, int stage) {
    const uint32_t sk = s_base + stage * kStageBytes;
    const uint32_t sv = sk + kChunk * kRowBytes;
#pragma unroll
    for (int i = 0; i < (kChunk * 16) / kThreads; ++i) {
      const int e = threadIdx.x + i * kThreads;  // 16-byte chunk index within the 64x256B tile
      const int r = e >> 4;
      const int cc = e & 15;
      const int kr = c * kChunk + r;
      const bool in = kr < n_keys;
      const int64_t row = in ? key0 + kr : 0;
      const size_t off = static_cast<size_t>(row) * row_stride + g * 128 + cc * 8;
      cp_async16(sk + swz(r, cc), p.k + off, in ? 16u : 0u);
      cp_async16(sv + swz(r, cc), p.v + off, in ? 16u : 0u);
    }
  };

#pragma unroll
  for (int s = 0; s < kStages - 1; ++s) {
    if (s < n_chunks) load_chunk(s, s);
    cp_async_commit();
  }

  // Q fragments: rows = query heads of the group (rows >= G are zero), 8 k-steps of 16 dims.
  const int gr = lane >> 2;  // fragment row
  const int tq = lane & 3;   // fragment column pair
  uint32_t qa[8][4];
  {
    const __nv_bfloat16* qb = p.q + (static_cast<size_t>(b) * p.n_h + g * p.group) * 128;
    const bool r0 = gr < p.group, r1 = gr + 8 < p.group;
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      const int c0 = ks * 16 + tq * 2;
      qa[ks][0] = r0 ? *reinterpret_cast<const uint32_t*>(qb + gr * 128 + c0) : 0u;
      qa[ks][1] = r1 ? *reinterpret_cast<const uint32_t*>(qb + (gr + 8) * 128 + c0) : 0u;
      qa[ks][2] = r0 ? *reinterpret_cast<const uint32_t*>(qb + gr * 128 + c0 + 8) : 0u;
      qa[ks][3] = r1 ? *reinterpret_cast<const uint32_t*>(qb + (gr + 8) * 128 + c0 + 8) : 0u;
    }
  }

  float o[16][4];
#pragma unroll
  for (int j = 0; j < 16; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.0f;
  float m0 = -INFINITY, m1 = -INFINITY;  // running max (log2 units) of rows gr, gr+8
  float l0 = 0.0f, l1 = 0.0f;            // thread-partial running sums
  const float sl2 = p.scale_log2;

  for (int c = 0; c < n_chunks; ++c) {
    cp_async_wait<kStages - 2>();
    __syncthreads();
    if (c + kStages - 1 < n_chunks) load_chunk(c + kStages - 1, (c + kStages - 1) % kStages);
    cp_async_commit();

    const uint32_t sk = s_base + (c % kStages) * kStageBytes;
    const uint32_t sv = sk + kChunk * kRowBytes;
    const int kw = warp * 16;  // this warp's 16 keys of the chunk

    // S = Q K^T for 16 keys: two n-tiles of 8 keys
    float s[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
    {
      const int mi = lane >> 3, rr = lane & 7;
      const int key = kw + (mi >> 1) * 8 + rr;
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        uint32_t b0, b1, b2, b3;
        ldsm_x4(sk + swz(key, ks * 2 + (mi & 1)), b0, b1, b2, b3);
        mma16816(s[0], qa[ks], b0, b1);
        mma16816(s[1], qa[ks], b2, b3);
      }
    }
    // mask keys past the split end
    const int valid = n_keys - c * kChunk - kw;  // keys of this warp's 16 that exist
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      const int col = nt * 8 + tq * 2;
      if (col >= valid) { s[nt][0] = -INFINITY; s[nt][2] = -INFINITY; }
      if (col + 1 >= valid) { s[nt][1] = -INFINITY; s[nt][3] = -INFINITY; }
    }
    float mx0 = fmaxf(fmaxf(s[0][0], s[0][1]), fmaxf(s[1][0], s[1][1]));
    float mx1 = fmaxf(fmaxf(s[0][2], s[0][3]), fmaxf(s[1][2], s[1][3]));
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
    const float n0 = fmaxf(m0, mx0 * sl2);
    const float n1 = fmaxf(m1, mx1 * sl2);
    const float u0 = (n0 == -INFINITY) ? 0.0f : n0;
    const float u1 = (n1 == -INFINITY) ? 0.0f : n1;
    const float a0 = ex2(m0 - u0);
    const float a1 = ex2(m1 - u1);
    m0 = n0;
    m1 = n1;
    float pr[2][4];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      pr[nt][0] = ex2(fmaf(s[nt][0], sl2, -u0));
      pr[nt][1] = ex2(fmaf(s[nt][1], sl2, -u0));
      pr[nt][2] = ex2(fmaf(s[nt][2], sl2, -u1));
      pr[nt][3] = ex2(fmaf(s[nt][3], sl2, -u1));
    }
    l0 = l0 * a0 + pr[0][0] + pr[0][1] + pr[1][0] + pr[1][1];
    l1 = l1 * a1 + pr[0][2] + pr[0][3] + pr[1][2] + pr[1][3];
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      o[j][0] *= a0;
      o[j][1] *= a0;
      o[j][2] *= a1;
      o[j][3] *= a1;
    }
    uint32_t pa[4];
    pa[0] = pack_bf16x2(pr[0][0], pr[0][1]);
    pa[1] = pack_bf16x2(pr[0][2], pr[0][3]);
    pa[2] = pack_bf16x2(pr[1][0], pr[1][1]);
    pa[3] = pack_bf16x2(pr[1][2], pr[1][3]);
    // O += P V: 16 d-tiles of 8, two per transposed ldmatrix.x4
    {
      const int mi = lane >> 3, rr = lane & 7;
      const int key = kw + (mi & 1) * 8 + rr;
#pragma unroll
      for (int j = 0; j < 16; j += 2) {
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(sv + swz(key, j + (mi >> 1)), b0, b1, b2, b3);
        mma16816(o[j], pa, b0, b1);
        mma16816(o[j + 1], pa, b2, b3);
      }
    }
  }
  cp_async_wait<0>();
  __syncthreads();

  // combine the four warps: rows gr and gr+8 of each warp
  float* sm_o = reinterpret_cast<float*>(smem);                 // [4][16][128]
  float* sm_m = sm_o + 4 * 16 * 128;                            // [4][16]
  float* sm_l = sm_m + 4 * 16;                                  // [4][16]
  l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
  l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
  if (tq == 0) {
    sm_m[warp * 16 + gr] = m0;
    sm_m[warp * 16 + gr + 8] = m1;
    sm_l[warp * 16 + gr] = l0;
    sm_l[warp * 16 + gr + 8] = l1;
  }
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    const int col = j * 8 + tq * 2;
    sm_o[(warp * 16 + gr) * 128 + col] = o[j][0];
    sm_o[(warp * 16 + gr) * 128 + col + 1] = o[j][1];
    sm_o[(warp * 16 + gr + 8) * 128 + col] = o[j][2];
    sm_o[(warp * 16 + gr + 8) * 128 + col + 1] = o[j][3];
  }
  __syncthreads();
  {
    const int row = threadIdx.x >> 3;  // 16 rows, 8 threads each, 16 columns per thread
    const int c0 = (threadIdx.x & 7) * 16;
    float mw[4], M = -INFINITY;
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      mw[w] = sm_m[w * 16 + row];
      M = fmaxf(M, mw[w]);
    }
    float L = 0.0f, sc[4];
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      sc[w] = (M == -INFINITY) ? 0.0f : ex2(mw[w] - M);
      L += sm_l[w * 16 + row] * sc[w];
    }
    if (row < p.group) {
      const float inv = (L > 0.0f) ? 1.0f / L : 0.0f;
      const size_t prow = (static_cast<size_t>(split) * p.batch + b) * p.n_h + g * p.group + row;
      float* dst = p.o_part + prow * 128 + c0;
#pragma unroll
      for (int i = 0; i < 16; i += 4) {
        float4 acc;
        acc.x = (sm_o[(0 * 16 + row) * 128 + c0 + i + 0] * sc[0] + sm_o[(1 * 16 + row) * 128 + c0 + i + 0] * sc[1] +
                 sm_o[(2 * 16 + row) * 128 + c0 + i + 0] * sc[2] + sm_o[(3 * 16 + row) * 128 + c0 + i + 0] * sc[3]) * inv;
        acc.y = (sm_o[(0 * 16 + row) * 128 + c0 + i + 1] * sc[0] + sm_o[(1 * 16 + row) * 128 + c0 + i + 1] * sc[1] +
                 sm_o[(2 * 16 + row) * 128 + c0 + i + 1] * sc[2] + sm_o[(3 * 16 + row) * 128 + c0 + i + 1] * sc[3]) * inv;
        acc.z = (sm_o[(0 * 16 + row) * 128 + c0 + i + 2] * sc[0] + sm_o[(1 * 16 + row) * 128 + c0 + i + 2] * sc[1] +
                 sm_o[(2 * 16 + row) * 128 + c0 + i + 2] * sc[2] + sm_o[(3 * 16 + row) * 128 + c0 + i + 2] * sc[3]) * inv;
        acc.w = (sm_o[(0 * 16 + row) * 128 + c0 + i + 3] * sc[0] + sm_o[(1 * 16 + row) * 128 + c0 + i + 3] * sc[1] +
                 sm_o[(2 * 16 + row) * 128 + c0 + i + 3] * sc[2] + sm_o[(3 * 16 + row) * 128 + c0 + i + 3] * sc[3]) * inv;
        *reinterpret_cast<float4*>(dst + i) = acc;
      }
      if ((threadIdx.x & 7) == 0)
        p.lse_part[prow] = (L > 0.0f) ? (M + log2f(L)) * 0.69314718055994531f : -INFINITY;
    }
  }
}

// Merge of the split partials of one (request, head) per CTA: the 8 warps take
// every 8th split, each keeps an online (max, sum, O) over its splits with
// float4 loads eight splits deep, and the eight results are combined in shared
// memory. Same formula as the generic merge (LSE weighting, -inf splits weigh
// 0); more warps per row so the 256 splits stream at full bandwidth.
constexpr int kMergeThreads = 256;
constexpr int kMergeUnroll = 8;

__global__ void __launch_bounds__(kMergeThreads) decode_merge_kernel(const float* __restrict__ o_parts,
                                                                      const float* __restrict__ lse_parts,
                                                                      int n_splits, int64_t n_rowheads,
                                                                      __nv_bfloat16* out, float* lse_out) {
  __shared__ float sm_m[8], sm_l[8];
  __shared__ float4 sm_o[8][32];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t rh = blockIdx.x;
  const int64_t o_stride = n_rowheads * 128;   // floats between splits
  float m = -INFINITY, l = 0.0f;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int j0 = warp; j0 < n_splits; j0 += 8 * kMergeUnroll) {
    float4 x[kMergeUnroll];
    float lj[kMergeUnroll];
#pragma unroll
    for (int u = 0; u < kMergeUnroll; ++u) {
      const int j = j0 + u * 8;
      lj[u] = -INFINITY;
      x[u] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (j < n_splits) {
        lj[u] = __ldg(lse_parts + j * n_rowheads + rh);
        x[u] = __ldcs(reinterpret_cast<const float4*>(o_parts + j * o_stride + rh * 128) + lane);
      }
    }
#pragma unroll
    for (int u = 0; u < kMergeUnroll; ++u) {
      if (lj[u] == -INFINITY) continue;
      const float m_new = fmaxf(m, lj[u]);
      const float so = __expf(m - m_new);   // 0 when m was -inf
      const float wj = __expf(lj[u] - m_new);
      l = l * so + wj;
      acc.x = fmaf(wj, x[u].x, acc.x * so);
      acc.y = fmaf(wj, x[u].y, acc.y * so);
      acc.z = fmaf(wj, x[u].z, acc.z * so);
      acc.w = fmaf(wj, x[u].w, acc.w * so);
      m = m_new;
    }
  }
  if (lane == 0) {
    sm_m[warp] = m;
    sm_l[warp] = l;
  }
  sm_o[warp][lane] = acc;
  __syncthreads();
  if (warp == 0) {
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < 8; ++w) M = fmaxf(M, sm_m[w]);
    float L = 0.0f;
    float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
    if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < 8; ++w) {
        const float sc = expf(sm_m[w] - M);   // 0 for warps that saw no split
        L += sm_l[w] * sc;
        const float4 a = sm_o[w][lane];
        o.x = fmaf(sc, a.x, o.x);
        o.y = fmaf(sc, a.y, o.y);
        o.z = fmaf(sc, a.z, o.z);
        o.w = fmaf(sc, a.w, o.w);
      }
    }
    const float inv = (L > 0.0f) ? 1.0f / L : 0.0f;
    uint2 u;
    u.x = pack_bf16x2(o.x * inv, o.y * inv);
    u.y = pack_bf16x2(o.z * inv, o.w * inv);
    *reinterpret_cast<uint2*>(out + rh * 128 + lane * 4) = u;
    if (lse_out && lane == 0) lse_out[rh] = (L > 0.0f) ? M + logf(L) : -INFINITY;
  }
}

}  // namespace dec
}  // namespace cpk
