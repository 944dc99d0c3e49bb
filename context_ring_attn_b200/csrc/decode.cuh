// Split-KV decode: one query token per request against its whole KV cache,
// the keys cut into splits, one partial (O, LSE) per split, then the LSE merge
// ("Context Parallelism for Scalable Million-Token Inference", section 5
// software stack: Flash Decoding; decode itself per "Context Parallelism과
// Expert Parallelism" section 5.2).
//
// The work is HBM-bound (every K/V byte is read once; 16 flop per byte with
// 16 query heads per KV head), so the design goal is streaming K/V at full
// bandwidth with the least fixed cost and no tail.
//
// Units. The query heads of one KV head are taken 16 at a time: a group of
// G <= 16 heads is one unit (rows past G are zero), a group of G = 16u heads
// is u units that each stream the KV head's keys (GQA section 8.2 of the GQA
// page: heads h of one group share the KV head floor(h / G)).
//
// The splits are cut over the whole batch: the keys of all (request, KV head,
// unit) triples, in order, form one flattened sequence of
// Kt = n_kv * U * (offsets[B] - offsets[0]) keys, and warp w of the persistent
// grid of W warps owns the range [w*Kt/W, (w+1)*Kt/W). Every warp thus streams
// the same number of keys (within one key), whatever the mix of request
// lengths, and writes one partial per triple its range overlaps: about
// W + B*n_kv*U partials in all. Warp w's partial for triple bg lands in slot
// w + bg, which is unique because both the ranges and the triples are in
// flattened order.
//
// Each warp works alone: a private ring of 16-key steps of K and V in shared
// memory, filled by 16-byte cp.async copies (whole key rows, fully coalesced)
// that run ahead across triple boundaries. The 16 query heads of a unit share
// every K/V load: they are the 16 rows of m16n8k16 bf16 MMAs (S = q K^T, then
// O += P V with P kept in registers).
#pragma once

#include "common.cuh"

namespace cpk {
namespace dec {

constexpr int kWarps = 8;                 // warps per CTA, one CTA per SM
constexpr int kThreads = kWarps * 32;
constexpr int kStepKeys = 16;             // keys per pipeline step of a warp
constexpr int kWarpBytes = 24 * 1024;     // shared ring per warp (K + V steps in flight)
constexpr int kSmemBytes = kWarps * kWarpBytes;   // 192 KB
constexpr int kMaxSplits = 1024;
constexpr int kUnitRows = 16;             // query heads per unit (MMA rows)

template <int D>
struct Cfg {
  static constexpr int kRowBytes = D * 2;                        // one key row of K (or V), bf16
  static constexpr int kChunks = D / 8;                          // 16-byte chunks per row
  static constexpr int kStepBytes = 2 * kStepKeys * kRowBytes;   // K + V of one step: 4 or 8 KB
  static constexpr int kStages = kWarpBytes / kStepBytes;        // 6 or 3 steps in flight
  static_assert(kStages >= 3, "ring too shallow");
};

struct Params {
  const __nv_bfloat16* q;
  const __nv_bfloat16* k;
  const __nv_bfloat16* v;
  const int64_t* offsets;
  int64_t kv_rows;
  float* o_part;   // [slot][R][D], slot = warp + triple
  float* lse_part; // [slot][R]
  uint32_t* status;
  int32_t batch;
  int32_t n_h;
  int32_t n_kv;
  int32_t group;   // G = n_h / n_kv
  int32_t units;   // U: units per KV head (1 for G <= 16, G / 16 above)
  int32_t rows;    // R: partial rows per slot, min(G, 16)
  int32_t n_warps; // W: warps of the split grid = ranges of the flattened keys
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

// byte offset of 16-byte chunk c of key row r inside a K or V step (rows of
// `row_bytes`, chunks XOR-swizzled by the row so ldmatrix is conflict-free)
template <int D>
__device__ __forceinline__ uint32_t swz(int r, int c) {
  return r * Cfg<D>::kRowBytes + ((c ^ (r & 7)) << 4);
}

// floor(x / y) for 0 <= x < 2^53, 0 < y < 2^53, exactly: the double quotient
// is correctly rounded, so its truncation is the true quotient or one above it
// (when x / y lies just below an integer); one integer check settles it.
__device__ __forceinline__ int64_t floordiv(int64_t x, int64_t y) {
  int64_t q = static_cast<int64_t>(static_cast<double>(x) / static_cast<double>(y));
  if (q * y > x) --q;
  return q;
}

// First key of range w of the flattened sequence of kt keys cut into n ranges.
__device__ __forceinline__ int64_t range_start(int64_t w, int64_t kt, int64_t n) { return floordiv(w * kt, n); }

// The range holding flattened key x (0 <= x < kt): the largest w with start(w) <= x.
__device__ __forceinline__ int64_t range_of(int64_t x, int64_t kt, int64_t n) {
  const int64_t w = floordiv((x + 1) * n - 1, kt);
  return w < n - 1 ? w : n - 1;
}

// Part of one warp's range inside one (request, KV head, unit) triple.
struct Piece {
  int64_t row0;  // first K/V row
  int n_keys;
  int b, g, u, bg;
};

// Walks the triples that overlap [a, e) in flattened order. Every triple it
// looks at is checked (rows inside [0, kv_rows)), so the walk stays in bounds
// even for offsets that break the non-decreasing contract; the merge reports
// those.
struct Walker {
  int bg;        // next triple to look at
  int64_t a, e;  // the range
  int64_t o0;    // offsets[0]

  __device__ __forceinline__ void init(const Params& p, int64_t a_, int64_t e_, int64_t o0_) {
    a = a_;
    e = e_;
    o0 = o0_;
    const int64_t per_tok = static_cast<int64_t>(p.n_kv) * p.units;   // flattened keys per token row
    int lo = 0, hi = p.batch - 1;   // last request whose first flattened key is <= a
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if ((p.offsets[mid] - o0) * per_tok <= a) lo = mid;
      else hi = mid - 1;
    }
    const int64_t base = p.offsets[lo], len = p.offsets[lo + 1] - base;
    int64_t gu = 0;
    if (len > 0) {
      gu = (a - (base - o0) * per_tok) / len;
      gu = gu < 0 ? 0 : (gu >= per_tok ? per_tok - 1 : gu);
    }
    bg = lo * static_cast<int>(per_tok) + static_cast<int>(gu);
  }

  // next non-empty piece; false once the range is done
  __device__ __forceinline__ bool next(const Params& p, Piece& t) {
    const int per_tok = p.n_kv * p.units;
    const int n_bg = p.batch * per_tok;
    while (bg < n_bg) {
      const int cur = bg++;
      const int b = cur / per_tok;
      const int gu = cur - b * per_tok;
      const int64_t base = p.offsets[b], end = p.offsets[b + 1];
      if (!(base >= o0 && end >= base && end <= p.kv_rows)) continue;
      const int64_t len = end - base;
      const int64_t vs = (base - o0) * per_tok + gu * len;
      if (vs >= e) {
        bg = n_bg;
        return false;
      }
      const int64_t lo = a > vs ? a : vs;
      const int64_t hi = e < vs + len ? e : vs + len;
      if (hi > lo) {
        t.row0 = base + (lo - vs);
        t.n_keys = static_cast<int>(hi - lo);
        t.b = b;
        t.g = gu / p.units;
        t.u = gu - t.g * p.units;
        t.bg = cur;
        return true;
      }
    }
    return false;
  }
};

// Let the merge launch (a programmatic dependent of this grid) proceed while
// this grid runs: its blocks are placed as SMs free up and wait in
// griddepcontrol.wait until this grid has finished and its writes are
// visible, so no launch gap separates the two kernels.
__device__ __forceinline__ void allow_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void wait_primary() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

template <int D>
__global__ void __launch_bounds__(kThreads, 1) decode_split_kernel(const __grid_constant__ Params p) {
  using C = Cfg<D>;
  constexpr int KS = D / 16;   // k-steps of the S product
  constexpr int NT = D / 8;    // 8-wide column tiles of O
  extern __shared__ __align__(128) uint8_t smem[];
  allow_dependents();
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int gw = blockIdx.x * kWarps + warp;
  const uint32_t ring = smem_u32(smem) + warp * kWarpBytes;
  const int row_stride = p.n_kv * D;   // elements between consecutive keys
  const float sl2 = p.scale_log2;
  const int gr = lane >> 2;  // fragment row (query head in the unit)
  const int tq = lane & 3;   // fragment column pair

  const int64_t o0 = p.offsets[0];
  const int64_t oB = p.offsets[p.batch];
  if (!(o0 >= 0 && oB >= o0 && oB <= p.kv_rows)) return;   // reported by the merge
  const int64_t kt = (oB - o0) * p.n_kv * p.units;
  if (kt == 0) return;
  const int64_t a = range_start(gw, kt, p.n_warps);
  const int64_t e = range_start(gw + 1, kt, p.n_warps);

  // ---- loader: walks the same pieces and 16-key steps as the compute loop
  Walker lw;
  lw.init(p, a, e, o0);
  Piece lp;
  bool l_more = lw.next(p, lp);
  int l_step = 0;
  int l_slot = 0;
  auto issue_step = [&]() {   // copies of one step, or nothing once the range is done
    if (l_more) {
      const uint32_t sk = ring + l_slot * C::kStepBytes;
      const uint32_t sv = sk + kStepKeys * C::kRowBytes;
#pragma unroll
      for (int i = 0; i < (kStepKeys * C::kChunks) / 32; ++i) {
        const int c = lane + i * 32;   // 16-byte chunk of the step's rows
        const int r = c / C::kChunks;
        const int cc = c % C::kChunks;
        const int kr = l_step * kStepKeys + r;
        const bool in = kr < lp.n_keys;
        const int64_t row = in ? lp.row0 + kr : 0;
        const size_t off = static_cast<size_t>(row) * row_stride + lp.g * D + cc * 8;
        cp_async16(sk + swz<D>(r, cc), p.k + off, in ? 16u : 0u);
        cp_async16(sv + swz<D>(r, cc), p.v + off, in ? 16u : 0u);
      }
      l_slot = (l_slot + 1) % C::kStages;
      if (++l_step * kStepKeys >= lp.n_keys) {
        l_step = 0;
        l_more = lw.next(p, lp);
      }
    }
    cp_async_commit();
  };
#pragma unroll
  for (int s = 0; s < C::kStages - 1; ++s) issue_step();

  Walker cw;
  cw.init(p, a, e, o0);
  Piece t;
  int c_slot = 0;
  while (cw.next(p, t)) {
    const size_t prow = static_cast<size_t>(gw + t.bg) * p.rows;   // first partial row of this piece
    // Q fragments: rows = the unit's query heads (rows past the group are zero), D/16 k-steps
    const int h_first = t.u * kUnitRows;   // first head of the unit within the group
    const bool r0 = h_first + gr < p.group, r1 = h_first + gr + 8 < p.group;
    uint32_t qa[KS][4];
    {
      const __nv_bfloat16* qb = p.q + (static_cast<size_t>(t.b) * p.n_h + t.g * p.group + h_first) * D;
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) {
        const int c0 = ks * 16 + tq * 2;
        qa[ks][0] = r0 ? *reinterpret_cast<const uint32_t*>(qb + gr * D + c0) : 0u;
        qa[ks][1] = r1 ? *reinterpret_cast<const uint32_t*>(qb + (gr + 8) * D + c0) : 0u;
        qa[ks][2] = r0 ? *reinterpret_cast<const uint32_t*>(qb + gr * D + c0 + 8) : 0u;
        qa[ks][3] = r1 ? *reinterpret_cast<const uint32_t*>(qb + (gr + 8) * D + c0 + 8) : 0u;
      }
    }
    float o[NT][4];
#pragma unroll
    for (int j = 0; j < NT; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.0f;
    float m0 = -INFINITY, m1 = -INFINITY;  // running max (log2 units) of rows gr, gr+8
    float l0 = 0.0f, l1 = 0.0f;            // thread-partial running sums
    const int n_steps = (t.n_keys + kStepKeys - 1) / kStepKeys;

    for (int st = 0; st < n_steps; ++st) {
      cp_async_wait<C::kStages - 2>();
      __syncwarp();
      issue_step();
      const uint32_t sk = ring + c_slot * C::kStepBytes;
      const uint32_t sv = sk + kStepKeys * C::kRowBytes;
      c_slot = (c_slot + 1) % C::kStages;

      // S = Q K^T for 16 keys: two n-tiles of 8 keys
      float s[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
      {
        const int mi = lane >> 3, rr = lane & 7;
        const int key = (mi >> 1) * 8 + rr;
#pragma unroll
        for (int ks = 0; ks < KS; ++ks) {
          uint32_t b0, b1, b2, b3;
          ldsm_x4(sk + swz<D>(key, ks * 2 + (mi & 1)), b0, b1, b2, b3);
          mma16816(s[0], qa[ks], b0, b1);
          mma16816(s[1], qa[ks], b2, b3);
        }
      }
      // mask keys past the piece end
      const int valid = t.n_keys - st * kStepKeys;
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
      for (int j = 0; j < NT; ++j) {
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
      // O += P V: D/8 column tiles of 8, two per transposed ldmatrix.x4
      {
        const int mi = lane >> 3, rr = lane & 7;
        const int key = (mi & 1) * 8 + rr;
#pragma unroll
        for (int j = 0; j < NT; j += 2) {
          uint32_t b0, b1, b2, b3;
          ldsm_x4_t(sv + swz<D>(key, j + (mi >> 1)), b0, b1, b2, b3);
          mma16816(o[j], pa, b0, b1);
          mma16816(o[j + 1], pa, b2, b3);
        }
      }
      __syncwarp();   // this slot is refilled only after every lane has read it
    }
    // partial of this piece: normalise and write the unit's rows
    l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
    l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
    const float inv0 = (l0 > 0.0f) ? 1.0f / l0 : 0.0f;
    const float inv1 = (l1 > 0.0f) ? 1.0f / l1 : 0.0f;
    if (r0) {
      float* dst = p.o_part + (prow + gr) * D;
#pragma unroll
      for (int j = 0; j < NT; ++j)
        *reinterpret_cast<float2*>(dst + j * 8 + tq * 2) = make_float2(o[j][0] * inv0, o[j][1] * inv0);
      if (tq == 0) p.lse_part[prow + gr] = (l0 > 0.0f) ? (m0 + log2f(l0)) * 0.69314718055994531f : -INFINITY;
    }
    if (r1) {
      float* dst = p.o_part + (prow + gr + 8) * D;
#pragma unroll
      for (int j = 0; j < NT; ++j)
        *reinterpret_cast<float2*>(dst + j * 8 + tq * 2) = make_float2(o[j][2] * inv1, o[j][3] * inv1);
      if (tq == 0) p.lse_part[prow + gr + 8] = (l1 > 0.0f) ? (m1 + log2f(l1)) * 0.69314718055994531f : -INFINITY;
    }
  }
  cp_async_wait<0>();
}

// Merge of the partials of one (request, head) per CTA. The pieces of triple
// bg come from the warps whose ranges hold its first and last flattened keys
// and every warp in between with a non-empty range; warp w's piece is in slot
// w + bg. The 8 warps take every 8th piece, each keeps an online (max, sum, O)
// with vector loads four pieces deep, and the eight results are combined in
// shared memory. Same formula as the generic merge (LSE weighting, -inf
// partials weigh 0). This kernel also checks the offsets of its request and
// records kStatusInternal for offsets that break the contract. It is launched
// as a programmatic dependent of the split kernel and waits for it first.
constexpr int kMergeThreads = 256;
constexpr int kMergeUnroll = 4;

template <int VW>
struct VecF;
template <>
struct VecF<4> {
  using T = float4;
  static __device__ __forceinline__ T zero() { return make_float4(0.f, 0.f, 0.f, 0.f); }
};
template <>
struct VecF<2> {
  using T = float2;
  static __device__ __forceinline__ T zero() { return make_float2(0.f, 0.f); }
};

__device__ __forceinline__ float4 vfma(float a, float4 x, float4 y) {
  return make_float4(fmaf(a, x.x, y.x), fmaf(a, x.y, y.y), fmaf(a, x.z, y.z), fmaf(a, x.w, y.w));
}
__device__ __forceinline__ float2 vfma(float a, float2 x, float2 y) { return make_float2(fmaf(a, x.x, y.x), fmaf(a, x.y, y.y)); }
__device__ __forceinline__ float4 vscale(float a, float4 x) { return make_float4(a * x.x, a * x.y, a * x.z, a * x.w); }
__device__ __forceinline__ float2 vscale(float a, float2 x) { return make_float2(a * x.x, a * x.y); }

__device__ __forceinline__ void store_vec(__nv_bfloat16* dst, float4 v) {
  uint2 u;
  u.x = pack_bf16x2(v.x, v.y);
  u.y = pack_bf16x2(v.z, v.w);
  *reinterpret_cast<uint2*>(dst) = u;
}
__device__ __forceinline__ void store_vec(__nv_bfloat16* dst, float2 v) {
  *reinterpret_cast<uint32_t*>(dst) = pack_bf16x2(v.x, v.y);
}
__device__ __forceinline__ void store_vec(float* dst, float4 v) { *reinterpret_cast<float4*>(dst) = v; }
__device__ __forceinline__ void store_vec(float* dst, float2 v) { *reinterpret_cast<float2*>(dst) = v; }

// OutT: bf16 for the decoded output, float for a partial (O, LSE) that a
// later LSE merge combines with other ranks' partials. D/32 floats per lane.
template <typename OutT, int D>
__global__ void __launch_bounds__(kMergeThreads, 4) decode_merge_kernel(const __grid_constant__ Params p,
                                                                      OutT* out, float* lse_out) {
  constexpr int VW = D / 32;
  using V = typename VecF<VW>::T;
  __shared__ float sm_m[8], sm_l[8];
  __shared__ V sm_o[8][32];
  wait_primary();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t rh = blockIdx.x;
  const int b = static_cast<int>(rh / p.n_h);
  const int h = static_cast<int>(rh - static_cast<int64_t>(b) * p.n_h);
  const int g = h / p.group;
  const int hr = h - g * p.group;         // head within the group
  const int u = hr / kUnitRows;           // its unit
  const int hl = hr - u * kUnitRows;      // its row in the unit's partials
  const int per_tok = p.n_kv * p.units;
  const int bg = b * per_tok + g * p.units + u;
  const int64_t o0 = p.offsets[0], oB = p.offsets[p.batch];
  const int64_t base = p.offsets[b], end = p.offsets[b + 1];
  const bool ok = o0 >= 0 && oB >= o0 && oB <= p.kv_rows && base >= o0 && end >= base && end <= oB;
  if (!ok && threadIdx.x == 0) atomicOr(p.status, kStatusInternal);
  const int64_t len = ok ? end - base : 0;
  const int64_t kt = (oB - o0) * per_tok;
  const int64_t W = p.n_warps;
  int64_t w_first = 0, n_pieces = 0;
  if (len > 0) {
    const int64_t vs = (base - o0) * per_tok + static_cast<int64_t>(bg - b * per_tok) * len;
    w_first = range_of(vs, kt, W);
    n_pieces = range_of(vs + len - 1, kt, W) - w_first + 1;
  }
  float m = -INFINITY, l = 0.0f;
  V acc = VecF<VW>::zero();
  for (int64_t j0 = warp; j0 < n_pieces; j0 += 8 * kMergeUnroll) {
    // pieces present (a range is empty only when there are fewer keys than ranges)
    uint32_t present = 0;
#pragma unroll 1
    for (int uu = 0; uu < kMergeUnroll; ++uu) {
      const int64_t w = w_first + j0 + uu * 8;
      if (j0 + uu * 8 < n_pieces && (kt >= W || range_start(w, kt, W) < range_start(w + 1, kt, W)))
        present |= 1u << uu;
    }
    V x[kMergeUnroll];
    float lj[kMergeUnroll];
#pragma unroll
    for (int uu = 0; uu < kMergeUnroll; ++uu) {
      lj[uu] = -INFINITY;
      x[uu] = VecF<VW>::zero();
      if (present & (1u << uu)) {
        const int64_t row = (w_first + j0 + uu * 8 + bg) * p.rows + hl;
        lj[uu] = __ldcs(p.lse_part + row);
        x[uu] = __ldcs(reinterpret_cast<const V*>(p.o_part + row * D) + lane);
      }
    }
#pragma unroll
    for (int uu = 0; uu < kMergeUnroll; ++uu) {
      if (lj[uu] == -INFINITY) continue;   // a part at -inf weighs 0 and its O is not read
      const float m_new = fmaxf(m, lj[uu]);
      const float so = __expf(m - m_new);   // 0 when m was -inf
      const float wj = __expf(lj[uu] - m_new);
      l = l * so + wj;
      acc = vfma(wj, x[uu], vscale(so, acc));
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
    V o = VecF<VW>::zero();
    if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < 8; ++w) {
        if (sm_m[w] == -INFINITY) continue;   // a warp that saw no piece
        const float sc = expf(sm_m[w] - M);
        L += sm_l[w] * sc;
        o = vfma(sc, sm_o[w][lane], o);
      }
    }
    const float inv = (L > 0.0f) ? 1.0f / L : 0.0f;
    store_vec(out + rh * D + lane * VW, vscale(inv, o));
    if (lse_out && lane == 0) lse_out[rh] = (L > 0.0f) ? M + logf(L) : -INFINITY;
  }
}

}  // namespace dec
}  // namespace cpk
