// LSE merge of attention partials ("merge attention", method page section 5,
// implementation detail 3; the same step closes the pass-KV ring).
//
// Per (row, head): M = max_j lse_j, lse = M + ln sum_j exp(lse_j - M),
// out = sum_j exp(lse_j - lse) * o_j; parts at -inf weigh 0.
//
// HBM-bound: every partial is read once with 16-byte loads and the output is
// written once. The weights are folded in online, eight partial rows per lane
// per round: a warp takes R (row, head) pairs at a time and C = 8 / R parts of
// each per round, loads their C LSEs (broadcast) together with the C float4s
// of each row, then rescales its running (max, sum, O) once per round. So a
// round costs one memory latency whatever n_parts is (R = 1, C = 8 for the
// 8-way merge; R = 4, C = 2 for the running 2-way merge and for a single
// part), and lane l owns the float4 columns l, l+32, ... of the rows.
//
// out may alias o_parts (part 0) and lse_out may alias lse_parts (part 0):
// each lane reads all parts of its columns before writing them, and the LSE
// is written after the warp has read every LSE it needs.
#pragma once

#include "common.cuh"

namespace cpk {
namespace merge {

constexpr int kThreads = 256;
constexpr int kLoads = 8;   // float4 loads per lane per round

// Four consecutive partial elements (fp32, or bf16 partial buffers) as fp32,
// streamed (read once).
__device__ __forceinline__ float4 load4(const float* src) { return __ldcs(reinterpret_cast<const float4*>(src)); }

__device__ __forceinline__ float4 load4(const __nv_bfloat16* src) {
  const uint2 u = __ldcs(reinterpret_cast<const uint2*>(src));
  return make_float4(__uint_as_float(u.x << 16), __uint_as_float(u.x & 0xffff0000u), __uint_as_float(u.y << 16),
                     __uint_as_float(u.y & 0xffff0000u));
}

__device__ __forceinline__ void store4(float* dst, float4 v) { *reinterpret_cast<float4*>(dst) = v; }

__device__ __forceinline__ void store4(__nv_bfloat16* dst, float4 v) {
  uint2 u;
  u.x = pack_bf16x2(v.x, v.y);
  u.y = pack_bf16x2(v.z, v.w);
  *reinterpret_cast<uint2*>(dst) = u;
}

// InT: fp32 partials, or bf16 partial buffers (rounded O, fp32 LSE).
// kInPlace: out / lse_out may be part 0, so the part pointers carry no
// __restrict__ promise; otherwise they do (the compiler may then schedule the
// loads of a round freely around the stores).
template <typename InT, typename OutT, int R, bool kInPlace>
__device__ __forceinline__ void merge_body(const InT* o_parts, const float* lse_parts, int n_parts, int64_t o_stride,
                                           int64_t l_stride, int64_t n_rowheads, int d, OutT* out, float* lse_out) {
  constexpr int C = kLoads / R;
  const int lane = threadIdx.x & 31;
  const int64_t warp_global = (static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x) >> 5;
  const int64_t n_warps = (static_cast<int64_t>(gridDim.x) * kThreads) >> 5;
  const int n_vec = d >> 2;

  for (int64_t rh0 = warp_global * R; rh0 < n_rowheads; rh0 += n_warps * R) {
    float lse_r[R];
    for (int vbase = 0; vbase < n_vec; vbase += 32) {
      const int vi = vbase + lane;
      const bool active = vi < n_vec;
      float m[R], l[R];
      float4 acc[R];
#pragma unroll
      for (int r = 0; r < R; ++r) {
        m[r] = -INFINITY;
        l[r] = 0.0f;
        acc[r] = make_float4(0.f, 0.f, 0.f, 0.f);
      }
      for (int jb = 0; jb < n_parts; jb += C) {
        float lj[R][C];
        float4 x[R][C];
#pragma unroll
        for (int r = 0; r < R; ++r) {
#pragma unroll
          for (int c = 0; c < C; ++c) {
            const int64_t rh = rh0 + r;
            const int j = jb + c;
            lj[r][c] = -INFINITY;
            x[r][c] = make_float4(0.f, 0.f, 0.f, 0.f);
            if (rh < n_rowheads && j < n_parts) {
              lj[r][c] = lse_parts[j * l_stride + rh];
              if (active) x[r][c] = load4(o_parts + j * o_stride + rh * d + vi * 4);
            }
          }
        }
#pragma unroll
        for (int r = 0; r < R; ++r) {
          float mx = lj[r][0];
#pragma unroll
          for (int c = 1; c < C; ++c) mx = fmaxf(mx, lj[r][c]);
          const float m_new = fmaxf(m[r], mx);
          const float mu = (m_new == -INFINITY) ? 0.0f : m_new;   // parts at -inf weigh 0
          const float sc = expf(m[r] - mu);
          l[r] *= sc;
          acc[r].x *= sc;
          acc[r].y *= sc;
          acc[r].z *= sc;
          acc[r].w *= sc;
#pragma unroll
          for (int c = 0; c < C; ++c) {
            // a part at -inf weighs 0: its O row is not used (it may hold anything)
            const bool used = lj[r][c] != -INFINITY;
            const float w = used ? expf(lj[r][c] - mu) : 0.0f;
            const float4 xv = used ? x[r][c] : make_float4(0.f, 0.f, 0.f, 0.f);
            l[r] += w;
            acc[r].x = fmaf(w, xv.x, acc[r].x);
            acc[r].y = fmaf(w, xv.y, acc[r].y);
            acc[r].z = fmaf(w, xv.z, acc[r].z);
            acc[r].w = fmaf(w, xv.w, acc[r].w);
          }
          m[r] = m_new;
        }
      }
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const int64_t rh = rh0 + r;
        const float inv = (l[r] > 0.0f) ? 1.0f / l[r] : 0.0f;
        lse_r[r] = (l[r] > 0.0f) ? m[r] + logf(l[r]) : -INFINITY;
        if (rh < n_rowheads && active)
          store4(out + rh * d + vi * 4, make_float4(acc[r].x * inv, acc[r].y * inv, acc[r].z * inv, acc[r].w * inv));
      }
    }
    __syncwarp();   // every lane has read the LSEs before part 0's may be overwritten
    if (lse_out && lane == 0) {
#pragma unroll
      for (int r = 0; r < R; ++r)
        if (rh0 + r < n_rowheads) lse_out[rh0 + r] = lse_r[r];
    }
  }
}

template <typename InT, typename OutT, int R>
__global__ void __launch_bounds__(kThreads, R <= 2 ? 3 : 2)
    merge_kernel(const InT* __restrict__ o_parts, const float* __restrict__ lse_parts, int n_parts, int64_t o_stride,
                 int64_t l_stride, int64_t n_rowheads, int d, OutT* __restrict__ out, float* __restrict__ lse_out) {
  merge_body<InT, OutT, R, false>(o_parts, lse_parts, n_parts, o_stride, l_stride, n_rowheads, d, out, lse_out);
}

// out and lse_out may be part 0: no aliasing promise.
template <typename InT, typename OutT, int R>
__global__ void __launch_bounds__(kThreads, R <= 2 ? 3 : 2)
    merge_kernel_in_place(const InT* o_parts, const float* lse_parts, int n_parts, int64_t o_stride,
                          int64_t l_stride, int64_t n_rowheads, int d, OutT* out, float* lse_out) {
  merge_body<InT, OutT, R, true>(o_parts, lse_parts, n_parts, o_stride, l_stride, n_rowheads, d, out, lse_out);
}

// The same merge over bf16 partial buffers. A lane loads 8 bf16 (16 bytes) of
// a part per round, so one row-head of D columns takes D/8 lanes and a warp
// covers 32*8/D row-heads at a time; each round brings 8 parts of every
// row-head (as many bytes in flight per lane as the fp32 kernel). Needs
// D % 8 == 0 and D <= 256; out may not alias the parts.
constexpr int kMergeParts16 = 8;

__device__ __forceinline__ void unpack8(const uint4 u, float (&f)[8]) {
  f[0] = __uint_as_float(u.x << 16); f[1] = __uint_as_float(u.x & 0xffff0000u);
  f[2] = __uint_as_float(u.y << 16); f[3] = __uint_as_float(u.y & 0xffff0000u);
  f[4] = __uint_as_float(u.z << 16); f[5] = __uint_as_float(u.z & 0xffff0000u);
  f[6] = __uint_as_float(u.w << 16); f[7] = __uint_as_float(u.w & 0xffff0000u);
}

// Three CTAs per SM (at most 85 registers a thread; 76 used, no spills): more
// loads in flight than two, +5% measured on an 8-way merge of bf16 parts.
template <typename OutT>
__global__ void __launch_bounds__(kThreads, 3)
    merge_bf16_parts_kernel(const __nv_bfloat16* __restrict__ o_parts, const float* __restrict__ lse_parts,
                            int n_parts, int64_t o_stride, int64_t l_stride, int64_t n_rowheads, int d,
                            OutT* __restrict__ out, float* __restrict__ lse_out) {
  const int lane = threadIdx.x & 31;
  const int lanes_per_row = d >> 3;                 // 8 columns per lane
  const int rows_per_warp = 32 / lanes_per_row;
  const int sub = lane / lanes_per_row;             // row-head of this lane within the warp's group
  const int vi = lane - sub * lanes_per_row;        // its 8-column slice
  const bool active = sub < rows_per_warp;
  const int64_t warp_global = (static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x) >> 5;
  const int64_t n_warps = (static_cast<int64_t>(gridDim.x) * kThreads) >> 5;
  for (int64_t rh0 = warp_global * rows_per_warp; rh0 < n_rowheads; rh0 += n_warps * rows_per_warp) {
    const int64_t rh = rh0 + sub;
    const bool mine = active && rh < n_rowheads;
    float m = -INFINITY, l = 0.0f;
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (int jb = 0; jb < n_parts; jb += kMergeParts16) {
      float lj[kMergeParts16];
      uint4 x[kMergeParts16];
#pragma unroll
      for (int c = 0; c < kMergeParts16; ++c) {
        const int j = jb + c;
        lj[c] = -INFINITY;
        x[c] = make_uint4(0u, 0u, 0u, 0u);
        if (mine && j < n_parts) {
          lj[c] = lse_parts[j * l_stride + rh];
          x[c] = __ldcs(reinterpret_cast<const uint4*>(o_parts + j * o_stride + rh * d) + vi);
        }
      }
      float mx = lj[0];
#pragma unroll
      for (int c = 1; c < kMergeParts16; ++c) mx = fmaxf(mx, lj[c]);
      const float m_new = fmaxf(m, mx);
      const float mu = (m_new == -INFINITY) ? 0.0f : m_new;   // parts at -inf weigh 0
      const float sc = expf(m - mu);
      l *= sc;
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] *= sc;
#pragma unroll
      for (int c = 0; c < kMergeParts16; ++c) {
        if (lj[c] == -INFINITY) continue;   // its O row is not used (it may hold anything)
        const float w = expf(lj[c] - mu);
        float f[8];
        unpack8(x[c], f);
        l += w;
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] = fmaf(w, f[i], acc[i]);
      }
      m = m_new;
    }
    if (mine) {
      const float inv = (l > 0.0f) ? 1.0f / l : 0.0f;
      OutT* dst = out + rh * d + vi * 8;
      store4(dst, make_float4(acc[0] * inv, acc[1] * inv, acc[2] * inv, acc[3] * inv));
      store4(dst + 4, make_float4(acc[4] * inv, acc[5] * inv, acc[6] * inv, acc[7] * inv));
      if (lse_out && vi == 0) lse_out[rh] = (l > 0.0f) ? m + logf(l) : -INFINITY;
    }
  }
}

}  // namespace merge
}  // namespace cpk
