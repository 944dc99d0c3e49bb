// LSE merge of attention partials ("merge attention", method page section 5,
// implementation detail 3; the same step closes the pass-KV ring).
//
// Per (row, head): M = max_j lse_j, lse = M + ln sum_j exp(lse_j - M),
// out = sum_j exp(lse_j - lse) * o_j; parts at -inf weigh 0.
//
// HBM-bound: every partial is read once with 16-byte loads and the output is
// written once. One warp per (row, head); lane l owns float4 columns
// l, l+32, ...; the part weights are computed 32 parts at a time, one per lane,
// and broadcast with shuffles while eight parts' loads are in flight.
#pragma once

#include "common.cuh"

namespace cpk {
namespace merge {

constexpr int kThreads = 256;
constexpr int kUnroll = 8;

__device__ __forceinline__ void store4(float* dst, float4 v) { *reinterpret_cast<float4*>(dst) = v; }

__device__ __forceinline__ void store4(__nv_bfloat16* dst, float4 v) {
  uint2 u;
  u.x = pack_bf16x2(v.x, v.y);
  u.y = pack_bf16x2(v.z, v.w);
  *reinterpret_cast<uint2*>(dst) = u;
}

template <typename OutT>
__global__ void __launch_bounds__(kThreads) merge_kernel(const float* __restrict__ o_parts,
                                                          const float* __restrict__ lse_parts, int n_parts,
                                                          int64_t o_stride, int64_t l_stride, int64_t n_rowheads,
                                                          int d, OutT* out, float* lse_out) {
  const int lane = threadIdx.x & 31;
  const int64_t warp_global = (static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x) >> 5;
  const int64_t n_warps = (static_cast<int64_t>(gridDim.x) * kThreads) >> 5;
  const int n_vec = d >> 2;

  for (int64_t rh = warp_global; rh < n_rowheads; rh += n_warps) {
    // pass 1: max and sum of the part LSEs
    float mx = -INFINITY;
    for (int j = lane; j < n_parts; j += 32) mx = fmaxf(mx, lse_parts[j * l_stride + rh]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    float lse;
    if (mx == -INFINITY) {
      lse = -INFINITY;
    } else {
      float sum = 0.0f;
      for (int j = lane; j < n_parts; j += 32) sum += expf(lse_parts[j * l_stride + rh] - mx);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
      lse = mx + logf(sum);
    }
    // pass 2: weighted sum of the part outputs
    for (int vbase = 0; vbase < n_vec; vbase += 32) {
      const int vi = vbase + lane;
      const bool active = vi < n_vec;
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
      if (lse != -INFINITY) {
        for (int jb = 0; jb < n_parts; jb += 32) {
          const int jl = jb + lane;
          const float w_lane = (jl < n_parts) ? expf(lse_parts[jl * l_stride + rh] - lse) : 0.0f;
          const int cnt = min(32, n_parts - jb);
          for (int jj = 0; jj < cnt; jj += kUnroll) {
            float4 x[kUnroll];
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) {
              x[u] = make_float4(0.f, 0.f, 0.f, 0.f);
              if (active && jj + u < cnt)
                x[u] = __ldcs(reinterpret_cast<const float4*>(o_parts + (jb + jj + u) * o_stride + rh * d) + vi);
            }
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) {
              const float w = __shfl_sync(0xffffffffu, w_lane, (jj + u) & 31);
              if (jj + u < cnt && w != 0.0f) {
                acc.x = fmaf(w, x[u].x, acc.x);
                acc.y = fmaf(w, x[u].y, acc.y);
                acc.z = fmaf(w, x[u].z, acc.z);
                acc.w = fmaf(w, x[u].w, acc.w);
              }
            }
          }
        }
      }
      if (active) store4(out + rh * d + vi * 4, acc);
    }
    if (lse_out && lane == 0) lse_out[rh] = lse;
  }
}

}  // namespace merge
}  // namespace cpk
