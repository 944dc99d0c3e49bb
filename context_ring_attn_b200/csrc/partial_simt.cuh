// Exact fp32 partial attention on the CUDA cores (the fp32 check path).
//
// Same computation and work table as the tensor-core kernel (method page,
// section 3: a query shard against a KV shard, online softmax over KV tiles,
// output normalised within the block plus LSE), in fp32 FMA with the accurate
// expf/logf, so results agree with the fp64 reference to about 1e-6.
//
// One CTA = one query tile of one KV head: up to 64 packed rows
// (floor(64/G) tokens x G heads), two threads per row, each holding half of the
// head dimension of q and of the output accumulator. K/V tiles of 32 keys are
// staged in shared memory; each key's dot product is two half-sums joined by a
// lane shuffle.
#pragma once

#include "common.cuh"
#include "work.cuh"

namespace cpk {
namespace simt {

constexpr int kThreads = 128;
constexpr int kRows = 64;
constexpr int kKeys = 32;

struct Params {
  const float* q;
  const float* k;
  const float* v;
  float* o_part;
  float* lse_part;
  int32_t n_h;
  int32_t n_kv;
  int32_t group;
  int32_t tok_per_tile;
  int32_t causal;
  float scale;
  WorkTable wt;
};

template <int D>
__global__ void __launch_bounds__(kThreads) partial_f32_kernel(const __grid_constant__ Params p) {
  constexpr int H = D / 2;
  __shared__ float sK[kKeys][D];
  __shared__ float sV[kKeys][D];

  int32_t seg, tile;
  locate_tile(p.wt, blockIdx.x, seg, tile);
  const WorkSeg ws = p.wt.segs[seg];
  const cp_range qr = p.wt.ranges[ws.q_range];
  const int kvh = blockIdx.y;
  const int tpt = p.tok_per_tile;
  const int64_t tok0 = static_cast<int64_t>(tile) * tpt;
  const int n_tok = static_cast<int>(min(static_cast<int64_t>(tpt), qr.len - tok0));
  const int64_t q_pos_lo = qr.pos0 + tok0;
  const int64_t q_pos_hi = q_pos_lo + n_tok - 1;

  const int row = threadIdx.x >> 1;
  const int half = threadIdx.x & 1;
  const int tok = row / p.group;
  const int hg = row - tok * p.group;
  const bool row_valid = (row < tpt * p.group) && (tok < n_tok);
  const int64_t q_row = qr.row0 + tok0 + tok;
  const int64_t qpos = q_pos_lo + tok;
  const int head = kvh * p.group + hg;

  float qv[H];
  float acc[H];
#pragma unroll
  for (int i = 0; i < H; ++i) {
    qv[i] = row_valid ? p.q[(q_row * p.n_h + head) * D + half * H + i] : 0.0f;
    acc[i] = 0.0f;
  }
  float m_run = -INFINITY;
  float l_run = 0.0f;

  for (int r = 0; r < ws.kv_count; ++r) {
    const cp_range kr = p.wt.ranges[ws.kv_begin + r];
    if (kr.seq != qr.seq) continue;
    const int64_t nv = visible_keys(kr, q_pos_hi, p.causal);
    for (int64_t k0 = 0; k0 < nv; k0 += kKeys) {
      const int n_valid = static_cast<int>(min(static_cast<int64_t>(kKeys), nv - k0));
      __syncthreads();
      for (int e = threadIdx.x; e < kKeys * D; e += kThreads) {
        const int j = e / D, c = e - (e / D) * D;
        float kx = 0.0f, vx = 0.0f;
        if (j < n_valid) {
          const int64_t src = ((kr.row0 + k0 + j) * p.n_kv + kvh) * D + c;
          kx = p.k[src];
          vx = p.v[src];
        }
        sK[j][c] = kx;
        sV[j][c] = vx;
      }
      __syncthreads();
      float s[kKeys];
      float mx = -INFINITY;
#pragma unroll
      for (int j = 0; j < kKeys; ++j) {
        float part = 0.0f;
#pragma unroll
        for (int i = 0; i < H; ++i) part = fmaf(qv[i], sK[j][half * H + i], part);
        part += __shfl_xor_sync(0xffffffffu, part, 1);
        const int64_t kpos = kr.pos0 + k0 + j;
        const bool vis = (j < n_valid) && (!p.causal || kpos <= qpos);
        s[j] = vis ? part * p.scale : -INFINITY;
        mx = fmaxf(mx, s[j]);
      }
      const float m_new = fmaxf(m_run, mx);
      if (m_new == -INFINITY) continue;  // nothing visible yet for this row
      const float alpha = expf(m_run - m_new);
      l_run *= alpha;
#pragma unroll
      for (int i = 0; i < H; ++i) acc[i] *= alpha;
#pragma unroll
      for (int j = 0; j < kKeys; ++j) {
        const float pj = expf(s[j] - m_new);
        l_run += pj;
#pragma unroll
        for (int i = 0; i < H; ++i) acc[i] = fmaf(pj, sV[j][half * H + i], acc[i]);
      }
      m_run = m_new;
    }
  }

  if (row_valid) {
    const int64_t out_row = ws.out_row0 + q_row;
    const float inv_l = (l_run > 0.0f) ? 1.0f / l_run : 0.0f;
    float* dst = p.o_part + (out_row * p.n_h + head) * D + half * H;
#pragma unroll
    for (int i = 0; i < H; ++i) dst[i] = acc[i] * inv_l;
    if (half == 0) p.lse_part[out_row * p.n_h + head] = (l_run > 0.0f) ? m_run + logf(l_run) : -INFINITY;
  }
}

}  // namespace simt
}  // namespace cpk
