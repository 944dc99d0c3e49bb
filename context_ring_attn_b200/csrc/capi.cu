// Device entry points of libcpattn.so: argument checks, work tables, tensor
// maps and kernel launches. Every check happens before the first launch; the
// library allocates nothing and keeps no state beyond a cached driver entry
// point.
#include <algorithm>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <vector>

#include "cp_attn.h"
#include "common.cuh"
#include "decode.cuh"
#include "merge.cuh"
#include "partial_simt.cuh"
#include "partial_tc.cuh"
#include "work.cuh"

namespace {

using namespace cpk;

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  return fn;
}

inline bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

inline int ilog2_exact(int x) {
  int l = 0;
  while ((1 << l) < x) ++l;
  return ((1 << l) == x) ? l : -1;
}

cp_status last_cuda_status() { return cudaGetLastError() == cudaSuccess ? CP_OK : CP_ERR_CUDA; }

bool range_ok(const cp_range& r) { return r.len >= 0 && r.row0 >= 0 && r.pos0 >= 0 && r.reserved == 0; }

// ---------------------------------------------------------------------------
// work tables
// ---------------------------------------------------------------------------
struct SegSort {
  WorkSeg seg;
  int64_t cost;  // visible keys of the segment's most expensive tile
};

// Split the blocks into launches whose tables fit the kernel parameter space.
// Within a launch, segments run longest-first so the tail of the grid holds
// the cheap tiles.
bool build_tables(const cp_range* ranges, const cp_block* blocks, int32_t n_blocks, int tok_per_tile, int causal,
                  std::vector<WorkTable>& tables) {
  tables.clear();
  std::vector<SegSort> segs;
  std::vector<int32_t> local;  // global range index -> local index, -1 if absent
  std::vector<cp_range> lranges;
  std::vector<int32_t> touched;

  auto flush = [&]() {
    if (segs.empty()) return;
    std::stable_sort(segs.begin(), segs.end(), [](const SegSort& a, const SegSort& b) { return a.cost > b.cost; });
    tables.emplace_back();
    WorkTable& wt = tables.back();
    std::memset(&wt, 0, sizeof(WorkTable));
    wt.n_segs = static_cast<int32_t>(segs.size());
    int32_t acc = 0;
    for (size_t i = 0; i < segs.size(); ++i) {
      wt.segs[i] = segs[i].seg;
      wt.tile_prefix[i] = acc;
      acc += segs[i].seg.n_tiles;
    }
    wt.tile_prefix[segs.size()] = acc;
    wt.total_tiles = acc;
    std::copy(lranges.begin(), lranges.end(), wt.ranges);
    segs.clear();
    lranges.clear();
    for (int32_t g : touched) local[g] = -1;
    touched.clear();
  };

  int32_t max_index = 0;
  for (int32_t b = 0; b < n_blocks; ++b)
    max_index = std::max(max_index, std::max(blocks[b].q_begin + blocks[b].q_count, blocks[b].kv_begin + blocks[b].kv_count));
  local.assign(max_index + 1, -1);

  for (int32_t b = 0; b < n_blocks; ++b) {
    const cp_block& bl = blocks[b];
    if (bl.q_count > kMaxSegs || bl.q_count + bl.kv_count > kMaxRanges) return false;
    // ranges this block needs that the current table lacks
    int need = 0;
    for (int32_t j = 0; j < bl.q_count; ++j) need += local[bl.q_begin + j] < 0;
    bool kv_contiguous = true;
    for (int32_t j = 0; j < bl.kv_count; ++j) {
      const int32_t g = bl.kv_begin + j;
      if (local[g] < 0) ++need;
      else if (j > 0 && local[g] != local[g - 1] + 1) kv_contiguous = false;
    }
    if (!kv_contiguous) need += bl.kv_count;  // KV slice is re-added contiguously
    if (static_cast<int>(lranges.size()) + need > kMaxRanges || static_cast<int>(segs.size()) + bl.q_count > kMaxSegs)
      flush();
    // KV slice: contiguous in the local table
    int32_t kv_local = -1;
    {
      bool have = bl.kv_count > 0 && local[bl.kv_begin] >= 0;
      for (int32_t j = 1; j < bl.kv_count && have; ++j)
        have = local[bl.kv_begin + j] == local[bl.kv_begin] + j;
      if (have) {
        kv_local = local[bl.kv_begin];
      } else {
        kv_local = static_cast<int32_t>(lranges.size());
        for (int32_t j = 0; j < bl.kv_count; ++j) {
          const int32_t g = bl.kv_begin + j;
          lranges.push_back(ranges[g]);
          if (local[g] < 0) touched.push_back(g);
          local[g] = kv_local + j;
        }
      }
    }
    for (int32_t j = 0; j < bl.q_count; ++j) {
      const int32_t g = bl.q_begin + j;
      const cp_range& qr = ranges[g];
      if (qr.len == 0) continue;
      int32_t ql = local[g];
      if (ql < 0) {
        ql = static_cast<int32_t>(lranges.size());
        lranges.push_back(qr);
        local[g] = ql;
        touched.push_back(g);
      }
      const int64_t n_tiles = (qr.len + tok_per_tile - 1) / tok_per_tile;
      int64_t cost = 0;
      for (int32_t r = 0; r < bl.kv_count; ++r) {
        const cp_range& kr = ranges[bl.kv_begin + r];
        if (kr.seq == qr.seq) cost += visible_keys(kr, qr.pos0 + qr.len - 1, causal);
      }
      SegSort s;
      s.seg.q_range = ql;
      s.seg.kv_begin = kv_local;
      s.seg.kv_count = bl.kv_count;
      s.seg.n_tiles = static_cast<int32_t>(n_tiles);
      s.seg.out_row0 = bl.out_row0;
      s.cost = cost;
      segs.push_back(s);
    }
  }
  flush();
  return true;
}

// Tensor maps (bf16, 128-byte swizzle): Q as [rows][N_KV][G][HD] with a box of
// 64 columns x G heads x 1 KV head x 128/G tokens (128 packed query rows);
// K and V as [rows][N_KV][HD] with a box of 64 columns x 1 KV head x
// kv_box_rows keys.
bool make_qkv_maps(CUtensorMap* tm_q, CUtensorMap* tm_k, CUtensorMap* tm_v, const void* q, const void* k,
                   const void* v, int64_t q_rows, int64_t kv_rows, int n_h, int n_kv, int group, int hd,
                   int kv_box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const cuuint32_t estr4[4] = {1, 1, 1, 1};
  const cuuint64_t row_bytes = static_cast<cuuint64_t>(hd) * 2;
  {
    const cuuint64_t dims[4] = {static_cast<cuuint64_t>(hd), static_cast<cuuint64_t>(group),
                                static_cast<cuuint64_t>(n_kv), static_cast<cuuint64_t>(q_rows)};
    const cuuint64_t strides[3] = {row_bytes, static_cast<cuuint64_t>(group) * row_bytes,
                                   static_cast<cuuint64_t>(n_h) * row_bytes};
    const cuuint32_t box[4] = {64, static_cast<cuuint32_t>(group), 1, static_cast<cuuint32_t>(128 / group)};
    if (enc(tm_q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(q), dims, strides, box, estr4,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return false;
  }
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(hd), static_cast<cuuint64_t>(n_kv),
                              static_cast<cuuint64_t>(kv_rows)};
  const cuuint64_t strides[2] = {row_bytes, static_cast<cuuint64_t>(n_kv) * row_bytes};
  const void* src[2] = {k, v};
  CUtensorMap* dst[2] = {tm_k, tm_v};
  for (int i = 0; i < 2; ++i) {
    const cuuint32_t box[3] = {64, 1, static_cast<cuuint32_t>(kv_box_rows)};
    if (enc(dst[i], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(src[i]), dims, strides, box, estr4,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return false;
  }
  return true;
}

constexpr size_t kStatusBytes = 256;

inline size_t round256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// Ranges of the flattened decode keys (one per warp of the persistent split
// grid): dec::kWarps per SM of the current device, at most n_splits per flattened
// (request, KV head, unit) triple.
cp_status decode_ranges(int32_t n_splits, int32_t batch, int32_t triples_per_request, int32_t* n_warps) {
  int n_sm = 0, dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return CP_ERR_CUDA;
  const int64_t want = (static_cast<int64_t>(n_splits) * batch * triples_per_request + dec::kWarps - 1) / dec::kWarps;
  *n_warps = static_cast<int32_t>(std::max<int64_t>(1, std::min<int64_t>(n_sm, want)) * dec::kWarps);
  return CP_OK;
}

// A decode call after its arguments have been checked: the unit split of the
// query heads and the grid and workspace sizes it will use.
struct DecodeShape {
  int32_t group;    // G = n_h / n_kv
  int32_t units;    // U: 16-head units per KV head (1 for G <= 16)
  int32_t rows;     // R: partial rows per slot, min(G, 16)
  int32_t n_warps;  // W: ranges of the flattened keys
  size_t part_rows; // (W + batch * n_kv * U) * R
  size_t bytes;     // workspace bytes the call uses (never above cp_workspace_size)
};

// Every argument check of cp_decode / cp_decode_partial / cp_decode_static,
// with nothing launched, nothing written and no CUDA call; fills in the unit
// split of the query heads.
cp_status decode_validate(const void* q, const void* k, const void* v, cp_dtype dtype, const int64_t* kv_offsets,
                          int32_t batch, int64_t kv_rows, int32_t n_h, int32_t n_kv, int32_t d, int32_t n_splits,
                          float softmax_scale, const void* out, bool out_f32, DecodeShape* s) {
  if (!q || !k || !v || !kv_offsets || !out) return CP_ERR_INVALID_ARG;
  if (batch < 0 || kv_rows < 0 || n_h < 1 || n_kv < 1 || d < 1 || n_h % n_kv) return CP_ERR_INVALID_ARG;
  if (!(softmax_scale > 0.0f) || !(softmax_scale < INFINITY)) return CP_ERR_INVALID_ARG;
  if (n_splits < 1 || n_splits > dec::kMaxSplits) return CP_ERR_UNSUPPORTED;
  const int group = n_h / n_kv;
  if (dtype != CP_BF16 || (d != 64 && d != 128)) return CP_ERR_UNSUPPORTED;
  if (group > 128 || (group > dec::kUnitRows && group % dec::kUnitRows != 0)) return CP_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(batch) * n_h > 0x7fffffffLL) return CP_ERR_UNSUPPORTED;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, out_f32 ? 16 : 8) || !aligned(kv_offsets, 8))
    return CP_ERR_INVALID_ARG;
  s->group = group;
  s->units = group > dec::kUnitRows ? group / dec::kUnitRows : 1;
  s->rows = group > dec::kUnitRows ? dec::kUnitRows : group;
  s->n_warps = 0;
  s->part_rows = 0;
  s->bytes = 0;
  return CP_OK;
}

// Partial rows and workspace bytes of a decode with n_warps ranges.
void decode_sizes(DecodeShape* s, int32_t n_warps, int32_t batch, int32_t n_kv, int32_t d) {
  s->n_warps = n_warps;
  s->part_rows = (static_cast<size_t>(n_warps) + static_cast<size_t>(batch) * n_kv * s->units) * s->rows;
  s->bytes = kStatusBytes + round256(s->part_rows * d * 4) + round256(s->part_rows * 4);
}

// Grid of the current device (the one CUDA query of a decode call before its
// launches) and the sizes that follow from it.
cp_status decode_grid(DecodeShape* s, int32_t n_splits, int32_t batch, int64_t kv_rows, int32_t n_kv, int32_t d) {
  int32_t n_warps = 0;
  if (decode_ranges(n_splits, batch, n_kv * s->units, &n_warps) != CP_OK) return CP_ERR_CUDA;
  // the range arithmetic is exact while (flattened keys) x W stays below 2^53
  const double kt_max = static_cast<double>(kv_rows) * n_kv * s->units;
  if (kt_max * (static_cast<double>(n_warps) + 1.0) >= 9007199254740992.0) return CP_ERR_UNSUPPORTED;
  decode_sizes(s, n_warps, batch, n_kv, d);
  return CP_OK;
}

// Launch the split kernel and, as its programmatic dependent, the merge. The
// status word is at `ws`, the partials follow it.
template <int D>
cp_status decode_launch_d(const DecodeShape& s, const void* q, const void* k, const void* v,
                                 const int64_t* kv_offsets, int32_t batch, int64_t kv_rows, int32_t n_h, int32_t n_kv,
                                 float softmax_scale, void* out, bool out_f32, float* lse_out, void* ws,
                                 cudaStream_t stream) {
  float* o_ws = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + kStatusBytes);
  float* l_ws = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + kStatusBytes + round256(s.part_rows * D * 4));
  dec::Params p;
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.k = static_cast<const __nv_bfloat16*>(k);
  p.v = static_cast<const __nv_bfloat16*>(v);
  p.offsets = kv_offsets;
  p.kv_rows = kv_rows;
  p.o_part = o_ws;
  p.lse_part = l_ws;
  p.status = static_cast<uint32_t*>(ws);
  p.batch = batch;
  p.n_h = n_h;
  p.n_kv = n_kv;
  p.group = s.group;
  p.units = s.units;
  p.rows = s.rows;
  p.n_warps = s.n_warps;
  p.scale_log2 = softmax_scale * 1.4426950408889634f;
  if (cudaFuncSetAttribute(dec::decode_split_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           dec::kSmemBytes) != cudaSuccess)
    return CP_ERR_CUDA;
  // persistent: up to one CTA per SM, each warp streaming one range of the flattened keys
  dec::decode_split_kernel<D><<<static_cast<unsigned>(s.n_warps / dec::kWarps), dec::kThreads, dec::kSmemBytes, stream>>>(p);
  if (last_cuda_status() != CP_OK) return CP_ERR_CUDA;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(static_cast<int64_t>(batch) * n_h));
  cfg.blockDim = dim3(dec::kMergeThreads);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e;
  if (out_f32)
    e = cudaLaunchKernelEx(&cfg, dec::decode_merge_kernel<float, D>, p, static_cast<float*>(out), lse_out);
  else
    e = cudaLaunchKernelEx(&cfg, dec::decode_merge_kernel<__nv_bfloat16, D>, p, static_cast<__nv_bfloat16*>(out),
                           lse_out);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return CP_ERR_CUDA;
  }
  return last_cuda_status();
}

cp_status decode_launch(const DecodeShape& s, const void* q, const void* k, const void* v,
                               const int64_t* kv_offsets, int32_t batch, int64_t kv_rows, int32_t n_h, int32_t n_kv,
                               int32_t d, float softmax_scale, void* out, bool out_f32, float* lse_out, void* ws,
                               cudaStream_t stream) {
  if (d == 64)
    return decode_launch_d<64>(s, q, k, v, kv_offsets, batch, kv_rows, n_h, n_kv, softmax_scale, out, out_f32,
                               lse_out, ws, stream);
  return decode_launch_d<128>(s, q, k, v, kv_offsets, batch, kv_rows, n_h, n_kv, softmax_scale, out, out_f32,
                              lse_out, ws, stream);
}

// One launch of the tensor-core partial kernel per work table.
template <int HD>
cp_status launch_partial_tc(tc::Params& params, const std::vector<WorkTable>& tables, int n_kv, cudaStream_t stream) {
  if (cudaFuncSetAttribute(tc::partial_bf16_kernel<HD>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           tc::Cfg<HD>::kSmemBytes) != cudaSuccess)
    return CP_ERR_CUDA;
  for (const WorkTable& wt : tables) {
    if (wt.total_tiles == 0) continue;
    std::memcpy(&params.wt, &wt, sizeof(WorkTable));
    dim3 grid(wt.total_tiles, n_kv);
    tc::partial_bf16_kernel<HD><<<grid, tc::kThreads, tc::Cfg<HD>::kSmemBytes, stream>>>(params);
    if (last_cuda_status() != CP_OK) return CP_ERR_CUDA;
  }
  return CP_OK;
}

}  // namespace

extern "C" {

size_t cp_workspace_size(cp_op op, int64_t rows, int32_t n_h, int32_t d, int32_t n_splits) {
  if (op == CP_OP_DECODE) {
    if (rows < 0 || n_h < 1 || d < 1 || n_splits < 1) return kStatusBytes;
    // at most n_splits*batch*n_kv + 7 ranges + batch*n_kv pairs, G = n_h/n_kv rows each
    const size_t part = (static_cast<size_t>(n_splits) + 1) * static_cast<size_t>(rows) * static_cast<size_t>(n_h) +
                        7 * static_cast<size_t>(n_h);
    return kStatusBytes + round256(part * static_cast<size_t>(d) * 4) + round256(part * 4);
  }
  return kStatusBytes;
}

namespace {
// One thread waits on a barrier that nothing arrives at, through the same
// bounded wait as every kernel of the library, with a short budget.
__global__ void wait_selftest_kernel(uint32_t* status, uint64_t budget_ns) {
  __shared__ uint64_t bar;
  __shared__ uint32_t abort_flag;
  if (threadIdx.x != 0) return;
  cpk::mbar_init(&bar, 1u);
  abort_flag = 0u;
  cpk::fence_mbar_init();
  (void)cpk::mbar_wait(&bar, 0u, &abort_flag, status, budget_ns);
}
}  // namespace

cp_status cp_wait_selftest(void* workspace, size_t ws_bytes, uint64_t budget_ns, void* cuda_stream) {
  if (!workspace || ws_bytes < kStatusBytes || !aligned(workspace, 256)) return CP_ERR_WORKSPACE;
  if (budget_ns == 0 || budget_ns > cpk::kWaitBudgetNs) return CP_ERR_INVALID_ARG;
  wait_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(cuda_stream)>>>(static_cast<uint32_t*>(workspace),
                                                                              budget_ns);
  return last_cuda_status();
}

cp_status cp_reset_status(void* workspace, void* cuda_stream) {
  if (!workspace) return CP_ERR_WORKSPACE;
  if (cudaMemsetAsync(workspace, 0, sizeof(uint32_t), static_cast<cudaStream_t>(cuda_stream)) != cudaSuccess)
    return CP_ERR_CUDA;
  return CP_OK;
}

cp_status cp_check_status(const void* workspace, void* cuda_stream) {
  if (!workspace) return CP_ERR_WORKSPACE;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(cuda_stream)) != cudaSuccess) return CP_ERR_CUDA;
  uint32_t word = 0;
  if (cudaMemcpy(&word, workspace, sizeof(word), cudaMemcpyDeviceToHost) != cudaSuccess) return CP_ERR_CUDA;
  if (word & kStatusTimeout) return CP_ERR_TIMEOUT;
  if (word & kStatusInternal) return CP_ERR_INTERNAL;
  return CP_OK;
}

static cp_status partial_impl(const void* q, const void* k, const void* v, cp_dtype dtype, int64_t q_rows,
                              int64_t kv_rows, int32_t n_h, int32_t n_kv, int32_t d, float softmax_scale,
                              int32_t causal, const cp_range* ranges, int32_t n_ranges, const cp_block* blocks,
                              int32_t n_blocks, float* o_part, float* lse_part, int64_t out_rows, int32_t accumulate,
                              void* out_final, void* workspace, size_t ws_bytes, void* cuda_stream) {
  // ---- arguments (o_part is not read or written when every row goes to out_final unmerged)
  if (!q || !k || !v || !lse_part || (!o_part && (accumulate || !out_final))) return CP_ERR_INVALID_ARG;
  const bool fused = accumulate != 0 || out_final != nullptr;
  if (fused && dtype != CP_BF16) return CP_ERR_UNSUPPORTED;
  if (out_final && !aligned(out_final, 16)) return CP_ERR_INVALID_ARG;
  if (n_blocks < 0 || n_ranges < 0 || (n_blocks > 0 && (!ranges || !blocks))) return CP_ERR_INVALID_ARG;
  if (n_h < 1 || n_kv < 1 || d < 1 || q_rows < 0 || kv_rows < 0 || out_rows < 0) return CP_ERR_INVALID_ARG;
  if (!(softmax_scale > 0.0f) || !(softmax_scale < INFINITY)) return CP_ERR_INVALID_ARG;
  if (n_h % n_kv != 0) return CP_ERR_INVALID_ARG;
  if (!workspace || ws_bytes < kStatusBytes || !aligned(workspace, 256)) return CP_ERR_WORKSPACE;
  const int group = n_h / n_kv;
  if (dtype == CP_BF16) {
    if ((d != 64 && d != 128) || ilog2_exact(group) < 0 || group > 128) return CP_ERR_UNSUPPORTED;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16)) return CP_ERR_INVALID_ARG;
    if (q_rows >= (int64_t(1) << 31) || kv_rows >= (int64_t(1) << 31)) return CP_ERR_UNSUPPORTED;
  } else if (dtype == CP_F32) {
    if ((d != 64 && d != 128) || group > simt::kRows) return CP_ERR_UNSUPPORTED;
    if (!aligned(q, 4) || !aligned(k, 4) || !aligned(v, 4)) return CP_ERR_INVALID_ARG;
  } else {
    return CP_ERR_UNSUPPORTED;
  }
  if ((o_part && !aligned(o_part, 16)) || !aligned(lse_part, 4)) return CP_ERR_INVALID_ARG;
  for (int32_t b = 0; b < n_blocks; ++b) {
    const cp_block& bl = blocks[b];
    if (bl.q_begin < 0 || bl.q_count < 0 || bl.kv_begin < 0 || bl.kv_count < 0) return CP_ERR_INVALID_ARG;
    if (int64_t(bl.q_begin) + bl.q_count > n_ranges || int64_t(bl.kv_begin) + bl.kv_count > n_ranges)
      return CP_ERR_INVALID_ARG;
    for (int32_t j = 0; j < bl.q_count; ++j) {
      const cp_range& r = ranges[bl.q_begin + j];
      if (!range_ok(r) || r.row0 + r.len > q_rows) return CP_ERR_INVALID_ARG;
      if (r.len > 0 && (bl.out_row0 + r.row0 < 0 || bl.out_row0 + r.row0 + r.len > out_rows)) return CP_ERR_INVALID_ARG;
    }
    for (int32_t j = 0; j < bl.kv_count; ++j) {
      const cp_range& r = ranges[bl.kv_begin + j];
      if (!range_ok(r) || r.row0 + r.len > kv_rows) return CP_ERR_INVALID_ARG;
    }
  }
  if (fused) {
    // each output row may belong to at most one block of the call (read-modify-write)
    std::vector<std::pair<int64_t, int64_t>> rows;
    for (int32_t b = 0; b < n_blocks; ++b)
      for (int32_t j = 0; j < blocks[b].q_count; ++j) {
        const cp_range& r = ranges[blocks[b].q_begin + j];
        if (r.len > 0) rows.emplace_back(blocks[b].out_row0 + r.row0, blocks[b].out_row0 + r.row0 + r.len);
      }
    std::sort(rows.begin(), rows.end());
    for (size_t i = 1; i < rows.size(); ++i)
      if (rows[i].first < rows[i - 1].second) return CP_ERR_INVALID_ARG;
  }
  // tokens per CTA tile: the tensor-core kernel takes two 128-row query tiles per CTA
  const int tok_per_tile = (dtype == CP_BF16) ? tc::kQTiles * (128 / group) : simt::kRows / group;
  std::vector<WorkTable> tables;
  if (!build_tables(ranges, blocks, n_blocks, tok_per_tile, causal != 0, tables)) return CP_ERR_UNSUPPORTED;

  int64_t total_tiles = 0;
  for (const WorkTable& wt : tables) total_tiles += wt.total_tiles;
  if (total_tiles == 0) return CP_OK;

  cudaStream_t stream = static_cast<cudaStream_t>(cuda_stream);
  uint32_t* status = static_cast<uint32_t*>(workspace);
  const float log2e = 1.4426950408889634f;

  if (dtype == CP_BF16) {
    static tc::Params params;  // large: kept off the stack; copied at launch
    static std::mutex mu;
    std::lock_guard<std::mutex> lock(mu);
    if (!make_qkv_maps(&params.tm_q, &params.tm_k, &params.tm_v, q, k, v, q_rows, kv_rows, n_h, n_kv, group, d,
                       tc::BN))
      return CP_ERR_CUDA;
    params.o_part = o_part;
    params.lse_part = lse_part;
    params.out_final = static_cast<__nv_bfloat16*>(out_final);
    params.accumulate = accumulate != 0;
    params.status = status;
    params.n_h = n_h;
    params.log2_group = ilog2_exact(group);
    params.causal = causal != 0;
    params.scale_log2 = softmax_scale * log2e;
    const cp_status st = d == 64 ? launch_partial_tc<64>(params, tables, n_kv, stream)
                                 : launch_partial_tc<128>(params, tables, n_kv, stream);
    if (st != CP_OK) return st;
  } else {
    static simt::Params params;
    static std::mutex mu;
    std::lock_guard<std::mutex> lock(mu);
    params.q = static_cast<const float*>(q);
    params.k = static_cast<const float*>(k);
    params.v = static_cast<const float*>(v);
    params.o_part = o_part;
    params.lse_part = lse_part;
    params.n_h = n_h;
    params.n_kv = n_kv;
    params.group = group;
    params.tok_per_tile = tok_per_tile;
    params.causal = causal != 0;
    params.scale = softmax_scale;
    for (const WorkTable& wt : tables) {
      if (wt.total_tiles == 0) continue;
      std::memcpy(&params.wt, &wt, sizeof(WorkTable));
      dim3 grid(wt.total_tiles, n_kv);
      if (d == 64)
        simt::partial_f32_kernel<64><<<grid, simt::kThreads, 0, stream>>>(params);
      else
        simt::partial_f32_kernel<128><<<grid, simt::kThreads, 0, stream>>>(params);
      if (last_cuda_status() != CP_OK) return CP_ERR_CUDA;
    }
  }
  return CP_OK;
}

cp_status cp_attn_partial(const void* q, const void* k, const void* v, cp_dtype dtype, int64_t q_rows,
                          int64_t kv_rows, int32_t n_h, int32_t n_kv, int32_t d, float softmax_scale, int32_t causal,
                          const cp_range* ranges, int32_t n_ranges, const cp_block* blocks, int32_t n_blocks,
                          float* o_part, float* lse_part, int64_t out_rows, void* workspace, size_t ws_bytes,
                          void* cuda_stream) {
  return partial_impl(q, k, v, dtype, q_rows, kv_rows, n_h, n_kv, d, softmax_scale, causal, ranges, n_ranges, blocks,
                      n_blocks, o_part, lse_part, out_rows, 0, nullptr, workspace, ws_bytes, cuda_stream);
}

cp_status cp_attn_partial_fused(const void* q, const void* k, const void* v, cp_dtype dtype, int64_t q_rows,
                                int64_t kv_rows, int32_t n_h, int32_t n_kv, int32_t d, float softmax_scale,
                                int32_t causal, const cp_range* ranges, int32_t n_ranges, const cp_block* blocks,
                                int32_t n_blocks, float* o_acc, float* lse_acc, int64_t out_rows, int32_t accumulate,
                                void* out, void* workspace, size_t ws_bytes, void* cuda_stream) {
  return partial_impl(q, k, v, dtype, q_rows, kv_rows, n_h, n_kv, d, softmax_scale, causal, ranges, n_ranges, blocks,
                      n_blocks, o_acc, lse_acc, out_rows, accumulate, out, workspace, ws_bytes, cuda_stream);
}

cp_status cp_attn_partial_bf16_parts(const void* q, const void* k, const void* v, cp_dtype dtype, int64_t q_rows,
                                     int64_t kv_rows, int32_t n_h, int32_t n_kv, int32_t d, float softmax_scale,
                                     int32_t causal, const cp_range* ranges, int32_t n_ranges, const cp_block* blocks,
                                     int32_t n_blocks, void* o_part, float* lse_part, int64_t out_rows, void* workspace,
                                     size_t ws_bytes, void* cuda_stream) {
  if (!o_part) return CP_ERR_INVALID_ARG;
  return partial_impl(q, k, v, dtype, q_rows, kv_rows, n_h, n_kv, d, softmax_scale, causal, ranges, n_ranges, blocks,
                      n_blocks, nullptr, lse_part, out_rows, 0, o_part, workspace, ws_bytes, cuda_stream);
}

static cp_status merge_impl(const void* o_parts, cp_dtype parts_dtype, const float* lse_parts, int32_t n_parts,
                            int64_t part_stride_rows, int64_t rows, int32_t n_h, int32_t d, void* out,
                            cp_dtype out_dtype, float* lse_out, void* cuda_stream) {
  if (!o_parts || !lse_parts || !out) return CP_ERR_INVALID_ARG;
  if (n_parts < 1 || rows < 0 || n_h < 1 || d < 4 || (d & 3)) return CP_ERR_INVALID_ARG;
  if (n_parts > 1 && part_stride_rows < rows) return CP_ERR_INVALID_ARG;
  if (!aligned(o_parts, parts_dtype == CP_F32 ? 16 : 8) || !aligned(lse_parts, 4)) return CP_ERR_INVALID_ARG;
  if (out_dtype == CP_F32) {
    if (!aligned(out, 16)) return CP_ERR_INVALID_ARG;
  } else if (out_dtype == CP_BF16) {
    if (!aligned(out, 8)) return CP_ERR_INVALID_ARG;
  } else {
    return CP_ERR_UNSUPPORTED;
  }
  const int64_t n_rowheads = rows * n_h;
  if (n_rowheads == 0) return CP_OK;
  cudaStream_t stream = static_cast<cudaStream_t>(cuda_stream);
  const int64_t o_stride = part_stride_rows * n_h * d;
  const int64_t l_stride = part_stride_rows * n_h;
  // (row, head) pairs per warp and round: 8 four-element loads per lane split over the parts
  const int c = n_parts > 4 ? 8 : n_parts > 2 ? 4 : 2;
  const int r = 8 / c;
  const int64_t warps_per_block = merge::kThreads / 32;
  int64_t grid = (n_rowheads + warps_per_block * r - 1) / (warps_per_block * r);
  grid = std::min<int64_t>(grid, 148 * 32);
  const unsigned g = static_cast<unsigned>(grid);
  const unsigned t = merge::kThreads;
  // out on part 0 (or lse_out on LSE part 0): the in-place instantiation
  const uintptr_t o_lo = reinterpret_cast<uintptr_t>(o_parts), o_hi = o_lo + static_cast<uintptr_t>(rows * n_h * d) *
                                                                                  (parts_dtype == CP_F32 ? 4 : 2);
  const uintptr_t ob = reinterpret_cast<uintptr_t>(out);
  const uintptr_t l_lo = reinterpret_cast<uintptr_t>(lse_parts), l_hi = l_lo + static_cast<uintptr_t>(rows * n_h) * 4;
  const uintptr_t lb = reinterpret_cast<uintptr_t>(lse_out);
  const bool in_place = (ob >= o_lo && ob < o_hi) || (lse_out && lb >= l_lo && lb < l_hi);
#define CP_MERGE_LAUNCH(InT, OutT, R_)                                                                              \
  do {                                                                                                              \
    if (in_place)                                                                                                   \
      merge::merge_kernel_in_place<InT, OutT, R_><<<g, t, 0, stream>>>(                                           \
          static_cast<const InT*>(o_parts), lse_parts, n_parts, o_stride, l_stride, n_rowheads, d,                \
          static_cast<OutT*>(out), lse_out);                                                                        \
    else                                                                                                            \
      merge::merge_kernel<InT, OutT, R_><<<g, t, 0, stream>>>(static_cast<const InT*>(o_parts), lse_parts,       \
                                                              n_parts, o_stride, l_stride, n_rowheads, d,         \
                                                              static_cast<OutT*>(out), lse_out);                  \
  } while (0)
#define CP_MERGE_BY_R(InT, OutT)                \
  do {                                          \
    if (r == 1) CP_MERGE_LAUNCH(InT, OutT, 1);  \
    else if (r == 2) CP_MERGE_LAUNCH(InT, OutT, 2); \
    else CP_MERGE_LAUNCH(InT, OutT, 4);         \
  } while (0)
  if (parts_dtype == CP_F32) {
    if (out_dtype == CP_F32) CP_MERGE_BY_R(float, float);
    else CP_MERGE_BY_R(float, __nv_bfloat16);
  } else {
    if (out_dtype == CP_F32) CP_MERGE_BY_R(__nv_bfloat16, float);
    else CP_MERGE_BY_R(__nv_bfloat16, __nv_bfloat16);
  }
#undef CP_MERGE_BY_R
#undef CP_MERGE_LAUNCH
  return last_cuda_status();
}

cp_status cp_attn_merge(const float* o_parts, const float* lse_parts, int32_t n_parts, int64_t part_stride_rows,
                        int64_t rows, int32_t n_h, int32_t d, void* out, cp_dtype out_dtype, float* lse_out,
                        void* cuda_stream) {
  return merge_impl(o_parts, CP_F32, lse_parts, n_parts, part_stride_rows, rows, n_h, d, out, out_dtype, lse_out,
                    cuda_stream);
}

cp_status cp_attn_merge_bf16_parts(const void* o_parts, const float* lse_parts, int32_t n_parts,
                                   int64_t part_stride_rows, int64_t rows, int32_t n_h, int32_t d, void* out,
                                   cp_dtype out_dtype, float* lse_out, void* cuda_stream) {
  if (!o_parts || !lse_parts || !out) return CP_ERR_INVALID_ARG;
  if (n_parts < 1 || rows < 0 || n_h < 1 || d < 8 || (d & 7) || d > 256) return CP_ERR_INVALID_ARG;
  if (n_parts > 1 && part_stride_rows < rows) return CP_ERR_INVALID_ARG;
  if (!aligned(o_parts, 16) || !aligned(lse_parts, 4)) return CP_ERR_INVALID_ARG;
  if (out_dtype == CP_F32) {
    if (!aligned(out, 16)) return CP_ERR_INVALID_ARG;
  } else if (out_dtype == CP_BF16) {
    if (!aligned(out, 8)) return CP_ERR_INVALID_ARG;
  } else {
    return CP_ERR_UNSUPPORTED;
  }
  // out and lse_out may not overlap the parts (rows are read and written by different lanes)
  const uintptr_t o_lo = reinterpret_cast<uintptr_t>(o_parts);
  const uintptr_t o_hi = o_lo + static_cast<uintptr_t>((n_parts > 1 ? (n_parts - 1) * part_stride_rows : 0) + rows) *
                                    n_h * d * 2;
  const uintptr_t ob = reinterpret_cast<uintptr_t>(out);
  const uintptr_t oe = ob + static_cast<uintptr_t>(rows) * n_h * d * (out_dtype == CP_F32 ? 4 : 2);
  if (rows > 0 && ob < o_hi && oe > o_lo) return CP_ERR_INVALID_ARG;
  const int64_t n_rowheads = rows * n_h;
  if (n_rowheads == 0) return CP_OK;
  cudaStream_t stream = static_cast<cudaStream_t>(cuda_stream);
  const int64_t rows_per_warp = 32 / (d / 8);
  const int64_t warps_per_block = merge::kThreads / 32;
  int64_t grid = (n_rowheads + warps_per_block * rows_per_warp - 1) / (warps_per_block * rows_per_warp);
  grid = std::min<int64_t>(grid, 148 * 32);
  const int64_t o_stride = part_stride_rows * n_h * d, l_stride = part_stride_rows * n_h;
  if (out_dtype == CP_F32)
    merge::merge_bf16_parts_kernel<float><<<static_cast<unsigned>(grid), merge::kThreads, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(o_parts), lse_parts, n_parts, o_stride, l_stride, n_rowheads, d,
        static_cast<float*>(out), lse_out);
  else
    merge::merge_bf16_parts_kernel<__nv_bfloat16><<<static_cast<unsigned>(grid), merge::kThreads, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(o_parts), lse_parts, n_parts, o_stride, l_stride, n_rowheads, d,
        static_cast<__nv_bfloat16*>(out), lse_out);
  return last_cuda_status();
}

static cp_status decode_impl(const void* q, const void* k, const void* v, cp_dtype dtype, const int64_t* kv_offsets,
                             int32_t batch, int64_t kv_rows, int32_t n_h, int32_t n_kv, int32_t d, int32_t n_splits,
                             float softmax_scale, void* out, bool out_f32, float* lse_out, void* workspace,
                             size_t ws_bytes, void* cuda_stream) {
  DecodeShape s;
  cp_status st = decode_validate(q, k, v, dtype, kv_offsets, batch, kv_rows, n_h, n_kv, d, n_splits, softmax_scale,
                                 out, out_f32, &s);
  if (st != CP_OK) return st;
  decode_sizes(&s, dec::kWarps, batch, n_kv, d);   // below what even the smallest grid needs
  if (!workspace || !aligned(workspace, 256) || ws_bytes < s.bytes) return CP_ERR_WORKSPACE;
  st = decode_grid(&s, n_splits, batch, kv_rows, n_kv, d);
  if (st != CP_OK) return st;
  if (ws_bytes < s.bytes) return CP_ERR_WORKSPACE;
  if (batch == 0) return CP_OK;
  return decode_launch(s, q, k, v, kv_offsets, batch, kv_rows, n_h, n_kv, d, softmax_scale, out, out_f32, lse_out,
                       workspace, static_cast<cudaStream_t>(cuda_stream));
}

cp_status cp_decode(const void* q, const void* k, const void* v, cp_dtype dtype, const int64_t* kv_offsets,
                    int32_t batch, int64_t kv_rows, int32_t n_h, int32_t n_kv, int32_t d, int32_t n_splits,
                    float softmax_scale, void* out, float* lse_out, void* workspace, size_t ws_bytes,
                    void* cuda_stream) {
  return decode_impl(q, k, v, dtype, kv_offsets, batch, kv_rows, n_h, n_kv, d, n_splits, softmax_scale, out, false,
                     lse_out, workspace, ws_bytes, cuda_stream);
}

cp_status cp_decode_partial(const void* q, const void* k, const void* v, cp_dtype dtype, const int64_t* kv_offsets,
                            int32_t batch, int64_t kv_rows, int32_t n_h, int32_t n_kv, int32_t d, int32_t n_splits,
                            float softmax_scale, float* o_part, float* lse_part, void* workspace, size_t ws_bytes,
                            void* cuda_stream) {
  if (!lse_part) return CP_ERR_INVALID_ARG;
  return decode_impl(q, k, v, dtype, kv_offsets, batch, kv_rows, n_h, n_kv, d, n_splits, softmax_scale, o_part, true,
                     lse_part, workspace, ws_bytes, cuda_stream);
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Split-KV decode without a caller-provided workspace.
//
// Some callers cannot allocate device memory at the point where they decode:
// code running inside a custom allocator or a memory pool that must not
// re-enter itself, plugins handed only input and output buffers by a host
// framework, and serving loops that forbid allocation after start-up. For
// them the split partials live in one fixed array in the library's own device
// memory (every GPU that loads the library holds it until the process exits).
// ---------------------------------------------------------------------------
namespace {

constexpr size_t kStaticScratchBytes = 32ull << 20;  // 32 MiB per device
static __device__ __align__(256) uint8_t g_decode_scratch[kStaticScratchBytes];

// Device address of g_decode_scratch on each device. In host code the array's
// name is only a stand-in; the address must be looked up with that device current.
std::mutex g_scratch_mu;
void* g_scratch_addr[64] = {nullptr};

cp_status scratch_for_current_device(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return CP_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_addr[dev]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_decode_scratch) != cudaSuccess || !ptr) return CP_ERR_CUDA;
    g_scratch_addr[dev] = ptr;
  }
  *out = g_scratch_addr[dev];
  return CP_OK;
}

}  // namespace

extern "C" cp_status cp_decode_static(const void* q, const void* k, const void* v, cp_dtype dtype,
                                      const int64_t* kv_offsets, int32_t batch, int64_t kv_rows, int32_t n_h,
                                      int32_t n_kv, int32_t d, int32_t n_splits, float softmax_scale, void* out,
                                      float* lse_out, void* cuda_stream) {
  // every argument is checked before anything is enqueued
  DecodeShape s;
  cp_status st = decode_validate(q, k, v, dtype, kv_offsets, batch, kv_rows, n_h, n_kv, d, n_splits, softmax_scale,
                                 out, false, &s);
  if (st != CP_OK) return st;
  st = decode_grid(&s, n_splits, batch, kv_rows, n_kv, d);
  if (st != CP_OK) return st;
  if (s.bytes > kStaticScratchBytes) return CP_ERR_WORKSPACE;
  void* scratch = nullptr;
  st = scratch_for_current_device(&scratch);
  if (st != CP_OK) return st;
  cudaStream_t stream = static_cast<cudaStream_t>(cuda_stream);
  // The status word starts at zero for every call (so that
  // cp_decode_static_status reports this call); the split partials are fully
  // rewritten before the merge reads them.
  if (cudaMemsetAsync(scratch, 0, sizeof(uint32_t), stream) != cudaSuccess) return CP_ERR_CUDA;
  if (batch == 0) return CP_OK;
  return decode_launch(s, q, k, v, kv_offsets, batch, kv_rows, n_h, n_kv, d, softmax_scale, out, false, lse_out,
                       scratch, stream);
}

extern "C" cp_status cp_decode_static_status(void* cuda_stream) {
  void* scratch = nullptr;
  const cp_status st = scratch_for_current_device(&scratch);
  if (st != CP_OK) return st;
  return cp_check_status(scratch, cuda_stream);
}
