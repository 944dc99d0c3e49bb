/*
 * cp_attn.h -- C ABI of libcpattn.so: the hot path of context-parallel ring
 * attention on one B200 (sm_100a), with the N context-parallel ranks as
 * virtual shards of one GPU's buffers.
 *
 * Method: "Context Parallelism for Scalable Million-Token Inference" (review of
 * arXiv:2411.01783). Exact GQA softmax attention is computed as partial blocks
 * (one query shard against one KV shard, online softmax over KV tiles), each
 * yielding an output normalised within the block plus a per-row log-sum-exp,
 * and the partials are combined by LSE weighting ("merge attention").
 *
 * Conventions shared by every entry point:
 *  - The caller owns and allocates every buffer. The library never allocates
 *    or frees device memory and holds no state between calls; the one
 *    exception is the fixed scratch array behind cp_decode_static (below).
 *  - Tensors are row-major and token-major: Q [rows, N_H, D], K and V
 *    [rows, N_KV, D], partial outputs [rows, N_H, D] fp32, LSE [rows, N_H] fp32
 *    (natural logarithm of the sum of exp(scaled scores)).
 *  - Device entry points are asynchronous on the given CUDA stream
 *    (a cudaStream_t passed as void*, NULL = legacy default stream). They
 *    validate every argument before launching anything and return a status;
 *    they never abort or print. A launch failure maps to CP_ERR_CUDA. A fault
 *    inside a kernel surfaces at the caller's next synchronisation.
 *  - Device-side waits are bounded. A wait that runs out writes a code into the
 *    status word at the start of the workspace and the kernel returns early;
 *    cp_check_status() reports it.
 *  - Host planning entry points are deterministic and bit-exact.
 */
#ifndef CP_ATTN_H
#define CP_ATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define CP_ABI_VERSION 2

typedef enum {
  CP_OK = 0,
  CP_ERR_INVALID_ARG = 1,  /* null pointer, negative size, range outside a buffer */
  CP_ERR_UNSUPPORTED = 2,  /* valid but not implemented: head dim, dtype, group size */
  CP_ERR_WORKSPACE = 3,    /* workspace missing, misaligned or too small */
  CP_ERR_CUDA = 4,         /* a CUDA runtime or driver call failed */
  CP_ERR_TIMEOUT = 5,      /* a device-side wait ran out (see cp_check_status) */
  CP_ERR_INTERNAL = 6      /* a device-side consistency check failed */
} cp_status;

typedef enum { CP_F32 = 0, CP_BF16 = 1 } cp_dtype;

/* Load-balanced: a segment of length L is cut into 2N chunks,
 * chunk c = [floor(c*L/2N), floor((c+1)*L/2N)), and rank i holds chunks i and
 * 2N-1-i (method page, section 4, load-balanced sharding).
 * Contiguous: rank i holds chunks 2i and 2i+1, i.e. [floor(iL/N), floor((i+1)L/N)). */
typedef enum { CP_SHARD_LOAD_BALANCED = 0, CP_SHARD_CONTIGUOUS = 1 } cp_shard_mode;

/* Ring variants (method page, section 3). Rank r sends to r+1, so at step t
 * rank r holds the visiting shard of rank (r - t) mod N.
 *  pass-KV: rank i keeps its Q shard and sees the KV shard of (i - t) mod N;
 *           that block's partial is arrival number t.
 *  pass-Q:  rank i keeps its KV shard and sees the Q shard of (i - t) mod N;
 *           after the all-to-all the Q owner holds one partial per KV owner,
 *           indexed by the KV owner i. */
typedef enum { CP_PASS_KV = 0, CP_PASS_Q = 1 } cp_ring_variant;

typedef enum { CP_PAIR_FULL = 0, CP_PAIR_PARTIAL = 1, CP_PAIR_SKIP = 2 } cp_pair_class;

/* A sharding unit: `len` consecutive rows of a buffer starting at `row0`,
 * holding tokens of sequence `seq` at global positions pos0..pos0+len-1.
 * A persistent-KV prefill describes the cached prefix and the new tokens as
 * two segments of the same sequence, each sharded on its own. */
typedef struct {
  int64_t len;
  int64_t row0;
  int64_t pos0;
  int32_t seq;
  int32_t reserved; /* must be 0 */
} cp_segment;

/* A contiguous run of rows of one buffer (a chunk of a shard). 32 bytes. */
typedef struct {
  int64_t row0; /* first row in the Q (or K/V) buffer */
  int64_t pos0; /* global causal position of that row */
  int64_t len;  /* number of rows */
  int32_t seq;  /* sequence id: attention never crosses sequences */
  int32_t reserved; /* must be 0 */
} cp_range;

/* One block of the ring: the query ranges ranges[q_begin .. q_begin+q_count)
 * against the key/value ranges ranges[kv_begin .. kv_begin+kv_count).
 * Query row r of the Q buffer writes output row out_row0 + r. 24 bytes. */
typedef struct {
  int32_t q_begin, q_count;
  int32_t kv_begin, kv_count;
  int64_t out_row0;
} cp_block;

typedef enum { CP_OP_PARTIAL = 0, CP_OP_DECODE = 1, CP_OP_MERGE = 2 } cp_op;

const char* cp_status_string(cp_status s);
int32_t cp_abi_version(void);

/* ---------------------------------------------------------------------------
 * Host planning (method page, sections 3 and 4). No device work.
 * ------------------------------------------------------------------------- */

/* Shard plan of `n_seg` segments over `n_ranks` ranks.
 *  chunk_bounds [n_seg][2N+1]: per segment, chunk boundaries relative to the
 *                segment start (floor(c*len/2N)).
 *  rank_rows    [N+1]: prefix offsets of each rank's rows in token_index.
 *  token_index  [sum of len]: buffer rows held by rank 0, then rank 1, ...;
 *                per rank, segment by segment, chunks in ascending order.
 *  sizes_out    [3]: the element counts of the three arrays above,
 *                n_seg*(2N+1), N+1 and sum of len, so that a caller can call
 *                once with NULL arrays to size them, then again to fill them.
 * Any output pointer may be NULL to skip it. Errors: CP_ERR_INVALID_ARG for
 * n_ranks < 1, n_seg < 0, a negative len/row0/pos0 or a nonzero reserved field. */
cp_status cp_shard_plan(const cp_segment* segs, int32_t n_seg, int32_t n_ranks,
                        cp_shard_mode mode, int64_t* chunk_bounds, int64_t* rank_rows,
                        int64_t* token_index, int64_t* sizes_out);

/* The ranges rank `rank` holds: for each segment in order, its two chunks in
 * ascending chunk order, empty chunks left out. `out` holds up to 2*n_seg
 * entries; *n_out receives the count. */
cp_status cp_rank_ranges(const cp_segment* segs, int32_t n_seg, int32_t n_ranks,
                         cp_shard_mode mode, int32_t rank, cp_range* out, int32_t* n_out);

/* Full ring schedule. ranges receives the Q shards of ranks 0..N-1 followed by
 * the KV shards of ranks 0..N-1 (at most 2*N*(n_q_seg+n_kv_seg) entries;
 * `ranges_cap` is the capacity, *n_ranges the count). blocks [N*N]:
 * blocks[t*N + i] is the block rank i computes at ring step t, with
 * out_row0 = 0; block_part [N*N] (may be NULL) is the index (0..N-1) of the
 * partial that block produces for its query rows (see cp_ring_variant). */
cp_status cp_ring_schedule(const cp_segment* q_segs, int32_t n_q_seg,
                           const cp_segment* kv_segs, int32_t n_kv_seg, int32_t n_ranks,
                           cp_shard_mode mode, cp_ring_variant variant, cp_range* ranges,
                           int32_t ranges_cap, int32_t* n_ranges, cp_block* blocks,
                           int32_t* block_part);

/* FULL: every query row of q sees every key of kv; PARTIAL: a mask is needed;
 * SKIP: no pair is visible (other sequence, or every key after every query
 * when causal). Causal visibility: key position <= query position. */
cp_pair_class cp_classify_pair(const cp_range* q, const cp_range* kv, int32_t causal);

/* Number of (query, key) pairs of a block that the mask keeps, per query head. */
int64_t cp_block_pairs(const cp_range* ranges, const cp_block* block, int32_t causal);

/* Elements a real ring would move (the virtual ring moves none). hop_elems
 * [(N-1)*N]: at hop t (1..N-1), what rank i receives, at [(t-1)*N + i]:
 * pass-KV counts one KV tensor (K or V), rows*N_KV*D; pass-Q counts the Q
 * shard, rows*N_H*D. *total sums hop_elems; *all_to_all counts pass-Q's
 * return of partials, rows*N_H*(D+1) per non-local block (0 for pass-KV).
 * Any output may be NULL. */
cp_status cp_ring_comm_volume(const cp_range* ranges, const cp_block* blocks, int32_t n_ranks,
                              cp_ring_variant variant, int32_t n_h, int32_t n_kv, int32_t d,
                              int64_t* hop_elems, int64_t* total, int64_t* all_to_all);

/* Ring variant by Algorithm 1 (method page, section 3, "Pass-KV vs Pass-Q"):
 *  1. pass-KV if the KV-cache miss rate t/(t+p) is above 2*n_kv/n_h (12.5%
 *     for 128 query heads on 8 KV heads);
 *  2. else pass-KV if one ring hop's SendRecv of a KV shard, (t+p)/n_ranks
 *     tokens of K and V at elem_bytes each, over link_bytes_per_s, takes no
 *     longer than step_attn_s, the caller's time for one ring step of
 *     attention (so the transfer hides under compute);
 *  3. else pass-Q.
 * t: new tokens, p: cached tokens (t+p > 0). Writes the variant and the
 * condition that chose pass-KV (1 or 2; 0 for pass-Q) to *reason (may be NULL).
 * CP_ERR_INVALID_ARG on a negative size, n_h % n_kv != 0, a non-positive link
 * bandwidth or a negative step time. Host only. */
cp_status cp_select_ring_variant(int64_t t, int64_t p, int32_t n_h, int32_t n_kv, int32_t d, int32_t n_ranks,
                                 int32_t elem_bytes, double link_bytes_per_s, double step_attn_s,
                                 cp_ring_variant* variant, int32_t* reason);

/* ---------------------------------------------------------------------------
 * Device entry points (sm_100a). Pointers named q/k/v/o/lse/out/workspace are
 * device pointers; ranges/blocks are host arrays read during the call.
 * ------------------------------------------------------------------------- */

/* Bytes of workspace an entry point needs (always a multiple of 256).
 *  CP_OP_PARTIAL, CP_OP_MERGE: 256 (the status word).
 *  CP_OP_DECODE: 256 + room for ((n_splits+1)*batch + 7)*n_h partial rows of
 *  d+1 floats (O and LSE), each part rounded up to 256; a bound on what
 *  cp_decode uses on any device. `rows` is the batch for decode. */
size_t cp_workspace_size(cp_op op, int64_t rows, int32_t n_h, int32_t d, int32_t n_splits);

/* Self-test of the library's device-side wait bound (no counterpart on the
 * method's pages): one GPU thread waits on a barrier that nothing completes,
 * through the same bounded wait every kernel uses, gives up after budget_ns
 * (1 .. 1e9 ns; every other wait in the library gives up after 1 s) and
 * records the timeout in the workspace status word, so that cp_check_status
 * then returns CP_ERR_TIMEOUT. Nothing faults or hangs; the context stays
 * usable. Asynchronous on the stream. */
cp_status cp_wait_selftest(void* workspace, size_t ws_bytes, uint64_t budget_ns, void* cuda_stream);

/* Zero the status word of a workspace (stream-ordered). */
cp_status cp_reset_status(void* workspace, void* cuda_stream);

/* Synchronise `cuda_stream` and report the status word of `workspace`:
 * CP_OK, CP_ERR_TIMEOUT or CP_ERR_INTERNAL. */
cp_status cp_check_status(const void* workspace, void* cuda_stream);

/* Partial attention of every block (method page, section 3: ring pass-KV and
 * pass-Q; shapes from section 3, core formulas). For block b, query row r of
 * range ranges[j] (j in the block's query slice), at position
 * pos_r = ranges[j].pos0 + (r - ranges[j].row0), and query head h, the visible
 * keys are the rows of the block's KV ranges of the same sequence with
 * position <= pos_r (all positions when causal == 0); KV head
 * g = floor(h / (n_h / n_kv)). Writes, at output row out_row0 + r:
 *   lse_part[row, h] = ln sum_visible exp(scale * <q, k>)   (-inf if none)
 *   o_part[row, h, :] = sum_visible exp(scale*<q,k> - lse) * v   (0 if none)
 * Rows of the output not named by any block are left untouched. Blocks must
 * not write the same output row twice.
 *
 * dtype CP_BF16: tensor-core path (tcgen05/TMEM/TMA), fp32 accumulation,
 *   probabilities rounded to bf16 before the PV product; needs d == 128,
 *   n_h % n_kv == 0, the group size n_h/n_kv a power of two <= 128, and
 *   16-byte aligned q/k/v.
 * dtype CP_F32: exact fp32 SIMT path; d in {64, 128}.
 * q_rows / kv_rows / out_rows: rows allocated in q, k/v and o_part/lse_part;
 * every range must lie inside its buffer (CP_ERR_INVALID_ARG otherwise).
 * workspace: >= cp_workspace_size(CP_OP_PARTIAL, ...) bytes, 256-byte aligned. */
cp_status cp_attn_partial(const void* q, const void* k, const void* v, cp_dtype dtype,
                          int64_t q_rows, int64_t kv_rows, int32_t n_h, int32_t n_kv, int32_t d,
                          float softmax_scale, int32_t causal, const cp_range* ranges,
                          int32_t n_ranges, const cp_block* blocks, int32_t n_blocks,
                          float* o_part, float* lse_part, int64_t out_rows, void* workspace,
                          size_t ws_bytes, void* cuda_stream);

/* cp_attn_partial with the LSE merge in its epilogue ("merge attention",
 * method page section 5, fused into the attention kernel), so that a ring
 * schedule keeps one running (O, LSE) and needs no separate merge pass.
 * Arguments as cp_attn_partial, with o_acc / lse_acc in the roles of o_part /
 * lse_part, and:
 *   accumulate = 0: each computed row is written as cp_attn_partial writes it;
 *   accumulate != 0: each computed row is merged into the (O, LSE) already at
 *     its place in o_acc / lse_acc (LSE weighting; -inf weighs 0);
 *   out (bf16 [out_rows, n_h, d], 16-byte aligned) not NULL: the resulting row
 *     is written there normalised instead of to o_acc (lse_acc still gets its
 *     LSE): the last step of a ring.
 * A row written by this call must belong to one block only (the host checks
 * this and returns CP_ERR_INVALID_ARG otherwise). dtype CP_BF16 only
 * (CP_ERR_UNSUPPORTED for CP_F32). */
cp_status cp_attn_partial_fused(const void* q, const void* k, const void* v, cp_dtype dtype, int64_t q_rows,
                                int64_t kv_rows, int32_t n_h, int32_t n_kv, int32_t d, float softmax_scale,
                                int32_t causal, const cp_range* ranges, int32_t n_ranges, const cp_block* blocks,
                                int32_t n_blocks, float* o_acc, float* lse_acc, int64_t out_rows, int32_t accumulate,
                                void* out, void* workspace, size_t ws_bytes, void* cuda_stream);

/* cp_attn_partial writing its partial O rows in bf16 (round to nearest even)
 * instead of fp32; the LSE stays fp32. A ring's partials then move half the
 * bytes (the merge after the ring reads every partial once: method page,
 * section 5, implementation detail 3), for about 2^-9 of relative rounding
 * in each partial. Arguments as cp_attn_partial with o_part bf16
 * [out_rows, n_h, d], 16-byte aligned. dtype CP_BF16 only (CP_ERR_UNSUPPORTED
 * for CP_F32). Merge such partials with cp_attn_merge_bf16_parts. */
cp_status cp_attn_partial_bf16_parts(const void* q, const void* k, const void* v, cp_dtype dtype,
                                     int64_t q_rows, int64_t kv_rows, int32_t n_h, int32_t n_kv,
                                     int32_t d, float softmax_scale, int32_t causal,
                                     const cp_range* ranges, int32_t n_ranges, const cp_block* blocks,
                                     int32_t n_blocks, void* o_part, float* lse_part, int64_t out_rows,
                                     void* workspace, size_t ws_bytes, void* cuda_stream);

/* LSE merge of n_parts partials of the same rows (method page, section 5,
 * implementation detail 3: the merge after pass-Q; the same step closes
 * pass-KV). Part j lives at o_parts + j*part_stride_rows*n_h*d and
 * lse_parts + j*part_stride_rows*n_h. Per (row, head):
 *   M = max_j lse_j;  lse = M + ln sum_j exp(lse_j - M);
 *   out = sum_j exp(lse_j - lse) * o_j.
 * Parts with lse = -inf get weight 0; if all are -inf, out = 0 and lse = -inf.
 * out [rows, n_h, d] is written as out_dtype (bf16: round to nearest even);
 * lse_out [rows, n_h] may be NULL. With out_dtype CP_F32, out may be the
 * same buffer as part 0 (and lse_out as lse part 0): each element is read
 * before it is written, by the same thread. Requires d % 4 == 0 and 16-byte
 * aligned o_parts/out. */
cp_status cp_attn_merge(const float* o_parts, const float* lse_parts, int32_t n_parts,
                        int64_t part_stride_rows, int64_t rows, int32_t n_h, int32_t d, void* out,
                        cp_dtype out_dtype, float* lse_out, void* cuda_stream);

/* cp_attn_merge of bf16 partials (as cp_attn_partial_bf16_parts writes them):
 * o_parts bf16 at o_parts + j*part_stride_rows*n_h*d elements, 16-byte
 * aligned; LSE parts fp32; the arithmetic is fp32 as in cp_attn_merge.
 * Needs d % 8 == 0 and d <= 256; out may not overlap the parts
 * (CP_ERR_INVALID_ARG otherwise). */
cp_status cp_attn_merge_bf16_parts(const void* o_parts, const float* lse_parts, int32_t n_parts,
                                   int64_t part_stride_rows, int64_t rows, int32_t n_h, int32_t d,
                                   void* out, cp_dtype out_dtype, float* lse_out, void* cuda_stream);

/* Split-KV decode (Flash Decoding; method page, section 5 software stack).
 * Request b has one query row q[b] at position L_b - 1 and keys k/v rows
 * kv_offsets[b] .. kv_offsets[b+1]-1 (L_b = difference), all visible.
 * The query heads of a KV head (G = n_h/n_kv of them, GQA) are taken 16 at a
 * time: G <= 16 is one unit, G = 16u is u units. The splits are cut over the
 * whole batch rather than per request: the keys of every (request, KV head,
 * unit) triple, in order, form one sequence of
 * Kt = n_kv*U*(kv_offsets[batch] - kv_offsets[0]) keys (U units per KV head),
 * cut into W equal ranges, W = 8*min(SM count, ceil(n_splits*batch*n_kv*U/8)).
 * So n_splits caps the average number of splits per triple, and every range
 * holds the same number of keys whatever the mix of lengths. Each range leaves
 * one partial per triple it overlaps in the workspace; the partials of each
 * (request, head) are then merged as in cp_attn_merge (a second launch that
 * starts as a programmatic dependent of the first). The result does not
 * depend on the cut beyond rounding.
 *   q [batch, n_h, d] bf16; k, v [kv_rows, n_kv, d] bf16;
 *   kv_offsets: DEVICE int64 [batch+1], non-decreasing, last <= kv_rows
 *   (with offsets that break this no K/V row outside [0, kv_rows) is read,
 *   and cp_check_status then reports CP_ERR_INTERNAL);
 *   out [batch, n_h, d] bf16; lse_out [batch, n_h] fp32 (may be NULL).
 * Supports dtype CP_BF16, d in {64, 128}, a group G = n_h/n_kv <= 16 or a
 * multiple of 16 up to 128 (CP_ERR_UNSUPPORTED otherwise), 1 <= n_splits <=
 * 1024, kv_rows*n_kv*U*(W+1) < 2^53. Every argument is checked before
 * anything is launched. A request with L_b = 0 yields out = 0, lse = -inf.
 * workspace: >= cp_workspace_size(CP_OP_DECODE, batch, n_h, d, n_splits),
 * 256-byte aligned, status word zeroed (cp_reset_status). */
cp_status cp_decode(const void* q, const void* k, const void* v, cp_dtype dtype,
                    const int64_t* kv_offsets, int32_t batch, int64_t kv_rows, int32_t n_h,
                    int32_t n_kv, int32_t d, int32_t n_splits, float softmax_scale, void* out,
                    float* lse_out, void* workspace, size_t ws_bytes, void* cuda_stream);

/* The decode of cp_decode as a partial: O (fp32, normalised over the keys this
 * call sees) and its LSE, for context-parallel decode, where every rank holds
 * a shard of each request's KV cache, decodes the queries against its shard
 * and the per-rank partials are merged with cp_attn_merge (method page,
 * section 3: ring pass-Q for decode; the merge after the final all-to-all is
 * the "merge attention" step of section 5). Arguments, limits and workspace as
 * in cp_decode, with o_part [batch, n_h, d] fp32 (16-byte aligned) in place of
 * out and lse_part [batch, n_h] fp32 required. A request with no keys here
 * yields O = 0, LSE = -inf, which the merge weighs 0. */
cp_status cp_decode_partial(const void* q, const void* k, const void* v, cp_dtype dtype,
                            const int64_t* kv_offsets, int32_t batch, int64_t kv_rows, int32_t n_h,
                            int32_t n_kv, int32_t d, int32_t n_splits, float softmax_scale,
                            float* o_part, float* lse_part, void* workspace, size_t ws_bytes,
                            void* cuda_stream);

/* Split-KV decode for callers that cannot allocate device memory when they
 * decode (code inside an allocator or memory pool, plugins that are given only
 * their inputs and outputs, serving loops that forbid allocation after
 * start-up). The method's pages have no counterpart to this entry point.
 *
 * Same arguments, results and limits as cp_decode, without the workspace: the
 * split partials and the status word live in a fixed 32 MiB array in the
 * library's device memory, which every GPU that loads the library holds until
 * the process exits.
 *  - Every argument is checked first; a call that returns an error has
 *    enqueued nothing. Requests whose partials, (W + batch*n_kv*U)*min(G, 16)
 *    rows of d+1 floats with W and U as in cp_decode for the current device,
 *    need more than the array are rejected with CP_ERR_WORKSPACE.
 *  - The first call on a device looks up the array's device address for that
 *    device (the device current at the call); make that first call before any
 *    stream capture.
 *  - Every call shares the one array, which keeps the last call's contents;
 *    each call clears the status word (stream-ordered) and rewrites every
 *    partial it reads. Calls that overlap on the GPU (different streams
 *    without ordering, or several host threads) race on the array.
 *  - Device-side failures of a call (offsets that break the contract) are
 *    reported by cp_decode_static_status until the next call clears them.
 *  - Nothing is allocated or freed. */
cp_status cp_decode_static(const void* q, const void* k, const void* v, cp_dtype dtype,
                           const int64_t* kv_offsets, int32_t batch, int64_t kv_rows, int32_t n_h,
                           int32_t n_kv, int32_t d, int32_t n_splits, float softmax_scale, void* out,
                           float* lse_out, void* cuda_stream);

/* The device-side status of the latest cp_decode_static call on the current
 * device (the counterpart of cp_check_status for the fixed array):
 * synchronises `cuda_stream` (pass the stream that call used), then returns
 * CP_OK, CP_ERR_INTERNAL (offsets that break the contract) or CP_ERR_TIMEOUT.
 * Allocates nothing. */
cp_status cp_decode_static_status(void* cuda_stream);

#ifdef __cplusplus
}
#endif
#endif /* CP_ATTN_H */
