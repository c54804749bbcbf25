/*
 * zsa.h -- C ABI of libzsa: zigzag-sharded causal (GQA) attention on B200 (sm_100a).
 *
 * The operation.  A sequence of S positions is cut into 2D equal chunks of
 * C = S/(2D) positions; logical shard r holds chunk r followed by chunk 2D-1-r
 * ("Folding Tensor and Sequence Parallelism", summary page, section 2, attention
 * layer: a zigzag partition balances the causal work across shards).  Every shard's
 * queries attend to the full, all-gathered K/V (same page and section: an
 * all-gather rebuilds the full K/V for FlashAttention), with the causal mask taken
 * on GLOBAL positions ("AutoSP" summary page, section 2.A, step 4: index tensors
 * such as causal masks are recomputed for the sharded layout).  q head h reads kv
 * head h / (Hq/Hkv) (grouped-query attention, "Tensor, pipeline e sequence
 * parallelism", 01 Conceito: 24 q heads over 4 kv heads).  On one GPU all D
 * shards run in one launch reading one K/V buffer.
 *
 *   forward : for shard row (r, j) at position p and q head h,
 *             s_k = scale * q . k_k for keys k <= p (all k when causal == 0),
 *             lse = ln sum_k exp(s_k),  O = sum_k exp(s_k - lse) v_k
 *   backward: the exact gradient of <dO, O>:  Delta = <dO, O>,
 *             dS_k = P_k (dO . v_k - Delta),  dQ = scale sum_k dS_k k_k,
 *             dK_k = scale sum dS_k q,  dV_k = sum P_k dO   (sums over every shard
 *             and every q head of the kv group)
 *
 * Layouts (all tensors contiguous, row-major, bf16 unless stated):
 *   Q, O, dO, dQ : [D][B][2C][Hq][d]   shard-major: shard r's slab is what one rank holds
 *   K, V, dK, dV : [B][S][Hkv][d]      natural position order (the gathered buffer)
 *   lse          : fp32 [D][B][Hq][2C] natural logarithm
 *
 * Ownership.  The caller owns every buffer: device pointers for tensors and the
 * workspace, host pointers for zsa_partition's outputs.  The library allocates no
 * device memory; it caches host-side schedules per shape (thread-safe).
 *
 * Asynchrony.  zsa_attn_fwd / zsa_attn_bwd enqueue work on `cuda_stream` (a
 * cudaStream_t; NULL = legacy default stream) and return without synchronising.
 * Launch-time CUDA errors return ZSA_ERR_CUDA.  Every device-side wait is bounded;
 * a wait that gives up records a timeout in the workspace's status word, which
 * zsa_device_status() reads.
 *
 * Errors: every call returns ZSA_OK (0) or a negative ZSA_ERR_* code and never
 * throws across the ABI.  Argument errors are detected before anything is enqueued.
 */
#ifndef ZSA_H
#define ZSA_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define ZSA_API __attribute__((visibility("default")))
#else
#define ZSA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

enum {
  ZSA_OK = 0,
  ZSA_ERR_INVALID = -1,     /* null pointer, non-positive size or scale, misaligned pointer,
                               bad kv_layout or shard range                                 */
  ZSA_ERR_SHAPE = -2,       /* S % (2*D*64) != 0, Hq % Hkv != 0                              */
  ZSA_ERR_UNSUPPORTED = -3, /* head dim not in {64, 128, 256}; device is not sm_100          */
  ZSA_ERR_WORKSPACE = -4,   /* workspace (or schedule capacity) too small                    */
  ZSA_ERR_CUDA = -5,        /* a CUDA runtime call failed                                    */
  ZSA_ERR_TIMEOUT = -6      /* a bounded device-side wait gave up (see zsa_device_status)   */
};

/* K / V layouts (zsa_problem.kv_layout). */
enum {
  ZSA_KV_NATURAL = 0,     /* K, V, dK, dV : [B][S][Hkv][d] in position order               */
  ZSA_KV_SHARD_MAJOR = 1  /* K, V, dK, dV : [D][B][2C][Hkv][d], rows in the Q layout's
                             zigzag order: exactly what an all-gather of every shard's own
                             K/V rows produces, and what a reduce-scatter of dK/dV back to
                             the owning shards consumes, with no reorder pass           */
};

/* One attention problem, and the part of it one call computes.
 *  softmax_scale: applied as an fp32 value (callers usually pass 1/sqrt(d) rounded to
 *    fp32).  causal = 0 gives full (non-causal) attention with the same layouts.
 *  kv_layout: ZSA_KV_NATURAL or ZSA_KV_SHARD_MAJOR (above); K/V always hold the whole
 *    gathered sequence.
 *  shard_begin, shard_count: the call computes the queries of the logical shards
 *    [shard_begin, shard_begin + shard_count) only (shard_count = 0: all D shards).  The
 *    Q-layout tensors (Q, O, dO, dQ, lse) then hold just those shards, [shard_count][B]
 *    [2C][Hq][d] (lse [shard_count][B][Hq][2C]), and dK/dV are the partial sums over
 *    those shards' queries: one rank's share of a D-rank run, whose reduce-scatter gives
 *    every owner its slab.  A zero-initialised struct tail keeps the one-launch default
 *    (natural K/V, all shards).
 * The sharded reading ("Folding Tensor and Sequence Parallelism" summary, section 2,
 * attention layer: each rank holds one zigzag shard and an all-gather rebuilds the K/V
 * context) is what the shard range and the shard-major K/V layout express. */
typedef struct {
  int64_t B, S;
  int32_t Hq, Hkv, d, D;
  int32_t causal;
  float softmax_scale;
  int32_t kv_layout;
  int32_t shard_begin, shard_count;
} zsa_problem;

/* Tiling of the forward schedule: block_q query rows per tile, block_k keys per key
 * tile, `slots` query tiles per work unit (the tiles of one unit share one K/V
 * stream).  Zero fields mean "library default for d" and are filled in on return. */
typedef struct {
  int32_t block_q, block_k, slots;
} zsa_tiling;

/* One forward work unit: up to two (q tile, q head) slots of shard `shard`, batch
 * `b`, both q heads in kv group `kv_head`.  k_tile_end = number of key tiles the
 * slot's rows can see (key tiles 0 .. k_tile_end-1).  An absent second slot has
 * q_tile1 = q_head1 = -1 and k_tile_end1 = 0. */
typedef struct {
  int32_t shard, b, kv_head;
  int32_t q_tile0, q_head0, q_tile1, q_head1;
  int32_t k_tile_end0, k_tile_end1;
} zsa_work;

/*
 * zsa_partition -- the zigzag index map and the balanced causal tile schedule
 * (host only, no GPU needed).
 * Defined by: "Folding Tensor and Sequence Parallelism" summary, section 2, attention
 * layer (a zigzag partition balances causal work across shards; chunks r and 2D-1-r
 * per shard is the reading taken), and the global-position causal mask of "AutoSP"
 * summary, section 2.A step 4 (which key tiles a query tile sees).  The unit order is
 * this library's own definition (the pages give none).
 *   perm_host        [S]  or NULL: perm[r*2C + j] = global position of row j of shard r
 *   inv_perm_host    [S]  or NULL: inverse of perm
 *   shard_tiles_host [D]  or NULL: QK^T tile products (block_q x block_k) of shard r,
 *                         summed over b and q heads; equal for every r (the balance
 *                         the zigzag provides)
 *   sched_host       [cap] or NULL: work units in launch order (see zsa_work)
 *   *n_work_out      number of units (always set when the shape is valid)
 * Tiling: q tile i of shard r covers rows [i*block_q, (i+1)*block_q) of the shard;
 * its k_tile_end is (largest position in the tile)/block_k + 1 (causal) or S/block_k.
 * Units list, per (b, kv head g, shard r), the tile-major slots s = i*G + e (q head
 * g*G + e) in consecutive runs of `slots`; they are ordered by b, then g (ascending),
 * and within one (b, g) by max k_tile_end descending, then shard, then run index.
 * Returns ZSA_ERR_WORKSPACE when cap < *n_work_out and sched_host != NULL.
 */
ZSA_API int zsa_partition(const zsa_problem* problem, zsa_tiling* tiling, int32_t* perm_host,
                  int32_t* inv_perm_host, int64_t* shard_tiles_host, zsa_work* sched_host,
                  int64_t cap, int64_t* n_work_out);

/* Workspace bytes needed by zsa_attn_fwd (pass = 0) or zsa_attn_bwd (pass = 1).
 * No passage defines it: the caller owns all device memory, so the library states how
 * much scratch each pass needs.
 * The workspace must be device memory, 256-byte aligned, not shared between calls in
 * flight.  fwd: status word + the unit table.  bwd: status word + -Delta and
 * -lse*log2(e) (fp32 [D][B][Hq][2C] each) + a dQ accumulator (fp32, head-major
 * [Hq][D*B*2C][d]). */
ZSA_API int zsa_workspace_bytes(const zsa_problem* problem, int pass, size_t* bytes_out);

/* Forward: o (bf16, Q layout) and lse (fp32 [D][B][Hq][2C]).  q, k, v, o, lse and the
 * workspace are device pointers, 16-byte aligned.
 * Defined by: "Folding Tensor and Sequence Parallelism" summary, section 2, attention
 * layer (each shard's queries run FlashAttention over the all-gathered K/V), with the
 * causal mask on global positions ("AutoSP" summary, section 2.A step 4) and GQA head
 * sharing ("Tensor, pipeline e sequence parallelism", 01 Conceito). */
ZSA_API int zsa_attn_fwd(const zsa_problem* problem, const void* q, const void* k, const void* v,
                 void* o, float* lse, void* workspace, size_t ws_bytes, void* cuda_stream);

/* Backward: dq (Q layout), dk, dv (K layout), all bf16, overwritten (not accumulated).
 * o and lse must come from zsa_attn_fwd on the same inputs.  dk and dv are the same on
 * every run; dq sums the key tiles' contributions with fp32 reduce-adds whose order
 * between thread blocks is not fixed, so runs may differ by that fp32 rounding (seen
 * through the bf16 output).
 * Defined by: the pages describe only the forward; this is the exact gradient of
 * <dO, O> for the forward above (the reading taken where the pages are silent), with
 * dK/dV summed over every shard as the reduce-scatter back to the owning shards of the
 * "Folding Tensor and Sequence Parallelism" attention layer would deliver them. */
ZSA_API int zsa_attn_bwd(const zsa_problem* problem, const void* q, const void* k, const void* v,
                 const void* o, const float* lse, const void* dout, void* dq, void* dk,
                 void* dv, void* workspace, size_t ws_bytes, void* cuda_stream);

/* Most partial results one zsa_attn_merge call combines. */
#define ZSA_MERGE_MAX_PARTS 32

/* Merge of partial attention results over disjoint key sets: the combining step of ring
 * attention ("AutoSP" summary, sections 1 and 4, where ring attention is the
 * sequence-parallel baseline; the pages give no formula, and the reading taken is the
 * definition of a softmax over a union of disjoint key sets):
 *   lse = ln sum_i exp(lse_i),   O = sum_i exp(lse_i - lse) O_i,
 * an empty key set (lse_i = -inf, O_i = 0) contributing nothing; a (row, head) whose parts
 * are all empty gets lse = -inf and O = 0.
 *   problem   : shapes; the Q-layout rows are those of its shard range (all D by default)
 *   n_parts   : 1 .. ZSA_MERGE_MAX_PARTS
 *   o_parts   : HOST array of n_parts device pointers, bf16 in the Q layout
 *   lse_parts : HOST array of n_parts device pointers, fp32 [shards][B][Hq][2C]
 *   o, lse    : device outputs in the same layouts; they may alias one of the parts (a
 *               running merge in place)
 * Pointers 16-byte aligned; rows * Hq * d < 2^31 (ZSA_ERR_SHAPE otherwise).  Asynchronous
 * on cuda_stream; HBM-bound (reads n_parts * (2d + 4) bytes and writes 2d + 4 per
 * (row, head)). */
ZSA_API int zsa_attn_merge(const zsa_problem* problem, int32_t n_parts, const void* const* o_parts,
                           const float* const* lse_parts, void* o, float* lse,
                           void* cuda_stream);

/* K5: copy a tensor of one bf16 row of heads*d values per position between the natural
 * order [B][S][heads][d] and the zigzag shard-major order [shards][B][2C][heads][d] of the
 * problem's shard range (all D by default): shard r holds chunk r, then chunk 2D-1-r, of
 * C = S/(2D) positions ("Folding Tensor and Sequence Parallelism" summary, section 2,
 * attention layer: the zigzag partition of the sequence).  For callers whose Q, O, dO or
 * K/V are in position order; the attention calls themselves need no such pass
 * (ZSA_KV_SHARD_MAJOR reads an all-gather's output as it lands).
 *   heads          : Hq for Q / O / dO / dQ, Hkv for K / V / dK / dV (any value >= 1)
 *   to_shard_major : 1: src natural -> dst shard-major; 0: src shard-major -> dst natural.
 *                    With a shard range, natural -> shard-major reads only the range's
 *                    chunks, and shard-major -> natural writes only those (the other rows
 *                    of dst are left as they are).
 *   src, dst       : device pointers, 16-byte aligned, not overlapping.
 * Uses the problem's B, S, D, d and shard range (d a multiple of 8; Hq, Hkv, the scale and
 * kv_layout are checked as everywhere but not used).  ZSA_ERR_SHAPE when 2 * shards * B >
 * 65535.  Asynchronous on cuda_stream; HBM-bound (reads and writes each byte once). */
ZSA_API int zsa_permute(const zsa_problem* problem, int32_t heads, int32_t to_shard_major,
                        const void* src, void* dst, void* cuda_stream);

/* A block of keys for zsa_attn_fwd_block: the positions [key_lo, key_hi) of the
 * sequence (0 <= key_lo <= key_hi <= S, any values), held in K/V tensors
 * [rows][Hkv][d] bf16 with the key at position p of batch b in row
 *   b * rows_per_batch + row_offset + (p - key_lo).
 * E.g. one zigzag chunk c of a natural [B][S][Hkv][d] buffer: rows_per_batch = S,
 * row_offset = c*C; the first chunk of a received shard block [B][2C][Hkv][d]:
 * rows_per_batch = 2C, row_offset = 0 (its second chunk: row_offset = C).
 * rows, rows_per_batch and row_offset are below 2^31, and every row the block names lies
 * inside the tensor: (B-1)*rows_per_batch + row_offset + (key_hi - key_lo) <= rows, with
 * rows_per_batch >= key_hi - key_lo when B > 1. */
typedef struct {
  int64_t key_lo, key_hi;
  int64_t rows_per_batch;
  int64_t row_offset;
  int64_t rows;
} zsa_key_block;

/* Forward restricted to one block of keys: the partial result one ring-attention step
 * computes ("AutoSP" summary, sections 1 and 4, ring attention as the sequence-parallel
 * baseline: each rank's queries meet the K/V blocks one at a time).  For every query
 * row of the problem's shard range and q head: the causal softmax attention over the
 * keys of the block only (the mask on global positions as in zsa_attn_fwd), written as
 * o (bf16, Q layout) and lse (fp32 [shards][B][Hq][2C]) exactly as zsa_attn_fwd writes
 * them.  A row that sees no key of the block gets o = 0 and lse = -inf, the empty part
 * zsa_attn_merge skips; merging the results of blocks that tile [0, S) gives
 * zsa_attn_fwd's.  problem->kv_layout is not used (the block describes K/V).  Workspace
 * as zsa_attn_fwd's (zsa_workspace_bytes pass 0); pointers 16-byte aligned; errors as
 * zsa_attn_fwd, plus ZSA_ERR_INVALID for a block outside the bounds above. */
ZSA_API int zsa_attn_fwd_block(const zsa_problem* problem, const zsa_key_block* block,
                               const void* q, const void* k, const void* v, void* o, float* lse,
                               void* workspace, size_t ws_bytes, void* cuda_stream);

/* One run of output columns of a TSP projection step (zsa_tsp_project). */
typedef struct {
  void* out;                 /* device: element (0, 0) of this run's output */
  int64_t ld;                /* row stride of out, in elements (a multiple of 8) */
  int32_t cols;              /* columns of W routed here (a multiple of 32) */
  int32_t fp32_accumulate;   /* 0: out is bf16 and overwritten; 1: out is fp32, out += */
} zsa_proj_segment;

#define ZSA_PROJ_MAX_SEGMENTS 8

/* One step of the TSP attention-layer weight schedule on one rank ("Folding Tensor and
 * Sequence Parallelism" summary, section 2, attention layer: each rank holds 1/D of the
 * tokens and one packed shard of W_Q/W_K/W_V/W_O; step s broadcasts rank s's shard and
 * every rank projects its own tokens with it):
 *   Y = X W,   X [T][K] bf16 (row stride ldx), W [K][N] bf16 (row stride ldw),
 * with Y's columns routed, in order, to segs[0], segs[1], ... (segs[i].cols each, summing
 * to N): e.g. the Q, K and V columns of the shard's heads written into the rank's Q, K
 * and V (bf16), or the output projection's partial added into an fp32 accumulator.
 * N a multiple of 32, K a multiple of 8 (any T); ldx, ldw multiples of 8; x, w and every
 * out 16-byte aligned.  `status_ws` is a 256-byte device workspace whose status word
 * zsa_device_status reads (a bounded wait that gave up).  Asynchronous on cuda_stream.
 * fp32 tensor-core accumulation; bf16 outputs rounded to nearest even. */
ZSA_API int zsa_tsp_project(int64_t T, int64_t K, int64_t N, const void* x, int64_t ldx,
                            const void* w, int64_t ldw, const zsa_proj_segment* segs,
                            int32_t n_segs, void* status_ws, void* cuda_stream);

/* Size of the fixed device scratch behind zsa_attn_bwd_noalloc (64 MiB per device). */
#define ZSA_NOALLOC_SCRATCH_BYTES (64u * 1024u * 1024u)

/* Backward without a workspace argument and without allocating anything.  The pages
 * have no counterpart to this call.  It exists for callers that cannot allocate device
 * memory where they call the backward: plugins inside a host runtime that owns and
 * pre-plans all device memory (they may not call cudaMalloc and get no scratch hook),
 * or C callers without an allocator of their own.  Arguments and results are those of
 * zsa_attn_bwd; the scratch (status word, -Delta, -lse*log2(e), fp32 dQ accumulator) is
 * a fixed static device array of ZSA_NOALLOC_SCRATCH_BYTES, resident until the process
 * exits on every GPU on which the library's module is loaded (under CUDA's eager module
 * loading, every GPU the process has a context on).
 *  - Problems needing more scratch than that (zsa_workspace_bytes(problem, 1) >
 *    ZSA_NOALLOC_SCRATCH_BYTES) return ZSA_ERR_WORKSPACE before anything is enqueued.
 *  - All calls on a device share the array and it keeps the last call's contents:
 *    calls whose GPU work overlaps (other streams or host threads) race and produce
 *    wrong results.  Each call re-zeroes what must start at zero.
 *  - The first call on each device looks up the array's device address
 *    (cudaGetSymbolAddress) with that device current; make it before any stream
 *    capture begins.
 *  - zsa_set_wait_limit_ns and zsa_debug_inject_stall apply as for zsa_attn_bwd; a
 *    device-side wait that gives up is reported by zsa_noalloc_status. */
ZSA_API int zsa_attn_bwd_noalloc(const zsa_problem* problem, const void* q, const void* k,
                                 const void* v, const void* o, const float* lse,
                                 const void* dout, void* dq, void* dk, void* dv,
                                 void* cuda_stream);

/* Synchronises `cuda_stream`, reads and clears the status word of the current device's
 * zsa_attn_bwd_noalloc scratch: ZSA_OK, or ZSA_ERR_TIMEOUT if a device-side wait of an
 * earlier zsa_attn_bwd_noalloc call gave up (its outputs are then undefined). */
ZSA_API int zsa_noalloc_status(void* cuda_stream);

/* Synchronises `cuda_stream`, reads and clears the status word at the start of
 * `workspace`: ZSA_OK, or ZSA_ERR_TIMEOUT if a device-side wait gave up.  Failure
 * detection of this library (bounded waits); the pages define nothing here. */
ZSA_API int zsa_device_status(void* workspace, void* cuda_stream);

/* Upper bound, in nanoseconds, on any single device-side wait of later launches
 * (default 2e9).  Test hook: a tiny limit makes the first real wait time out so the
 * error path can be exercised without hanging anything. */
ZSA_API int zsa_set_wait_limit_ns(uint64_t limit_ns);

/* Test hook: when `enable` is nonzero, later launches make their MMA-issuing thread
 * first wait on a barrier that nothing ever arrives at, so the bounded wait must give
 * up; the launch then tears down (draining its copies and MMAs in flight, releasing
 * TMEM) and records ZSA_ERR_TIMEOUT in the status word.  Outputs of such a launch are
 * undefined.  Call with 0 to restore normal operation. */
ZSA_API int zsa_debug_inject_stall(int enable);

/* Tracing hook: while set, every later launch of kernel `which` records the CUDA
 * events `begin_event` / `end_event` (cudaEvent_t handles owned by the caller) on the
 * launch stream immediately before / after the kernel, so the caller can time that
 * kernel alone with cudaEventElapsedTime.  which: ZSA_TRACE_FWD (forward kernel),
 * ZSA_TRACE_BWD_PRE (Delta preprocess), ZSA_TRACE_BWD_MAIN (backward main kernel),
 * ZSA_TRACE_BWD_DQ (dQ conversion), ZSA_TRACE_MERGE (partial-result merge),
 * ZSA_TRACE_PROJ (TSP projection GEMM), ZSA_TRACE_PERMUTE (K5 permute).  Pass NULL events
 * to stop tracing that kernel. */
enum {
  ZSA_TRACE_FWD = 0, ZSA_TRACE_BWD_PRE = 1, ZSA_TRACE_BWD_MAIN = 2, ZSA_TRACE_BWD_DQ = 3,
  ZSA_TRACE_MERGE = 4, ZSA_TRACE_PROJ = 5, ZSA_TRACE_PERMUTE = 6
};
ZSA_API int zsa_trace_events(int which, void* begin_event, void* end_event);

/* Static string for a status code.  Library bookkeeping; no passage defines it. */
ZSA_API const char* zsa_status_string(int status);

#ifdef __cplusplus
}
#endif

#endif /* ZSA_H */
