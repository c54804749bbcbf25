// zsa_kernels.h -- host-side launch interface of the sm_100a kernels.
#pragma once
#include <cstdint>
#include <cuda_runtime.h>

#include "zsa_schedule.h"

namespace zsa {

struct FwdArgs {
  const void* q;           // [D][B][2C][Hq][d] bf16
  const void* k;           // [B][S][Hkv][d] bf16
  const void* v;
  void* o;                 // [D][B][2C][Hq][d] bf16
  float* lse;              // [D][B][Hq][2C]
  const DevUnit* units;    // device copy of the schedule
  int32_t n_units;
  int64_t S;
  int32_t B, Hq, Hkv, d, D, causal;
  float scale;
  int32_t kv_layout;       // 0: K/V [B][S][Hkv][d]; 1: shard-major [D][B][2C][Hkv][d]
  int32_t shard_begin;     // the call computes the queries of shards
  int32_t shard_count;     //   [shard_begin, shard_begin + shard_count)
  int* status;
  uint64_t wait_limit_ns;
  int inject_stall;        // test hook: the MMA threads first wait on a barrier nobody arrives at
  // key-block launch (key_block != 0): only keys at positions [key_lo, key_hi) count, and
  // K/V are a [kv_rows][Hkv][d] tensor holding the key at position p of batch b in row
  // b * kv_rows_per_batch + kv_row_offset + p - key_lo (kv_layout is not used)
  int32_t key_block = 0;
  int32_t key_lo = 0, key_hi = 0;
  int32_t kv_rows_per_batch = 0, kv_row_offset = 0, kv_rows = 0;
};

struct BwdArgs {
  const void* q;
  const void* k;
  const void* v;
  const void* o;
  const float* lse;
  const void* dout;
  void* dq;
  void* dk;
  void* dv;
  float* delta;            // [shards][B][Hq][2C] workspace: -Delta (written by K2)
  float* nlse2;            // [shards][B][Hq][2C] workspace: -lse * log2(e) (written by K2)
  float* dq_acc;           // [Hq][shards*B*2C][d] workspace (head-major)
  int64_t S;
  int32_t B, Hq, Hkv, d, D, causal;
  float scale;
  int32_t kv_layout;       // as in FwdArgs; dK / dV are written in the same layout
  int32_t shard_begin, shard_count;
  int* status;
  uint64_t wait_limit_ns;
  int inject_stall;        // test hook: the MMA threads first wait on a barrier nobody arrives at
};

// Partial results to merge (ring attention): n parts of the Q layout (bf16 O) and the
// lse layout (fp32), rows = local Q-layout rows of the problem.
constexpr int kMergeMaxParts = 32;
// K5: natural [B][S][H][d] <-> shard-major [shards][B][2C][H][d] copy (bf16 rows).
struct PermuteArgs {
  const void* src;
  void* dst;
  int64_t chunk_words;     // 16-byte words in one chunk of one batch: C * H * d * 2 / 16
  int32_t B, D;
  int32_t shard_begin, shard_count;
  int32_t to_shard_major;  // 1: src natural, dst shard-major; 0: the reverse
};

struct MergeArgs {
  const void* o[kMergeMaxParts];
  const float* lse[kMergeMaxParts];
  void* o_out;
  float* lse_out;
  int64_t S, rows;
  int32_t Hq, d, D, n;
};

// One TSP step's local projection Y = X W (zsa_gemm.cu): X [T][K] (row stride ldx),
// W [K][N] (row stride ldw), columns of Y routed by segments.
constexpr int kProjMaxSegs = 8;
struct ProjSegment {
  void* out;               // element (0, 0) of the segment's output
  int64_t ld;              // its row stride (elements)
  int64_t col_begin, col_end;   // the columns of W it receives
  int32_t fp32_accumulate; // 0: bf16 output, overwritten; 1: fp32 output, +=
};
struct ProjArgs {
  const void* x;
  const void* w;
  int64_t T, N, K, ldx, ldw;
  int32_t n_segs;
  ProjSegment segs[kProjMaxSegs];
  int* status;
  uint64_t wait_limit_ns;
};

// Tiling the forward kernel is built for, per head dim.
inline void fwd_tiling(int d, int32_t* bq, int32_t* bk, int32_t* slots) {
  *bq = 128;
  *bk = d <= 128 ? 128 : 64;
  *slots = d <= 128 ? 2 : 1;
}

// Caller-owned CUDA events recorded around one kernel's launches (null = not traced).
struct TraceEvents {
  cudaEvent_t begin, end;
};
TraceEvents trace_events(int which);  // 0 fwd, 1 bwd pre, 2 bwd main, 3 dQ convert, 4 merge,
                                      // 5 projection GEMM, 6 permute

// Raises `func`'s dynamic shared-memory limit to `bytes` on the current device, once
// per (kernel, device): cudaFuncSetAttribute applies to the device current at the time
// of the call only.  Thread-safe.  Returns a cudaError_t.
int ensure_smem_attr(const void* func, int bytes);

// Wait limit and stall hook set through zsa_set_wait_limit_ns / zsa_debug_inject_stall;
// every entry point that launches a kernel reads them.
uint64_t wait_limit_ns();
int inject_stall();

// Returns a cudaError_t (cudaSuccess on success).
int launch_fwd(const FwdArgs& a, cudaStream_t stream);
int launch_bwd(const BwdArgs& a, cudaStream_t stream);
int launch_merge(const MergeArgs& a, cudaStream_t stream);
int launch_permute(const PermuteArgs& a, cudaStream_t stream);
int launch_proj_gemm(const ProjArgs& a, cudaStream_t stream);

}  // namespace zsa
