// zsa_bwd_common.cuh -- pieces shared by the backward main kernels: launch parameters,
// the key-tile unit decode and the slot walk (which q slots see a key tile).
#pragma once
#include <cuda_bf16.h>

#include "zsa_kernels.h"
#include "zsa_ptx.cuh"

namespace zsa {
namespace bwd {

constexpr float kLog2e = 1.4426950408889634f;
constexpr int kUnitRing = 4;   // claimed units in flight between the producer and the others

struct BwdParams {
  const float* nlse2;         // -lse * log2(e), [shards][B][Hq][2C] (K2)
  const float* ndelta;        // -Delta, same layout (K2)
  float* dq_acc;
  __nv_bfloat16* dk;
  __nv_bfloat16* dv;
  int64_t S, C;
  int32_t B, Hq, Hkv, G, D, causal;
  int32_t n_units, n_qtiles;  // n_qtiles = BQ-row tiles per shard
  int32_t bq;                 // query rows per slot
  int32_t n_ktiles;           // S / 128
  int32_t kv_shard_major;     // K/V/dK/dV rows in the shard-major zigzag order
  int32_t kv_box;             // rows per K / V TMA box (128, or 64 when C % 128 != 0)
  int32_t shard_begin, shard_end;   // the launch computes the queries of these shards
  int64_t rows;               // local Q-layout rows: (shard_end - shard_begin) * B * 2C
  float scale, scale_log2;
  int* status;
  int* counter;       // next unclaimed unit (zeroed before every launch)
  uint64_t wait_limit_ns;
  int inject_stall;
};

// One key tile of work.
struct KvUnit {
  int32_t n, b, g;   // key tile, batch, kv head
};

// Units are claimed dynamically in the order (b, kv head g, key tile n): CTAs busy at
// the same time work on one head group, sharing its Q / dO stream and its dQ
// accumulator rows in L2; within a group n ascends, i.e. the work per unit (the number
// of q tiles that see key tile n) descends, so each group ends with its shortest units.
__device__ __forceinline__ KvUnit decode_kv_unit(int idx, int Hkv, int NT) {
  KvUnit u;
  u.n = idx % NT;
  u.g = (idx / NT) % Hkv;
  u.b = idx / (NT * Hkv);
  return u;
}

// Enumerates the q slots (shard r, BQ-row tile i, head offset e) that see key tile n,
// in (r, i, e) order.  Every role walks the same sequence.  A BQ-row tile never
// straddles a zigzag chunk (C is a multiple of 64), so its positions are contiguous.
struct SlotWalk {
  int32_t r, i, e;
  int64_t p0;   // position of the tile's first row (its rows are p0 .. p0+BQ-1)
};

__device__ __forceinline__ int64_t zz_pos(int64_t C, int32_t D, int32_t r, int64_t j) {
  return j < C ? int64_t(r) * C + j : int64_t(2 * D - 1 - r) * C + (j - C);
}

__device__ __forceinline__ bool tile_sees(const BwdParams& p, int32_t r, int32_t i, int32_t n,
                                          int64_t* p0) {
  *p0 = zz_pos(p.C, p.D, r, int64_t(i) * p.bq);
  // positions rise along a shard, so the tile's last row holds its largest position
  return !p.causal || (zz_pos(p.C, p.D, r, int64_t(i) * p.bq + p.bq - 1) >= int64_t(n) * 128);
}

// First slot at or after (r, i, 0); false when the walk is over.  Only the launch's
// shards [shard_begin, shard_end) are walked.
__device__ __forceinline__ bool walk_seek(const BwdParams& p, int32_t n, SlotWalk& w) {
  while (w.r < p.shard_end) {
    if (tile_sees(p, w.r, w.i, n, &w.p0)) return true;
    if (++w.i == p.n_qtiles) {
      w.i = 0;
      ++w.r;
    }
  }
  return false;
}
__device__ __forceinline__ bool walk_first(const BwdParams& p, int32_t n, SlotWalk& w) {
  w.r = p.shard_begin; w.i = 0; w.e = 0;
  return walk_seek(p, n, w);
}
__device__ __forceinline__ bool walk_next(const BwdParams& p, int32_t n, SlotWalk& w) {
  if (++w.e < p.G) return true;
  w.e = 0;
  if (++w.i == p.n_qtiles) {
    w.i = 0;
    ++w.r;
  }
  return walk_seek(p, n, w);
}

__device__ __forceinline__ bool warp_wait_b(uint64_t* bar, uint32_t parity, const WaitCtx& w) {
  bool ok = mbar_wait(bar, parity, w);
  return __all_sync(0xffffffffu, ok);
}

// d = 256 backward main kernel on clusters of two CTAs (zsa_bwd_pair.cu).
int launch_pair_main(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                     const CUtensorMap& mdo, const CUtensorMap& mdq, const BwdParams& p,
                     cudaStream_t stream);

}  // namespace bwd
}  // namespace zsa
