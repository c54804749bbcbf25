// zsa_schedule.h -- zigzag index map and forward tile schedule (host side).
#pragma once
#include <cstdint>
#include <vector>

#if defined(__CUDACC__)
#define ZSA_HD __host__ __device__ __forceinline__
#else
#define ZSA_HD inline
#endif

namespace zsa {

// Zigzag rule: shard r holds chunk r then chunk 2D-1-r, chunks of C = S/(2D) positions.
ZSA_HD int64_t zigzag_pos(int64_t C, int32_t D, int32_t r, int64_t j) {
  return j < C ? int64_t(r) * C + j : int64_t(2 * D - 1 - r) * C + (j - C);
}

// Inverse of zigzag_pos: the (shard, row) holding position p, as the shard-major row
// index r*2C + j.
ZSA_HD int64_t zigzag_row(int64_t C, int32_t D, int64_t p) {
  const int64_t c = p / C, o = p % C;
  return c < D ? c * 2 * C + o : (2 * D - 1 - c) * 2 * C + C + o;
}

// Row of a K / V tensor ([rows][Hkv][d]) holding position p of batch b: b*S + p in
// position order, or the zigzag owner's row (r*B + b)*2C + j in the shard-major order
// (the all-gather of every shard's own rows).  C = S/(2D) is passed in (no division by
// a 64-bit value on the device); positions and rows fit in 32 bits (B*S < 2^31).  A
// 64-key box starting at a multiple of 64 lies inside one zigzag chunk (C % 64 == 0),
// so its rows are contiguous either way.
ZSA_HD int32_t kv_tensor_row(int32_t p, int32_t b, int32_t S, int32_t C, int32_t B, int32_t D,
                             int32_t shard_major) {
  if (!shard_major) return b * S + p;
  const uint32_t c = uint32_t(p) / uint32_t(C);
  const int32_t o = p - int32_t(c) * C;
  const int32_t r = int32_t(c) < D ? int32_t(c) : 2 * D - 1 - int32_t(c);
  const int32_t j = int32_t(c) < D ? o : C + o;
  return (r * B + b) * 2 * C + j;
}

// Device-side record of one forward work unit (32 bytes).
struct DevUnit {
  int32_t r, b, g;
  int32_t tile0, head0, tile1, head1;
  int32_t kend;  // kend0 | kend1 << 16
};

struct Schedule {
  int64_t S;
  int32_t D, B, Hq, Hkv, causal, bq, bk, slots;
  int32_t shard_begin, shard_count;  // units of shards [begin, begin + count) only
  std::vector<int64_t> shard_tiles;  // [D]
  std::vector<DevUnit> units;        // launch order
};

// Returns false for an invalid tiling.  shard_tiles covers every shard; the unit list
// only the shards [shard_begin, shard_begin + shard_count), in the order the full list
// would have them.
bool build_schedule(int64_t S, int32_t D, int32_t B, int32_t Hq, int32_t Hkv, int32_t causal,
                    int32_t bq, int32_t bk, int32_t slots, int32_t shard_begin,
                    int32_t shard_count, Schedule* out);

}  // namespace zsa
