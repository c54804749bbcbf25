// zsa_schedule.h -- zigzag index map and forward tile schedule (host side).
#pragma once
#include <cstdint>
#include <vector>

namespace zsa {

// Zigzag rule: shard r holds chunk r then chunk 2D-1-r, chunks of C = S/(2D) positions.
inline int64_t zigzag_pos(int64_t C, int32_t D, int32_t r, int64_t j) {
  return j < C ? int64_t(r) * C + j : int64_t(2 * D - 1 - r) * C + (j - C);
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
  std::vector<int64_t> shard_tiles;  // [D]
  std::vector<DevUnit> units;        // launch order
};

// Returns false for an invalid tiling.
bool build_schedule(int64_t S, int32_t D, int32_t B, int32_t Hq, int32_t Hkv, int32_t causal,
                    int32_t bq, int32_t bk, int32_t slots, Schedule* out);

}  // namespace zsa
