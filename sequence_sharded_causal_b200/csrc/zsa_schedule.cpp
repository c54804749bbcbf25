// zsa_schedule.cpp -- the forward tile schedule.
//
// Balance (the reason for the zigzag, "Folding Tensor and Sequence Parallelism"
// summary, section 2, attention layer): with block_q | C and block_k | block_q the
// per-(b, q head) tile work of shard r is
//   (block_q/block_k) * (T^2 (2D-1) + T (T+1)),  T = C / block_q,
// independent of r.  Positions rise along a shard's rows (its second chunk lies
// wholly after its first), so a tile's largest position is that of its last row.
#include "zsa_schedule.h"

#include <algorithm>

namespace zsa {

bool build_schedule(int64_t S, int32_t D, int32_t B, int32_t Hq, int32_t Hkv, int32_t causal,
                    int32_t bq, int32_t bk, int32_t slots, int32_t shard_begin,
                    int32_t shard_count, Schedule* out) {
  if (S <= 0 || D <= 0 || B <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0) return false;
  if (shard_begin < 0 || shard_count <= 0 || shard_begin + shard_count > D) return false;
  if (bq <= 0 || bk <= 0 || (slots != 1 && slots != 2)) return false;
  if (S % (2 * int64_t(D)) != 0 || (S / D) % bq != 0 || S % bk != 0) return false;
  const int64_t C = S / (2 * int64_t(D));
  const int64_t T = (2 * C) / bq;
  const int32_t G = Hq / Hkv;
  const int64_t n_key_tiles = S / bk;

  std::vector<int32_t> kend(size_t(D * T));
  for (int32_t r = 0; r < D; ++r)
    for (int64_t i = 0; i < T; ++i) {
      int64_t last = zigzag_pos(C, D, r, (i + 1) * bq - 1);
      kend[size_t(r * T + i)] = int32_t(causal ? last / bk + 1 : n_key_tiles);
    }

  out->S = S; out->D = D; out->B = B; out->Hq = Hq; out->Hkv = Hkv;
  out->causal = causal; out->bq = bq; out->bk = bk; out->slots = slots;
  out->shard_begin = shard_begin; out->shard_count = shard_count;
  out->shard_tiles.assign(size_t(D), 0);
  for (int32_t r = 0; r < D; ++r) {
    int64_t w = 0;
    for (int64_t i = 0; i < T; ++i) w += kend[size_t(r * T + i)];
    out->shard_tiles[size_t(r)] = w * B * Hq;
  }

  struct Keyed {
    int32_t work, r, m, b, g;
    DevUnit u;
  };
  const int64_t runs = (T * G + slots - 1) / slots;
  std::vector<Keyed> list;
  list.reserve(size_t(int64_t(B) * Hkv * shard_count * runs));
  for (int32_t b = 0; b < B; ++b)
    for (int32_t g = 0; g < Hkv; ++g)
      for (int32_t r = shard_begin; r < shard_begin + shard_count; ++r)
        for (int64_t m = 0; m < runs; ++m) {
          Keyed x;
          const int64_t s0 = m * slots, s1 = s0 + 1;
          x.u.r = r; x.u.b = b; x.u.g = g;
          x.u.tile0 = int32_t(s0 / G);
          x.u.head0 = int32_t(g * G + s0 % G);
          const int32_t k0 = kend[size_t(r * T + x.u.tile0)];
          int32_t k1 = 0;
          if (slots == 2 && s1 < T * G) {
            x.u.tile1 = int32_t(s1 / G);
            x.u.head1 = int32_t(g * G + s1 % G);
            k1 = kend[size_t(r * T + x.u.tile1)];
          } else {
            x.u.tile1 = -1;
            x.u.head1 = -1;
          }
          x.u.kend = k0 | (k1 << 16);
          x.work = std::max(k0, k1);
          x.r = r; x.m = int32_t(m); x.b = b; x.g = g;
          list.push_back(x);
        }
  // Grouped by (b, kv head) so that units running at the same time share one head's
  // K/V in L2; longest first within a group so each group ends with its shortest units.
  std::sort(list.begin(), list.end(), [](const Keyed& a, const Keyed& c) {
    if (a.b != c.b) return a.b < c.b;
    if (a.g != c.g) return a.g < c.g;
    if (a.work != c.work) return a.work > c.work;
    if (a.r != c.r) return a.r < c.r;
    return a.m < c.m;
  });
  out->units.resize(list.size());
  for (size_t k = 0; k < list.size(); ++k) out->units[k] = list[k].u;
  return true;
}

}  // namespace zsa
