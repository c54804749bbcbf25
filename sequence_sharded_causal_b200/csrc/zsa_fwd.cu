// zsa_fwd.cu -- forward kernel (K1): zigzag-sharded causal GQA attention on sm_100a.
//
// Method: every shard's queries attend FlashAttention-style to the full gathered K/V
// ("Folding Tensor and Sequence Parallelism" summary, section 2, attention layer), the
// causal mask on global positions ("AutoSP" summary, section 2.A step 4), q heads
// sharing kv heads ("Tensor, pipeline e sequence parallelism", 01 Conceito).  The
// pages give no kernel design; this one is built for the B200:
//
//  * persistent CTAs, one per SM, claim units of the host-built table from a global
//    counter (the table is grouped by (b, kv head), longest first within a group, so
//    CTAs busy at the same time share one head's K/V in L2);
//  * a unit is up to NSLOT (q tile, q head) slots of 128 query rows that share one K/V
//    stream: two q heads of one kv group (GQA) or two adjacent q tiles (MHA), so a
//    K/V tile fetched once feeds 2 x 128 rows of MMAs;
//  * warp roles: 4 softmax warps per slot (one TMEM lane = one query row per thread),
//    1 TMA producer warp, 2 MMA warps (one thread each issues tcgen05.mma: one the QK
//    list, one the PV list);
//  * S = Q K^T goes to one TMEM buffer (128 x BK fp32) shared by the slots; the softmax
//    warps of the slot it belongs to copy it to registers and release it at once
//    (s_free), apply the global-position mask, keep a running max (rescaling O in TMEM
//    only when the max grows by more than 2^8) and write P as bf16 to the slot's own P
//    columns; O += P V is a TMEM-A MMA (P from TMEM, V from shared memory as an
//    MN-major operand);
//  * shared memory: Q tiles resident for the unit, a K ring and a V ring of ST stages,
//    all 128B-swizzled TMA tiles; TMEM: S | P0 | P1 | O0 | O1 (512 columns at d = 128).
// The QK MMAs of a unit run in (key tile, slot) order through the S buffer, each one
// issued as soon as the previous S has been copied out, so the next tile's scores are
// computed while the softmax still works on the current one.  PV_s(n) is issued as soon
// as P_s(n) is published (p_full), by the other issuing thread, so neither list waits
// behind the other.  The softmax waits for PV_s(n-1) (pv_done) only before it
// overwrites P_s or rescales O_s, after its exponentials.
//
// The key-block build (KR = true, zsa_attn_fwd_block) is the same kernel restricted to the
// keys of one K/V block, the partial of a ring-attention step ("AutoSP" summary, sections
// 1 and 4): each slot's key tiles are clamped to the block's, K/V rows come from the
// block's linear row map, the mask adds the block's bounds, and a row that sees no key of
// the block ends as O = 0, lse = -inf.
#include <cuda_bf16.h>

#include <cmath>

#include "zsa_kernels.h"
#include "zsa_ptx.cuh"
#include "zsa_tma_host.h"

namespace zsa {
namespace {

template <int HD>
struct FwdCfg {
  static constexpr int NSLOT = HD <= 128 ? 2 : 1;
  static constexpr int BQ = 128;
  static constexpr int BK = HD <= 128 ? 128 : 64;
  static constexpr int ST = HD == 64 ? 4 : 2;
  static constexpr int KB = HD / 64;                  // 64-wide (128-byte) d blocks
  static constexpr int Q_BYTES = BQ * HD * 2;
  static constexpr int KV_BYTES = BK * HD * 2;
  static constexpr int SMEM_Q = 0;
  static constexpr int SMEM_K = SMEM_Q + NSLOT * Q_BYTES;
  static constexpr int SMEM_V = SMEM_K + ST * KV_BYTES;
  static constexpr int SMEM_BYTES = SMEM_V + ST * KV_BYTES;
  static constexpr int NWARP_SOFTMAX = 4 * NSLOT;
  static constexpr int WARP_LOAD = NWARP_SOFTMAX;
  static constexpr int WARP_MMA = NWARP_SOFTMAX + 1;   // QK issuer (and TMEM owner)
  static constexpr int WARP_PV = NWARP_SOFTMAX + 2;    // PV issuer
  static constexpr int NTHREADS = (NWARP_SOFTMAX + 3) * 32;
  static constexpr uint32_t TM_COLS = 512;
  static constexpr uint32_t TM_S = 0;                                     // BK columns
  __device__ static constexpr uint32_t tm_p(int s) { return uint32_t(BK + s * (BK / 2)); }
  __device__ static constexpr uint32_t tm_o(int s) { return uint32_t(256 + s * HD); }
  static_assert(SMEM_BYTES + 1024 <= 227 * 1024, "shared memory budget");
  static_assert(BK + NSLOT * (BK / 2) <= 256 && 256 + NSLOT * HD <= 512, "TMEM budget");
};

struct FwdParams {
  const DevUnit* units;
  int32_t n_units;
  __nv_bfloat16* o;
  float* lse;
  int64_t S, C;
  int32_t B, Hq, Hkv, D, causal;
  // A key-block launch (KR) reuses the two K/V layout fields for its linear row map.
  // (The parameter block is kept this small on purpose: at the d <= 128 register budget
  // a few more words of it made ptxas spill in the softmax warps.)
  union {
    int32_t kv_shard_major;  // K/V rows in the shard-major zigzag order instead of position order
    int32_t kb_rpb;          // KR: K/V rows per batch
  };
  int32_t shard_begin;       // first shard this launch computes (Q-layout rows are local)
  union {
    int32_t kv_box;          // rows per K / V TMA box: BK when a key tile never straddles a
                             // zigzag chunk (C % BK == 0), else 64 (C is a multiple of 64)
    int32_t kb_off;          // KR: K/V row of (batch 0, position key_lo)
  };
  int32_t key_lo, key_hi;    // KR: only keys at positions [key_lo, key_hi) count; the key at
                             // position p of batch b is K/V row b * kb_rpb + kb_off + p - key_lo
  float scale_log2;
  int* status;
  int* counter;       // next unclaimed unit (zeroed before every launch)
  uint64_t wait_limit_ns;
  int inject_stall;
};

constexpr int kUnitRing = 4;  // claimed units in flight between the producer and the others

struct FwdBars {
  uint64_t q_full[2], q_empty[2];
  uint64_t k_full[4], k_empty[4], v_full[4], v_empty[4];
  uint64_t s_full[2], s_free, p_full[2], pv_done[2], o_full[2], o_empty[2];
  uint64_t unit_full[kUnitRing], unit_empty[kUnitRing];
  uint64_t drain;
  uint64_t never;  // test hook: no one ever arrives here
};

// kend[s] counts the slot's key tiles from n0 on: all tiles up to the causal limit
// (n0 = 0), or, in a key-range launch, those inside [n_lo, n_hi) (n0 = n_lo; a present
// slot may then have none: its rows see no key of the range).
struct UnitInfo {
  int32_t r, b, g;
  int32_t tile[2], head[2], kend[2];
  int32_t nmax, n0;
  uint32_t live;           // bit s: slot s holds a q tile (its kend before any clamp > 0)
};

template <int HD, bool KR>
__device__ __forceinline__ UnitInfo load_unit(const DevUnit* units, int idx, const FwdParams& prm) {
  const int4* p = reinterpret_cast<const int4*>(units + idx);
  int4 a = __ldg(p), c = __ldg(p + 1);
  UnitInfo u;
  u.r = a.x; u.b = a.y; u.g = a.z;
  u.tile[0] = a.w; u.head[0] = c.x; u.tile[1] = c.y; u.head[1] = c.z;
  u.kend[0] = c.w & 0xFFFF;
  u.kend[1] = (c.w >> 16) & 0xFFFF;
  u.n0 = 0;
  u.live = (u.kend[0] > 0 ? 1u : 0u) | (u.kend[1] > 0 ? 2u : 0u);
  if constexpr (KR) {
    // the block's key tiles are [n_lo, n_hi)
    const int32_t n_lo = prm.key_lo / FwdCfg<HD>::BK;
    const int32_t n_hi = (prm.key_hi + FwdCfg<HD>::BK - 1) / FwdCfg<HD>::BK;
    u.n0 = n_lo;
    for (int s = 0; s < 2; ++s) {
      const int32_t e = u.kend[s] < n_hi ? u.kend[s] : n_hi;
      u.kend[s] = e > n_lo ? e - n_lo : 0;
    }
  }
  u.nmax = u.kend[0] > u.kend[1] ? u.kend[0] : u.kend[1];
  return u;
}

// K/V tensor row of the key at position p of batch b.  A key-block launch maps positions
// linearly, so a whole BK tile is one box even where it overhangs the block: rows before
// the block (a negative coordinate reads zeros) or past it hold keys the mask removes.
template <bool KR>
__device__ __forceinline__ int32_t kv_row(const FwdParams& prm, int32_t p, int32_t b) {
  if constexpr (KR) return b * prm.kb_rpb + prm.kb_off + (p - prm.key_lo);
  else return kv_tensor_row(p, b, int32_t(prm.S), int32_t(prm.C), prm.B, prm.D, prm.kv_shard_major);
}


// Every lane polls; the outcome is made warp-uniform so .sync.aligned TMEM ops that
// follow are executed by the full warp or by none of it.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, const WaitCtx& w) {
  bool ok = mbar_wait(bar, parity, w);
  return __all_sync(0xffffffffu, ok);
}

template <int HD, bool KR>
__global__ void __launch_bounds__(FwdCfg<HD>::NTHREADS, 1)
    zsa_fwd_kernel(const __grid_constant__ CUtensorMap map_q,
                   const __grid_constant__ CUtensorMap map_k,
                   const __grid_constant__ CUtensorMap map_v, const FwdParams prm) {
  using Cfg = FwdCfg<HD>;
  constexpr int NSLOT = Cfg::NSLOT, BK = Cfg::BK, ST = Cfg::ST, KB = Cfg::KB;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  __shared__ FwdBars bars;
  __shared__ uint32_t tmem_base_s;
  __shared__ int abort_s;
  __shared__ int unit_ring[kUnitRing];

  const int warp = int(warp_id()), lane = int(lane_id());
  if (threadIdx.x == 0) {
    abort_s = 0;
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars.q_full[s], 1);
      mbar_init(&bars.q_empty[s], 1);
      mbar_init(&bars.s_full[s], 1);
      mbar_init(&bars.p_full[s], 4);
      mbar_init(&bars.pv_done[s], 1);
      mbar_init(&bars.o_full[s], 1);
      mbar_init(&bars.o_empty[s], 4);
    }
    for (int s = 0; s < 4; ++s) {
      mbar_init(&bars.k_full[s], 1);
      mbar_init(&bars.k_empty[s], 1);
      mbar_init(&bars.v_full[s], 1);
      mbar_init(&bars.v_empty[s], 1);
    }
    for (int s = 0; s < kUnitRing; ++s) {
      mbar_init(&bars.unit_full[s], 1);
      mbar_init(&bars.unit_empty[s], 2 + 4 * Cfg::NSLOT);   // 2 MMA threads + softmax warps
    }
    mbar_init(&bars.s_free, 4);                             // the 4 warps of the slot it held
    mbar_init(&bars.drain, 2);                              // one commit per MMA thread
    mbar_init(&bars.never, 1);
    fence_mbar_init();
  }
  if (warp == Cfg::WARP_MMA) {
    tmem_alloc(&tmem_base_s, Cfg::TM_COLS);
    tmem_relinquish();
  }
  if (warp == Cfg::WARP_LOAD && lane == 0) {
    tma_prefetch_desc(&map_q);
    tma_prefetch_desc(&map_k);
    tma_prefetch_desc(&map_v);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_s;
  const WaitCtx wctx{&abort_s, prm.status, prm.wait_limit_ns};
  const uint32_t sQ = smem_u32(smem + Cfg::SMEM_Q);
  const uint32_t sK = smem_u32(smem + Cfg::SMEM_K);
  const uint32_t sV = smem_u32(smem + Cfg::SMEM_V);
  const int64_t twoC = 2 * prm.C;

  if (warp == Cfg::WARP_LOAD) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      uint32_t kv_it = 0;
      uint32_t q_fills[2] = {0, 0};
      uint32_t k_fills[ST], v_fills[ST];
      for (int st = 0; st < ST; ++st) k_fills[st] = v_fills[st] = 0;
      bool ok = true;
      for (int k = 0; ok; ++k) {
        // Claim the next unit of the table (dynamic scheduling: the table is grouped
        // by kv head, so CTAs busy at the same time share that head's K/V in L2) and
        // hand it to the MMA threads and the softmax warps through the ring.
        const int slot = k % kUnitRing;
        if (k >= kUnitRing) ok = mbar_wait(&bars.unit_empty[slot], ((k / kUnitRing) - 1) & 1, wctx);
        if (!ok) break;
        int idx = atomicAdd(prm.counter, 1);
        if (idx >= prm.n_units) idx = -1;
        unit_ring[slot] = idx;
        mbar_arrive(&bars.unit_full[slot]);
        if (idx < 0) break;
        const UnitInfo u = load_unit<HD, KR>(prm.units, idx, prm);
        for (int s = 0; s < NSLOT && ok; ++s) {
          if (u.kend[s] == 0) continue;
          if (q_fills[s] > 0) ok = mbar_wait(&bars.q_empty[s], (q_fills[s] - 1) & 1, wctx);
          if (!ok) break;
          mbar_expect_tx(&bars.q_full[s], Cfg::Q_BYTES);
          const int32_t row0 =
              int32_t((int64_t(u.r - prm.shard_begin) * prm.B + u.b) * twoC + int64_t(u.tile[s]) * 128);
          for (int kb = 0; kb < KB; ++kb)
            tma_load_3d(smem + Cfg::SMEM_Q + s * Cfg::Q_BYTES + kb * 128 * 128, &map_q,
                        &bars.q_full[s], kb * 64, u.head[s], row0);
          ++q_fills[s];
        }
        // K runs one tile ahead of V: the MMA threads need K(n+1) (for QK(n+1)) before
        // V(n) (for PV(n)).
        for (int n = 0; n <= u.nmax && ok; ++n) {
          if (n < u.nmax) {
            const uint32_t it = kv_it + uint32_t(n);
            const int st = int(it % ST);
            const uint32_t use = it / ST;
            if (use > 0) ok = mbar_wait(&bars.k_empty[st], (use - 1) & 1, wctx);
            if (!ok) break;
            mbar_expect_tx(&bars.k_full[st], Cfg::KV_BYTES);
            if (KR || prm.kv_box == BK) { // the tile's rows are contiguous: one box per d block
              const int32_t krow = kv_row<KR>(prm, (u.n0 + n) * BK, u.b);
              for (int kb = 0; kb < KB; ++kb)
                tma_load_3d(smem + Cfg::SMEM_K + st * Cfg::KV_BYTES + kb * BK * 128, &map_k,
                            &bars.k_full[st], kb * 64, u.g, krow);
            } else {                      // 64-key boxes, one zigzag chunk each
              for (int hb = 0; hb < BK / 64; ++hb) {
                const int32_t krow = kv_tensor_row((u.n0 + n) * BK + hb * 64, u.b, int32_t(prm.S),
                                                   int32_t(prm.C), prm.B, prm.D, prm.kv_shard_major);
                for (int kb = 0; kb < KB; ++kb)
                  tma_load_3d(smem + Cfg::SMEM_K + st * Cfg::KV_BYTES + kb * BK * 128 + hb * 64 * 128,
                              &map_k, &bars.k_full[st], kb * 64, u.g, krow);
              }
            }
            ++k_fills[st];
          }
          if (n >= 1) {
            const uint32_t it = kv_it + uint32_t(n - 1);
            const int st = int(it % ST);
            const uint32_t use = it / ST;
            if (use > 0) ok = mbar_wait(&bars.v_empty[st], (use - 1) & 1, wctx);
            if (!ok) break;
            mbar_expect_tx(&bars.v_full[st], Cfg::KV_BYTES);
            if (KR || prm.kv_box == BK) {
              const int32_t vrow = kv_row<KR>(prm, (u.n0 + n - 1) * BK, u.b);
              for (int kb = 0; kb < KB; ++kb)
                tma_load_3d(smem + Cfg::SMEM_V + st * Cfg::KV_BYTES + kb * BK * 128, &map_v,
                            &bars.v_full[st], kb * 64, u.g, vrow);
            } else {
              for (int hb = 0; hb < BK / 64; ++hb) {
                const int32_t vrow = kv_tensor_row((u.n0 + n - 1) * BK + hb * 64, u.b, int32_t(prm.S),
                                                   int32_t(prm.C), prm.B, prm.D, prm.kv_shard_major);
                for (int kb = 0; kb < KB; ++kb)
                  tma_load_3d(smem + Cfg::SMEM_V + st * Cfg::KV_BYTES + kb * BK * 128 + hb * 64 * 128,
                              &map_v, &bars.v_full[st], kb * 64, u.g, vrow);
              }
            }
            ++v_fills[st];
          }
        }
        kv_it += uint32_t(u.nmax);
      }
      if (!ok) {
        // Teardown after an abort: wait (bounded) for every fill still in flight.
        const uint64_t lim = 1000000000ull;
        for (int s = 0; s < NSLOT; ++s)
          if (q_fills[s] > 0) mbar_drain(&bars.q_full[s], (q_fills[s] - 1) & 1, lim);
        for (int st = 0; st < ST; ++st) {
          if (k_fills[st] > 0) mbar_drain(&bars.k_full[st], (k_fills[st] - 1) & 1, lim);
          if (v_fills[st] > 0) mbar_drain(&bars.v_full[st], (v_fills[st] - 1) & 1, lim);
        }
      }
    }
  } else if (warp == Cfg::WARP_MMA || warp == Cfg::WARP_PV) {
    // ------------------------------------------------------------ MMA issuers
    // Two threads issue tcgen05.mma: one the QK list, one the PV list, each in (key tile
    // n, slot s) order over the pairs with n < kend[s].  They share the tensor pipe but
    // not their bookkeeping, so one thread's barrier waits and index arithmetic never
    // leave the pipe idle while the other has work.  tcgen05.commit tracks the issuing
    // thread's own MMAs, so each commits what it issued.
    if (lane == 0) {
      const bool qk_role = warp == Cfg::WARP_MMA;
      const uint32_t idesc_qk = idesc_bf16(128, BK, false, false);
      const uint32_t idesc_pv = idesc_bf16(128, HD, false, true);
      uint32_t kv_it = 0, qk_total = 0;
      // per-slot phase bits (bit s), kept in registers: the slot index is dynamic here
      uint32_t q_ph = 0, p_ph = 0, oe_ph = 0, o_pending = 0;
      bool ok = true;
      if (prm.inject_stall) ok = mbar_wait(&bars.never, 0, wctx);
      for (int k = 0; ok; ++k) {
        const int slot = k % kUnitRing;
        ok = mbar_wait(&bars.unit_full[slot], (k / kUnitRing) & 1, wctx);
        if (!ok) break;
        const int idx = *reinterpret_cast<volatile int*>(&unit_ring[slot]);
        mbar_arrive(&bars.unit_empty[slot]);
        if (idx < 0) break;
        const UnitInfo u = load_unit<HD, KR>(prm.units, idx, prm);
        const int k0 = u.kend[0], k1 = NSLOT == 2 ? u.kend[1] : 0;
        // (n, s) walk over present pairs; first / last: s opens / closes key tile n
        int n = 0, sl = k0 > 0 ? 0 : 1;
        if (qk_role) {
          for (int s = 0; s < NSLOT && ok; ++s) {
            if (u.kend[s] == 0) continue;
            ok = mbar_wait(&bars.q_full[s], (q_ph >> s) & 1u, wctx);
            q_ph ^= 1u << s;
          }
          for (int i = 0; i < k0 + k1 && ok; ++i) {
            // ---- QK_sl(n): S = Q_sl K(n)^T into the shared S buffer
            const uint32_t it = kv_it + uint32_t(n);
            const int st = int(it % ST);
            const bool first = sl == 0 || n >= k0;
            const bool last = sl == 1 || n >= k1;
            if (qk_total > 0) ok = mbar_wait(&bars.s_free, (qk_total - 1) & 1, wctx);
            if (ok && first) ok = mbar_wait(&bars.k_full[st], (it / ST) & 1, wctx);
            if (!ok) break;
            tc_fence_after();
            for (int kb = 0; kb < KB; ++kb)
#pragma unroll
              for (int ks = 0; ks < 4; ++ks) {
                const uint64_t a = sdesc_sw128(sQ + sl * Cfg::Q_BYTES + kb * 128 * 128 + ks * 32, 16, 1024);
                const uint64_t b = sdesc_sw128(sK + st * Cfg::KV_BYTES + kb * BK * 128 + ks * 32, 16, 1024);
                mma_ss(tmem + Cfg::TM_S, a, b, idesc_qk, (kb | ks) != 0);
              }
            mma_commit(&bars.s_full[sl]);
            if (n == (sl == 0 ? k0 : k1) - 1) mma_commit(&bars.q_empty[sl]);
            if (last) mma_commit(&bars.k_empty[st]);
            ++qk_total;
            if (sl == 0 && n < k1) {
              sl = 1;
            } else {
              ++n;
              sl = n < k0 ? 0 : 1;
            }
          }
        } else {
          for (int i = 0; i < k0 + k1 && ok; ++i) {
            // ---- PV_sl(n): O_sl += P_sl V(n)
            const uint32_t it = kv_it + uint32_t(n);
            const int st = int(it % ST);
            const bool first = sl == 0 || n >= k0;
            const bool last = sl == 1 || n >= k1;
            if (first) ok = mbar_wait(&bars.v_full[st], (it / ST) & 1, wctx);
            if (ok) ok = mbar_wait(&bars.p_full[sl], (p_ph >> sl) & 1u, wctx);
            p_ph ^= 1u << sl;
            if (ok && n == 0 && ((o_pending >> sl) & 1u)) {
              ok = mbar_wait(&bars.o_empty[sl], (oe_ph >> sl) & 1u, wctx);
              oe_ph ^= 1u << sl;
              o_pending &= ~(1u << sl);
            }
            if (!ok) break;
            tc_fence_after();
            const uint32_t tO = tmem + Cfg::tm_o(sl), tP = tmem + Cfg::tm_p(sl);
#pragma unroll
            for (int ks = 0; ks < BK / 16; ++ks) {
              const uint64_t b = sdesc_sw128(sV + st * Cfg::KV_BYTES + ks * 2048, BK * 128, 1024);
              mma_ts(tO, tP + ks * 8, b, idesc_pv, (n > 0) || (ks > 0));
            }
            mma_commit(&bars.pv_done[sl]);
            if (n == (sl == 0 ? k0 : k1) - 1) {
              mma_commit(&bars.o_full[sl]);
              o_pending |= 1u << sl;
            }
            if (last) mma_commit(&bars.v_empty[st]);
            if (sl == 0 && n < k1) {
              sl = 1;
            } else {
              ++n;
              sl = n < k0 ? 0 : 1;
            }
          }
        }
        kv_it += uint32_t(u.nmax);
      }
      // Teardown: every MMA issued so far completes before TMEM is released.
      mma_commit(&bars.drain);
      mbar_drain(&bars.drain, 0, 1000000000ull);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax warps
    const int s = warp / 4;            // slot
    const int qw = warp % 4;           // TMEM lane quarter
    const int row = qw * 32 + lane;    // query row within the tile = TMEM lane
    const uint32_t lane_addr = uint32_t(qw * 32) << 16;
    const uint32_t tS = tmem + Cfg::TM_S + lane_addr;
    const uint32_t tP = tmem + Cfg::tm_p(s) + lane_addr;
    const uint32_t tO = tmem + Cfg::tm_o(s) + lane_addr;
    uint32_t s_ph = 0, o_ph = 0;
    uint32_t pv_base = 0;              // PV_s MMAs committed in earlier units
    bool ok = true;
    for (int k = 0; ok; ++k) {
      const int slot = k % kUnitRing;
      ok = warp_wait(&bars.unit_full[slot], (k / kUnitRing) & 1, wctx);
      if (!ok) break;
      const int idx = *reinterpret_cast<volatile int*>(&unit_ring[slot]);
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.unit_empty[slot]);
      if (idx < 0) break;
      const UnitInfo u = load_unit<HD, KR>(prm.units, idx, prm);
      if (u.kend[s] == 0) {
        if constexpr (KR) {
          // a q tile that sees no key of the block: O = 0, lse = -inf, no MMA involved
          if ((u.live >> s) & 1u) {
            const int64_t j = int64_t(u.tile[s]) * 128 + row;
            const int64_t rb = int64_t(u.r - prm.shard_begin) * prm.B + u.b;
            uint4* dst = reinterpret_cast<uint4*>(prm.o + ((rb * twoC + j) * prm.Hq + u.head[s]) * HD);
#pragma unroll 4
            for (int v4 = 0; v4 < HD / 8; ++v4) dst[v4] = make_uint4(0u, 0u, 0u, 0u);
            prm.lse[(rb * prm.Hq + u.head[s]) * twoC + j] = -INFINITY;
          }
        }
        continue;
      }
      const int64_t j = int64_t(u.tile[s]) * 128 + row;             // row within the shard
      const int64_t pos = j < prm.C ? int64_t(u.r) * prm.C + j
                                    : int64_t(2 * prm.D - 1 - u.r) * prm.C + (j - prm.C);
      float m_run = -INFINITY, l_run = 0.f, r_run = 0.f;
      for (int n = 0; n < u.kend[s]; ++n) {
        ok = warp_wait(&bars.s_full[s], s_ph, wctx);
        s_ph ^= 1;
        if (!ok) break;
        tc_fence_after();
        uint32_t sr[BK / 32][32];
#pragma unroll
        for (int c = 0; c < BK / 32; ++c) tmem_ld32(tS + c * 32, sr[c]);
        tmem_ld_wait();
        // the scores are in registers: the S buffer may take the next QK
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars.s_free);
        // Causal mask on the tiles that cross this warp's diagonal only: keys past
        // `lim` (relative to the tile) are invisible to this row.  Off-diagonal tiles
        // (all but about one in kend) skip the mask entirely.
        if constexpr (!KR) {
          const int64_t rel = pos - int64_t(n) * BK;
          const int lim = rel >= BK ? BK : int(rel);            // >= 0: key 0 is always visible
          if (prm.causal && __any_sync(0xffffffffu, lim < BK - 1)) {
#pragma unroll
            for (int c = 0; c < BK / 32; ++c)
#pragma unroll
              for (int e = 0; e < 32; ++e)
                if (c * 32 + e > lim) sr[c][e] = 0xFF800000u;  // -inf
          }
        } else {
          // visible: keys e of the tile with lo <= e <= hi (the block's bounds, and the
          // causal limit); a row may see none of them (lo > hi)
          const int32_t k0 = (u.n0 + n) * BK;
          int hi = prm.key_hi - k0 - 1;
          if (prm.causal && pos - k0 < hi) hi = int(pos - k0);
          const int lo = prm.key_lo - k0;
          if (__any_sync(0xffffffffu, lo > 0 || hi < BK - 1)) {
#pragma unroll
            for (int c = 0; c < BK / 32; ++c)
#pragma unroll
              for (int e = 0; e < 32; ++e)
                if (c * 32 + e > hi || c * 32 + e < lo) sr[c][e] = 0xFF800000u;
          }
        }
        // row max of the raw scores (three-input max, four independent chains)
        float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int c = 0; c < BK / 32; ++c)
#pragma unroll
          for (int e = 0; e < 32; e += 2)
            mx[(e >> 1) & 3] = max3f(mx[(e >> 1) & 3], __uint_as_float(sr[c][e]),
                                     __uint_as_float(sr[c][e + 1]));
        const float m_new = fmaxf(m_run, fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])) * prm.scale_log2);
        // The running max (log2 units) moves only when it grows by more than 2^8; O was
        // accumulated against the old max, so it (and l) are scaled down by alpha.  The
        // decision is per row, but the TMEM access is warp-collective (.sync.aligned),
        // so the whole warp takes the rescale branch when any of its rows needs it
        // (alpha = 1 for the others).
        float alpha = 1.0f;
        const bool grow = m_new > m_run + 8.0f;       // always true at n == 0
        if (grow) {
          if (n > 0) alpha = ex2_approx(m_run - m_new);
          m_run = m_new;
        }
        // P = 2^(s*scale*log2e - m), two elements per packed FMA.  Two row sums, in
        // packed adds: of the fp32 P (for lse) and of the bf16-rounded P the PV MMA
        // consumes (normalises O, keeping it a convex combination of V rows: exact when
        // one key dominates a row).
        const uint64_t scale2 = f2_pack(prm.scale_log2, prm.scale_log2);
        // a row with no visible key so far keeps m = -inf; it subtracts 0 instead (its
        // P is exactly 0 either way)
        const float m_sub = (KR && m_run == -INFINITY) ? 0.f : m_run;
        const uint64_t negm2 = f2_pack(-m_sub, -m_sub);
        uint64_t lsum2[2] = {f2_pack(0.f, 0.f), f2_pack(0.f, 0.f)};
        uint64_t rsum2[2] = {f2_pack(0.f, 0.f), f2_pack(0.f, 0.f)};
        uint32_t pk[BK / 32][16];
#pragma unroll
        for (int c = 0; c < BK / 32; ++c) {
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const uint64_t x2 = f2_fma(f2_pack(__uint_as_float(sr[c][2 * e]), __uint_as_float(sr[c][2 * e + 1])),
                                       scale2, negm2);
            float x0, x1;
            f2_unpack(x2, x0, x1);
            const float p0 = ex2_approx(x0);
            const float p1 = ex2_approx(x1);
            lsum2[e & 1] = f2_add(lsum2[e & 1], f2_pack(p0, p1));
            pk[c][e] = pack_bf16x2(p0, p1);
            rsum2[e & 1] = f2_add(rsum2[e & 1], bf16x2_widen(pk[c][e]));
          }
        }
        // P_s and O_s are free once PV_s(n-1) has completed
        if (n > 0) {
          ok = warp_wait(&bars.pv_done[s], (pv_base + uint32_t(n) - 1) & 1, wctx);
          if (!ok) break;
          tc_fence_after();
        }
        if (__any_sync(0xffffffffu, grow && n > 0)) {
          l_run *= alpha;
          r_run *= alpha;
#pragma unroll 1
          for (int c = 0; c < HD / 32; ++c) {
            uint32_t orow[32];
            tmem_ld32(tO + c * 32, orow);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 32; ++e) orow[e] = __float_as_uint(__uint_as_float(orow[e]) * alpha);
            tmem_st32(tO + c * 32, orow);
          }
        }
#pragma unroll
        for (int c = 0; c < BK / 32; ++c) tmem_st16(tP + c * 16, pk[c]);
        float a0, a1, b0, b1;
        f2_unpack(f2_add(lsum2[0], lsum2[1]), a0, a1);
        f2_unpack(f2_add(rsum2[0], rsum2[1]), b0, b1);
        l_run += a0 + a1;
        r_run += b0 + b1;
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars.p_full[s]);
      }
      if (!ok) break;
      pv_base += uint32_t(u.kend[s]);
      // ---- epilogue: O / l -> bf16, lse
      ok = warp_wait(&bars.o_full[s], o_ph, wctx);
      o_ph ^= 1;
      if (!ok) break;
      tc_fence_after();
      // a row that saw no key of the block (key-block launches only): O = 0, lse = -inf
      const float inv_l = (KR && r_run == 0.f) ? 0.f : 1.0f / r_run;
      const int64_t rb = int64_t(u.r - prm.shard_begin) * prm.B + u.b;   // local (shard, b)
      const int64_t grow = rb * twoC + j;                                 // shard-major row
      __nv_bfloat16* orow_g = prm.o + (grow * prm.Hq + u.head[s]) * HD;
#pragma unroll 1
      for (int c = 0; c < HD / 32; ++c) {
        uint32_t orow[32];
        tmem_ld32(tO + c * 32, orow);
        tmem_ld_wait();
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e)
          pk[e] = pack_bf16x2(__uint_as_float(orow[2 * e]) * inv_l,
                              __uint_as_float(orow[2 * e + 1]) * inv_l);
        uint4* dst = reinterpret_cast<uint4*>(orow_g + c * 32);
#pragma unroll
        for (int v4 = 0; v4 < 4; ++v4)
          dst[v4] = make_uint4(pk[4 * v4], pk[4 * v4 + 1], pk[4 * v4 + 2], pk[4 * v4 + 3]);
      }
      prm.lse[(rb * prm.Hq + u.head[s]) * twoC + j] =
          (KR && l_run == 0.f) ? -INFINITY : (m_run + log2f(l_run)) * 0.69314718055994530942f;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.o_empty[s]);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == Cfg::WARP_MMA) tmem_dealloc(tmem, Cfg::TM_COLS);
}

template <int HD, bool KR>
int launch_fwd_hd(const FwdArgs& a, cudaStream_t stream) {
  using Cfg = FwdCfg<HD>;
  const int64_t rows = int64_t(a.shard_count) * a.B * (a.S / a.D);  // local shard-major rows
  const int32_t kv_box = KR || (a.S / (2 * int64_t(a.D))) % Cfg::BK == 0 ? Cfg::BK : 64;
  const uint64_t kv_rows = KR ? uint64_t(a.kv_rows) : uint64_t(a.B * a.S);
  CUtensorMap mq, mk, mv;
  {
    const uint64_t dims[3] = {uint64_t(HD), uint64_t(a.Hq), uint64_t(rows)};
    const uint64_t strides[2] = {uint64_t(HD) * 2, uint64_t(a.Hq) * HD * 2};
    const uint32_t box[3] = {64, 1, 128};
    if (!make_map_bf16_sw128(&mq, a.q, 3, dims, strides, box)) return int(cudaErrorInvalidValue);
  }
  {
    const uint64_t dims[3] = {uint64_t(HD), uint64_t(a.Hkv), kv_rows};
    const uint64_t strides[2] = {uint64_t(HD) * 2, uint64_t(a.Hkv) * HD * 2};
    // a box never straddles a zigzag chunk: the K/V rows it covers are contiguous in
    // both layouts
    const uint32_t box[3] = {64, 1, uint32_t(kv_box)};
    if (!make_map_bf16_sw128(&mk, a.k, 3, dims, strides, box)) return int(cudaErrorInvalidValue);
    if (!make_map_bf16_sw128(&mv, a.v, 3, dims, strides, box)) return int(cudaErrorInvalidValue);
  }
  FwdParams p;
  p.units = a.units;
  p.n_units = a.n_units;
  p.o = reinterpret_cast<__nv_bfloat16*>(a.o);
  p.lse = a.lse;
  p.S = a.S;
  p.C = a.S / (2 * int64_t(a.D));
  p.B = a.B; p.Hq = a.Hq; p.Hkv = a.Hkv; p.D = a.D; p.causal = a.causal;
  p.shard_begin = a.shard_begin;
  if (KR) {
    p.kb_rpb = a.kv_rows_per_batch;
    p.kb_off = a.kv_row_offset;
  } else {
    p.kv_shard_major = a.kv_layout;
    p.kv_box = kv_box;
  }
  p.scale_log2 = float(double(a.scale) * 1.4426950408889634);
  p.status = a.status;
  p.counter = a.status + 32;
  p.wait_limit_ns = a.wait_limit_ns;
  p.inject_stall = a.inject_stall;
  p.key_lo = a.key_lo;
  p.key_hi = a.key_hi;
  const int smem = Cfg::SMEM_BYTES + 1024;
  {
    const int e = ensure_smem_attr(reinterpret_cast<const void*>(zsa_fwd_kernel<HD, KR>), smem);
    if (e != int(cudaSuccess)) return e;
  }
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int grid = a.n_units < sms ? a.n_units : sms;
  if (grid <= 0) return int(cudaSuccess);
  const TraceEvents tr = trace_events(0);
  if (tr.begin) cudaEventRecord(tr.begin, stream);
  zsa_fwd_kernel<HD, KR><<<grid, Cfg::NTHREADS, smem, stream>>>(mq, mk, mv, p);
  const cudaError_t e = cudaGetLastError();
  if (tr.end) cudaEventRecord(tr.end, stream);
  return int(e);
}

}  // namespace

int launch_fwd(const FwdArgs& a, cudaStream_t stream) {
  switch (a.d) {
    case 64: return a.key_block ? launch_fwd_hd<64, true>(a, stream) : launch_fwd_hd<64, false>(a, stream);
    case 128: return a.key_block ? launch_fwd_hd<128, true>(a, stream) : launch_fwd_hd<128, false>(a, stream);
    case 256: return a.key_block ? launch_fwd_hd<256, true>(a, stream) : launch_fwd_hd<256, false>(a, stream);
    default: return int(cudaErrorInvalidValue);
  }
}

}  // namespace zsa
