// zsa_bwd_pair.cu -- backward main kernel (K3) for head dim 256, on clusters of two CTAs.
//
// At d = 256 the fp32 dK and dV of a 128-key tile fill 512 TMEM columns, all of one
// SM's TMEM.  This kernel splits the work of a key tile (b, kv head g, tile n) between
// the two CTAs of a cluster by role, so that no product is computed twice:
//
//   CTA 0 ("K side"): K tile resident, Q slots streamed; S^T = K Q^T, P^T = exp(scale S^T
//     - lse) -> sent to CTA 1; dK += dS^T Q, dQ^T = K^T dS^T (two 128-row d halves).
//     TMEM: dK (256) | ST x2 (64 each) | XT (dQ^T, 2 x 64).
//   CTA 1 ("V side"): V tile resident, dO slots streamed; dP^T = V dO^T; on receiving
//     P^T, dS^T = P^T (dP^T - Delta) -> sent to CTA 0; dV += P^T dO.
//     TMEM: dV (256) | DT x2 (64 each).
//
// q slots are 64 rows: with K (or V) resident (64 KB) that leaves room for a 3-stage
// Q (dO) ring, double-buffered exchange buffers and a dedicated dQ staging buffer, so
// the next slots' loads, products and exchanges overlap the current slot's.  S^T, dP^T
// and dQ^T are N = 64 MMAs; dK and dV are N = 256.
//
// P^T and dS^T (bf16, 128 keys x 64 q rows, 16 KB) cross between the CTAs through
// distributed shared memory: the producing compute warps store them straight into the
// peer's buffer (st.shared::cluster, already in the 128B-swizzled K-major layout the
// peer's MMA reads), gather on a local barrier, and one thread arrives on the peer's
// barrier with a cluster-scope release; the consuming MMA thread fences the async proxy
// after its acquire.  A buffer goes back to its writer
// once the peer's MMA has read it (tcgen05.commit multicast to the writer's CTA) and, on
// CTA 1, once its compute warps have read P^T.
//
// dQ^T (fp32) leaves through TMEM -> the staging buffer -> one TMA bulk reduce-add per
// warp and half into the head-major accumulator.
//
// Units (key tiles) are claimed dynamically by CTA 0's producer and handed to both CTAs
// through a unit ring whose slots every consumer of both CTAs releases.  Every wait is
// bounded (WaitCtx); a CTA that gives up raises its abort flag, and its peer's waits on
// it then run out their own limit.
#include <cuda_bf16.h>

#include "zsa_bwd_common.cuh"
#include "zsa_kernels.h"
#include "zsa_ptx.cuh"
#include "zsa_tma_host.h"

namespace zsa {
namespace {
using namespace bwd;

struct PairCfg {
  static constexpr int HD = 256;
  static constexpr int BKV = 128;                   // keys per tile (TMEM lanes)
  static constexpr int BQ = 64;                     // q rows per slot
  static constexpr int KB = HD / 64;                // 64-wide d blocks
  static constexpr int NST = 3;                     // Q / dO stages
  static constexpr int TILE_BYTES = BKV * HD * 2;   // K or V tile: 64 KB, [4 d blocks][128 keys][128 B]
  static constexpr int SLOT_BYTES = BQ * HD * 2;    // Q or dO slot: 32 KB, [4 d blocks][64 q][128 B]
  static constexpr int X_BYTES = BKV * BQ * 2;      // P^T or dS^T: 16 KB, [128 keys][64 q]
  static constexpr int STG_BYTES = 128 * BQ * 4;    // one dQ^T half: [4 warps][64 q][32 d] fp32
  static constexpr int SMEM_T = 0;                          // K (CTA 0) or V (CTA 1)
  static constexpr int SMEM_S = SMEM_T + TILE_BYTES;        // Q (CTA 0) or dO (CTA 1) stages
  static constexpr int SMEM_X = SMEM_S + NST * SLOT_BYTES;  // received: dS^T (CTA 0) / P^T (CTA 1), x2
  static constexpr int SMEM_STG = SMEM_X + 2 * X_BYTES;     // dQ^T staging (CTA 0)
  static constexpr int SMEM_STAT = SMEM_STG + STG_BYTES;    // NST x 64 fp32: lse or Delta
  static constexpr int SMEM_BYTES = SMEM_STAT + NST * BQ * 4;
  static constexpr int WARP_DQ = 8;      // warps 8..11 (CTA 0)
  static constexpr int WARP_LOAD = 12;
  static constexpr int WARP_MMA = 13;    // CTA 0: S^T;  CTA 1: dP^T  (and TMEM owner)
  static constexpr int WARP_MMA2 = 14;   // CTA 0: dK, dQ^T;  CTA 1: dV
  static constexpr int NTHREADS = 15 * 32;
  static constexpr uint32_t TM_ACC = 0;      // dK (CTA 0) / dV (CTA 1): 256 columns
  static constexpr uint32_t TM_ST = 256;     // S^T / dP^T, two buffers of BQ columns
  static constexpr uint32_t TM_XT = 384;     // dQ^T: d half h at TM_XT + h * BQ (CTA 0)
  static constexpr uint32_t TM_COLS = 512;
  static_assert(SMEM_BYTES <= 227 * 1024 - 1024, "shared memory budget");
  static_assert(TM_XT + 2 * BQ <= TM_COLS, "TMEM budget");
};

// The same barrier struct sits at the same offset in both CTAs, so a barrier of the peer
// is addressed by mapping the local one (mapa) or by a multicast commit.
struct PairBars {
  uint64_t unit_full[kUnitRing], unit_empty[kUnitRing];  // unit_empty used in CTA 0 only
  uint64_t t_full, t_empty;                       // K / V tile
  uint64_t s_full[PairCfg::NST], s_empty[PairCfg::NST];   // Q / dO (+ lse / Delta) stages
  uint64_t mm_full[2], mm_free[2];   // S^T (CTA 0) / dP^T (CTA 1) buffers in TMEM
  uint64_t x_full[2];                // the peer's P^T (CTA 1) / dS^T (CTA 0) has arrived
  uint64_t x_free[2];                // CTA 0: CTA 1 is done with P^T;  CTA 1: CTA 0 with dS^T
  uint64_t x_sent[2];                // local: all 8 compute warps have stored their rows
  uint64_t x_read[2];                // local (CTA 1): all 8 compute warps have read P^T
  uint64_t dq_full[2], dq_empty[2];  // dQ^T half h in XT (CTA 0), per half
  uint64_t acc_full, acc_empty;      // dK / dV accumulators
  uint64_t drain, never;
};

// Units claimed by the producer of CTA 0 and consumed by both CTAs' roles:
//   CTA 0: two MMA threads + 8 compute warps + 4 dQ warps;  CTA 1: producer + two MMA
//   threads + 8 compute warps.  All of them release a ring slot on CTA 0's unit_empty.
constexpr uint32_t kUnitConsumers = (2 + 8 + 4) + (1 + 2 + 8);

__device__ __forceinline__ uint32_t peer_addr(const void* p, uint32_t peer) {
  return mapa_shared(smem_u32(p), peer);
}

// Read the claimed unit of ring slot `slot` and release the slot on CTA 0.
__device__ __forceinline__ int take_unit(PairBars& bars, int* unit_ring, int slot, uint32_t rank) {
  const int idx = *reinterpret_cast<volatile int*>(&unit_ring[slot]);
  if (rank == 0) mbar_arrive(&bars.unit_empty[slot]);
  else mbar_arrive_cluster(peer_addr(&bars.unit_empty[slot], 0));
  return idx;
}

__global__ void __launch_bounds__(PairCfg::NTHREADS, 1)
    zsa_bwd_pair_kernel(const __grid_constant__ CUtensorMap map_q,
                        const __grid_constant__ CUtensorMap map_k,
                        const __grid_constant__ CUtensorMap map_v,
                        const __grid_constant__ CUtensorMap map_do,
                        const __grid_constant__ CUtensorMap map_dq, const BwdParams prm) {
  using Cfg = PairCfg;
  constexpr int KB = Cfg::KB, BQ = Cfg::BQ, BKV = Cfg::BKV, NST = Cfg::NST;
  extern __shared__ __align__(1024) uint8_t smem[];
  __shared__ PairBars bars;
  __shared__ uint32_t tmem_base_s;
  __shared__ int abort_s;
  __shared__ int unit_ring[kUnitRing];

  const uint32_t rank = cluster_ctarank();
  const uint32_t peer = rank ^ 1u;
  const int warp = int(warp_id()), lane = int(lane_id());
  if (smem_u32(smem) & 1023u) {       // never expected (both CTAs share the layout)
    if (threadIdx.x == 0) atomicOr(prm.status, kDevTimeout);
    return;
  }
  if (threadIdx.x == 0) {
    abort_s = 0;
    for (int s = 0; s < kUnitRing; ++s) {
      mbar_init(&bars.unit_full[s], 1);
      mbar_init(&bars.unit_empty[s], kUnitConsumers);
    }
    mbar_init(&bars.t_full, 1);
    mbar_init(&bars.t_empty, 1);
    for (int s = 0; s < NST; ++s) {
      mbar_init(&bars.s_full[s], 1);
      // 8 compute warps (lse / Delta read) + the commit after the last MMA reading the
      // stage (dK on CTA 0, dV on CTA 1)
      mbar_init(&bars.s_empty[s], 8 + 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bars.mm_full[b], 1);
      mbar_init(&bars.mm_free[b], 8);
      // one cluster-scope arrival per slot and direction: the peer's 8 compute warps
      // gather on its local x_sent / x_read first, and one thread forwards them
      mbar_init(&bars.x_full[b], 1);
      mbar_init(&bars.x_free[b], rank == 0 ? 1 + 1 : 1);   // CTA 1: dV commit + compute warps
      mbar_init(&bars.x_sent[b], 8);
      mbar_init(&bars.x_read[b], 8);
    }
    for (int h = 0; h < 2; ++h) {
      mbar_init(&bars.dq_full[h], 1);
      mbar_init(&bars.dq_empty[h], 4);
    }
    mbar_init(&bars.acc_full, 1);
    mbar_init(&bars.acc_empty, 8);
    mbar_init(&bars.drain, 2);
    mbar_init(&bars.never, 1);
    fence_mbar_init();
  }
  if (warp == Cfg::WARP_MMA) {
    tmem_alloc(&tmem_base_s, Cfg::TM_COLS);
    tmem_relinquish();
  }
  if (warp == Cfg::WARP_LOAD && lane == 0) {
    tma_prefetch_desc(rank == 0 ? &map_k : &map_v);
    tma_prefetch_desc(rank == 0 ? &map_q : &map_do);
    if (rank == 0) tma_prefetch_desc(&map_dq);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  cluster_sync();                      // the peer's barriers are initialised
  const uint32_t tmem = tmem_base_s;
  const WaitCtx wctx{&abort_s, prm.status, prm.wait_limit_ns};
  const int64_t twoC = 2 * prm.C;
  const uint32_t sT = smem_u32(smem + Cfg::SMEM_T);
  const uint32_t sS = smem_u32(smem + Cfg::SMEM_S);
  const uint32_t sX = smem_u32(smem + Cfg::SMEM_X);

  if (warp == Cfg::WARP_LOAD) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      uint32_t s_it = 0, t_fills = 0;
      uint32_t s_fills[NST];
      for (int s = 0; s < NST; ++s) s_fills[s] = 0;
      bool ok = true;
      for (int k = 0; ok; ++k) {
        const int slot = k % kUnitRing;
        int idx;
        if (rank == 0) {
          // claim the next key tile and hand it to both CTAs
          if (k >= kUnitRing)
            ok = mbar_wait_cluster(&bars.unit_empty[slot], ((k / kUnitRing) - 1) & 1, wctx);
          if (!ok) break;
          idx = atomicAdd(prm.counter, 1);
          if (idx >= prm.n_units) idx = -1;
          unit_ring[slot] = idx;
          st_cluster_b32(peer_addr(&unit_ring[slot], peer), uint32_t(idx));
          mbar_arrive(&bars.unit_full[slot]);
          mbar_arrive_cluster(peer_addr(&bars.unit_full[slot], peer));
        } else {
          ok = mbar_wait_cluster(&bars.unit_full[slot], (k / kUnitRing) & 1, wctx);
          if (!ok) break;
          idx = take_unit(bars, unit_ring, slot, rank);
        }
        if (idx < 0) break;
        const KvUnit u = decode_kv_unit(idx, prm.Hkv, prm.n_ktiles);
        // the unit's K (CTA 0) or V (CTA 1) tile
        if (t_fills > 0) ok = mbar_wait(&bars.t_empty, (t_fills - 1) & 1, wctx);
        if (!ok) break;
        mbar_expect_tx(&bars.t_full, Cfg::TILE_BYTES);
        for (int hb = 0; hb < BKV / prm.kv_box; ++hb) {
          const int32_t krow = kv_tensor_row(u.n * BKV + hb * prm.kv_box, u.b, int32_t(prm.S),
                                             int32_t(prm.C), prm.B, prm.D, prm.kv_shard_major);
          for (int kb = 0; kb < KB; ++kb)
            tma_load_3d(smem + Cfg::SMEM_T + kb * BKV * 128 + hb * prm.kv_box * 128,
                        rank == 0 ? &map_k : &map_v, &bars.t_full, kb * 64, u.g, krow);
        }
        ++t_fills;
        // the q slots: Q + lse (CTA 0) or dO + Delta (CTA 1)
        SlotWalk w;
        for (bool more = walk_first(prm, u.n, w); more && ok; more = walk_next(prm, u.n, w)) {
          const int st = int(s_it % NST);
          const uint32_t use = s_it / NST;
          if (use > 0) ok = mbar_wait(&bars.s_empty[st], (use - 1) & 1, wctx);
          if (!ok) break;
          const int32_t h = u.g * prm.G + w.e;
          const int64_t rb = int64_t(w.r - prm.shard_begin) * prm.B + u.b;
          const int32_t row0 = int32_t(rb * twoC + int64_t(w.i) * BQ);
          mbar_expect_tx(&bars.s_full[st], Cfg::SLOT_BYTES + BQ * 4);
          for (int kb = 0; kb < KB; ++kb)
            tma_load_3d(smem + Cfg::SMEM_S + st * Cfg::SLOT_BYTES + kb * BQ * 128,
                        rank == 0 ? &map_q : &map_do, &bars.s_full[st], kb * 64, h, row0);
          const int64_t stat = (rb * prm.Hq + h) * twoC + int64_t(w.i) * BQ;
          bulk_load(smem + Cfg::SMEM_STAT + st * BQ * 4, (rank == 0 ? prm.nlse2 : prm.ndelta) + stat,
                    BQ * 4, &bars.s_full[st]);
          ++s_fills[st];
          ++s_it;
        }
      }
      if (!ok) {
        const uint64_t lim = 1000000000ull;
        if (t_fills > 0) mbar_drain(&bars.t_full, (t_fills - 1) & 1, lim);
        for (int s = 0; s < NST; ++s)
          if (s_fills[s] > 0) mbar_drain(&bars.s_full[s], (s_fills[s] - 1) & 1, lim);
      }
    }
  } else if (warp == Cfg::WARP_MMA || warp == Cfg::WARP_MMA2) {
    // ------------------------------------------------------------ MMA issuers
    //  thread A (WARP_MMA): S^T = K Q^T (CTA 0) or dP^T = V dO^T (CTA 1) into ST buffer
    //    j % 2, as soon as the slot's stage is loaded and the compute warps have read
    //    slot j-2's product out of that buffer;
    //  thread B (WARP_MMA2): CTA 0: dK += dS^T Q, then both 128-row halves of
    //    dQ^T = K^T dS^T into XT;  CTA 1: dV += P^T dO.  Both read the operand the peer
    //    stored into this CTA's exchange buffer j % 2, and hand it back to the peer with a
    //    multicast commit.
    if (lane == 0) {
      const bool role_a = warp == Cfg::WARP_MMA;
      const uint32_t idesc_s = idesc_bf16(128, BQ, false, false);      // S^T, dP^T
      const uint32_t idesc_acc = idesc_bf16(128, 256, false, true);    // dK, dV (N = d = 256)
      const uint32_t idesc_dq = idesc_bf16(128, BQ, true, true);       // dQ^T half
      uint32_t t_ph = 0, q_it = 0;
      uint32_t s_uses[NST];
      for (int s = 0; s < NST; ++s) s_uses[s] = 0;
      uint32_t dq_commits = 0, acc_commits = 0;
      bool ok = true;
      if (prm.inject_stall) ok = mbar_wait(&bars.never, 0, wctx);
      for (int k = 0; ok; ++k) {
        const int slot = k % kUnitRing;
        ok = mbar_wait_cluster(&bars.unit_full[slot], (k / kUnitRing) & 1, wctx);
        if (!ok) break;
        const int idx = take_unit(bars, unit_ring, slot, rank);
        if (idx < 0) break;
        const KvUnit u = decode_kv_unit(idx, prm.Hkv, prm.n_ktiles);
        if (role_a) {
          ok = mbar_wait(&bars.t_full, t_ph, wctx);
          t_ph ^= 1;
          if (!ok) break;
        }
        SlotWalk w;
        for (bool more = walk_first(prm, u.n, w), j0 = true; more && ok;
             more = walk_next(prm, u.n, w), j0 = false) {
          const int st = int(q_it % NST);
          const int xb = int(q_it & 1);                 // ST / exchange buffer of this slot
          const uint32_t sSt = sS + uint32_t(st * Cfg::SLOT_BYTES);
          const uint32_t sXb = sX + uint32_t(xb * Cfg::X_BYTES);
          if (role_a) {
            ok = mbar_wait(&bars.s_full[st], s_uses[st] & 1, wctx);
            ++s_uses[st];
            if (ok && q_it >= 2) ok = mbar_wait(&bars.mm_free[xb], ((q_it >> 1) - 1) & 1, wctx);
            if (!ok) break;
            tc_fence_after();
            for (int kb = 0; kb < KB; ++kb)
#pragma unroll
              for (int ks = 0; ks < 4; ++ks)
                mma_ss(tmem + Cfg::TM_ST + uint32_t(xb * BQ),
                       sdesc_sw128(sT + kb * BKV * 128 + ks * 32, 16, 1024),
                       sdesc_sw128(sSt + kb * BQ * 128 + ks * 32, 16, 1024), idesc_s, (kb | ks) != 0);
            mma_commit(&bars.mm_full[xb]);
          } else {
            // the peer's operand for this slot: dS^T (CTA 0) or P^T (CTA 1)
            ok = mbar_wait_cluster(&bars.x_full[xb], (q_it >> 1) & 1, wctx);
            // The peer's stores are performed before its cluster-scope release, which this
            // acquire observed; the proxy fence then orders them (as seen by this thread)
            // before the tensor core's reads of the buffer.  One fence per slot here
            // replaces one per storing thread on the peer (measured: +11% on this kernel).
            fence_proxy_async_cluster();
            if (ok && j0 && acc_commits > 0)
              ok = mbar_wait(&bars.acc_empty, (acc_commits - 1) & 1, wctx);
            if (!ok) break;
            tc_fence_after();
            // dK += dS^T Q  /  dV += P^T dO: A = the exchange buffer (K-major, one 64-q
            // block), B = the stage (MN-major, N = 256 over four 64-wide d blocks)
#pragma unroll
            for (int ks = 0; ks < BQ / 16; ++ks)
              mma_ss(tmem + Cfg::TM_ACC, sdesc_sw128(sXb + ks * 32, 16, 1024),
                     sdesc_sw128(sSt + ks * 2048, BQ * 128, 1024), idesc_acc, !j0 || (ks > 0));
            mma_commit(&bars.s_empty[st]);              // the stage's last MMA reader
            if (rank == 0) {
              // dQ^T rows 128hh .. 128hh+127: A = K^T (MN-major, d blocks 2hh, 2hh+1),
              // B = dS^T (MN-major: the 64 q of each key row), K = the 128 keys.  Each
              // half has its own TMEM columns and hand-off, so half 0 of this slot only
              // waits for half 0 of the previous one to be read out.
              for (int hh = 0; hh < 2 && ok; ++hh) {
                if (dq_commits > 0) {
                  ok = mbar_wait(&bars.dq_empty[hh], (dq_commits - 1) & 1, wctx);
                  if (!ok) break;
                  tc_fence_after();
                }
#pragma unroll
                for (int ks = 0; ks < BKV / 16; ++ks)
                  mma_ss(tmem + Cfg::TM_XT + uint32_t(hh * BQ),
                         sdesc_sw128(sT + (2 * hh) * (BKV * 128) + ks * 2048, BKV * 128, 1024),
                         sdesc_sw128(sXb + ks * 2048, BKV * 128, 1024), idesc_dq, ks > 0);
                mma_commit(&bars.dq_full[hh]);
              }
              if (!ok) break;
              ++dq_commits;
            }
            mma_commit_multicast(&bars.x_free[xb], uint16_t(1u << peer));   // buffer back
          }
          ++q_it;
        }
        if (!ok) break;
        if (role_a) {
          if (rank == 1) mma_commit(&bars.t_empty);      // V is read by dP^T only
        } else {
          mma_commit(&bars.acc_full);
          ++acc_commits;
          if (rank == 0) mma_commit(&bars.t_empty);      // K: last read by this unit's dQ^T
        }
      }
      mma_commit(&bars.drain);
      mbar_drain(&bars.drain, 0, 1000000000ull);
    }
    __syncwarp();
  } else if (warp >= Cfg::WARP_DQ) {
    // ------------------------------------------------------------ dQ warps (CTA 0)
    // Each dQ^T half of a slot (TMEM lane = d within the half, column = q row) is staged
    // as [32 q][32 d] fp32 boxes (128-byte rows, 128-byte swizzle) in a ring of two per
    // warp in the staging buffer, each reduced into the accumulator by one TMA bulk
    // reduce-add: a box is rewritten once the reduce issued two boxes earlier has read
    // it, so staging overlaps the reduces instead of waiting for each to drain.
    if (rank == 0) {
      const int qw = warp - Cfg::WARP_DQ;
      const uint32_t tXT = tmem + Cfg::TM_XT + (uint32_t(qw * 32) << 16);
      uint8_t* box = smem + Cfg::SMEM_STG + qw * (BQ * 128);
      uint32_t dq_ph = 0;
      bool ok = true;
      for (int k = 0; ok; ++k) {
        const int slot = k % kUnitRing;
        ok = warp_wait_b(&bars.unit_full[slot], (k / kUnitRing) & 1, wctx);
        if (!ok) break;
        const int idx = *reinterpret_cast<volatile int*>(&unit_ring[slot]);
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars.unit_empty[slot]);
        if (idx < 0) break;
        const KvUnit u = decode_kv_unit(idx, prm.Hkv, prm.n_ktiles);
        SlotWalk w;
        for (bool more = walk_first(prm, u.n, w); more && ok; more = walk_next(prm, u.n, w)) {
          const int32_t h = u.g * prm.G + w.e;
          const int32_t row0 =
              int32_t((int64_t(w.r - prm.shard_begin) * prm.B + u.b) * twoC + int64_t(w.i) * BQ);
          for (int hh = 0; hh < 2; ++hh) {
            ok = warp_wait_b(&bars.dq_full[hh], dq_ph, wctx);
            if (!ok) break;
            tc_fence_after();
            uint32_t v[2][32];
            tmem_ld32(tXT + uint32_t(hh * BQ), v[0]);
            tmem_ld32(tXT + uint32_t(hh * BQ + 32), v[1]);
            tmem_ld_wait();
            tc_fence_before();                 // the half is in registers: its columns
            __syncwarp();                      // may take the next slot's half
            if (lane == 0) mbar_arrive(&bars.dq_empty[hh]);
            const uint32_t within = uint32_t(lane & 3) * 4;
#pragma unroll
            for (int t = 0; t < 2; ++t) {
              // [32 q][32 d] boxes in a ring of two per warp: the box written now was last
              // used two reduces ago, which must have read it (at most one in flight)
              uint8_t* bx = box + ((hh * 2 + t) & 1) * (32 * 128);
              if (lane == 0) bulk_wait_group_read1();
              __syncwarp();
#pragma unroll
              for (int c = 0; c < 32; ++c)
                *reinterpret_cast<uint32_t*>(bx + sw128_offset(uint32_t(c), uint32_t(lane >> 2)) + within) =
                    v[t][c];
              fence_proxy_async_smem();
              __syncwarp();
              if (lane == 0) {
                tma_reduce_add_3d(&map_dq, bx, hh * 128 + qw * 32, row0 + t * 32, h);
                bulk_commit_group();
              }
            }
          }
          dq_ph ^= 1;
        }
      }
      if (lane == 0) bulk_wait_group0();
      __syncwarp();
    }
  } else {
    // ------------------------------------------------------------ compute warps
    // group hg = warp / 4 handles q rows 32hg .. 32hg+31 of each 64-row slot (contiguous
    // positions: a 64-row slot lies inside one zigzag chunk); thread = key row.
    //  CTA 0: P^T = exp(scale S^T - lse) (masked) -> the peer's P^T buffer.
    //  CTA 1: dS^T = P^T (dP^T - Delta) -> the peer's dS^T buffer.
    const int hg = warp / 4;
    const int qw = warp % 4;
    const int row = qw * 32 + lane;
    const uint32_t lane_addr = uint32_t(qw * 32) << 16;
    const float* stat = reinterpret_cast<const float*>(smem + Cfg::SMEM_STAT);
    uint32_t q_it = 0, acc_ph = 0;
    uint32_t s_uses[NST];
    for (int s = 0; s < NST; ++s) s_uses[s] = 0;
    bool ok = true;
    for (int k = 0; ok; ++k) {
      const int slot = k % kUnitRing;
      ok = __all_sync(0xffffffffu, mbar_wait_cluster(&bars.unit_full[slot], (k / kUnitRing) & 1, wctx));
      if (!ok) break;
      const int idx = *reinterpret_cast<volatile int*>(&unit_ring[slot]);
      __syncwarp();
      if (lane == 0) {
        if (rank == 0) mbar_arrive(&bars.unit_empty[slot]);
        else mbar_arrive_cluster(peer_addr(&bars.unit_empty[slot], 0));
      }
      if (idx < 0) break;
      const KvUnit u = decode_kv_unit(idx, prm.Hkv, prm.n_ktiles);
      const int64_t key = int64_t(u.n) * BKV + row;
      int nslots = 0;
      SlotWalk w;
      for (bool more = walk_first(prm, u.n, w); more && ok; more = walk_next(prm, u.n, w)) {
        ++nslots;
        const int st = int(q_it % NST);
        const int xb = int(q_it & 1);
        const uint32_t ph = (q_it >> 1) & 1;              // phase of the slot's buffers
        ok = warp_wait_b(&bars.s_full[st], s_uses[st] & 1, wctx);
        ++s_uses[st];
        if (!ok) break;
        const float* stat_c = stat + st * BQ + 32 * hg;
        // ---- this slot's product (S^T or dP^T), 32 columns per thread
        ok = warp_wait_b(&bars.mm_full[xb], ph, wctx);
        if (!ok) break;
        tc_fence_after();
        uint32_t sv[32];
        tmem_ld32(tmem + Cfg::TM_ST + uint32_t(xb * BQ + 32 * hg) + lane_addr, sv);
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars.mm_free[xb]);    // the buffer may take slot j+2
        uint32_t pk[16];
        if (rank == 0) {
          // P^T: columns c < nvis_lo lie above the diagonal for this key
          const int64_t p0 = zz_pos(prm.C, prm.D, w.r, int64_t(w.i) * BQ + 32 * hg);
          const int nvis_lo = prm.causal ? int(key - p0) : 0;
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const int c0 = 2 * e;
            const float x0 = fmaf(__uint_as_float(sv[c0]), prm.scale_log2, stat_c[c0]);        // -lse log2 e
            const float x1 = fmaf(__uint_as_float(sv[c0 + 1]), prm.scale_log2, stat_c[c0 + 1]);
            pk[e] = pack_bf16x2(c0 < nvis_lo ? 0.f : ex2_approx(x0),
                                c0 + 1 < nvis_lo ? 0.f : ex2_approx(x1));
          }
        } else {
          // dS^T needs this slot's P^T from the peer
          ok = __all_sync(0xffffffffu, mbar_wait_cluster(&bars.x_full[xb], ph, wctx));
          if (!ok) break;
          const uint8_t* x_local = smem + Cfg::SMEM_X + xb * Cfg::X_BYTES;
          uint4 pv[4];
#pragma unroll
          for (int m = 0; m < 4; ++m)
            pv[m] = *reinterpret_cast<const uint4*>(x_local + sw128_offset(uint32_t(row), uint32_t(4 * hg + m)));
          __syncwarp();
          if (lane == 0) mbar_arrive(&bars.x_read[xb]);
          if (warp == 0 && lane == 0) {        // forward "P^T read" once all 8 warps have
            ok = mbar_wait(&bars.x_read[xb], ph, wctx);
            mbar_arrive_cluster(peer_addr(&bars.x_free[xb], peer));
          }
          ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
          if (!ok) break;
#pragma unroll
          for (int m = 0; m < 4; ++m) {
            const uint32_t pw[4] = {pv[m].x, pv[m].y, pv[m].z, pv[m].w};
#pragma unroll
            for (int t = 0; t < 4; ++t) {
              const int c0 = 8 * m + 2 * t;
              pk[4 * m + t] =
                  pack_bf16x2(__uint_as_float(pw[t] << 16) * (__uint_as_float(sv[c0]) + stat_c[c0]),   // -Delta
                              __uint_as_float(pw[t] & 0xFFFF0000u) * (__uint_as_float(sv[c0 + 1]) + stat_c[c0 + 1]));
            }
          }
        }
        // the peer's buffer must be done with slot j-2's operand
        if (q_it >= 2) {
          ok = __all_sync(0xffffffffu, mbar_wait_cluster(&bars.x_free[xb], ph ^ 1u, wctx));
          if (!ok) break;
        }
        const uint32_t x_peer = peer_addr(smem + Cfg::SMEM_X + xb * Cfg::X_BYTES, peer);
#pragma unroll
        for (int m = 0; m < 4; ++m)
          st_cluster_v4(x_peer + sw128_offset(uint32_t(row), uint32_t(4 * hg + m)),
                        make_uint4(pk[4 * m], pk[4 * m + 1], pk[4 * m + 2], pk[4 * m + 3]));
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&bars.x_sent[xb]);
          mbar_arrive(&bars.s_empty[st]);             // lse / Delta of the stage consumed
        }
        if (warp == 0 && lane == 0) {                 // forward "rows stored" once all 8
          ok = mbar_wait(&bars.x_sent[xb], ph, wctx); // warps have (their release is
          mbar_arrive_cluster(peer_addr(&bars.x_full[xb], peer));   // acquired here)
        }
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        if (!ok) break;
        ++q_it;
      }
      if (!ok) break;
      // ---- epilogue: dK (CTA 0) / dV (CTA 1) rows of this key tile; group hg writes d
      //      columns 128hg .. 128hg+127
      ok = warp_wait_b(&bars.acc_full, acc_ph, wctx);
      acc_ph ^= 1;
      if (!ok) break;
      tc_fence_after();
      const float mul = rank == 0 ? prm.scale : 1.0f;
      const int64_t krow = kv_tensor_row(int32_t(key), u.b, int32_t(prm.S), int32_t(prm.C), prm.B, prm.D,
                                           prm.kv_shard_major);
      __nv_bfloat16* dst = (rank == 0 ? prm.dk : prm.dv) + (krow * prm.Hkv + u.g) * Cfg::HD + 128 * hg;
      const bool empty = nslots == 0;   // no query of the launch's shards sees this tile
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        uint32_t a[32];
        if (!empty) {
          tmem_ld32(tmem + Cfg::TM_ACC + 128 * hg + c * 32 + lane_addr, a);
          tmem_ld_wait();
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) a[e] = 0u;
        }
        uint32_t o16[16];
#pragma unroll
        for (int e = 0; e < 16; ++e)
          o16[e] = pack_bf16x2(__uint_as_float(a[2 * e]) * mul, __uint_as_float(a[2 * e + 1]) * mul);
        uint4* d4 = reinterpret_cast<uint4*>(dst + c * 32);
#pragma unroll
        for (int v4 = 0; v4 < 4; ++v4)
          d4[v4] = make_uint4(o16[4 * v4], o16[4 * v4 + 1], o16[4 * v4 + 2], o16[4 * v4 + 3]);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.acc_empty);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  cluster_sync();            // the peer no longer stores into or arrives on this CTA
  if (warp == Cfg::WARP_MMA) tmem_dealloc(tmem, Cfg::TM_COLS);
}

}  // namespace

namespace bwd {
int launch_pair_main(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                     const CUtensorMap& mdo, const CUtensorMap& mdq, const BwdParams& p,
                     cudaStream_t stream) {
  const int smem = PairCfg::SMEM_BYTES;
  int e = ensure_smem_attr(reinterpret_cast<const void*>(zsa_bwd_pair_kernel), smem);
  if (e != int(cudaSuccess)) return e;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(PairCfg::NTHREADS);
  cfg.dynamicSmemBytes = size_t(smem);
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  cfg.gridDim = dim3(unsigned(sms & ~1));
  int max_clusters = 0;
  if (cudaOccupancyMaxActiveClusters(&max_clusters, zsa_bwd_pair_kernel, &cfg) != cudaSuccess ||
      max_clusters <= 0)
    max_clusters = sms / 2;
  const int clusters = p.n_units < max_clusters ? p.n_units : max_clusters;
  if (clusters <= 0) return int(cudaSuccess);
  cfg.gridDim = dim3(unsigned(2 * clusters));
  const TraceEvents tr = trace_events(2);
  if (tr.begin) cudaEventRecord(tr.begin, stream);
  cudaError_t err = cudaLaunchKernelEx(&cfg, zsa_bwd_pair_kernel, mq, mk, mv, mdo, mdq, p);
  if (err == cudaSuccess) err = cudaGetLastError();
  if (tr.end) cudaEventRecord(tr.end, stream);
  return int(err);
}
}  // namespace bwd

}  // namespace zsa
