// zsa_bwd.cu -- backward of zigzag-sharded causal GQA attention on sm_100a.
//
// The pages describe only the forward (all-gathered K/V + FlashAttention with a zigzag
// partition, "Folding Tensor and Sequence Parallelism" summary, section 2); the
// backward here is the exact gradient of <dO, O>, recomputing P from the saved lse:
//   Delta = rowsum(dO * O)                                            (K2, HBM-bound)
//   per key tile (b, kv head g, n), over every (shard, q tile, q head of g) that sees it:
//     S^T = K Q^T,  P^T = exp(scale S^T - lse),  dP^T = V dO^T,
//     dS^T = P^T * (dP^T - Delta),
//     dV += P^T dO,  dK += dS^T Q,  dQ (+)= dS K                       (K3, tensor-bound)
//   dQ = bf16(scale * dQacc)                                          (K4, HBM-bound)
// dK and dV are summed over every shard and the G q heads of the group inside one CTA
// (the single-GPU stand-in for the reduce-scatter back to the owning shards); dQ is
// summed across key tiles with fp32 reductions into a workspace accumulator.
//
// K3 has two builds, chosen by head dim.  Both claim 128-key-tile units (b, kv head, key
// tile) from a global counter in that order, keep the unit's K and V tiles in shared
// memory, stream the q slots that see the tile through a TMA ring (Q, dO, lse, Delta),
// send dQ through shared memory into TMA bulk reduce-adds, and bound every wait.
//
//  zsa_bwd_wide_kernel (d <= 128, this file): one CTA per key tile;
//   * 128-row q slots, so all five MMAs of a slot are N = 128; a 128-row slot may
//     straddle two zigzag chunks, so the 8 compute warps work in two groups of 64
//     rows, each over contiguous positions;
//   * TMEM: dV | dK (fp32, lanes = keys) | ST | XT.  ST receives S^T, then the bf16 P^T
//     and dS^T (TMEM A operands of dV and dK); XT receives dP^T and, once the compute
//     warps have read it, dQ = dS K (A = dS^T in shared memory read M-major, B = the
//     resident K tile read N-major), so a TMEM lane is a q row;
//   * two MMA-issuing threads: one issues S^T and dP^T, the other dV, dK and dQ;
//   * 4 dQ warps stage dQ, a q row per thread, in the slot's own Q / dO stage and
//     reduce it into the fp32 accumulator.
//
//  zsa_bwd_pair_kernel (d = 256, zsa_bwd_pair.cu): a cluster of two CTAs per key tile,
//  one holding K and dK, the other V and dV, exchanging P^T and dS^T through
//  distributed shared memory (dK + dV of the tile alone would fill one SM's TMEM); it
//  computes dQ transposed, dQ^T = K^T dS^T, in two 128-row d halves.
#include <cuda_bf16.h>

#include "zsa_bwd_common.cuh"
#include "zsa_kernels.h"
#include "zsa_ptx.cuh"
#include "zsa_tma_host.h"

namespace zsa {
namespace {
using namespace bwd;


// ------------------------------------------------------------------ K2: Delta + zero dQacc
// Per (row, head): -Delta = -rowsum(dO * O) and -lse * log2(e), the two per-row terms of
// the main kernel's element formulas stored ready to add (P^T = 2^(scale log2(e) S^T +
// (-lse log2 e)) is one FMA, dS^T = P^T (dP^T + (-Delta)) one add and one multiply), and
// the zeroed dQ accumulator.
// A warp takes 32 consecutive (row, head) pairs in the stats order (rb, h, j) -- the
// order of the fp32 [rows-block][Hq][2C] arrays -- so it reads 32 rows of O and dO (HD*2
// contiguous bytes each), writes each of the two stats arrays with one 128-byte store,
// and zeroes a contiguous 32*HD-float block of the accumulator (the pairs tile it, so any
// order zeroes all of it).  2C is a multiple of 128, so 32 consecutive pairs share (rb, h).
template <int HD>
__global__ void __launch_bounds__(256) zsa_bwd_pre_kernel(const __nv_bfloat16* __restrict__ o,
                                                          const __nv_bfloat16* __restrict__ dout,
                                                          const float* __restrict__ lse,
                                                          float* __restrict__ ndelta,
                                                          float* __restrict__ nlse2,
                                                          float* __restrict__ dq_acc,
                                                          int64_t n_pairs, int32_t Hq,
                                                          int64_t twoC) {
  constexpr int LPP = HD / 8;   // lanes per pair, 8 bf16 (16 B) per lane
  constexpr int PPI = 32 / LPP; // pairs per warp iteration
  const int lane = int(threadIdx.x & 31);
  const int sub = lane % LPP, grp = lane / LPP;
  const int64_t warp_global = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) / 32;
  const int64_t n_warps = int64_t(gridDim.x) * blockDim.x / 32;
  for (int64_t base = warp_global * 32; base < n_pairs; base += n_warps * 32) {
    const int64_t rbh = base / twoC;
    const int64_t j0 = base - rbh * twoC;
    const int64_t rb = rbh / Hq;
    const int64_t h = rbh - rb * Hq;
    float mine = 0.f;                         // lane l ends with pair base + l's rowsum
#pragma unroll 4
    for (int it = 0; it < 32 / PPI; ++it) {
      const int pi = it * PPI + grp;
      const int64_t el = ((rb * twoC + j0 + pi) * Hq + h) * HD;   // (row, h) in O's layout
      const uint4 a = reinterpret_cast<const uint4*>(o + el)[sub];
      const uint4 b = reinterpret_cast<const uint4*>(dout + el)[sub];
      const __nv_bfloat162* a2 = reinterpret_cast<const __nv_bfloat162*>(&a);
      const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&b);
      float acc = 0.f;
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const float2 x = __bfloat1622float2(a2[t]);
        const float2 y = __bfloat1622float2(b2[t]);
        acc = fmaf(x.x, y.x, acc);
        acc = fmaf(x.y, y.y, acc);
      }
#pragma unroll
      for (int off = LPP / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
      const float v = __shfl_sync(0xffffffffu, acc, (lane % PPI) * LPP);
      if (lane / PPI == it) mine = v;
      float4* z = reinterpret_cast<float4*>(dq_acc + (base + pi) * HD) + 2 * sub;
      z[0] = make_float4(0.f, 0.f, 0.f, 0.f);
      z[1] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    ndelta[base + lane] = -mine;
    nlse2[base + lane] = -lse[base + lane] * kLog2e;
  }
}

// ------------------------------------------------------------------ K4: dQ = bf16(scale*acc)
// The accumulator is head-major, [Hq][rows][d] (one q head's rows contiguous, so the
// reductions of a 128-row slot land in one 64 KB block instead of 128 lines 16 KB
// apart); dQ is [rows][Hq][d].  One block per row (grid-stride): each thread turns 8
// consecutive fp32 of one head into one 16-byte bf16 store.
template <int HD>
__global__ void __launch_bounds__(256) zsa_dq_convert_kernel(const float* __restrict__ acc,
                                                             __nv_bfloat16* __restrict__ dq,
                                                             int64_t rows, int32_t Hq, float scale) {
  constexpr int V8 = HD / 8;
  for (int64_t row = blockIdx.x; row < rows; row += gridDim.x) {
    for (int t = threadIdx.x; t < Hq * V8; t += blockDim.x) {
      const int h = t / V8, d8 = t % V8;
      const float4* src = reinterpret_cast<const float4*>(acc + (int64_t(h) * rows + row) * HD) + 2 * d8;
      const float4 a = src[0];
      const float4 b = src[1];
      uint4 r;
      r.x = pack_bf16x2(a.x * scale, a.y * scale);
      r.y = pack_bf16x2(a.z * scale, a.w * scale);
      r.z = pack_bf16x2(b.x * scale, b.y * scale);
      r.w = pack_bf16x2(b.z * scale, b.w * scale);
      reinterpret_cast<uint4*>(dq + row * int64_t(Hq) * HD)[t] = r;
    }
  }
}

// ------------------------------------------------------------------ K3 for d <= 128
// 128-row q slots, so every MMA of the slot is N = 128 (the tensor core loses most of
// its rate on N = 64 shapes whose operands all come from shared memory).  TMEM holds
// dV | dK | ST | XT: ST receives S^T and then the bf16 P^T and dS^T (half its columns
// each, A operands of dV and dK); XT receives dP^T and, once the compute warps have
// loaded it, dQ.  One slot is in flight; the next slot's S^T is issued as soon as
// dK has consumed ST, its dP^T as soon as the dQ warps have read XT.
template <int HD>
struct BwdWideCfg {
  static constexpr int BKV = 128;
  static constexpr int BQ = 128;
  static constexpr int KB = HD / 64;
  static constexpr int NQST = 2;
  static constexpr int KV_BYTES = BKV * HD * 2;
  static constexpr int QT_BYTES = BQ * HD * 2;
  static constexpr int DS_BYTES = BKV * BQ * 2;     // [2 q blocks][128 keys][64 q], 128B swizzle
  static constexpr int SMEM_K = 0;
  static constexpr int SMEM_V = SMEM_K + KV_BYTES;
  static constexpr int SMEM_Q = SMEM_V + KV_BYTES;
  static constexpr int SMEM_DO = SMEM_Q + NQST * QT_BYTES;
  static constexpr int SMEM_DS = SMEM_DO + NQST * QT_BYTES;
  static constexpr int SMEM_LSE = SMEM_DS + DS_BYTES;
  static constexpr int SMEM_DELTA = SMEM_LSE + NQST * BQ * 4;
  static constexpr int SMEM_BYTES = SMEM_DELTA + NQST * BQ * 4;
  static constexpr int WARP_DQ = 8;
  static constexpr int WARP_LOAD = 12;
  static constexpr int WARP_MMA = 13;   // S^T, dP^T issuer (and TMEM owner)
  static constexpr int WARP_MMA2 = 14;  // dV, dK, dQ issuer
  static constexpr int NTHREADS = 15 * 32;
  static constexpr uint32_t TM_DV = 0;
  static constexpr uint32_t TM_DK = HD;
  static constexpr uint32_t TM_ST = 2 * HD;
  static constexpr uint32_t TM_XT = 2 * HD + BQ;
  static constexpr uint32_t TM_COLS = 512;
  static_assert(2 * HD + 2 * BQ <= 512, "TMEM budget");
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
};

struct BwdWideBars {
  uint64_t kv_full, kv_empty;
  uint64_t q_full[2], q_empty[2];
  uint64_t s_full, p_full, dp_full, ds_full;
  uint64_t st_free, dsm_free, dq_full, dq_empty;
  uint64_t acc_full, acc_empty;
  uint64_t unit_full[kUnitRing], unit_empty[kUnitRing];
  uint64_t drain, never;
};

template <int HD>
__global__ void __launch_bounds__(BwdWideCfg<HD>::NTHREADS, 1)
    zsa_bwd_wide_kernel(const __grid_constant__ CUtensorMap map_q,
                        const __grid_constant__ CUtensorMap map_k,
                        const __grid_constant__ CUtensorMap map_v,
                        const __grid_constant__ CUtensorMap map_do,
                        const __grid_constant__ CUtensorMap map_dq, const BwdParams prm) {
  using Cfg = BwdWideCfg<HD>;
  constexpr int KB = Cfg::KB, BQ = Cfg::BQ, BKV = Cfg::BKV;
  // the 128B-swizzled operand tiles need a 1024-byte aligned base; the shared-memory
  // budget leaves no slack for aligning by hand, so the array itself is aligned
  extern __shared__ __align__(1024) uint8_t smem_w[];
  uint8_t* smem = smem_w;
  __shared__ BwdWideBars bars;
  __shared__ uint32_t tmem_base_s;
  __shared__ int abort_s;
  __shared__ int unit_ring[kUnitRing];

  const int warp = int(warp_id()), lane = int(lane_id());
  if (smem_u32(smem) & 1023u) {          // never expected; refuse rather than misread tiles
    if (threadIdx.x == 0) atomicOr(prm.status, kDevTimeout);
    return;
  }
  if (threadIdx.x == 0) {
    abort_s = 0;
    mbar_init(&bars.kv_full, 1);
    mbar_init(&bars.kv_empty, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars.q_full[s], 1);
      // 8 compute warps (lse / Delta read) + 4 dQ warps (their reduces have read the
      // dQ staged in this stage's Q / dO space, after every MMA of the slot)
      mbar_init(&bars.q_empty[s], 8 + 4);
    }
    mbar_init(&bars.s_full, 1);
    mbar_init(&bars.p_full, 8);
    mbar_init(&bars.dp_full, 1);
    mbar_init(&bars.ds_full, 8);
    mbar_init(&bars.st_free, 1);
    mbar_init(&bars.dsm_free, 1);
    mbar_init(&bars.dq_full, 1);
    mbar_init(&bars.dq_empty, 4);
    mbar_init(&bars.acc_full, 1);
    mbar_init(&bars.acc_empty, 8);
    for (int s = 0; s < kUnitRing; ++s) {
      mbar_init(&bars.unit_full[s], 1);
      mbar_init(&bars.unit_empty[s], 2 + 8 + 4);   // 2 MMA threads + compute + dQ warps
    }
    mbar_init(&bars.drain, 2);                     // one commit per MMA thread
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
    tma_prefetch_desc(&map_do);
    tma_prefetch_desc(&map_dq);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_s;
  const WaitCtx wctx{&abort_s, prm.status, prm.wait_limit_ns};
  const int64_t twoC = 2 * prm.C;

  if (warp == Cfg::WARP_LOAD) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      uint32_t q_it = 0, kv_fills = 0;
      uint32_t q_fills[2] = {0, 0};
      bool ok = true;
      for (int k = 0; ok; ++k) {
        const int slot = k % kUnitRing;
        if (k >= kUnitRing) ok = mbar_wait(&bars.unit_empty[slot], ((k / kUnitRing) - 1) & 1, wctx);
        if (!ok) break;
        int idx = atomicAdd(prm.counter, 1);
        if (idx >= prm.n_units) idx = -1;
        unit_ring[slot] = idx;
        mbar_arrive(&bars.unit_full[slot]);
        if (idx < 0) break;
        const KvUnit u = decode_kv_unit(idx, prm.Hkv, prm.n_ktiles);
        if (kv_fills > 0) ok = mbar_wait(&bars.kv_empty, (kv_fills - 1) & 1, wctx);
        if (!ok) break;
        mbar_expect_tx(&bars.kv_full, 2 * Cfg::KV_BYTES);
        for (int hb = 0; hb < BKV / prm.kv_box; ++hb) {
          const int32_t krow = kv_tensor_row(u.n * BKV + hb * prm.kv_box, u.b, int32_t(prm.S), int32_t(prm.C), prm.B, prm.D,
                                             prm.kv_shard_major);
          for (int kb = 0; kb < KB; ++kb) {
            tma_load_3d(smem + Cfg::SMEM_K + kb * BKV * 128 + hb * prm.kv_box * 128, &map_k, &bars.kv_full,
                        kb * 64, u.g, krow);
            tma_load_3d(smem + Cfg::SMEM_V + kb * BKV * 128 + hb * prm.kv_box * 128, &map_v, &bars.kv_full,
                        kb * 64, u.g, krow);
          }
        }
        ++kv_fills;
        SlotWalk w;
        for (bool more = walk_first(prm, u.n, w); more && ok; more = walk_next(prm, u.n, w)) {
          const int st = int(q_it & 1);
          const uint32_t use = q_it >> 1;
          if (use > 0) ok = mbar_wait(&bars.q_empty[st], (use - 1) & 1, wctx);
          if (!ok) break;
          const int32_t h = u.g * prm.G + w.e;
          const int64_t rb = int64_t(w.r - prm.shard_begin) * prm.B + u.b;   // local (shard, b)
          const int32_t row0 = int32_t(rb * twoC + int64_t(w.i) * BQ);
          mbar_expect_tx(&bars.q_full[st], 2 * Cfg::QT_BYTES + 2 * BQ * 4);
          for (int kb = 0; kb < KB; ++kb) {
            tma_load_3d(smem + Cfg::SMEM_Q + st * Cfg::QT_BYTES + kb * BQ * 128, &map_q,
                        &bars.q_full[st], kb * 64, h, row0);
            tma_load_3d(smem + Cfg::SMEM_DO + st * Cfg::QT_BYTES + kb * BQ * 128, &map_do,
                        &bars.q_full[st], kb * 64, h, row0);
          }
          const int64_t stat = (rb * prm.Hq + h) * twoC + int64_t(w.i) * BQ;
          bulk_load(smem + Cfg::SMEM_LSE + st * BQ * 4, prm.nlse2 + stat, BQ * 4, &bars.q_full[st]);
          bulk_load(smem + Cfg::SMEM_DELTA + st * BQ * 4, prm.ndelta + stat, BQ * 4, &bars.q_full[st]);
          ++q_fills[st];
          ++q_it;
        }
      }
      if (!ok) {
        const uint64_t lim = 1000000000ull;
        if (kv_fills > 0) mbar_drain(&bars.kv_full, (kv_fills - 1) & 1, lim);
        for (int s = 0; s < 2; ++s)
          if (q_fills[s] > 0) mbar_drain(&bars.q_full[s], (q_fills[s] - 1) & 1, lim);
      }
    }
  } else if (warp == Cfg::WARP_MMA || warp == Cfg::WARP_MMA2) {
    // ------------------------------------------------------------ MMA issuers
    // Thread A (WARP_MMA) issues each slot's S^T and dP^T, thread B (WARP_MMA2) its dV,
    // dK and dQ.  Their TMEM hand-offs are barriers already (st_free: B's dK has
    // consumed ST; dq_empty: the dQ warps have read XT; ds_full: the compute warps have
    // read dP^T), so neither waits on the other's issue order, and one thread's barrier
    // latency no longer idles the tensor pipe.  tcgen05.commit tracks the issuing
    // thread's own MMAs: everything that needs both threads' MMAs finished (q_empty,
    // kv_empty, acc_full) is committed by B, whose MMAs start only after A's of the same
    // slot have completed (p_full / ds_full follow s_full / dp_full).
    if (lane == 0) {
      const bool role_a = warp == Cfg::WARP_MMA;
      const uint32_t idesc_s = idesc_bf16(128, BQ, false, false);   // S^T, dP^T
      const uint32_t idesc_kv = idesc_bf16(128, HD, false, true);   // dV, dK (A from TMEM)
      const uint32_t idesc_dq = idesc_bf16(BQ, HD, true, true);     // dQ = dS K
      const uint32_t sK = smem_u32(smem + Cfg::SMEM_K);
      const uint32_t sV = smem_u32(smem + Cfg::SMEM_V);
      const uint32_t sQ = smem_u32(smem + Cfg::SMEM_Q);
      const uint32_t sDO = smem_u32(smem + Cfg::SMEM_DO);
      const uint32_t sDS = smem_u32(smem + Cfg::SMEM_DS);
      uint32_t kv_ph = 0, q_it = 0, p_ph = 0, ds_ph = 0;
      uint32_t q_full_uses[2] = {0, 0};
      uint32_t st_waits = 0, xt_waits = 0, acc_commits = 0;
      bool ok = true;
      if (prm.inject_stall) ok = mbar_wait(&bars.never, 0, wctx);
      // bf16 column of q rows 16ks .. 16ks+15 of P^T in ST: compute group h holds q rows
      // 64h .. 64h+63 as 32 packed columns at 64h (dS^T at 64h + 32)
      auto p_col = [](int ks) -> uint32_t { return uint32_t((ks >> 2) * 64 + (ks & 3) * 8); };
      for (int k = 0; ok; ++k) {
        const int slot = k % kUnitRing;
        ok = mbar_wait(&bars.unit_full[slot], (k / kUnitRing) & 1, wctx);
        if (!ok) break;
        const int idx = *reinterpret_cast<volatile int*>(&unit_ring[slot]);
        mbar_arrive(&bars.unit_empty[slot]);
        if (idx < 0) break;
        const KvUnit u = decode_kv_unit(idx, prm.Hkv, prm.n_ktiles);
        if (role_a) {
          ok = mbar_wait(&bars.kv_full, kv_ph, wctx);
          kv_ph ^= 1;
          if (!ok) break;
        }
        SlotWalk w;
        for (bool more = walk_first(prm, u.n, w), j0 = true; more && ok;
             more = walk_next(prm, u.n, w), j0 = false) {
          const int st = int(q_it & 1);
          if (role_a) {
            // S^T into ST once this stage's Q is in and B's dK has consumed ST
            ok = mbar_wait(&bars.q_full[st], q_full_uses[st] & 1, wctx);
            ++q_full_uses[st];
            if (ok && q_it > 0) ok = mbar_wait(&bars.st_free, st_waits++ & 1, wctx);
            if (!ok) break;
            tc_fence_after();
            for (int kb = 0; kb < KB; ++kb)
#pragma unroll
              for (int ks = 0; ks < 4; ++ks)
                mma_ss(tmem + Cfg::TM_ST, sdesc_sw128(sK + kb * BKV * 128 + ks * 32, 16, 1024),
                       sdesc_sw128(sQ + st * Cfg::QT_BYTES + kb * BQ * 128 + ks * 32, 16, 1024),
                       idesc_s, (kb | ks) != 0);
            mma_commit(&bars.s_full);
            // dP^T into XT once the dQ warps have read the previous dQ out of it
            if (q_it > 0) ok = mbar_wait(&bars.dq_empty, xt_waits++ & 1, wctx);
            if (!ok) break;
            tc_fence_after();
            for (int kb = 0; kb < KB; ++kb)
#pragma unroll
              for (int ks = 0; ks < 4; ++ks)
                mma_ss(tmem + Cfg::TM_XT, sdesc_sw128(sV + kb * BKV * 128 + ks * 32, 16, 1024),
                       sdesc_sw128(sDO + st * Cfg::QT_BYTES + kb * BQ * 128 + ks * 32, 16, 1024),
                       idesc_s, (kb | ks) != 0);
            mma_commit(&bars.dp_full);
          } else {
            // dV += P^T dO
            ok = mbar_wait(&bars.p_full, p_ph, wctx);
            p_ph ^= 1;
            if (ok && j0 && acc_commits > 0) ok = mbar_wait(&bars.acc_empty, (acc_commits - 1) & 1, wctx);
            if (!ok) break;
            tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < BQ / 16; ++ks)
              mma_ts(tmem + Cfg::TM_DV, tmem + Cfg::TM_ST + p_col(ks),
                     sdesc_sw128(sDO + st * Cfg::QT_BYTES + ks * 2048, BQ * 128, 1024), idesc_kv,
                     !j0 || (ks > 0));
            // dK += dS^T Q, then dQ = dS K into XT (dP^T there was loaded already)
            ok = mbar_wait(&bars.ds_full, ds_ph, wctx);
            ds_ph ^= 1;
            if (!ok) break;
            tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < BQ / 16; ++ks)
              mma_ts(tmem + Cfg::TM_DK, tmem + Cfg::TM_ST + p_col(ks) + 32,
                     sdesc_sw128(sQ + st * Cfg::QT_BYTES + ks * 2048, BQ * 128, 1024), idesc_kv,
                     !j0 || (ks > 0));
            mma_commit(&bars.st_free);
            // A = dS: the dS^T tile read M-major (two 64-wide q blocks 16 KB apart);
            // B = K: the resident K tile read N-major (64-wide d blocks 16 KB apart)
#pragma unroll
            for (int ks = 0; ks < BKV / 16; ++ks)
              mma_ss(tmem + Cfg::TM_XT, sdesc_sw128(sDS + ks * 2048, BKV * 128, 1024),
                     sdesc_sw128(sK + ks * 2048, BKV * 128, 1024), idesc_dq, ks > 0);
            mma_commit(&bars.dq_full);
            mma_commit(&bars.dsm_free);
            // the stage's Q / dO are released by the dQ warps, which stage dQ there
          }
          ++q_it;
        }
        if (!ok) break;
        if (!role_a) {
          mma_commit(&bars.acc_full);
          ++acc_commits;
          mma_commit(&bars.kv_empty);
        }
      }
      mma_commit(&bars.drain);
      mbar_drain(&bars.drain, 0, 1000000000ull);
    }
    __syncwarp();
  } else if (warp >= Cfg::WARP_DQ) {
    // ------------------------------------------------------------ dQ warps
    // dQ = dS K of a slot lies in XT with TMEM lane = q row and column = d, so dQ warp
    // qw holds q rows 32qw .. 32qw+31 and each thread one row: it moves its row in 16-byte
    // pieces into [32 q][32 d] fp32 boxes (128-byte rows, 128-byte swizzle: conflict-free
    // for 8 threads a wavefront) and one TMA bulk reduce-add per box adds them into the
    // head-major fp32 accumulator.  The boxes live in the slot's own Q and dO stage (HD *
    // 512 bytes, exactly the size of dQ): once dQ exists every MMA that reads that stage
    // has completed, and the producer refills it only after the reduces have read it out
    // (q_empty).  XT is read in pairs of 32-column chunks and released after the last
    // pair's load, before that pair is staged.  No per-element atomics leave the SM.
    const int qw = warp - Cfg::WARP_DQ;
    const uint32_t tXT = tmem + Cfg::TM_XT + (uint32_t(qw * 32) << 16);
    constexpr int NCH = HD / 32;                   // 32-column chunks of a row of dQ
    uint32_t sw_off[8];                            // this thread's row, 16-byte piece j
#pragma unroll
    for (int j = 0; j < 8; ++j) sw_off[j] = sw128_offset(uint32_t(lane), uint32_t(j));
    uint32_t dq_ph = 0, q_it = 0;
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
      for (bool more = walk_first(prm, u.n, w); more; more = walk_next(prm, u.n, w)) {
        ok = warp_wait_b(&bars.dq_full, dq_ph, wctx);
        dq_ph ^= 1;
        if (!ok) break;
        tc_fence_after();
        const int st = int(q_it & 1);
        const int32_t h = u.g * prm.G + w.e;
        const int32_t row0 = int32_t((int64_t(w.r - prm.shard_begin) * prm.B + u.b) * twoC +
                                     int64_t(w.i) * BQ + qw * 32);
#pragma unroll 1
        for (int c0 = 0; c0 < NCH; c0 += 2) {
          uint32_t v[2][32];
          tmem_ld32(tXT + c0 * 32, v[0]);
          tmem_ld32(tXT + c0 * 32 + 32, v[1]);
          tmem_ld_wait();
          if (c0 + 2 == NCH) {             // all of dQ read: XT may be overwritten
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars.dq_empty);
          }
#pragma unroll
          for (int cc = 0; cc < 2; ++cc) {
            const int bi = qw * NCH + c0 + cc;   // box index within the stage's 16*HD rows
            uint8_t* box = bi * 4096 < Cfg::QT_BYTES
                               ? smem + Cfg::SMEM_Q + st * Cfg::QT_BYTES + bi * 4096
                               : smem + Cfg::SMEM_DO + st * Cfg::QT_BYTES + (bi * 4096 - Cfg::QT_BYTES);
#pragma unroll
            for (int j = 0; j < 8; ++j)
              *reinterpret_cast<uint4*>(box + sw_off[j]) =
                  make_uint4(v[cc][4 * j], v[cc][4 * j + 1], v[cc][4 * j + 2], v[cc][4 * j + 3]);
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
              tma_reduce_add_3d(&map_dq, box, (c0 + cc) * 32, row0, h);
              bulk_commit_group();
            }
          }
        }
        if (lane == 0) bulk_wait_group_read0();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars.q_empty[st]);
        ++q_it;
      }
    }
    // every reduce issued by this warp has been performed before the kernel ends
    if (lane == 0) bulk_wait_group0();
    __syncwarp();
  } else {
    // ------------------------------------------------------------ compute warps
    // group h = warp / 4 handles q rows 64h .. 64h+63 of every slot (contiguous
    // positions: a 64-row half never straddles a zigzag chunk); thread = key row
    const int hgrp = warp / 4;
    const int qw = warp % 4;
    const int row = qw * 32 + lane;
    const uint32_t lane_addr = uint32_t(qw * 32) << 16;
    const uint32_t tS = tmem + Cfg::TM_ST + 64 * hgrp + lane_addr;
    const uint32_t tX = tmem + Cfg::TM_XT + 64 * hgrp + lane_addr;
    uint8_t* dsb = smem + Cfg::SMEM_DS + hgrp * (BKV * 128);
    uint32_t q_it = 0, s_ph = 0, dp_ph = 0, acc_ph = 0, dsm_uses = 0;
    uint32_t q_full_uses[2] = {0, 0};
    bool ok = true;
    int nslots = 0;                            // slots of the current unit
    for (int k = 0; ok; ++k) {
      const int slot = k % kUnitRing;
      ok = warp_wait_b(&bars.unit_full[slot], (k / kUnitRing) & 1, wctx);
      if (!ok) break;
      const int idx = *reinterpret_cast<volatile int*>(&unit_ring[slot]);
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.unit_empty[slot]);
      if (idx < 0) break;
      const KvUnit u = decode_kv_unit(idx, prm.Hkv, prm.n_ktiles);
      const int64_t key = int64_t(u.n) * BKV + row;
      SlotWalk w;
      nslots = 0;
      for (bool more = walk_first(prm, u.n, w); more && ok; more = walk_next(prm, u.n, w)) {
        ++nslots;
        const int st = int(q_it & 1);
        ok = warp_wait_b(&bars.q_full[st], q_full_uses[st] & 1, wctx);
        ++q_full_uses[st];
        if (!ok) break;
        // this group's 64 columns of -lse log2(e) and -Delta (K2), as float4s
        const float4* nl4 = reinterpret_cast<const float4*>(smem + Cfg::SMEM_LSE) + (st * BQ + 64 * hgrp) / 4;
        const float4* nd4 = reinterpret_cast<const float4*>(smem + Cfg::SMEM_DELTA) + (st * BQ + 64 * hgrp) / 4;
        const int64_t p0 = zz_pos(prm.C, prm.D, w.r, int64_t(w.i) * BQ + 64 * hgrp);
        const int nvis_lo = prm.causal ? int(key - p0) : 0;   // columns c < nvis_lo are masked
        // only slots whose columns cross this warp's keys need the mask (warp-uniform)
        const bool masked = __any_sync(0xffffffffu, nvis_lo > 0);
        const uint64_t scale2 = f2_pack(prm.scale_log2, prm.scale_log2);
        // ---- P^T = 2^(scale log2(e) S^T - lse log2(e)) -> bf16 over the first half of
        //      this group's columns
        ok = warp_wait_b(&bars.s_full, s_ph, wctx);
        s_ph ^= 1;
        if (!ok) break;
        tc_fence_after();
        uint32_t pk[2][16];
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
          uint32_t sv[32];
          tmem_ld32(tS + cc * 32, sv);
          tmem_ld_wait();
#pragma unroll
          for (int q4 = 0; q4 < 8; ++q4) {
            const float4 nl = nl4[cc * 8 + q4];
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
              const int e = 2 * q4 + hh;
              const uint64_t x2 = f2_fma(f2_pack(__uint_as_float(sv[2 * e]), __uint_as_float(sv[2 * e + 1])),
                                         scale2, hh == 0 ? f2_pack(nl.x, nl.y) : f2_pack(nl.z, nl.w));
              float x0, x1;
              f2_unpack(x2, x0, x1);
              float e0 = ex2_approx(x0), e1 = ex2_approx(x1);
              if (masked) {
                const int c0 = cc * 32 + 2 * e;
                e0 = c0 < nvis_lo ? 0.f : e0;
                e1 = c0 + 1 < nvis_lo ? 0.f : e1;
              }
              pk[cc][e] = pack_bf16x2(e0, e1);
            }
          }
          tmem_st16(tS + cc * 16, pk[cc]);     // S^T columns already loaded
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars.p_full);
        // ---- dS^T = P^T (dP^T - Delta) -> bf16 into the second half of the columns and
        //      into shared memory (A operand of dQ)
        ok = warp_wait_b(&bars.dp_full, dp_ph, wctx);
        dp_ph ^= 1;
        if (ok && dsm_uses > 0) ok = warp_wait_b(&bars.dsm_free, (dsm_uses - 1) & 1, wctx);
        if (!ok) break;
        ++dsm_uses;
        tc_fence_after();
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
          uint32_t sv[32];
          tmem_ld32(tX + cc * 32, sv);
          tmem_ld_wait();
          uint32_t dk[16];
#pragma unroll
          for (int q4 = 0; q4 < 8; ++q4) {
            const float4 nd = nd4[cc * 8 + q4];
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
              const int e = 2 * q4 + hh;
              const uint64_t t2 = f2_add(f2_pack(__uint_as_float(sv[2 * e]), __uint_as_float(sv[2 * e + 1])),
                                         hh == 0 ? f2_pack(nd.x, nd.y) : f2_pack(nd.z, nd.w));
              float d0, d1;
              f2_unpack(f2_mul(bf16x2_widen(pk[cc][e]), t2), d0, d1);
              dk[e] = pack_bf16x2(d0, d1);
            }
          }
          tmem_st16(tS + 32 + cc * 16, dk);
#pragma unroll
          for (int m = 0; m < 4; ++m)
            *reinterpret_cast<uint4*>(dsb + sw128_offset(uint32_t(row), uint32_t(4 * cc + m))) =
                make_uint4(dk[4 * m], dk[4 * m + 1], dk[4 * m + 2], dk[4 * m + 3]);
        }
        fence_proxy_async_smem();
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&bars.ds_full);
          mbar_arrive(&bars.q_empty[st]);     // lse / Delta of this stage consumed
        }
        ++q_it;
      }
      if (!ok) break;
      // ---- epilogue: dV (group 0) / dK (group 1) rows of this key tile
      ok = warp_wait_b(&bars.acc_full, acc_ph, wctx);
      acc_ph ^= 1;
      if (!ok) break;
      tc_fence_after();
      const uint32_t tAcc = tmem + (hgrp == 0 ? Cfg::TM_DV : Cfg::TM_DK) + lane_addr;
      const float mul = hgrp == 0 ? 1.0f : prm.scale;
      const int64_t krow = kv_tensor_row(int32_t(key), u.b, int32_t(prm.S), int32_t(prm.C), prm.B, prm.D,
                                           prm.kv_shard_major);
      __nv_bfloat16* dst = (hgrp == 0 ? prm.dv : prm.dk) + (krow * prm.Hkv + u.g) * HD;
      // a key tile no query of the launch's shards sees has no MMA behind its
      // accumulators: its dK / dV rows are zero
      const bool empty = nslots == 0;
#pragma unroll 1
      for (int c = 0; c < HD / 32; ++c) {
        uint32_t a[32];
        if (!empty) {
          tmem_ld32(tAcc + c * 32, a);
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
  if (warp == Cfg::WARP_MMA) tmem_dealloc(tmem, Cfg::TM_COLS);
}

int num_sms() {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return sms;
}

template <int HD>
int launch_bwd_hd(const BwdArgs& a, cudaStream_t stream) {
  // 128-key tiles.  d <= 128: one CTA per key tile with 128-row q slots, every MMA
  // N = 128 (zsa_bwd_wide_kernel); d = 256: a cluster of two CTAs per key tile with
  // 64-row q slots (zsa_bwd_pair_kernel), since dK + dV of the tile alone fill one SM's
  // TMEM.
  constexpr bool kWide = HD <= 128;
  constexpr int BQ = kWide ? 128 : 64, BKV = 128;
  const int64_t twoC = a.S / a.D;
  const int64_t rows = int64_t(a.shard_count) * a.B * twoC;   // local shard-major rows
  const int sms = num_sms();
  // K2: Delta and a zeroed dQ accumulator
  {
    const int64_t pairs = rows * a.Hq;
    const int64_t warps_needed = (pairs + 31) / 32;
    int64_t blocks = (warps_needed + 7) / 8;
    if (blocks > int64_t(sms) * 16) blocks = int64_t(sms) * 16;
    if (blocks < 1) blocks = 1;
    const TraceEvents tr = trace_events(1);
    if (tr.begin) cudaEventRecord(tr.begin, stream);
    zsa_bwd_pre_kernel<HD><<<int(blocks), 256, 0, stream>>>(
        reinterpret_cast<const __nv_bfloat16*>(a.o), reinterpret_cast<const __nv_bfloat16*>(a.dout),
        a.lse, a.delta, a.nlse2, a.dq_acc, pairs, a.Hq, twoC);
    cudaError_t e = cudaGetLastError();
    if (tr.end) cudaEventRecord(tr.end, stream);
    if (e != cudaSuccess) return int(e);
  }
  // K3
  CUtensorMap mq, mk, mv, mdo;
  {
    const uint64_t dims[3] = {uint64_t(HD), uint64_t(a.Hq), uint64_t(rows)};
    const uint64_t strides[2] = {uint64_t(HD) * 2, uint64_t(a.Hq) * HD * 2};
    const uint32_t box[3] = {64, 1, uint32_t(BQ)};
    if (!make_map_bf16_sw128(&mq, a.q, 3, dims, strides, box)) return int(cudaErrorInvalidValue);
    if (!make_map_bf16_sw128(&mdo, a.dout, 3, dims, strides, box)) return int(cudaErrorInvalidValue);
  }
  {
    const uint64_t dims[3] = {uint64_t(HD), uint64_t(a.Hkv), uint64_t(a.B * a.S)};
    const uint64_t strides[2] = {uint64_t(HD) * 2, uint64_t(a.Hkv) * HD * 2};
    // a box never straddles a zigzag chunk: its rows are contiguous in both layouts
    const uint32_t box[3] = {64, 1, uint32_t((a.S / (2 * int64_t(a.D))) % BKV == 0 ? BKV : 64)};
    if (!make_map_bf16_sw128(&mk, a.k, 3, dims, strides, box)) return int(cudaErrorInvalidValue);
    if (!make_map_bf16_sw128(&mv, a.v, 3, dims, strides, box)) return int(cudaErrorInvalidValue);
  }
  CUtensorMap mdq;   // the head-major fp32 dQ accumulator: [32 rows][32 d] reduce boxes
  {
    const uint64_t dims[3] = {uint64_t(HD), uint64_t(rows), uint64_t(a.Hq)};
    const uint64_t strides[2] = {uint64_t(HD) * 4, uint64_t(rows) * HD * 4};
    const uint32_t box[3] = {32, 32, 1};
    if (!make_map_f32_sw128(&mdq, a.dq_acc, 3, dims, strides, box)) return int(cudaErrorInvalidValue);
  }
  BwdParams p;
  p.nlse2 = a.nlse2;
  p.ndelta = a.delta;
  p.dq_acc = a.dq_acc;
  p.dk = reinterpret_cast<__nv_bfloat16*>(a.dk);
  p.dv = reinterpret_cast<__nv_bfloat16*>(a.dv);
  p.S = a.S;
  p.C = a.S / (2 * int64_t(a.D));
  p.B = a.B; p.Hq = a.Hq; p.Hkv = a.Hkv; p.G = a.Hq / a.Hkv; p.D = a.D; p.causal = a.causal;
  p.n_units = int32_t(int64_t(a.B) * a.Hkv * (a.S / BKV));
  p.n_qtiles = int32_t(twoC / BQ);
  p.bq = BQ;
  p.n_ktiles = int32_t(a.S / BKV);
  p.kv_shard_major = a.kv_layout;
  p.kv_box = (a.S / (2 * int64_t(a.D))) % BKV == 0 ? BKV : 64;
  p.shard_begin = a.shard_begin;
  p.shard_end = a.shard_begin + a.shard_count;
  p.rows = rows;
  p.counter = a.status + 32;
  p.scale = a.scale;
  p.scale_log2 = float(double(a.scale) * 1.4426950408889634);
  p.status = a.status;
  p.wait_limit_ns = a.wait_limit_ns;
  p.inject_stall = a.inject_stall;
  cudaError_t e = cudaSuccess;
  if constexpr (kWide) {
    using Cfg = BwdWideCfg<HD>;
    const int smem = Cfg::SMEM_BYTES;   // the kernel aligns its dynamic shared memory itself
    {
      const int err = ensure_smem_attr(reinterpret_cast<const void*>(zsa_bwd_wide_kernel<HD>), smem);
      if (err != int(cudaSuccess)) return err;
    }
    const int grid = p.n_units < sms ? p.n_units : sms;
    const TraceEvents tr = trace_events(2);
    if (tr.begin) cudaEventRecord(tr.begin, stream);
    zsa_bwd_wide_kernel<HD><<<grid, Cfg::NTHREADS, smem, stream>>>(mq, mk, mv, mdo, mdq, p);
    e = cudaGetLastError();
    if (tr.end) cudaEventRecord(tr.end, stream);
  } else {
    e = cudaError_t(launch_pair_main(mq, mk, mv, mdo, mdq, p, stream));
  }
  if (e != cudaSuccess) return int(e);
  // K4
  {
    int64_t blocks = rows;
    if (blocks > int64_t(sms) * 16) blocks = int64_t(sms) * 16;
    const TraceEvents tr4 = trace_events(3);
    if (tr4.begin) cudaEventRecord(tr4.begin, stream);
    zsa_dq_convert_kernel<HD><<<int(blocks), 256, 0, stream>>>(
        a.dq_acc, reinterpret_cast<__nv_bfloat16*>(a.dq), rows, a.Hq, a.scale);
    e = cudaGetLastError();
    if (tr4.end) cudaEventRecord(tr4.end, stream);
  }
  return int(e);
}

}  // namespace

int launch_bwd(const BwdArgs& a, cudaStream_t stream) {
  switch (a.d) {
    case 64: return launch_bwd_hd<64>(a, stream);
    case 128: return launch_bwd_hd<128>(a, stream);
    case 256: return launch_bwd_hd<256>(a, stream);
    default: return int(cudaErrorNotSupported);
  }
}

}  // namespace zsa
