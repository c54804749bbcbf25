// zsa_gemm.cu -- the local projection of one step of the TSP attention-layer schedule.
//
// "Folding Tensor and Sequence Parallelism" (summary page, section 2, attention layer):
// each rank holds 1/D of the tokens and one packed shard of the attention weights
// (W_Q, W_K, W_V, W_O); step s broadcasts rank s's shard and every rank multiplies its
// own tokens by it.  One step on one rank is the GEMM
//     Y = X W_s,   X [T][K] (the rank's tokens), W_s [K][N] (the shard, row-major)
// whose N output columns are routed, in runs of columns ("segments"), to where they
// belong: Q, K and V columns of the shard's heads (bf16, overwritten), or an fp32
// accumulator that sums the output projection's per-step partials.
//
// Any T; N a multiple of 32; K a multiple of 8: tiles past the edges load zeros (TMA
// out-of-bounds fill) and the epilogue stores only rows < T and 32-column chunks < N.
//
// Kernel: persistent CTAs over 128 x BN output tiles (BN = 256 where N and the tile
// count allow, else 128), rastered in bands of 16 row blocks (m fastest inside a band,
// then n, then the next band): the tiles running together cover a few row blocks of X and
// a few column blocks of W_s, so each X row block is read from HBM about once instead of
// once per column block (an m-fastest order over all of T re-read X for every column
// block: 12x its size at T = 16384, N = 2048).  One TMA warp streams [128 m][64 k] tiles
// of X (K-major) and [64 k][BN n] tiles of W_s (64-wide n boxes, MN-major) through a ring
// of 4 (BN = 256) or 6 stages; one thread issues tcgen05.mma (M = 128, N = BN, K = 16)
// into one of two TMEM accumulators; 4 epilogue warps (thread = output row) drain the
// other accumulator meanwhile.  fp32-accumulate chunks leave by TMA bulk
// reduce-add (each warp stages its [32 rows][32 columns] in a double-buffered,
// 128B-swizzled box), so the accumulator is never read back by the SM; bf16 chunks are
// stored directly.  Every wait is bounded.
#include <cuda_bf16.h>

#include "zsa_kernels.h"
#include "zsa_ptx.cuh"
#include "zsa_tma_host.h"

namespace zsa {
namespace {

// Output tile t -> (m block, n block): bands of kBand row blocks, m fastest in a band.
constexpr int32_t kBand = 16;
__device__ __forceinline__ void tile_mn(int32_t t, int32_t mt, int32_t nt, int32_t& mb, int32_t& nb) {
  const int32_t band = t / (kBand * nt);
  const int32_t in = t - band * (kBand * nt);
  const int32_t rows = mt - band * kBand < kBand ? mt - band * kBand : kBand;  // rows in this band
  nb = in / rows;
  mb = band * kBand + (in - nb * rows);
}

// Tiles of 128 x TBN outputs: TBN = 256 (N = 256 MMAs) halves the operand bytes staged per
// FLOP against TBN = 128 (every 128 rows of X feed twice the columns), for GEMMs with
// enough tiles; TBN = 128 keeps small-N steps (a few tiles per SM) from wasting columns.
template <int TBN>
struct GemmCfg {
  static constexpr int BM = 128, BN = TBN, BK = 64;
  static constexpr int STAGES = TBN == 256 ? 4 : 6;
  static constexpr int A_BYTES = BM * BK * 2;     // 16 KB
  static constexpr int B_BYTES = BK * BN * 2;     // [BN / 64 n blocks][64 k][128 B]
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int STG_BYTES = 4 * 2 * 32 * 128;   // 4 warps x 2 boxes of [32 rows][32 fp32]
  static constexpr int SMEM_STG = STAGES * STAGE_BYTES;
  static constexpr int SMEM_BYTES = SMEM_STG + STG_BYTES;
  static constexpr int WARP_LOAD = 4;
  static constexpr int WARP_MMA = 5;
  static constexpr int NTHREADS = 6 * 32;
  static constexpr uint32_t TM_COLS = 2 * BN;     // two BN-column accumulators
  static_assert(SMEM_BYTES + 1024 <= 227 * 1024, "shared memory budget");
};

// Tensor maps of the fp32-accumulate segments ([T][cols] fp32, [32 rows][32 cols] boxes).
struct SegMaps {
  CUtensorMap m[kProjMaxSegs];
};

struct GemmParams {
  int64_t T, N, K;
  int32_t mt, nt;                  // 128-row and 128-column tile counts
  int32_t n_segs;
  ProjSegment segs[kProjMaxSegs];  // column runs of W_s, in order
  int* status;
  uint64_t wait_limit_ns;
};

struct GemmBars {
  uint64_t full[6], empty[6];                      // GemmCfg<BN>::STAGES <= 6
  uint64_t acc_full[2], acc_empty[2];
  uint64_t drain;
};

template <int TBN>
__global__ void __launch_bounds__(GemmCfg<TBN>::NTHREADS, 1)
    zsa_proj_gemm_kernel(const __grid_constant__ CUtensorMap map_x,
                         const __grid_constant__ CUtensorMap map_w,
                         const __grid_constant__ SegMaps seg_maps, const GemmParams prm) {
  using Cfg = GemmCfg<TBN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  __shared__ GemmBars bars;
  __shared__ uint32_t tmem_base_s;
  __shared__ int abort_s;
  const int warp = int(warp_id()), lane = int(lane_id());
  if (threadIdx.x == 0) {
    abort_s = 0;
    for (int s = 0; s < Cfg::STAGES; ++s) {
      mbar_init(&bars.full[s], 1);
      mbar_init(&bars.empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars.acc_full[s], 1);
      mbar_init(&bars.acc_empty[s], 4);
    }
    mbar_init(&bars.drain, 1);
    fence_mbar_init();
  }
  if (warp == Cfg::WARP_MMA) {
    tmem_alloc(&tmem_base_s, Cfg::TM_COLS);
    tmem_relinquish();
  }
  if (warp == Cfg::WARP_LOAD && lane == 0) {
    tma_prefetch_desc(&map_x);
    tma_prefetch_desc(&map_w);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_s;
  const WaitCtx wctx{&abort_s, prm.status, prm.wait_limit_ns};
  const int32_t n_tiles = prm.mt * prm.nt;
  const int32_t kblocks = int32_t((prm.K + Cfg::BK - 1) / Cfg::BK);

  if (warp == Cfg::WARP_LOAD) {
    if (lane == 0) {
      uint32_t it = 0;
      uint32_t fills[Cfg::STAGES];
      for (int s = 0; s < Cfg::STAGES; ++s) fills[s] = 0;
      bool ok = true;
      for (int32_t t = blockIdx.x; t < n_tiles && ok; t += gridDim.x) {
        int32_t mb, nb;
        tile_mn(t, prm.mt, prm.nt, mb, nb);
        const int32_t m0 = mb * Cfg::BM, n0 = nb * Cfg::BN;
        for (int32_t kb = 0; kb < kblocks; ++kb, ++it) {
          const int st = int(it % Cfg::STAGES);
          if (it >= uint32_t(Cfg::STAGES)) ok = mbar_wait(&bars.empty[st], ((it / Cfg::STAGES) - 1) & 1, wctx);
          if (!ok) break;
          uint8_t* sa = smem + st * Cfg::STAGE_BYTES;
          mbar_expect_tx(&bars.full[st], Cfg::STAGE_BYTES);
          tma_load_3d(sa, &map_x, &bars.full[st], kb * Cfg::BK, m0, 0);
          for (int nb = 0; nb < Cfg::BN / 64; ++nb)
            tma_load_3d(sa + Cfg::A_BYTES + nb * (Cfg::BK * 128), &map_w, &bars.full[st],
                        n0 + nb * 64, kb * Cfg::BK, 0);
          ++fills[st];
        }
      }
      if (!ok)   // teardown: let the copies in flight land before the CTA exits
        for (int s = 0; s < Cfg::STAGES; ++s)
          if (fills[s] > 0) mbar_drain(&bars.full[s], (fills[s] - 1) & 1, 1000000000ull);
    }
  } else if (warp == Cfg::WARP_MMA) {
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16(128, Cfg::BN, false, true);   // A K-major, B N-major
      uint32_t it = 0, tile_it = 0;
      bool ok = true;
      for (int32_t t = blockIdx.x; t < n_tiles && ok; t += gridDim.x, ++tile_it) {
        const int acc = int(tile_it & 1);
        if (tile_it >= 2) ok = mbar_wait(&bars.acc_empty[acc], ((tile_it / 2) - 1) & 1, wctx);
        if (!ok) break;
        tc_fence_after();
        for (int32_t kb = 0; kb < kblocks; ++kb, ++it) {
          const int st = int(it % Cfg::STAGES);
          ok = mbar_wait(&bars.full[st], (it / Cfg::STAGES) & 1, wctx);
          if (!ok) break;
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + st * Cfg::STAGE_BYTES);
          const uint32_t sb = sa + Cfg::A_BYTES;
#pragma unroll
          for (int ks = 0; ks < Cfg::BK / 16; ++ks)
            mma_ss(tmem + uint32_t(acc * Cfg::BN), sdesc_sw128(sa + ks * 32, 16, 1024),
                   sdesc_sw128(sb + ks * 2048, Cfg::BK * 128, 1024), idesc, (kb | ks) != 0);
          mma_commit(&bars.empty[st]);
        }
        if (!ok) break;
        mma_commit(&bars.acc_full[acc]);
      }
      mma_commit(&bars.drain);
      mbar_drain(&bars.drain, 0, 1000000000ull);
    }
    __syncwarp();
  } else {
    // epilogue: thread = output row; 32-column chunks go to their segment
    const uint32_t lane_addr = uint32_t(warp * 32) << 16;
    const int row = warp * 32 + lane;
    uint8_t* stg = smem + Cfg::SMEM_STG + warp * (2 * 32 * 128);   // this warp's two boxes
    uint32_t tile_it = 0, n_red = 0;
    bool ok = true;
    for (int32_t t = blockIdx.x; t < n_tiles; t += gridDim.x, ++tile_it) {
      const int acc = int(tile_it & 1);
      ok = mbar_wait(&bars.acc_full[acc], (tile_it / 2) & 1, wctx);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      int32_t mb, nb;
      tile_mn(t, prm.mt, prm.nt, mb, nb);
      const int64_t m = int64_t(mb) * Cfg::BM + row;
      const int64_t n0 = int64_t(nb) * Cfg::BN;
      const bool row_in = m < prm.T;
#pragma unroll 1
      for (int c = 0; c < Cfg::BN / 32; ++c) {
        uint32_t v[32];
        tmem_ld32(tmem + uint32_t(acc * Cfg::BN + c * 32) + lane_addr, v);
        tmem_ld_wait();
        int64_t col = n0 + c * 32;
        if (col >= prm.N) continue;                  // past the output's edge
        int si = 0;
        while (si + 1 < prm.n_segs && col >= prm.segs[si].col_end) ++si;
        const ProjSegment& sg = prm.segs[si];
        const int64_t oc = col - sg.col_begin;
        if (sg.fp32_accumulate) {
          // stage [32 rows][32 fp32] (row = lane, 128-byte rows, 128-byte swizzle) and
          // reduce-add it; the box's other buffer may still be read by the previous reduce
          uint8_t* box = stg + (n_red & 1) * (32 * 128);
          if (lane == 0) bulk_wait_group_read1();
          __syncwarp();
#pragma unroll
          for (int q4 = 0; q4 < 8; ++q4)
            *reinterpret_cast<uint4*>(box + sw128_offset(uint32_t(lane), uint32_t(q4))) =
                make_uint4(v[4 * q4], v[4 * q4 + 1], v[4 * q4 + 2], v[4 * q4 + 3]);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_reduce_add_3d(&seg_maps.m[si], box, int32_t(oc),
                              int32_t(int64_t(mb) * Cfg::BM + warp * 32), 0);
            bulk_commit_group();
          }
          ++n_red;
        } else if (row_in) {
          uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(sg.out) + m * sg.ld + oc);
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4)
            dst[q4] = make_uint4(pack_bf16x2(__uint_as_float(v[8 * q4]), __uint_as_float(v[8 * q4 + 1])),
                                 pack_bf16x2(__uint_as_float(v[8 * q4 + 2]), __uint_as_float(v[8 * q4 + 3])),
                                 pack_bf16x2(__uint_as_float(v[8 * q4 + 4]), __uint_as_float(v[8 * q4 + 5])),
                                 pack_bf16x2(__uint_as_float(v[8 * q4 + 6]), __uint_as_float(v[8 * q4 + 7])));
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.acc_empty[acc]);
    }
    if (lane == 0) bulk_wait_group0();        // every reduce-add performed before exit
    __syncwarp();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == Cfg::WARP_MMA) tmem_dealloc(tmem, Cfg::TM_COLS);
}

template <int TBN>
int launch_proj_gemm_bn(const ProjArgs& a, cudaStream_t stream) {
  using Cfg = GemmCfg<TBN>;
  CUtensorMap mx, mw;
  {
    const uint64_t dims[3] = {uint64_t(a.K), uint64_t(a.T), 1};
    const uint64_t strides[2] = {uint64_t(a.ldx) * 2, uint64_t(a.ldx) * 2 * uint64_t(a.T)};
    const uint32_t box[3] = {64, uint32_t(Cfg::BM), 1};
    if (!make_map_bf16_sw128(&mx, a.x, 3, dims, strides, box)) return int(cudaErrorInvalidValue);
  }
  {
    const uint64_t dims[3] = {uint64_t(a.N), uint64_t(a.K), 1};
    const uint64_t strides[2] = {uint64_t(a.ldw) * 2, uint64_t(a.ldw) * 2 * uint64_t(a.K)};
    const uint32_t box[3] = {64, uint32_t(Cfg::BK), 1};
    if (!make_map_bf16_sw128(&mw, a.w, 3, dims, strides, box)) return int(cudaErrorInvalidValue);
  }
  SegMaps sm;
  for (int i = 0; i < a.n_segs; ++i) {
    if (!a.segs[i].fp32_accumulate) continue;
    const uint64_t cols = uint64_t(a.segs[i].col_end - a.segs[i].col_begin);
    const uint64_t dims[3] = {cols, uint64_t(a.T), 1};
    const uint64_t strides[2] = {uint64_t(a.segs[i].ld) * 4, uint64_t(a.segs[i].ld) * 4 * uint64_t(a.T)};
    const uint32_t box[3] = {32, 32, 1};
    if (!make_map_f32_sw128(&sm.m[i], a.segs[i].out, 3, dims, strides, box))
      return int(cudaErrorInvalidValue);
  }
  GemmParams p;
  p.T = a.T; p.N = a.N; p.K = a.K;
  p.mt = int32_t((a.T + Cfg::BM - 1) / Cfg::BM);
  p.nt = int32_t((a.N + Cfg::BN - 1) / Cfg::BN);
  p.n_segs = a.n_segs;
  for (int i = 0; i < a.n_segs; ++i) p.segs[i] = a.segs[i];
  p.status = a.status;
  p.wait_limit_ns = a.wait_limit_ns;
  const int smem = Cfg::SMEM_BYTES + 1024;
  int e = ensure_smem_attr(reinterpret_cast<const void*>(zsa_proj_gemm_kernel<TBN>), smem);
  if (e != int(cudaSuccess)) return e;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t tiles = int64_t(p.mt) * p.nt;
  const int grid = int(tiles < sms ? tiles : sms);
  if (grid <= 0) return int(cudaSuccess);
  const TraceEvents tr = trace_events(5);
  if (tr.begin) cudaEventRecord(tr.begin, stream);
  zsa_proj_gemm_kernel<TBN><<<grid, Cfg::NTHREADS, smem, stream>>>(mx, mw, sm, p);
  const cudaError_t err = cudaGetLastError();
  if (tr.end) cudaEventRecord(tr.end, stream);
  return int(err);
}

}  // namespace

// 256-wide tiles when N divides into them and they still give every SM at least two
// tiles; 128-wide otherwise.
int launch_proj_gemm(const ProjArgs& a, cudaStream_t stream) {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t tiles256 = ((a.T + 127) / 128) * (a.N / 256);
  if (a.N % 256 == 0 && tiles256 >= 2 * int64_t(sms)) return launch_proj_gemm_bn<256>(a, stream);
  return launch_proj_gemm_bn<128>(a, stream);
}

}  // namespace zsa
