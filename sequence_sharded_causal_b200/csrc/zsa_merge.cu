// zsa_merge.cu -- merge of partial attention results over disjoint key sets.
//
// Ring attention ("AutoSP" summary, sections 1 and 4, the sequence-parallel baseline)
// gives each rank's queries the K/V blocks one after another; each block yields the
// softmax attention restricted to its keys, (O_i, lse_i).  Over the union of the blocks
//   lse = ln sum_i exp(lse_i),   O = sum_i exp(lse_i - lse) O_i,
// an empty block (lse_i = -inf) contributing nothing.  This kernel evaluates that for
// every (row, q head) of a Q-layout tensor in one pass: a running maximum over the parts
// with the sum and the weighted O rescaled whenever the maximum grows (the same
// bookkeeping as an online softmax, here over parts instead of keys).
//
// HBM-bound: per (row, head) it reads n * (2d + 4) bytes and writes 2d + 4.  Lanes
// take 16 bytes (8 bf16) each, d/8 lanes per (row, head), so each part's O is read in
// fully coalesced 256-byte rows at d = 128; the parts' lse values for one (row, head)
// are the same address for all of its lanes.  The output may alias any part (each lane
// reads all of its inputs before it writes).
#include <cuda_bf16.h>

#include <cmath>

#include "zsa_kernels.h"
#include "zsa_ptx.cuh"

namespace zsa {
namespace {

// Index arithmetic is 32-bit (the launcher checks that rows * Hq * d < 2^31): 64-bit
// divisions per (row, head) would make this HBM-bound kernel issue-bound.  Each warp
// takes U = 2 groups of (row, head) pairs per iteration and issues the loads of both,
// PG = 2 parts at a time, before any arithmetic; with 4 CTAs of 256 threads per SM
// (registers capped at 64) that keeps about 64 KB of loads in flight per SM, what the
// HBM latency-bandwidth product asks for.  Weights are computed in log2 units with
// ex2.approx.
template <int HD>
__global__ void __launch_bounds__(256, 4) zsa_merge_kernel(const __grid_constant__ MergeArgs a,
                                                        uint32_t n_pairs, uint32_t twoC) {
  constexpr uint32_t LPP = HD / 8;            // lanes per (row, head), 16 bytes each
  constexpr uint32_t PPW = 32u / LPP;         // (row, head) pairs per warp and group
  constexpr int U = 2;                        // groups per iteration
  constexpr int PG = 2;                       // parts loaded together
  constexpr float kL2e = 1.4426950408889634f, kLn2 = 0.6931471805599453f;
  const uint32_t lane = threadIdx.x & 31u;
  const uint32_t sub = lane % LPP;
  const uint32_t Hq = uint32_t(a.Hq);
  const uint32_t warp_global = (blockIdx.x * blockDim.x + threadIdx.x) / 32u;
  const uint32_t n_warps = gridDim.x * blockDim.x / 32u;
  const uint32_t stride = n_warps * PPW;      // pairs between a warp's two groups
  for (uint32_t base = warp_global * PPW; base < n_pairs; base += U * stride) {
    uint32_t off[U], lidx[U];
    bool live[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const uint32_t pair = base + uint32_t(u) * stride + lane / LPP;   // O layout's order
      live[u] = pair < n_pairs;
      const uint32_t row = live[u] ? pair / Hq : 0u;
      const uint32_t h = live[u] ? pair - row * Hq : 0u;
      const uint32_t rb = row / twoC;
      lidx[u] = (rb * Hq + h) * twoC + (row - rb * twoC);            // lse layout
      off[u] = (live[u] ? pair : 0u) * LPP + sub;                      // 16-byte word
    }
    float m[U], l[U], acc[U][8];                // m: running max of lse * log2(e)
#pragma unroll
    for (int u = 0; u < U; ++u) {
      m[u] = -INFINITY;
      l[u] = 0.f;
#pragma unroll
      for (int t = 0; t < 8; ++t) acc[u][t] = 0.f;
    }
    for (int i0 = 0; i0 < a.n; i0 += PG) {
      float li[U][PG];
      uint4 x[U][PG];
#pragma unroll
      for (int t = 0; t < PG; ++t) {
        const bool have = i0 + t < a.n;
        const int i = have ? i0 + t : i0;
#pragma unroll
        for (int u = 0; u < U; ++u) {
          li[u][t] = have && live[u] ? a.lse[i][lidx[u]] : -INFINITY;
          x[u][t] = reinterpret_cast<const uint4*>(a.o[i])[off[u]];
        }
      }
#pragma unroll
      for (int u = 0; u < U; ++u)
#pragma unroll
        for (int t = 0; t < PG; ++t) {
          if (li[u][t] == -INFINITY) continue;   // an empty key set (or no part) adds nothing
          const float l2 = li[u][t] * kL2e;
          if (l2 > m[u]) {                       // rescale what was summed against the old max
            const float c = ex2_approx(m[u] - l2);   // m = -inf at the first live part: c = 0
            l[u] *= c;
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[u][e] *= c;
            m[u] = l2;
          }
          const float w = ex2_approx(l2 - m[u]);
          l[u] += w;
          const uint32_t xs[4] = {x[u][t].x, x[u][t].y, x[u][t].z, x[u][t].w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            acc[u][2 * e] = fmaf(w, __uint_as_float(xs[e] << 16), acc[u][2 * e]);
            acc[u][2 * e + 1] = fmaf(w, __uint_as_float(xs[e] & 0xFFFF0000u), acc[u][2 * e + 1]);
          }
        }
    }
    __syncwarp();                              // every lane has read its inputs
#pragma unroll
    for (int u = 0; u < U; ++u) {
      if (!live[u]) continue;
      const bool empty = m[u] == -INFINITY;
      const float inv = empty ? 0.f : 1.0f / l[u];
      uint4 y;
      y.x = pack_bf16x2(acc[u][0] * inv, acc[u][1] * inv);
      y.y = pack_bf16x2(acc[u][2] * inv, acc[u][3] * inv);
      y.z = pack_bf16x2(acc[u][4] * inv, acc[u][5] * inv);
      y.w = pack_bf16x2(acc[u][6] * inv, acc[u][7] * inv);
      reinterpret_cast<uint4*>(a.o_out)[off[u]] = y;
      if (sub == 0) a.lse_out[lidx[u]] = empty ? -INFINITY : (m[u] + __log2f(l[u])) * kLn2;
    }
  }
}

template <int HD>
int launch_merge_hd(const MergeArgs& a, cudaStream_t stream) {
  const int64_t twoC = a.S / a.D;
  const int64_t n_pairs = a.rows * a.Hq;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  // 8 warps x pairs per warp x 2 groups per iteration; at most the 4 resident CTAs per
  // SM, which then stride over the rest
  const int64_t pairs_per_block = 8 * (32 / (HD / 8)) * 2;
  int64_t blocks = (n_pairs + pairs_per_block - 1) / pairs_per_block;
  if (blocks > int64_t(sms) * 4) blocks = int64_t(sms) * 4;
  if (blocks < 1) return int(cudaSuccess);
  const TraceEvents tr = trace_events(4);
  if (tr.begin) cudaEventRecord(tr.begin, stream);
  zsa_merge_kernel<HD><<<int(blocks), 256, 0, stream>>>(a, uint32_t(n_pairs), uint32_t(twoC));
  const cudaError_t e = cudaGetLastError();
  if (tr.end) cudaEventRecord(tr.end, stream);
  return int(e);
}

}  // namespace

int launch_merge(const MergeArgs& a, cudaStream_t stream) {
  switch (a.d) {
    case 64: return launch_merge_hd<64>(a, stream);
    case 128: return launch_merge_hd<128>(a, stream);
    case 256: return launch_merge_hd<256>(a, stream);
    default: return int(cudaErrorInvalidValue);
  }
}

}  // namespace zsa
