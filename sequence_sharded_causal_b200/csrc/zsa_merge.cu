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
// fully coalesced 512-byte rows at d = 128; the parts' lse values for one (row, head)
// are the same address for all of its lanes.  The output may alias any part (each lane
// reads all of its inputs before it writes).
#include <cuda_bf16.h>

#include <cmath>

#include "zsa_kernels.h"
#include "zsa_ptx.cuh"

namespace zsa {
namespace {

template <int HD>
// Index arithmetic is 32-bit (the launcher checks that rows * Hq * d < 2^31): 64-bit
// divisions per (row, head) would make this HBM-bound kernel issue-bound.
__global__ void __launch_bounds__(256) zsa_merge_kernel(const __grid_constant__ MergeArgs a,
                                                        uint32_t n_pairs, uint32_t twoC) {
  constexpr uint32_t LPP = HD / 8;            // lanes per (row, head), 16 bytes each
  const uint32_t lane = threadIdx.x & 31u;
  const uint32_t sub = lane % LPP;
  const uint32_t Hq = uint32_t(a.Hq);
  const uint32_t warp_global = (blockIdx.x * blockDim.x + threadIdx.x) / 32u;
  const uint32_t n_warps = gridDim.x * blockDim.x / 32u;
  for (uint32_t base = warp_global * (32u / LPP); base < n_pairs; base += n_warps * (32u / LPP)) {
    const uint32_t pair = base + lane / LPP;  // (row, head) in the O layout's order
    const bool live = pair < n_pairs;
    const uint32_t row = live ? pair / Hq : 0u;
    const uint32_t h = live ? pair - row * Hq : 0u;
    const uint32_t rb = row / twoC;
    const uint32_t lidx = (rb * Hq + h) * twoC + (row - rb * twoC);   // lse layout
    float m = -INFINITY, l = 0.f;
    float acc[8];
#pragma unroll
    for (int t = 0; t < 8; ++t) acc[t] = 0.f;
    if (live) {
      // parts in groups of four: every load of a group is issued before any arithmetic,
      // so their latencies overlap instead of chaining part after part
      for (int i0 = 0; i0 < a.n; i0 += 4) {
        float li[4];
        uint4 x[4];
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          const int i = i0 + t < a.n ? i0 + t : i0;
          li[t] = i0 + t < a.n ? a.lse[i][lidx] : -INFINITY;
          x[t] = reinterpret_cast<const uint4*>(
              reinterpret_cast<const __nv_bfloat16*>(a.o[i]) + size_t(pair) * HD)[sub];
        }
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          if (li[t] == -INFINITY) continue;      // an empty key set (or no part) adds nothing
          if (li[t] > m) {                       // rescale what was summed against the old max
            const float c = expf(m - li[t]);     // m = -inf at the first live part: c = 0
            l *= c;
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[e] *= c;
            m = li[t];
          }
          const float w = expf(li[t] - m);
          l += w;
          const uint32_t xs[4] = {x[t].x, x[t].y, x[t].z, x[t].w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            acc[2 * e] = fmaf(w, __uint_as_float(xs[e] << 16), acc[2 * e]);
            acc[2 * e + 1] = fmaf(w, __uint_as_float(xs[e] & 0xFFFF0000u), acc[2 * e + 1]);
          }
        }
      }
    }
    __syncwarp();                              // every lane has read its inputs
    if (live) {
      const bool empty = m == -INFINITY;
      const float inv = empty ? 0.f : 1.0f / l;
      uint4 y;
      y.x = pack_bf16x2(acc[0] * inv, acc[1] * inv);
      y.y = pack_bf16x2(acc[2] * inv, acc[3] * inv);
      y.z = pack_bf16x2(acc[4] * inv, acc[5] * inv);
      y.w = pack_bf16x2(acc[6] * inv, acc[7] * inv);
      reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(a.o_out) + size_t(pair) * HD)[sub] = y;
      if (sub == 0) a.lse_out[lidx] = empty ? -INFINITY : m + logf(l);
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
  const int64_t pairs_per_block = 8 * (32 / (HD / 8));
  int64_t blocks = (n_pairs + pairs_per_block - 1) / pairs_per_block;
  if (blocks > int64_t(sms) * 16) blocks = int64_t(sms) * 16;
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
