// zsa_permute.cu -- K5: natural <-> zigzag shard-major copy of a row tensor.
//
// The zigzag partition ("Folding Tensor and Sequence Parallelism" summary, section 2,
// attention layer) gives shard r the chunks r and 2D-1-r of C = S/(2D) positions.  A
// tensor with one row of H*d bf16 values per position exists in two orders:
//   natural      [B][S][H][d]          (position order),
//   shard-major  [D'][B][2C][H][d]     (shard r's chunk r, then its chunk 2D-1-r),
// D' the shards of the problem's range.  Both orders store each chunk of one batch as
// C contiguous rows, so the permutation is 2 * D' * B copies of C*H*d*2 bytes, chunk
// block cb = (r_local * B + b) * 2 + half sitting at cb * chunk in the shard-major
// tensor and at (b * 2D + chunk index) * chunk in the natural one.
//
// HBM-bound: every byte is read once and written once.  grid.y enumerates the chunk
// blocks (no index division per element); grid.x cuts each block into contiguous spans,
// sized so the whole grid is a few waves of 148 SMs; every thread moves 16-byte words
// with four loads in flight before their stores.  Loads and stores are streaming
// (evict-first): the copy is used once and should not displace L2 residents.
#include <cuda_runtime.h>

#include "zsa_kernels.h"

namespace zsa {
namespace {

constexpr int kPermThreads = 256;
constexpr int kPermUnroll = 4;

__global__ void __launch_bounds__(kPermThreads) zsa_permute_kernel(const __grid_constant__ PermuteArgs a,
                                                                   uint32_t span) {
  const uint32_t cb = blockIdx.y;                      // chunk block
  const uint32_t half = cb & 1u;
  const uint32_t rb = cb >> 1;                         // r_local * B + b
  const uint32_t r = uint32_t(a.shard_begin) + rb / uint32_t(a.B);
  const uint32_t b = rb % uint32_t(a.B);
  const uint32_t c = half == 0 ? r : 2u * uint32_t(a.D) - 1u - r;   // chunk index
  const int64_t smj = int64_t(cb) * a.chunk_words;
  const int64_t nat = (int64_t(b) * 2 * a.D + c) * a.chunk_words;
  const uint4* src = reinterpret_cast<const uint4*>(a.src) + (a.to_shard_major ? nat : smj);
  uint4* dst = reinterpret_cast<uint4*>(a.dst) + (a.to_shard_major ? smj : nat);
  const int64_t begin = int64_t(blockIdx.x) * span;
  int64_t end = begin + span;
  if (end > a.chunk_words) end = a.chunk_words;
  constexpr int64_t step = int64_t(kPermThreads) * kPermUnroll;
  int64_t w = begin + threadIdx.x;
  for (; w + (kPermUnroll - 1) * kPermThreads < end; w += step) {
    uint4 x[kPermUnroll];
#pragma unroll
    for (int u = 0; u < kPermUnroll; ++u) x[u] = __ldcs(src + w + u * kPermThreads);
#pragma unroll
    for (int u = 0; u < kPermUnroll; ++u) __stcs(dst + w + u * kPermThreads, x[u]);
  }
  for (; w < end; w += kPermThreads) __stcs(dst + w, __ldcs(src + w));
}

}  // namespace

int launch_permute(const PermuteArgs& a, cudaStream_t stream) {
  const int64_t blocks = 2 * int64_t(a.shard_count) * a.B;
  if (blocks <= 0 || a.chunk_words <= 0) return int(cudaSuccess);
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  // about 8 CTAs per SM in total, each span a whole number of unrolled steps
  const int64_t step = int64_t(kPermThreads) * kPermUnroll;
  int64_t per_block = (int64_t(sms) * 8 + blocks - 1) / blocks;
  int64_t span = (a.chunk_words + per_block - 1) / per_block;
  span = (span + step - 1) / step * step;
  per_block = (a.chunk_words + span - 1) / span;
  const TraceEvents tr = trace_events(6);
  if (tr.begin) cudaEventRecord(tr.begin, stream);
  zsa_permute_kernel<<<dim3(unsigned(per_block), unsigned(blocks)), kPermThreads, 0, stream>>>(
      a, uint32_t(span));
  const cudaError_t e = cudaGetLastError();
  if (tr.end) cudaEventRecord(tr.end, stream);
  return int(e);
}

}  // namespace zsa
