// zsa_tma_host.h -- host-side construction of TMA tensor maps.
//
// cuTensorMapEncodeTiled is a driver-API call; it is fetched through the runtime's
// cudaGetDriverEntryPoint so the shared library has no link-time dependency on
// libcuda and can be loaded (e.g. to list its symbols) on a machine without a GPU.
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace zsa {

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFn encode_tiled_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// Tensor of `rank` dims (dim 0 innermost, contiguous) with elements of `dtype`; strides
// in BYTES for dims 1..rank-1; box in elements; 128-byte swizzle (box dim 0 must span
// 128 bytes: 64 bf16 or 32 fp32).
inline bool make_map_sw128(CUtensorMap* map, CUtensorMapDataType dtype, const void* base,
                           int rank, const uint64_t* dims, const uint64_t* strides_bytes,
                           const uint32_t* box) {
  EncodeTiledFn fn = encode_tiled_fn();
  if (!fn) return false;
  cuuint64_t gdim[5];
  cuuint64_t gstr[4];
  cuuint32_t bx[5];
  cuuint32_t es[5];
  for (int i = 0; i < rank; ++i) {
    gdim[i] = dims[i];
    bx[i] = box[i];
    es[i] = 1;
  }
  for (int i = 0; i + 1 < rank; ++i) gstr[i] = strides_bytes[i];
  CUresult r = fn(map, dtype, (cuuint32_t)rank, const_cast<void*>(base), gdim, gstr, bx, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

inline bool make_map_bf16_sw128(CUtensorMap* map, const void* base, int rank,
                                const uint64_t* dims, const uint64_t* strides_bytes,
                                const uint32_t* box) {
  return make_map_sw128(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, base, rank, dims, strides_bytes,
                        box);
}

inline bool make_map_f32_sw128(CUtensorMap* map, const void* base, int rank,
                               const uint64_t* dims, const uint64_t* strides_bytes,
                               const uint32_t* box) {
  return make_map_sw128(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, base, rank, dims, strides_bytes,
                        box);
}

}  // namespace zsa
