// tma_host.h -- host-side construction of TMA tensor maps (cuTensorMapEncodeTiled),
// fetched through the runtime's driver entry-point query so the library does not
// link libcuda directly.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>
#include <cstdint>

namespace nsa {

inline PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess) {
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
  }
  return fn;
}

// Tensor map over a row-major bf16 tensor viewed as [n2][n1][n0] (n0 contiguous),
// with byte strides s1 (between consecutive index-1 entries) and s2 (index 2).
// Box (b0, b1, b2); b0 * 2 bytes must be <= 128 for the 128-byte swizzle.
// Out-of-range box elements read as zero. Returns false if the encoder rejects it.
inline bool make_tmap_16bit_3d(CUtensorMap* map, CUtensorMapDataType dtype, const void* base, uint64_t n0,
                               uint64_t n1, uint64_t n2, uint64_t s1, uint64_t s2, uint32_t b0, uint32_t b1,
                               uint32_t b2) {
  auto enc = tensor_map_encoder();
  if (enc == nullptr) return false;
  cuuint64_t dims[3] = {n0, n1, n2};
  cuuint64_t strides[2] = {s1, s2};
  cuuint32_t box[3] = {b0, b1, b2};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(map, dtype, 3, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}
inline bool make_tmap_bf16_3d(CUtensorMap* map, const void* base, uint64_t n0, uint64_t n1, uint64_t n2,
                              uint64_t s1, uint64_t s2, uint32_t b0, uint32_t b1, uint32_t b2) {
  return make_tmap_16bit_3d(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, base, n0, n1, n2, s1, s2, b0, b1, b2);
}
inline bool make_tmap_f16_3d(CUtensorMap* map, const void* base, uint64_t n0, uint64_t n1, uint64_t n2,
                             uint64_t s1, uint64_t s2, uint32_t b0, uint32_t b1, uint32_t b2) {
  return make_tmap_16bit_3d(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, base, n0, n1, n2, s1, s2, b0, b1, b2);
}

}  // namespace nsa
