// Host-side construction of TMA tensor maps (CUtensorMap) for bf16 tensors.
// The driver's cuTensorMapEncodeTiled is reached through the runtime's
// entry-point query, so the library needs no link-time dependency on libcuda.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cstdint>

namespace pkv {

inline PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    else
      cudaGetLastError();
  }
  return fn;
}

// 2-D bf16 tensor [rows][cols] with a row pitch of `pitch_bytes` (a multiple of
// 16), read in boxes of box_cols x box_rows (box_cols * 2 <= 128 bytes) with the
// 128-byte swizzle the UMMA SW128 descriptors expect; rows past the end read
// as zeros. Returns false if the driver rejects the map.
inline bool make_map_2d(CUtensorMap* m, const void* base, int64_t cols, int64_t rows, int64_t pitch_bytes,
                        int box_cols, int box_rows) {
  auto fn = tensor_map_encoder();
  if (!fn || rows <= 0 || cols <= 0) return false;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)pitch_bytes};
  cuuint32_t box[2] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace pkv
