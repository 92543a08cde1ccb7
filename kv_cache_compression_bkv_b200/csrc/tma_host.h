// tma_host.h -- host side of TMA: the driver's tensor-map encoder, obtained
// through the runtime (so the library needs no link to libcuda), and a helper
// for the row-major 2-D bf16 tensors the kernels stream.
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <mutex>

namespace bkv {

inline PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// A [rows][128] bf16 tensor read in boxes of 64 columns x box_rows rows with
// the 128-byte swizzle (rows past the end read as zero).
inline bool make_bf16_rows_map(CUtensorMap *map, const void *base, unsigned long long rows,
                               int box_rows) {
  auto encode = tensor_map_encoder();
  if (!encode || rows == 0) return false;
  cuuint64_t dims[2] = {128u, static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {256u};
  cuuint32_t box[2] = {64u, static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1u, 1u};
  return encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides,
                box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace bkv
