// Host-side construction of TMA tensor maps for [B, N, H, D] bf16 tensors.
// The driver's encoder is fetched once through the runtime's entry-point
// query, so the library needs no link-time dependency on libcuda.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>
#include <mutex>

#include "rtp_internal.h"

namespace rtp {

static PFN_cuTensorMapEncodeTiled_v12000 encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

// Tensor map over x[b, n, h, d] (D = 128 contiguous, element strides sb/sn/sh)
// whose box is 64 elements of D (128 bytes, 128-byte swizzle) x 1 head x
// `box_rows` rows x 1 batch. Out-of-range rows read as zero.
bool make_tmap_bnhd(CUtensorMap* map, const void* ptr, int B, int N, int H, int64_t sb, int64_t sn,
                    int64_t sh, int box_rows) {
  auto fn = encoder();
  if (!fn) return false;
  cuuint64_t dims[4] = {128, (cuuint64_t)H, (cuuint64_t)N, (cuuint64_t)B};
  cuuint64_t strides[3] = {(cuuint64_t)sh * 2, (cuuint64_t)sn * 2, (cuuint64_t)sb * 2};
  // A stride of a size-1 dimension is never used; keep it a valid multiple of 16.
  if (H == 1 && strides[0] == 0) strides[0] = 256;
  if (B == 1 && strides[2] == 0) strides[2] = 256;
  cuuint32_t box[4] = {64, 1, (cuuint32_t)box_rows, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(ptr), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Tensor map over rows 0 .. N-1 of an index x~[b, h, n, 0..16) (bf16; `cap`
// rows per (b, h), contiguous): box of one 32-byte row x `box_rows` rows,
// 32-byte swizzle.
bool make_tmap_index(CUtensorMap* map, const void* ptr, int B, int H, int N, int64_t cap, int box_rows) {
  auto fn = encoder();
  if (!fn) return false;
  cuuint64_t dims[4] = {16, (cuuint64_t)N, (cuuint64_t)H, (cuuint64_t)B};
  cuuint64_t strides[3] = {32, (cuuint64_t)cap * 32, (cuuint64_t)H * cap * 32};
  cuuint32_t box[4] = {16, (cuuint32_t)box_rows, 1, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(ptr), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_32B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace rtp
