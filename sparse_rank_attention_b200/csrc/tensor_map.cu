// Host-side TMA descriptors of the activation tensors ([B, N, H*d], row-major), built
// with the driver's cuTensorMapEncodeTiled obtained through the runtime (no link-time
// dependency on libcuda).
#include <cuda.h>
#include <cudaTypedefs.h>

#include "rola_internal.cuh"

namespace rola {
namespace {

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

}  // namespace

// [B, N, H*d] activation tensor as a 3D map with [box_rows tokens x 128 bytes] boxes (64
// channels of a 16-bit type, 128 of an 8-bit one); rows past N read as zeros.
bool make_act_map(CUtensorMap* m, CUtensorMapDataType dt, uint32_t el_bytes, const void* ptr, const Dims& dm,
                  CUtensorMapSwizzle sw, uint32_t box_rows) {
  auto enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t HD = (cuuint64_t)dm.H * dm.d;
  cuuint64_t dims[3] = {HD, (cuuint64_t)dm.N, (cuuint64_t)dm.B};
  cuuint64_t strides[2] = {HD * el_bytes, HD * el_bytes * (cuuint64_t)dm.N};
  cuuint32_t box[3] = {128 / el_bytes, box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, dt, 3, const_cast<void*>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// A [d2][d1][d0] tensor (d0 contiguous) with [box1 x box0] boxes; rows past d1 read as zeros
// and are clipped on stores.  The row pitch d0 * el_bytes must be a multiple of 16 bytes.
bool make_map_3d(CUtensorMap* m, CUtensorMapDataType dt, uint32_t el_bytes, const void* ptr, uint64_t d0,
                 uint64_t d1, uint64_t d2, uint32_t box0, uint32_t box1, CUtensorMapSwizzle sw) {
  auto enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {d0, d1, d2};
  cuuint64_t strides[2] = {d0 * el_bytes, d0 * el_bytes * d1};
  cuuint32_t box[3] = {box0, box1, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, dt, 3, const_cast<void*>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace rola
