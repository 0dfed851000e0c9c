// Tensor-map construction and device queries shared by the tensor-core
// kernels.  cuTensorMapEncodeTiled is a driver entry point; it is looked up
// through the runtime so the library links against cudart only.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "internal.cuh"

namespace nabla {
namespace {

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    cudaDriverEntryPointQueryResult qr;
    void* p = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &qr) == cudaSuccess &&
        qr == cudaDriverEntryPointSuccess)
      fn = (PFN_cuTensorMapEncodeTiled_v12000)p;
  }
  return fn;
}

bool encode(CUtensorMap* map, CUtensorMapDataType type, int elem, const void* base, const Dims& d, int rows,
            int inner, int box_inner) {
  auto enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {(cuuint64_t)d.D, (cuuint64_t)rows, (cuuint64_t)d.BH()};
  cuuint64_t strides[2] = {(cuuint64_t)d.D * elem, (cuuint64_t)rows * d.D * elem};
  cuuint32_t box[3] = {(cuuint32_t)box_inner, (cuuint32_t)inner, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(map, type, 3, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace

bool make_map_bf16(CUtensorMap* map, const void* base, const Dims& d, int box_rows) {
  return encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, d, d.S, box_rows, 64);
}

bool make_map_pooled_f32(CUtensorMap* map, const float* base, const Dims& d) {
  return encode(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, base, d, d.nb, 128, 32);
}

bool make_map_bf16_rows(CUtensorMap* map, const void* base, int inner, long long rows, int outer, int box_rows) {
  auto enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {(cuuint64_t)inner, (cuuint64_t)rows, (cuuint64_t)outer};
  cuuint64_t strides[2] = {(cuuint64_t)inner * 2, (cuuint64_t)rows * inner * 2};
  cuuint32_t box[3] = {64, (cuuint32_t)box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

int sm_count() {
  static int n = 0;
  if (!n) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
  }
  return n;
}

}  // namespace nabla
