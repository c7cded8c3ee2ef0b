// Tensor maps (TMA descriptors) of bf16 and float32 tensors in the 128-byte
// swizzle that the tensor-core operand descriptors expect.
#include <cudaTypedefs.h>

#include <mutex>

#include "hils_common.cuh"

namespace hils {
namespace {

// cuTensorMapEncodeTiled from the driver, looked up once through the runtime.
PFN_cuTensorMapEncodeTiled_v12000 tmap_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

}  // namespace

cudaError_t encode_tmap(CUtensorMap* tm, int dtype, int rank, const void* base,
                        const uint64_t* dims, const uint64_t* strides, const uint32_t* box) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = tmap_encoder();
  if (!enc) return cudaErrorNotSupported;
  cuuint64_t d[5], s[4];
  cuuint32_t b[5], e[5];
  for (int x = 0; x < rank; ++x) {
    d[x] = dims[x];
    b[x] = box[x];
    e[x] = 1;
    if (x + 1 < rank) s[x] = strides[x];
  }
  const CUresult r = enc(tm, dtype == HILS_F32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32
                                               : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                         (cuuint32_t)rank, const_cast<void*>(base), d, s, b, e,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

cudaError_t encode_tmap_bf16(CUtensorMap* tm, int rank, const void* base, const uint64_t* dims,
                             const uint64_t* strides, const uint32_t* box) {
  return encode_tmap(tm, HILS_BF16, rank, base, dims, strides, box);
}

}  // namespace hils
