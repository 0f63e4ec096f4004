// Host-side runtime helpers shared by the device entry points: the device
// check and TMA tensor-map encoding.  The driver's encoder is reached through
// the runtime's entry-point query, so the library does not link libcuda and
// loads on hosts without a GPU driver (where every device call then fails
// with VARK_E_DEVICE / VARK_E_CUDA instead of at load time).
#include <cudaTypedefs.h>

#include <mutex>

#include "vark_common.cuh"

namespace vark {

int check_device_sm100() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return VARK_E_DEVICE;
  }
  int major = 0, minor = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) {
    cudaGetLastError();
    return VARK_E_DEVICE;
  }
  return (major == 10 && minor == 0) ? VARK_OK : VARK_E_DEVICE;
}

static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    else
      cudaGetLastError();
  });
  return fn;
}

int encode_bf16_map(CUtensorMap* map, const void* base, int rank, const uint64_t* dims,
                    const uint64_t* strides_bytes, uint32_t box_rows) {
  auto fn = encode_fn();
  if (fn == nullptr) return VARK_E_CUDA;
  cuuint64_t gdim[5];
  cuuint64_t gstride[4];
  cuuint32_t box[5];
  cuuint32_t estride[5];
  for (int i = 0; i < rank; ++i) {
    gdim[i] = dims[i];
    estride[i] = 1;
    box[i] = (i == 0) ? 64u : (i == 1 ? box_rows : 1u);
  }
  for (int i = 0; i < rank - 1; ++i) gstride[i] = strides_bytes[i];
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, cuuint32_t(rank), const_cast<void*>(base), gdim, gstride,
                  box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? VARK_OK : VARK_E_CUDA;
}

}  // namespace vark
