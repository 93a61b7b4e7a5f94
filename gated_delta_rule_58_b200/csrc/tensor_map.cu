// Host-side TMA descriptors: cuTensorMapEncodeTiled, reached through the runtime's
// driver entry-point lookup so that the library needs no link against libcuda.
#include <mutex>
#include <string>

#include "tensor_map.cuh"

namespace gdn {
namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

gdn_status_t encode_tiled(EncodeTiledFn* fn) {
  static EncodeTiledFn cached = nullptr;
  static std::mutex mu;
  std::lock_guard<std::mutex> lock(mu);
  if (!cached) {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    const cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q);
    if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || f == nullptr)
      return fail(GDN_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
    cached = reinterpret_cast<EncodeTiledFn>(f);
  }
  *fn = cached;
  return GDN_OK;
}

}  // namespace

gdn_status_t make_tensor_map_3d(CUtensorMap* map, CUtensorMapDataType type, const void* base,
                                const uint64_t dims[3], const uint64_t strides[2], const uint32_t box[3],
                                const char* what, CUtensorMapSwizzle swizzle) {
  EncodeTiledFn encode = nullptr;
  const gdn_status_t st = encode_tiled(&encode);
  if (st != GDN_OK) return st;
  const cuuint64_t d[3] = {dims[0], dims[1], dims[2]};
  const cuuint64_t s[2] = {strides[0], strides[1]};
  const cuuint32_t b[3] = {box[0], box[1], box[2]};
  const cuuint32_t e[3] = {1, 1, 1};
  const CUresult r = encode(map, type, 3, const_cast<void*>(base), d, s, b, e, CU_TENSOR_MAP_INTERLEAVE_NONE,
                            swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS)
    return fail(GDN_ERR_CUDA, std::string(what) + ": cuTensorMapEncodeTiled failed (CUresult " +
                                  std::to_string((int)r) + ")");
  return GDN_OK;
}

}  // namespace gdn
