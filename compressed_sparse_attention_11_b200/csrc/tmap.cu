// Host-side helpers: TMA tensor-map encoding through the driver entry point
// (no link-time dependency on libcuda) and the device's SM count.
#include <mutex>

#include "launch.h"
#include "sm100.cuh"

namespace csa {

namespace {
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;
std::once_flag g_once;

void resolve() {
  void* fn = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) ==
          cudaSuccess &&
      q == cudaDriverEntryPointSuccess)
    g_encode = reinterpret_cast<EncodeTiledFn>(fn);
}
}  // namespace

bool make_tmap_3d(CUtensorMap* map, const void* base, int elem_bytes, uint64_t x, uint64_t y,
                  uint64_t z, uint64_t stride_y_bytes, uint64_t stride_z_bytes, uint32_t box_x,
                  uint32_t box_y) {
  std::call_once(g_once, resolve);
  if (!g_encode) return false;
  const cuuint64_t dims[3] = {x, y, z};
  const cuuint64_t strides[2] = {stride_y_bytes, stride_z_bytes};
  const cuuint32_t box[3] = {box_x, box_y, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUtensorMapDataType dt =
      elem_bytes == 1 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  CUresult r = g_encode(map, dt, 3, const_cast<void*>(base), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

int sm_count() {
  constexpr int kMaxDev = 64;
  static int counts[kMaxDev] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) dev = 0;
  if (counts[dev] <= 0) {
    int count = 0;
    cudaDeviceGetAttribute(&count, cudaDevAttrMultiProcessorCount, dev);
    counts[dev] = count > 0 ? count : 148;
  }
  return counts[dev];
}

}  // namespace csa
