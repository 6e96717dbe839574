#include "tmap.h"

#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <mutex>

namespace {
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_once;
std::string g_init_err;

void resolve() {
  void* fn = nullptr;
  cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
  const cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
  if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || fn == nullptr) {
    g_init_err = std::string("cuTensorMapEncodeTiled unavailable: ") + cudaGetErrorString(e);
    return;
  }
  g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
}

bool encode(CUtensorMap* m, CUtensorMapDataType dt, int rank, const void* base, const cuuint64_t* dims,
            const cuuint64_t* strides_bytes, const cuuint32_t* box, std::string& err) {
  if (!g_encode) {
    err = g_init_err.empty() ? "tensor-map encoder not initialised" : g_init_err;
    return false;
  }
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  const CUresult r = g_encode(m, dt, static_cast<cuuint32_t>(rank),
                              const_cast<void*>(base), dims, strides_bytes, box, estr,
                              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    err = "cuTensorMapEncodeTiled failed with CUresult " + std::to_string(static_cast<int>(r));
    return false;
  }
  return true;
}
}  // namespace

bool tmap_init(std::string& err) {
  std::call_once(g_once, resolve);
  if (!g_encode) {
    err = g_init_err;
    return false;
  }
  return true;
}

bool tmap_2d_bf16(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint64_t ld, uint32_t box_rows,
                  std::string& err) {
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {ld * 2};
  const cuuint32_t box[2] = {64, box_rows};
  return encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, dims, strides, box, err);
}

bool tmap_2d_u8(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint64_t ld, uint32_t box_rows,
                std::string& err) {
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {ld};
  const cuuint32_t box[2] = {128, box_rows};
  return encode(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, base, dims, strides, box, err);
}

bool tmap_planes_bf16(CUtensorMap* m, const void* base, uint64_t d, uint64_t rows, uint64_t H, uint64_t slices,
                     std::string& err) {
  const cuuint64_t dims[4] = {d, rows, H, slices};
  const cuuint64_t strides[3] = {d * 2, rows * d * 2, H * rows * d * 2};
  const cuuint32_t box[4] = {64, 128, 1, 1};
  return encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, base, dims, strides, box, err);
}

bool tmap_planes_u8(CUtensorMap* m, const void* base, uint64_t d, uint64_t rows, uint64_t H, uint64_t slices,
                    std::string& err) {
  const cuuint64_t dims[4] = {d, rows, H, slices};
  const cuuint64_t strides[3] = {d, rows * d, H * rows * d};
  const cuuint32_t box[4] = {128, 128, 1, 1};
  return encode(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, base, dims, strides, box, err);
}
