// ABI-wide host code: version, status strings, tensor-map encoding through the
// driver entry point, device properties.
#include <mutex>

#include <cudaTypedefs.h>

#include "common.cuh"
#include "host_util.h"

namespace df {

namespace {
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

void load_encode() {
  void* fn = nullptr;
  cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
  if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault,
                                       &q) == cudaSuccess &&
      q == cudaDriverEntryPointSuccess) {
    g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  }
}
}  // namespace

bool encode_tmap_bf16_2d(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                         uint64_t row_pitch_bytes, uint32_t box_rows, uint32_t box_cols) {
  std::call_once(g_encode_once, load_encode);
  if (!g_encode) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {row_pitch_bytes};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t elem_strides[2] = {1, 1};
  CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims,
                        strides, box, elem_strides, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool encode_tmap_bf16_3d(CUtensorMap* map, const void* base, uint64_t batch, uint64_t rows,
                         uint64_t cols, uint64_t row_pitch_bytes, uint64_t batch_pitch_bytes,
                         uint32_t box_rows, uint32_t box_cols) {
  std::call_once(g_encode_once, load_encode);
  if (!g_encode) return false;
  cuuint64_t dims[3] = {cols, rows, batch};
  cuuint64_t strides[2] = {row_pitch_bytes, batch_pitch_bytes};
  cuuint32_t box[3] = {box_cols, box_rows, 1};
  cuuint32_t elem_strides[3] = {1, 1, 1};
  CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims,
                        strides, box, elem_strides, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool encode_tmap_bf16_3d_box(CUtensorMap* map, const void* base, const uint64_t dims[3],
                             const uint64_t strides_bytes[2], const uint32_t box[3]) {
  std::call_once(g_encode_once, load_encode);
  if (!g_encode) return false;
  cuuint64_t gdims[3] = {dims[0], dims[1], dims[2]};
  cuuint64_t gstrides[2] = {strides_bytes[0], strides_bytes[1]};
  cuuint32_t gbox[3] = {box[0], box[1], box[2]};
  cuuint32_t elem_strides[3] = {1, 1, 1};
  CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), gdims,
                        gstrides, gbox, elem_strides, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool encode_tmap_f32_3d_box(CUtensorMap* map, const void* base, const uint64_t dims[3],
                            const uint64_t strides_bytes[2], const uint32_t box[3]) {
  std::call_once(g_encode_once, load_encode);
  if (!g_encode) return false;
  cuuint64_t gdims[3] = {dims[0], dims[1], dims[2]};
  cuuint64_t gstrides[2] = {strides_bytes[0], strides_bytes[1]};
  cuuint32_t gbox[3] = {box[0], box[1], box[2]};
  cuuint32_t elem_strides[3] = {1, 1, 1};
  CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<void*>(base), gdims,
                        gstrides, gbox, elem_strides, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

int device_sm_count() {
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (cached[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
    cached[dev] = n;
  }
  return cached[dev];
}

}  // namespace df

extern "C" int dualflow_abi_version(void) { return 1; }

extern "C" const char* dualflow_status_string(int status) {
  switch (status) {
    case DF_OK: return "DF_OK";
    case DF_ERR_NULL: return "DF_ERR_NULL: a required pointer is NULL";
    case DF_ERR_SHAPE: return "DF_ERR_SHAPE: sizes inconsistent or out of range";
    case DF_ERR_UNSUPPORTED: return "DF_ERR_UNSUPPORTED: request not implemented by this build";
    case DF_ERR_WORKSPACE: return "DF_ERR_WORKSPACE: workspace missing, too small or misaligned";
    case DF_ERR_ALIGN: return "DF_ERR_ALIGN: pointer or stride misaligned";
    case DF_ERR_CUDA: return "DF_ERR_CUDA: a CUDA call or kernel launch failed";
    default: return "unknown dualflow status";
  }
}

// ------------------------------------------------------------------ failure-detection self-test

namespace df {

// One CTA of one warp waits, with the bounded waits every kernel of this
// library uses (one thread, then the whole warp), on an mbarrier that nothing
// ever arrives on. Each wait gives up after kWaitLimitCycles and the kernel
// records DF_DEVERR_TIMEOUT and returns normally.
__global__ void __launch_bounds__(32) wait_timeout_selftest_kernel(int32_t* err) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_barrier_init();
  }
  __syncwarp();
  if (threadIdx.x == 0 && !mbar_wait(&bar, 0)) set_err(err, DF_DEVERR_TIMEOUT);
  __syncwarp();
  const bool ok = mbar_wait_warp(&bar, 0);
  if (!ok && threadIdx.x == 0) set_err(err, DF_DEVERR_TIMEOUT);
}

}  // namespace df

extern "C" df_status dualflow_selftest_wait_timeout(int32_t* err_flag, void* stream) {
  if (err_flag == nullptr) return DF_ERR_NULL;
  df::wait_timeout_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(err_flag);
  return cudaGetLastError() == cudaSuccess ? DF_OK : DF_ERR_CUDA;
}
