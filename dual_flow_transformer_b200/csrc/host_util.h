// Host-side helpers shared by the ABI entry points: tensor-map encoding via the
// driver entry point (no link-time dependency on libcuda, so the library loads
// on machines without a GPU driver), and small arithmetic helpers.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>
#include <utility>
#include <vector>

namespace df {

inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }
inline size_t round_up(size_t a, size_t m) { return (a + m - 1) / m * m; }
inline bool aligned(const void* p, uintptr_t n) {
  return (reinterpret_cast<uintptr_t>(p) & (n - 1)) == 0;
}

// Encode a 2-D row-major bf16 tensor map: `rows` rows of `cols` elements with a
// row pitch of `row_pitch_bytes`, box = box_rows x box_cols, 128-byte swizzle.
// Returns false if the driver entry point is unavailable or encoding fails.
bool encode_tmap_bf16_2d(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                         uint64_t row_pitch_bytes, uint32_t box_rows, uint32_t box_cols);

// 3-D variant: `batch` matrices of [rows][cols], batch_pitch_bytes apart
// (a multiple of 16); boxes of [box_rows][box_cols] in one matrix.
bool encode_tmap_bf16_3d(CUtensorMap* map, const void* base, uint64_t batch, uint64_t rows,
                         uint64_t cols, uint64_t row_pitch_bytes, uint64_t batch_pitch_bytes,
                         uint32_t box_rows, uint32_t box_cols);

// General 3-D tensor map (128-byte swizzle): dims[0] contiguous elements,
// dims[1], dims[2] at the given byte strides (multiples of 16, in any
// order), box[0..2] elements per dimension. The box lands in shared memory
// dimension 0 fastest, then 1, then 2.
bool encode_tmap_bf16_3d_box(CUtensorMap* map, const void* base, const uint64_t dims[3],
                             const uint64_t strides_bytes[2], const uint32_t box[3]);

// The same for fp32 elements (box[0] * 4 bytes <= 128 with the swizzle).
bool encode_tmap_f32_3d_box(CUtensorMap* map, const void* base, const uint64_t dims[3],
                            const uint64_t strides_bytes[2], const uint32_t box[3]);

// Opt `kernel` into `bytes` of dynamic shared memory on the current device.
// The attribute belongs to the device, so it is set once per (kernel,
// device) pair; later calls only look the pair up.
inline cudaError_t ensure_dynamic_smem(const void* kernel, size_t bytes) {
  static std::mutex mu;
  static std::vector<std::pair<const void*, int>> done;
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(mu);
  for (const auto& d : done)
    if (d.first == kernel && d.second == dev) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(bytes));
  if (e == cudaSuccess) done.emplace_back(kernel, dev);
  return e;
}

// Streaming-multiprocessor count of the current device (cached per device).
int device_sm_count();

// Launch with programmatic stream serialization (the kernel may begin while
// the previous kernel on the stream drains; it synchronises with pdl_wait()).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t stream, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

}  // namespace df
