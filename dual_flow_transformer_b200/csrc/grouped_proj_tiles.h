// Internal interface between the grouped-projection entry point and its
// tile-parallel / cluster split-K plan (grouped_proj_tiles.cu).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace df {
namespace tgemm {

struct Request {
  const void* x;
  int64_t ldx;
  int m_primary, m_aux;
  const void* w;
  int N, K, n_aux;
  void* y;
  int64_t ldy;
  int epilogue;
  const void* coupling;
  const void* residual;
  int64_t ldr;
  int32_t* err;
  cudaStream_t stream;
  void* workspace;  // fp32 partial slots of the cluster split-K reduction
  size_t workspace_bytes;
  // Optional: the projection launched next on the stream (same rows and
  // workspace size); its first k-blocks are prefetched into L2 during this
  // launch's tail. w_next NULL = none.
  const void* w_next;
  int N_next, K_next, epilogue_next;
  // Batched form (batch > 1): `batch` independent projections of the same
  // shape, entry b at x + b*x_bstride, w + b*w_bstride, y + b*y_bstride
  // (elements); the next projection may be batched too.
  int batch;
  int64_t x_bstride, w_bstride, y_bstride;
  int batch_next;
  int64_t w_next_bstride;
};

// Launches the tile plan when it is modelled to beat stream-K on this device.
// Returns 1 when launched, 0 when the caller should use stream-K, -1 on a CUDA
// error. Arguments must already be validated.
int launch_if_better(const Request& r);

// 1 if the tile plan would be used for this shape on the current device with
// a workspace of ws_bytes, else 0.
int planned_launches(int M, int N, int K, int epilogue, size_t ws_bytes, int batch = 1);

}  // namespace tgemm
}  // namespace df
