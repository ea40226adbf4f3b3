// Row RMS normalisation for the layer step (pre-attention and pre-MLP norm of
// both flows' rows in one launch). One CTA per row, 16-byte loads, fp32 sums.
#include "common.cuh"
#include "host_util.h"

namespace df {
namespace norm {

constexpr int kThreads = 256;

__global__ void __launch_bounds__(kThreads) rmsnorm_kernel(const __nv_bfloat16* x, int64_t ldx,
                                                           const __nv_bfloat16* gain,
                                                           __nv_bfloat16* y, int64_t ldy, int cols,
                                                           float eps) {
  const int r = blockIdx.x;
  pdl_wait();
  pdl_trigger();
  const uint4* xr = reinterpret_cast<const uint4*>(x + r * ldx);
  const int nvec = cols / 8;
  float ss = 0.f;
  for (int v = threadIdx.x; v < nvec; v += kThreads) {
    const uint4 u = xr[v];
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float a = bf16_bits_to_float(static_cast<uint16_t>(w[k] & 0xffffu));
      const float c = bf16_bits_to_float(static_cast<uint16_t>(w[k] >> 16));
      ss = fmaf(a, a, ss);
      ss = fmaf(c, c, ss);
    }
  }
  __shared__ float red[kThreads / 32];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
  __syncthreads();
  float tot = 0.f;
#pragma unroll
  for (int w = 0; w < kThreads / 32; ++w) tot += red[w];
  const float inv = 1.0f / sqrtf(tot / static_cast<float>(cols) + eps);
  uint4* yr = reinterpret_cast<uint4*>(y + r * ldy);
  const uint4* gr = reinterpret_cast<const uint4*>(gain);
  for (int v = threadIdx.x; v < nvec; v += kThreads) {
    const uint4 u = xr[v];
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
    uint32_t gw[4] = {0x3f803f80u, 0x3f803f80u, 0x3f803f80u, 0x3f803f80u};  // bf16 1.0 pairs
    if (gain) {
      const uint4 gu = gr[v];
      gw[0] = gu.x;
      gw[1] = gu.y;
      gw[2] = gu.z;
      gw[3] = gu.w;
    }
    uint32_t out[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float a = bf16_bits_to_float(static_cast<uint16_t>(w[k] & 0xffffu)) * inv *
                      bf16_bits_to_float(static_cast<uint16_t>(gw[k] & 0xffffu));
      const float c = bf16_bits_to_float(static_cast<uint16_t>(w[k] >> 16)) * inv *
                      bf16_bits_to_float(static_cast<uint16_t>(gw[k] >> 16));
      out[k] = pack_bf16x2(__float2bfloat16_rn(a), __float2bfloat16_rn(c));
    }
    yr[v] = make_uint4(out[0], out[1], out[2], out[3]);
  }
}

}  // namespace norm
}  // namespace df

extern "C" df_status dualflow_rmsnorm(const void* x, int64_t ldx, const void* gain, void* y,
                                      int64_t ldy, int rows, int cols, float eps, void* stream) {
  using namespace df;
  if (!x || !y) return DF_ERR_NULL;
  if (rows < 1 || cols < 1 || rows > 2147483647) return DF_ERR_SHAPE;
  if (cols % 8 != 0) return DF_ERR_UNSUPPORTED;
  const int64_t lx = ldx ? ldx : cols, ly = ldy ? ldy : cols;
  if (lx < cols || ly < cols || !(eps >= 0.f)) return DF_ERR_SHAPE;
  if (lx % 8 != 0 || ly % 8 != 0 || !aligned(x, 16) || !aligned(y, 16) ||
      (gain && !aligned(gain, 16)))
    return DF_ERR_ALIGN;
  if (launch_pdl(norm::rmsnorm_kernel, dim3(rows), dim3(norm::kThreads), 0,
                 static_cast<cudaStream_t>(stream), static_cast<const __nv_bfloat16*>(x), lx,
                 static_cast<const __nv_bfloat16*>(gain), static_cast<__nv_bfloat16*>(y), ly, cols,
                 eps) != cudaSuccess)
    return DF_ERR_CUDA;
  return DF_OK;
}
