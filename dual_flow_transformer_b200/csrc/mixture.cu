// Mixture head: the mixed next-token distribution of both flows.
//
// "Sintesi Tecnica: Dual-Flow Transformers", section "Meccanismi Chiave"
// (mixture objective): p_mix = alpha p_primary + (1 - alpha) p_aux, with the
// mixing weight set by the primary distribution's confidence (its collision
// probability) and keeping the primary at least half of the mixture. The map
// from confidence to weight is not printed; this library reads it as
//   alpha = 1/2 + 1/2 * sum_v p1_v^2.
//
// Input: the grouped LM-head projection's logits [2B][V] (primary rows, then
// auxiliary rows). Output: p_mix [B][V] fp32 and alpha [B].
//
// Design (sm_100a, HBM-bound: the logits are read from HBM once and p_mix is
// written once):
//  * one thread-block cluster of S <= 8 CTAs per sequence splits the
//    vocabulary into S slices so that B * S CTAs fill the GPU;
//  * pass 1: each thread keeps online statistics over its elements -- running
//    max m, sum z = sum 2^(x - m) and, for the primary flow, the sum of
//    squares c = sum 2^(2 (x - m)) (x = logit * log2(e)); warps and CTAs merge
//    them by rescaling to the larger max;
//  * the S CTAs exchange their 5 statistics through distributed shared memory
//    and combine them in rank order, so every CTA derives the same alpha;
//  * pass 2 re-reads the slice (an L2 hit: it was just read) and writes
//    p_mix = (alpha / z1) 2^(x1 - m1) + ((1 - alpha) / z2) 2^(x2 - m2) with
//    16-byte stores.
// alpha reads only the primary rows, so it is bit-identical whatever the
// auxiliary logits are (NaN included).
#include <math.h>

#include "common.cuh"
#include "host_util.h"

namespace df {
namespace mix {

constexpr int kThreads = 256;
constexpr int kMaxCluster = 8;
constexpr int kTargetCtas = 148 * 2;
constexpr float kLog2e = 1.4426950408889634f;

struct Params {
  const void* logits;
  int64_t ld;  // logits row stride, elements
  int B, V, chunk;
  float* p_mix;
  int64_t ldp;
  float* alpha;
};

// max that propagates NaN (fmaxf drops it)
__device__ __forceinline__ float max_nan(float a, float b) { return (a != a || a > b) ? a : b; }

// Online statistics of one flow: running max m (log2 domain), z = sum 2^(x-m),
// c = sum 2^(2(x-m)).
struct Stat {
  float m, z, c;
};

__device__ __forceinline__ Stat stat_empty() { return Stat{-INFINITY, 0.f, 0.f}; }

// Merge b into a (rescale both to the larger max). An empty side (m = -inf)
// contributes nothing; NaN maxima propagate.
__device__ __forceinline__ Stat stat_merge(Stat a, Stat b) {
  const float M = max_nan(a.m, b.m);
  if (M == -INFINITY) return a;
  const float sa = (a.m == -INFINITY) ? 0.f : exp2f(a.m - M);
  const float sb = (b.m == -INFINITY) ? 0.f : exp2f(b.m - M);
  return Stat{M, a.z * sa + b.z * sb, a.c * sa * sa + b.c * sb * sb};
}

// Accumulate n values (already scaled by log2 e) into s: one max update per
// group, then the exponentials.
template <int N>
__device__ __forceinline__ void stat_add(Stat& s, const float (&x)[N], bool squares) {
  float gm = x[0];
#pragma unroll
  for (int i = 1; i < N; ++i) gm = max_nan(gm, x[i]);
  const float M = max_nan(s.m, gm);
  if (M == -INFINITY) return;  // all -inf so far: nothing to add
  if (M != s.m) {
    const float r = (s.m == -INFINITY) ? 0.f : exp2f(s.m - M);
    s.z *= r;
    if (squares) s.c *= r * r;
    s.m = M;
  }
#pragma unroll
  for (int i = 0; i < N; ++i) {
    const float e = exp2f(x[i] - M);
    s.z += e;
    if (squares) s.c = fmaf(e, e, s.c);
  }
}

__device__ __forceinline__ Stat stat_shfl_xor(Stat s, int o) {
  return Stat{__shfl_xor_sync(0xffffffffu, s.m, o), __shfl_xor_sync(0xffffffffu, s.z, o),
              __shfl_xor_sync(0xffffffffu, s.c, o)};
}

// 8 consecutive logits of a row, scaled by log2 e.
template <typename T>
__device__ __forceinline__ void load8(const T* src, float (&x)[8]);
template <>
__device__ __forceinline__ void load8<float>(const float* src, float (&x)[8]) {
  const float4 a = reinterpret_cast<const float4*>(src)[0];
  const float4 b = reinterpret_cast<const float4*>(src)[1];
  x[0] = a.x * kLog2e; x[1] = a.y * kLog2e; x[2] = a.z * kLog2e; x[3] = a.w * kLog2e;
  x[4] = b.x * kLog2e; x[5] = b.y * kLog2e; x[6] = b.z * kLog2e; x[7] = b.w * kLog2e;
}
template <>
__device__ __forceinline__ void load8<__nv_bfloat16>(const __nv_bfloat16* src, float (&x)[8]) {
  const uint4 u = *reinterpret_cast<const uint4*>(src);
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    x[2 * k] = bf16_bits_to_float(static_cast<uint16_t>(w[k] & 0xffffu)) * kLog2e;
    x[2 * k + 1] = bf16_bits_to_float(static_cast<uint16_t>(w[k] >> 16)) * kLog2e;
  }
}

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                   : "memory");
}
__device__ __forceinline__ float ld_cluster_f32(const float* local, uint32_t rank) {
  uint32_t addr;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(addr) : "r"(smem_u32(local)), "r"(rank));
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
  return v;
}

template <typename T>
__global__ void __launch_bounds__(kThreads) mixture_kernel(const Params p) {
  __shared__ Stat warp_st[2][kThreads / 32];
  __shared__ float cta_st[5];  // this CTA's (m1, z1, c1, m2, z2), read by the cluster
  const int b = blockIdx.y;
  const uint32_t rank = cluster_rank();
  const int S = static_cast<int>(gridDim.x);
  const int v0 = static_cast<int>(rank) * p.chunk;
  const int v1 = min(p.V, v0 + p.chunk);
  const T* row1 = static_cast<const T*>(p.logits) + static_cast<int64_t>(b) * p.ld;
  const T* row2 = static_cast<const T*>(p.logits) + static_cast<int64_t>(p.B + b) * p.ld;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  pdl_wait();
  pdl_trigger();

  // ---- pass 1: statistics of this slice
  Stat s1 = stat_empty(), s2 = stat_empty();
  for (int v = v0 + tid * 8; v < v1; v += kThreads * 8) {
    float x1[8], x2[8];
    load8<T>(row1 + v, x1);
    load8<T>(row2 + v, x2);
    stat_add<8>(s1, x1, true);
    stat_add<8>(s2, x2, false);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    s1 = stat_merge(s1, stat_shfl_xor(s1, o));
    s2 = stat_merge(s2, stat_shfl_xor(s2, o));
  }
  if (lane == 0) {
    warp_st[0][warp] = s1;
    warp_st[1][warp] = s2;
  }
  __syncthreads();
  if (tid == 0) {
    Stat a = warp_st[0][0], c = warp_st[1][0];
    for (int w = 1; w < kThreads / 32; ++w) {
      a = stat_merge(a, warp_st[0][w]);
      c = stat_merge(c, warp_st[1][w]);
    }
    cta_st[0] = a.m;
    cta_st[1] = a.z;
    cta_st[2] = a.c;
    cta_st[3] = c.m;
    cta_st[4] = c.z;
  }
  // ---- combine the cluster's statistics in rank order (same result everywhere)
  cluster_sync();
  __shared__ float fin[5];
  if (tid == 0) {
    Stat a = stat_empty(), c = stat_empty();
    for (int q = 0; q < S; ++q) {
      const Stat qa{ld_cluster_f32(&cta_st[0], q), ld_cluster_f32(&cta_st[1], q),
                    ld_cluster_f32(&cta_st[2], q)};
      const Stat qc{ld_cluster_f32(&cta_st[3], q), ld_cluster_f32(&cta_st[4], q), 0.f};
      a = stat_merge(a, qa);
      c = stat_merge(c, qc);
    }
    const float alpha = 0.5f + 0.5f * (a.c / (a.z * a.z));
    fin[0] = a.m;
    fin[1] = alpha / a.z;
    fin[2] = c.m;
    fin[3] = (1.0f - alpha) / c.z;
    fin[4] = alpha;
    if (rank == 0 && p.alpha != nullptr) p.alpha[b] = alpha;
  }
  cluster_sync();  // no CTA leaves while others may still read its statistics
  const float m1 = fin[0], k1 = fin[1], m2 = fin[2], k2 = fin[3];

  // ---- pass 2: p_mix of this slice
  float* out = p.p_mix + static_cast<int64_t>(b) * p.ldp;
  for (int v = v0 + tid * 8; v < v1; v += kThreads * 8) {
    float x1[8], x2[8], o[8];
    load8<T>(row1 + v, x1);
    load8<T>(row2 + v, x2);
#pragma unroll
    for (int i = 0; i < 8; ++i) o[i] = k1 * exp2f(x1[i] - m1) + k2 * exp2f(x2[i] - m2);
    reinterpret_cast<float4*>(out + v)[0] = make_float4(o[0], o[1], o[2], o[3]);
    reinterpret_cast<float4*>(out + v)[1] = make_float4(o[4], o[5], o[6], o[7]);
  }
}

// Slices per sequence: enough CTAs to fill two per SM, at most 8 (a portable
// cluster), and no slice shorter than 4096 logits.
inline int slices(int B, int V) {
  int s = static_cast<int>(ceil_div(kTargetCtas, B));
  const int by_len = static_cast<int>(ceil_div(V, 4096));
  if (s > by_len) s = by_len;
  if (s > kMaxCluster) s = kMaxCluster;
  return s < 1 ? 1 : s;
}

}  // namespace mix
}  // namespace df

extern "C" df_status dualflow_mixture_head(const void* logits, int64_t ld, int B, int V, int dtype,
                                           float* p_mix, int64_t ldp, float* alpha,
                                           void* stream) {
  using namespace df;
  if (!logits || !p_mix) return DF_ERR_NULL;
  if (B < 1 || V < 1 || B > 65535) return DF_ERR_SHAPE;
  if (dtype != DF_FP32 && dtype != DF_BF16) return DF_ERR_UNSUPPORTED;
  if (V % 8 != 0) return DF_ERR_UNSUPPORTED;
  const int64_t l = ld ? ld : V, lp = ldp ? ldp : V;
  if (l < V || lp < V) return DF_ERR_SHAPE;
  if (l % 8 != 0 || lp % 4 != 0 || !aligned(logits, 16) || !aligned(p_mix, 16) ||
      (alpha && !aligned(alpha, 4)))
    return DF_ERR_ALIGN;
  mix::Params p;
  p.logits = logits;
  p.ld = l;
  p.B = B;
  p.V = V;
  const int S = mix::slices(B, V);
  p.chunk = static_cast<int>(round_up(ceil_div(V, S), 8));
  p.p_mix = p_mix;
  p.ldp = lp;
  p.alpha = alpha;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(S, B);
  cfg.blockDim = dim3(mix::kThreads);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = static_cast<cudaStream_t>(stream);
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = S;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  cudaError_t e = (dtype == DF_BF16)
                      ? cudaLaunchKernelEx(&cfg, mix::mixture_kernel<__nv_bfloat16>, p)
                      : cudaLaunchKernelEx(&cfg, mix::mixture_kernel<float>, p);
  return e == cudaSuccess ? DF_OK : DF_ERR_CUDA;
}

extern "C" int dualflow_mixture_head_slices(int B, int V) {
  if (B < 1 || V < 1) return 0;
  return df::mix::slices(B, V);
}
