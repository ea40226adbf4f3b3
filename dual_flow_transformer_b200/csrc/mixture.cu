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
//  * pass 1: per CTA, the maximum m of each row's slice, then z = sum 2^(x - m)
//    and, for the primary flow, the sum of squares c = sum 2^(2 (x - m))
//    (x = logit * log2(e)); the slice stays in registers as packed bf16
//    between the passes (slices longer than 8192 logits stream twice, with
//    online statistics); CTAs merge by rescaling to the larger max;
//  * the S CTAs exchange their 5 statistics through distributed shared memory
//    (one remote load per thread) and combine them in rank order, so every
//    CTA derives the same alpha;
//  * pass 2 writes p_mix = (alpha / z1) 2^(x1 - m1) + ((1 - alpha) / z2)
//    2^(x2 - m2) with 16-byte stores, from registers when each thread holds
//    at most 4 vectors of 8 logits per row, else re-reading the slice (an L2
//    hit: it was just read).
// alpha reads only the primary rows, so it is bit-identical whatever the
// auxiliary logits are (NaN included).
#include <math.h>

#include "common.cuh"
#include "host_util.h"

namespace df {
namespace mix {

constexpr int kThreads = 256;
constexpr int kMaxCluster = 8;
constexpr int kTargetCtas = 148 * 4;
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
__device__ __forceinline__ float ld_cluster_f32(const float* local, uint32_t rank) {
  uint32_t addr;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(addr) : "r"(smem_u32(local)), "r"(rank));
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
  return v;
}

__device__ __forceinline__ void cluster_arrive() {
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() {
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// 8 consecutive logits kept in their storage type (bf16: one 16-byte vector
// in 4 registers), decoded to the log2 domain on use.
template <typename T>
struct Raw8;
template <>
struct Raw8<__nv_bfloat16> {
  uint4 u;
  __device__ __forceinline__ void load(const __nv_bfloat16* src) {
    u = *reinterpret_cast<const uint4*>(src);
  }
  __device__ __forceinline__ float get(int i) const {
    const uint32_t w = (i < 2) ? u.x : (i < 4) ? u.y : (i < 6) ? u.z : u.w;
    return bf16_bits_to_float(static_cast<uint16_t>((i & 1) ? (w >> 16) : (w & 0xffffu))) * kLog2e;
  }
};
template <>
struct Raw8<float> {
  float4 a, b;
  __device__ __forceinline__ void load(const float* src) {
    a = reinterpret_cast<const float4*>(src)[0];
    b = reinterpret_cast<const float4*>(src)[1];
  }
  __device__ __forceinline__ float get(int i) const {
    const float v = (i == 0) ? a.x : (i == 1) ? a.y : (i == 2) ? a.z : (i == 3) ? a.w
                  : (i == 4) ? b.x : (i == 5) ? b.y : (i == 6) ? b.z : b.w;
    return v * kLog2e;
  }
};

// Vectors of 8 logits per row held in registers by each thread when the slice
// is short enough (every CTA of the launch resident at once); longer slices
// take the streaming path, which reads the slice twice.
constexpr int kRegVecs = 4;

__device__ __forceinline__ float warp_max_nan(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = max_nan(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

template <typename T>
__global__ void __launch_bounds__(kThreads) mixture_kernel(const Params p) {
  constexpr int kWarps = kThreads / 32;
  __shared__ float red[5][kWarps];
  __shared__ float cta_st[5];                 // this CTA's (m1, z1, c1, m2, z2)
  __shared__ float all_st[kMaxCluster][5];    // every rank's, gathered in one round trip
  __shared__ float fin[4];
  const int b = blockIdx.y;
  const uint32_t rank = cluster_rank();
  const int S = static_cast<int>(gridDim.x);
  const int v0 = static_cast<int>(rank) * p.chunk;
  const int v1 = min(p.V, v0 + p.chunk);
  const T* row1 = static_cast<const T*>(p.logits) + static_cast<int64_t>(b) * p.ld;
  const T* row2 = static_cast<const T*>(p.logits) + static_cast<int64_t>(p.B + b) * p.ld;
  float* out = p.p_mix + static_cast<int64_t>(b) * p.ldp;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const bool in_regs = (v1 - v0) <= kRegVecs * kThreads * 8;
  pdl_wait();
  pdl_trigger();

  float m1 = -INFINITY, m2 = -INFINITY;  // this CTA's maxima (after the first reduction)
  float z1 = 0.f, c1 = 0.f, z2 = 0.f;
  Raw8<T> r1[kRegVecs], r2[kRegVecs];
  if (in_regs) {
#pragma unroll
    for (int it = 0; it < kRegVecs; ++it) {  // every load issued before any use
      const int v = v0 + (it * kThreads + tid) * 8;
      if (v < v1) {
        r1[it].load(row1 + v);
        r2[it].load(row2 + v);
      }
    }
    // local maxima
#pragma unroll
    for (int it = 0; it < kRegVecs; ++it) {
      if (v0 + (it * kThreads + tid) * 8 < v1) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          m1 = max_nan(m1, r1[it].get(i));
          m2 = max_nan(m2, r2[it].get(i));
        }
      }
    }
    m1 = warp_max_nan(m1);
    m2 = warp_max_nan(m2);
    if (lane == 0) {
      red[0][warp] = m1;
      red[1][warp] = m2;
    }
    __syncthreads();
    m1 = red[0][0];
    m2 = red[1][0];
#pragma unroll
    for (int w = 1; w < kWarps; ++w) {
      m1 = max_nan(m1, red[0][w]);
      m2 = max_nan(m2, red[1][w]);
    }
    // sums against the CTA maxima (an all -inf slice contributes nothing)
    const float u1 = (m1 == -INFINITY) ? 0.f : m1, u2 = (m2 == -INFINITY) ? 0.f : m2;
#pragma unroll
    for (int it = 0; it < kRegVecs; ++it) {
      if (v0 + (it * kThreads + tid) * 8 < v1) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const float e1 = exp2f(r1[it].get(i) - u1);
          z1 += e1;
          c1 = fmaf(e1, e1, c1);
          z2 += exp2f(r2[it].get(i) - u2);
        }
      }
    }
  } else {
    // streaming: online statistics with rescaling, two vectors per step
    Stat s1 = stat_empty(), s2 = stat_empty();
    for (int v = v0 + tid * 8; v < v1; v += 2 * kThreads * 8) {
      float x1[8], x2[8], y1[8], y2[8];
      const int w = v + kThreads * 8;
      load8<T>(row1 + v, x1);
      load8<T>(row2 + v, x2);
      if (w < v1) {
        load8<T>(row1 + w, y1);
        load8<T>(row2 + w, y2);
      }
      stat_add<8>(s1, x1, true);
      stat_add<8>(s2, x2, false);
      if (w < v1) {
        stat_add<8>(s1, y1, true);
        stat_add<8>(s2, y2, false);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      s1 = stat_merge(s1, stat_shfl_xor(s1, o));
      s2 = stat_merge(s2, stat_shfl_xor(s2, o));
    }
    if (lane == 0) {
      red[0][warp] = s1.m;
      red[1][warp] = s2.m;
    }
    __syncthreads();
    m1 = red[0][0];
    m2 = red[1][0];
#pragma unroll
    for (int w = 1; w < kWarps; ++w) {
      m1 = max_nan(m1, red[0][w]);
      m2 = max_nan(m2, red[1][w]);
    }
    // this warp's sums rescaled to the CTA maxima
    const float f1 = (s1.m == -INFINITY) ? 0.f : exp2f(s1.m - m1);
    const float f2 = (s2.m == -INFINITY) ? 0.f : exp2f(s2.m - m2);
    if (lane == 0) {
      z1 = s1.z * f1;
      c1 = s1.c * f1 * f1;
      z2 = s2.z * f2;
    }
  }
  z1 = warp_sum(z1);
  c1 = warp_sum(c1);
  z2 = warp_sum(z2);
  __syncthreads();  // the maxima in red[] have been read
  if (lane == 0) {
    red[2][warp] = z1;
    red[3][warp] = c1;
    red[4][warp] = z2;
  }
  __syncthreads();
  if (tid == 0) {
    float a = 0.f, c = 0.f, d = 0.f;
    for (int w = 0; w < kWarps; ++w) {
      a += red[2][w];
      c += red[3][w];
      d += red[4][w];
    }
    cta_st[0] = m1;
    cta_st[1] = a;
    cta_st[2] = c;
    cta_st[3] = m2;
    cta_st[4] = d;
  }
  // ---- gather the cluster's statistics (one remote load per thread), combine
  // them in rank order (the same result in every CTA)
  cluster_arrive();
  cluster_wait();
  if (tid < 5 * S) all_st[tid / 5][tid % 5] = ld_cluster_f32(&cta_st[tid % 5], tid / 5);
  cluster_arrive();  // this CTA is done reading remote statistics
  __syncthreads();
  if (tid == 0) {
    Stat a = stat_empty(), c = stat_empty();
    for (int q = 0; q < S; ++q) {
      a = stat_merge(a, Stat{all_st[q][0], all_st[q][1], all_st[q][2]});
      c = stat_merge(c, Stat{all_st[q][3], all_st[q][4], 0.f});
    }
    const float alpha = 0.5f + 0.5f * (a.c / (a.z * a.z));
    fin[0] = a.m;
    fin[1] = alpha / a.z;
    fin[2] = c.m;
    fin[3] = (1.0f - alpha) / c.z;
    if (rank == 0 && p.alpha != nullptr) p.alpha[b] = alpha;
  }
  __syncthreads();
  const float M1 = fin[0], k1 = fin[1], M2 = fin[2], k2 = fin[3];

  // ---- pass 2: p_mix of this slice
  if (in_regs) {
#pragma unroll
    for (int it = 0; it < kRegVecs; ++it) {
      const int v = v0 + (it * kThreads + tid) * 8;
      if (v < v1) {
        float o[8];
#pragma unroll
        for (int i = 0; i < 8; ++i)
          o[i] = k1 * exp2f(r1[it].get(i) - M1) + k2 * exp2f(r2[it].get(i) - M2);
        reinterpret_cast<float4*>(out + v)[0] = make_float4(o[0], o[1], o[2], o[3]);
        reinterpret_cast<float4*>(out + v)[1] = make_float4(o[4], o[5], o[6], o[7]);
      }
    }
  } else {
    for (int v = v0 + tid * 8; v < v1; v += kThreads * 8) {
      float x1[8], x2[8], o[8];
      load8<T>(row1 + v, x1);
      load8<T>(row2 + v, x2);
#pragma unroll
      for (int i = 0; i < 8; ++i) o[i] = k1 * exp2f(x1[i] - M1) + k2 * exp2f(x2[i] - M2);
      reinterpret_cast<float4*>(out + v)[0] = make_float4(o[0], o[1], o[2], o[3]);
      reinterpret_cast<float4*>(out + v)[1] = make_float4(o[4], o[5], o[6], o[7]);
    }
  }
  cluster_wait();  // no CTA leaves while another may still read its statistics
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
