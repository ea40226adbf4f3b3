// MoE MLP block with router replay: routing, dispatch and combine kernels.
//
// "Sintesi Tecnica: Dual-Flow Transformers", section "Meccanismi Chiave"
// (router replay): the auxiliary flow reuses the set of experts selected by
// the primary router and applies them with its own mixing weights; section
// "Contributi Chiave": the two flows may have independent expert fan-outs.
// Readings: one router matrix shared by both flows; ids = the primary's
// top-k_aux experts by descending logit (ties: lower expert index); the
// primary uses the first k, the auxiliary all k_aux; gates are each flow's
// softmax over its set; experts are SwiGLU MLPs.
//
// The expert MLPs themselves run on the grouped tcgen05 projection: the
// dispatch kernel packs, for every expert e, the primary rows routed to it
// into rows 0..63 of a fixed [128][d] block and the auxiliary rows into rows
// 64..127, so each expert's gate/up and down weights stream from HBM once for
// both flows with launch shapes that do not depend on the routing. The
// combine kernel forms y_f[t] = sum_j g_f[t][j] * Y_{ids[t][j]}[slot_f[t][j]]
// (+ residual) in fp32 and stores bf16.
#include <math.h>

#include "common.cuh"
#include "host_util.h"

namespace df {
namespace moe {

constexpr int kRows = 64;      // rows per flow in an expert block (max tokens per call)
constexpr int kMaxK = 8;       // max experts per token
constexpr int kMaxE = 256;     // max experts
constexpr int kThreads = 256;
constexpr int kCopySplit = 16;  // CTAs per expert in the dispatch copy
constexpr float kLog2e = 1.4426950408889634f;

// ------------------------------------------------------------------ routing

struct RouteParams {
  const __nv_bfloat16* x;
  int64_t ldx;
  const __nv_bfloat16* w;  // [E][d]
  int B, d, E, k, k_aux;
  int32_t* ids;            // [B][k_aux]
  float* g1;               // [B][k]
  float* g2;               // [B][k_aux]
  float* logits;           // [2B][E] or null
};

// One CTA per token: both flows' router logits (fp32 dot products of the bf16
// rows), the primary's top-k_aux, and both gate vectors.
__global__ void __launch_bounds__(kThreads) route_kernel(const RouteParams p) {
  __shared__ float r[2][kMaxE];
  const int t = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  pdl_wait();
  pdl_trigger();
  const int nvec = p.d / 8;
  for (int pair = warp; pair < 2 * p.E; pair += kThreads / 32) {
    const int f = pair / p.E, e = pair % p.E;
    const uint4* xr = reinterpret_cast<const uint4*>(p.x + (static_cast<int64_t>(f) * p.B + t) * p.ldx);
    const uint4* wr = reinterpret_cast<const uint4*>(p.w + static_cast<int64_t>(e) * p.d);
    float acc = 0.f;
#pragma unroll 8
    for (int v = lane; v < nvec; v += 32) {  // loads of 8 iterations in flight
      const uint4 a = xr[v], b = wr[v];
      const uint32_t aw[4] = {a.x, a.y, a.z, a.w}, bw[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        acc = fmaf(bf16_bits_to_float(static_cast<uint16_t>(aw[q] & 0xffffu)),
                   bf16_bits_to_float(static_cast<uint16_t>(bw[q] & 0xffffu)), acc);
        acc = fmaf(bf16_bits_to_float(static_cast<uint16_t>(aw[q] >> 16)),
                   bf16_bits_to_float(static_cast<uint16_t>(bw[q] >> 16)), acc);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) r[f][e] = acc;
  }
  __syncthreads();
  if (threadIdx.x != 0) return;
  if (p.logits) {
    for (int e = 0; e < p.E; ++e) {
      p.logits[static_cast<int64_t>(t) * p.E + e] = r[0][e];
      p.logits[static_cast<int64_t>(p.B + t) * p.E + e] = r[1][e];
    }
  }
  // top-k_aux of the primary logits: repeated arg-max over the unchosen
  // experts, scanning in index order with a strict comparison (ties go to the
  // lower index)
  int sel[kMaxK];
  uint32_t taken[kMaxE / 32] = {};
  for (int j = 0; j < p.k_aux; ++j) {
    int best = -1;
    float bv = 0.f;
    for (int e = 0; e < p.E; ++e) {
      if (taken[e >> 5] & (1u << (e & 31))) continue;
      if (best < 0 || r[0][e] > bv) {
        best = e;
        bv = r[0][e];
      }
    }
    sel[j] = best;
    taken[best >> 5] |= 1u << (best & 31);
    p.ids[static_cast<int64_t>(t) * p.k_aux + j] = best;
  }
  // gates: softmax of each flow's logits over its set
  for (int f = 0; f < 2; ++f) {
    const int n = f == 0 ? p.k : p.k_aux;
    float m = -INFINITY;
    for (int j = 0; j < n; ++j) m = fmaxf(m, r[f][sel[j]]);
    float z = 0.f, ex[kMaxK];
    for (int j = 0; j < n; ++j) {
      ex[j] = exp2f((r[f][sel[j]] - m) * kLog2e);
      z += ex[j];
    }
    float* g = f == 0 ? p.g1 + static_cast<int64_t>(t) * p.k : p.g2 + static_cast<int64_t>(t) * p.k_aux;
    for (int j = 0; j < n; ++j) g[j] = ex[j] / z;
  }
}

// ------------------------------------------------------------------ dispatch

struct DispatchParams {
  const __nv_bfloat16* x;
  int64_t ldx;
  int B, d, E, k, k_aux;
  const int32_t* ids;
  __nv_bfloat16* xe;  // [E][128][d]
  int32_t* slot1;     // [B][k]: row of (t, j) in expert ids[t][j]'s block
  int32_t* slot2;     // [B][k_aux]: 64 + row
  int32_t* counts;    // [E][2] or null
  int32_t* err;
};

// kCopySplit CTAs per expert: each finds the tokens routed to it in token
// order (ballot prefix over the <= 64 tokens) and copies its share of their
// rows into the expert's block; the first also writes the row slots and
// counts. Rows past the counts are left as they were: every output row of the
// projections depends only on its own input row, and the combine reads only
// the rows listed in the slots.
__global__ void __launch_bounds__(kThreads) dispatch_kernel(const DispatchParams p) {
  __shared__ int rows1[kRows], rows2[kRows];
  __shared__ int n_s[2];
  const int e = blockIdx.x;
  const bool writer = blockIdx.y == 0;
  const int tid = threadIdx.x;
  pdl_wait();
  pdl_trigger();
  if (tid < 64) {  // two warps: warp 0 tokens 0..31, warp 1 tokens 32..63
    const int t = tid;
    int j1 = -1, j2 = -1;
    if (t < p.B) {
      for (int j = 0; j < p.k_aux; ++j) {
        const int id = p.ids[static_cast<int64_t>(t) * p.k_aux + j];
        if (id < 0 || id >= p.E) {
          if (writer) set_err(p.err, DF_DEVERR_BLOCK);
          continue;
        }
        if (id == e) {
          if (j < p.k) j1 = j;
          j2 = j;
        }
      }
    }
    const uint32_t m1 = __ballot_sync(0xffffffffu, j1 >= 0);
    const uint32_t m2 = __ballot_sync(0xffffffffu, j2 >= 0);
    const int lane = t & 31;
    const uint32_t below = (1u << lane) - 1u;
    __shared__ int c1[2], c2[2];
    if (lane == 0) {
      c1[t >> 5] = __popc(m1);
      c2[t >> 5] = __popc(m2);
    }
    asm volatile("bar.sync 1, 64;" ::: "memory");
    const int base1 = (t >> 5) ? c1[0] : 0, base2 = (t >> 5) ? c2[0] : 0;
    if (j1 >= 0) {
      const int row = base1 + __popc(m1 & below);
      rows1[row] = t;
      if (writer) p.slot1[static_cast<int64_t>(t) * p.k + j1] = row;
    }
    if (j2 >= 0) {
      const int row = base2 + __popc(m2 & below);
      rows2[row] = t;
      if (writer) p.slot2[static_cast<int64_t>(t) * p.k_aux + j2] = kRows + row;
    }
    if (t == 0) {
      n_s[0] = c1[0] + c1[1];
      n_s[1] = c2[0] + c2[1];
    }
  }
  __syncthreads();
  const int n1 = n_s[0], n2 = n_s[1];
  if (tid == 0 && writer && p.counts) {
    p.counts[2 * e] = n1;
    p.counts[2 * e + 1] = n2;
  }
  const int nvec = p.d / 8;
  uint4* dst = reinterpret_cast<uint4*>(p.xe + static_cast<int64_t>(e) * 2 * kRows * p.d);
  const int total = (n1 + n2) * nvec;
  const int per = (total + gridDim.y - 1) / gridDim.y;
  const int i0 = blockIdx.y * per, i1 = min(total, i0 + per);
  for (int i = i0 + tid; i < i1; i += kThreads) {
    const int rr = i / nvec, v = i % nvec;
    const bool aux = rr >= n1;
    const int row = aux ? kRows + (rr - n1) : rr;
    const int t = aux ? rows2[rr - n1] : rows1[rr];
    const uint4* src = reinterpret_cast<const uint4*>(
        p.x + (static_cast<int64_t>(aux ? p.B : 0) + t) * p.ldx);
    dst[static_cast<int64_t>(row) * nvec + v] = src[v];
  }
}

// ------------------------------------------------------------------ combine

struct CombineParams {
  const __nv_bfloat16* ye;  // [E][128][d]
  const int32_t* ids;
  const float* g1;
  const float* g2;
  const int32_t* slot1;
  const int32_t* slot2;
  int B, d, E, k, k_aux;
  const __nv_bfloat16* residual;  // [2B][d] or null
  int64_t ldr;
  __nv_bfloat16* y;               // [2B][d]
  int64_t ldy;
  int32_t* err;
};

// One CTA per (token, flow): the gate-weighted sum of its experts' output
// rows in fp32, plus the residual, one rounding to bf16.
__global__ void __launch_bounds__(kThreads) combine_kernel(const CombineParams p) {
  const int t = blockIdx.x, f = blockIdx.y;
  pdl_wait();
  pdl_trigger();
  const int n = f == 0 ? p.k : p.k_aux;
  const float* g = f == 0 ? p.g1 + static_cast<int64_t>(t) * p.k : p.g2 + static_cast<int64_t>(t) * p.k_aux;
  const int32_t* slot = f == 0 ? p.slot1 + static_cast<int64_t>(t) * p.k
                               : p.slot2 + static_cast<int64_t>(t) * p.k_aux;
  const uint4* src[kMaxK];
  float w[kMaxK];
  int nv = 0;
  for (int j = 0; j < n; ++j) {
    const int e = p.ids[static_cast<int64_t>(t) * p.k_aux + j];
    const int row = slot[j];
    if (e < 0 || e >= p.E || row < 0 || row >= 2 * kRows) {
      if (threadIdx.x == 0) set_err(p.err, DF_DEVERR_BLOCK);
      continue;
    }
    src[nv] = reinterpret_cast<const uint4*>(p.ye + (static_cast<int64_t>(e) * 2 * kRows + row) * p.d);
    w[nv] = g[j];
    ++nv;
  }
  const int nvec = p.d / 8;
  const int64_t r = static_cast<int64_t>(f) * p.B + t;
  for (int v = threadIdx.x; v < nvec; v += kThreads) {
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (int j = 0; j < nv; ++j) {
      const uint4 u = src[j][v];
      const uint32_t uw[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        acc[2 * q] = fmaf(w[j], bf16_bits_to_float(static_cast<uint16_t>(uw[q] & 0xffffu)), acc[2 * q]);
        acc[2 * q + 1] = fmaf(w[j], bf16_bits_to_float(static_cast<uint16_t>(uw[q] >> 16)), acc[2 * q + 1]);
      }
    }
    if (p.residual) {
      const uint4 u = reinterpret_cast<const uint4*>(p.residual + r * p.ldr)[v];
      const uint32_t uw[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        acc[2 * q] += bf16_bits_to_float(static_cast<uint16_t>(uw[q] & 0xffffu));
        acc[2 * q + 1] += bf16_bits_to_float(static_cast<uint16_t>(uw[q] >> 16));
      }
    }
    uint4 o;
    o.x = pack_bf16x2(__float2bfloat16_rn(acc[0]), __float2bfloat16_rn(acc[1]));
    o.y = pack_bf16x2(__float2bfloat16_rn(acc[2]), __float2bfloat16_rn(acc[3]));
    o.z = pack_bf16x2(__float2bfloat16_rn(acc[4]), __float2bfloat16_rn(acc[5]));
    o.w = pack_bf16x2(__float2bfloat16_rn(acc[6]), __float2bfloat16_rn(acc[7]));
    reinterpret_cast<uint4*>(p.y + r * p.ldy)[v] = o;
  }
}

inline df_status check_common(int B, int d, int E, int k, int k_aux) {
  if (B < 1 || d < 1 || E < 1 || k < 1 || k_aux < k) return DF_ERR_SHAPE;
  if (B > kRows || E > kMaxE || k_aux > kMaxK || k_aux > E) return DF_ERR_UNSUPPORTED;
  if (d % 8 != 0) return DF_ERR_UNSUPPORTED;
  return DF_OK;
}

}  // namespace moe
}  // namespace df

extern "C" df_status dualflow_moe_route(const void* x, int64_t ldx, int B, int d,
                                        const void* w_router, int E, int k, int k_aux,
                                        int32_t* ids, float* g1, float* g2, float* logits,
                                        void* stream) {
  using namespace df;
  if (!x || !w_router || !ids || !g1 || !g2) return DF_ERR_NULL;
  const df_status s = moe::check_common(B, d, E, k, k_aux);
  if (s != DF_OK) return s;
  const int64_t lx = ldx ? ldx : d;
  if (lx < d) return DF_ERR_SHAPE;
  if (lx % 8 != 0 || !aligned(x, 16) || !aligned(w_router, 16)) return DF_ERR_ALIGN;
  moe::RouteParams p{static_cast<const __nv_bfloat16*>(x), lx,
                     static_cast<const __nv_bfloat16*>(w_router), B, d, E, k, k_aux, ids, g1, g2,
                     logits};
  if (launch_pdl(moe::route_kernel, dim3(B), dim3(moe::kThreads), 0,
                 static_cast<cudaStream_t>(stream), p) != cudaSuccess)
    return DF_ERR_CUDA;
  return DF_OK;
}

extern "C" df_status dualflow_moe_dispatch(const void* x, int64_t ldx, int B, int d,
                                           const int32_t* ids, int E, int k, int k_aux, void* xe,
                                           int32_t* slot1, int32_t* slot2, int32_t* counts,
                                           int32_t* err_flag, void* stream) {
  using namespace df;
  if (!x || !ids || !xe || !slot1 || !slot2) return DF_ERR_NULL;
  const df_status s = moe::check_common(B, d, E, k, k_aux);
  if (s != DF_OK) return s;
  const int64_t lx = ldx ? ldx : d;
  if (lx < d) return DF_ERR_SHAPE;
  if (lx % 8 != 0 || !aligned(x, 16) || !aligned(xe, 16)) return DF_ERR_ALIGN;
  moe::DispatchParams p{static_cast<const __nv_bfloat16*>(x), lx, B, d, E, k, k_aux, ids,
                        static_cast<__nv_bfloat16*>(xe), slot1, slot2, counts, err_flag};
  if (launch_pdl(moe::dispatch_kernel, dim3(E, moe::kCopySplit), dim3(moe::kThreads), 0,
                 static_cast<cudaStream_t>(stream), p) != cudaSuccess)
    return DF_ERR_CUDA;
  return DF_OK;
}

extern "C" df_status dualflow_moe_combine(const void* ye, const int32_t* ids, const float* g1,
                                          const float* g2, const int32_t* slot1,
                                          const int32_t* slot2, int B, int d, int E, int k,
                                          int k_aux, const void* residual, int64_t ldr, void* y,
                                          int64_t ldy, int32_t* err_flag, void* stream) {
  using namespace df;
  if (!ye || !ids || !g1 || !g2 || !slot1 || !slot2 || !y) return DF_ERR_NULL;
  const df_status s = moe::check_common(B, d, E, k, k_aux);
  if (s != DF_OK) return s;
  const int64_t lr = ldr ? ldr : d, ly = ldy ? ldy : d;
  if (ly < d || (residual && lr < d)) return DF_ERR_SHAPE;
  if (ly % 8 != 0 || (residual && lr % 8 != 0) || !aligned(ye, 16) || !aligned(y, 16) ||
      (residual && !aligned(residual, 16)))
    return DF_ERR_ALIGN;
  moe::CombineParams p{static_cast<const __nv_bfloat16*>(ye), ids, g1, g2, slot1, slot2, B, d, E,
                       k, k_aux, static_cast<const __nv_bfloat16*>(residual), lr,
                       static_cast<__nv_bfloat16*>(y), ly, err_flag};
  if (launch_pdl(moe::combine_kernel, dim3(B, 2), dim3(moe::kThreads), 0,
                 static_cast<cudaStream_t>(stream), p) != cudaSuccess)
    return DF_ERR_CUDA;
  return DF_OK;
}
