// Post-attention half of the Dual-Flow decoder layer as ONE persistent kernel.
//
// Method: "Sintesi Tecnica: Dual-Flow Transformers", sections "Architettura
// Core" (both flows share the output and MLP matrices), "Meccanismi Chiave"
// (one-way coupling b_l at the MLP intermediate and c_l at the MLP output) and
// "Costi di Inferenza vs. Addestramento" (grouped decode reads the unique
// weights once for both flows). With X = [primary rows; auxiliary rows]:
//   x_mid = x + attn W_o^T                                   (residual)
//   xn2   = x_mid / sqrt(mean(x_mid^2) + eps)                 (RMSNorm, unit gain)
//   h     = SiLU(xn2 W_gate^T) * (xn2 W_up^T);  h_aux += b (.) h_primary
//   x_out = x_mid + h W_down^T;  aux rows add c (.) (h W_down^T)_primary
// x_mid, xn2, h and x_out are stored as bf16 (the same interfaces as the
// four-launch form of the same step).
//
// Why one kernel: at M = 128 rows every projection is a weight stream (about
// 128 flop per weight byte, below the B200 ridge). Separate launches leave
// HBM idle at every boundary: the next launch's CTAs cannot become resident
// until the previous launch's CTAs (one per SM) have run their tails, and
// then each pays a first TMA round trip. Here one CTA per SM walks all three
// GEMMs in order and its TMA producer streams the weights continuously, into
// a 4-stage ring, across the phase boundaries; only the activation tiles of a
// phase wait for the phase before it. The dependencies between phases are
// grid-wide counters in the workspace (every CTA is resident: one per SM,
// grid = SM count), each wait bounded.
//
// Phases (units are spread over the CTAs, CTA i takes units i, i + G, ...):
//   P0  W_o:    16 column tiles of 256 x S0 k-ranges -> fp32 partials
//   --- counter A --- R0: CTA r < M sums row r's partials in split order, adds
//                     the residual, stores x_mid, then xn2 (row-local norm)
//   --- counter B --- P1  W_gate/W_up: one tile of 2*H1 weight rows per CTA,
//                     SwiGLU + b coupling straight from TMEM -> h
//   --- counter C --- P2  W_down: column tiles of 256 x S2 k-ranges -> partials
//   --- counter D --- R2: (sequence, column half) units: residual + c
//                     coupling -> x_out
// Roles (224 threads): warp 0 weight producer, warp 1 MMA issuer (one thread,
// tcgen05.mma M = 128 into two 256-column TMEM accumulators), warp 2
// activation producer, warps 3-6 epilogue (TMEM lane quarter = warp % 4).
// Every split reduction sums in a fixed order: results are deterministic, and
// primary rows never read auxiliary rows.
#include <math.h>
#include <string.h>

#include <mutex>

#include "common.cuh"
#include "host_util.h"
#include "umma.cuh"

namespace df {
namespace post {

using namespace umma;

constexpr int kBM = 128;
constexpr int kBK = 64;
constexpr int kThreads = 224;
constexpr int kEpiThreads = 128;
constexpr int kStages = 4;
constexpr int kXBytes = kBM * kBK * 2;            // 16 KB activation tile
constexpr int kSlot = kXBytes + 256 * kBK * 2;    // + up to 32 KB of weights
constexpr int kTileN = 256;                       // W_o / W_down column tile
constexpr int kMaxHalf = 112;                     // SwiGLU output columns per tile
constexpr int kStgPitch = 36;                     // fp32 staging row pitch
constexpr int kXchgFloats = 64 * (kMaxHalf + 1);  // >= 4 * 32 * kStgPitch
constexpr int kCounters = 8;                      // A, B, C, D, exit
constexpr size_t kCounterBytes = 256;
constexpr size_t kSmemBytes = 1024 + static_cast<size_t>(kStages) * kSlot + kXchgFloats * 4 +
                              16 * 4 + 256;  // + barriers, TMEM slot and flags
static_assert(kXchgFloats >= 4 * 32 * kStgPitch, "staging must fit in the exchange area");
static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");

enum { kCntA = 0, kCntB = 1, kCntC = 2, kCntD = 3, kCntExit = 4 };

struct Gemm {
  int units, splits, kblocks;
  int BN;       // MMA N
  int half;     // SwiGLU output columns per tile (0: plain)
  int w_bytes;  // weight bytes per stage
  uint32_t idesc;
};

struct Params {
  int M, mp, d, qd, F;
  float eps;
  Gemm g[3];
  int r2_units;  // mp * 2 (sequence, column half)
  const __nv_bfloat16* x;
  const __nv_bfloat16* b;
  const __nv_bfloat16* c;
  __nv_bfloat16* x_mid;
  __nv_bfloat16* xn2;
  __nv_bfloat16* h;
  __nv_bfloat16* x_out;
  float* part;  // [units][128][256] fp32
  int* cnt;     // [kCounters]
  int32_t* err;
};

__device__ __forceinline__ void epi_bar() {
  asm volatile("bar.sync 1, %0;" ::"n"(kEpiThreads) : "memory");
}

__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

__device__ __forceinline__ int ld_acquire(const int* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ float4 ld_cg4(const float* p) {
  float4 v;
  asm volatile("ld.global.cg.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ void st_cg4(float* p, float4 v) {
  asm volatile("st.global.cg.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(p), "f"(v.x), "f"(v.y),
               "f"(v.z), "f"(v.w)
               : "memory");
}

// 16 bf16 values through L2 only (rows written by other CTAs of this grid).
__device__ __forceinline__ void load_bf16x16_cg(const __nv_bfloat16* src, float (&v)[16]) {
#pragma unroll
  for (int q = 0; q < 2; ++q) {
    uint32_t w[4];
    asm volatile("ld.global.cg.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3])
                 : "l"(src + 8 * q));
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      v[q * 8 + 2 * k] = bf16_bits_to_float(static_cast<uint16_t>(w[k] & 0xffffu));
      v[q * 8 + 2 * k + 1] = bf16_bits_to_float(static_cast<uint16_t>(w[k] >> 16));
    }
  }
}

// Single-thread bounded wait until *cnt >= target (every CTA of the grid has
// passed the corresponding point). false: gave up.
__device__ bool wait_count(const int* cnt, int target) {
  if (ld_acquire(cnt) >= target) return true;
  const long long t0 = clock64();
  while (ld_acquire(cnt) < target) {
    if (clock64() - t0 > kWaitLimitCycles) return false;
    __nanosleep(100);
  }
  return true;
}

// (tile, first k-block, end k-block) of unit u of GEMM g.
__device__ __forceinline__ void unit_range(const Gemm& g, int u, int& tile, int& k0, int& k1) {
  if (g.splits > 1) {
    tile = u / g.splits;
    const int s = u - tile * g.splits;
    k0 = s * g.kblocks / g.splits;
    k1 = (s + 1) * g.kblocks / g.splits;
  } else {
    tile = u;
    k0 = 0;
    k1 = g.kblocks;
  }
}

// The epilogue threads' arrival at a grid counter: every thread's stores are
// made visible (also to TMA reads of other CTAs) before one thread adds.
__device__ __forceinline__ void arrive_count(int* cnt, int et) {
  fence_proxy_async_global();
  epi_bar();
  if (et == 0) {
    __threadfence();
    atomicAdd(cnt, 1);
  }
}

// All epilogue threads wait for a grid counter; returns false if it gave up.
__device__ __forceinline__ bool epi_wait_count(const int* cnt, int target, int et,
                                               volatile int* flag) {
  if (et == 0) *flag = wait_count(cnt, target) ? 1 : 0;
  epi_bar();
  const bool ok = *flag != 0;
  epi_bar();
  return ok;
}

// Accumulator (this warp's 32 rows, BN = 256 columns) -> fp32 partial slab
// part[unit][row][256], staged through shared memory so that each store
// instruction writes whole 128-byte row segments.
__device__ void store_partial(const Params& p, float* slab, uint32_t taddr, int quarter, int lane,
                              float* stg) {
  for (int c = 0; c < kTileN; c += 32) {
    float v[32];
    tmem_ld<32>(taddr + c, v);
    float4* srow = reinterpret_cast<float4*>(stg + lane * kStgPitch);
#pragma unroll
    for (int i = 0; i < 8; ++i)
      srow[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
    __syncwarp();
#pragma unroll
    for (int rr = 0; rr < 8; ++rr) {
      const int rl = rr * 4 + (lane >> 3), cg = (lane & 7) * 4;
      const int r = quarter * 32 + rl;
      if (r < p.M)
        st_cg4(slab + static_cast<size_t>(r) * kTileN + c + cg,
               *reinterpret_cast<const float4*>(stg + rl * kStgPitch + cg));
    }
    __syncwarp();
  }
}

// P1 epilogue of tile t: h[row][t*H + j] = SiLU(gate) * up (+ b * primary row's
// value for auxiliary rows). Pass 1 stores the primary rows (and every row
// without coupling) and parks the primary values in `xchg`; pass 2 re-reads
// the accumulator for the auxiliary rows and adds the coupling.
__device__ void swiglu_epilogue(const Params& p, int t, uint32_t taddr, int quarter, int lane,
                                float* xchg) {
  const int H = p.g[1].half;
  const int row = quarter * 32 + lane;
  const int col0 = t * H;
  const bool coupled = p.b != nullptr;
  const int pitch = H + 1;
  // pass 1
  if (!coupled || quarter * 32 < p.mp) {
    for (int c = 0; c < H; c += 8) {
      float g[8], u[8];
      tmem_ld<8>(taddr + c, g);
      tmem_ld<8>(taddr + H + c, u);
#pragma unroll
      for (int i = 0; i < 8; ++i) g[i] = silu_f(g[i]) * u[i];
      const bool prim = row < p.mp;
      if (coupled && prim) {
#pragma unroll
        for (int i = 0; i < 8; ++i) xchg[row * pitch + c + i] = g[i];
      }
      if ((!coupled || prim) && row < p.M && col0 + c < p.F)
        store_bf16<8>(p.h + static_cast<size_t>(row) * p.F + col0 + c, g);
    }
  }
  if (!coupled) return;
  epi_bar();
  // pass 2: auxiliary rows mp .. 2mp-1, paired with primary row row - mp
  if (quarter * 32 + 31 >= p.mp) {
    for (int c = 0; c < H; c += 8) {
      float g[8], u[8];
      tmem_ld<8>(taddr + c, g);
      tmem_ld<8>(taddr + H + c, u);
      const bool aux = row >= p.mp && row < p.M;
      if (aux && col0 + c < p.F) {
        float bv[8];
        load_bf16<8>(p.b + col0 + c, bv);
        const float* src = xchg + (row - p.mp) * pitch + c;
#pragma unroll
        for (int i = 0; i < 8; ++i) g[i] = fmaf(bv[i], src[i], silu_f(g[i]) * u[i]);
        store_bf16<8>(p.h + static_cast<size_t>(row) * p.F + col0 + c, g);
      }
    }
  }
  epi_bar();  // xchg is reused by the next tile / the staging of P2
}

// R0 for row r: x_mid = x + sum of the W_o partials (split order), stored
// bf16; then xn2 = bf16(x_mid / sqrt(mean(x_mid^2) + eps)) from the stored
// (rounded) values.
__device__ void reduce_o_row(const Params& p, int r, int et, float* red) {
  const Gemm& g = p.g[0];
  const int groups = p.d / 32;
  float ss = 0.f;
  for (int cg = et; cg < groups; cg += kEpiThreads) {
    const int col = cg * 32;
    const int tile = col / kTileN, off = col - tile * kTileN;
    float acc[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) acc[i] = 0.f;
    for (int s = 0; s < g.splits; ++s) {
      const float* src =
          p.part + (static_cast<size_t>(tile * g.splits + s) * kBM + r) * kTileN + off;
      float4 v[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) v[i] = ld_cg4(src + 4 * i);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        acc[4 * i] += v[i].x;
        acc[4 * i + 1] += v[i].y;
        acc[4 * i + 2] += v[i].z;
        acc[4 * i + 3] += v[i].w;
      }
    }
    float res[32];
    load_bf16<32>(p.x + static_cast<size_t>(r) * p.d + col, res);
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      acc[i] += res[i];
      const float q = __bfloat162float(__float2bfloat16_rn(acc[i]));
      ss = fmaf(q, q, ss);
    }
    store_bf16<32>(p.x_mid + static_cast<size_t>(r) * p.d + col, acc);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  if ((et & 31) == 0) red[et >> 5] = ss;
  epi_bar();
  const float tot = red[0] + red[1] + red[2] + red[3];
  const float inv = 1.0f / sqrtf(tot / static_cast<float>(p.d) + p.eps);
  for (int cg = et; cg < groups; cg += kEpiThreads) {
    const int col = cg * 32;
    float v[32];
    load_bf16<32>(p.x_mid + static_cast<size_t>(r) * p.d + col, v);  // this thread's own stores
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] *= inv;
    store_bf16<32>(p.xn2 + static_cast<size_t>(r) * p.d + col, v);
  }
  epi_bar();  // red is reused
}

// R2 for unit v = (sequence j, column half hf): x_out rows j (primary) and
// mp + j (auxiliary) over that half: residual x_mid + sum of the W_down
// partials (split order); the auxiliary row adds c * (primary row's sum).
__device__ void reduce_down_pair(const Params& p, int v, int et) {
  const Gemm& g = p.g[2];
  const int j = v >> 1, hf = v & 1;
  const int half_cols = p.d / 2;
  const int rp = j, ra = p.mp + j;
  for (int cg = et; cg < half_cols / 16; cg += kEpiThreads) {
    const int col = hf * half_cols + cg * 16;
    const int tile = col / kTileN, off = col - tile * kTileN;
    float ap[16], aa[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) ap[i] = aa[i] = 0.f;
    for (int s = 0; s < g.splits; ++s) {
      const float* base = p.part + static_cast<size_t>(tile * g.splits + s) * kBM * kTileN + off;
      float4 vp[4], va[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        vp[i] = ld_cg4(base + static_cast<size_t>(rp) * kTileN + 4 * i);
        va[i] = ld_cg4(base + static_cast<size_t>(ra) * kTileN + 4 * i);
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        ap[4 * i] += vp[i].x; ap[4 * i + 1] += vp[i].y; ap[4 * i + 2] += vp[i].z;
        ap[4 * i + 3] += vp[i].w;
        aa[4 * i] += va[i].x; aa[4 * i + 1] += va[i].y; aa[4 * i + 2] += va[i].z;
        aa[4 * i + 3] += va[i].w;
      }
    }
    if (p.c != nullptr) {
      float cv[16];
      load_bf16<16>(p.c + col, cv);
#pragma unroll
      for (int i = 0; i < 16; ++i) aa[i] = fmaf(cv[i], ap[i], aa[i]);
    }
    float rv[16];
    load_bf16x16_cg(p.x_mid + static_cast<size_t>(rp) * p.d + col, rv);
#pragma unroll
    for (int i = 0; i < 16; ++i) ap[i] += rv[i];
    load_bf16x16_cg(p.x_mid + static_cast<size_t>(ra) * p.d + col, rv);
#pragma unroll
    for (int i = 0; i < 16; ++i) aa[i] += rv[i];
    store_bf16<16>(p.x_out + static_cast<size_t>(rp) * p.d + col, ap);
    store_bf16<16>(p.x_out + static_cast<size_t>(ra) * p.d + col, aa);
  }
}

__global__ void __launch_bounds__(kThreads, 1)
    post_kernel(const __grid_constant__ CUtensorMap tmXo, const __grid_constant__ CUtensorMap tmWo,
                const __grid_constant__ CUtensorMap tmXg, const __grid_constant__ CUtensorMap tmWg,
                const __grid_constant__ CUtensorMap tmXd, const __grid_constant__ CUtensorMap tmWd,
                const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  float* xchg = reinterpret_cast<float*>(smem + static_cast<size_t>(kStages) * kSlot);
  float* red = xchg + kXchgFloats;                                // [16]
  uint64_t* full = reinterpret_cast<uint64_t*>(red + 16);         // [kStages]
  uint64_t* empty = full + kStages;                               // [kStages]
  uint64_t* acc_full = empty + kStages;                           // [2]
  uint64_t* acc_empty = acc_full + 2;                             // [2]
  uint64_t* mma_done = acc_empty + 2;                             // [1]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
  // [0] abort, [1] epilogue broadcast, [2] / [3] stages issued by the weight /
  // activation producer
  volatile int* flags = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = gridDim.x, cta = blockIdx.x;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&full[i], 2);  // weight producer + activation producer
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], kEpiThreads / 32);
    }
    mbar_init(mma_done, 1);
    flags[0] = 0;
    flags[1] = 0;
    flags[2] = 0;
    flags[3] = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)),
                 "n"(512)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // Only the weight producer may run ahead of the kernel launched before this
  // one (the weights are constants); every other role waits for it first.
  if (warp != 0) pdl_wait();

  if (warp == 0) {
    // ------------------------------------------------------------ weight producer
    if (lane == 0) {
      prefetch_tensormap(&tmWo);
      prefetch_tensormap(&tmWg);
      prefetch_tensormap(&tmWd);
      const uint64_t pol = l2_policy_evict_first();
      int s = 0;
      uint32_t ph = 0;
      long long n = 0;
      bool ok = true;
      for (int q = 0; q < 3 && ok; ++q) {
        const Gemm& g = p.g[q];
        const CUtensorMap* tm = q == 0 ? &tmWo : (q == 1 ? &tmWg : &tmWd);
        for (int u = cta; u < g.units && ok; u += G) {
          int tile, k0, k1;
          unit_range(g, u, tile, k0, k1);
          for (int kb = k0; kb < k1; ++kb, ++n) {
            if (n >= kStages && !mbar_wait(&empty[s], ph ^ 1u)) {
              set_err(p.err, DF_DEVERR_TIMEOUT);
              flags[0] = 1;
              ok = false;
              break;
            }
            if (flags[0]) {
              ok = false;
              break;
            }
            uint8_t* wdst = smem + static_cast<size_t>(s) * kSlot + kXBytes;
            mbar_arrive_expect_tx(&full[s], static_cast<uint32_t>(g.w_bytes));
            if (q == 1) {
              tma_load_2d_hint(wdst, tm, &full[s], kb * kBK, tile * g.half, pol);
              tma_load_2d_hint(wdst + g.half * 128, tm, &full[s], kb * kBK,
                               p.F + tile * g.half, pol);
            } else {
              tma_load_2d_hint(wdst, tm, &full[s], kb * kBK, tile * kTileN, pol);
            }
            if (++s == kStages) {
              s = 0;
              ph ^= 1u;
            }
          }
        }
      }
      flags[2] = static_cast<int>(n);
      pdl_trigger();
    }
  } else if (warp == 2) {
    // ------------------------------------------------------------ activation producer
    if (lane == 0) {
      prefetch_tensormap(&tmXo);
      prefetch_tensormap(&tmXg);
      prefetch_tensormap(&tmXd);
      const uint64_t pol = l2_policy_evict_last();
      int s = 0;
      uint32_t ph = 0;
      long long n = 0;
      bool ok = true;
      for (int q = 0; q < 3 && ok; ++q) {
        const Gemm& g = p.g[q];
        const CUtensorMap* tm = q == 0 ? &tmXo : (q == 1 ? &tmXg : &tmXd);
        bool ready = q == 0;  // P0 reads the attention output: pdl_wait above
        for (int u = cta; u < g.units && ok; u += G) {
          int tile, k0, k1;
          unit_range(g, u, tile, k0, k1);
          if (!ready) {
            // P1 needs every row's xn2 (counter B), P2 every column of h (C)
            if (!wait_count(p.cnt + (q == 1 ? kCntB : kCntC), G)) {
              set_err(p.err, DF_DEVERR_TIMEOUT);
              flags[0] = 1;
              ok = false;
              break;
            }
            fence_proxy_async_global();
            ready = true;
          }
          for (int kb = k0; kb < k1; ++kb, ++n) {
            if (n >= kStages && !mbar_wait(&empty[s], ph ^ 1u)) {
              set_err(p.err, DF_DEVERR_TIMEOUT);
              flags[0] = 1;
              ok = false;
              break;
            }
            if (flags[0]) {
              ok = false;
              break;
            }
            mbar_arrive_expect_tx(&full[s], kXBytes);
            tma_load_2d_hint(smem + static_cast<size_t>(s) * kSlot, tm, &full[s], kb * kBK, 0,
                             pol);
            if (++s == kStages) {
              s = 0;
              ph ^= 1u;
            }
          }
        }
      }
      flags[3] = static_cast<int>(n);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0;
      int seg = 0;
      bool ok = true;
      for (int q = 0; q < 3 && ok; ++q) {
        const Gemm& g = p.g[q];
        for (int u = cta; u < g.units && ok; u += G, ++seg) {
          int tile, k0, k1;
          unit_range(g, u, tile, k0, k1);
          const int acc = seg & 1;
          if (seg >= 2 &&
              !mbar_wait(&acc_empty[acc], static_cast<uint32_t>(((seg >> 1) - 1) & 1))) {
            set_err(p.err, DF_DEVERR_TIMEOUT);
            flags[0] = 1;
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * 256);
          for (int kb = k0; kb < k1; ++kb) {
            if (!mbar_wait(&full[s], ph) || flags[0]) {
              set_err(p.err, DF_DEVERR_TIMEOUT);
              flags[0] = 1;
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t a_addr = smem_u32(smem + static_cast<size_t>(s) * kSlot);
            const uint32_t b_addr = a_addr + kXBytes;
#pragma unroll
            for (int kk = 0; kk < kBK / 16; ++kk)
              umma_bf16(d_tmem, smem_desc(a_addr + kk * 32), smem_desc(b_addr + kk * 32), g.idesc,
                        (kb > k0 || kk > 0) ? 1u : 0u);
            umma_commit(&empty[s]);
            if (++s == kStages) {
              s = 0;
              ph ^= 1u;
            }
          }
          if (!ok) break;
          umma_commit(&acc_full[acc]);
        }
      }
      // no tensor-core operation may still be reading shared memory or TMEM
      // when the CTA leaves (this commit completes after every MMA above)
      umma_commit(mma_done);
      mbar_wait(mma_done, 0);
    }
  } else {
    // ------------------------------------------------------------ epilogue warps
    const int quarter = warp & 3;
    const int et = threadIdx.x - 3 * 32;
    float* stg = xchg + (warp - 3) * 32 * kStgPitch;
    volatile int* eflag = flags + 1;
    int seg = 0;
    bool ok = true;
    auto take_acc = [&](int acc, int sg) -> bool {
      const bool got = mbar_wait_warp(&acc_full[acc], static_cast<uint32_t>((sg >> 1) & 1));
      if (!got && lane == 0) {
        set_err(p.err, DF_DEVERR_TIMEOUT);
        flags[0] = 1;
      }
      return got;
    };
    auto give_acc = [&](int acc) {
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[acc]);
    };
    // P0: W_o partials
    for (int u = cta; u < p.g[0].units && ok; u += G, ++seg) {
      const int acc = seg & 1;
      if (!take_acc(acc, seg)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t taddr =
          tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + static_cast<uint32_t>(acc * 256);
      store_partial(p, p.part + static_cast<size_t>(u) * kBM * kTileN, taddr, quarter, lane, stg);
      give_acc(acc);
    }
    arrive_count(p.cnt + kCntA, et);
    // R0: rows
    for (int r = cta; r < p.M; r += G) {
      if (!epi_wait_count(p.cnt + kCntA, G, et, eflag)) {
        if (et == 0) set_err(p.err, DF_DEVERR_TIMEOUT);
        flags[0] = 1;
        break;
      }
      if (!flags[0]) reduce_o_row(p, r, et, red);
    }
    arrive_count(p.cnt + kCntB, et);
    // P1: SwiGLU tiles straight from TMEM
    for (int u = cta; u < p.g[1].units && ok; u += G, ++seg) {
      const int acc = seg & 1;
      if (!take_acc(acc, seg)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t taddr =
          tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + static_cast<uint32_t>(acc * 256);
      swiglu_epilogue(p, u, taddr, quarter, lane, xchg);
      give_acc(acc);
    }
    arrive_count(p.cnt + kCntC, et);
    // P2: W_down partials
    for (int u = cta; u < p.g[2].units && ok; u += G, ++seg) {
      const int acc = seg & 1;
      if (!take_acc(acc, seg)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t taddr =
          tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + static_cast<uint32_t>(acc * 256);
      store_partial(p, p.part + static_cast<size_t>(u) * kBM * kTileN, taddr, quarter, lane, stg);
      give_acc(acc);
    }
    arrive_count(p.cnt + kCntD, et);
    // R2: (sequence, column half) units
    for (int v = cta; v < p.r2_units; v += G) {
      if (!epi_wait_count(p.cnt + kCntD, G, et, eflag)) {
        if (et == 0) set_err(p.err, DF_DEVERR_TIMEOUT);
        flags[0] = 1;
        break;
      }
      if (!flags[0]) reduce_down_pair(p, v, et);
    }
  }

  // Every role of this CTA is done (all its waits have returned): count the
  // CTA out; the last one out rewinds the counters for the next call.
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (threadIdx.x == 0 && flags[0]) {
    // A wait gave up: a stage may have been filled by one producer only. The
    // missing arrivals are made here so that those phases complete once the
    // copies already issued have landed, and the last kStages stages are
    // awaited (bounded): no copy is left in flight into shared memory.
    const int nw = flags[2], nx = flags[3];
    const int lo = nw < nx ? nw : nx, hi = nw < nx ? nx : nw;
    for (int n = lo; n < hi; ++n) mbar_arrive(&full[n % kStages]);
    for (int n = hi > kStages ? hi - kStages : 0; n < hi; ++n)
      mbar_wait(&full[n % kStages], static_cast<uint32_t>((n / kStages) & 1));
  }
  if (threadIdx.x == 0) {
    __threadfence();
    const int before = atomicAdd(p.cnt + kCntExit, 1);
    if (before == G - 1) {
      for (int i = 0; i < kCounters; ++i) atomicExch(p.cnt + i, 0);
      __threadfence();
    }
  }
  if (warp == 1) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "n"(512)
                 : "memory");
  }
}

// ------------------------------------------------------------------ planning

struct Plan {
  bool ok;
  int G, S0, T0, S2, T2, H1, T1;
};

Plan make_plan(int M, int mp, int d, int qd, int F) {
  Plan pl{};
  pl.ok = false;
  const int G = device_sm_count();
  if (M != 2 * mp || mp < 1 || mp > 64 || d % kTileN != 0 || qd % kBK != 0 || F % kBK != 0 ||
      d < kTileN)
    return pl;
  pl.G = G;
  pl.T0 = d / kTileN;
  const int kb0 = qd / kBK, kb2 = F / kBK;
  pl.S0 = G / pl.T0;
  if (pl.S0 < 1) pl.S0 = 1;
  if (pl.S0 > kb0) pl.S0 = kb0;
  pl.T2 = pl.T0;
  pl.S2 = G / pl.T2;
  if (pl.S2 < 1) pl.S2 = 1;
  if (pl.S2 > kb2) pl.S2 = kb2;
  // smallest multiple of 8 with at most G SwiGLU tiles
  int H = static_cast<int>(ceil_div(F, G));
  H = static_cast<int>(ceil_div(H, 8)) * 8;
  if (H < 8) H = 8;
  if (H > kMaxHalf) return pl;
  pl.H1 = H;
  pl.T1 = static_cast<int>(ceil_div(F, H));
  pl.ok = true;
  return pl;
}

size_t workspace_bytes(const Plan& pl) {
  const int units = pl.T0 * pl.S0 > pl.T2 * pl.S2 ? pl.T0 * pl.S0 : pl.T2 * pl.S2;
  return kCounterBytes + static_cast<size_t>(units) * kBM * kTileN * 4;
}

std::mutex g_mu;
bool g_attr[64] = {};

}  // namespace post
}  // namespace df

extern "C" size_t dualflow_layer_post_attention_workspace_size(int m_primary, int d_model,
                                                               int q_dim, int F) {
  const df::post::Plan pl = df::post::make_plan(2 * m_primary, m_primary, d_model, q_dim, F);
  return pl.ok ? df::post::workspace_bytes(pl) : 0;
}

extern "C" df_status dualflow_layer_post_attention(
    const void* attn, const void* x, const void* w_o, const void* w_gu, const void* w_down,
    const void* b, const void* c, int m_primary, int d_model, int q_dim, int F, float eps,
    void* x_mid, void* xn2, void* h, void* x_out, void* workspace, size_t workspace_bytes,
    int32_t* err_flag, void* stream) {
  using namespace df;
  using namespace df::post;
  if (!attn || !x || !w_o || !w_gu || !w_down || !x_mid || !xn2 || !h || !x_out)
    return DF_ERR_NULL;
  if (m_primary < 1 || d_model < 1 || q_dim < 1 || F < 1 || !(eps >= 0.f)) return DF_ERR_SHAPE;
  const int M = 2 * m_primary;
  const Plan pl = make_plan(M, m_primary, d_model, q_dim, F);
  if (!pl.ok) return DF_ERR_UNSUPPORTED;
  const void* ptrs[] = {attn, x, w_o, w_gu, w_down, x_mid, xn2, h, x_out};
  for (const void* ptr : ptrs)
    if (!aligned(ptr, 16)) return DF_ERR_ALIGN;
  if ((b && !aligned(b, 16)) || (c && !aligned(c, 16))) return DF_ERR_ALIGN;
  if (!workspace || workspace_bytes < df::post::workspace_bytes(pl) || !aligned(workspace, 256))
    return DF_ERR_WORKSPACE;

  Params p{};
  p.M = M;
  p.mp = m_primary;
  p.d = d_model;
  p.qd = q_dim;
  p.F = F;
  p.eps = eps;
  p.g[0] = Gemm{pl.T0 * pl.S0, pl.S0, q_dim / kBK, kTileN, 0, kTileN * kBK * 2,
                make_idesc(kBM, kTileN)};
  p.g[1] = Gemm{pl.T1, 1, d_model / kBK, 2 * pl.H1, pl.H1, 2 * pl.H1 * kBK * 2,
                make_idesc(kBM, 2 * pl.H1)};
  p.g[2] = Gemm{pl.T2 * pl.S2, pl.S2, F / kBK, kTileN, 0, kTileN * kBK * 2,
                make_idesc(kBM, kTileN)};
  p.r2_units = 2 * m_primary;
  p.x = static_cast<const __nv_bfloat16*>(x);
  p.b = static_cast<const __nv_bfloat16*>(b);
  p.c = static_cast<const __nv_bfloat16*>(c);
  p.x_mid = static_cast<__nv_bfloat16*>(x_mid);
  p.xn2 = static_cast<__nv_bfloat16*>(xn2);
  p.h = static_cast<__nv_bfloat16*>(h);
  p.x_out = static_cast<__nv_bfloat16*>(x_out);
  p.cnt = static_cast<int*>(workspace);
  p.part = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + kCounterBytes);
  p.err = err_flag;

  CUtensorMap tmXo, tmWo, tmXg, tmWg, tmXd, tmWd;
  const uint64_t Mu = static_cast<uint64_t>(M), du = static_cast<uint64_t>(d_model),
                 qu = static_cast<uint64_t>(q_dim), Fu = static_cast<uint64_t>(F);
  if (!encode_tmap_bf16_2d(&tmXo, attn, Mu, qu, qu * 2, kBM, kBK) ||
      !encode_tmap_bf16_2d(&tmWo, w_o, du, qu, qu * 2, kTileN, kBK) ||
      !encode_tmap_bf16_2d(&tmXg, xn2, Mu, du, du * 2, kBM, kBK) ||
      !encode_tmap_bf16_2d(&tmWg, w_gu, 2 * Fu, du, du * 2, static_cast<uint32_t>(pl.H1), kBK) ||
      !encode_tmap_bf16_2d(&tmXd, h, Mu, Fu, Fu * 2, kBM, kBK) ||
      !encode_tmap_bf16_2d(&tmWd, w_down, du, Fu, Fu * 2, kTileN, kBK))
    return DF_ERR_CUDA;

  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return DF_ERR_CUDA;
  {
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_attr[dev]) {
      if (cudaFuncSetAttribute(post_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(kSmemBytes)) != cudaSuccess)
        return DF_ERR_CUDA;
      g_attr[dev] = true;
    }
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(pl.G);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = static_cast<cudaStream_t>(stream);
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, post_kernel, tmXo, tmWo, tmXg, tmWg, tmXd, tmWd, p) != cudaSuccess)
    return DF_ERR_CUDA;
  return DF_OK;
}
