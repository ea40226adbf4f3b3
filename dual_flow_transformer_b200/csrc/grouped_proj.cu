// Grouped shared-weight projection on the 5th-generation tensor cores.
//
// Method: both flows share every attention, MLP and output matrix ("Sintesi
// Tecnica: Dual-Flow Transformers", section "Architettura Core"), so at a
// decode step the primary rows and the auxiliary rows are multiplied by the
// same weight in ONE GEMM and each weight byte is read from HBM once
// ("Costi di Inferenza": no growth in the unique weights read).
//
// Design (sm_100a, one CTA per SM, persistent stream-K):
//  * the whole M <= 128 rows form one UMMA M-tile; each k-step stages a
//    128 x 64 activation tile and a 256 x 64 weight tile (bf16, 128-byte
//    swizzle) by TMA into a 4-deep shared-memory ring. N = 256 per MMA halves
//    the activation bytes re-read from L2 per weight byte (with 128 columns
//    the L2 -> SM traffic, not DRAM, capped the weight stream);
//  * one elected thread issues tcgen05.mma (kind::f16, M=128, N=256, K=16,
//    fp32 accumulation in TMEM, two 256-column accumulators so the epilogue
//    of one segment overlaps the MMAs of the next) and tcgen05.commit frees
//    ring stages and publishes accumulators;
//  * the k-iterations of all tiles are divided evenly over the CTAs (stream-K)
//    so every SM streams the same number of weight bytes. A tile whose
//    k-range is cut between CTAs is published as fp32 partials (L2-resident
//    workspace) and summed by a second, fully parallel kernel in fixed
//    contributor order (deterministic); tiles owned by one CTA are finished
//    straight from TMEM;
//  * 4 epilogue warps read TMEM (tcgen05.ld 32x32b) and apply the fused
//    epilogue: plain store, SwiGLU with the b_l coupling, or residual add with
//    the c_l coupling. The coupling pairs auxiliary row m_primary + j with
//    primary row j of the same tile through shared memory.
// Every mbarrier wait is bounded; on a timeout the kernel flags it, drains its
// own copies/MMAs (bounded) and frees TMEM before returning.
#include <math.h>

#include "common.cuh"
#include "host_util.h"
#include "grouped_proj_tiles.h"
#include "umma.cuh"

namespace df {
namespace gemm {

using namespace umma;

constexpr int kBM = 128;           // rows per tile (all rows of both flows)
constexpr int kBN = 256;           // accumulator columns per tile (one N=256 MMA)
constexpr int kBK = 64;            // k per stage (one 128-byte swizzle atom)
constexpr int kStages = 4;
constexpr int kTileA = kBM * kBK * 2;   // 16 KB of activations
constexpr int kTileB = kBN * kBK * 2;   // 32 KB of weights
constexpr int kStageBytes = kTileA + kTileB;
constexpr int kThreads = 192;      // warp 0 TMA, warp 1 MMA/TMEM, warps 2-5 epilogue
constexpr int kEpiThreads = 128;
constexpr int kMaxCtas = 148;      // one CTA per SM of a B200
constexpr int kXRows = 64;         // coupled epilogues pair at most 64 primary rows
constexpr int kXPitch = 33;        // floats per row of the coupling exchange buffer
constexpr int kTmemCols = 512;     // two fp32 accumulators of 256 columns
constexpr int kRedThreads = 512;   // split-tile reduction: 16 rows x 32 column groups
constexpr int kStgPitch = 36;      // floats per row of a warp's 32 x 32 staging tile

struct Params {
  int M, m_primary, N, K, n_out, n_aux;
  int epilogue;
  int n_tiles, kblocks, ctas;
  long long total_iters;
  __nv_bfloat16* y;
  int64_t ldy;
  const __nv_bfloat16* coupling;
  const __nv_bfloat16* residual;
  int64_t ldr;
  float* partials;   // [2 * ctas][128][256] fp32
  int32_t* err;
  int F;             // SWIGLU: rows of W_gate (= output columns)
};

__host__ __device__ inline long long iter_begin(const Params& p, int cta) {
  return static_cast<long long>(cta) * p.total_iters / p.ctas;
}
__host__ __device__ inline int owner_of(const Params& p, long long it) {
  return static_cast<int>(((it + 1) * p.ctas - 1) / p.total_iters);
}
// First output column of a tile and output columns per tile.
__host__ __device__ inline int tile_col0(const Params& p, int tile) {
  return p.epilogue == DF_EPI_SWIGLU ? tile * (kBN / 2) : tile * kBN;
}

// kind::f16 instruction descriptor: D fp32, A/B bf16, both K-major, N=256, M=128.
constexpr uint32_t kIdesc = umma::make_idesc(kBM, kBN);

__device__ __forceinline__ void epi_bar() {
  asm volatile("bar.sync 2, %0;" ::"n"(kEpiThreads) : "memory");
}

// Residual add (RESIDUAL epilogue) and store of NV output columns of one row,
// honouring the output width and the auxiliary-row column limit.
template <int NV>
__device__ __forceinline__ void store_row(const Params& p, int row, int col0, float (&val)[NV]) {
  if (row >= p.M || col0 >= p.n_out) return;
  if (row >= p.m_primary && col0 >= p.n_aux) return;
  if (p.epilogue == DF_EPI_RESIDUAL) {
    float rv[NV];
    load_bf16<NV>(p.residual + row * p.ldr + col0, rv);
#pragma unroll
    for (int i = 0; i < NV; ++i) val[i] += rv[i];
  }
  store_bf16<NV>(p.y + row * p.ldy + col0, val);
}

// A warp holds a 32 x 32 fp32 block: lane = row (32 rows of its TMEM quarter),
// registers = 32 consecutive columns. Stage it through shared memory so that
// global stores are row-contiguous: each store instruction then covers 4 rows
// x 32 columns (8 lanes per row). Returns, per lane, 8 groups of 4 columns.
__device__ __forceinline__ void stage_block(const float (&v)[32], float* stg, int lane) {
  float4* srow = reinterpret_cast<float4*>(stg + lane * kStgPitch);
#pragma unroll
  for (int i = 0; i < 8; ++i) srow[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
  __syncwarp();
}

// fp32 partial of one 32-column chunk, coalesced (streamed to L2).
__device__ __forceinline__ void write_partial_chunk(const float (&v)[32], float* stg, float* slot,
                                                    int quarter, int c, int lane) {
  stage_block(v, stg, lane);
#pragma unroll
  for (int rr = 0; rr < 8; ++rr) {
    const int rl = rr * 4 + (lane >> 3), cg = (lane & 7) * 4;
    const float4 f = *reinterpret_cast<const float4*>(stg + rl * kStgPitch + cg);
    __stcg(reinterpret_cast<float4*>(slot + (quarter * 32 + rl) * kBN + 32 * c + cg), f);
  }
  __syncwarp();
}

// Epilogue of one 32-column output chunk of this warp's 32 rows (lane = row in
// `val`). Coupling: primary rows publish their values through shared memory,
// auxiliary rows add coupling[col] * value of their paired primary row. Then
// residual add and bf16 store, row-contiguous after the shared-memory transpose.
__device__ __forceinline__ void finish_chunk(const Params& p, int quarter, int lane, int col0,
                                             float (&val)[32], float* xbuf, float* stg) {
  const int row = quarter * 32 + lane;
  if (p.coupling != nullptr) {
    if (row < p.m_primary) {
#pragma unroll
      for (int i = 0; i < 32; ++i) xbuf[row * kXPitch + i] = val[i];
    }
    epi_bar();
    if (row >= p.m_primary && row < p.M && col0 < p.n_out) {
      float cv[32];
      load_bf16<32>(p.coupling + col0, cv);
      const float* src = xbuf + (row - p.m_primary) * kXPitch;
#pragma unroll
      for (int i = 0; i < 32; ++i) val[i] = fmaf(cv[i], src[i], val[i]);
    }
    epi_bar();
  }
  stage_block(val, stg, lane);
  if (col0 < p.n_out) {
#pragma unroll
    for (int rr = 0; rr < 8; ++rr) {
      const int rl = rr * 4 + (lane >> 3), cg = (lane & 7) * 4;
      const int r = quarter * 32 + rl;
      if (r >= p.M || (r >= p.m_primary && col0 >= p.n_aux)) continue;
      const float4 f = *reinterpret_cast<const float4*>(stg + rl * kStgPitch + cg);
      float o[4] = {f.x, f.y, f.z, f.w};
      if (p.epilogue == DF_EPI_RESIDUAL) {
        const uint2 u = *reinterpret_cast<const uint2*>(p.residual + r * p.ldr + col0 + cg);
        o[0] += bf16_bits_to_float(static_cast<uint16_t>(u.x & 0xffffu));
        o[1] += bf16_bits_to_float(static_cast<uint16_t>(u.x >> 16));
        o[2] += bf16_bits_to_float(static_cast<uint16_t>(u.y & 0xffffu));
        o[3] += bf16_bits_to_float(static_cast<uint16_t>(u.y >> 16));
      }
      *reinterpret_cast<uint2*>(p.y + r * p.ldy + col0 + cg) =
          make_uint2(pack_bf16x2(__float2bfloat16_rn(o[0]), __float2bfloat16_rn(o[1])),
                     pack_bf16x2(__float2bfloat16_rn(o[2]), __float2bfloat16_rn(o[3])));
    }
  }
  __syncwarp();
}

// Epilogue of a tile whose whole k-range this CTA accumulated (TMEM source).
__device__ void tile_epilogue_tmem(const Params& p, int tile, int quarter, int lane, uint32_t taddr,
                                   float* xbuf, float* stg) {
  const int col0 = tile_col0(p, tile);
  if (p.epilogue == DF_EPI_SWIGLU) {
#pragma unroll 1
    for (int c = 0; c < kBN / 64; ++c) {
      float g[32], u[32];
      tmem_ld<32>(taddr + 32 * c, g);
      tmem_ld<32>(taddr + kBN / 2 + 32 * c, u);
#pragma unroll
      for (int i = 0; i < 32; ++i) g[i] = silu_f(g[i]) * u[i];
      finish_chunk(p, quarter, lane, col0 + 32 * c, g, xbuf, stg);
    }
  } else {
#pragma unroll 1
    for (int c = 0; c < kBN / 32; ++c) {
      float v[32];
      tmem_ld<32>(taddr + 32 * c, v);
      finish_chunk(p, quarter, lane, col0 + 32 * c, v, xbuf, stg);
    }
  }
}

__device__ __forceinline__ const float* partial_row(const Params& p, int q, int tile, int row) {
  const int first_tile = static_cast<int>(iter_begin(p, q) / p.kblocks);
  const int slot = 2 * q + (first_tile == tile ? 0 : 1);
  return p.partials + (static_cast<size_t>(slot) * kBM + row) * kBN;
}

__global__ void __launch_bounds__(kThreads, 1)
    grouped_proj_kernel(const __grid_constant__ CUtensorMap tmX,
                        const __grid_constant__ CUtensorMap tmW, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  float* xbuf = reinterpret_cast<float*>(smem + kStages * kStageBytes);  // [64][33]
  float* stg_all = xbuf + kXRows * kXPitch;  // 4 epilogue warps x [32][36] (16-byte aligned)
  uint64_t* full = reinterpret_cast<uint64_t*>(stg_all + 4 * 32 * kStgPitch);
  uint64_t* empty = full + kStages;
  uint64_t* acc_full = empty + kStages;
  uint64_t* acc_empty = acc_full + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 2);
  int* flags = reinterpret_cast<int*>(tmem_slot + 1);  // [0] timeout

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int cta = blockIdx.x;
  const long long it_begin = iter_begin(p, cta);
  const long long it_end = iter_begin(p, cta + 1);

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], kEpiThreads / 32);
    }
    flags[0] = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)),
                 "n"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int KB = p.kblocks;
  // Set-up above overlaps the previous kernel (programmatic dependent launch).
  // Global memory that it may write (activations, residual, coupling,
  // partials, the output) only after the wait; the producer waits after its
  // first weights.
  if (warp != 0) {
    pdl_wait();
    pdl_trigger();
  }

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    if (lane == 0) {
      prefetch_tensormap(&tmX);
      prefetch_tensormap(&tmW);
      const uint64_t pol_w = l2_policy_evict_first();  // weights: streamed once
      const uint64_t pol_x = l2_policy_evict_last();   // activations: re-read by every CTA
      auto load_w = [&](int s, long long it) {
        const int tile = static_cast<int>(it / KB), kb = static_cast<int>(it % KB);
        uint8_t* sb = smem + s * kStageBytes + kTileA;
        if (p.epilogue == DF_EPI_SWIGLU) {
          tma_load_2d_hint(sb, &tmW, &full[s], kb * kBK, tile * (kBN / 2), pol_w);
          tma_load_2d_hint(sb + kTileB / 2, &tmW, &full[s], kb * kBK, p.F + tile * (kBN / 2),
                           pol_w);
        } else {
          tma_load_2d_hint(sb, &tmW, &full[s], kb * kBK, tile * kBN, pol_w);
        }
      };
      // The weights are no product of the previous kernel: the first ring
      // stages start streaming them before the wait for it.
      long long pre = 0;
      for (long long it = it_begin; it < it_end && pre < kStages; ++it, ++pre) {
        mbar_arrive_expect_tx(&full[pre], kStageBytes);
        load_w(static_cast<int>(pre), it);
      }
      pdl_wait();
      pdl_trigger();
      long long n = 0;  // stages issued
      for (long long it = it_begin; it < it_end; ++it, ++n) {
        const int s = static_cast<int>(n % kStages);
        const int kb = static_cast<int>(it % KB);
        uint8_t* sa = smem + s * kStageBytes;
        if (n < pre) {  // weights already on their way
          tma_load_2d_hint(sa, &tmX, &full[s], kb * kBK, 0, pol_x);
          continue;
        }
        if (n >= kStages && !mbar_wait(&empty[s], static_cast<uint32_t>(((n / kStages) - 1) & 1))) {
          set_err(p.err, DF_DEVERR_TIMEOUT);
          break;
        }
        mbar_arrive_expect_tx(&full[s], kStageBytes);
        tma_load_2d_hint(sa, &tmX, &full[s], kb * kBK, 0, pol_x);
        load_w(s, it);
      }
      // drain own copies still in flight
      for (long long i = (n > kStages ? n - kStages : 0); i < n; ++i)
        mbar_wait(&full[i % kStages], static_cast<uint32_t>((i / kStages) & 1));
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      long long n = 0;  // stages consumed
      int seg = 0;
      bool ok = true;
      long long it = it_begin;
      while (it < it_end && ok) {
        const int k0 = static_cast<int>(it % KB);
        const long long seg_len = min(static_cast<long long>(KB - k0), it_end - it);
        const int acc = seg & 1;
        if (seg >= 2 && !mbar_wait(&acc_empty[acc], static_cast<uint32_t>(((seg >> 1) - 1) & 1))) {
          set_err(p.err, DF_DEVERR_TIMEOUT);
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * kBN;
        for (long long j = 0; j < seg_len; ++j, ++n) {
          const int s = static_cast<int>(n % kStages);
          if (!mbar_wait(&full[s], static_cast<uint32_t>((n / kStages) & 1))) {
            set_err(p.err, DF_DEVERR_TIMEOUT);
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(smem + s * kStageBytes);
          const uint32_t b_addr = a_addr + kTileA;
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk) {
            umma_bf16(d_tmem, smem_desc(a_addr + kk * 32), smem_desc(b_addr + kk * 32), kIdesc,
                      (j > 0 || kk > 0) ? 1u : 0u);
          }
          umma_commit(&empty[s]);
        }
        if (!ok) break;
        umma_commit(&acc_full[acc]);
        it += seg_len;
        ++seg;
      }
      // drain: wait until the last committed MMAs have completed
      if (n > 0) mbar_wait(&empty[(n - 1) % kStages], static_cast<uint32_t>(((n - 1) / kStages) & 1));
    }
  } else {
    // ---------------------------------------------------------------- epilogue warps
    const int quarter = warp & 3;  // TMEM lane quarter this warp may access
    const int et = threadIdx.x - 64;  // 0..127
    float* stg = stg_all + (warp - 2) * 32 * kStgPitch;
    int seg = 0;
    long long it = it_begin;
    while (it < it_end) {
      const int tile = static_cast<int>(it / KB);
      const int k0 = static_cast<int>(it % KB);
      const long long seg_len = min(static_cast<long long>(KB - k0), it_end - it);
      const int acc = seg & 1;
      // bounded wait; the give-up decision is made uniform over the 4 warps
      const bool got = mbar_wait_warp(&acc_full[acc], static_cast<uint32_t>((seg >> 1) & 1));
      if (!got && lane == 0) atomicOr(&flags[0], 1);
      epi_bar();
      if (flags[0]) {
        if (et == 0) set_err(p.err, DF_DEVERR_TIMEOUT);
        break;
      }
      tc_fence_after();
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + acc * kBN;
      const long long t_first = static_cast<long long>(tile) * KB;
      if (owner_of(p, t_first) == owner_of(p, t_first + KB - 1)) {
        tile_epilogue_tmem(p, tile, quarter, lane, taddr, xbuf, stg);
      } else {
        // split tile: publish this CTA's fp32 partial; the reduce kernel sums them
        float* slot =
            p.partials + static_cast<size_t>(2 * cta + (it == it_begin ? 0 : 1)) * kBM * kBN;
#pragma unroll 1
        for (int c = 0; c < kBN / 32; ++c) {
          float v[32];
          tmem_ld<32>(taddr + 32 * c, v);
          write_partial_chunk(v, stg, slot, quarter, c, lane);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[acc]);
      it += seg_len;
      ++seg;
    }
  }

  // teardown: everyone done with TMEM before it is freed
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                 "n"(kTmemCols)
                 : "memory");
  }
}

// Sum of the fp32 partials of a split tile (contributors in k order, so the
// result is deterministic) followed by the same fused epilogue. One CTA per
// (tile, group of 16 rows), 512 threads = 16 rows x 32 column groups, two CTAs
// per SM; each thread keeps up to 4 contributors' loads in flight. A coupled group holds 8
// primary rows and their 8 paired auxiliary rows so the coupling stays inside
// the CTA.
__global__ void __launch_bounds__(kRedThreads, 2) reduce_kernel(const Params p) {
  const int tile = blockIdx.x, grp = blockIdx.y;
  pdl_wait();
  pdl_trigger();
  const long long t_first = static_cast<long long>(tile) * p.kblocks;
  const int q_a = owner_of(p, t_first), q_b = owner_of(p, t_first + p.kblocks - 1);
  if (q_a == q_b) return;  // handled by the GEMM kernel
  __shared__ float share[8][kBN];
  const int slot16 = threadIdx.x >> 5;  // row slot 0..15
  const int c = threadIdx.x & 31;       // column group 0..31
  const bool coupled = p.coupling != nullptr;
  int row;
  bool valid;
  if (coupled) {
    const int j = grp * 8 + (slot16 & 7);
    row = slot16 < 8 ? j : p.m_primary + j;
    valid = j < p.m_primary;
  } else {
    row = grp * 16 + slot16;
    valid = row < p.M;
  }
  const bool swiglu = p.epilogue == DF_EPI_SWIGLU;
  // accumulator columns of this thread: 8 contiguous (plain) or 4 gate + 4 up (SwiGLU)
  const int ca = swiglu ? 4 * c : 8 * c;
  const int cb = swiglu ? kBN / 2 + 4 * c : 8 * c + 4;
  float4 sa = make_float4(0.f, 0.f, 0.f, 0.f), sb = sa;
  if (valid) {
    for (int q0 = q_a; q0 <= q_b; q0 += 4) {
      float4 va[4], vb[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        if (q0 + i <= q_b) {
          const float* pr = partial_row(p, q0 + i, tile, row);
          va[i] = __ldcg(reinterpret_cast<const float4*>(pr + ca));
          vb[i] = __ldcg(reinterpret_cast<const float4*>(pr + cb));
        }
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        if (q0 + i <= q_b) {
          sa.x += va[i].x; sa.y += va[i].y; sa.z += va[i].z; sa.w += va[i].w;
          sb.x += vb[i].x; sb.y += vb[i].y; sb.z += vb[i].z; sb.w += vb[i].w;
        }
      }
    }
  }
  if (swiglu) {
    float v[4] = {silu_f(sa.x) * sb.x, silu_f(sa.y) * sb.y, silu_f(sa.z) * sb.z,
                  silu_f(sa.w) * sb.w};
    const int col0 = tile_col0(p, tile) + 4 * c;
    if (coupled) {
      if (slot16 < 8) {
#pragma unroll
        for (int i = 0; i < 4; ++i) share[slot16][4 * c + i] = v[i];
      }
      __syncthreads();
      if (slot16 >= 8 && valid && col0 < p.n_out) {
        const uint2 u = *reinterpret_cast<const uint2*>(p.coupling + col0);
        const float cv[4] = {bf16_bits_to_float(u.x & 0xffffu), bf16_bits_to_float(u.x >> 16),
                             bf16_bits_to_float(u.y & 0xffffu), bf16_bits_to_float(u.y >> 16)};
#pragma unroll
        for (int i = 0; i < 4; ++i) v[i] = fmaf(cv[i], share[slot16 - 8][4 * c + i], v[i]);
      }
    }
    if (!valid || row >= p.M || col0 >= p.n_out || (row >= p.m_primary && col0 >= p.n_aux)) return;
    const uint2 out = make_uint2(pack_bf16x2(__float2bfloat16_rn(v[0]), __float2bfloat16_rn(v[1])),
                                 pack_bf16x2(__float2bfloat16_rn(v[2]), __float2bfloat16_rn(v[3])));
    *reinterpret_cast<uint2*>(p.y + row * p.ldy + col0) = out;
  } else {
    float v[8] = {sa.x, sa.y, sa.z, sa.w, sb.x, sb.y, sb.z, sb.w};
    const int col0 = tile_col0(p, tile) + 8 * c;
    if (coupled) {
      if (slot16 < 8) {
#pragma unroll
        for (int i = 0; i < 8; ++i) share[slot16][8 * c + i] = v[i];
      }
      __syncthreads();
      if (slot16 >= 8 && valid && col0 < p.n_out) {
        float cv[8];
        load_bf16<8>(p.coupling + col0, cv);
#pragma unroll
        for (int i = 0; i < 8; ++i) v[i] = fmaf(cv[i], share[slot16 - 8][8 * c + i], v[i]);
      }
    }
    if (valid) store_row<8>(p, row, col0, v);
  }
}

struct Layout {
  int n_tiles, kblocks, ctas;
  long long total;
  size_t partial_bytes;
};

inline Layout make_layout(int N, int K, int epilogue) {
  Layout l;
  l.n_tiles = (epilogue == DF_EPI_SWIGLU) ? static_cast<int>(ceil_div(N / 2, kBN / 2))
                                          : static_cast<int>(ceil_div(N, kBN));
  l.kblocks = K / kBK;
  l.total = static_cast<long long>(l.n_tiles) * l.kblocks;
  l.ctas = static_cast<int>(l.total < kMaxCtas ? l.total : kMaxCtas);
  l.partial_bytes = static_cast<size_t>(2) * kMaxCtas * kBM * kBN * sizeof(float);
  return l;
}

constexpr size_t kSmemBytes =
    1024 + kStages * kStageBytes + kXRows * kXPitch * 4 + 4 * 32 * kStgPitch * 4 + 256;

}  // namespace gemm
}  // namespace df

extern "C" size_t dualflow_grouped_proj_workspace_size(int M, int N, int K, int epilogue) {
  using namespace df::gemm;
  if (M < 1 || N < 1 || K < 1 || epilogue < 0 || epilogue > 2) return 0;
  const Layout l = make_layout(N, K, epilogue);
  if (l.total < 1) return 0;
  return l.partial_bytes;
}

extern "C" int dualflow_grouped_proj_num_launches(int M, int N, int K, int epilogue) {
  using namespace df::gemm;
  if (M < 1 || N < 1 || K < 1 || epilogue < 0 || epilogue > 2) return 0;
  const Layout l = make_layout(N, K, epilogue);
  if (l.total < 1) return 0;
  if (df::tgemm::planned_launches(M, N, K, epilogue, l.partial_bytes)) return 1;
  Params p{};
  p.total_iters = l.total;
  p.ctas = l.ctas;
  for (int t = 0; t < l.n_tiles; ++t) {
    const long long f = static_cast<long long>(t) * l.kblocks;
    if (owner_of(p, f) != owner_of(p, f + l.kblocks - 1)) return 2;
  }
  return 1;
}

namespace {

df_status grouped_proj_impl(const void* x, int64_t ldx, int m_primary, int m_aux, const void* w,
                            int N, int K, int n_aux, void* y, int64_t ldy, int epilogue,
                            const void* coupling, const void* residual, int64_t ldr,
                            void* workspace, size_t workspace_bytes, const void* w_next,
                            int N_next, int K_next, int epilogue_next, int32_t* err_flag,
                            void* stream, int batch = 1, int64_t x_bstride = 0,
                            int64_t w_bstride = 0, int64_t y_bstride = 0, int batch_next = 1,
                            int64_t w_next_bstride = 0) {
  using namespace df;
  using namespace df::gemm;
  if (!x || !w || !y) return DF_ERR_NULL;
  if (w_next) {
    if (epilogue_next < DF_EPI_NONE || epilogue_next > DF_EPI_RESIDUAL) return DF_ERR_UNSUPPORTED;
    if (N_next < 128 || K_next < kBK || N_next % 128 != 0 || K_next % kBK != 0)
      return DF_ERR_UNSUPPORTED;
    if (!aligned(w_next, 16)) return DF_ERR_ALIGN;
  }
  if (epilogue < DF_EPI_NONE || epilogue > DF_EPI_RESIDUAL) return DF_ERR_UNSUPPORTED;
  if (epilogue == DF_EPI_RESIDUAL && !residual) return DF_ERR_NULL;
  if (epilogue == DF_EPI_NONE && (coupling || residual)) return DF_ERR_SHAPE;
  const int M = m_primary + m_aux;
  if (m_primary < 0 || m_aux < 0 || M < 1 || N < 1 || K < 1) return DF_ERR_SHAPE;
  if (coupling && m_aux != m_primary) return DF_ERR_SHAPE;
  if (M > kBM) return DF_ERR_UNSUPPORTED;
  if (K % kBK != 0) return DF_ERR_UNSUPPORTED;
  if (N % 128 != 0) return DF_ERR_UNSUPPORTED;  // SWIGLU: F = N / 2 must be a multiple of 64
  const int n_out = epilogue == DF_EPI_SWIGLU ? N / 2 : N;
  if (n_aux < 0 || n_aux > n_out) return DF_ERR_SHAPE;
  if (n_aux % 32 != 0 && n_aux != n_out) return DF_ERR_UNSUPPORTED;
  const int64_t lx = ldx ? ldx : K, ly = ldy ? ldy : n_out, lr = ldr ? ldr : n_out;
  if (lx < K || ly < n_out || (residual && lr < n_out)) return DF_ERR_SHAPE;
  if (lx % 8 || ly % 8 || (residual && lr % 8)) return DF_ERR_ALIGN;
  if (!aligned(x, 16) || !aligned(w, 16) || !aligned(y, 16) || (residual && !aligned(residual, 16)) ||
      (coupling && !aligned(coupling, 16)))
    return DF_ERR_ALIGN;
  const Layout l = make_layout(N, K, epilogue);
  if (l.n_tiles > 65535) return DF_ERR_UNSUPPORTED;
  const size_t need = l.partial_bytes;
  if (!workspace || workspace_bytes < need || !aligned(workspace, 256)) return DF_ERR_WORKSPACE;

  Params p{};
  p.M = M;
  p.m_primary = m_primary;
  p.N = N;
  p.K = K;
  p.n_aux = n_aux;
  p.n_out = n_out;
  p.epilogue = epilogue;
  p.n_tiles = l.n_tiles;
  p.kblocks = l.kblocks;
  p.ctas = l.ctas;
  p.total_iters = l.total;
  p.y = static_cast<__nv_bfloat16*>(y);
  p.ldy = ly;
  p.coupling = static_cast<const __nv_bfloat16*>(coupling);
  p.residual = static_cast<const __nv_bfloat16*>(residual);
  p.ldr = lr;
  p.partials = static_cast<float*>(workspace);
  p.err = err_flag;
  p.F = N / 2;

  cudaStream_t st = static_cast<cudaStream_t>(stream);
  {
    // tile-parallel / cluster split-K plan when it is modelled to be faster
    tgemm::Request rq{x, lx, m_primary, m_aux, w, N, K, n_aux, y, ly, epilogue, coupling,
                      residual, lr, err_flag, st, workspace, workspace_bytes,
                      w_next, N_next, K_next, epilogue_next, batch, x_bstride, w_bstride,
                      y_bstride, batch_next, w_next_bstride};
    const int launched = tgemm::launch_if_better(rq);
    if (launched < 0) return DF_ERR_CUDA;
    if (launched > 0) return DF_OK;
  }
  if (batch > 1) {  // no single-launch plan: one projection per batch entry
    for (int b = 0; b < batch; ++b) {
      const df_status sb = grouped_proj_impl(
          static_cast<const __nv_bfloat16*>(x) + b * x_bstride, ldx, m_primary, m_aux,
          static_cast<const __nv_bfloat16*>(w) + b * w_bstride, N, K, n_aux,
          static_cast<__nv_bfloat16*>(y) + b * y_bstride, ldy, epilogue, nullptr, nullptr, 0,
          workspace, workspace_bytes, nullptr, 0, 0, 0, err_flag, stream);
      if (sb != DF_OK) return sb;
    }
    return DF_OK;
  }
  CUtensorMap tmX, tmW;
  if (!encode_tmap_bf16_2d(&tmX, x, static_cast<uint64_t>(M), static_cast<uint64_t>(K),
                           static_cast<uint64_t>(lx) * 2, kBM, kBK) ||
      !encode_tmap_bf16_2d(&tmW, w, static_cast<uint64_t>(N), static_cast<uint64_t>(K),
                           static_cast<uint64_t>(K) * 2,
                           epilogue == DF_EPI_SWIGLU ? kBN / 2 : kBN, kBK))
    return DF_ERR_CUDA;
  if (ensure_dynamic_smem(reinterpret_cast<const void*>(grouped_proj_kernel), kSmemBytes) !=
      cudaSuccess)
    return DF_ERR_CUDA;
  if (launch_pdl(grouped_proj_kernel, dim3(l.ctas), dim3(kThreads), kSmemBytes, st, tmX, tmW, p) !=
      cudaSuccess)
    return DF_ERR_CUDA;
  // split tiles (a k-range shared by several CTAs) are summed by a second kernel
  bool any_split = false;
  for (int t = 0; t < l.n_tiles && !any_split; ++t) {
    const long long f = static_cast<long long>(t) * l.kblocks;
    any_split = owner_of(p, f) != owner_of(p, f + l.kblocks - 1);
  }
  if (any_split) {
    const int groups = coupling ? static_cast<int>(ceil_div(m_primary, 8))
                                : static_cast<int>(ceil_div(M, 16));
    if (launch_pdl(reduce_kernel, dim3(l.n_tiles, groups), dim3(kRedThreads), 0, st, p) !=
        cudaSuccess)
      return DF_ERR_CUDA;
  }
  return cudaGetLastError() == cudaSuccess ? DF_OK : DF_ERR_CUDA;
}

}  // namespace

extern "C" df_status dualflow_grouped_proj(const void* x, int64_t ldx, int m_primary, int m_aux,
                                           const void* w, int N, int K, int n_aux, void* y,
                                           int64_t ldy, int epilogue, const void* coupling,
                                           const void* residual, int64_t ldr, void* workspace,
                                           size_t workspace_bytes, int32_t* err_flag,
                                           void* stream) {
  return grouped_proj_impl(x, ldx, m_primary, m_aux, w, N, K, n_aux, y, ldy, epilogue, coupling,
                           residual, ldr, workspace, workspace_bytes, nullptr, 0, 0, 0, err_flag,
                           stream);
}

extern "C" df_status dualflow_grouped_proj_batched(
    const void* x, int64_t ldx, int64_t x_bstride, int m_primary, int m_aux, const void* w, int N,
    int K, int64_t w_bstride, void* y, int64_t ldy, int64_t y_bstride, int batch, int epilogue,
    void* workspace, size_t workspace_bytes, const void* w_next, int N_next, int K_next,
    int epilogue_next, int batch_next, int64_t w_next_bstride, int32_t* err_flag, void* stream) {
  using namespace df;
  if (!x || !w || !y) return DF_ERR_NULL;
  if (batch < 1 || batch > 65535 || (w_next && (batch_next < 1 || batch_next > 65535)))
    return DF_ERR_SHAPE;
  if (epilogue != DF_EPI_NONE && epilogue != DF_EPI_SWIGLU) return DF_ERR_UNSUPPORTED;
  const int M = m_primary + m_aux;
  const int n_out = epilogue == DF_EPI_SWIGLU ? N / 2 : N;
  const int64_t lx = ldx ? ldx : K, ly = ldy ? ldy : n_out;
  const int64_t xs = x_bstride ? x_bstride : lx * M;
  const int64_t wsd = w_bstride ? w_bstride : static_cast<int64_t>(N) * K;
  const int64_t ys = y_bstride ? y_bstride : ly * M;
  if (M < 1 || N < 1 || K < 1 || xs < lx * M || wsd < static_cast<int64_t>(N) * K ||
      ys < ly * M)
    return DF_ERR_SHAPE;
  if (xs % 8 || wsd % 8 || ys % 8) return DF_ERR_ALIGN;
  const int64_t wns = w_next_bstride ? w_next_bstride : static_cast<int64_t>(N_next) * K_next;
  if (w_next && (wns < static_cast<int64_t>(N_next) * K_next || wns % 8)) return DF_ERR_SHAPE;
  return grouped_proj_impl(x, lx, m_primary, m_aux, w, N, K, n_out, y, ly, epilogue, nullptr,
                           nullptr, 0, workspace, workspace_bytes, w_next, N_next, K_next,
                           epilogue_next, err_flag, stream, batch, xs, wsd, ys,
                           w_next ? batch_next : 1, wns);
}

extern "C" int dualflow_grouped_proj_batched_num_launches(int M, int N, int K, int epilogue,
                                                          int batch) {
  using namespace df::gemm;
  if (M < 1 || N < 1 || K < 1 || batch < 1 || (epilogue != DF_EPI_NONE && epilogue != DF_EPI_SWIGLU))
    return 0;
  const Layout l = make_layout(N, K, epilogue);
  if (l.total < 1) return 0;
  if (df::tgemm::planned_launches(M, N, K, epilogue, l.partial_bytes, batch)) return 1;
  return batch * dualflow_grouped_proj_num_launches(M, N, K, epilogue);
}

extern "C" df_status dualflow_grouped_proj_chain(
    const void* x, int64_t ldx, int m_primary, int m_aux, const void* w, int N, int K, int n_aux,
    void* y, int64_t ldy, int epilogue, const void* coupling, const void* residual, int64_t ldr,
    void* workspace, size_t workspace_bytes, const void* w_next, int N_next, int K_next,
    int epilogue_next, int32_t* err_flag, void* stream) {
  return grouped_proj_impl(x, ldx, m_primary, m_aux, w, N, K, n_aux, y, ldy, epilogue, coupling,
                           residual, ldr, workspace, workspace_bytes, w_next, N_next, K_next,
                           epilogue_next, err_flag, stream);
}
