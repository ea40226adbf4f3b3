// Grouped shared-weight projection, tile-parallel / cluster split-K plan.
//
// Same product as the stream-K kernel (both flows' rows times one shared bf16
// weight, fp32 accumulation in TMEM, fused SwiGLU/residual/coupling epilogues;
// "Sintesi Tecnica: Dual-Flow Transformers", sections "Architettura Core" and
// "Meccanismi Chiave"), but every output tile is finished without fp32
// partials in global memory:
//  * the tile width BN (the MMA's N, a multiple of 16 up to 256) is chosen per
//    shape so that the tile count fills the 148 SMs; with C = 1 each CTA owns
//    whole tiles (persistent over tiles, two TMEM accumulators);
//  * when there are too few tiles, a thread-block cluster of C <= 8 CTAs
//    splits one tile's k-range. Each CTA parks its fp32 accumulator in shared
//    memory and writes it with one bulk TMA store to its slot of an
//    L2-resident workspace; after a cluster barrier each CTA bulk-loads the C
//    partials of its share of the tile's rows, sums them in rank order
//    (deterministic), applies the epilogue and stores. (Distributed shared
//    memory moves these ~100 KB per CTA at only ~20 GB/s per SM on B200; the
//    TMA engine through L2 is several times faster.)
// The producer/MMA/epilogue warp roles, the TMA ring and the bounded waits are
// as in the stream-K kernel.
#include <math.h>
#include <string.h>

#include <mutex>

#include "common.cuh"
#include "grouped_proj_tiles.h"
#include "host_util.h"
#include "umma.cuh"

namespace df {
namespace tgemm {

using namespace umma;

constexpr int kBM = 128;
constexpr int kBK = 64;
constexpr int kThreads = 192;
constexpr int kEpiThreads = 128;
constexpr int kMaxStages = 8;
constexpr int kXRows = 64;
constexpr int kXPitch = 33;
constexpr int kStgPitch = 36;
constexpr int kTileX = kBM * kBK * 2;  // 16 KB activation tile per stage
constexpr int kRingBytes = 196 * 1024;
// The ring plus the epilogue staging (the primary rows' results for the
// coupling and the output staging). A CTA with one tile and no cluster
// partner needs the staging only after its last MMA, when the ring is idle:
// its ring then spans the whole region (one stage more at the wide tiles).
constexpr int kStagingBytes = 64 * 33 * 4 + 4 * 32 * 36 * 4;
constexpr int kRingRegion = kRingBytes + kStagingBytes;
constexpr int kMaxCluster = 8;
constexpr int kSms = 148;
constexpr int kMaxOut = 256;  // output columns per tile (coupling prefetch buffer)
static_assert(kStagingBytes == kXRows * kXPitch * 4 + 4 * 32 * kStgPitch * 4, "staging size");
constexpr size_t kSmemBytes = 1024 + kRingRegion + kMaxOut * 4 + 256;

struct Params {
  int M, m_primary, n_out, n_aux, epilogue;
  int kblocks, BN, half, out_per_tile, n_tiles, C, stages, stage_bytes;
  int staging_in_ring;  // 1: the epilogue staging starts at the ring's base (see kRingRegion)
  int tpb;            // tiles per batch entry: tile t is (batch t / tpb, column tile t % tpb)
  int64_t ystride_b;  // output batch stride (elements)
  int batched;        // X / W tensor maps are 3-D (batch > 1); 2-D otherwise
  int pf_batched;     // the next projection's W map is 3-D
  uint32_t idesc;
  int F;
  __nv_bfloat16* y;
  int64_t ldy;
  const __nv_bfloat16* coupling;
  const __nv_bfloat16* residual;
  int64_t ldr;
  float* part;  // C > 1: [ctas][kBM][BN + 4] fp32 partial accumulators
  int32_t* err;
  // L2 prefetch for the next projection (pf_stages 0 = none): its plan's tile
  // width, cluster size, tile and CTA counts, k-blocks, SwiGLU half width and
  // gate/up offset; pf_stages k-blocks from the start of each of its CTAs'
  // slices.
  int pf_stages, pf_BN, pf_C, pf_ntiles, pf_ctas, pf_kblocks, pf_half, pf_F, pf_tpb;
};

__device__ __forceinline__ void epi_bar() {
  asm volatile("bar.sync 2, %0;" ::"n"(kEpiThreads) : "memory");
}

__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                   : "memory");
}

// Bulk (untiled) TMA copies; addresses 16-byte aligned, sizes multiples of 16.
__device__ __forceinline__ void bulk_store_s2g(void* gdst, uint32_t ssrc, uint32_t bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(gdst),
               "r"(ssrc), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void bulk_store_commit_and_wait() {
  asm volatile("cp.async.bulk.commit_group;\n\tcp.async.bulk.wait_group 0;" ::: "memory");
}
__device__ __forceinline__ void bulk_load_g2s(uint32_t sdst, const void* gsrc, uint32_t bytes,
                                              uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          sdst),
      "l"(gsrc), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

// Cluster plan (C > 1): rank q owns rows [lo, hi) of the rows it splits --
// the primary rows when a coupling pairs aux row m_primary + j with primary
// row j (both then belong to the same rank), else all M rows.
__device__ __forceinline__ void owned_rows(const Params& p, int q, int& lo, int& hi) {
  const int base = p.coupling != nullptr ? p.m_primary : p.M;
  lo = q * base / p.C;
  hi = (q + 1) * base / p.C;
}

__device__ __forceinline__ bool store_ok(const Params& p, int row, int col) {
  return row < p.M && col < p.n_out && !(row >= p.m_primary && col >= p.n_aux);
}

// Epilogue of one chunk of W output columns held row-wise (lane = row of this
// warp's TMEM quarter): coupling through shared memory, then residual add and
// bf16 store. W = 32 goes through the warp's staging tile so that stores are
// row-contiguous; W = 8 (tile tails) stores per row.
template <int W>
__device__ __forceinline__ void finish_chunk(const Params& p, __nv_bfloat16* y, int quarter,
                                             int lane, int col0, float (&val)[W], float* xbuf,
                                             float* stg, const float* cpl) {
  const int row = quarter * 32 + lane;
  if (p.coupling != nullptr) {
    if (row < p.m_primary) {
#pragma unroll
      for (int i = 0; i < W; ++i) xbuf[row * kXPitch + i] = val[i];
    }
    epi_bar();
    if (row >= p.m_primary && row < p.M) {
      const float* src = xbuf + (row - p.m_primary) * kXPitch;
#pragma unroll
      for (int i = 0; i < W; ++i) val[i] = fmaf(cpl[i], src[i], val[i]);
    }
    epi_bar();
  }
  if constexpr (W == 32) {
    float4* srow = reinterpret_cast<float4*>(stg + lane * kStgPitch);
#pragma unroll
    for (int i = 0; i < 8; ++i)
      srow[i] = make_float4(val[4 * i], val[4 * i + 1], val[4 * i + 2], val[4 * i + 3]);
    __syncwarp();
#pragma unroll
    for (int rr = 0; rr < 8; ++rr) {
      const int rl = rr * 4 + (lane >> 3), cg = (lane & 7) * 4;
      const int r = quarter * 32 + rl;
      if (!store_ok(p, r, col0 + cg)) continue;
      const float4 f = *reinterpret_cast<const float4*>(stg + rl * kStgPitch + cg);
      float o[4] = {f.x, f.y, f.z, f.w};
      if (p.epilogue == DF_EPI_RESIDUAL) {
        float rv[4];
        load_bf16x4(p.residual + r * p.ldr + col0 + cg, rv);
#pragma unroll
        for (int i = 0; i < 4; ++i) o[i] += rv[i];
      }
      store_bf16x4(y + r * p.ldy + col0 + cg, o);
    }
    __syncwarp();
  } else {
    if (store_ok(p, row, col0)) {
      if (p.epilogue == DF_EPI_RESIDUAL) {
        float rv[W];
        load_bf16<W>(p.residual + row * p.ldr + col0, rv);
#pragma unroll
        for (int i = 0; i < W; ++i) val[i] += rv[i];
      }
      store_bf16<W>(y + row * p.ldy + col0, val);
    }
  }
}

// Epilogue of a whole tile straight from TMEM (C = 1); tile = column tile,
// y = the output matrix of its batch entry.
__device__ void tile_epilogue(const Params& p, int tile, __nv_bfloat16* y, int quarter, int lane,
                              uint32_t taddr, float* xbuf, float* stg, const float* cpl_s) {
  const int col0 = tile * p.out_per_tile;
  if (p.epilogue == DF_EPI_SWIGLU) {
    const int H = p.half;
    int c = 0;
    for (; c + 32 <= H; c += 32) {
      float g[32], u[32];
      tmem_ld<32>(taddr + c, g);
      tmem_ld<32>(taddr + H + c, u);
#pragma unroll
      for (int i = 0; i < 32; ++i) g[i] = silu_f(g[i]) * u[i];
      finish_chunk<32>(p, y, quarter, lane, col0 + c, g, xbuf, stg, cpl_s + c);
    }
    for (; c < H; c += 8) {
      float g[8], u[8];
      tmem_ld<8>(taddr + c, g);
      tmem_ld<8>(taddr + H + c, u);
#pragma unroll
      for (int i = 0; i < 8; ++i) g[i] = silu_f(g[i]) * u[i];
      finish_chunk<8>(p, y, quarter, lane, col0 + c, g, xbuf, stg, cpl_s + c);
    }
  } else {
    int c = 0;
    for (; c + 32 <= p.BN; c += 32) {
      float v[32];
      tmem_ld<32>(taddr + c, v);
      finish_chunk<32>(p, y, quarter, lane, col0 + c, v, xbuf, stg, cpl_s + c);
    }
    for (; c < p.BN; c += 8) {
      float v[8];
      tmem_ld<8>(taddr + c, v);
      finish_chunk<8>(p, y, quarter, lane, col0 + c, v, xbuf, stg, cpl_s + c);
    }
  }
}

// C > 1: this CTA's rows of the tile, summed over the C partials loaded into
// `recv` ([src rank][own row][BN + 4] fp32, own primary rows first), in rank
// order, then the epilogue. Thread t keeps one 4-column group (t % groups)
// and walks rows t / groups, + nthreads / groups, ... two at a time, with
// the C partial loads of both rows issued before any sum (this loop runs on
// six warps, so its latency is not hidden by other warps).
template <int C>
__device__ void cluster_epilogue_c(const Params& p, int tile, __nv_bfloat16* y, int rank,
                                   const float* recv, float* prim, int tid, int nthreads,
                                   const __nv_bfloat16* res_s, const float* cpl_s) {
  const int pitch = p.BN + 4;
  const bool coupled = p.coupling != nullptr;
  const bool swiglu = p.epilogue == DF_EPI_SWIGLU;
  const bool resid = p.epilogue == DF_EPI_RESIDUAL;
  const int opt = p.out_per_tile;
  const int groups = opt / 4;  // 4-column groups per row
  int r0, r1;
  owned_rows(p, rank, r0, r1);
  const int n = r1 - r0;
  const int nloc = coupled ? 2 * n : n;
  const int rstep = nthreads / groups;
  const int g = tid % groups, rfirst = tid / groups;
  const int j = g * 4;
  const int col = tile * opt + j;
  const bool active = rfirst < rstep;
  float cv[4] = {0.f, 0.f, 0.f, 0.f};
  if (coupled && col < p.n_out) {
#pragma unroll
    for (int i = 0; i < 4; ++i) cv[i] = cpl_s[j + i];
  }
  for (int pass = 0; pass < (coupled ? 2 : 1); ++pass) {
    const int row_off = (pass == 1 ? p.m_primary : 0) + r0;
    for (int rl0 = rfirst; active && rl0 < n; rl0 += 2 * rstep) {
      float4 va[2][C], vu[2][C];
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        const int rl = rl0 + k * rstep;
        if (rl >= n) continue;
        const float* src = recv + (pass * n + rl) * pitch + j;
#pragma unroll
        for (int q = 0; q < C; ++q) {
          va[k][q] = *reinterpret_cast<const float4*>(src + q * nloc * pitch);
          if (swiglu) vu[k][q] = *reinterpret_cast<const float4*>(src + q * nloc * pitch + p.half);
        }
      }
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        const int rl = rl0 + k * rstep;
        if (rl >= n) continue;
        const int row = row_off + rl;
        float4 a = va[k][0], u = vu[k][0];
#pragma unroll
        for (int q = 1; q < C; ++q) {
          a.x += va[k][q].x; a.y += va[k][q].y; a.z += va[k][q].z; a.w += va[k][q].w;
          if (swiglu) {
            u.x += vu[k][q].x; u.y += vu[k][q].y; u.z += vu[k][q].z; u.w += vu[k][q].w;
          }
        }
        float o[4] = {a.x, a.y, a.z, a.w};
        if (swiglu) {
          o[0] = silu_f(a.x) * u.x;
          o[1] = silu_f(a.y) * u.y;
          o[2] = silu_f(a.z) * u.z;
          o[3] = silu_f(a.w) * u.w;
        }
        if (coupled && pass == 0) {
#pragma unroll
          for (int i = 0; i < 4; ++i) prim[rl * opt + j + i] = o[i];
        }
        if (coupled && pass == 1) {
#pragma unroll
          for (int i = 0; i < 4; ++i) o[i] = fmaf(cv[i], prim[rl * opt + j + i], o[i]);
        }
        if (!store_ok(p, row, col)) continue;
        if (resid) {
          float rv[4];
          if (res_s != nullptr) {
            load_bf16x4(res_s + (pass * n + rl) * opt + j, rv);
          } else {
            load_bf16x4(p.residual + row * p.ldr + col, rv);
          }
#pragma unroll
          for (int i = 0; i < 4; ++i) o[i] += rv[i];
        }
        store_bf16x4(y + row * p.ldy + col, o);
      }
    }
    if (coupled && pass == 0) __syncthreads();
  }
}

__device__ void cluster_epilogue(const Params& p, int tile, __nv_bfloat16* y, int rank,
                                 const float* recv, float* prim, int tid, int nthreads,
                                 const __nv_bfloat16* res_s, const float* cpl_s) {
  switch (p.C) {
    case 2: cluster_epilogue_c<2>(p, tile, y, rank, recv, prim, tid, nthreads, res_s, cpl_s); break;
    case 3: cluster_epilogue_c<3>(p, tile, y, rank, recv, prim, tid, nthreads, res_s, cpl_s); break;
    case 4: cluster_epilogue_c<4>(p, tile, y, rank, recv, prim, tid, nthreads, res_s, cpl_s); break;
    case 5: cluster_epilogue_c<5>(p, tile, y, rank, recv, prim, tid, nthreads, res_s, cpl_s); break;
    case 6: cluster_epilogue_c<6>(p, tile, y, rank, recv, prim, tid, nthreads, res_s, cpl_s); break;
    case 7: cluster_epilogue_c<7>(p, tile, y, rank, recv, prim, tid, nthreads, res_s, cpl_s); break;
    default: cluster_epilogue_c<8>(p, tile, y, rank, recv, prim, tid, nthreads, res_s, cpl_s); break;
  }
}

__global__ void __launch_bounds__(kThreads, 1)
    tile_gemm_kernel(const __grid_constant__ CUtensorMap tmX,
                     const __grid_constant__ CUtensorMap tmW,
                     const __grid_constant__ CUtensorMap tmWn, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  float* xbuf = reinterpret_cast<float*>(smem + (p.staging_in_ring ? 0 : kRingBytes));  // [64][33]
  float* stg_all = xbuf + kXRows * kXPitch;                        // 4 x [32][36]
  float* cpl_s = reinterpret_cast<float*>(smem + kRingRegion);     // [256] coupling of a tile
  uint64_t* full = reinterpret_cast<uint64_t*>(cpl_s + kMaxOut);
  uint64_t* empty = full + kMaxStages;
  uint64_t* acc_full = empty + kMaxStages;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* red_full = acc_empty + 2;  // C > 1: the partials of this CTA's rows have landed
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(red_full + 1);
  int* flags = reinterpret_cast<int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int S = p.stages;
  const int KB = p.kblocks;
  int tile_first, tile_stride, kb0, kb1, rank;
  if (p.C > 1) {
    tile_first = blockIdx.x / p.C;
    rank = blockIdx.x % p.C;
    tile_stride = p.n_tiles;  // one tile per cluster
    kb0 = rank * KB / p.C;
    kb1 = (rank + 1) * KB / p.C;
  } else {
    tile_first = blockIdx.x;
    rank = 0;
    tile_stride = gridDim.x;
    kb0 = 0;
    kb1 = KB;
  }
  const uint32_t tmem_cols = p.C > 1 ? 256u : 512u;

  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], kEpiThreads / 32);
    }
    mbar_init(red_full, 1);
    flags[0] = 0;  // a wait gave up
    flags[1] = 0;  // C > 1: the residual rows were prefetched into the staging area
    fence_barrier_init();
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"(tmem_cols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // Set-up above overlaps the previous kernel (programmatic dependent launch).
  // Global memory that it may write (activations, residual, coupling, the
  // output) only after the wait; the producer waits after its first weights.
  if (warp != 0) {
    pdl_wait();
    pdl_trigger();
  }

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    if (lane == 0) {
      prefetch_tensormap(&tmX);
      prefetch_tensormap(&tmW);
      const uint64_t pol_w = l2_policy_evict_first();
      const uint64_t pol_x = l2_policy_evict_last();
      // (e, tn) = (batch entry, column tile) of tile t, split once per tile:
      // nothing on the per-stage issue path divides (the ring is only a few
      // DRAM round trips deep, so issue latency costs bandwidth)
      auto load_w = [&](int s, int e, int tn, int kb) {
        uint8_t* sb = smem + s * p.stage_bytes + kTileX;
        const int r0 = p.epilogue == DF_EPI_SWIGLU ? tn * p.half : tn * p.BN;
        const int r1 = p.F + tn * p.half;
        if (p.batched) {
          tma_load_3d_hint(sb, &tmW, &full[s], kb * kBK, r0, e, pol_w);
          if (p.epilogue == DF_EPI_SWIGLU)
            tma_load_3d_hint(sb + p.half * 128, &tmW, &full[s], kb * kBK, r1, e, pol_w);
        } else {
          tma_load_2d_hint(sb, &tmW, &full[s], kb * kBK, r0, pol_w);
          if (p.epilogue == DF_EPI_SWIGLU)
            tma_load_2d_hint(sb + p.half * 128, &tmW, &full[s], kb * kBK, r1, pol_w);
        }
      };
      auto load_x = [&](uint8_t* sa, int s, int e, int kb) {
        if (p.batched)
          tma_load_3d_hint(sa, &tmX, &full[s], kb * kBK, 0, e, pol_x);
        else
          tma_load_2d_hint(sa, &tmX, &full[s], kb * kBK, 0, pol_x);
      };
      // The weights are no product of the previous kernel: the first ring
      // stages start streaming them before the wait for it.
      long long pre = 0;
      for (int t = tile_first; t < p.n_tiles && pre < S; t += tile_stride) {
        const int e = t / p.tpb, tn = t - e * p.tpb;
        for (int kb = kb0; kb < kb1 && pre < S; ++kb, ++pre) {
          mbar_arrive_expect_tx(&full[pre], p.stage_bytes);
          load_w(static_cast<int>(pre), e, tn, kb);
        }
      }
      pdl_wait();
      pdl_trigger();
      long long n = 0;
      int s = 0;         // n % S
      uint32_t ph = 0;   // (n / S) & 1
      bool ok = true;
      for (int t = tile_first; t < p.n_tiles && ok; t += tile_stride) {
        const int e = t / p.tpb, tn = t - e * p.tpb;
        for (int kb = kb0; kb < kb1; ++kb, ++n) {
          uint8_t* sa = smem + s * p.stage_bytes;
          if (n < pre) {  // weights already on their way
            load_x(sa, s, e, kb);
          } else {
            if (n >= S && !mbar_wait(&empty[s], ph ^ 1u)) {
              set_err(p.err, DF_DEVERR_TIMEOUT);
              ok = false;
              break;
            }
            mbar_arrive_expect_tx(&full[s], p.stage_bytes);
            load_x(sa, s, e, kb);
            load_w(s, e, tn, kb);
          }
          if (++s == S) {
            s = 0;
            ph ^= 1u;
          }
        }
      }
      for (long long i = (n > S ? n - S : 0); i < n; ++i)
        mbar_wait(&full[i % S], static_cast<uint32_t>((i / S) & 1));
      // This CTA's weights have landed: while the tile finishes (DRAM is
      // otherwise idle in the tail), warm L2 with the first k-blocks that the
      // next projection's CTAs j = blockIdx.x (mod gridDim.x) stream first.
      if (ok && p.pf_stages > 0) {
        prefetch_tensormap(&tmWn);
        for (int j = blockIdx.x; j < p.pf_ctas; j += gridDim.x) {
          int t = j, k0 = 0, k1 = p.pf_kblocks;
          if (p.pf_C > 1) {
            t = j / p.pf_C;
            const int r = j % p.pf_C;
            k0 = r * p.pf_kblocks / p.pf_C;
            k1 = (r + 1) * p.pf_kblocks / p.pf_C;
          }
          if (t >= p.pf_ntiles) continue;
          const int e = t / p.pf_tpb, tn = t - e * p.pf_tpb;
          const int r0 = p.pf_half > 0 ? tn * p.pf_half : tn * p.pf_BN;
          const int r1 = p.pf_F + tn * p.pf_half;
          for (int kb = k0; kb < k1 && kb < k0 + p.pf_stages; ++kb) {
            if (p.pf_batched) {
              tma_prefetch_3d(&tmWn, kb * kBK, r0, e);
              if (p.pf_half > 0) tma_prefetch_3d(&tmWn, kb * kBK, r1, e);
            } else {
              tma_prefetch_2d(&tmWn, kb * kBK, r0);
              if (p.pf_half > 0) tma_prefetch_2d(&tmWn, kb * kBK, r1);
            }
          }
        }
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      long long n = 0;
      int ms = 0;        // n % S
      uint32_t mph = 0;  // (n / S) & 1
      int seg = 0;
      bool ok = true;
      for (int t = tile_first; t < p.n_tiles && ok; t += tile_stride, ++seg) {
        const int acc = seg & 1;
        if (seg >= 2 && !mbar_wait(&acc_empty[acc], static_cast<uint32_t>(((seg >> 1) - 1) & 1))) {
          set_err(p.err, DF_DEVERR_TIMEOUT);
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * p.BN;
        for (int kb = kb0; kb < kb1; ++kb, ++n) {
          const int s = ms;  // n % S and (n / S) & 1, kept as counters
          if (!mbar_wait(&full[s], mph)) {
            set_err(p.err, DF_DEVERR_TIMEOUT);
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(smem + s * p.stage_bytes);
          const uint32_t b_addr = a_addr + kTileX;
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk) {
            umma_bf16(d_tmem, smem_desc(a_addr + kk * 32), smem_desc(b_addr + kk * 32), p.idesc,
                      (kb > kb0 || kk > 0) ? 1u : 0u);
          }
          umma_commit(&empty[s]);
          if (++ms == S) {
            ms = 0;
            mph ^= 1u;
          }
        }
        if (!ok) break;
        umma_commit(&acc_full[acc]);
      }
      if (n > 0) mbar_wait(&empty[(n - 1) % S], static_cast<uint32_t>(((n - 1) / S) & 1));
    }
  } else {
    // ---------------------------------------------------------------- epilogue warps
    const int quarter = warp & 3;
    const int et = threadIdx.x - 64;
    float* stg = stg_all + (warp - 2) * 32 * kStgPitch;
    if (p.C > 1) {
      // While the MMAs run: this rank's epilogue inputs into the (idle)
      // staging area -- the tile's coupling slice and, when they fit, the
      // residual rows it will write.
      const int opt = p.out_per_tile;
      const int col0 = (tile_first % p.tpb) * opt;  // coupling / residual: one batch entry
      const bool coupled = p.coupling != nullptr;
      const int rows_base = coupled ? p.m_primary : p.M;
      const int r0 = rank * rows_base / p.C, r1 = (rank + 1) * rows_base / p.C;
      const int nrows = (r1 - r0) * (coupled ? 2 : 1);
      if (coupled) {
        for (int i = et; i < opt; i += kEpiThreads)
          cpl_s[i] = (col0 + i < p.n_out) ? __bfloat162float(p.coupling[col0 + i]) : 0.f;
      }
      if (p.epilogue == DF_EPI_RESIDUAL && nrows * opt * 2 <= 4 * 32 * kStgPitch * 4) {
        __nv_bfloat16* rs = reinterpret_cast<__nv_bfloat16*>(stg_all);
        const int vec = opt / 8;  // 16-byte vectors per row
        for (int i = et; i < nrows * vec; i += kEpiThreads) {
          const int rl = i / vec, v = i % vec;
          const int pass = rl / (r1 - r0), rr = rl % (r1 - r0);
          const int row = (pass == 1 ? p.m_primary : 0) + r0 + rr;
          const int col = col0 + v * 8;
          uint4 val = make_uint4(0u, 0u, 0u, 0u);
          if (row < p.M && col < p.n_out)
            val = *reinterpret_cast<const uint4*>(p.residual + row * p.ldr + col);
          reinterpret_cast<uint4*>(rs)[i] = val;
        }
        if (et == 0) flags[1] = 1;
      }
    }
    int seg = 0;
    for (int t = tile_first; t < p.n_tiles; t += tile_stride, ++seg) {
      const int acc = seg & 1;
      if (p.C == 1 && p.coupling != nullptr) {
        // this tile's coupling vector, fetched while the MMAs run
        const int c0 = (t % p.tpb) * p.out_per_tile;
        for (int i = et; i < p.out_per_tile; i += kEpiThreads)
          cpl_s[i] = (c0 + i < p.n_out) ? __bfloat162float(p.coupling[c0 + i]) : 0.f;
      }
      const bool got = mbar_wait_warp(&acc_full[acc], static_cast<uint32_t>((seg >> 1) & 1));
      if (!got && lane == 0) atomicOr(&flags[0], 1);
      epi_bar();
      if (flags[0]) {
        if (et == 0) set_err(p.err, DF_DEVERR_TIMEOUT);
        break;
      }
      tc_fence_after();
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + acc * p.BN;
      if (p.C == 1) {
        tile_epilogue(p, t % p.tpb, p.y + (t / p.tpb) * p.ystride_b, quarter, lane, taddr, xbuf,
                      stg, cpl_s);
      } else {
        // park the fp32 accumulator rows in this CTA's shared memory (the ring
        // is idle: every stage has been consumed by the MMAs that completed)
        float* arow = reinterpret_cast<float*>(smem) + (quarter * 32 + lane) * (p.BN + 4);
        int c = 0;
        for (; c + 32 <= p.BN; c += 32) {
          float v[32];
          tmem_ld<32>(taddr + c, v);
#pragma unroll
          for (int i = 0; i < 8; ++i)
            reinterpret_cast<float4*>(arow + c)[i] =
                make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
        }
        for (; c < p.BN; c += 8) {
          float v[8];
          tmem_ld<8>(taddr + c, v);
          reinterpret_cast<float4*>(arow + c)[0] = make_float4(v[0], v[1], v[2], v[3]);
          reinterpret_cast<float4*>(arow + c)[1] = make_float4(v[4], v[5], v[6], v[7]);
        }
        fence_proxy_async_smem();  // the parked rows leave through a bulk TMA store
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[acc]);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const __nv_bfloat16* res_s =
      flags[1] ? reinterpret_cast<const __nv_bfloat16*>(stg_all) : nullptr;
  if (p.C > 1) {
    const int pitch = p.BN + 4;
    const size_t slot_floats = static_cast<size_t>(kBM) * pitch;
    if (threadIdx.x == 0) {
      // parked rows -> this CTA's slot (every parking thread fenced its writes
      // toward the async proxy before the CTA barrier above)
      bulk_store_s2g(p.part + blockIdx.x * slot_floats, smem_u32(smem),
                     static_cast<uint32_t>(slot_floats * 4));
      bulk_store_commit_and_wait();
      fence_proxy_async_global();
    }
    cluster_sync_all();  // every slot of the cluster is written; the rings are free
    int r0, r1;
    owned_rows(p, rank, r0, r1);
    const int n = r1 - r0;
    const bool coupled = p.coupling != nullptr;
    const int nloc = (coupled ? 2 : 1) * n;
    float* recv = reinterpret_cast<float*>(smem);  // [C][nloc][pitch]
    float* prim = recv + p.C * nloc * pitch;       // [n][out_per_tile]
    bool ok = !flags[0];
    if (threadIdx.x == 0) {
      fence_proxy_async_global();
      const uint32_t row_bytes = static_cast<uint32_t>(pitch * 4);
      mbar_arrive_expect_tx(red_full, static_cast<uint32_t>(p.C * nloc) * row_bytes);
      if (n > 0) {
        const float* base = p.part + (blockIdx.x - rank) * slot_floats;  // rank 0's slot
        for (int q = 0; q < p.C; ++q) {
          const float* slot = base + q * slot_floats;
          bulk_load_g2s(smem_u32(recv + (q * nloc) * pitch), slot + r0 * pitch,
                        static_cast<uint32_t>(n) * row_bytes, red_full);
          if (coupled)
            bulk_load_g2s(smem_u32(recv + (q * nloc + n) * pitch),
                          slot + (p.m_primary + r0) * pitch, static_cast<uint32_t>(n) * row_bytes,
                          red_full);
        }
      }
    }
    if (!mbar_wait(red_full, 0)) ok = false;
    ok = __syncthreads_and(ok) != 0;  // uniform: cluster_epilogue has CTA barriers
    if (!ok) {
      if (threadIdx.x == 0) set_err(p.err, DF_DEVERR_TIMEOUT);
    } else {
      cluster_epilogue(p, tile_first % p.tpb, p.y + (tile_first / p.tpb) * p.ystride_b, rank,
                       recv, prim, threadIdx.x, kThreads, res_s, cpl_s);
    }
  }
  if (warp == 1) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                 "r"(tmem_cols)
                 : "memory");
  }
}

// ------------------------------------------------------------------ planning

struct ClusterCaps {
  int max_clusters[kMaxCluster + 1];  // resident clusters of size C (0 = unavailable)
};

std::mutex g_mu;
bool g_attr_set[64] = {};
bool g_caps_ok[64] = {};
ClusterCaps g_caps[64];

// Resident-cluster capacity of this kernel on the current device, per cluster
// size (depends on the GPC layout); queried once per device.
const ClusterCaps* caps_for_device() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_attr_set[dev]) {
    if (cudaFuncSetAttribute(tile_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(kSmemBytes)) != cudaSuccess)
      return nullptr;
    g_attr_set[dev] = true;
  }
  if (!g_caps_ok[dev]) {
    ClusterCaps c{};
    for (int C = 1; C <= kMaxCluster; ++C) {
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(C * kSms);
      cfg.blockDim = dim3(kThreads);
      cfg.dynamicSmemBytes = kSmemBytes;
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = C;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      int n = 0;
      if (cudaOccupancyMaxActiveClusters(&n, tile_gemm_kernel, &cfg) != cudaSuccess) {
        cudaGetLastError();
        n = 0;
      }
      c.max_clusters[C] = n;
    }
    g_caps[dev] = c;
    g_caps_ok[dev] = true;
  }
  return &g_caps[dev];
}

struct Plan {
  bool ok;
  int BN, C, n_tiles, ctas, stages, stage_bytes;
  bool staging_in_ring;
  double est_us;
  int tpb;  // tiles per batch entry (n_tiles = batch * tpb)
};

// Pick the tile width and cluster size with the lowest modelled time. Rates:
// ~46 GB/s of DRAM and ~77 GB/s of total TMA traffic per SM (measured with a
// TMA streaming probe on B200), plus fixed costs for the cluster exchange and
// per-tile epilogues.
Plan make_plan(int M, int N, int K, int epilogue, const ClusterCaps* caps, size_t ws_bytes,
               int batch = 1) {
  Plan best{};
  best.ok = false;
  best.est_us = 1e30;
  const bool swiglu = epilogue == DF_EPI_SWIGLU;
  const int n_out = swiglu ? N / 2 : N;
  const int KB = K / kBK;
  for (int BN = 256; BN >= 64; BN -= 16) {
    const int opt = swiglu ? BN / 2 : BN;
    const int tpb = static_cast<int>(ceil_div(n_out, opt));
    const int n_tiles = tpb * batch;
    const int stage_bytes = kTileX + BN * 128;
    int stages = kRingBytes / stage_bytes;
    if (stages > kMaxStages) stages = kMaxStages;
    if (stages < 3) continue;
    int stages_region = kRingRegion / stage_bytes;  // one tile, no cluster partner
    if (stages_region > kMaxStages) stages_region = kMaxStages;
    for (int C = 1; C <= kMaxCluster && C <= KB; ++C) {
      int ctas, tpc;
      if (C == 1) {
        ctas = n_tiles < kSms ? n_tiles : kSms;
        tpc = static_cast<int>(ceil_div(n_tiles, ctas));
      } else {
        if (!caps || n_tiles > caps->max_clusters[C]) continue;
        // parked tile; then C partials of <= ceil(rows / C) (x2 coupled) own
        // rows plus the coupled primary results, all within the ring
        if (kBM * (BN + 4) * 4 > kRingBytes) continue;
        if ((kBM + 2 * C) * (BN + 4) * 4 + 32 * BN * 4 > kRingBytes) continue;
        if (static_cast<size_t>(n_tiles) * C * kBM * (BN + 4) * 4 > ws_bytes) continue;
        ctas = n_tiles * C;
        tpc = 1;
      }
      if (C > 1 && ctas > kSms) continue;
      const double kbpc = static_cast<double>(ceil_div(KB, C));
      const double w = tpc * kbpc * BN * 128.0;
      const double tot = tpc * kbpc * (BN * 128.0 + kTileX);
      double t = w / 46e3;  // bytes / (46 GB/s) in microseconds
      if (tot / 77e3 > t) t = tot / 77e3;
      t += (C > 1 ? 2.5 : 0.0) + tpc * 1.5 + 2.5;
      if (t < best.est_us) {
        const bool in_ring = C == 1 && tpc == 1;
        best = Plan{true, BN, C, n_tiles, ctas, in_ring ? stages_region : stages, stage_bytes,
                    in_ring, t, tpb};
      }
    }
  }
  (void)M;
  return best;
}

// Modelled time of the stream-K kernel for the same shape (same rates), used
// to choose between the two plans.
double stream_k_estimate(int N, int K, int epilogue) {
  const bool swiglu = epilogue == DF_EPI_SWIGLU;
  const int n_tiles = static_cast<int>(swiglu ? ceil_div(N / 2, 128) : ceil_div(N, 256));
  const double units = static_cast<double>(n_tiles) * (K / kBK);
  const double per_cta = units / kSms;
  double t = per_cta * 32768.0 / 46e3;
  const double tot = per_cta * 49152.0 / 77e3;
  if (tot > t) t = tot;
  const bool split = (static_cast<long long>(K / kBK) * n_tiles) % kSms != 0 || n_tiles < kSms;
  return t + 2.5 + 3.0 + (split ? 7.0 : 0.0);
}

// The tile plan is taken when it fills at least 3/4 of the SMs and beats the
// stream-K kernel run once per batch entry.
bool tile_plan_wins(const Plan& pl, int N, int K, int epilogue, int batch) {
  return pl.ok && pl.ctas >= kSms * 3 / 4 &&
         pl.est_us < batch * stream_k_estimate(N, K, epilogue);
}

int planned_launches(int M, int N, int K, int epilogue, size_t ws_bytes, int batch) {
  const Plan pl = make_plan(M, N, K, epilogue, caps_for_device(), ws_bytes, batch);
  return tile_plan_wins(pl, N, K, epilogue, batch) ? 1 : 0;
}

int launch_if_better(const Request& r) {
  const int M = r.m_primary + r.m_aux;
  const ClusterCaps* caps = caps_for_device();
  if (!caps) return 0;
  const int batch = r.batch > 0 ? r.batch : 1;
  const Plan pl =
      make_plan(M, r.N, r.K, r.epilogue, caps, r.workspace ? r.workspace_bytes : 0, batch);
  if (!tile_plan_wins(pl, r.N, r.K, r.epilogue, batch)) return 0;
  const bool swiglu = r.epilogue == DF_EPI_SWIGLU;
  Params p{};
  p.M = M;
  p.m_primary = r.m_primary;
  p.n_out = swiglu ? r.N / 2 : r.N;
  p.n_aux = r.n_aux;
  p.epilogue = r.epilogue;
  p.kblocks = r.K / kBK;
  p.BN = pl.BN;
  p.half = swiglu ? pl.BN / 2 : 0;
  p.out_per_tile = swiglu ? pl.BN / 2 : pl.BN;
  p.n_tiles = pl.n_tiles;
  p.tpb = pl.tpb;
  p.ystride_b = r.y_bstride;
  p.C = pl.C;
  p.stages = pl.stages;
  p.stage_bytes = pl.stage_bytes;
  p.staging_in_ring = pl.staging_in_ring ? 1 : 0;
  p.idesc = make_idesc(kBM, pl.BN);
  p.F = r.N / 2;
  p.y = static_cast<__nv_bfloat16*>(r.y);
  p.ldy = r.ldy;
  p.coupling = static_cast<const __nv_bfloat16*>(r.coupling);
  p.residual = static_cast<const __nv_bfloat16*>(r.residual);
  p.ldr = r.ldr;
  p.part = static_cast<float*>(r.workspace);
  p.err = r.err;
  CUtensorMap tmWn;
  memset(&tmWn, 0, sizeof(tmWn));
  if (r.w_next != nullptr) {
    const size_t ws = r.workspace ? r.workspace_bytes : 0;
    const int nb = r.batch_next > 0 ? r.batch_next : 1;
    const Plan nx = make_plan(M, r.N_next, r.K_next, r.epilogue_next, caps, ws, nb);
    const bool nx_tiles = tile_plan_wins(nx, r.N_next, r.K_next, r.epilogue_next, nb);
    const bool nx_swiglu = r.epilogue_next == DF_EPI_SWIGLU;
    const int box_rows = nx_swiglu ? nx.BN / 2 : nx.BN;
    const int64_t wn_stride =
        r.w_next_bstride > 0 ? r.w_next_bstride : static_cast<int64_t>(r.N_next) * r.K_next;
    const bool nx_map =
        nb > 1 ? encode_tmap_bf16_3d(&tmWn, r.w_next, static_cast<uint64_t>(nb),
                                     static_cast<uint64_t>(r.N_next),
                                     static_cast<uint64_t>(r.K_next),
                                     static_cast<uint64_t>(r.K_next) * 2,
                                     static_cast<uint64_t>(wn_stride) * 2, box_rows, kBK)
               : encode_tmap_bf16_2d(&tmWn, r.w_next, static_cast<uint64_t>(r.N_next),
                                     static_cast<uint64_t>(r.K_next),
                                     static_cast<uint64_t>(r.K_next) * 2, box_rows, kBK);
    if (nx_tiles && nx_map) {
      p.pf_batched = nb > 1 ? 1 : 0;
      // ~28 MB in all: what DRAM delivers in a few microseconds of tail
      const double per_stage = static_cast<double>(nx.ctas) * nx.BN * kBK * 2;
      int st = static_cast<int>(28.0 * 1024 * 1024 / per_stage);
      p.pf_stages = st < 1 ? 1 : (st > 16 ? 16 : st);
      p.pf_BN = nx.BN;
      p.pf_C = nx.C;
      p.pf_ntiles = nx.n_tiles;
      p.pf_ctas = nx.ctas;
      p.pf_kblocks = r.K_next / kBK;
      p.pf_half = nx_swiglu ? nx.BN / 2 : 0;
      p.pf_F = r.N_next / 2;
      p.pf_tpb = nx.tpb;
    }
  }
  CUtensorMap tmX, tmW;
  const int64_t xs = r.x_bstride > 0 ? r.x_bstride : static_cast<int64_t>(M) * r.ldx;
  const int64_t wsd = r.w_bstride > 0 ? r.w_bstride : static_cast<int64_t>(r.N) * r.K;
  // batch 1 keeps 2-D maps and loads (measured faster than a 3-D map whose
  // third dimension is 1)
  p.batched = batch > 1 ? 1 : 0;
  const uint32_t wbox = swiglu ? pl.BN / 2 : pl.BN;
  const bool maps_ok =
      batch > 1
          ? encode_tmap_bf16_3d(&tmX, r.x, static_cast<uint64_t>(batch), static_cast<uint64_t>(M),
                                static_cast<uint64_t>(r.K), static_cast<uint64_t>(r.ldx) * 2,
                                static_cast<uint64_t>(xs) * 2, kBM, kBK) &&
                encode_tmap_bf16_3d(&tmW, r.w, static_cast<uint64_t>(batch),
                                    static_cast<uint64_t>(r.N), static_cast<uint64_t>(r.K),
                                    static_cast<uint64_t>(r.K) * 2,
                                    static_cast<uint64_t>(wsd) * 2, wbox, kBK)
          : encode_tmap_bf16_2d(&tmX, r.x, static_cast<uint64_t>(M), static_cast<uint64_t>(r.K),
                                static_cast<uint64_t>(r.ldx) * 2, kBM, kBK) &&
                encode_tmap_bf16_2d(&tmW, r.w, static_cast<uint64_t>(r.N),
                                    static_cast<uint64_t>(r.K), static_cast<uint64_t>(r.K) * 2,
                                    wbox, kBK);
  if (!maps_ok) return -1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(pl.ctas);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = r.stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = pl.C;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  if (cudaLaunchKernelEx(&cfg, tile_gemm_kernel, tmX, tmW, tmWn, p) != cudaSuccess) return -1;
  return 1;
}

}  // namespace tgemm
}  // namespace df
