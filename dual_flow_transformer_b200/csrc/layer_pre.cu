// Pre-attention half of the Dual-Flow decoder layer as ONE launch of 4-CTA
// clusters: RMSNorm, the grouped QKV projection and the primary-only KV append.
//
// Method: "Sintesi Tecnica: Dual-Flow Transformers", sections "Architettura
// Core" (both flows share the projection matrices; only the primary flow
// writes the persistent KV cache; the auxiliary flow needs only its query) and
// "Costi di Inferenza vs. Addestramento" (grouped decode reads the unique
// weights once for both flows). With X = [primary rows; auxiliary rows]:
//   r     = 1 / sqrt(mean(x^2) + eps)                   (RMSNorm, unit gain)
//   qkv   = bf16(r (x W_qkv^T))   primary rows: Q, K, V columns;
//                                 auxiliary rows: Q columns only
//   cache[page of positions[b]][g][slot][:] = the primary row b's K / V
//   columns of KV head g (the same bf16 values), nothing else.
// The row scale multiplies the accumulator (r (x W^T) = (r x) W^T), so the
// normalised rows are never rounded to bf16 and stored.
//
// Layout of the work: the Q, K, V columns are cut into T column tiles of TN
// (a multiple of 32, at most 256), one per cluster; rank r of the cluster
// multiplies the r-th quarter of K, so its 4 CTAs stream disjoint quarters of
// the tile's weights. A rank's epilogue warps also add up, from the
// activation tiles already in its shared-memory ring, each row's squares over
// its quarter. When the four partial products are done, a cluster barrier
// retires the ring, which then becomes the receive buffer of a reduce-scatter
// through distributed shared memory: rank r owns columns r TN/4 .. of the
// tile, the others write their fp32 slices of those columns (and their row
// sums of squares) into it with st.async, and r adds the four in rank order.
// There is one phase and no grid-wide dependency: no counters, no workspace.
// Roles (224 threads): warp 0 weight producer, warp 1 MMA issuer (one thread,
// tcgen05.mma M = 128, N = TN, fp32 accumulator in TMEM), warp 2 activation
// producer, warps 3-6 epilogue (TMEM lane quarter = warp % 4, thread = row).
// Sums are taken in a fixed order: results are deterministic, and primary
// rows never read auxiliary rows.
#include <math.h>
#include <string.h>

#include <mutex>

#include "cluster.cuh"
#include "common.cuh"
#include "host_util.h"
#include "umma.cuh"

namespace df {
namespace pre {

using namespace umma;
using namespace cl;

constexpr int kBM = 128;
constexpr int kBK = 64;
constexpr int kThreads = 224;  // warps 3-6: the 128 epilogue threads of cl::epi_bar
constexpr int kCluster = 4;
constexpr int kMaxTileN = 256;
constexpr int kMaxStages = 8;
constexpr int kXBytes = kBM * kBK * 2;     // 16 KB activation tile
constexpr size_t kRingBytes = 208 * 1024;  // e.g. 5 stages of 16 + 24 KB at TN = 192
constexpr size_t kSmemBytes = 1024 + kRingBytes + 512;  // + barriers, flags
// The retired ring holds the receive buffer [3 senders][TN/16 + 1 chunks][128
// rows][16 B] and, after it, the outgoing slices in the same layout.
static_assert(6 * (kMaxTileN / 16 + 1) * kBM * 16 <= kRingBytes, "reduce buffers fit the ring");
static_assert(kSmemBytes <= 232448, "shared memory budget");

struct Params {
  int M, mp, d;
  int nq;    // Q columns (Hq * D)
  int nout;  // Q, K and V columns (Hq * D + 2 Hkv * D)
  int TN;    // columns per tile (cluster)
  int kblocks, nst, stage, w_bytes;
  uint32_t idesc;
  float eps;
  __nv_bfloat16* qkv;  // [M][nout]
  __nv_bfloat16* k_cache;
  __nv_bfloat16* v_cache;
  const int32_t* block_table;
  const int32_t* positions;
  int max_blocks, Hkv, D, block_size, num_blocks;
  int32_t* err;
  // partials mode (part != nullptr): each rank stores its fp32 partial
  // product [rank][row][column] and the first cluster each rank's row sums
  // of squares ss_out [rank][row]; no reduction, no norm, no append here
  float* part;
  float* ss_out;
};

// Cache element offset of (sequence b, KV head 0, dimension 0) at b's
// position (head g adds g block_size D), or -1 (and the error bit) when b's
// position or page is outside the table.
__device__ __forceinline__ int64_t cache_row_base(const Params& p, int b) {
  const int pos = p.positions[b];
  if (pos < 0 || pos / p.block_size >= p.max_blocks) {
    set_err(p.err, DF_DEVERR_POSITION);
    return -1;
  }
  const int page =
      p.block_table[static_cast<int64_t>(b) * p.max_blocks + pos / p.block_size];
  if (page < 0 || page >= p.num_blocks) {
    set_err(p.err, DF_DEVERR_BLOCK);
    return -1;
  }
  return (static_cast<int64_t>(page) * p.Hkv * p.block_size + pos % p.block_size) * p.D;
}

// 8 bf16 values (16 bytes) from 8 floats.
__device__ __forceinline__ uint4 pack8(const float (&v)[8]) {
  uint32_t w[4];
#pragma unroll
  for (int k = 0; k < 4; ++k)
    w[k] = pack_bf16x2(__float2bfloat16_rn(v[2 * k]), __float2bfloat16_rn(v[2 * k + 1]));
  return make_uint4(w[0], w[1], w[2], w[3]);
}

__global__ void __launch_bounds__(kThreads, 1)
    pre_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
               const __grid_constant__ CUtensorMap tmP, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* recv = smem;  // the ring, once retired
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kRingBytes);  // [kMaxStages]
  uint64_t* empty = full + kMaxStages;                              // [kMaxStages]
  uint64_t* acc_full = empty + kMaxStages;
  uint64_t* mma_done = acc_full + 1;
  uint64_t* red_full = mma_done + 1;  // this rank's slices from the other 3 ranks have landed
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(red_full + 1);
  volatile int* flags = reinterpret_cast<volatile int*>(tmem_slot + 1);  // [0] abort
  int* fills = reinterpret_cast<int*>(tmem_slot + 2);  // [2][kMaxStages]: weight / activation

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const int tile = static_cast<int>(cluster_index());
  const int k0 = static_cast<int>(rank) * p.kblocks / kCluster;
  const int k1 = (static_cast<int>(rank) + 1) * p.kblocks / kCluster;
  const int W = p.TN / kCluster;                     // columns this rank owns
  const int nchunk = W / 4;                          // its 4-column chunks
  const int slot_bytes = (nchunk + 1) * kBM * 16;    // + one chunk of row sums of squares

  if (threadIdx.x == 0) {
    for (int i = 0; i < kMaxStages; ++i) {
      mbar_init(&full[i], 2);           // weight producer + activation producer
      mbar_init(&empty[i], 1 + 4);      // MMA commit + the 4 epilogue warps (row sums)
      fills[i] = 0;
      fills[kMaxStages + i] = 0;
    }
    mbar_init(acc_full, 1);
    mbar_init(mma_done, 1);
    mbar_init(red_full, 1);  // this rank's expect_tx arrival + the senders' bytes
    flags[0] = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)),
                 "n"(kMaxTileN)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  // every CTA of the cluster has initialised its barriers before any remote write
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // Only the weight producer may run ahead of the kernel launched before this
  // one (the weights are constants); every other role waits for it first.
  if (warp != 0) pdl_wait();

  bool ok = true;
  if (warp == 0 || warp == 2) {
    // ------------------------------------------------------------ producers
    if (lane == 0) {
      const bool wrole = warp == 0;
      prefetch_tensormap(wrole ? &tmW : &tmX);
      const uint64_t pol = wrole ? l2_policy_evict_first() : l2_policy_evict_last();
      int* fl = fills + (wrole ? 0 : kMaxStages);
      int s = 0;
      uint32_t ph = 0;
      for (int kb = k0, n = 0; kb < k1; ++kb, ++n) {
        if (n >= p.nst && !mbar_wait(&empty[s], ph ^ 1u)) {
          set_err(p.err, DF_DEVERR_TIMEOUT);
          flags[0] = 1;
          break;
        }
        if (flags[0]) break;
        uint8_t* st = smem + static_cast<size_t>(s) * p.stage;
        if (wrole) {
          mbar_arrive_expect_tx(&full[s], static_cast<uint32_t>(p.w_bytes));
          tma_load_2d_hint(st + kXBytes, &tmW, &full[s], kb * kBK, tile * p.TN, pol);
        } else {
          mbar_arrive_expect_tx(&full[s], kXBytes);
          tma_load_2d_hint(st, &tmX, &full[s], kb * kBK, 0, pol);
        }
        ++fl[s];
        if (++s == p.nst) {
          s = 0;
          ph ^= 1u;
        }
      }
      if (wrole) pdl_trigger();
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0;
      bool mok = true;
      for (int kb = k0; kb < k1; ++kb) {
        if (!mbar_wait(&full[s], ph) || flags[0]) {
          set_err(p.err, DF_DEVERR_TIMEOUT);
          flags[0] = 1;
          mok = false;
          break;
        }
        tc_fence_after();
        const uint32_t a_addr = smem_u32(smem + static_cast<size_t>(s) * p.stage);
        const uint32_t b_addr = a_addr + kXBytes;
#pragma unroll
        for (int kk = 0; kk < kBK / 16; ++kk)
          umma_bf16(tmem_base, smem_desc(a_addr + kk * 32), smem_desc(b_addr + kk * 32), p.idesc,
                    (kb > k0 || kk > 0) ? 1u : 0u);
        umma_commit(&empty[s]);
        if (++s == p.nst) {
          s = 0;
          ph ^= 1u;
        }
      }
      // (a rank without k-blocks commits at once: its partial is zero)
      if (mok) umma_commit(acc_full);
      // no tensor-core operation may still be reading shared memory or TMEM
      // past this point (this commit completes after every MMA above)
      umma_commit(mma_done);
      mbar_wait(mma_done, 0);
    }
  } else {
    // ------------------------------------------------------------ epilogue warps:
    // this row's sum of squares over this rank's K quarter, from the
    // activation tiles in the ring (a row's 128 bytes in any chunk order)
    const int row = (warp & 3) * 32 + lane;
    // a primary row's cache slot, looked up while the MMAs run
    const int64_t cbase = (p.part == nullptr && row < p.mp) ? cache_row_base(p, row) : -1;
    float ss = 0.f;
    int s = 0;
    uint32_t ph = 0;
    for (int kb = k0; kb < k1; ++kb) {
      if (!mbar_wait(&full[s], ph)) {
        ok = false;
        break;
      }
      const uint8_t* xr = smem + static_cast<size_t>(s) * p.stage + row * 128;
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const uint4 u = *reinterpret_cast<const uint4*>(xr + ((c ^ (row & 7)) * 16));
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float a = bf16_bits_to_float(static_cast<uint16_t>(w[k] & 0xffffu));
          const float b = bf16_bits_to_float(static_cast<uint16_t>(w[k] >> 16));
          ss = fmaf(a, a, ss);
          ss = fmaf(b, b, ss);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
      if (++s == p.nst) {
        s = 0;
        ph ^= 1u;
      }
    }
    ok = __all_sync(0xffffffffu, ok);
    ok = ok && mbar_wait_warp(acc_full, 0);
    ok = epi_bar_and(ok);
    if (!ok && lane == 0) {
      set_err(p.err, DF_DEVERR_TIMEOUT);
      flags[0] = 1;
    }
    if (p.part != nullptr) {
      // Partials mode: this rank's fp32 partial product, staged in its own
      // ring (retired: all its MMAs have completed) as boxes of 32 columns
      // in the 128-byte-swizzled layout, then stored by TMA.
      if (ok) {
        const uint32_t taddr = tmem_base + (static_cast<uint32_t>((warp & 3) * 32) << 16);
        const bool empty_rank = k1 == k0;
#pragma unroll 1
        for (int j = 0; j < p.TN / 32; ++j) {
          float v[32];
          if (empty_rank) {
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] = 0.f;
          } else {
            tmem_ld<32>(taddr + 32 * j, v);
          }
          uint8_t* box = smem + static_cast<size_t>(j) * (kBM * 128) + row * 128;
#pragma unroll
          for (int c = 0; c < 8; ++c)
            *reinterpret_cast<float4*>(box + ((c ^ (row & 7)) * 16)) =
                make_float4(v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
        }
        if (tile == 0 && row < p.M) p.ss_out[static_cast<size_t>(rank) * p.M + row] = ss;
        fence_proxy_async_smem();  // the generic writes above -> the TMA stores' reads
        epi_bar();
        if (threadIdx.x == 3 * 32) {
          for (int j = 0; j < p.TN / 32; ++j)
            tma_store_3d(&tmP, smem + static_cast<size_t>(j) * (kBM * 128), tile * p.TN + 32 * j,
                         0, static_cast<int>(rank));
          bulk_commit_group();
          bulk_wait_all();
        }
      }
    } else {
    tc_fence_before();
    // every rank's ring is retired (all its MMAs have completed: the MMA
    // thread waited for them) before any rank writes into another's
    cluster_sync();
    tc_fence_after();
    if (ok) {
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>((warp & 3) * 32) << 16);
      const bool empty_rank = k1 == k0;
      if (threadIdx.x == 3 * 32)
        mbar_arrive_expect_tx(red_full, static_cast<uint32_t>(3 * slot_bytes));
      // the other ranks' slices of this row, then its sum of squares, into
      // this rank's outgoing buffers (the layout of a receive slot), each
      // then sent by one bulk copy
      uint8_t* out = recv + 3 * slot_bytes;
#pragma unroll 1
      for (uint32_t o = 0; o < kCluster; ++o) {
        if (o == rank) continue;
        uint8_t* dst = out + ((o - rank - 1u) & 3u) * slot_bytes + row * 16;
#pragma unroll 1
        for (int j = 0; j < W / 8; ++j) {
          float v[8];
          if (empty_rank) {
#pragma unroll
            for (int i = 0; i < 8; ++i) v[i] = 0.f;
          } else {
            tmem_ld<8>(taddr + o * W + 8 * j, v);
          }
          *reinterpret_cast<float4*>(dst + (2 * j) * (kBM * 16)) = make_float4(v[0], v[1], v[2], v[3]);
          *reinterpret_cast<float4*>(dst + (2 * j + 1) * (kBM * 16)) =
              make_float4(v[4], v[5], v[6], v[7]);
        }
        *reinterpret_cast<float4*>(dst + nchunk * (kBM * 16)) = make_float4(ss, 0.f, 0.f, 0.f);
      }
      fence_proxy_async_smem();  // the generic writes above -> the bulk copies' reads
      epi_bar();
      if (threadIdx.x == 3 * 32) {
        for (uint32_t o = 0; o < kCluster; ++o) {
          if (o == rank) continue;
          bulk_s2cluster(map_rank(smem_u32(recv + recv_slot(rank, o) * slot_bytes), o),
                         out + ((o - rank - 1u) & 3u) * slot_bytes,
                         static_cast<uint32_t>(slot_bytes), map_rank(smem_u32(red_full), o));
        }
      }
      ok = epi_bar_and(mbar_wait(red_full, 0));
      if (ok) {
        // the row's sum of squares over all of K (rank order), its scale
        float sst = 0.f;
        for (uint32_t k = 0; k < kCluster; ++k)
          sst += k == rank ? ss
                           : *reinterpret_cast<const float*>(recv + recv_slot(k, rank) * slot_bytes +
                                                             nchunk * (kBM * 16) + row * 16);
        const float r = 1.0f / sqrtf(sst / static_cast<float>(p.d) + p.eps);
        const bool primary = row < p.mp, live = row < p.M;
#pragma unroll 1
        for (int j = 0; j < W / 8; ++j) {
          float sum[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) sum[i] = 0.f;
          for (uint32_t k = 0; k < kCluster; ++k) {
            float v[8];
            if (k == rank) {
              if (empty_rank) {
#pragma unroll
                for (int i = 0; i < 8; ++i) v[i] = 0.f;
              } else {
                tmem_ld<8>(taddr + rank * W + 8 * j, v);
              }
            } else {
              const uint8_t* src = recv + recv_slot(k, rank) * slot_bytes + row * 16;
              const float4 a = *reinterpret_cast<const float4*>(src + (2 * j) * (kBM * 16));
              const float4 b = *reinterpret_cast<const float4*>(src + (2 * j + 1) * (kBM * 16));
              v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
              v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
            }
#pragma unroll
            for (int i = 0; i < 8; ++i) sum[i] += v[i];
          }
#pragma unroll
          for (int i = 0; i < 8; ++i) sum[i] *= r;
          const int c0 = tile * p.TN + static_cast<int>(rank) * W + 8 * j;
          if (!live || c0 >= p.nout || (!primary && c0 >= p.nq)) continue;
          const uint4 packed = pack8(sum);
          *reinterpret_cast<uint4*>(p.qkv + static_cast<size_t>(row) * p.nout + c0) = packed;
          if (primary && c0 >= p.nq && cbase >= 0) {
            // primary K / V columns: also into the cache slot of this position
            const int kvd = p.Hkv * p.D;
            const bool is_v = c0 >= p.nq + kvd;
            const int c = c0 - p.nq - (is_v ? kvd : 0);
            const int g = c / p.D;
            const int64_t off =
                cbase + static_cast<int64_t>(g) * p.block_size * p.D + (c - g * p.D);
            *reinterpret_cast<uint4*>((is_v ? p.v_cache : p.k_cache) + off) = packed;
          }
        }
      } else if (lane == 0) {
        set_err(p.err, DF_DEVERR_TIMEOUT);
      }
    }
    }  // reduce mode
  }
  if (warp < 3 && p.part == nullptr) {
    // the roles outside the epilogue meet the epilogue's cluster barrier
    tc_fence_before();
    cluster_sync();
    tc_fence_after();
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (threadIdx.x == 0 && flags[0]) {
    // A wait gave up: a stage may have been filled by one producer only. Its
    // missing arrival is made here, so that the phase completes once the copy
    // already issued has landed, and the last fill of every slot is awaited
    // (bounded): no copy is left in flight into shared memory.
    for (int i = 0; i < kMaxStages; ++i) {
      const int nw = fills[i], nx = fills[kMaxStages + i];
      if (nw != nx) mbar_arrive(&full[i]);
      const int n = nw > nx ? nw : nx;
      if (n > 0) mbar_wait(&full[i], static_cast<uint32_t>((n - 1) & 1));
    }
  }
  // no CTA leaves while another rank may still write into its shared memory
  cluster_sync();
  if (warp == 1) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                 "n"(kMaxTileN)
                 : "memory");
  }
}

}  // namespace pre
}  // namespace df

namespace df {
namespace pre {

std::mutex g_mu;
bool g_attr[64] = {};
int g_clusters[64] = {};  // co-resident 4-CTA clusters per device (0: not queried)

// Sets the kernel's shared-memory attribute on the current device and returns
// how many 4-CTA clusters of it fit on the device at once (0 on error).
int max_clusters() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_attr[dev]) {
    if (cudaFuncSetAttribute(pre_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(kSmemBytes)) != cudaSuccess)
      return 0;
    g_attr[dev] = true;
  }
  if (g_clusters[dev] == 0) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(kCluster * 64);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = kSmemBytes;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = kCluster;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, pre_kernel, &cfg) != cudaSuccess || n < 1) return 0;
    g_clusters[dev] = n;
  }
  return g_clusters[dev];
}

struct Plan {
  bool ok;
  int nq, nout, TN, T;
};

// One column tile per cluster: TN = the smallest multiple of 32 with at most
// as many tiles as co-resident clusters, at most 256.
Plan make_plan(int mp, int d, int Hq, int Hkv, int D) {
  Plan pl{};
  pl.ok = false;
  if (mp < 1 || mp > 64 || d < kBK || d % kBK != 0 || Hq < 1 || Hkv < 1 || D < 8 || D % 8 != 0)
    return pl;
  const int nc = max_clusters();
  if (nc < 1) return pl;
  pl.nq = Hq * D;
  pl.nout = pl.nq + 2 * Hkv * D;
  pl.TN = static_cast<int>(round_up(static_cast<size_t>(ceil_div(pl.nout, nc)), 32));
  if (pl.TN > kMaxTileN) return pl;
  pl.T = static_cast<int>(ceil_div(pl.nout, pl.TN));
  pl.ok = pl.T <= nc;
  return pl;
}

}  // namespace pre
}  // namespace df

extern "C" int dualflow_layer_pre_attention_supported(int m_primary, int d_model, int Hq, int Hkv,
                                                      int D) {
  return df::pre::make_plan(m_primary, d_model, Hq, Hkv, D).ok ? 1 : 0;
}

namespace df {
namespace pre {

// Fills the shape fields of Params from the plan, encodes the tensor maps and
// launches (tmP: the partials store map, or any valid map in reduce mode).
df_status launch(Params& p, const Plan& pl, const void* x, const void* w_qkv, int m_primary,
                 int d_model, void* stream) {
  const int M = 2 * m_primary;
  p.M = M;
  p.mp = m_primary;
  p.d = d_model;
  p.nq = pl.nq;
  p.nout = pl.nout;
  p.TN = pl.TN;
  p.kblocks = d_model / kBK;
  p.w_bytes = pl.TN * kBK * 2;
  p.stage = static_cast<int>(round_up(static_cast<size_t>(kXBytes + p.w_bytes), 1024));
  p.nst = static_cast<int>(kRingBytes / static_cast<size_t>(p.stage));
  if (p.nst > kMaxStages) p.nst = kMaxStages;
  p.idesc = make_idesc(kBM, pl.TN);

  CUtensorMap tmX, tmW, tmP;
  const uint64_t du = static_cast<uint64_t>(d_model);
  if (!encode_tmap_bf16_2d(&tmX, x, static_cast<uint64_t>(M), du, du * 2, kBM, kBK) ||
      !encode_tmap_bf16_2d(&tmW, w_qkv, static_cast<uint64_t>(pl.nout), du, du * 2,
                           static_cast<uint32_t>(pl.TN), kBK))
    return DF_ERR_CUDA;
  if (p.part != nullptr) {
    // [rank][row][column] fp32, boxes of 32 columns x 128 rows of one rank
    const uint64_t nout = static_cast<uint64_t>(pl.nout), Mu = static_cast<uint64_t>(M);
    const uint64_t dims[3] = {nout, Mu, kCluster};
    const uint64_t strides[2] = {nout * 4, Mu * nout * 4};
    const uint32_t box[3] = {32, kBM, 1};
    if (!encode_tmap_f32_3d_box(&tmP, p.part, dims, strides, box)) return DF_ERR_CUDA;
  } else {
    tmP = tmX;
  }

  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(pl.T * kCluster);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = static_cast<cudaStream_t>(stream);
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = kCluster;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  if (cudaLaunchKernelEx(&cfg, pre_kernel, tmX, tmW, tmP, p) != cudaSuccess) return DF_ERR_CUDA;
  return DF_OK;
}

}  // namespace pre
}  // namespace df

extern "C" df_status dualflow_layer_pre_attention(
    const void* x, const void* w_qkv, int m_primary, int d_model, int Hq, int Hkv, int D,
    float eps, void* qkv, void* k_cache, void* v_cache, const int32_t* block_table,
    int max_blocks_per_seq, const int32_t* positions, int block_size, int num_blocks,
    int32_t* err_flag, void* stream) {
  using namespace df;
  using namespace df::pre;
  if (!x || !w_qkv || !qkv || !k_cache || !v_cache || !block_table || !positions)
    return DF_ERR_NULL;
  if (m_primary < 1 || d_model < 1 || Hq < 1 || Hkv < 1 || D < 1 || block_size < 1 ||
      num_blocks < 1 || max_blocks_per_seq < 1 || !(eps >= 0.f))
    return DF_ERR_SHAPE;
  const Plan pl = make_plan(m_primary, d_model, Hq, Hkv, D);
  if (!pl.ok) return DF_ERR_UNSUPPORTED;
  const void* ptrs[] = {x, w_qkv, qkv, k_cache, v_cache};
  for (const void* ptr : ptrs)
    if (!aligned(ptr, 16)) return DF_ERR_ALIGN;
  Params p{};
  p.eps = eps;
  p.qkv = static_cast<__nv_bfloat16*>(qkv);
  p.k_cache = static_cast<__nv_bfloat16*>(k_cache);
  p.v_cache = static_cast<__nv_bfloat16*>(v_cache);
  p.block_table = block_table;
  p.positions = positions;
  p.max_blocks = max_blocks_per_seq;
  p.Hkv = Hkv;
  p.D = D;
  p.block_size = block_size;
  p.num_blocks = num_blocks;
  p.err = err_flag;
  return launch(p, pl, x, w_qkv, m_primary, d_model, stream);
}

extern "C" df_status dualflow_layer_qkv_partials(const void* x, const void* w_qkv, int m_primary,
                                                 int d_model, int Hq, int Hkv, int D, void* part,
                                                 void* ss_part, int32_t* err_flag, void* stream) {
  using namespace df;
  using namespace df::pre;
  if (!x || !w_qkv || !part || !ss_part) return DF_ERR_NULL;
  if (m_primary < 1 || d_model < 1 || Hq < 1 || Hkv < 1 || D < 1) return DF_ERR_SHAPE;
  const Plan pl = make_plan(m_primary, d_model, Hq, Hkv, D);
  if (!pl.ok) return DF_ERR_UNSUPPORTED;
  const void* ptrs[] = {x, w_qkv, part, ss_part};
  for (const void* ptr : ptrs)
    if (!aligned(ptr, 16)) return DF_ERR_ALIGN;
  Params p{};
  p.Hkv = Hkv;
  p.D = D;
  p.err = err_flag;
  p.part = static_cast<float*>(part);
  p.ss_out = static_cast<float*>(ss_part);
  return launch(p, pl, x, w_qkv, m_primary, d_model, stream);
}
