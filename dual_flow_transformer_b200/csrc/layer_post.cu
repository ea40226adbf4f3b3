// Post-attention half of the Dual-Flow decoder layer as ONE persistent kernel
// launched as clusters of 4 CTAs.
//
// Method: "Sintesi Tecnica: Dual-Flow Transformers", sections "Architettura
// Core" (both flows share the output and MLP matrices), "Meccanismi Chiave"
// (one-way coupling b_l at the MLP intermediate and c_l at the MLP output) and
// "Costi di Inferenza vs. Addestramento" (grouped decode reads the unique
// weights once for both flows). With X = [primary rows; auxiliary rows]:
//   x_mid = x + attn W_o^T                                   (residual)
//   r     = 1 / sqrt(mean(x_mid^2) + eps)                    (RMSNorm, unit gain)
//   h     = SiLU(r x_mid W_gate^T) * (r x_mid W_up^T);  h_aux += b (.) h_primary
//   x_out = x_mid + h W_down^T;  aux rows add c (.) (h W_down^T)_primary
// x_mid, h and x_out are stored as bf16. The norm's row scale r is applied to
// the gate/up accumulators (r (x_mid W^T) = (r x_mid) W^T), so the normalised
// rows are never rounded to bf16 and stored: the gate/up product reads x_mid.
//
// Why one kernel: at M = 128 rows every projection is a weight stream (about
// 128 flop per weight byte, below the B200 ridge). Separate launches leave
// HBM idle at every boundary. Here one CTA per SM walks all three GEMMs in
// order and its TMA producer streams the weights continuously, into a 4-stage
// ring, across the phase boundaries; only the activation tiles of a phase
// wait for the phase before it.
//
// Why clusters: W_o and W_down have only d / 128 output tiles of 128 columns,
// too few for the SMs, so their K dimension is split 4 ways. The 4 splits of
// a tile run on the 4 CTAs of one cluster, and the split sum is a
// reduce-scatter through distributed shared memory: rank r owns columns
// 32 r .. 32 r + 31 of the tile, every other rank writes its fp32 slice of
// those columns straight from its TMEM accumulator into r's receive buffer
// (st.async, completing on r's mbarrier), and r adds the four slices in rank
// order. No partial sum goes through global memory and no grid-wide barrier
// is needed for a split reduction.
//
// Phases (cluster c = blockIdx.x / 4, rank = blockIdx.x % 4, G CTAs):
//   P0  W_o: cluster c < d/128 takes column tile c, rank r the r-th quarter
//       of K; reduce-scatter; the owner of a 32-column slice stores x_mid =
//       bf16(x + sum) and its rows' sums of squares over the slice
//   --- grid counter A2: x_mid and every slice's sums of squares are stored
//   P1  W_gate/W_up: tiles of 2*H1 weight rows spread over all CTAs (CTA i
//       takes i, i + G, ...); each CTA sums the slices' squares of its rows
//       (slice order) for r; SwiGLU + b coupling straight from TMEM -> h
//   --- grid counter C: every column of h is stored
//   P2  W_down: as P0 over K = F; the owner adds x_mid and the c coupling
//       -> x_out
// (Per-tile readiness flags in place of the two counters were measured
// slower: each flag read is an L2 round trip of a microsecond or more while
// the weight stream fills the memory system, and the tiles finish together.)
// The activation tiles interleave the flows (sequence j's primary row at tile
// row 2j, its auxiliary row at 2j + 1, by a [sequence][flow][K] tensor map),
// so both rows of a sequence sit in neighbouring TMEM lanes of one warp and
// the one-way b and c couplings are a warp shuffle from the primary lane.
// Every cluster is resident (one CTA per SM, grid = 4 x the device's maximum
// of co-resident 4-CTA clusters), so the grid counters cannot deadlock;
// every wait is bounded.
// Roles (352 threads): warp 0 weight producer, warp 1 MMA issuer (one thread,
// tcgen05.mma M = 128 into two 256-column TMEM accumulators), warp 2
// activation producer, warps 3-10 epilogue (TMEM lane quarter = warp % 4,
// thread = accumulator row; the two warps of a quarter take one half of the
// columns each, so two epilogue warps share each SM sub-partition).
// One ring holds a k-block's activation tile and weight tile per stage; its
// stage size follows the phase (5 stages of 32 KB for W_o in the low 176 KB,
// 5 of 44 KB for gate/up and 7 of 32 KB for W_down over 224 KB, whose top
// 48 KB is the W_o / W_down receive buffer when a reduction needs it), so
// every phase keeps the ring in flight: at these loads the DRAM and L2
// latency under full HBM traffic (1.5-2 us) needs all of it. The producers
// drain the ring at each phase boundary, where the MMAs wait for the phase
// before anyway; the gate/up stage in the top is filled once the W_o
// reduction has consumed its slices and counter A2 is complete (more weight
// traffic in flight delays the counter). (L2 prefetches
// of the next phase's weights at a boundary were measured to delay the grid
// counters behind them by more than they saved.)
// Every split sum is taken in a fixed order: results are deterministic, and
// primary rows never read auxiliary rows.
#include <math.h>
#include <string.h>

#include <mutex>

#include "cluster.cuh"
#include "common.cuh"
#include "host_util.h"
#include "umma.cuh"

namespace df {
namespace post {

using namespace umma;
using namespace cl;

constexpr int kBM = 128;
constexpr int kBK = 64;
constexpr int kThreads = 352;
constexpr int kEpiThreads = 256;                     // warps 3-10: two per TMEM lane quarter
constexpr int kMaxStages = 8;                        // ring stages (barrier pairs)
constexpr int kCluster = 4;                          // CTAs per cluster = K splits
constexpr int kTileN = 128;                          // W_o / W_down columns per cluster
constexpr int kSliceN = kTileN / kCluster;           // columns a rank owns: 32
constexpr int kHalfN = kSliceN / 2;                  // of which one epilogue thread takes 16
constexpr int kMaxHalf = 112;                        // SwiGLU output columns per tile
constexpr int kXBytes = kBM * kBK * 2;               // 16 KB activation tile
constexpr int kRecvSlotBytes = kBM * kSliceN * 4;    // one sender's slice: 16 KB
constexpr int kRecvBytes = (kCluster - 1) * kRecvSlotBytes;
constexpr int kCounters = 8;
constexpr size_t kCounterBytes = 256;
// The ring: P0 uses its low 176 KB (5 stages of 16 + 16 KB); P1 and P2 also
// the top 48 KB, which is the W_o / W_down receive buffer when a reduction
// needs it (P1: 5 stages of 16 + 28 KB, P2: 7 of 16 + 16 KB).
constexpr size_t kRingLow = 4 * (kXBytes + 2 * kMaxHalf * kBK * 2);
constexpr size_t kRingBytes = kRingLow + kRecvBytes;
constexpr size_t kSmemBytes = 1024 + kRingBytes + kMaxHalf * 4 + kBM * 4 +
                              512;                   // + barriers, fill counts, flags
static_assert(kRingLow % 1024 == 0 && kRingBytes % 1024 == 0 && kXBytes % 1024 == 0,
              "1024-byte swizzle alignment");
static_assert(kSmemBytes <= 232448, "shared memory budget");

// grid counters: CTAs past P0 (x_mid and the sums of squares stored), past
// P1 (h stored), done, past P2 (x_out and its sums of squares stored; P3 only)
enum { kCntA2 = 0, kCntC = 1, kCntExit = 2, kCntD = 3 };

// Weight stages filled before counter A2 (gate/up) and C (W_down) is seen.
constexpr int kEarlyGateUpStages = 4;
constexpr int kEarlyDownStages = 7;
// Weight stages of P3 filled before counter D is seen (the ones below the
// receive buffer, which P2's reduction still uses).
constexpr int kEarlyQkvStages = 4;

struct Gemm {
  int units;    // P0 / P2: column tiles (one per cluster); P1: SwiGLU tiles
  int kblocks;  // 64-wide K blocks of the whole product
  int BN;       // MMA N
  int half;     // SwiGLU output columns per tile (0: plain)
  int w_bytes;  // weight bytes per stage
  int stage;    // bytes per ring stage (activation tile first; multiple of 1024)
  int nst;      // ring stages in this phase
  uint32_t idesc;
};

struct Params {
  int M, mp, d, qd, F;
  float eps;
  Gemm g[4];  // P0 W_o, P1 W_gate / W_up, P2 W_down, P3 the next layer's W_qkv
  const __nv_bfloat16* x;
  const __nv_bfloat16* b;
  const __nv_bfloat16* c;
  __nv_bfloat16* x_mid;
  __nv_bfloat16* h;
  __nv_bfloat16* x_out;
  float* ss_part;  // [d / 32 slices][128 rows] sums of squares of stored x_mid values
  int* cnt;        // [kCounters]
  int32_t* err;
  int early[4];    // weight stages of phase q filled before its grid counter is complete
  // P3 (part != nullptr): rank r's fp32 partial product of x_out W_qkv^T over
  // its K quarter, part[r][row][column] (nout columns), and ss_out[r][row],
  // the sum of squares of the stored x_out row over that quarter
  float* part;
  float* ss_out;
  int nout;
};

__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

__device__ __forceinline__ int ld_acquire(const int* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// 16 bf16 values written by other CTAs of this launch (read through L2).
__device__ __forceinline__ void load_bf16x16_cg(const __nv_bfloat16* src, float (&v)[16]) {
#pragma unroll
  for (int q = 0; q < 2; ++q) {
    uint32_t w[4];
    asm volatile("ld.global.cg.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3])
                 : "l"(src + 8 * q));
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      v[8 * q + 2 * k] = bf16_bits_to_float(static_cast<uint16_t>(w[k] & 0xffffu));
      v[8 * q + 2 * k + 1] = bf16_bits_to_float(static_cast<uint16_t>(w[k] >> 16));
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

// This CTA's units of GEMM q: P0 / P2 one column tile per cluster (the
// cluster's index, if it has one), P1 tiles cta, cta + G, ...; and the
// k-blocks [k0, k1) of a unit (rank r's quarter for P0 / P2; may be empty
// when the product has fewer than 4 k-blocks).
struct Units {
  int first, step;
};
__device__ __forceinline__ Units units_of(const Gemm& g, int q, int cta, int cid, int G) {
  return q == 1 ? Units{cta, G} : Units{cid, g.units};
}
__device__ __forceinline__ void k_range(const Gemm& g, int q, int rank, int& k0, int& k1) {
  if (q == 1) {
    k0 = 0;
    k1 = g.kblocks;
  } else {
    k0 = rank * g.kblocks / kCluster;
    k1 = (rank + 1) * g.kblocks / kCluster;
  }
}

// The epilogue threads' arrival at a grid counter: every thread's stores are
// made visible (also to TMA reads of other CTAs) before one thread adds.
__device__ __forceinline__ void arrive_count(int* cnt, int et) {
  fence_proxy_async_global();
  epi_bar<kEpiThreads>();
  if (et == 0) {
    __threadfence();
    atomicAdd(cnt, 1);
  }
}

// All epilogue threads wait for a grid counter; returns false if it gave up.
__device__ __forceinline__ bool epi_wait_count(const int* cnt, int target, int et,
                                               volatile int* flag) {
  if (et == 0) *flag = wait_count(cnt, target) ? 1 : 0;
  epi_bar<kEpiThreads>();
  const bool ok = *flag != 0;
  epi_bar<kEpiThreads>();
  return ok;
}

// Reduce-scatter of a split-K accumulator over the cluster (thread = row and
// column half). reduce_send writes the given 16-column half of the other
// ranks' 32-column slices of this thread's row into their receive buffers and
// returns the same half of this rank's own slice in `own`; the TMEM
// accumulator may be reused once it returns. `empty`: this rank had no
// k-blocks (its partial is 0). A receive slot is laid out [8 chunks of 4
// columns][128 rows][16 bytes], so the 32 lanes of a warp (32 consecutive
// rows) write, and later read, one contiguous 512-byte block per chunk.
__device__ __forceinline__ void reduce_send(uint32_t taddr, bool empty, int row, int half,
                                            uint32_t rank, uint8_t* recv, uint64_t* red_full,
                                            float (&own)[kHalfN]) {
#pragma unroll 1
  for (uint32_t o = 0; o < kCluster; ++o) {
    if (o == rank) continue;
    float v[kHalfN];
    if (empty) {
#pragma unroll
      for (int i = 0; i < kHalfN; ++i) v[i] = 0.f;
    } else {
      tmem_ld<kHalfN>(taddr + o * kSliceN + half * kHalfN, v);
    }
    const uint32_t base = map_rank(
        smem_u32(recv + recv_slot(rank, o) * kRecvSlotBytes + (half * 4) * (kBM * 16) + row * 16),
        o);
    const uint32_t rbar = map_rank(smem_u32(red_full), o);
#pragma unroll
    for (int c = 0; c < 4; ++c)
      st_async16(base + c * (kBM * 16), v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3], rbar);
  }
  if (empty) {
#pragma unroll
    for (int i = 0; i < kHalfN; ++i) own[i] = 0.f;
  } else {
    tmem_ld<kHalfN>(taddr + rank * kSliceN + half * kHalfN, own);
  }
}

// reduce_gather waits (phase `parity`) for the other ranks' slices and sums
// the four in rank order into `sum` (this thread's half); false (for every
// epilogue thread) if the wait gave up.
__device__ __forceinline__ bool reduce_gather(int row, int half, uint32_t rank,
                                              const uint8_t* recv, uint64_t* red_full,
                                              uint32_t parity, const float (&own)[kHalfN],
                                              float (&sum)[kHalfN]) {
  bool ok = mbar_wait(red_full, parity);
  ok = epi_bar_and<kEpiThreads>(ok);
  if (!ok) return false;
#pragma unroll
  for (int i = 0; i < kHalfN; ++i) sum[i] = 0.f;
#pragma unroll 1
  for (uint32_t k = 0; k < kCluster; ++k) {
    if (k == rank) {
#pragma unroll
      for (int i = 0; i < kHalfN; ++i) sum[i] += own[i];
    } else {
      const uint8_t* src =
          recv + recv_slot(k, rank) * kRecvSlotBytes + (half * 4) * (kBM * 16) + row * 16;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const float4 v = *reinterpret_cast<const float4*>(src + c * (kBM * 16));
        sum[4 * c] += v.x;
        sum[4 * c + 1] += v.y;
        sum[4 * c + 2] += v.z;
        sum[4 * c + 3] += v.w;
      }
    }
  }
  return true;
}

// Row scale of this thread's row: 1 / sqrt(sum over the d/32 column slices of
// their sums of squares / d + eps). The two threads of a row (one per column
// half) sum one half of the slices each, in slice order, and the halves are
// added in a fixed order (uniform call: every epilogue thread).
__device__ float row_scale(const Params& p, int row, int tl, int half, bool live, float* red) {
  const int slices = p.d / kSliceN;
  const int k0 = half * (slices / 2), k1 = half ? slices : slices / 2;
  float s = 0.f;
  if (live) {
    int k = k0;
    for (; k + 16 <= k1; k += 16) {
      float v[16];
#pragma unroll
      for (int i = 0; i < 16; ++i)
        v[i] = __ldcg(p.ss_part + static_cast<size_t>(k + i) * kBM + row);
#pragma unroll
      for (int i = 0; i < 16; ++i) s += v[i];
    }
    for (; k < k1; ++k) s += __ldcg(p.ss_part + static_cast<size_t>(k) * kBM + row);
  }
  if (half == 1) red[tl] = s;
  epi_bar<kEpiThreads>();
  float r = 0.f;
  if (half == 0) r = 1.0f / sqrtf((s + red[tl]) / static_cast<float>(p.d) + p.eps);
  epi_bar<kEpiThreads>();
  if (half == 0) red[tl] = r;
  epi_bar<kEpiThreads>();
  r = red[tl];
  epi_bar<kEpiThreads>();
  return live ? r : 0.f;
}

// P1 epilogue of tile t: h[row][t*H + j] = SiLU(rs g) * (rs u) (+ b * primary
// row's value for auxiliary rows), in 32-column chunks (8-column tail). The
// primary row of a sequence is the neighbouring TMEM lane of its auxiliary
// row (lanes 2j, 2j + 1), so its values arrive by one warp shuffle.
template <int W>
__device__ __forceinline__ void swiglu_chunk(const Params& p, uint32_t taddr, int H, int c, int col0,
                                             int row, bool live, bool aux, float rs,
                                             const float* bsl) {
  float g[W], u[W];
  tmem_ld<W>(taddr + c, g);
  tmem_ld<W>(taddr + H + c, u);
#pragma unroll
  for (int i = 0; i < W; ++i) g[i] = silu_f(rs * g[i]) * (rs * u[i]);
  if (p.b != nullptr) {
#pragma unroll
    for (int i = 0; i < W; ++i) {
      const float pv = __shfl_xor_sync(0xffffffffu, g[i], 1);
      if (aux) g[i] = fmaf(bsl[c + i], pv, g[i]);
    }
  }
  if (live) {
    // a chunk of the last tile may reach past F: store its 8-column groups
    // that lie inside (F and H are multiples of 8)
#pragma unroll
    for (int q = 0; q < W / 8; ++q) {
      if (col0 + c + 8 * q >= p.F) break;
      float o[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) o[i] = g[8 * q + i];
      store_bf16<8>(p.h + static_cast<size_t>(row) * p.F + col0 + c + 8 * q, o);
    }
  }
}

// (this thread's half of the tile's H columns: H is a multiple of 16)
__device__ void swiglu_epilogue(const Params& p, int t, uint32_t taddr, int row, int half,
                                bool live, bool aux, float rs, const float* bsl) {
  const int H = p.g[1].half;
  const int col0 = t * H;
  int c = half * (H / 2);
  const int c1 = c + H / 2;
  for (; c + 32 <= c1; c += 32) swiglu_chunk<32>(p, taddr, H, c, col0, row, live, aux, rs, bsl);
  for (; c < c1; c += 8) swiglu_chunk<8>(p, taddr, H, c, col0, row, live, aux, rs, bsl);
}

// Tile t's slice of the coupling vector b into shared memory (zeros past F),
// fetched while the tile's MMAs run.
__device__ void load_b_slice(const Params& p, int t, int et, float* bsl) {
  const int H = p.g[1].half;
  for (int i = et; i < H; i += kEpiThreads) {
    const int col = t * H + i;
    bsl[i] = (p.b != nullptr && col < p.F) ? __bfloat162float(p.b[col]) : 0.f;
  }
  epi_bar<kEpiThreads>();
}

__global__ void __launch_bounds__(kThreads, 1)
    post_kernel(const __grid_constant__ CUtensorMap tmXo, const __grid_constant__ CUtensorMap tmWo,
                const __grid_constant__ CUtensorMap tmXg, const __grid_constant__ CUtensorMap tmWg,
                const __grid_constant__ CUtensorMap tmXd, const __grid_constant__ CUtensorMap tmWd,
                const __grid_constant__ CUtensorMap tmXq, const __grid_constant__ CUtensorMap tmWq,
                const __grid_constant__ CUtensorMap tmP, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* recv = smem + kRingLow;  // [3][8 chunks][128 rows][16 B], the ring's top in P1 / P2
  float* bsl = reinterpret_cast<float*>(smem + kRingBytes);      // [kMaxHalf] b of a tile
  float* red = bsl + kMaxHalf;  // [128]: one value per TMEM lane passed between the halves
  uint64_t* full = reinterpret_cast<uint64_t*>(red + kBM);       // [kMaxStages]
  uint64_t* empty = full + kMaxStages;                           // [kMaxStages]
  uint64_t* acc_full = empty + kMaxStages;                       // [2]
  uint64_t* acc_empty = acc_full + 2;                            // [2]
  uint64_t* mma_done = acc_empty + 2;                            // [1]
  uint64_t* red_full = mma_done + 1;  // this rank's slices from the other 3 ranks have landed
  uint64_t* recv_free = red_full + 1;  // P0's received slices are consumed: P1 may use the top
  int* wfills = reinterpret_cast<int*>(recv_free + 1);  // [kMaxStages] fills per slot: weights
  int* xfills = wfills + kMaxStages;                     // [kMaxStages] activation tiles
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(xfills + kMaxStages);
  // [0] abort, [1] epilogue broadcast, [2] / [3] / [4] counter A2 / C / D
  // seen by the activation producer
  volatile int* flags = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = gridDim.x, cta = blockIdx.x;
  const uint32_t rank = cluster_rank();
  const int cid = static_cast<int>(cluster_index());

  if (threadIdx.x == 0) {
    for (int i = 0; i < kMaxStages; ++i) {
      mbar_init(&full[i], 2);  // weight producer + activation producer
      mbar_init(&empty[i], 1);
      wfills[i] = 0;
      xfills[i] = 0;
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], kEpiThreads / 32);
    }
    mbar_init(mma_done, 1);
    mbar_init(red_full, 1);  // this rank's expect_tx arrival + the senders' bytes
    mbar_init(recv_free, 1);
    flags[0] = 0;
    flags[1] = 0;
    flags[2] = 0;
    flags[3] = 0;
    flags[4] = 0;
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
  // every CTA of the cluster has initialised its barriers before any remote write
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // Only the weight producer may run ahead of the kernel launched before this
  // one (the weights are constants); every other role waits for it first.
  if (warp != 0) pdl_wait();

  if (warp == 0 || warp == 2) {
    // ------------------------------------------------------------ producers
    // warp 0: weights (may run ahead of the kernel launched before this one:
    // the weights are constants); warp 2: activation tiles.
    const bool wrole = warp == 0;
    const uint64_t pol = wrole ? l2_policy_evict_first() : l2_policy_evict_last();
    int* fills = wrole ? wfills : xfills;
    uint32_t par = 0;  // bit i: parity of this producer's fills of slot i
    bool recv_ok = false;
    bool ok = true;
    const bool qkv = p.part != nullptr;  // phase P3: the next layer's QKV partials
    // one phase's fills (lane 0)
    auto fill_phase = [&](int q) {
      const Gemm& g = p.g[q];
      const CUtensorMap* tm =
          wrole ? (q == 0 ? &tmWo : (q == 1 ? &tmWg : (q == 2 ? &tmWd : &tmWq)))
                : (q == 0 ? &tmXo : (q == 1 ? &tmXg : (q == 2 ? &tmXd : &tmXq)));
      // The ring changes its stage size at a phase boundary: every earlier
      // fill of every slot must have been consumed first.
      if (q > 0) {
        for (int i = 0; i < kMaxStages && ok; ++i) {
          if (!mbar_wait(&empty[i], ((par >> i) & 1u) ^ 1u)) {
            set_err(p.err, DF_DEVERR_TIMEOUT);
            flags[0] = 1;
            ok = false;
          }
        }
      }
      int s = 0;
      int fills_q = 0;  // this producer's fills in this phase
      const Units us = units_of(g, q, cta, cid, G);
      for (int u = us.first; u < g.units && ok; u += us.step) {
        int k0, k1;
        k_range(g, q, static_cast<int>(rank), k0, k1);
        if (!wrole && q > 0 && k1 > k0) {
          // P1 reads x_mid (counter A2), P2 every column of h (counter C),
          // P3 x_out (counter D)
          if (!wait_count(p.cnt + (q == 1 ? kCntA2 : (q == 2 ? kCntC : kCntD)), G)) {
            set_err(p.err, DF_DEVERR_TIMEOUT);
            flags[0] = 1;
            ok = false;
            break;
          }
          fence_proxy_async_global();
          flags[1 + q] = 1;  // counter A2 / C / D seen (see the weight producer)
        }
        for (int kb = k0; kb < k1 && ok; ++kb) {
          if (wrole && q > 0 && fills_q == p.early[q]) {
            // Weight traffic in flight delays the grid counter the phase's
            // activations wait for: beyond p.early[q] stages, wait until
            // the activation producer has seen it (counter A2 / C / D).
            const long long t0 = clock64();
            while (flags[1 + q] == 0 && !flags[0]) {
              if (clock64() - t0 > kWaitLimitCycles) {
                set_err(p.err, DF_DEVERR_TIMEOUT);
                flags[0] = 1;
              }
              __nanosleep(64);
            }
            if (flags[0]) {
              ok = false;
              break;
            }
          }
          if (!recv_ok && static_cast<size_t>(s + 1) * g.stage > kRingLow) {
            // this slot reaches into the receive buffer: wait until this
            // CTA's epilogue has consumed the received slices (P0's before
            // P1, P2's before P3)
            if (!mbar_wait(recv_free, q == 3 ? 1u : 0u)) {
              set_err(p.err, DF_DEVERR_TIMEOUT);
              flags[0] = 1;
              ok = false;
              break;
            }
            recv_ok = true;
          }
          if (!mbar_wait(&empty[s], ((par >> s) & 1u) ^ 1u)) {
            set_err(p.err, DF_DEVERR_TIMEOUT);
            flags[0] = 1;
            ok = false;
            break;
          }
          if (flags[0]) {
            ok = false;
            break;
          }
          uint8_t* st = smem + static_cast<size_t>(s) * g.stage;
          if (wrole) {
            mbar_arrive_expect_tx(&full[s], static_cast<uint32_t>(g.w_bytes));
            if (q == 1) {
              tma_load_2d_hint(st + kXBytes, tm, &full[s], kb * kBK, u * g.half, pol);
              tma_load_2d_hint(st + kXBytes + g.half * 128, tm, &full[s], kb * kBK,
                               p.F + u * g.half, pol);
            } else {
              tma_load_2d_hint(st + kXBytes, tm, &full[s], kb * kBK, u * g.BN, pol);
            }
          } else {
            mbar_arrive_expect_tx(&full[s], kXBytes);
            tma_load_3d_hint(st, tm, &full[s], kb * kBK, 0, 0, pol);
          }
          ++fills[s];
          ++fills_q;
          par ^= 1u << s;
          if (++s == g.nst) s = 0;
        }
      }
        };
    if (lane == 0) {
      if (wrole) {
        prefetch_tensormap(&tmWo);
        prefetch_tensormap(&tmWg);
        prefetch_tensormap(&tmWd);
        if (qkv) prefetch_tensormap(&tmWq);
      } else {
        prefetch_tensormap(&tmXo);
        prefetch_tensormap(&tmXg);
        prefetch_tensormap(&tmXd);
        if (qkv) prefetch_tensormap(&tmXq);
      }
      for (int q = 0; q < 3 && ok; ++q) fill_phase(q);
      if (wrole && !qkv) pdl_trigger();
    }
    // P2's reduction may write into this CTA's ring once every role of every
    // rank is done with it (the epilogue meets this barrier after P2's MMAs)
    tc_fence_before();
    cluster_sync();
    tc_fence_after();
    if (lane == 0 && qkv) {
      // P3: the low stages are free (every P2 MMA has completed); a stage
      // that reaches into the receive buffer waits for P2's reduction
      recv_ok = false;
      if (ok) fill_phase(3);
      if (wrole) pdl_trigger();
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    uint32_t par = 0;  // bit i: parity of the next phase of full[i] to wait for
    int seg = 0;
    bool ok = true;
    auto mma_phase = [&](int q) {
      const Gemm& g = p.g[q];
      int s = 0;  // the producers restart the ring at every phase
      const Units us = units_of(g, q, cta, cid, G);
      for (int u = us.first; u < g.units && ok; u += us.step, ++seg) {
        int k0, k1;
        k_range(g, q, static_cast<int>(rank), k0, k1);
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
          if (!mbar_wait(&full[s], (par >> s) & 1u) || flags[0]) {
            set_err(p.err, DF_DEVERR_TIMEOUT);
            flags[0] = 1;
            ok = false;
            break;
          }
          par ^= 1u << s;
          tc_fence_after();
          const uint32_t a_addr = smem_u32(smem + static_cast<size_t>(s) * g.stage);
          const uint32_t b_addr = a_addr + kXBytes;
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk)
            umma_bf16(d_tmem, smem_desc(a_addr + kk * 32), smem_desc(b_addr + kk * 32), g.idesc,
                      (kb > k0 || kk > 0) ? 1u : 0u);
          umma_commit(&empty[s]);
          if (++s == g.nst) s = 0;
        }
        if (!ok) break;
        // (a unit without k-blocks commits at once: its partial is zero)
        umma_commit(&acc_full[acc]);
      }
    };
    if (lane == 0) {
      for (int q = 0; q < 3 && ok; ++q) mma_phase(q);
      // no tensor-core operation may still be reading shared memory or TMEM
      // when the ring retires or the CTA leaves (this commit completes after
      // every MMA above)
      umma_commit(mma_done);
      mbar_wait(mma_done, 0);
    }
    tc_fence_before();
    cluster_sync();  // the ring retires (see the producers)
    tc_fence_after();
    if (lane == 0 && p.part != nullptr) {
      if (ok) mma_phase(3);
      umma_commit(mma_done);
      mbar_wait(mma_done, 1);
    }
  } else {
    // ------------------------------------------------------------ epilogue warps
    // Two warps per TMEM lane quarter (warps q + 3 and q + 7 take quarter
    // (q + 3) % 4), each taking one half of the columns.
    const int quarter = warp & 3;
    const int et = threadIdx.x - 3 * 32;
    const int half = et >> 7;
    // The activation tiles hold the rows interleaved, sequence j's primary
    // row at tile row 2j and its auxiliary row at 2j + 1: this thread's TMEM
    // lane tl is tile row tl, which is `row` of x / x_mid / h / x_out.
    const int tl = quarter * 32 + lane;
    const int seq = tl >> 1;
    const bool aux = (tl & 1) != 0;
    const bool live = seq < p.mp;
    const int row = aux ? p.mp + seq : seq;
    volatile int* eflag = flags + 1;
    int seg = 0;
    bool ok = true;
    // (uniform over the epilogue threads, like every other epilogue wait, so
    // that all of them pass the same named barriers on every path)
    auto take_acc = [&](int acc, int sg) -> bool {
      const bool got = mbar_wait_warp(&acc_full[acc], static_cast<uint32_t>((sg >> 1) & 1));
      return epi_bar_and<kEpiThreads>(got);
    };
    auto give_acc = [&](int acc) {
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[acc]);
    };
    auto grid_wait = [&](int which) -> bool {
      if (epi_wait_count(p.cnt + which, G, et, eflag)) return true;
      if (et == 0) set_err(p.err, DF_DEVERR_TIMEOUT);
      flags[0] = 1;
      return false;
    };
    auto acc_addr = [&](int acc) -> uint32_t {
      return tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) +
             static_cast<uint32_t>(acc * 256);
    };
    auto fail = [&]() {
      if (et == 0) set_err(p.err, DF_DEVERR_TIMEOUT);
      flags[0] = 1;
      ok = false;
    };
    // P0: W_o tile `cid` over this rank's K quarter; reduce-scatter; x_mid
    if (cid < p.g[0].units) {
      const int acc = seg & 1;
      int k0, k1;
      k_range(p.g[0], 0, static_cast<int>(rank), k0, k1);
      const int slice = (cid * kCluster + static_cast<int>(rank)) * 2 + half;  // 16 columns
      const int col0 = slice * kHalfN;
      float res[kHalfN];  // residual, loaded while the MMAs run
      if (live) {
        load_bf16<kHalfN>(p.x + static_cast<size_t>(row) * p.d + col0, res);
      } else {
#pragma unroll
        for (int i = 0; i < kHalfN; ++i) res[i] = 0.f;
      }
      if (et == 0) mbar_arrive_expect_tx(red_full, kRecvBytes);
      if (!take_acc(acc, seg)) {
        fail();
      } else {
        tc_fence_after();
        float own[kHalfN], sum[kHalfN];
        reduce_send(acc_addr(acc), k1 == k0, tl, half, rank, recv, red_full, own);
        give_acc(acc);
        if (!reduce_gather(tl, half, rank, recv, red_full, 0, own, sum)) {
          fail();
        } else {
          float ss = 0.f;
#pragma unroll
          for (int i = 0; i < kHalfN; ++i) {
            sum[i] = __bfloat162float(__float2bfloat16_rn(sum[i] + res[i]));
            ss = fmaf(sum[i], sum[i], ss);
          }
          if (live) store_bf16<kHalfN>(p.x_mid + static_cast<size_t>(row) * p.d + col0, sum);
          // the 32-column slice's sum of squares: this half's, then the other's
          if (half == 1) red[tl] = ss;
          epi_bar<kEpiThreads>();
          if (half == 0 && live)
            p.ss_part[static_cast<size_t>(slice >> 1) * kBM + row] = ss + red[tl];
        }
      }
      ++seg;
    }
    ok = epi_bar_and<kEpiThreads>(ok);
    if (et == 0) mbar_arrive(recv_free);  // every epilogue thread is done with recv
    arrive_count(p.cnt + kCntA2, et);
    // P1: SwiGLU tiles straight from TMEM
    float rs = 0.f;
    bool have_rs = false;
    for (int u = cta; u < p.g[1].units && ok; u += G, ++seg) {
      const int acc = seg & 1;
      if (p.b != nullptr) load_b_slice(p, u, et, bsl);
      if (!have_rs) {
        if (!grid_wait(kCntA2)) {
          ok = false;
          break;
        }
        rs = row_scale(p, row, tl, half, live, red);
        have_rs = true;
      }
      if (!take_acc(acc, seg)) {
        fail();
        break;
      }
      tc_fence_after();
      swiglu_epilogue(p, u, acc_addr(acc), row, half, live, aux, rs, bsl);
      give_acc(acc);
    }
    ok = epi_bar_and<kEpiThreads>(ok);
    arrive_count(p.cnt + kCntC, et);
    // P2: W_down tile `cid` over this rank's K quarter; reduce-scatter; x_out.
    // (Counter C orders this rank's sends after the receivers' last use of
    // P0's data; a rank without k-blocks would otherwise send at once.)
    const bool p2 = ok && cid < p.g[2].units && grid_wait(kCntC);
    bool got = false;
    float res[kHalfN], cc[kHalfN];
    int col0 = 0;
    const int acc2 = seg & 1;
    if (p2) {
      const int acc = acc2;
      int k0, k1;
      k_range(p.g[2], 2, static_cast<int>(rank), k0, k1);
      col0 = ((cid * kCluster + static_cast<int>(rank)) * 2 + half) * kHalfN;
      // residual (x_mid, stored by other CTAs before counter A2) and coupling,
      // loaded while the MMAs run
      if (live) {
        load_bf16x16_cg(p.x_mid + static_cast<size_t>(row) * p.d + col0, res);
      } else {
#pragma unroll
        for (int i = 0; i < kHalfN; ++i) res[i] = 0.f;
      }
      if (aux && live && p.c != nullptr) {
        load_bf16<kHalfN>(p.c + col0, cc);
      } else {
#pragma unroll
        for (int i = 0; i < kHalfN; ++i) cc[i] = 0.f;
      }
      if (et == 0) mbar_arrive_expect_tx(red_full, kRecvBytes);
      got = take_acc(acc, seg);
      if (!got) fail();
    }
    // every role of every rank of the cluster is done with its ring (the
    // receive buffer is its top in P2)
    tc_fence_before();
    cluster_sync();
    tc_fence_after();
    if (p2 && got) {
      const int acc = acc2;
      int k0, k1;
      k_range(p.g[2], 2, static_cast<int>(rank), k0, k1);
      {
        float own[kHalfN], sum[kHalfN];
        reduce_send(acc_addr(acc), k1 == k0, tl, half, rank, recv, red_full, own);
        give_acc(acc);
        if (!reduce_gather(tl, half, rank, recv, red_full, 1, own, sum)) {
          fail();
        } else {
          if (p.c != nullptr) {
            // the primary row's sum from the neighbouring lane
#pragma unroll
            for (int i = 0; i < kHalfN; ++i) {
              const float pv = __shfl_xor_sync(0xffffffffu, sum[i], 1);
              if (aux) sum[i] = fmaf(cc[i], pv, sum[i]);
            }
          }
#pragma unroll
          for (int i = 0; i < kHalfN; ++i) sum[i] += res[i];
          if (p.part != nullptr) {
            // P3 reads x_out and needs its rows' sums of squares: per
            // 32-column slice, over the stored (bf16) values, as for x_mid
            float ss = 0.f;
#pragma unroll
            for (int i = 0; i < kHalfN; ++i) {
              sum[i] = __bfloat162float(__float2bfloat16_rn(sum[i]));
              ss = fmaf(sum[i], sum[i], ss);
            }
            if (half == 1) red[tl] = ss;
            epi_bar<kEpiThreads>();
            if (half == 0 && live)
              p.ss_part[static_cast<size_t>(cid * kCluster + static_cast<int>(rank)) * kBM + row] =
                  ss + red[tl];
          }
          if (live) store_bf16<kHalfN>(p.x_out + static_cast<size_t>(row) * p.d + col0, sum);
        }
      }
      ++seg;
    }
    if (p.part != nullptr) {
      // P3: the next layer's QKV partial products over x_out (the rows'
      // sums of squares of each K quarter from the slices above)
      ok = epi_bar_and<kEpiThreads>(ok);
      if (et == 0) mbar_arrive(recv_free);  // P2's received slices are consumed
      arrive_count(p.cnt + kCntD, et);
      if (ok && cid < p.g[3].units) {
        const int acc = seg & 1;
        int k0, k1;
        k_range(p.g[3], 3, static_cast<int>(rank), k0, k1);
        float ssq = 0.f;
        if (cid == 0) {
          // cluster 0 stores ss_out: this half's slices of the quarter in
          // slice order, then the two halves added in a fixed order
          if (!grid_wait(kCntD)) {
            ok = false;
          } else {
            const int per = p.d / kSliceN / kCluster;  // slices per K quarter
            const int k_first = static_cast<int>(rank) * per + half * (per / 2);
            if (live)
              for (int k = 0; k < per / 2; ++k)
                ssq += __ldcg(p.ss_part + static_cast<size_t>(k_first + k) * kBM + row);
            if (half == 1) red[tl] = ssq;
            epi_bar<kEpiThreads>();
            if (half == 0) ssq += red[tl];
          }
        }
        if (ok && !take_acc(acc, seg)) fail();
        if (ok) {
          tc_fence_after();
          // this thread's half of the tile, in boxes of 32 columns (128-byte
          // swizzle), staged in the retired ring at the output row: every
          // MMA of this CTA has completed, and no other rank writes here
          const int nbox = p.g[3].BN / 32;
          for (int j = half * (nbox / 2); j < (half + 1) * (nbox / 2); ++j) {
            float v[32];
            if (k1 == k0) {
#pragma unroll
              for (int i = 0; i < 32; ++i) v[i] = 0.f;
            } else {
              tmem_ld<32>(acc_addr(acc) + 32 * j, v);
            }
            if (live) {
              uint8_t* box = smem + static_cast<size_t>(j) * (kBM * 128) + row * 128;
#pragma unroll
              for (int c = 0; c < 8; ++c)
                *reinterpret_cast<float4*>(box + ((c ^ (row & 7)) * 16)) =
                    make_float4(v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
            }
          }
          give_acc(acc);
          if (cid == 0 && half == 0 && live)
            p.ss_out[static_cast<size_t>(rank) * p.M + row] = ssq;
          fence_proxy_async_smem();  // the generic writes above -> the TMA stores' reads
          epi_bar<kEpiThreads>();
          if (et == 0) {
            for (int j = 0; j < nbox; ++j)
              tma_store_3d(&tmP, smem + static_cast<size_t>(j) * (kBM * 128),
                           cid * p.g[3].BN + 32 * j, 0, static_cast<int>(rank));
            bulk_commit_group();
            bulk_wait_all();
          }
        }
        ++seg;
      }
    }
  }

  // Every role of this CTA is done (all its waits have returned): count the
  // CTA out; the last one out rewinds the counters for the next call.
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (threadIdx.x == 0 && flags[0]) {
    // A wait gave up: a stage may have been filled by one producer only. Its
    // missing arrival is made here, so that the phase completes once the copy
    // already issued has landed, and the last fill of every slot is awaited
    // (bounded): no copy is left in flight into shared memory.
    for (int i = 0; i < kMaxStages; ++i) {
      const int nw = wfills[i], nx = xfills[i];
      if (nw != nx) mbar_arrive(&full[i]);
      const int n = nw > nx ? nw : nx;
      if (n > 0) mbar_wait(&full[i], static_cast<uint32_t>((n - 1) & 1));
    }
  }
  if (threadIdx.x == 0) {
    __threadfence();
    const int before = atomicAdd(p.cnt + kCntExit, 1);
    if (before == G - 1) {
      for (int i = 0; i < kCounters; ++i) atomicExch(p.cnt + i, 0);
      __threadfence();
    }
  }
  // no CTA leaves while another rank may still write into its shared memory
  cluster_sync();
  if (warp == 1) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "n"(512)
                 : "memory");
  }
}

// ------------------------------------------------------------------ planning

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
    if (cudaFuncSetAttribute(post_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
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
    if (cudaOccupancyMaxActiveClusters(&n, post_kernel, &cfg) != cudaSuccess || n < 1) return 0;
    g_clusters[dev] = n;
  }
  return g_clusters[dev];
}

struct Plan {
  bool ok;
  int G, T0, H1, T1;
};

Plan make_plan(int M, int mp, int d, int qd, int F) {
  Plan pl{};
  pl.ok = false;
  if (M != 2 * mp || mp < 1 || mp > 64 || d % kTileN != 0 || qd % kBK != 0 || F % kBK != 0 ||
      d < kTileN || qd < kBK || F < kBK)
    return pl;
  const int nc = max_clusters();
  pl.T0 = d / kTileN;
  if (nc < 1 || pl.T0 > nc) return pl;  // one W_o / W_down tile per cluster
  pl.G = nc * kCluster;
  // smallest multiple of 16 with at most G SwiGLU tiles (two epilogue warps
  // take 8-column multiples each; the MMA's N = 2 H steps by 16 at M = 128)
  int H = static_cast<int>(ceil_div(F, pl.G));
  H = static_cast<int>(ceil_div(H, 16)) * 16;
  if (H > kMaxHalf) return pl;
  pl.H1 = H;
  pl.T1 = static_cast<int>(ceil_div(F, H));
  pl.ok = true;
  return pl;
}

// A phase's GEMM: MMA N = BN (weight rows per k-block), ring stages of the
// activation tile plus BN x 64 weights, as many as the ring holds (at most
// kMaxStages).
Gemm ring_gemm(int units, int kblocks, int BN, int half, size_t ring_bytes) {
  Gemm g{};
  g.units = units;
  g.kblocks = kblocks;
  g.BN = BN;
  g.half = half;
  g.w_bytes = BN * kBK * 2;
  g.stage = static_cast<int>(round_up(static_cast<size_t>(kXBytes + g.w_bytes), 1024));
  g.nst = static_cast<int>(ring_bytes / static_cast<size_t>(g.stage));
  if (g.nst > kMaxStages) g.nst = kMaxStages;
  g.idesc = make_idesc(kBM, BN);
  return g;
}

// Workspace: counters | ss_part [d / 32][128].
size_t ws_bytes(int d) {
  return kCounterBytes + static_cast<size_t>(d / kSliceN) * kBM * 4;
}

// P3's column tile: the narrowest multiple of 64 (at most 256) that divides
// nout with at most one tile per cluster (0: none fits).
int qkv_tile(int nout, int d, int clusters) {
  if (d % (kSliceN * kCluster * 2) != 0) return 0;  // whole slices per half quarter
  for (int tn = 64; tn <= 256; tn += 64)
    if (nout % tn == 0 && nout / tn <= clusters) return tn;
  return 0;
}

struct QkvNext {  // P3's operands (w == nullptr: no P3)
  const void* w;
  int nout;
  void* part;
  void* ss_out;
};

df_status launch_post(const void* attn, const void* x, const void* w_o, const void* w_gu,
                      const void* w_down, const void* b, const void* c, int m_primary,
                      int d_model, int q_dim, int F, float eps, void* x_mid, void* h,
                      void* x_out, void* workspace, size_t workspace_bytes, int32_t* err_flag,
                      const QkvNext& nx, void* stream) {
  if (!attn || !x || !w_o || !w_gu || !w_down || !x_mid || !h || !x_out)
    return DF_ERR_NULL;
  if (m_primary < 1 || d_model < 1 || q_dim < 1 || F < 1 || !(eps >= 0.f)) return DF_ERR_SHAPE;
  const int M = 2 * m_primary;
  const Plan pl = make_plan(M, m_primary, d_model, q_dim, F);
  if (!pl.ok) return DF_ERR_UNSUPPORTED;
  const void* ptrs[] = {attn, x, w_o, w_gu, w_down, x_mid, h, x_out};
  for (const void* ptr : ptrs)
    if (!aligned(ptr, 16)) return DF_ERR_ALIGN;
  if ((b && !aligned(b, 16)) || (c && !aligned(c, 16))) return DF_ERR_ALIGN;
  if (!workspace || workspace_bytes < ws_bytes(d_model) || !aligned(workspace, 256))
    return DF_ERR_WORKSPACE;
  int tn3 = 0;
  if (nx.w != nullptr) {
    if (!nx.part || !nx.ss_out) return DF_ERR_NULL;
    if (!aligned(nx.w, 16) || !aligned(nx.part, 16) || !aligned(nx.ss_out, 16))
      return DF_ERR_ALIGN;
    tn3 = qkv_tile(nx.nout, d_model, pl.G / kCluster);
    if (tn3 == 0) return DF_ERR_UNSUPPORTED;
  }

  Params p{};
  p.M = M;
  p.mp = m_primary;
  p.d = d_model;
  p.qd = q_dim;
  p.F = F;
  p.eps = eps;
  p.g[0] = ring_gemm(pl.T0, q_dim / kBK, kTileN, 0, kRingLow);
  p.g[1] = ring_gemm(pl.T1, d_model / kBK, 2 * pl.H1, pl.H1, kRingBytes);
  p.g[2] = ring_gemm(pl.T0, F / kBK, kTileN, 0, kRingBytes);
  p.x = static_cast<const __nv_bfloat16*>(x);
  p.b = static_cast<const __nv_bfloat16*>(b);
  p.c = static_cast<const __nv_bfloat16*>(c);
  p.x_mid = static_cast<__nv_bfloat16*>(x_mid);
  p.h = static_cast<__nv_bfloat16*>(h);
  p.x_out = static_cast<__nv_bfloat16*>(x_out);
  uint8_t* w8 = static_cast<uint8_t*>(workspace);
  p.cnt = reinterpret_cast<int*>(w8);
  p.ss_part = reinterpret_cast<float*>(w8 + kCounterBytes);
  p.err = err_flag;
  p.early[0] = 0;                    // (P0 waits for no counter)
  p.early[1] = kEarlyGateUpStages;
  p.early[2] = kEarlyDownStages;
  if (tn3 > 0) {
    p.g[3] = ring_gemm(nx.nout / tn3, d_model / kBK, tn3, 0, kRingBytes);
    p.early[3] = kEarlyQkvStages;
    p.part = static_cast<float*>(nx.part);
    p.ss_out = static_cast<float*>(nx.ss_out);
    p.nout = nx.nout;
  }

  CUtensorMap tmXo, tmWo, tmXg, tmWg, tmXd, tmWd;
  const uint64_t du = static_cast<uint64_t>(d_model),
                 qu = static_cast<uint64_t>(q_dim), Fu = static_cast<uint64_t>(F);
  // Activations [M][K] viewed as [sequence][flow][K]: a 64 x 2 x 64 box puts
  // sequence j's primary row at tile row 2j and its auxiliary row at 2j + 1
  // (sequences past m_primary read as zeros).
  const uint64_t mpu = static_cast<uint64_t>(m_primary);
  auto x_map = [&](CUtensorMap* m, const void* base, uint64_t K) {
    const uint64_t dims[3] = {K, 2, mpu};
    const uint64_t strides[2] = {mpu * K * 2, K * 2};
    const uint32_t box[3] = {kBK, 2, kBM / 2};
    return encode_tmap_bf16_3d_box(m, base, dims, strides, box);
  };
  if (!x_map(&tmXo, attn, qu) ||
      !encode_tmap_bf16_2d(&tmWo, w_o, du, qu, qu * 2, kTileN, kBK) ||
      !x_map(&tmXg, x_mid, du) ||
      !encode_tmap_bf16_2d(&tmWg, w_gu, 2 * Fu, du, du * 2, static_cast<uint32_t>(pl.H1), kBK) ||
      !x_map(&tmXd, h, Fu) ||
      !encode_tmap_bf16_2d(&tmWd, w_down, du, Fu, Fu * 2, kTileN, kBK))
    return DF_ERR_CUDA;
  CUtensorMap tmXq = tmXo, tmWq = tmWo, tmP = tmXo;  // (unused without P3)
  if (tn3 > 0) {
    // P3: x_out interleaved like the other activations; the partials
    // [rank][row][column] fp32 stored in boxes of 32 columns x 128 rows
    const uint64_t nout = static_cast<uint64_t>(nx.nout), Mu = static_cast<uint64_t>(M);
    const uint64_t dims[3] = {nout, Mu, kCluster};
    const uint64_t strides[2] = {nout * 4, Mu * nout * 4};
    const uint32_t box[3] = {32, kBM, 1};
    if (!x_map(&tmXq, x_out, du) ||
        !encode_tmap_bf16_2d(&tmWq, nx.w, nout, du, du * 2, static_cast<uint32_t>(tn3), kBK) ||
        !encode_tmap_f32_3d_box(&tmP, nx.part, dims, strides, box))
      return DF_ERR_CUDA;
  }

  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(pl.G);
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
  if (cudaLaunchKernelEx(&cfg, post_kernel, tmXo, tmWo, tmXg, tmWg, tmXd, tmWd, tmXq, tmWq, tmP,
                         p) != cudaSuccess)
    return DF_ERR_CUDA;
  return DF_OK;
}

}  // namespace post
}  // namespace df

extern "C" size_t dualflow_layer_post_attention_workspace_size(int m_primary, int d_model,
                                                               int q_dim, int F) {
  const df::post::Plan pl = df::post::make_plan(2 * m_primary, m_primary, d_model, q_dim, F);
  return pl.ok ? df::post::ws_bytes(d_model) : 0;
}

extern "C" df_status dualflow_layer_post_attention(
    const void* attn, const void* x, const void* w_o, const void* w_gu, const void* w_down,
    const void* b, const void* c, int m_primary, int d_model, int q_dim, int F, float eps,
    void* x_mid, void* h, void* x_out, void* workspace, size_t workspace_bytes,
    int32_t* err_flag, void* stream) {
  const df::post::QkvNext none{nullptr, 0, nullptr, nullptr};
  return df::post::launch_post(attn, x, w_o, w_gu, w_down, b, c, m_primary, d_model, q_dim, F,
                               eps, x_mid, h, x_out, workspace, workspace_bytes, err_flag, none,
                               stream);
}

extern "C" df_status dualflow_layer_post_attention_qkv(
    const void* attn, const void* x, const void* w_o, const void* w_gu, const void* w_down,
    const void* b, const void* c, int m_primary, int d_model, int q_dim, int F, float eps,
    void* x_mid, void* h, void* x_out, void* workspace, size_t workspace_bytes,
    const void* w_qkv_next, int Hq, int Hkv, int D, void* part, void* ss_part,
    int32_t* err_flag, void* stream) {
  if (!w_qkv_next) return DF_ERR_NULL;
  if (Hq < 1 || Hkv < 1 || D < 1 || Hq % Hkv != 0 || q_dim != Hq * D) return DF_ERR_SHAPE;
  const df::post::QkvNext nx{w_qkv_next, (Hq + 2 * Hkv) * D, part, ss_part};
  return df::post::launch_post(attn, x, w_o, w_gu, w_down, b, c, m_primary, d_model, q_dim, F,
                               eps, x_mid, h, x_out, workspace, workspace_bytes, err_flag, nx,
                               stream);
}
