// Post-attention half of the Dual-Flow decoder layer as ONE persistent kernel.
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
//   P0  W_o:    column tiles of 256 x S0 k-ranges -> fp32 partials
//   --- counter A --- R0: 4-column groups over all CTAs: x_mid = x + the sum
//                     of the partials (split order), and each CTA's partial
//                     sum of squares per row
//   --- counter A2 --- P1 may read x_mid; CTA r < M sums row r's squares in
//                     CTA order -> r_row   --- counter I ---
//   P1  W_gate/W_up: one tile of 2*H1 weight rows per CTA, SwiGLU (row scale
//                     r) + b coupling straight from TMEM -> h
//   --- counter C --- P2  W_down: column tiles of 256 x S2 k-ranges -> partials
//   --- counter D --- R2: 4-column groups over all CTAs: residual + c
//                     coupling -> x_out
// Partials are stored [unit][column group of 4][row][4] fp32: a warp's store
// (32 consecutive rows of one group) is one contiguous 512-byte segment, and a
// (group, split) item is one contiguous 2 KB block. The reductions bring all
// their items into the idle 192 KB weight ring with bulk TMA copies, one
// round trip at the layer's sizes (a latency-bound loop of loads took 13 us);
// the gate/up weight loads wait for the ring, and the gap is covered by L2
// prefetches of the next phase's first weight tiles, issued at each phase
// boundary only (prefetching ahead all the time took TMA bandwidth from the
// loads).
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
constexpr int kMaxHalf = 128;                     // SwiGLU output columns per tile
constexpr int kXchgPitch = 33;                    // coupling exchange: [64 rows][32 + 1]
constexpr int kXchgFloats = 64 * kXchgPitch;
constexpr int kCounters = 8;
constexpr size_t kCounterBytes = 256;
constexpr int kGroupBytes = kBM * 4 * 4;          // one 4-column group of a partial: 2 KB
constexpr int kRedItems = kStages * kSlot / kGroupBytes;  // reduction batch: the whole ring
constexpr int kBoundaryPrefetch = 16;             // next-phase weight stages prefetched to L2
constexpr size_t kSmemBytes = 1024 + static_cast<size_t>(kStages) * kSlot + kXchgFloats * 4 +
                              kEpiThreads * 4 + kMaxHalf * 4 + 256;  // + barriers, flags
static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");

enum { kCntA = 0, kCntA2 = 1, kCntI = 2, kCntC = 3, kCntD = 4, kCntExit = 5 };

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
  const __nv_bfloat16* x;
  const __nv_bfloat16* b;
  const __nv_bfloat16* c;
  __nv_bfloat16* x_mid;
  __nv_bfloat16* h;
  __nv_bfloat16* x_out;
  float* part;     // [units][64 groups][128 rows][4] fp32
  float* ss_part;  // [G][128] per-CTA partial sums of squares of x_mid rows
  float* rscale;   // [128] RMSNorm row scales
  int* cnt;        // [kCounters]
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

// Walks this CTA's stage sequence (GEMM q, its units u = cta, cta + G, ...,
// their k-blocks) in the order the producers and the MMA issuer use.
struct StageCursor {
  int q, u, kb, k1, tile;
  bool done;
  __device__ StageCursor(const Params& p, int cta, int G) : q(0), u(cta), kb(0), k1(0), tile(0),
                                                          done(false) {
    seek(p, G);
  }
  // first stage of unit u of GEMM q, or of the next GEMM that has one
  __device__ void seek(const Params& p, int G) {
    while (q < 3 && u >= p.g[q].units) {
      ++q;
      u = u % G;  // this CTA's index
    }
    if (q >= 3) {
      done = true;
      return;
    }
    int k0;
    unit_range(p.g[q], u, tile, k0, k1);
    kb = k0;
  }
  __device__ void next(const Params& p, int cta, int G) {
    if (++kb < k1) return;
    u += G;
    if (u >= p.g[q].units) {
      ++q;
      u = cta;
    }
    seek(p, G);
  }
};

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

// Two 32-column TMEM loads (this thread's lane), one wait.
__device__ __forceinline__ void tmem_ld64(uint32_t taddr, float (&v)[64]) {
  uint32_t r[64];
  __syncwarp();
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "
      "%28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "
      "%28, %29, %30, %31}, [%32];"
      : "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]), "=r"(r[37]),
        "=r"(r[38]), "=r"(r[39]), "=r"(r[40]), "=r"(r[41]), "=r"(r[42]), "=r"(r[43]),
        "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]), "=r"(r[48]), "=r"(r[49]),
        "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]), "=r"(r[55]),
        "=r"(r[56]), "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]), "=r"(r[61]),
        "=r"(r[62]), "=r"(r[63])
      : "r"(taddr + 32));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 64; ++i) v[i] = __uint_as_float(r[i]);
}

// Accumulator (row = this thread's TMEM lane, 256 columns) -> the unit's fp32
// partial slab [64 groups][128 rows][4]: for each group the warp's 32 lanes
// store one contiguous 512-byte segment, straight from registers.
__device__ void store_partial(const Params& p, float* slab, uint32_t taddr, int row) {
  for (int c = 0; c < kTileN; c += 64) {
    float v[64];
    tmem_ld64(taddr + c, v);
    if (row < p.M) {
#pragma unroll
      for (int q = 0; q < 16; ++q)
        st_cg4(slab + (static_cast<size_t>(c / 4 + q) * kBM + row) * 4,
               make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]));
    }
  }
}

__device__ __forceinline__ void load_bf16x4_cg(const __nv_bfloat16* src, float (&v)[4]) {
  uint32_t w0, w1;
  asm volatile("ld.global.cg.v2.u32 {%0, %1}, [%2];" : "=r"(w0), "=r"(w1) : "l"(src));
  v[0] = bf16_bits_to_float(static_cast<uint16_t>(w0 & 0xffffu));
  v[1] = bf16_bits_to_float(static_cast<uint16_t>(w0 >> 16));
  v[2] = bf16_bits_to_float(static_cast<uint16_t>(w1 & 0xffffu));
  v[3] = bf16_bits_to_float(static_cast<uint16_t>(w1 >> 16));
}

__device__ __forceinline__ void bulk_g2s(uint32_t sdst, const void* gsrc, uint32_t bytes,
                                         uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          sdst),
      "l"(gsrc), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// Streams the S split partials of each of this CTA's 4-column groups (gi =
// cta, cta + G, ...) into shared memory by bulk TMA copies (one 2 KB copy
// per (group, split): all 128 rows of those 4 columns), as many at once as
// the idle weight ring holds (all of them at the layer's sizes: one round
// trip), and hands every item to on_item(gi, s, bytes) in split order, then
// on_group(gi) after its last split. Thread et == 0 issues the copies;
// `batches` counts the batches of earlier calls (it sets the barrier phase).
// Returns false if a wait gave up. The caller guarantees that no weight or
// activation copy targets the ring meanwhile.
template <class OnItem, class OnGroup>
__device__ bool stream_partials(const Params& p, int S, int cta, int G, uint8_t* rbuf,
                                uint64_t* rfull, int& batches, int et, OnItem on_item,
                                OnGroup on_group) {
  const int groups = p.d / 4;
  const int mine = groups > cta ? (groups - cta + G - 1) / G : 0;
  const int n = mine * S;
  const int nb = (n + kRedItems - 1) / kRedItems;
  bool ok = true;
  for (int b = 0; b < nb; ++b) {
    const int gb = batches + b;
    const int k0 = b * kRedItems, k1 = min(n, k0 + kRedItems);
    if (et == 0) {
      if (b == 0) fence_proxy_async_global();  // partials stored by other CTAs -> bulk copies
      mbar_arrive_expect_tx(rfull, static_cast<uint32_t>((k1 - k0) * kGroupBytes));
      for (int k = k0; k < k1; ++k) {
        const int gi = cta + (k / S) * G, sp = k % S;
        const int tile = gi / (kTileN / 4), g = gi - tile * (kTileN / 4);
        const float* src =
            p.part + (static_cast<size_t>(tile * S + sp) * (kTileN / 4) + g) * (kBM * 4);
        bulk_g2s(smem_u32(rbuf + (k - k0) * kGroupBytes), src, kGroupBytes, rfull);
      }
    }
    if (!mbar_wait(rfull, static_cast<uint32_t>(gb & 1))) ok = false;
    if (ok) {
      for (int k = k0; k < k1; ++k) {
        const int gi = cta + (k / S) * G, sp = k % S;
        on_item(gi, sp, rbuf + (k - k0) * kGroupBytes);
        if (sp == S - 1) on_group(gi);
      }
    }
    epi_bar();  // every thread is done with the batch before the next one lands
  }
  batches += nb;
  return ok;
}

// R0 on this CTA's 4-column groups (thread = row): x_mid = bf16(x + sum of the
// W_o partials in split order); this CTA's sum of squares of each row's
// stored values goes to ss_part[cta][row].
constexpr int kPreGroups = 8;  // residual values of up to this many groups held in registers

__device__ bool reduce_o(const Params& p, int cta, int G, int et, uint8_t* rbuf, uint64_t* rfull,
                         int& batches) {
  const int row = et;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  float ss = 0.f;
  const bool live = row < p.M;
  // The residual values of this thread's groups are loaded before the partials
  // arrive, so no group waits for a load of its own.
  const int groups = p.d / 4;
  uint2 pre[kPreGroups];
#pragma unroll
  for (int i = 0; i < kPreGroups; ++i) {
    const int gi = cta + i * G;
    pre[i] = (live && gi < groups)
                 ? *reinterpret_cast<const uint2*>(p.x + static_cast<size_t>(row) * p.d + gi * 4)
                 : make_uint2(0u, 0u);
  }
  const bool ok = stream_partials(
      p, p.g[0].splits, cta, G, rbuf, rfull, batches, et,
      [&](int, int, const uint8_t* item) {
        const float4 v = *reinterpret_cast<const float4*>(item + row * 16);
        acc.x += v.x;
        acc.y += v.y;
        acc.z += v.z;
        acc.w += v.w;
      },
      [&](int gi) {
        if (live) {
          const int i = (gi - cta) / G;
          float res[4];
          if (i < kPreGroups) {
            uint2 w = make_uint2(0u, 0u);
#pragma unroll
            for (int k = 0; k < kPreGroups; ++k)
              if (k == i) w = pre[k];
            res[0] = bf16_bits_to_float(static_cast<uint16_t>(w.x & 0xffffu));
            res[1] = bf16_bits_to_float(static_cast<uint16_t>(w.x >> 16));
            res[2] = bf16_bits_to_float(static_cast<uint16_t>(w.y & 0xffffu));
            res[3] = bf16_bits_to_float(static_cast<uint16_t>(w.y >> 16));
          } else {
            load_bf16x4(p.x + static_cast<size_t>(row) * p.d + gi * 4, res);
          }
          float o[4] = {acc.x + res[0], acc.y + res[1], acc.z + res[2], acc.w + res[3]};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            o[i] = __bfloat162float(__float2bfloat16_rn(o[i]));
            ss = fmaf(o[i], o[i], ss);
          }
          store_bf16x4(p.x_mid + static_cast<size_t>(row) * p.d + gi * 4, o);
        }
        acc = make_float4(0.f, 0.f, 0.f, 0.f);
      });
  p.ss_part[static_cast<size_t>(cta) * kBM + row] = ss;
  return ok;
}

// Row scale of row r: 1 / sqrt(sum over CTAs of ss_part[.][r] / d + eps),
// summed in a fixed order (thread et adds CTAs et, et + 128, ...; then a
// fixed tree over the 128 threads).
__device__ void row_scale(const Params& p, int G, int r, int et, float* red) {
  float v = 0.f;
  for (int k = et; k < G; k += kEpiThreads) v += __ldcg(p.ss_part + static_cast<size_t>(k) * kBM + r);
  red[et] = v;
  epi_bar();
  for (int w = kEpiThreads / 2; w > 0; w >>= 1) {
    if (et < w) red[et] += red[et + w];
    epi_bar();
  }
  if (et == 0) p.rscale[r] = 1.0f / sqrtf(red[0] / static_cast<float>(p.d) + p.eps);
  epi_bar();
}

// P1 epilogue of tile t: h[row][t*H + j] = SiLU(rs g) * (rs u) (+ b * primary
// row's value for auxiliary rows), in 32-column chunks (8-column tail); the
// primary rows' values reach their auxiliary rows through `xchg`.
template <int W>
__device__ __forceinline__ void swiglu_chunk(const Params& p, uint32_t taddr, int H, int c, int col0,
                                             int row, float rs, float* xchg, const float* bsl) {
  float g[W], u[W];
  tmem_ld<W>(taddr + c, g);
  tmem_ld<W>(taddr + H + c, u);
#pragma unroll
  for (int i = 0; i < W; ++i) g[i] = silu_f(rs * g[i]) * (rs * u[i]);
  if (p.b != nullptr) {
    if (row < p.mp) {
#pragma unroll
      for (int i = 0; i < W; ++i) xchg[row * kXchgPitch + i] = g[i];
    }
    epi_bar();
    if (row >= p.mp && row < p.M && col0 + c < p.F) {
#pragma unroll
      for (int i = 0; i < W; ++i) g[i] = fmaf(bsl[c + i], xchg[(row - p.mp) * kXchgPitch + i], g[i]);
    }
    epi_bar();
  }
  if (row < p.M) {
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

__device__ void swiglu_epilogue(const Params& p, int t, uint32_t taddr, int row, float rs,
                                float* xchg, const float* bsl) {
  const int H = p.g[1].half;
  const int col0 = t * H;
  int c = 0;
  for (; c + 32 <= H; c += 32) swiglu_chunk<32>(p, taddr, H, c, col0, row, rs, xchg, bsl);
  for (; c < H; c += 8) swiglu_chunk<8>(p, taddr, H, c, col0, row, rs, xchg, bsl);
}

// Tile t's slice of the coupling vector b into shared memory (zeros past F),
// fetched while the tile's MMAs run.
__device__ void load_b_slice(const Params& p, int t, int et, float* bsl) {
  const int H = p.g[1].half;
  for (int i = et; i < H; i += kEpiThreads) {
    const int col = t * H + i;
    bsl[i] = (p.b != nullptr && col < p.F) ? __bfloat162float(p.b[col]) : 0.f;
  }
  epi_bar();
}

// R2 on this CTA's 4-column groups: thread et handles sequence j = et % 64
// (rows j and mp + j), columns 2 (et / 64) .. + 1 of each group: x_out =
// x_mid + the sum of the W_down partials in split order, the auxiliary row
// adding c * (primary row's sum) first.
__device__ bool reduce_down(const Params& p, int cta, int G, int et, uint8_t* rbuf,
                            uint64_t* rfull, int& batches) {
  const int j = et & 63, hc = (et >> 6) * 2;
  const bool live = j < p.mp;
  float2 ap = make_float2(0.f, 0.f), aa = make_float2(0.f, 0.f);
  // residual (x_mid, written by other CTAs: read through L2) and coupling
  // values of this thread's groups, loaded before the partials arrive
  const int groups = p.d / 4;
  uint32_t pre_p[kPreGroups], pre_a[kPreGroups], pre_c[kPreGroups];
#pragma unroll
  for (int i = 0; i < kPreGroups; ++i) {
    const int gi = cta + i * G;
    const bool in = live && gi < groups;
    const int col = gi * 4 + hc;
    pre_p[i] = in ? __ldcg(reinterpret_cast<const unsigned int*>(
                        p.x_mid + static_cast<size_t>(j) * p.d + col))
                  : 0u;
    pre_a[i] = in ? __ldcg(reinterpret_cast<const unsigned int*>(
                        p.x_mid + static_cast<size_t>(p.mp + j) * p.d + col))
                  : 0u;
    pre_c[i] = (in && p.c != nullptr) ? *reinterpret_cast<const uint32_t*>(p.c + col) : 0u;
  }
  return stream_partials(
      p, p.g[2].splits, cta, G, rbuf, rfull, batches, et,
      [&](int, int, const uint8_t* item) {
        if (!live) return;
        const float2 vp = *reinterpret_cast<const float2*>(item + j * 16 + hc * 4);
        const float2 va = *reinterpret_cast<const float2*>(item + (p.mp + j) * 16 + hc * 4);
        ap.x += vp.x;
        ap.y += vp.y;
        aa.x += va.x;
        aa.y += va.y;
      },
      [&](int gi) {
        if (live) {
          const int col = gi * 4 + hc;
          const int i = (gi - cta) / G;
          uint32_t wp = 0u, wa = 0u, wc = 0u;
          if (i < kPreGroups) {
#pragma unroll
            for (int k = 0; k < kPreGroups; ++k)
              if (k == i) {
                wp = pre_p[k];
                wa = pre_a[k];
                wc = pre_c[k];
              }
          } else {
            wp = __ldcg(reinterpret_cast<const unsigned int*>(p.x_mid + static_cast<size_t>(j) * p.d + col));
            wa = __ldcg(reinterpret_cast<const unsigned int*>(
                p.x_mid + static_cast<size_t>(p.mp + j) * p.d + col));
            if (p.c != nullptr) wc = *reinterpret_cast<const uint32_t*>(p.c + col);
          }
          float op[2] = {ap.x, ap.y}, oa[2] = {aa.x, aa.y};
          if (p.c != nullptr) {
            oa[0] = fmaf(bf16_bits_to_float(static_cast<uint16_t>(wc & 0xffffu)), op[0], oa[0]);
            oa[1] = fmaf(bf16_bits_to_float(static_cast<uint16_t>(wc >> 16)), op[1], oa[1]);
          }
          op[0] += bf16_bits_to_float(static_cast<uint16_t>(wp & 0xffffu));
          op[1] += bf16_bits_to_float(static_cast<uint16_t>(wp >> 16));
          oa[0] += bf16_bits_to_float(static_cast<uint16_t>(wa & 0xffffu));
          oa[1] += bf16_bits_to_float(static_cast<uint16_t>(wa >> 16));
          *reinterpret_cast<__nv_bfloat162*>(p.x_out + static_cast<size_t>(j) * p.d + col) =
              __floats2bfloat162_rn(op[0], op[1]);
          *reinterpret_cast<__nv_bfloat162*>(p.x_out + static_cast<size_t>(p.mp + j) * p.d + col) =
              __floats2bfloat162_rn(oa[0], oa[1]);
        }
        ap = make_float2(0.f, 0.f);
        aa = make_float2(0.f, 0.f);
      });
}

__global__ void __launch_bounds__(kThreads, 1)
    post_kernel(const __grid_constant__ CUtensorMap tmXo, const __grid_constant__ CUtensorMap tmWo,
                const __grid_constant__ CUtensorMap tmXg, const __grid_constant__ CUtensorMap tmWg,
                const __grid_constant__ CUtensorMap tmXd, const __grid_constant__ CUtensorMap tmWd,
                const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* rbuf = smem;  // the weight ring, while a reduction has it
  float* xchg = reinterpret_cast<float*>(smem + static_cast<size_t>(kStages) * kSlot);
  float* red = xchg + kXchgFloats;                                // [kEpiThreads]
  float* bsl = red + kEpiThreads;                                 // [kMaxHalf] b of a tile
  uint64_t* full = reinterpret_cast<uint64_t*>(bsl + kMaxHalf);   // [kStages]
  uint64_t* empty = full + kStages;                               // [kStages]
  uint64_t* acc_full = empty + kStages;                           // [2]
  uint64_t* acc_empty = acc_full + 2;                             // [2]
  uint64_t* mma_done = acc_empty + 2;                             // [1]
  uint64_t* rfull = mma_done + 1;     // reduction batch landed
  uint64_t* ring_free = rfull + 1;    // R0 is done with the ring: gate/up weights may load
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(ring_free + 1);
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
    mbar_init(rfull, 1);
    mbar_init(ring_free, 1);
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
      // At a phase boundary the MMAs wait for the next phase's activations:
      // the next phase's first weight tiles are prefetched into L2 there, so
      // DRAM keeps streaming and those stages later load from L2. Before the
      // first gate/up stage the ring is lent to the W_o reduction (R0): its
      // loads wait until R0 has released it.
      auto prefetch_phase = [&](int q, int count) {
        StageCursor pf(p, cta, G);
        while (!pf.done && pf.q < q) pf.next(p, cta, G);
        for (int i = 0; i < count && !pf.done && pf.q == q; ++i) {
          const Gemm& gq = p.g[q];
          const CUtensorMap* tq = q == 0 ? &tmWo : (q == 1 ? &tmWg : &tmWd);
          if (q == 1) {
            tma_prefetch_2d(tq, pf.kb * kBK, pf.tile * gq.half);
            tma_prefetch_2d(tq, pf.kb * kBK, p.F + pf.tile * gq.half);
          } else {
            tma_prefetch_2d(tq, pf.kb * kBK, pf.tile * kTileN);
          }
          pf.next(p, cta, G);
        }
      };
      int s = 0;
      uint32_t ph = 0;
      long long n = 0;
      bool ok = true;
      for (int q = 0; q < 3 && ok; ++q) {
        const Gemm& g = p.g[q];
        const CUtensorMap* tm = q == 0 ? &tmWo : (q == 1 ? &tmWg : &tmWd);
        if (q >= 1) prefetch_phase(q, kBoundaryPrefetch);
        if (q == 1 && !mbar_wait(ring_free, 0)) {
          set_err(p.err, DF_DEVERR_TIMEOUT);
          flags[0] = 1;
          ok = false;
          break;
        }
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
            // P1 reads x_mid (counter A2), P2 every column of h (C)
            if (!wait_count(p.cnt + (q == 1 ? kCntA2 : kCntC), G)) {
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
    const int row = quarter * 32 + lane;  // this thread's TMEM lane = accumulator row
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
    // P0: W_o partials
    for (int u = cta; u < p.g[0].units && ok; u += G, ++seg) {
      const int acc = seg & 1;
      if (!take_acc(acc, seg)) {
        ok = false;
        break;
      }
      tc_fence_after();
      store_partial(p, p.part + static_cast<size_t>(u) * kBM * kTileN, acc_addr(acc), row);
      give_acc(acc);
    }
    arrive_count(p.cnt + kCntA, et);
    // R0: x_mid and this CTA's row sums of squares
    // (the ring is idle: every W_o stage has been consumed, and the producers
    // hold back the gate/up stages until ring_free)
    int rbatches = 0;
    if (grid_wait(kCntA) && !flags[0] && !reduce_o(p, cta, G, et, rbuf, rfull, rbatches)) {
      if (et == 0) set_err(p.err, DF_DEVERR_TIMEOUT);
      flags[0] = 1;
    }
    if (et == 0) mbar_arrive(ring_free);
    arrive_count(p.cnt + kCntA2, et);
    // row scales of the norm (CTA r < M computes row r)
    if (cta < p.M && grid_wait(kCntA2) && !flags[0]) row_scale(p, G, cta, et, red);
    arrive_count(p.cnt + kCntI, et);
    // P1: SwiGLU tiles straight from TMEM
    float rs = 0.f;
    bool have_rs = false;
    for (int u = cta; u < p.g[1].units && ok; u += G, ++seg) {
      const int acc = seg & 1;
      if (!have_rs) {
        if (!grid_wait(kCntI)) {
          ok = false;
          break;
        }
        rs = row < p.M ? __ldcg(p.rscale + row) : 0.f;
        have_rs = true;
      }
      if (p.b != nullptr) load_b_slice(p, u, et, bsl);
      if (!take_acc(acc, seg)) {
        ok = false;
        break;
      }
      tc_fence_after();
      swiglu_epilogue(p, u, acc_addr(acc), row, rs, xchg, bsl);
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
      store_partial(p, p.part + static_cast<size_t>(u) * kBM * kTileN, acc_addr(acc), row);
      give_acc(acc);
    }
    arrive_count(p.cnt + kCntD, et);
    // R2: x_out (the ring is idle again: every W_down stage has been consumed)
    if (grid_wait(kCntD) && !flags[0] && !reduce_down(p, cta, G, et, rbuf, rfull, rbatches)) {
      if (et == 0) set_err(p.err, DF_DEVERR_TIMEOUT);
      flags[0] = 1;
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

// Workspace: counters | ss_part [G][128] | rscale [128] | partials.
struct WsLayout {
  size_t ss, rscale, part, total;
};

WsLayout ws_layout(const Plan& pl) {
  const int units = pl.T0 * pl.S0 > pl.T2 * pl.S2 ? pl.T0 * pl.S0 : pl.T2 * pl.S2;
  WsLayout l;
  l.ss = kCounterBytes;
  l.rscale = l.ss + round_up(static_cast<size_t>(pl.G) * kBM * 4, 256);
  l.part = l.rscale + round_up(kBM * 4, 256);
  l.total = l.part + static_cast<size_t>(units) * kBM * kTileN * 4;
  return l;
}

std::mutex g_mu;
bool g_attr[64] = {};

}  // namespace post
}  // namespace df

extern "C" size_t dualflow_layer_post_attention_workspace_size(int m_primary, int d_model,
                                                               int q_dim, int F) {
  const df::post::Plan pl = df::post::make_plan(2 * m_primary, m_primary, d_model, q_dim, F);
  return pl.ok ? df::post::ws_layout(pl).total : 0;
}

extern "C" df_status dualflow_layer_post_attention(
    const void* attn, const void* x, const void* w_o, const void* w_gu, const void* w_down,
    const void* b, const void* c, int m_primary, int d_model, int q_dim, int F, float eps,
    void* x_mid, void* h, void* x_out, void* workspace, size_t workspace_bytes,
    int32_t* err_flag, void* stream) {
  using namespace df;
  using namespace df::post;
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
  const WsLayout wl = ws_layout(pl);
  if (!workspace || workspace_bytes < wl.total || !aligned(workspace, 256))
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
  p.x = static_cast<const __nv_bfloat16*>(x);
  p.b = static_cast<const __nv_bfloat16*>(b);
  p.c = static_cast<const __nv_bfloat16*>(c);
  p.x_mid = static_cast<__nv_bfloat16*>(x_mid);
  p.h = static_cast<__nv_bfloat16*>(h);
  p.x_out = static_cast<__nv_bfloat16*>(x_out);
  uint8_t* w8 = static_cast<uint8_t*>(workspace);
  p.cnt = reinterpret_cast<int*>(w8);
  p.ss_part = reinterpret_cast<float*>(w8 + wl.ss);
  p.rscale = reinterpret_cast<float*>(w8 + wl.rscale);
  p.part = reinterpret_cast<float*>(w8 + wl.part);
  p.err = err_flag;

  CUtensorMap tmXo, tmWo, tmXg, tmWg, tmXd, tmWd;
  const uint64_t Mu = static_cast<uint64_t>(M), du = static_cast<uint64_t>(d_model),
                 qu = static_cast<uint64_t>(q_dim), Fu = static_cast<uint64_t>(F);
  if (!encode_tmap_bf16_2d(&tmXo, attn, Mu, qu, qu * 2, kBM, kBK) ||
      !encode_tmap_bf16_2d(&tmWo, w_o, du, qu, qu * 2, kTileN, kBK) ||
      !encode_tmap_bf16_2d(&tmXg, x_mid, Mu, du, du * 2, kBM, kBK) ||
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
