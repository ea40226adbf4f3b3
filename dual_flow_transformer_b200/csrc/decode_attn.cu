// Dual-flow decode attention: asymmetric shared-KV attention of the primary
// query Q1 and the coupled auxiliary query Q2 = Q2raw + a (.) Q1 over the single
// primary cache (K1, V1), optionally split over the sequence (flash-decoding).
//
// Method: "Sintesi Tecnica: Dual-Flow Transformers", section "Meccanismi
// Chiave" -- the auxiliary flow attends to the primary flow's keys and values
// without writing its own, so each KV region can be loaded once for both flows.
//
// bf16 kernel design (sm_100a):
//  * one CTA per (split, KV head g, sequence b); 4 consumer warps + 1 TMA
//    producer warp; 64-token pages of K and V arrive by TMA (128-byte swizzle)
//    into a STAGES-deep shared-memory ring guarded by mbarriers;
//  * each page is read from HBM exactly once and serves all 2*G query rows of
//    KV head g: rows 0..3 = primary heads, 4..7 = auxiliary heads (bf16 "hi"
//    part of the fp32 coupled Q2), 12..15 = the auxiliary "lo" part
//    (bf16(Q2 - hi)), 8..11 = the primary lo part (zero, Q1 is bf16-exact).
//    The m16n8k16 fragment keeps row r and r+8 in the same thread, so hi + lo
//    scores add in registers: Q2 enters the scores at ~16 significant bits;
//  * QK^T and PV run on mma.sync (bf16 in, fp32 accumulate; one 16-row tile
//    per page needs a small fraction of the tensor rate the HBM stream
//    allows). The softmax weights P are split the same way (hi in rows r, lo
//    in rows r+8) so PV also sees ~16-bit weights. Each warp owns 16 tokens of
//    every page and keeps its own running max / sum per row (online softmax
//    in the exp2 domain, quad shuffles), merged across warps through shared
//    memory;
//  * splits only when the (b, g) units cannot fill the two resident CTAs per
//    SM (see make_plan); split partials are combined inside the kernel by the
//    last split CTA of each unit to finish (arrival counter, split order);
//  * every query row's arithmetic is independent of every other row's, and
//    the split plan depends only on (B, Hkv, max_seqlen), so O1 is
//    bit-identical whatever the auxiliary inputs are.
#include <math.h>

#include <cudaTypedefs.h>

#include <mutex>
#include <utility>
#include <vector>

#include "common.cuh"
#include "host_util.h"

namespace df {
namespace attn {

constexpr int kPage = 64;                 // tokens per page (block_size)
constexpr int kConsumerWarps = 4;         // each owns 16 tokens of a page
constexpr int kThreads = (kConsumerWarps + 1) * 32;
constexpr int kStagesBf16 = 3;            // pipeline depth of the bf16 kernel
constexpr int kSlots = 148 * 2;            // resident split CTAs (two per SM)
constexpr int kSplitWaves = 2;             // split plans aim at ~2 waves of CTAs
constexpr int kMinChunkPages = 8;         // >= 512 tokens per split

struct Params {
  const void* q1;
  const void* q2raw;
  const void* a;
  int64_t q_stride_b;
  const void* k_cache;
  const void* v_cache;
  const int32_t* block_table;
  int max_blocks_per_seq;
  const int32_t* seqlens;
  int max_seqlen;
  void* o1;
  void* o2;
  int64_t o_stride_b;
  int B, Hq, Hkv, G, num_blocks;
  float scale_log2;  // softmax scale * log2(e)
  int chunk_pages;   // pages per split
  int num_splits;
  float* part_o;     // [B][2Hq][S][D]
  float* part_ml;
  int* counters;     // bf16 path with splits: [B][Hkv] arrival counters (zero between calls)    // [B][2Hq][S][2] (running max in log2 units, sum)
  int32_t* err;
  int dual;          // auxiliary rows computed
  int write1;        // store O1
  int write2;        // store O2
  // Partials mode (qpart != nullptr; bf16 kernel): Q1, Q2raw and this
  // step's K / V rows are not read from memory but built in the prologue
  // from qparts fp32 partial products [part][row][column] of the QKV
  // projection (row b primary, qmp + b auxiliary; columns: Q of head h at
  // h D, K of KV head g at qkcol + g D, V at qvcol + g D) and the parts'
  // row sums of squares qss [part][row]: with r = 1 / sqrt(sum qss / qd +
  // qeps), each value is bf16(r (sum of the parts in part order)); K and V
  // are appended to the cache at position seqlens[b] - 1 before its page is
  // read.
  const float* qpart;
  const float* qss;
  int qparts, qmp, qd, qkcol, qvcol;
  int64_t qrow;   // floats between rows
  int64_t qpstr;  // floats between parts
  float qeps;
};

struct Plan {
  int splits;
  int chunk_pages;
};

// Partials mode: most partial products a call may sum (the QKV partials
// launch writes 4, one per quarter of d_model).
constexpr int kMaxParts = 4;

__device__ __forceinline__ float4 ldg_f4(const float* ptr) {
  return *reinterpret_cast<const float4*>(ptr);
}
__device__ __forceinline__ float4 f4_add(float4 a, float4 b) {
  return make_float4(a.x + b.x, a.y + b.y, a.z + b.z, a.w + b.w);
}
__device__ __forceinline__ float4 f4_scale(float4 a, float r) {
  return make_float4(a.x * r, a.y * r, a.z * r, a.w * r);
}
// 4 bf16 (round to nearest even) to an 8-byte-aligned address
__device__ __forceinline__ void store_bf16x4(__nv_bfloat16* dst, float4 v) {
  __nv_bfloat162 lo = __floats2bfloat162_rn(v.x, v.y), hi = __floats2bfloat162_rn(v.z, v.w);
  uint2 u;
  u.x = *reinterpret_cast<uint32_t*>(&lo);
  u.y = *reinterpret_cast<uint32_t*>(&hi);
  *reinterpret_cast<uint2*>(dst) = u;
}

inline Plan make_plan(int B, int Hkv, int max_seqlen, int block_size, int requested) {
  const int max_pages = static_cast<int>(ceil_div(max_seqlen, block_size));
  int s0;
  if (requested > 0) {
    s0 = requested < max_pages ? requested : max_pages;
  } else {
    // Measured on B200: a CTA that streams a whole (sequence, KV head) unit
    // ends at no cost (its successor's start overlaps the other CTA of the
    // SM), while a split CTA adds ~3-6 us of slot time (partials, fence,
    // arrival, merge). So one CTA per unit whenever the units fill every
    // slot; otherwise enough splits for ~kSplitWaves waves at the longest
    // length, each of at least kMinChunkPages pages.
    const int64_t units = static_cast<int64_t>(B) * Hkv;
    int64_t want = units >= kSlots ? 1 : ceil_div(int64_t(kSplitWaves) * kSlots, units);
    int64_t cap = max_pages / kMinChunkPages;
    if (cap < 1) cap = 1;
    if (want > cap) want = cap;
    if (want < 1) want = 1;
    s0 = static_cast<int>(want);
  }
  Plan p;
  p.chunk_pages = static_cast<int>(ceil_div(max_pages, s0));
  p.splits = static_cast<int>(ceil_div(max_pages, p.chunk_pages));
  return p;
}

// max that propagates NaN (fmaxf drops it), so NaN inputs give NaN outputs.
__device__ __forceinline__ float max_nan(float a, float b) { return (a != a || a > b) ? a : b; }

// Normalise; an empty row (no attended token) gives 0, a NaN row stays NaN.
__device__ __forceinline__ float safe_div(float o, float l) { return (l == 0.f) ? 0.f : o / l; }

__device__ __forceinline__ int clamp_len(const Params& p, int L) {
  if (L < 1) return 0;
  return L < p.max_seqlen ? L : p.max_seqlen;
}

__device__ __forceinline__ int attended_len(const Params& p, int b) {
  return clamp_len(p, p.seqlens[b]);
}

__device__ __forceinline__ void flag_len(const Params& p, int b) {
  const int L = p.seqlens[b];
  if (L < 1 || L > p.max_seqlen) set_err(p.err, DF_DEVERR_SEQLEN);
}

// Byte address of 16-byte chunk `ch` of token row `tok` inside a TMA-written
// [64 tokens][D] bf16 tile stored as D/64 column halves of [64][128 B] with the
// 128-byte swizzle (chunk index XOR row index within each 8-row group).
__device__ __forceinline__ uint32_t swz(uint32_t base, int tok, int ch) {
  return base + (ch >> 3) * (kPage * 128) + tok * 128 + (((ch & 7) ^ (tok & 7)) << 4);
}

template <typename T>
__device__ __forceinline__ float ld_f(const T* p);
template <>
__device__ __forceinline__ float ld_f<float>(const float* p) { return *p; }
template <>
__device__ __forceinline__ float ld_f<__nv_bfloat16>(const __nv_bfloat16* p) {
  return __bfloat162float(*p);
}

template <typename T>
__device__ __forceinline__ void st_f(T* p, float v);
template <>
__device__ __forceinline__ void st_f<float>(float* p, float v) { *p = v; }
template <>
__device__ __forceinline__ void st_f<__nv_bfloat16>(__nv_bfloat16* p, float v) {
  *p = __float2bfloat16_rn(v);
}

// Write zeros for every requested output row of (b, g): used when a sequence
// has no attended token (seqlens[b] < 1) and there is a single split.
template <typename T, int D>
__device__ void write_zero_rows(const Params& p, int b, int g, int tid, int nthreads) {
  for (int idx = tid; idx < 2 * p.G * D; idx += nthreads) {
    const int r = idx / D, d = idx % D;
    const int flow = r / p.G, h = g * p.G + (r % p.G);
    if (flow == 0 && p.write1)
      st_f(static_cast<T*>(p.o1) + b * p.o_stride_b + h * D + d, 0.f);
    if (flow == 1 && p.write2)
      st_f(static_cast<T*>(p.o2) + b * p.o_stride_b + h * D + d, 0.f);
  }
}

// ------------------------------------------------------------------ bf16 split

template <int D, int STAGES>
__global__ void __launch_bounds__(kThreads, 2)
    split_bf16_kernel(const __grid_constant__ CUtensorMap tmK,
                      const __grid_constant__ CUtensorMap tmV, const Params p) {
  constexpr int kTileBytes = kPage * D * 2;  // one K (or V) page
  constexpr int kStageBytes = 2 * kTileBytes;
  constexpr int KS = D / 16;  // k-steps of Q K^T
  constexpr int NT = D / 8;   // n-tiles of P V
  constexpr float kNegInf = -INFINITY;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * kStageBytes);
  uint64_t* empty = full + STAGES;
  int* stage_valid = reinterpret_cast<int*>(empty + STAGES);
  uint64_t* kv_ready = reinterpret_cast<uint64_t*>(smem + STAGES * kStageBytes + 64);
  __nv_bfloat16* q1s = reinterpret_cast<__nv_bfloat16*>(smem + STAGES * kStageBytes + 128);
  __nv_bfloat16* q2s = q1s + 4 * D;  // partials mode: this KV head's Q1 / Q2raw rows

  const int split = blockIdx.x, g = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  pdl_wait();
  pdl_trigger();

  // Longest sequences first: with one CTA per (sequence, KV head) and ragged
  // lengths, the CTAs are issued roughly in blockIdx order, so a long
  // sequence that comes late sets the tail. Grid row z takes the sequence
  // of rank z by descending length (ties in index order: a uniform batch
  // keeps its order), ranked by every CTA from the lengths in shared memory
  // (the one load of them replaces the load of its own length).
  int b = blockIdx.z;
  int len_b = -1;  // seqlens[b], when already loaded
  if (p.qpart == nullptr && gridDim.x == 1 && p.B > 1 && p.B <= kThreads) {
    __shared__ int s_len[kThreads];
    __shared__ int s_b;
    const int t = threadIdx.x;
    const int Lt = t < p.B ? p.seqlens[t] : 0;
    const int L0 = p.seqlens[0];
    if (t < p.B) s_len[t] = Lt;
    // (a uniform batch keeps its order: no ranking)
    if (!__syncthreads_and(t >= p.B || Lt == L0)) {
      if (t < p.B) {
        int rank = 0;
#pragma unroll 8
        for (int j = 0; j < p.B; ++j) {
          const int Lj = s_len[j];
          rank += (Lj > Lt || (Lj == Lt && j < t)) ? 1 : 0;
        }
        if (rank == static_cast<int>(blockIdx.z)) s_b = t;
      }
      __syncthreads();
      b = s_b;
    }
    len_b = s_len[b];
  }

  // Partials mode: the query rows' partial products and row sums of squares
  // are loaded first (one L2 round trip, overlapping the set-up below);
  // consumer thread ct owns 4 consecutive Q columns of both rows.
  const int G = p.G;
  const bool has_q = p.qpart != nullptr && warp < kConsumerWarps && 4 * static_cast<int>(threadIdx.x) < G * D;
  float4 v1[kMaxParts], v2[kMaxParts];
  float ss1[kMaxParts], ss2[kMaxParts];
#pragma unroll
  for (int k = 0; k < kMaxParts; ++k) {
    const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
    const bool pk = has_q && k < p.qparts;
    const int64_t o = static_cast<int64_t>(k) * p.qpstr + g * G * D + 4 * threadIdx.x;
    v1[k] = pk ? ldg_f4(p.qpart + static_cast<int64_t>(b) * p.qrow + o) : z;
    v2[k] = pk && p.dual ? ldg_f4(p.qpart + static_cast<int64_t>(p.qmp + b) * p.qrow + o) : z;
    // (every consumer thread: those without Q columns may append K / V)
    const bool sk = p.qpart != nullptr && warp < kConsumerWarps && k < p.qparts;
    ss1[k] = sk ? p.qss[k * 2 * p.qmp + b] : 0.f;
    ss2[k] = sk ? p.qss[k * 2 * p.qmp + p.qmp + b] : 0.f;
  }

  if (split == 0 && g == 0 && threadIdx.x == 0) flag_len(p, b);
  const int L = len_b >= 0 ? clamp_len(p, len_b) : attended_len(p, b);
  const int npages = (L + kPage - 1) / kPage;
  const int pg0 = split * p.chunk_pages;
  const int pg1 = min(npages, pg0 + p.chunk_pages);
  if (pg0 >= pg1) {
    // no page in this split; split 0 owns the zero output of an empty sequence
    if (split == 0) write_zero_rows<__nv_bfloat16, D>(p, b, g, threadIdx.x, blockDim.x);
    return;
  }
  const int ntiles = pg1 - pg0;

  // Partials mode: the CTA whose pages include this step's position writes
  // its K / V rows into the cache (page append_pg, relative to pg0).
  int append_pg = -1;
  if (p.qpart != nullptr && p.seqlens[b] >= 1 && p.seqlens[b] - 1 < L) {
    const int pg = (p.seqlens[b] - 1) / kPage;
    if (pg >= pg0 && pg < pg1) append_pg = pg - pg0;
  }
  if (threadIdx.x == 0) {
    for (int i = 0; i < STAGES; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], kConsumerWarps);
    }
    mbar_init(kv_ready, 1);
    fence_barrier_init();
  }
  __syncthreads();

  // ------------------------------------------------------------ producer warp
  if (warp == kConsumerWarps) {
    if (lane == 0) {
      prefetch_tensormap(&tmK);
      prefetch_tensormap(&tmV);
      const uint64_t policy = l2_policy_evict_first();
      const int32_t* tbl = p.block_table + static_cast<int64_t>(b) * p.max_blocks_per_seq;
      int issued = 0;
      for (int i = 0; i < ntiles; ++i) {
        const int st = i % STAGES;
        if (i >= STAGES && !mbar_wait(&empty[st], ((i / STAGES) - 1) & 1)) {
          set_err(p.err, DF_DEVERR_TIMEOUT);
          break;
        }
        const int page = tbl[pg0 + i];
        if (page < 0 || page >= p.num_blocks) {
          set_err(p.err, DF_DEVERR_BLOCK);
          stage_valid[st] = 0;
          mbar_arrive(&full[st]);
          ++issued;
          continue;
        }
        // this step's K / V row lands in this page first (partials mode)
        if (i == append_pg && !mbar_wait(kv_ready, 0)) set_err(p.err, DF_DEVERR_TIMEOUT);
        stage_valid[st] = 1;
        mbar_arrive_expect_tx(&full[st], kStageBytes);
        const int row = (page * p.Hkv + g) * kPage;
        uint8_t* sK = smem + st * kStageBytes;
        uint8_t* sV = sK + kTileBytes;
#pragma unroll
        for (int h = 0; h < D / 64; ++h) {
          tma_load_2d_hint(sK + h * kPage * 128, &tmK, &full[st], h * 64, row, policy);
          tma_load_2d_hint(sV + h * kPage * 128, &tmV, &full[st], h * 64, row, policy);
        }
        ++issued;
      }
      // Do not leave the CTA with copies in flight: wait (bounded) for the last
      // issued pages, whose completion the consumers may not have observed.
      for (int i = issued > STAGES ? issued - STAGES : 0; i < issued; ++i)
        mbar_wait(&full[i % STAGES], (i / STAGES) & 1);
    }
    return;
  }

  // ------------------------------------------------------------ consumer warps
  const int gid = lane >> 2, tq = lane & 3;

  if (p.qpart != nullptr) {
    // Partials mode prologue: this KV head's Q1 / Q2raw rows into shared
    // memory (their loads were issued at the start), and (the CTA holding
    // this step's page) its K / V row into the cache, while the producer
    // already streams the other pages. Thread ct owns 4 consecutive Q
    // columns of both rows and, for ct < D / 2, 4 of the 2 D K / V columns.
    const int ct = threadIdx.x;  // 0 .. 127
    const bool has_kv = append_pg >= 0 && 4 * ct < 2 * D;
    const float* pr1 = p.qpart + static_cast<int64_t>(b) * p.qrow;
    const int kvi = 4 * ct, kvsel = kvi >= D ? 1 : 0, kvd = kvi - kvsel * D;
    const int kvcol = (kvsel ? p.qvcol : p.qkcol) + g * D + kvd;
    float4 vk[kMaxParts];
#pragma unroll
    for (int k = 0; k < kMaxParts; ++k)
      vk[k] = has_kv && k < p.qparts ? ldg_f4(pr1 + k * p.qpstr + kvcol)
                                     : make_float4(0.f, 0.f, 0.f, 0.f);
    float s1 = 0.f, s2 = 0.f;
    float4 a1 = make_float4(0.f, 0.f, 0.f, 0.f), a2 = a1, ak = a1;
#pragma unroll
    for (int k = 0; k < kMaxParts; ++k) {
      if (k < p.qparts) {
        s1 += ss1[k];
        s2 += ss2[k];
        a1 = f4_add(a1, v1[k]);
        a2 = f4_add(a2, v2[k]);
        ak = f4_add(ak, vk[k]);
      }
    }
    const float r1 = 1.0f / sqrtf(s1 / static_cast<float>(p.qd) + p.qeps);
    const float r2 = 1.0f / sqrtf(s2 / static_cast<float>(p.qd) + p.qeps);
    if (has_q) {
      store_bf16x4(q1s + 4 * ct, f4_scale(a1, r1));
      store_bf16x4(q2s + 4 * ct, f4_scale(a2, r2));
    }
    if (append_pg >= 0) {
      const int pos = p.seqlens[b] - 1;
      const int page = p.block_table[static_cast<int64_t>(b) * p.max_blocks_per_seq + pos / kPage];
      if (page < 0 || page >= p.num_blocks) {
        if (ct == 0) set_err(p.err, DF_DEVERR_BLOCK);
      } else if (has_kv) {
        const int64_t row = (static_cast<int64_t>(page) * p.Hkv + g) * kPage + pos % kPage;
        __nv_bfloat16* cache =
            static_cast<__nv_bfloat16*>(const_cast<void*>(kvsel ? p.v_cache : p.k_cache));
        store_bf16x4(cache + row * D + kvd, f4_scale(ak, r1));
      }
      asm volatile("fence.proxy.async.global;" ::: "memory");  // -> the page's TMA load
    }
    asm volatile("bar.sync 1, %0;" ::"n"(kConsumerWarps * 32) : "memory");
    if (ct == 0 && append_pg >= 0) {
      __threadfence();
      mbar_arrive(kv_ready);
    }
  }

  // Q fragments (A operand of Q K^T): rows gid and gid + 8 of the 16-row tile.
  uint32_t qa[KS][4];
  {
    // (q1 / q2: this KV head's G rows, in shared memory in partials mode)
    const bool own = p.qpart != nullptr;
    const __nv_bfloat16* q1 =
        own ? q1s : static_cast<const __nv_bfloat16*>(p.q1) + b * p.q_stride_b + g * G * D;
    const __nv_bfloat16* q2 =
        own ? q2s : static_cast<const __nv_bfloat16*>(p.q2raw) + b * p.q_stride_b + g * G * D;
    const __nv_bfloat16* av = static_cast<const __nv_bfloat16*>(p.a);
    const int j = gid & 3;
    const bool aux = gid >= 4;
    const bool valid = (j < G) && (!aux || p.dual);
    const int h = g * G + j;
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) {
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        const int d0 = ks * 16 + half * 8 + 2 * tq;
        __nv_bfloat16 lo_row[2], hi_row[2];  // rows gid (hi part) and gid + 8 (lo part)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          __nv_bfloat16 top = __float2bfloat16_rn(0.f), bot = __float2bfloat16_rn(0.f);
          if (valid) {
            const __nv_bfloat16 x1 = q1[j * D + d0 + e];
            if (!aux) {
              top = x1;
            } else {
              float q = __bfloat162float(q2[j * D + d0 + e]);
              if (av != nullptr) q = fmaf(__bfloat162float(av[h * D + d0 + e]), __bfloat162float(x1), q);
              split_bf16(q, top, bot);
            }
          }
          hi_row[e] = top;
          lo_row[e] = bot;
        }
        qa[ks][half * 2 + 0] = pack_bf16x2(hi_row[0], hi_row[1]);
        qa[ks][half * 2 + 1] = pack_bf16x2(lo_row[0], lo_row[1]);
      }
    }
  }

  float acc[NT][4];
#pragma unroll
  for (int n = 0; n < NT; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.f;
  float m_run = kNegInf, l_run = 0.f;
  const int tok0 = warp * 16;
  bool timed_out = false;

  for (int i = 0; i < ntiles; ++i) {
    const int st = i % STAGES;
    if (!mbar_wait_warp(&full[st], (i / STAGES) & 1)) {
      timed_out = true;
      break;
    }
    bool zeroed = false;
    const int nvalid = L - (pg0 + i) * kPage - tok0;  // valid tokens among this warp's 16
    if (stage_valid[st] && nvalid > 0) {
      const uint32_t kb = smem_u32(smem + st * kStageBytes);
      const uint32_t vb = kb + kTileBytes;

      // S = Q K^T for the warp's 16 tokens (two n-tiles of 8).
      float sc[2][4];
#pragma unroll
      for (int n = 0; n < 2; ++n) sc[n][0] = sc[n][1] = sc[n][2] = sc[n][3] = 0.f;
      {
        const int mi = lane >> 3, r = lane & 7;
        const int tok = tok0 + (mi >> 1) * 8 + r;
#pragma unroll
        for (int ks = 0; ks < KS; ++ks) {
          uint32_t b0, b1, b2, b3;
          ldsm_x4(swz(kb, tok, 2 * ks + (mi & 1)), b0, b1, b2, b3);
          mma_bf16_16816(sc[0], qa[ks][0], qa[ks][1], qa[ks][2], qa[ks][3], b0, b1);
          mma_bf16_16816(sc[1], qa[ks][0], qa[ks][1], qa[ks][2], qa[ks][3], b2, b3);
        }
      }
      // Scores of row gid: hi rows + lo rows, scaled to log2 units, masked.
      float sv[2][2];
      float mx = kNegInf;
#pragma unroll
      for (int n = 0; n < 2; ++n)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int t = n * 8 + 2 * tq + e;
          const float v = (sc[n][e] + sc[n][e + 2]) * p.scale_log2;
          sv[n][e] = (t < nvalid) ? v : kNegInf;
          mx = max_nan(mx, sv[n][e]);
        }
      mx = max_nan(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
      mx = max_nan(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
      const float m_new = max_nan(m_run, mx);
      const float m_use = (m_new == kNegInf) ? 0.f : m_new;
      const float alpha = exp2f(m_run - m_use);
      float pv[2][2], psum = 0.f;
#pragma unroll
      for (int n = 0; n < 2; ++n)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          pv[n][e] = exp2f(sv[n][e] - m_use);
          psum += pv[n][e];
        }
      l_run = l_run * alpha + psum;
      m_run = m_new;
      if (!__all_sync(0xffffffffu, alpha == 1.f)) {
#pragma unroll
        for (int n = 0; n < NT; ++n) {
          acc[n][0] *= alpha;
          acc[n][1] *= alpha;
          acc[n][2] *= alpha;
          acc[n][3] *= alpha;
        }
      }
      // P as the A operand of P V: hi parts in row gid, lo parts in row gid + 8.
      __nv_bfloat16 ph[2][2], pl[2][2];
#pragma unroll
      for (int n = 0; n < 2; ++n)
#pragma unroll
        for (int e = 0; e < 2; ++e) split_bf16(pv[n][e], ph[n][e], pl[n][e]);
      const uint32_t pa0 = pack_bf16x2(ph[0][0], ph[0][1]);
      const uint32_t pa1 = pack_bf16x2(pl[0][0], pl[0][1]);
      const uint32_t pa2 = pack_bf16x2(ph[1][0], ph[1][1]);
      const uint32_t pa3 = pack_bf16x2(pl[1][0], pl[1][1]);

      // Rows past the sequence end hold stale bytes (possibly NaN patterns);
      // a zero weight times NaN would still be NaN, so clear those V rows.
      if (nvalid < 16) {
        uint8_t* vrow = smem + st * kStageBytes + kTileBytes;
        for (int idx = lane; idx < (16 - nvalid) * (D / 8); idx += 32) {
          const int tok = tok0 + nvalid + idx / (D / 8);
          const int ch = idx % (D / 8);
          *reinterpret_cast<uint4*>(vrow + (ch >> 3) * (kPage * 128) + tok * 128 + (ch & 7) * 16) =
              make_uint4(0u, 0u, 0u, 0u);
        }
        zeroed = true;
        __syncwarp();
      }
      {
        const int mi = lane >> 3, r = lane & 7;
        const int tok = tok0 + (mi & 1) * 8 + r;
#pragma unroll
        for (int np = 0; np < NT / 2; ++np) {
          uint32_t v0, v1, v2, v3;
          ldsm_x4_trans(swz(vb, tok, 2 * np + (mi >> 1)), v0, v1, v2, v3);
          mma_bf16_16816(acc[2 * np], pa0, pa1, pa2, pa3, v0, v1);
          mma_bf16_16816(acc[2 * np + 1], pa0, pa1, pa2, pa3, v2, v3);
        }
      }
    }
    // Release the stage to the producer. Generic-proxy writes (the zeroing)
    // must be ordered before the next asynchronous (TMA) write of the buffer.
    if (zeroed) fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[st]);
  }

  // All consumer warps are done with the ring before it is reused as scratch.
  asm volatile("bar.sync 1, %0;" ::"n"(kConsumerWarps * 32) : "memory");
  if (__any_sync(0xffffffffu, timed_out)) timed_out = true;
  __shared__ int any_timeout;
  if (threadIdx.x == 0) any_timeout = 0;
  asm volatile("bar.sync 1, %0;" ::"n"(kConsumerWarps * 32) : "memory");
  if (timed_out && lane == 0) {
    any_timeout = 1;
    set_err(p.err, DF_DEVERR_TIMEOUT);
  }
  asm volatile("bar.sync 1, %0;" ::"n"(kConsumerWarps * 32) : "memory");
  if (any_timeout) return;

  // Merge the 4 warps' (max, sum, O) per logical row through shared memory.
  float* ms = reinterpret_cast<float*>(smem);      // [4 warps][8 rows]
  float* ls = ms + kConsumerWarps * 8;             // [4][8]
  float* os = ls + kConsumerWarps * 8;             // [4][8][D]
  float l_tot = l_run + __shfl_xor_sync(0xffffffffu, l_run, 1);
  l_tot += __shfl_xor_sync(0xffffffffu, l_tot, 2);
  if (tq == 0) {
    ms[warp * 8 + gid] = m_run;
    ls[warp * 8 + gid] = l_tot;
  }
  float* orow = os + (warp * 8 + gid) * D;
#pragma unroll
  for (int n = 0; n < NT; ++n) {
    *reinterpret_cast<float2*>(orow + n * 8 + 2 * tq) =
        make_float2(acc[n][0] + acc[n][2], acc[n][1] + acc[n][3]);
  }
  asm volatile("bar.sync 1, %0;" ::"n"(kConsumerWarps * 32) : "memory");

  for (int idx = threadIdx.x; idx < 8 * D; idx += kConsumerWarps * 32) {
    const int row = idx / D, d = idx % D;
    const int flow = row >> 2, j = row & 3;
    if (j >= G || (flow == 1 && !p.dual)) continue;
    float M = kNegInf;
#pragma unroll
    for (int w = 0; w < kConsumerWarps; ++w) M = max_nan(M, ms[w * 8 + row]);
    float Ls = 0.f, O = 0.f;
#pragma unroll
    for (int w = 0; w < kConsumerWarps; ++w) {
      const float mw = ms[w * 8 + row];
      const float wt = (mw == kNegInf) ? 0.f : exp2f(mw - M);
      Ls += wt * ls[w * 8 + row];
      O += wt * os[(w * 8 + row) * D + d];
    }
    const int h = g * G + j;
    if (p.num_splits == 1) {
      const float out = safe_div(O, Ls);
      if (flow == 0 && p.write1)
        static_cast<__nv_bfloat16*>(p.o1)[b * p.o_stride_b + h * D + d] = __float2bfloat16_rn(out);
      if (flow == 1 && p.write2)
        static_cast<__nv_bfloat16*>(p.o2)[b * p.o_stride_b + h * D + d] = __float2bfloat16_rn(out);
    } else {
      const int64_t slot =
          (static_cast<int64_t>(b) * 2 * p.Hq + flow * p.Hq + h) * p.num_splits + split;
      p.part_o[slot * D + d] = O;
      if (d == 0) {
        p.part_ml[slot * 2] = M;
        p.part_ml[slot * 2 + 1] = Ls;
      }
    }
  }
  if (p.num_splits == 1) return;

  // Split combine, done by whichever split of (b, g) finishes last: every
  // split publishes its partial (fence, then one arrival on the unit's
  // counter); the last arrival rewinds the counter for the next call and
  // merges the splits in split order:
  //   O = sum_s o_s 2^(m_s - M) / sum_s l_s 2^(m_s - M),  M = max_s m_s.
  __threadfence();
  asm volatile("bar.sync 1, %0;" ::"n"(kConsumerWarps * 32) : "memory");
  __shared__ int last_arrival;
  const int nsplit = (npages + p.chunk_pages - 1) / p.chunk_pages;
  if (threadIdx.x == 0) {
    int* ctr = p.counters + b * p.Hkv + g;
    const int last = (atomicAdd(ctr, 1) == nsplit - 1);
    if (last) atomicExch(ctr, 0);
    last_arrival = last;
  }
  asm volatile("bar.sync 1, %0;" ::"n"(kConsumerWarps * 32) : "memory");
  if (!last_arrival) return;
  __threadfence();
  {
    // thread t: row t / 16, columns [(t % 16) * D / 16, +D / 16)
    constexpr int kCols = D / 16;
    constexpr int kFastMerge = 8;
    const int row = threadIdx.x >> 4, c0 = (threadIdx.x & 15) * kCols;
    const int flow = row >> 2, j = row & 3;
    if (j >= G || (flow == 1 && !p.dual)) return;
    const int h = g * G + j;
    const int64_t slot0 = (static_cast<int64_t>(b) * 2 * p.Hq + flow * p.Hq + h) * p.num_splits;
    float M = kNegInf, Ls = 0.f, o[kCols];
#pragma unroll
    for (int c = 0; c < kCols; ++c) o[c] = 0.f;
    auto accumulate = [&](float ms2, float ls2, const float4* v) {
      const float wt = (ms2 == kNegInf) ? 0.f : exp2f(ms2 - M);
      Ls += wt * ls2;
#pragma unroll
      for (int c = 0; c < kCols / 4; ++c) {
        o[4 * c + 0] += wt * v[c].x;
        o[4 * c + 1] += wt * v[c].y;
        o[4 * c + 2] += wt * v[c].z;
        o[4 * c + 3] += wt * v[c].w;
      }
    };
    if (nsplit <= kFastMerge) {
      // every load issued before the first use: one L2 round trip
      float mv[kFastMerge], lv[kFastMerge];
      float4 ov[kFastMerge][kCols / 4];
#pragma unroll
      for (int s2 = 0; s2 < kFastMerge; ++s2) {
        if (s2 >= nsplit) break;
        const float2 ml = __ldcg(reinterpret_cast<const float2*>(p.part_ml + (slot0 + s2) * 2));
        mv[s2] = ml.x;
        lv[s2] = ml.y;
        const float4* src = reinterpret_cast<const float4*>(p.part_o + (slot0 + s2) * D + c0);
#pragma unroll
        for (int c = 0; c < kCols / 4; ++c) ov[s2][c] = __ldcg(src + c);
      }
#pragma unroll
      for (int s2 = 0; s2 < kFastMerge; ++s2)
        if (s2 < nsplit) M = max_nan(M, mv[s2]);
#pragma unroll
      for (int s2 = 0; s2 < kFastMerge; ++s2)
        if (s2 < nsplit) accumulate(mv[s2], lv[s2], ov[s2]);
    } else {
      for (int s2 = 0; s2 < nsplit; ++s2) M = max_nan(M, __ldcg(p.part_ml + (slot0 + s2) * 2));
      for (int s2 = 0; s2 < nsplit; ++s2) {
        const float2 ml = __ldcg(reinterpret_cast<const float2*>(p.part_ml + (slot0 + s2) * 2));
        float4 v[kCols / 4];
        const float4* src = reinterpret_cast<const float4*>(p.part_o + (slot0 + s2) * D + c0);
#pragma unroll
        for (int c = 0; c < kCols / 4; ++c) v[c] = __ldcg(src + c);
        accumulate(ml.x, ml.y, v);
      }
    }
    __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(flow == 0 ? (p.write1 ? p.o1 : nullptr)
                                                               : (p.write2 ? p.o2 : nullptr));
    if (dst == nullptr) return;
    uint32_t* out = reinterpret_cast<uint32_t*>(dst + b * p.o_stride_b + h * D + c0);
#pragma unroll
    for (int c = 0; c < kCols / 2; ++c)
      out[c] = pack_bf16x2(__float2bfloat16_rn(safe_div(o[2 * c], Ls)),
                           __float2bfloat16_rn(safe_div(o[2 * c + 1], Ls)));
  }
}

// ------------------------------------------------------------------ fp32 split
// Plain CUDA-core kernel for fp32 inputs (exact fp32 arithmetic throughout).

template <int D>
__global__ void __launch_bounds__(128) split_f32_kernel(const Params p) {
  constexpr float kNegInf = -INFINITY;
  extern __shared__ float fsm[];
  float* sq = fsm;             // [8][D] query rows (primary 0..G-1, aux G..2G-1)
  float* sk = sq + 8 * D;      // [64][D]
  float* sv = sk + kPage * D;  // [64][D]
  float* sp = sv + kPage * D;  // [8][64] scores / weights
  float* sm_ = sp + 8 * kPage; // [8] running max
  float* sl = sm_ + 8;         // [8] running sum
  float* sa = sl + 8;          // [8] rescale factor

  const int split = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int t = threadIdx.x;
  pdl_wait();
  pdl_trigger();
  if (split == 0 && g == 0 && t == 0) flag_len(p, b);
  const int L = attended_len(p, b);
  const int npages = (L + kPage - 1) / kPage;
  const int pg0 = split * p.chunk_pages;
  const int pg1 = min(npages, pg0 + p.chunk_pages);
  if (pg0 >= pg1) {
    if (p.num_splits == 1) write_zero_rows<float, D>(p, b, g, t, blockDim.x);
    return;
  }
  const int G = p.G;
  const int R = p.dual ? 2 * G : G;
  const float* q1 = static_cast<const float*>(p.q1) + b * p.q_stride_b;
  const float* q2 = static_cast<const float*>(p.q2raw) + b * p.q_stride_b;
  const float* av = static_cast<const float*>(p.a);
  for (int idx = t; idx < R * D; idx += 128) {
    const int r = idx / D, d = idx % D;
    const int h = g * G + (r % G);
    const float x1 = q1[h * D + d];
    float q = x1;
    if (r >= G) {
      q = q2[h * D + d];
      if (av) q = fmaf(av[h * D + d], x1, q);
    }
    sq[r * D + d] = q;
  }
  if (t < 8) {
    sm_[t] = kNegInf;
    sl[t] = 0.f;
  }
  constexpr int kPer = 8 * D / 128;
  float o[kPer];
#pragma unroll
  for (int k = 0; k < kPer; ++k) o[k] = 0.f;

  const float* kc = static_cast<const float*>(p.k_cache);
  const float* vc = static_cast<const float*>(p.v_cache);
  const int32_t* tbl = p.block_table + static_cast<int64_t>(b) * p.max_blocks_per_seq;
  for (int pg = pg0; pg < pg1; ++pg) {
    const int page = tbl[pg];
    if (page < 0 || page >= p.num_blocks) {
      if (t == 0) set_err(p.err, DF_DEVERR_BLOCK);
      continue;
    }
    const int nval = min(kPage, L - pg * kPage);
    __syncthreads();
    const int64_t base = (static_cast<int64_t>(page) * p.Hkv + g) * kPage * D;
    for (int idx = t; idx < nval * D; idx += 128) {
      sk[idx] = kc[base + idx];
      sv[idx] = vc[base + idx];
    }
    __syncthreads();
    for (int idx = t; idx < R * nval; idx += 128) {
      const int r = idx / nval, tok = idx % nval;
      float s = 0.f;
      for (int d = 0; d < D; ++d) s = fmaf(sq[r * D + d], sk[tok * D + d], s);
      sp[r * kPage + tok] = s * p.scale_log2;
    }
    __syncthreads();
    if (t < R) {
      float mx = kNegInf;
      for (int tok = 0; tok < nval; ++tok) mx = max_nan(mx, sp[t * kPage + tok]);
      const float m_new = max_nan(sm_[t], mx);
      const float m_use = (m_new == kNegInf) ? 0.f : m_new;
      const float al = exp2f(sm_[t] - m_use);
      float sum = 0.f;
      for (int tok = 0; tok < nval; ++tok) {
        const float e = exp2f(sp[t * kPage + tok] - m_use);
        sp[t * kPage + tok] = e;
        sum += e;
      }
      sl[t] = sl[t] * al + sum;
      sm_[t] = m_new;
      sa[t] = al;
    }
    __syncthreads();
#pragma unroll
    for (int k = 0; k < kPer; ++k) {
      const int idx = t + 128 * k;
      if (idx < R * D) {
        const int r = idx / D, d = idx % D;
        float acc = o[k] * sa[r];
        for (int tok = 0; tok < nval; ++tok) acc = fmaf(sp[r * kPage + tok], sv[tok * D + d], acc);
        o[k] = acc;
      }
    }
  }
  __syncthreads();
#pragma unroll
  for (int k = 0; k < kPer; ++k) {
    const int idx = t + 128 * k;
    if (idx >= R * D) continue;
    const int r = idx / D, d = idx % D;
    const int flow = r / G, h = g * G + (r % G);
    const float M = sm_[r], Ls = sl[r];
    if (p.num_splits == 1) {
      const float out = safe_div(o[k], Ls);
      if (flow == 0 && p.write1) static_cast<float*>(p.o1)[b * p.o_stride_b + h * D + d] = out;
      if (flow == 1 && p.write2) static_cast<float*>(p.o2)[b * p.o_stride_b + h * D + d] = out;
    } else {
      const int64_t slot =
          (static_cast<int64_t>(b) * 2 * p.Hq + flow * p.Hq + h) * p.num_splits + split;
      p.part_o[slot * D + d] = o[k];
      if (d == 0) {
        p.part_ml[slot * 2] = M;
        p.part_ml[slot * 2 + 1] = Ls;
      }
    }
  }
}

// ------------------------------------------------------------------ combine
// fp32 path: O = sum_s o_s 2^(m_s - M) / sum_s l_s 2^(m_s - M), M = max_s m_s,
// in split order (deterministic), then one rounding to the output dtype.

template <typename T, int D>
__global__ void __launch_bounds__(D) combine_kernel(const Params p) {
  constexpr float kNegInf = -INFINITY;
  const int row = blockIdx.x, b = blockIdx.y, d = threadIdx.x;
  const int flow = row / p.Hq, h = row % p.Hq;
  pdl_wait();
  pdl_trigger();
  if ((flow == 0 && !p.write1) || (flow == 1 && !p.write2)) return;
  const int L = attended_len(p, b);
  const int npages = (L + kPage - 1) / kPage;
  const int nsplit = (npages + p.chunk_pages - 1) / p.chunk_pages;
  const int64_t slot0 = (static_cast<int64_t>(b) * 2 * p.Hq + row) * p.num_splits;
  float M = kNegInf;
  for (int s = 0; s < nsplit; ++s) M = max_nan(M, p.part_ml[(slot0 + s) * 2]);
  float Ls = 0.f, O = 0.f;
  for (int s = 0; s < nsplit; ++s) {
    const float ms = p.part_ml[(slot0 + s) * 2];
    const float wt = (ms == kNegInf) ? 0.f : exp2f(ms - M);
    Ls += wt * p.part_ml[(slot0 + s) * 2 + 1];
    O += wt * p.part_o[(slot0 + s) * D + d];
  }
  const float out = safe_div(O, Ls);
  T* dst = static_cast<T*>(flow == 0 ? p.o1 : p.o2);
  st_f(dst + b * p.o_stride_b + h * D + d, out);
}

// ------------------------------------------------------------------ launch

template <int D>
size_t bf16_smem_bytes() {
  // ring | barriers, stage flags (64 B) | kv_ready (64 B) | Q1, Q2raw rows of
  // one KV head (partials mode)
  return 1024 + static_cast<size_t>(kStagesBf16) * 2 * kPage * D * 2 + 128 + 2 * 4 * D * 2;
}

template <int D>
size_t f32_smem_bytes() {
  return sizeof(float) * (8 * D + 2 * kPage * D + 8 * kPage + 24);
}

// Workspace carve-up when there are splits: the bf16 arrival counters first
// (the part that must start at zero), then the partial outputs and (max, sum).
struct WsLayout {
  size_t counters, part_o, part_ml;
  size_t total() const { return counters + part_o + part_ml; }
};

inline WsLayout ws_layout(int B, int Hq, int Hkv, int D, int splits) {
  WsLayout l{0, 0, 0};
  if (splits <= 1) return l;
  const size_t rows = static_cast<size_t>(B) * 2 * Hq * splits;
  l.counters = round_up(static_cast<size_t>(B) * Hkv * sizeof(int), 256);
  l.part_o = round_up(rows * D * sizeof(float), 256);
  l.part_ml = round_up(rows * 2 * sizeof(float), 256);
  return l;
}

template <int D>
cudaError_t launch(const Params& p, int dtype, const CUtensorMap* tmK, const CUtensorMap* tmV,
                   cudaStream_t stream) {
  const dim3 grid(p.num_splits, p.Hkv, p.B);
  if (dtype == DF_BF16) {
    const size_t smem = bf16_smem_bytes<D>();
    cudaError_t e = ensure_dynamic_smem(
        reinterpret_cast<const void*>(split_bf16_kernel<D, kStagesBf16>), smem);
    if (e != cudaSuccess) return e;
    e = launch_pdl(split_bf16_kernel<D, kStagesBf16>, grid, dim3(kThreads), smem, stream, *tmK,
                   *tmV, p);
    if (e != cudaSuccess) return e;
  } else {
    const size_t smem = f32_smem_bytes<D>();
    cudaError_t e = ensure_dynamic_smem(reinterpret_cast<const void*>(split_f32_kernel<D>), smem);
    if (e != cudaSuccess) return e;
    e = launch_pdl(split_f32_kernel<D>, grid, dim3(128), smem, stream, p);
    if (e != cudaSuccess) return e;
    if (p.num_splits > 1) {
      e = launch_pdl(combine_kernel<float, D>, dim3(2 * p.Hq, p.B), dim3(D), 0, stream, p);
      if (e != cudaSuccess) return e;
    }
  }
  return cudaGetLastError();
}

}  // namespace attn
}  // namespace df

using df::attn::make_plan;
using df::attn::Plan;

extern "C" int dualflow_decode_attn_num_splits(int B, int Hkv, int max_seqlen, int block_size,
                                               int num_splits) {
  if (B < 1 || Hkv < 1 || max_seqlen < 1 || block_size < 1 || num_splits < 0) return 0;
  return make_plan(B, Hkv, max_seqlen, block_size, num_splits).splits;
}

extern "C" int dualflow_decode_attn_num_launches(int B, int Hkv, int max_seqlen, int block_size,
                                                 int num_splits, int dtype) {
  if (B < 1 || Hkv < 1 || max_seqlen < 1 || block_size < 1 || num_splits < 0) return 0;
  if (dtype == DF_BF16) return 1;  // the split combine runs inside the kernel
  if (dtype != DF_FP32) return 0;
  return make_plan(B, Hkv, max_seqlen, block_size, num_splits).splits > 1 ? 2 : 1;
}

extern "C" size_t dualflow_decode_attn_workspace_size(int B, int Hq, int Hkv, int D,
                                                      int max_seqlen, int block_size,
                                                      int num_splits) {
  if (B < 1 || Hq < 1 || Hkv < 1 || D < 1 || max_seqlen < 1 || block_size < 1 || num_splits < 0)
    return 0;
  const Plan pl = make_plan(B, Hkv, max_seqlen, block_size, num_splits);
  return df::attn::ws_layout(B, Hq, Hkv, D, pl.splits).total();
}

namespace {

// Partials-mode source of Q1 / Q2raw and this step's K / V (see Params).
struct QParts {
  const float* part;
  const float* ss;
  int parts, mp, d, kcol, vcol;
  int64_t row, pstr;
  float eps;
};

// Every entry point: every argument check first, then (only for the no-alloc
// entry point, clear_counters) the clearing of the bf16 arrival counters, then
// the launch. A call rejected by a check has issued no device work.
df_status decode_attn_impl(
    const void* q1, const void* q2raw, const void* a, int64_t q_stride_b, const void* k_cache,
    const void* v_cache, const int32_t* block_table, int max_blocks_per_seq,
    const int32_t* seqlens, int max_seqlen, void* o1, void* o2, int64_t o_stride_b, int B, int Hq,
    int Hkv, int D, int block_size, int num_blocks, float scale, int dtype, int num_splits,
    void* workspace, size_t workspace_bytes, int32_t* err_flag, void* stream,
    bool clear_counters, const QParts* qp = nullptr) {
  using namespace df;
  if ((!q1 && !qp) || !k_cache || !v_cache || !block_table || !seqlens) return DF_ERR_NULL;
  const bool want2 = (o2 != nullptr) && (q2raw != nullptr || qp != nullptr);
  if (!o1 && !want2) return DF_ERR_NULL;
  if (B < 1 || Hq < 1 || Hkv < 1 || D < 1 || num_blocks < 1 || max_blocks_per_seq < 1 ||
      max_seqlen < 1 || num_splits < 0)
    return DF_ERR_SHAPE;
  if (Hq % Hkv != 0) return DF_ERR_SHAPE;
  if (B > 65535 || Hkv > 65535) return DF_ERR_SHAPE;
  if (static_cast<int64_t>(max_seqlen) > static_cast<int64_t>(max_blocks_per_seq) * block_size)
    return DF_ERR_SHAPE;
  if (block_size != attn::kPage) return DF_ERR_UNSUPPORTED;
  if (D != 64 && D != 128) return DF_ERR_UNSUPPORTED;
  if (Hq / Hkv > 4) return DF_ERR_UNSUPPORTED;
  if (dtype != DF_FP32 && dtype != DF_BF16) return DF_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(num_blocks) * Hkv * attn::kPage >= (int64_t(1) << 31))
    return DF_ERR_UNSUPPORTED;
  const int64_t qs = q_stride_b ? q_stride_b : static_cast<int64_t>(Hq) * D;
  const int64_t os = o_stride_b ? o_stride_b : static_cast<int64_t>(Hq) * D;
  if (qs < static_cast<int64_t>(Hq) * D || os < static_cast<int64_t>(Hq) * D) return DF_ERR_SHAPE;
  const uintptr_t esize = dtype == DF_BF16 ? 2 : 4;
  const uintptr_t qa_align = dtype == DF_BF16 ? 4 : 4;
  if ((q1 && !aligned(q1, qa_align)) || (q2raw && !aligned(q2raw, qa_align)) ||
      (a && !aligned(a, qa_align)) ||
      (o1 && !aligned(o1, esize)) || (o2 && !aligned(o2, esize)))
    return DF_ERR_ALIGN;
  if (dtype == DF_BF16 && (qs % 2 != 0)) return DF_ERR_ALIGN;
  if (!aligned(k_cache, 16) || !aligned(v_cache, 16)) return DF_ERR_ALIGN;

  const Plan pl = make_plan(B, Hkv, max_seqlen, block_size, num_splits);
  attn::Params p{};
  p.q1 = q1;
  p.q2raw = want2 ? q2raw : nullptr;
  p.a = want2 ? a : nullptr;
  p.q_stride_b = qs;
  p.k_cache = k_cache;
  p.v_cache = v_cache;
  p.block_table = block_table;
  p.max_blocks_per_seq = max_blocks_per_seq;
  p.seqlens = seqlens;
  p.max_seqlen = max_seqlen;
  p.o1 = o1;
  p.o2 = want2 ? o2 : nullptr;
  p.o_stride_b = os;
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.G = Hq / Hkv;
  p.num_blocks = num_blocks;
  const float sc = scale > 0.f ? scale : 1.0f / sqrtf(static_cast<float>(D));
  p.scale_log2 = sc * 1.4426950408889634f;
  p.chunk_pages = pl.chunk_pages;
  p.num_splits = pl.splits;
  p.err = err_flag;
  p.dual = want2 ? 1 : 0;
  p.write1 = o1 ? 1 : 0;
  p.write2 = want2 ? 1 : 0;
  if (qp != nullptr) {
    if (dtype != DF_BF16) return DF_ERR_UNSUPPORTED;
    p.qpart = qp->part;
    p.qss = qp->ss;
    p.qparts = qp->parts;
    p.qmp = qp->mp;
    p.qd = qp->d;
    p.qkcol = qp->kcol;
    p.qvcol = qp->vcol;
    p.qrow = qp->row;
    p.qpstr = qp->pstr;
    p.qeps = qp->eps;
  }
  if (pl.splits > 1) {
    const attn::WsLayout l = attn::ws_layout(B, Hq, Hkv, D, pl.splits);
    if (!workspace || workspace_bytes < l.total() || !aligned(workspace, 256))
      return DF_ERR_WORKSPACE;
    uint8_t* w = static_cast<uint8_t*>(workspace);
    p.counters = reinterpret_cast<int*>(w);
    p.part_o = reinterpret_cast<float*>(w + l.counters);
    p.part_ml = reinterpret_cast<float*>(w + l.counters + l.part_o);
  }

  CUtensorMap tmK, tmV;
  if (dtype == DF_BF16) {
    const uint64_t rows = static_cast<uint64_t>(num_blocks) * Hkv * attn::kPage;
    if (!encode_tmap_bf16_2d(&tmK, k_cache, rows, D, D * 2, attn::kPage, 64) ||
        !encode_tmap_bf16_2d(&tmV, v_cache, rows, D, D * 2, attn::kPage, 64))
      return DF_ERR_CUDA;
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (clear_counters && dtype == DF_BF16 && pl.splits > 1) {
    const size_t counters = attn::ws_layout(B, Hq, Hkv, D, pl.splits).counters;
    if (cudaMemsetAsync(p.counters, 0, counters, st) != cudaSuccess) return DF_ERR_CUDA;
  }
  cudaError_t e = (D == 64) ? attn::launch<64>(p, dtype, &tmK, &tmV, st)
                            : attn::launch<128>(p, dtype, &tmK, &tmV, st);
  return e == cudaSuccess ? DF_OK : DF_ERR_CUDA;
}

}  // namespace

extern "C" df_status dualflow_decode_attn(
    const void* q1, const void* q2raw, const void* a, int64_t q_stride_b, const void* k_cache,
    const void* v_cache, const int32_t* block_table, int max_blocks_per_seq,
    const int32_t* seqlens, int max_seqlen, void* o1, void* o2, int64_t o_stride_b, int B, int Hq,
    int Hkv, int D, int block_size, int num_blocks, float scale, int dtype, int num_splits,
    void* workspace, size_t workspace_bytes, int32_t* err_flag, void* stream) {
  return decode_attn_impl(q1, q2raw, a, q_stride_b, k_cache, v_cache, block_table,
                          max_blocks_per_seq, seqlens, max_seqlen, o1, o2, o_stride_b, B, Hq, Hkv,
                          D, block_size, num_blocks, scale, dtype, num_splits, workspace,
                          workspace_bytes, err_flag, stream, false);
}

extern "C" df_status dualflow_decode_attn_qkv_partials(
    const float* part, const float* ss_part, int parts, int m_primary, int d_model, float eps,
    const void* a, const void* k_cache, const void* v_cache, const int32_t* block_table,
    int max_blocks_per_seq, const int32_t* seqlens, int max_seqlen, void* o1, void* o2,
    int64_t o_stride_b, int Hq, int Hkv, int D, int block_size, int num_blocks, float scale,
    int num_splits, void* workspace, size_t workspace_bytes, int32_t* err_flag, void* stream) {
  using namespace df;
  if (!part || !ss_part) return DF_ERR_NULL;
  if (parts < 1 || parts > attn::kMaxParts || m_primary < 1 || d_model < 1 || !(eps >= 0.f) || Hq < 1 ||
      Hkv < 1 || D < 1)
    return DF_ERR_SHAPE;
  if (!aligned(part, 16) || !aligned(ss_part, 4)) return DF_ERR_ALIGN;
  QParts qp;
  qp.part = part;
  qp.ss = ss_part;
  qp.parts = parts;
  qp.mp = m_primary;
  qp.d = d_model;
  qp.kcol = Hq * D;
  qp.vcol = (Hq + Hkv) * D;
  qp.row = static_cast<int64_t>(Hq + 2 * Hkv) * D;
  qp.pstr = 2 * static_cast<int64_t>(m_primary) * qp.row;
  qp.eps = eps;
  return decode_attn_impl(nullptr, nullptr, a, 0, k_cache, v_cache, block_table,
                          max_blocks_per_seq, seqlens, max_seqlen, o1, o2, o_stride_b, m_primary,
                          Hq, Hkv, D, block_size, num_blocks, scale, DF_BF16, num_splits,
                          workspace, workspace_bytes, err_flag, stream, false, &qp);
}

// ------------------------------------------------------------------ no-alloc variant
// Some callers cannot give this library a workspace: a serving engine that has
// handed all free device memory to its own KV-page pool before decoding
// starts, or a plain C host program with no device allocator of its own. For
// them the split partials live in a fixed array in the library's own device
// memory (allocated when the module loads, held by every GPU that loads the
// library until the process exits). Only host code needs the array's device
// address; the name itself is a host-side stand-in.

namespace df {
namespace noalloc {

static __device__ __align__(256) uint8_t g_scratch[DF_DECODE_ATTN_NOALLOC_SCRATCH_BYTES];

// The array's device address belongs to a CUDA context (the module is loaded
// into each context separately): after a device reset, or under another
// driver-API context, the same device ordinal has a different address. So
// the looked-up address is cached per context, keyed by the context's unique
// id (never reused within a process), not per device ordinal.
PFN_cuCtxGetCurrent_v4000 g_ctx_current = nullptr;
PFN_cuCtxGetId_v12000 g_ctx_id = nullptr;
std::once_flag g_fn_once;

void load_ctx_fns() {
  void* fn = nullptr;
  cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
  if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &fn, 4000, cudaEnableDefault, &q) ==
          cudaSuccess && q == cudaDriverEntryPointSuccess)
    g_ctx_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(fn);
  fn = nullptr;
  q = cudaDriverEntryPointSymbolNotFound;
  if (cudaGetDriverEntryPointByVersion("cuCtxGetId", &fn, 12000, cudaEnableDefault, &q) ==
          cudaSuccess && q == cudaDriverEntryPointSuccess)
    g_ctx_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(fn);
}

// Unique id of the calling thread's current context; 0 if there is none or
// the driver cannot say.
unsigned long long current_ctx_id() {
  std::call_once(g_fn_once, load_ctx_fns);
  if (!g_ctx_current || !g_ctx_id) return 0;
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (g_ctx_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return 0;
  if (g_ctx_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return id;
}

std::mutex g_mu;
std::vector<std::pair<unsigned long long, void*>> g_addr;  // (context id, address)

// Device address of the scratch array in the current context: looked up with
// cudaGetSymbolAddress the first time a context calls (which also loads the
// module there, so make that first call before any stream capture), then
// taken from the cache. Without a context id the lookup runs on every call.
df_status scratch_address(void** out) {
  unsigned long long id = current_ctx_id();
  if (id != 0) {
    std::lock_guard<std::mutex> lock(g_mu);
    for (const auto& e : g_addr)
      if (e.first == id) {
        *out = e.second;
        return DF_OK;
      }
  }
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_scratch) != cudaSuccess || p == nullptr) return DF_ERR_CUDA;
  if (id == 0) id = current_ctx_id();  // the lookup made the primary context current
  if (id != 0) {
    std::lock_guard<std::mutex> lock(g_mu);
    g_addr.emplace_back(id, p);
  }
  *out = p;
  return DF_OK;
}

}  // namespace noalloc
}  // namespace df

extern "C" df_status dualflow_decode_attn_noalloc(
    const void* q1, const void* q2raw, const void* a, int64_t q_stride_b, const void* k_cache,
    const void* v_cache, const int32_t* block_table, int max_blocks_per_seq,
    const int32_t* seqlens, int max_seqlen, void* o1, void* o2, int64_t o_stride_b, int B, int Hq,
    int Hkv, int D, int block_size, int num_blocks, float scale, int dtype, int num_splits,
    int32_t* err_flag, void* stream) {
  if (!q1 || !k_cache || !v_cache || !block_table || !seqlens) return DF_ERR_NULL;
  if (!o1 && !(o2 && q2raw)) return DF_ERR_NULL;
  const size_t need = dualflow_decode_attn_workspace_size(B, Hq, Hkv, D, max_seqlen, block_size,
                                                          num_splits);
  if (need > DF_DECODE_ATTN_NOALLOC_SCRATCH_BYTES) return DF_ERR_WORKSPACE;
  void* scratch = nullptr;
  if (need > 0) {
    const df_status st = df::noalloc::scratch_address(&scratch);
    if (st != DF_OK) return st;
  }
  // the counters at the start of the scratch are cleared after the argument
  // checks, just before the launch (bf16 split calls only)
  return decode_attn_impl(q1, q2raw, a, q_stride_b, k_cache, v_cache, block_table,
                          max_blocks_per_seq, seqlens, max_seqlen, o1, o2, o_stride_b, B, Hq, Hkv,
                          D, block_size, num_blocks, scale, dtype, num_splits, scratch,
                          need > 0 ? DF_DECODE_ATTN_NOALLOC_SCRATCH_BYTES : 0, err_flag, stream,
                          true);
}
