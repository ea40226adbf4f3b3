// Primary prefill: the primary flow processes a prompt chunk causally and
// writes its K/V to the persistent paged cache; the auxiliary flow is skipped
// over the prompt and switched on only at the last prompt position.
//
// Method: page "Sintesi Tecnica: Dual-Flow Transformers", section
// "Architettura Core" (the primary flow is a standard causal Transformer that
// processes the whole prompt and writes the cache; the auxiliary flow is
// omitted during prefill and activated at the last prompt position) and
// section "Costi di Inferenza vs. Addestramento" (prefill costs what a
// standard Transformer's does).
//
// One call = up to four kernels on the caller's stream, all launched with
// programmatic dependent launch:
//  1. append_kernel: token t of sequence b goes to cache position
//     ctx_lens[b] + (t - cu_seqlens[b]) (one CTA per token, 16-byte copies);
//  2. causal flash attention of the chunk's primary queries over the cache
//     (prefix + chunk): tc::pair_kernel on the tcgen05 tensor cores (D = 64
//     or 128, at least 128 token rows, 16-byte aligned output rows; described at the
//     kernel), otherwise attn_kernel: one CTA per (query head, 64-row tile,
//     sequence), heads fastest so that the CTAs sharing a KV head run side by
//     side and meet its pages in L2; tiles of one sequence are issued longest
//     first. 4 consumer warps own 16 query rows each; 1 producer warp streams
//     64-token K and V pages by TMA (128-byte swizzle) through a 3-stage
//     mbarrier ring. S = Q K^T and O += P V run on mma.sync (bf16 in, fp32
//     accumulate), online softmax in the exp2 domain per row (P rounded once
//     to bf16 for P V, fp32 row sums);
//  3. gather_last_kernel: copies each sequence's last-position primary query
//     row and writes the attended length ctx + n, the inputs of
//  4. the decode attention kernel in auxiliary-only mode: the coupled
//     auxiliary query of the last prompt position attends to the same cache
//     exactly as it does at a generated position.
#include <math.h>

#include <algorithm>

#include "common.cuh"
#include "host_util.h"
#include "umma.cuh"

extern "C" size_t dualflow_decode_attn_workspace_size(int B, int Hq, int Hkv, int D,
                                                      int max_seqlen, int block_size,
                                                      int num_splits);
extern "C" df_status dualflow_decode_attn(
    const void* q1, const void* q2raw, const void* a, int64_t q_stride_b, const void* k_cache,
    const void* v_cache, const int32_t* block_table, int max_blocks_per_seq,
    const int32_t* seqlens, int max_seqlen, void* o1, void* o2, int64_t o_stride_b, int B, int Hq,
    int Hkv, int D, int block_size, int num_blocks, float scale, int dtype, int num_splits,
    void* workspace, size_t workspace_bytes, int32_t* err_flag, void* stream);
extern "C" int dualflow_decode_attn_num_splits(int B, int Hkv, int max_seqlen, int block_size,
                                               int num_splits);

namespace df {
namespace prefill {

constexpr int kPage = 64;           // tokens per cache page (block_size)
constexpr int kRows = 64;           // query rows per CTA
constexpr int kConsumerWarps = 4;   // 16 query rows each
constexpr int kThreads = (kConsumerWarps + 1) * 32;
constexpr int kStages = 3;

// ------------------------------------------------------------------ sequence lookup

struct Chunk {
  int t0, n, ctx;  // first token row, tokens in the chunk, cached tokens before it
  bool ok;
};

// Validates the chunk of sequence b: 0 <= t0, 1 <= n <= max_q_len,
// t0 + n <= T, ctx >= 0 and ctx + n <= max_seqlen.
__device__ __forceinline__ Chunk load_chunk(const int32_t* cu, const int32_t* ctx_lens, int b,
                                            int T, int max_q_len, int max_seqlen) {
  Chunk c;
  c.t0 = cu[b];
  const int t1 = cu[b + 1];
  c.n = t1 - c.t0;
  c.ctx = ctx_lens ? ctx_lens[b] : 0;
  c.ok = c.t0 >= 0 && t1 <= T && c.n >= 1 && c.n <= max_q_len && c.ctx >= 0 &&
         static_cast<int64_t>(c.ctx) + c.n <= max_seqlen;
  return c;
}

// ------------------------------------------------------------------ 1. append

struct AppendParams {
  const uint8_t* k_new;
  const uint8_t* v_new;
  int64_t new_stride_bytes;  // between token rows
  uint8_t* k_cache;
  uint8_t* v_cache;
  const int32_t* block_table;
  int max_blocks_per_seq;
  const int32_t* cu_seqlens;
  const int32_t* ctx_lens;
  int B, T, Hkv, row_bytes, num_blocks, max_q_len, max_seqlen;
  int32_t* err;
};

__global__ void __launch_bounds__(256) append_kernel(const AppendParams p) {
  const int t = blockIdx.x;
  pdl_wait();
  pdl_trigger();
  // sequence of token t: the last b with cu_seqlens[b] <= t
  int lo = 0, hi = p.B;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (p.cu_seqlens[mid] <= t) lo = mid; else hi = mid;
  }
  const Chunk c = load_chunk(p.cu_seqlens, p.ctx_lens, lo, p.T, p.max_q_len, p.max_seqlen);
  if (!c.ok || t < c.t0 || t >= c.t0 + c.n) {
    if (threadIdx.x == 0) set_err(p.err, DF_DEVERR_SEQLEN);
    return;
  }
  const int pos = c.ctx + (t - c.t0);
  if (pos / kPage >= p.max_blocks_per_seq) {
    if (threadIdx.x == 0) set_err(p.err, DF_DEVERR_POSITION);
    return;
  }
  const int page = p.block_table[static_cast<int64_t>(lo) * p.max_blocks_per_seq + pos / kPage];
  if (page < 0 || page >= p.num_blocks) {
    if (threadIdx.x == 0) set_err(p.err, DF_DEVERR_BLOCK);
    return;
  }
  const int slot = pos % kPage;
  const int vec_per_row = p.row_bytes / 16;
  for (int v = threadIdx.x; v < p.Hkv * vec_per_row; v += blockDim.x) {
    const int g = v / vec_per_row, off = (v % vec_per_row) * 16;
    const int64_t src = static_cast<int64_t>(t) * p.new_stride_bytes +
                        static_cast<int64_t>(g) * p.row_bytes + off;
    const int64_t dst =
        ((static_cast<int64_t>(page) * p.Hkv + g) * kPage + slot) * p.row_bytes + off;
    *reinterpret_cast<uint4*>(p.k_cache + dst) = *reinterpret_cast<const uint4*>(p.k_new + src);
    *reinterpret_cast<uint4*>(p.v_cache + dst) = *reinterpret_cast<const uint4*>(p.v_new + src);
  }
}

// ------------------------------------------------------------------ 2. attention

struct AttnParams {
  const __nv_bfloat16* q1;
  int64_t q_stride_t;  // elements between token rows
  const int32_t* block_table;
  int max_blocks_per_seq;
  const int32_t* cu_seqlens;
  const int32_t* ctx_lens;
  __nv_bfloat16* o1;
  int64_t o_stride_t;
  int T, Hkv, G, num_blocks, max_q_len, max_seqlen, tiles;
  float scale_log2;  // softmax scale * log2(e)
  int32_t* err;
  int pair_rows;     // two-tile kernel: pair row tiles of one head (1) or heads (0)
};

// Byte address of 16-byte chunk `ch` of token row `tok` in a TMA-written
// [64 tokens][D] bf16 page stored as D/64 column halves of [64][128 B] with the
// 128-byte swizzle (chunk index XOR row index within each 8-row group).
__device__ __forceinline__ uint32_t swz(uint32_t base, int tok, int ch) {
  return base + (ch >> 3) * (kPage * 128) + tok * 128 + (((ch & 7) ^ (tok & 7)) << 4);
}

__device__ __forceinline__ uint32_t pack_f32_bf16x2(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);  // lo in the low half
  return *reinterpret_cast<const uint32_t*>(&v);
}

// Zero the bf16 halves of a P V operand register whose key index is >= kend:
// the register holds keys k0 (low half) and k0 + 1 (high half).
__device__ __forceinline__ uint32_t keep_keys(uint32_t v, int k0, int kend) {
  if (k0 >= kend) return 0u;
  if (k0 + 1 >= kend) return v & 0x0000ffffu;
  return v;
}

template <int D>
__global__ void __launch_bounds__(kThreads, 2)
    attn_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                const AttnParams p) {
  constexpr int kTileBytes = kPage * D * 2;  // one K (or V) page
  constexpr int kStageBytes = 2 * kTileBytes;
  constexpr int KS = D / 16;  // k-steps of Q K^T
  constexpr int NT = D / 8;   // n-tiles of P V
  constexpr float kNegInf = -INFINITY;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kStages * kStageBytes);
  uint64_t* empty = full + kStages;
  int* stage_valid = reinterpret_cast<int*>(empty + kStages);

  const int h = blockIdx.x;
  const int tile = p.tiles - 1 - static_cast<int>(blockIdx.y);  // longest tiles first
  const int b = blockIdx.z;
  const int g = h / p.G;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  pdl_wait();
  pdl_trigger();

  const Chunk c = load_chunk(p.cu_seqlens, p.ctx_lens, b, p.T, p.max_q_len, p.max_seqlen);
  if (!c.ok) {
    if (h == 0 && tile == 0 && threadIdx.x == 0) set_err(p.err, DF_DEVERR_SEQLEN);
    return;
  }
  const int i0 = tile * kRows;
  if (i0 >= c.n) return;
  const int rows = min(kRows, c.n - i0);
  const int kend = c.ctx + i0 + rows;  // keys [0, kend) serve this tile
  const int npages = (kend + kPage - 1) / kPage;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], kConsumerWarps);
    }
    fence_barrier_init();
  }
  __syncthreads();

  // ------------------------------------------------------------ producer warp
  if (warp == kConsumerWarps) {
    if (lane == 0) {
      prefetch_tensormap(&tmK);
      prefetch_tensormap(&tmV);
      const int32_t* tbl = p.block_table + static_cast<int64_t>(b) * p.max_blocks_per_seq;
      int issued = 0;
      for (int i = 0; i < npages; ++i) {
        const int st = i % kStages;
        if (i >= kStages && !mbar_wait(&empty[st], ((i / kStages) - 1) & 1)) {
          set_err(p.err, DF_DEVERR_TIMEOUT);
          break;
        }
        const int page = tbl[i];
        if (page < 0 || page >= p.num_blocks) {
          set_err(p.err, DF_DEVERR_BLOCK);
          stage_valid[st] = 0;
          mbar_arrive(&full[st]);
          ++issued;
          continue;
        }
        stage_valid[st] = 1;
        mbar_arrive_expect_tx(&full[st], kStageBytes);
        const int row = (page * p.Hkv + g) * kPage;
        uint8_t* sK = smem + st * kStageBytes;
        uint8_t* sV = sK + kTileBytes;
#pragma unroll
        for (int hf = 0; hf < D / 64; ++hf) {
          tma_load_2d(sK + hf * kPage * 128, &tmK, &full[st], hf * 64, row);
          tma_load_2d(sV + hf * kPage * 128, &tmV, &full[st], hf * 64, row);
        }
        ++issued;
      }
      // Leave no copy in flight: wait (bounded) for the last issued pages.
      for (int i = issued > kStages ? issued - kStages : 0; i < issued; ++i)
        mbar_wait(&full[i % kStages], (i / kStages) & 1);
    }
    return;
  }

  // ------------------------------------------------------------ consumer warps
  const int gid = lane >> 2, tq = lane & 3;
  const int mi = lane >> 3, r8 = lane & 7;
  // The thread's two query rows (gid and gid + 8 of the warp's 16). A padding
  // row past the chunk end repeats the last real row (finite, never stored).
  const int r_lo = i0 + warp * 16 + gid, r_hi = r_lo + 8;
  const int pos_lo = c.ctx + min(r_lo, c.n - 1);
  const int pos_hi = c.ctx + min(r_hi, c.n - 1);
  const int w_first = c.ctx + min(i0 + warp * 16, c.n - 1);     // smallest row position
  const int w_last = c.ctx + min(i0 + warp * 16 + 15, c.n - 1);  // largest row position
  const int w_pages = w_last / kPage + 1;                        // pages the warp needs

  // Q fragments (A operand of Q K^T).
  uint32_t qa[KS][4];
  {
    const __nv_bfloat16* qlo =
        p.q1 + static_cast<int64_t>(c.t0 + min(r_lo, c.n - 1)) * p.q_stride_t + h * D;
    const __nv_bfloat16* qhi =
        p.q1 + static_cast<int64_t>(c.t0 + min(r_hi, c.n - 1)) * p.q_stride_t + h * D;
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) {
      qa[ks][0] = *reinterpret_cast<const uint32_t*>(qlo + ks * 16 + 2 * tq);
      qa[ks][1] = *reinterpret_cast<const uint32_t*>(qhi + ks * 16 + 2 * tq);
      qa[ks][2] = *reinterpret_cast<const uint32_t*>(qlo + ks * 16 + 8 + 2 * tq);
      qa[ks][3] = *reinterpret_cast<const uint32_t*>(qhi + ks * 16 + 8 + 2 * tq);
    }
  }

  float acc[NT][4];
#pragma unroll
  for (int n = 0; n < NT; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.f;
  float m_lo = kNegInf, m_hi = kNegInf, l_lo = 0.f, l_hi = 0.f;
  bool timed_out = false;

  for (int i = 0; i < npages; ++i) {
    const int st = i % kStages;
    if (!mbar_wait_warp(&full[st], (i / kStages) & 1)) {
      timed_out = true;
      break;
    }
    if (i < w_pages && stage_valid[st]) {
      const uint32_t kb = smem_u32(smem + st * kStageBytes);
      const uint32_t vb = kb + kTileBytes;
      const int kbase = i * kPage;
      const bool v_tail = kbase + kPage > kend;
      const int kend_rel = kend - kbase;

      // The page in two halves of 32 keys (fewer live registers); a half that
      // lies wholly past the warp's last row is skipped.
#pragma unroll
      for (int hk = 0; hk < 2; ++hk) {
        const int hbase = kbase + hk * 32;
        if (hbase > w_last) break;

        // S = Q K^T: 16 rows x 32 keys (4 n-tiles of 8 keys).
        float sc[4][4];
#pragma unroll
        for (int n = 0; n < 4; ++n) sc[n][0] = sc[n][1] = sc[n][2] = sc[n][3] = 0.f;
#pragma unroll
        for (int ks = 0; ks < KS; ++ks) {
#pragma unroll
          for (int kg = 0; kg < 2; ++kg) {
            uint32_t b0, b1, b2, b3;
            ldsm_x4(swz(kb, hk * 32 + kg * 16 + (mi >> 1) * 8 + r8, 2 * ks + (mi & 1)), b0, b1,
                    b2, b3);
            mma_bf16_16816(sc[2 * kg], qa[ks][0], qa[ks][1], qa[ks][2], qa[ks][3], b0, b1);
            mma_bf16_16816(sc[2 * kg + 1], qa[ks][0], qa[ks][1], qa[ks][2], qa[ks][3], b2, b3);
          }
        }

        // Causal mask (key j visible to the row at position pos iff j <= pos),
        // needed only where the half reaches past the warp's first row.
        if (hbase + 31 > w_first) {
#pragma unroll
          for (int n = 0; n < 4; ++n)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              const int j = hbase + n * 8 + 2 * tq + e;
              if (j > pos_lo) sc[n][e] = kNegInf;
              if (j > pos_hi) sc[n][e + 2] = kNegInf;
            }
        }
        // Row maxima of the raw scores as a tree (scale > 0 keeps the order).
        // fmaxf skips a NaN score, but the NaN still reaches the output
        // through its weight exp2(NaN) and the sums.
        float mx_lo = fmaxf(fmaxf(fmaxf(sc[0][0], sc[0][1]), fmaxf(sc[1][0], sc[1][1])),
                            fmaxf(fmaxf(sc[2][0], sc[2][1]), fmaxf(sc[3][0], sc[3][1])));
        float mx_hi = fmaxf(fmaxf(fmaxf(sc[0][2], sc[0][3]), fmaxf(sc[1][2], sc[1][3])),
                            fmaxf(fmaxf(sc[2][2], sc[2][3]), fmaxf(sc[3][2], sc[3][3])));
        mx_lo = fmaxf(mx_lo, __shfl_xor_sync(0xffffffffu, mx_lo, 1));
        mx_hi = fmaxf(mx_hi, __shfl_xor_sync(0xffffffffu, mx_hi, 1));
        mx_lo = fmaxf(mx_lo, __shfl_xor_sync(0xffffffffu, mx_lo, 2));
        mx_hi = fmaxf(mx_hi, __shfl_xor_sync(0xffffffffu, mx_hi, 2));
        // running maxima in log2 units
        const float mn_lo = fmaxf(m_lo, mx_lo * p.scale_log2);
        const float mn_hi = fmaxf(m_hi, mx_hi * p.scale_log2);
        const float mu_lo = (mn_lo == kNegInf) ? 0.f : mn_lo;
        const float mu_hi = (mn_hi == kNegInf) ? 0.f : mn_hi;
        const float al_lo = exp2f(m_lo - mu_lo), al_hi = exp2f(m_hi - mu_hi);
        m_lo = mn_lo;
        m_hi = mn_hi;

        // P = 2^(s * scale_log2 - m) in bf16 as the A operand of P V (k-step
        // ks = keys 16 ks .. 16 ks + 15 of the half); fp32 row sums.
        uint32_t pa[2][4];
        float ps_lo = 0.f, ps_hi = 0.f;
#pragma unroll
        for (int ks = 0; ks < 2; ++ks)
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            const int n = 2 * ks + half;
            const float p0 = exp2f(fmaf(sc[n][0], p.scale_log2, -mu_lo));
            const float p1 = exp2f(fmaf(sc[n][1], p.scale_log2, -mu_lo));
            const float p2 = exp2f(fmaf(sc[n][2], p.scale_log2, -mu_hi));
            const float p3 = exp2f(fmaf(sc[n][3], p.scale_log2, -mu_hi));
            ps_lo += p0 + p1;
            ps_hi += p2 + p3;
            pa[ks][2 * half + 0] = pack_f32_bf16x2(p0, p1);
            pa[ks][2 * half + 1] = pack_f32_bf16x2(p2, p3);
          }
        l_lo = fmaf(l_lo, al_lo, ps_lo);
        l_hi = fmaf(l_hi, al_hi, ps_hi);
        if (!__all_sync(0xffffffffu, al_lo == 1.f && al_hi == 1.f)) {
#pragma unroll
          for (int n = 0; n < NT; ++n) {
            acc[n][0] *= al_lo;
            acc[n][1] *= al_lo;
            acc[n][2] *= al_hi;
            acc[n][3] *= al_hi;
          }
        }

        // O += P V. Keys at or past kend hold other tokens' bytes (possibly
        // NaN patterns); their weights are 0, and their V halves are zeroed
        // too, as 0 * NaN would still be NaN.
#pragma unroll
        for (int ks = 0; ks < 2; ++ks) {
#pragma unroll
          for (int np = 0; np < NT / 2; ++np) {
            uint32_t v0, v1, v2, v3;
            ldsm_x4_trans(swz(vb, hk * 32 + ks * 16 + (mi & 1) * 8 + r8, 2 * np + (mi >> 1)), v0,
                          v1, v2, v3);
            if (v_tail) {
              const int k0 = hk * 32 + ks * 16 + 2 * tq;
              v0 = keep_keys(v0, k0, kend_rel);
              v2 = keep_keys(v2, k0, kend_rel);
              v1 = keep_keys(v1, k0 + 8, kend_rel);
              v3 = keep_keys(v3, k0 + 8, kend_rel);
            }
            mma_bf16_16816(acc[2 * np], pa[ks][0], pa[ks][1], pa[ks][2], pa[ks][3], v0, v1);
            mma_bf16_16816(acc[2 * np + 1], pa[ks][0], pa[ks][1], pa[ks][2], pa[ks][3], v2, v3);
          }
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[st]);
  }

  if (timed_out) {
    if (lane == 0) set_err(p.err, DF_DEVERR_TIMEOUT);
    return;
  }

  // Normalise and store the warp's rows (each warp owns whole rows: no merge).
  l_lo += __shfl_xor_sync(0xffffffffu, l_lo, 1);
  l_lo += __shfl_xor_sync(0xffffffffu, l_lo, 2);
  l_hi += __shfl_xor_sync(0xffffffffu, l_hi, 1);
  l_hi += __shfl_xor_sync(0xffffffffu, l_hi, 2);
  if (r_lo < c.n) {
    uint32_t* o = reinterpret_cast<uint32_t*>(
        p.o1 + static_cast<int64_t>(c.t0 + r_lo) * p.o_stride_t + h * D + 2 * tq);
#pragma unroll
    for (int n = 0; n < NT; ++n) o[n * 4] = pack_f32_bf16x2(acc[n][0] / l_lo, acc[n][1] / l_lo);
  }
  if (r_hi < c.n) {
    uint32_t* o = reinterpret_cast<uint32_t*>(
        p.o1 + static_cast<int64_t>(c.t0 + r_hi) * p.o_stride_t + h * D + 2 * tq);
#pragma unroll
    for (int n = 0; n < NT; ++n) o[n * 4] = pack_f32_bf16x2(acc[n][2] / l_hi, acc[n][3] / l_hi);
  }
}


// ------------------------------------------------------------------ 2'. attention, tcgen05
//
// The same computation on the 5th-generation tensor cores, for D = 64 or 128, over
// key blocks of 128 tokens (two cache pages): S = Q K^T (M 128, N 128) into
// TMEM, the softmax warps write P as bf16 into TMEM, and O += P V takes P
// from TMEM as its A operand. pair_kernel (described at its definition) holds
// two 128-row tiles per CTA, the tensor core alternating between them: two
// query heads of a KV group over one row tile when the group has an even
// number of heads, else two consecutive row tiles of one head. The
// reference max m of a row changes (and O is rescaled in TMEM) only when the
// row's max exceeds it by more than 2^8, so P stays <= 256 and O is rarely
// touched. After the last block: O / l from TMEM to bf16 rows.
namespace tc {

constexpr int kRows = 128;          // query rows per CTA (= TMEM lanes)
constexpr float kRescaleLog2 = 8.f; // keep a stale reference max up to 2^8 below

// Store 32 consecutive fp32 TMEM columns of this thread's lane and wait.
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, "
      "%29, %30, %31, %32};" ::"r"(taddr),
      "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
      "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
      "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
      "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
      "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
      "r"(__float_as_uint(v[15])), "r"(__float_as_uint(v[16])), "r"(__float_as_uint(v[17])),
      "r"(__float_as_uint(v[18])), "r"(__float_as_uint(v[19])), "r"(__float_as_uint(v[20])),
      "r"(__float_as_uint(v[21])), "r"(__float_as_uint(v[22])), "r"(__float_as_uint(v[23])),
      "r"(__float_as_uint(v[24])), "r"(__float_as_uint(v[25])), "r"(__float_as_uint(v[26])),
      "r"(__float_as_uint(v[27])), "r"(__float_as_uint(v[28])), "r"(__float_as_uint(v[29])),
      "r"(__float_as_uint(v[30])), "r"(__float_as_uint(v[31]))
      : "memory");
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// 2^x by the SFU's approximate base-2 exponential (relative error near
// 2^-22, far below the bf16 rounding of P; results under 2^-126 flush to 0,
// which only drops weights below 2^-126 of the row's largest).
__device__ __forceinline__ float exp2_sfu(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// ------------------------------------------------------------------ two tiles per CTA
// The same computation for two 128-row query tiles of one KV group, over key
// blocks of 128 tokens (two cache pages): either two query heads h0 = 2x,
// h1 = 2x + 1 over one row tile (pair_rows = 0, the group has an even number
// of heads) or one head over row tiles 2y and 2y + 1 (pair_rows = 1). Both
// tiles read the same K/V blocks (one load serves 256 query rows), and the
// tensor core alternates between them: it computes one tile's P V and next S
// while the other tile's softmax warps work. With row pairs the two tiles see
// different causal ends; the CTA loads K/V up to the later one, tile 0 stops
// at its own end, and a tile past the chunk (an odd tile count) does nothing.
//  * S_t = Q_t K_j^T: M 128, N 128 (both pages of block j), K 128, both
//    operands in shared memory, into tile t's 128-column TMEM region;
//  * P_t, bf16 with two keys per 32-bit column, overwrites the first 64
//    columns of that region, and O_t += P_t V_j reads P from TMEM (the A
//    operand) and V from shared memory (MN-major, N 128 = all of D): P never
//    passes through shared memory, and no MMA step reads more than 8 KB of
//    it for its 128 x 128 x 16 multiply-adds;
//  * per block j and tile t the MMA warp issues P V, then S of block j + 1
//    into the same region: the MMAs of one thread run in issue order, so
//    S_{j+1} overwrites P_j only after P_j V_j has read it, and the commit
//    after S_{j+1} also tells the softmax warps that O_t holds P_j V_j (a
//    rescale of O may then follow, and the next P may be written).
// Warp 0: TMA producer (both Q tiles once; K blocks through a 2-stage ring,
// V blocks through a 3-stage ring: a K block is released once both tiles'
// S are computed, long before its V block); warp 1: MMA issuer; warps 2-5 /
// 6-9: softmax of tile 0 / 1, one thread per query row. TMEM: S and P of
// tile t at columns [128 t, 128 t + 128), O of tile t at [256 + 128 t, ...).

constexpr int kPairThreads = 320;
constexpr uint32_t kPairTmemCols = 512;
constexpr int kBlk = 2 * kPage;       // keys per block
constexpr int kKStages = 2;           // K block ring depth
constexpr int kVStages = 3;           // V block ring depth
constexpr uint32_t kPairOCol = 256;   // first TMEM column of O (tile 0)

template <int D>
struct PairLayout {
  static constexpr int kQBytes = kRows * D * 2;   // one tile's Q: [D/64][128 rows][128 B]
  static constexpr int kBlkBytes = kBlk * D * 2;  // one K or V block: [D/64][128 keys][128 B]
  static constexpr int kHalf = kBlk * 128;        // bytes between a block's 64-column halves
  static constexpr int kOffK = 2 * kQBytes;
  static constexpr int kOffV = kOffK + kKStages * kBlkBytes;
  static constexpr int kOffBar = kOffV + kVStages * kBlkBytes;
  static constexpr int kNumBars = 1 + 2 * kKStages + 2 * kVStages + 3 * 2 + 1;
  static constexpr size_t kSmem = 1024 + kOffBar + kNumBars * 8 + 16;
};

// Descriptor of an MN-major bf16 operand with 128-byte swizzle, two swizzle
// atoms (128 elements) wide along N: 8-row groups along K 1024 bytes apart
// (stride byte offset), the second 64-element atom along N `atom_stride`
// bytes after the first (leading byte offset).
__device__ __forceinline__ uint64_t smem_desc_mn(uint32_t addr, uint32_t atom_stride) {
  return static_cast<uint64_t>((addr >> 4) & 0x3FFFu) |
         (static_cast<uint64_t>((atom_stride >> 4) & 0x3FFFu) << 16) |
         (static_cast<uint64_t>(1024 >> 4) << 32) | (static_cast<uint64_t>(1) << 46) |
         (static_cast<uint64_t>(2) << 61);
}

// D (TMEM) (+)= A B with A in TMEM (K-major: lane = row, two bf16 of
// consecutive k per 32-bit column) and B in shared memory (descriptor db).
__device__ __forceinline__ void umma_bf16_ts(uint32_t tmem_d, uint32_t tmem_a, uint64_t db,
                                             uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(tmem_d),
      "r"(tmem_a), "l"(db), "r"(idesc), "r"(accumulate)
      : "memory");
}

// 64 consecutive 32-bit TMEM columns of this thread's lane, waited for in the
// same statement (the registers are defined once the wait has returned).
__device__ __forceinline__ void tmem_ld64_wait(uint32_t taddr, uint32_t (&r)[64]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x64.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "
      "%28, %29, %30, %31, %32, %33, %34, %35, %36, %37, %38, %39, %40, %41, %42, %43, %44, "
      "%45, %46, %47, %48, %49, %50, %51, %52, %53, %54, %55, %56, %57, %58, %59, %60, %61, "
      "%62, %63}, [%64];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
        "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
        "=r"(r[31]), "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]),
        "=r"(r[37]), "=r"(r[38]), "=r"(r[39]), "=r"(r[40]), "=r"(r[41]), "=r"(r[42]),
        "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]), "=r"(r[48]),
        "=r"(r[49]), "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]),
        "=r"(r[55]), "=r"(r[56]), "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]),
        "=r"(r[61]), "=r"(r[62]), "=r"(r[63])
      : "r"(taddr)
      : "memory");
}

// 16 consecutive 32-bit TMEM columns of this thread's lane (no wait).
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
      "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]),
      "r"(v[15])
      : "memory");
}

__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// Packed fp32 pairs (sm_100): one instruction computes both lanes, which
// halves the softmax warps' issue slots for the scale and the row sums.
__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void f2_unpack(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t f2_mul(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

// 2^x of a pair on the FMA pipe, for part of the weights (the SFU
// exponential alone cannot keep up with the tensor core): x = j + f with j
// the nearest integer (adding and subtracting 1.5 * 2^23 leaves it in the
// low mantissa bits of t), 2^f for |f| <= 1/2 by a degree-3 polynomial with
// p(0) = 1 whose coefficients minimise the maximum relative error on
// [-1/2, 1/2] (fitted offline by iteratively reweighted least squares: max
// relative error 1.02e-4, far below P's bf16 rounding), times 2^j built in
// the exponent field. x is raised to -127 first, where 2^j = 0 (a masked
// key's weight is exactly 0); NaN stays NaN; the weights here never exceed
// 2^8.
constexpr float kExp2C1 = 0.6932829022407532f;
constexpr float kExp2C2 = 0.2422107756137848f;
constexpr float kExp2C3 = 0.055008821189403534f;

__device__ __forceinline__ uint64_t exp2_poly2(uint64_t x2) {
  float xa, xb;
  f2_unpack(x2, xa, xb);
  xa = xa < -127.f ? -127.f : xa;
  xb = xb < -127.f ? -127.f : xb;
  const uint64_t x = f2_pack(xa, xb);
  const uint64_t t = f2_add(x, f2_pack(12582912.f, 12582912.f));
  const uint64_t j = f2_add(t, f2_pack(-12582912.f, -12582912.f));
  const uint64_t f = f2_fma(j, f2_pack(-1.f, -1.f), x);
  uint64_t p = f2_fma(f2_pack(kExp2C3, kExp2C3), f, f2_pack(kExp2C2, kExp2C2));
  p = f2_fma(p, f, f2_pack(kExp2C1, kExp2C1));
  p = f2_fma(p, f, f2_pack(1.f, 1.f));
  float ta, tb;
  f2_unpack(t, ta, tb);
  // the low bits of t hold j: (t's bits << 23) is j << 23 modulo 2^32
  const float sa = __int_as_float((__float_as_int(ta) << 23) + 0x3F800000);
  const float sb = __int_as_float((__float_as_int(tb) << 23) + 0x3F800000);
  return f2_mul(p, f2_pack(sa, sb));
}

// Which key pairs of a 32-key chunk take the polynomial (the rest the SFU).
constexpr int kPolyPeriod = 3;  // one pair in kPolyPeriod (5 of 16: measured best)
__device__ __forceinline__ constexpr bool poly_pair(int k) {
  return kPolyPeriod > 0 && (k % kPolyPeriod) == kPolyPeriod - 1;
}

// Three-input maximum (sm_100; NaN inputs are ignored as by fmaxf).
__device__ __forceinline__ float max3f(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

template <int D>
__global__ void __launch_bounds__(kPairThreads, 1)
    pair_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                const __grid_constant__ CUtensorMap tmV, const AttnParams p) {
  using Lay = PairLayout<D>;
  constexpr int H = D / 64;
  constexpr float kNegInf = -INFINITY;
  static_assert(D == 64 || D == 128, "the two-tile prefill kernel is built for head_dim 64 / 128");
  static_assert(PairLayout<D>::kSmem <= 227 * 1024, "shared memory budget");

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Lay::kOffBar);
  uint64_t* q_full = bars;
  uint64_t* k_full = q_full + 1;          // [kKStages] K block landed
  uint64_t* k_empty = k_full + kKStages;  // [kKStages] both tiles' S have read it
  uint64_t* v_full = k_empty + kKStages;  // [kVStages]
  uint64_t* v_empty = v_full + kVStages;  // [kVStages] both tiles' P V have read it
  uint64_t* s_full = v_empty + kVStages;  // [tile] S_j in TMEM (and every earlier MMA done)
  uint64_t* p_full = s_full + 2;          // [tile] P_j in TMEM (4 softmax warps)
  uint64_t* pv_done = p_full + 2;         // [tile] O += P_j V_j completed
  uint64_t* mma_done = pv_done + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);

  // The CTA's two tiles: two heads of one KV group over the same row tile
  // (p.pair_rows = 0), or two consecutive row tiles of one head (1), which
  // share every key block of the first; longest work first.
  int hd[2], i0s[2];
  if (p.pair_rows) {
    const int pr = (p.tiles + 1) / 2 - 1 - static_cast<int>(blockIdx.y);
    hd[0] = hd[1] = static_cast<int>(blockIdx.x);
    i0s[0] = 2 * pr * kRows;
    i0s[1] = i0s[0] + kRows;
  } else {
    hd[0] = 2 * static_cast<int>(blockIdx.x);
    hd[1] = hd[0] + 1;
    i0s[0] = i0s[1] = (p.tiles - 1 - static_cast<int>(blockIdx.y)) * kRows;
  }
  const int b = blockIdx.z;
  const int g = hd[0] / p.G;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  pdl_wait();
  pdl_trigger();

  const Chunk c = load_chunk(p.cu_seqlens, p.ctx_lens, b, p.T, p.max_q_len, p.max_seqlen);
  if (!c.ok) {
    if (hd[0] == 0 && i0s[0] == 0 && threadIdx.x == 0) set_err(p.err, DF_DEVERR_SEQLEN);
    return;
  }
  if (i0s[0] >= c.n) return;  // before any barrier or TMEM allocation
  // per tile: rows, keys [0, kend) it attends to, its key blocks (0 = no tile)
  int rows_t[2], kend_t[2], nb_t[2];
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    rows_t[t] = i0s[t] < c.n ? min(kRows, c.n - i0s[t]) : 0;
    kend_t[t] = c.ctx + i0s[t] + rows_t[t];
    nb_t[t] = rows_t[t] > 0 ? ((kend_t[t] + kPage - 1) / kPage + 1) / 2 : 0;
  }
  const int kend = max(kend_t[0], rows_t[1] > 0 ? kend_t[1] : 0);  // keys of the CTA
  const int npages = (kend + kPage - 1) / kPage;
  const int nblk = (npages + 1) / 2;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < kKStages; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&k_empty[i], 1);
    }
    for (int i = 0; i < kVStages; ++i) {
      mbar_init(&v_full[i], 1);
      mbar_init(&v_empty[i], 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&s_full[t], 1);
      mbar_init(&p_full[t], 4);
      mbar_init(&pv_done[t], 1);
    }
    mbar_init(mma_done, 1);
    fence_barrier_init();
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"(kPairTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  umma::tc_fence_before();
  __syncthreads();
  umma::tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    if (lane == 0) {
      prefetch_tensormap(&tmQ);
      prefetch_tensormap(&tmK);
      prefetch_tensormap(&tmV);
      mbar_arrive_expect_tx(q_full, (rows_t[1] > 0 ? 2 : 1) * Lay::kQBytes);
#pragma unroll
      for (int t = 0; t < 2; ++t)
        if (rows_t[t] > 0) {
#pragma unroll
          for (int hf = 0; hf < H; ++hf)
            tma_load_2d(smem + t * Lay::kQBytes + hf * (kRows * 128), &tmQ, q_full,
                        hd[t] * D + hf * 64, c.t0 + i0s[t]);
        }
      const int32_t* tbl = p.block_table + static_cast<int64_t>(b) * p.max_blocks_per_seq;
      // One block = pages 2j and (if the key range reaches it) 2j + 1; a
      // missing second page leaves its rows stale: their keys are masked and
      // their V rows cleared by the softmax warps.
      auto load_block = [&](const CUtensorMap* tm, uint64_t* bar, uint8_t* dst, int j) {
        const int np = min(2, npages - 2 * j);
        mbar_arrive_expect_tx(bar, static_cast<uint32_t>(np * H * kPage * 128));
        for (int q = 0; q < np; ++q) {
          int page = tbl[2 * j + q];
          if (page < 0 || page >= p.num_blocks) {  // flagged; page 0 stands in (outputs invalid)
            set_err(p.err, DF_DEVERR_BLOCK);
            page = 0;
          }
          const int row = (page * p.Hkv + g) * kPage;
#pragma unroll
          for (int hf = 0; hf < H; ++hf)
            tma_load_2d(dst + hf * Lay::kHalf + q * (kPage * 128), tm, bar, hf * 64, row);
        }
      };
      int kissued = 0, vissued = 0;
      for (int j = 0; j < nblk; ++j) {
        const int sk = j % kKStages, sv = j % kVStages;
        if (j >= kKStages && !mbar_wait(&k_empty[sk], ((j / kKStages) - 1) & 1)) {
          set_err(p.err, DF_DEVERR_TIMEOUT);
          break;
        }
        load_block(&tmK, &k_full[sk], smem + Lay::kOffK + sk * Lay::kBlkBytes, j);
        ++kissued;
        if (j >= kVStages && !mbar_wait(&v_empty[sv], ((j / kVStages) - 1) & 1)) {
          set_err(p.err, DF_DEVERR_TIMEOUT);
          break;
        }
        load_block(&tmV, &v_full[sv], smem + Lay::kOffV + sv * Lay::kBlkBytes, j);
        ++vissued;
      }
      // Leave no copy in flight (bounded waits).
      mbar_wait(q_full, 0);
      for (int j = kissued > kKStages ? kissued - kKStages : 0; j < kissued; ++j)
        mbar_wait(&k_full[j % kKStages], (j / kKStages) & 1);
      for (int j = vissued > kVStages ? vissued - kVStages : 0; j < vissued; ++j)
        mbar_wait(&v_full[j % kVStages], (j / kVStages) & 1);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t kIdS = umma::make_idesc(kRows, kBlk);          // Q K^T, N 128
      constexpr uint32_t kIdPV = umma::make_idesc(kRows, D) | (1u << 16);  // P V, V MN-major
      bool ok = mbar_wait(q_full, 0);
      // Descriptors are affine in the byte address (its bits 4..17 sit in the
      // low field): each one below is a base plus a constant.
      const uint64_t dq0 = umma::smem_desc(smem_u32(smem));
      const uint64_t dk0 = umma::smem_desc(smem_u32(smem + Lay::kOffK));
      const uint64_t dv0 = smem_desc_mn(smem_u32(smem + Lay::kOffV), Lay::kHalf);
      // S_j of tile t into its TMEM region (the block's first user waits for it)
      auto issue_s = [&](int t, int j) -> bool {
        const int st = j % kKStages;
        if ((t == 0 || j >= nb_t[0]) && !mbar_wait(&k_full[st], (j / kKStages) & 1)) return false;
        umma::tc_fence_after();
        const uint64_t dq = dq0 + static_cast<uint64_t>((t * Lay::kQBytes) >> 4);
        const uint64_t dk = dk0 + static_cast<uint64_t>((st * Lay::kBlkBytes) >> 4);
        const uint32_t d_tmem = tmem + t * kBlk;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const int hf = kk >> 2, kq = kk & 3;
          umma::umma_bf16(d_tmem, dq + ((hf * (kRows * 128) + kq * 32) >> 4),
                          dk + ((hf * Lay::kHalf + kq * 32) >> 4), kIdS, kk > 0 ? 1u : 0u);
        }
        umma::umma_commit(&s_full[t]);
        return true;
      };
      // O_t += P_j V_j once tile t's softmax has written P_j
      auto issue_pv = [&](int t, int j) -> bool {
        const int st = j % kVStages;
        if (!mbar_wait(&p_full[t], j & 1)) return false;
        if ((t == 0 || j >= nb_t[0]) && !mbar_wait(&v_full[st], (j / kVStages) & 1)) return false;
        umma::tc_fence_after();
        const uint64_t dv = dv0 + static_cast<uint64_t>((st * Lay::kBlkBytes) >> 4);
        const uint32_t a_tmem = tmem + t * kBlk;
        const uint32_t d_tmem = tmem + kPairOCol + t * D;
#pragma unroll
        for (int kk = 0; kk < kBlk / 16; ++kk)
          umma_bf16_ts(d_tmem, a_tmem + kk * 8, dv + ((kk * 16 * 128) >> 4), kIdPV,
                       (j > 0 || kk > 0) ? 1u : 0u);
        umma::umma_commit(&pv_done[t]);
        return true;
      };
      // a block's K (V) stage is released after the S (P V) of every tile
      // that reads it
      if (ok) ok = issue_s(0, 0) && (nb_t[1] == 0 || issue_s(1, 0));
      if (ok) umma::umma_commit(&k_empty[0]);
      for (int j = 0; ok && j < nblk; ++j) {
#pragma unroll
        for (int t = 0; t < 2; ++t) {
          if (ok && j < nb_t[t] && !issue_pv(t, j)) ok = false;
          if (ok && j + 1 < nb_t[t] && !issue_s(t, j + 1)) ok = false;
        }
        if (ok) {
          umma::umma_commit(&v_empty[j % kVStages]);
          if (j + 1 < nblk) umma::umma_commit(&k_empty[(j + 1) % kKStages]);
        }
      }
      if (!ok) set_err(p.err, DF_DEVERR_TIMEOUT);
      umma::umma_commit(mma_done);  // completes when every MMA issued above has
      mbar_wait(mma_done, 0);
    }
  } else {
    // ---------------------------------------------------------------- softmax warps
    const int t = warp >= 6 ? 1 : 0;  // the tile this warp serves
    const int quarter = warp & 3;     // this warp may access TMEM lanes 32 quarter .. + 31
    const int r = quarter * 32 + lane;
    const int i0 = i0s[t], rows = rows_t[t], tnb = nb_t[t];
    const int pos = c.ctx + min(i0 + r, c.n - 1);  // a padding row repeats the last real row
    const uint32_t t_lane = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    const uint32_t t_s = t_lane + t * kBlk;             // S / P of this tile
    const uint32_t t_o = t_lane + kPairOCol + t * D;    // O of this tile
    float m_ref = kNegInf, l = 0.f;
    bool ok = true;
    for (int j = 0; j < tnb; ++j) {
      const int kbase = j * kBlk;
      // S_j landed; every earlier MMA of this CTA (P_{j-1} V_{j-1} included)
      // has completed with it.
      if (!mbar_wait_warp(&s_full[t], j & 1)) {
        ok = false;
        break;
      }
      umma::tc_fence_after();
      float s[kBlk];
      {
        uint32_t rr[64];
        tmem_ld64_wait(t_s, rr);
#pragma unroll
        for (int k = 0; k < 64; ++k) s[k] = __uint_as_float(rr[k]);
        tmem_ld64_wait(t_s + 64, rr);
#pragma unroll
        for (int k = 0; k < 64; ++k) s[64 + k] = __uint_as_float(rr[k]);
      }
      if (kbase + kBlk - 1 > pos) {  // causal mask (and keys past the chunk end)
#pragma unroll
        for (int k = 0; k < kBlk; ++k)
          if (kbase + k > pos) s[k] = kNegInf;
      }
      // row max: 8 chains of three-input maxima, then their maximum
      float mx[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) mx[q] = s[q];
#pragma unroll
      for (int k = 8; k < kBlk; k += 16) {
#pragma unroll
        for (int q = 0; q < 8; ++q) mx[q] = max3f(mx[q], s[k + q], s[k + 8 + q]);
      }
      const float m_cand =
          fmaxf(max3f(mx[0], mx[1], mx[2]), max3f(max3f(mx[3], mx[4], mx[5]), mx[6], mx[7])) *
          p.scale_log2;
      // The reference max moves (and O and l are rescaled) only when the
      // block's max exceeds it by more than 2^kRescaleLog2.
      const bool rescale = (m_ref != kNegInf) && (m_cand > m_ref + kRescaleLog2);
      float alpha = 1.f;
      if (m_ref == kNegInf) {
        m_ref = m_cand;  // first block: O holds nothing yet
      } else if (rescale) {
        alpha = exp2f(m_ref - m_cand);
        m_ref = m_cand;
      }
      const float mu = (m_ref == kNegInf) ? 0.f : m_ref;

      // P_j = 2^(s scale_log2 - mu) as bf16 pairs over the first 64 columns
      // of the S region (this thread's lane); fp32 row sum of the weights.
      const uint64_t c2 = f2_pack(p.scale_log2, p.scale_log2);
      const uint64_t nmu2 = f2_pack(-mu, -mu);
      uint64_t sum2[4] = {0ull, 0ull, 0ull, 0ull};  // 8 partial sums (+0.0f pairs)
#pragma unroll
      for (int q = 0; q < kBlk / 32; ++q) {
        uint32_t w[16];
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          const uint64_t x2 = f2_fma(f2_pack(s[32 * q + 2 * k], s[32 * q + 2 * k + 1]), c2, nmu2);
          uint64_t e2;
          if (poly_pair(k)) {
            e2 = exp2_poly2(x2);
          } else {
            float xa, xb;
            f2_unpack(x2, xa, xb);
            e2 = f2_pack(exp2_sfu(xa), exp2_sfu(xb));
          }
          sum2[k & 3] = f2_add(sum2[k & 3], e2);
          float a, bb;
          f2_unpack(e2, a, bb);
          w[k] = pack_f32_bf16x2(a, bb);
        }
        tmem_st16(t_s + 16 * q, w);
      }
      float sum[2];
      {
        float e[8];
#pragma unroll
        for (int i = 0; i < 4; ++i) f2_unpack(sum2[i], e[2 * i], e[2 * i + 1]);
        sum[0] = (e[0] + e[1]) + (e[2] + e[3]);
        sum[1] = (e[4] + e[5]) + (e[6] + e[7]);
      }
      if (__any_sync(0xffffffffu, rescale)) {
        // O holds P_{j-1} V_{j-1} (see the wait above): rescale it in place
        // (alpha = 1 on the rows that keep their reference).
#pragma unroll
        for (int cc = 0; cc < D; cc += 32) {
          float o[32];
          umma::tmem_ld<32>(t_o + cc, o);
#pragma unroll
          for (int k = 0; k < 32; ++k) o[k] *= alpha;
          tmem_st32(t_o + cc, o);
        }
      }
      tmem_wait_st();
      l = fmaf(l, alpha, sum[0] + sum[1]);

      // Keys at or past the CTA's kend in its last block hold other tokens'
      // bytes (or stale rows where the block has one page): their weights
      // are 0, and their V rows are zeroed, as 0 * NaN would still be NaN in
      // the accumulator. Every tile that reads that block clears the same
      // rows (the same zero bytes) before its own P is published. (Keys a
      // first row tile masks inside the CTA's range are its partner's
      // tokens: zero weights on finite values.)
      if (kbase + kBlk > kend) {
        const int sv = j % kVStages;
        if (!mbar_wait_warp(&v_full[sv], (j / kVStages) & 1)) {  // the block has landed
          ok = false;
          break;
        }
        const int kend_rel = kend - kbase;
        uint8_t* sV = smem + Lay::kOffV + sv * Lay::kBlkBytes;
        const int nvec = (kBlk - kend_rel) * H * 8;  // 16-byte chunks to clear
        for (int v = r; v < nvec; v += kRows) {
          const int row = kend_rel + v / (H * 8), hf = (v / 8) % H, ch = v % 8;
          *reinterpret_cast<uint4*>(sV + hf * Lay::kHalf + row * 128 + ch * 16) =
              make_uint4(0u, 0u, 0u, 0u);
        }
        fence_proxy_async_smem();  // cleared V rows -> the tensor core's proxy
      }
      umma::tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[t]);
    }
    if (ok && tnb > 0) ok = mbar_wait_warp(&pv_done[t], (tnb - 1) & 1);
    if (tnb == 0) {
      // no tile here (a last row tile past the chunk): nothing to store
    } else if (ok) {
      umma::tc_fence_after();
      __nv_bfloat16* orow = p.o1 + static_cast<int64_t>(c.t0 + i0 + min(r, rows - 1)) * p.o_stride_t +
                            hd[t] * D;
#pragma unroll
      for (int cc = 0; cc < D; cc += 32) {
        float o[32];
        umma::tmem_ld<32>(t_o + cc, o);
#pragma unroll
        for (int k = 0; k < 32; ++k) o[k] = o[k] / l;
        if (r < rows) umma::store_bf16<32>(orow + cc, o);
      }
    } else if (lane == 0) {
      set_err(p.err, DF_DEVERR_TIMEOUT);
    }
  }

  umma::tc_fence_before();
  __syncthreads();
  umma::tc_fence_after();
  if (warp == 1) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(kPairTmemCols)
                 : "memory");
  }
}

}  // namespace tc

// ------------------------------------------------------------------ 3. last-row gather

struct GatherParams {
  const uint8_t* q1;
  int64_t q_stride_bytes;  // between token rows
  const int32_t* cu_seqlens;
  const int32_t* ctx_lens;
  int T, max_q_len, max_seqlen, row_bytes;  // row_bytes = Hq * D * 2
  uint8_t* q_last;               // [B][Hq][D]
  int32_t* seqlens;              // [B]: ctx + n (0 for an invalid chunk)
};

__global__ void __launch_bounds__(256) gather_last_kernel(const GatherParams p) {
  const int b = blockIdx.x;
  pdl_wait();
  pdl_trigger();
  const Chunk c = load_chunk(p.cu_seqlens, p.ctx_lens, b, p.T, p.max_q_len, p.max_seqlen);
  // An invalid chunk gets length 0: the decode kernel then flags it and
  // writes a zero auxiliary output.
  if (threadIdx.x == 0) p.seqlens[b] = c.ok ? c.ctx + c.n : 0;
  if (!c.ok) return;
  const uint8_t* src = p.q1 + static_cast<int64_t>(c.t0 + c.n - 1) * p.q_stride_bytes;
  uint8_t* dst = p.q_last + static_cast<int64_t>(b) * p.row_bytes;
  for (int v = threadIdx.x; v < p.row_bytes / 16; v += blockDim.x)
    reinterpret_cast<uint4*>(dst)[v] = reinterpret_cast<const uint4*>(src)[v];
}

// ------------------------------------------------------------------ host

template <int D>
size_t attn_smem_bytes() {
  return 1024 + static_cast<size_t>(kStages) * 2 * kPage * D * 2 + 2 * kStages * 8 +
         kStages * 4 + 64;
}

template <int D>
cudaError_t launch_attn(const AttnParams& p, int Hq, int B, const CUtensorMap* tmK,
                        const CUtensorMap* tmV, cudaStream_t stream) {
  const size_t smem = attn_smem_bytes<D>();
  cudaError_t e = ensure_dynamic_smem(reinterpret_cast<const void*>(attn_kernel<D>), smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(attn_kernel<D>, dim3(Hq, p.tiles, B), dim3(kThreads), smem, stream, *tmK, *tmV,
                    p);
}

// Two query heads of one KV group per CTA when the group has an even number
// of heads (both tiles then read the same pages), else one head per CTA.
template <int D>
cudaError_t launch_pair(AttnParams p, int Hq, int B, const CUtensorMap* tmQ,
                        const CUtensorMap* tmK, const CUtensorMap* tmV, cudaStream_t stream) {
  constexpr size_t smem2 = tc::PairLayout<D>::kSmem;
  cudaError_t e2 = ensure_dynamic_smem(reinterpret_cast<const void*>(tc::pair_kernel<D>), smem2);
  if (e2 != cudaSuccess) return e2;
  // two query heads of a KV group per CTA when the group has an even number
  // of heads, else two consecutive row tiles of one head
  p.pair_rows = p.G % 2 == 0 ? 0 : 1;
  const dim3 grid = p.pair_rows ? dim3(Hq, (p.tiles + 1) / 2, B) : dim3(Hq / 2, p.tiles, B);
  return launch_pdl(tc::pair_kernel<D>, grid, dim3(tc::kPairThreads), smem2, stream, *tmQ, *tmK,
                    *tmV, p);
}

cudaError_t launch_attn_tc(AttnParams p, int Hq, int B, int D, const CUtensorMap* tmQ,
                           const CUtensorMap* tmK, const CUtensorMap* tmV, cudaStream_t stream) {
  return D == 64 ? launch_pair<64>(p, Hq, B, tmQ, tmK, tmV, stream)
                 : launch_pair<128>(p, Hq, B, tmQ, tmK, tmV, stream);
}

// Workspace of the auxiliary step: the decode workspace (its arrival counters
// first), then the gathered last-position queries, then the attended lengths.
struct WsLayout {
  size_t decode, q_last, seqlens;
  size_t total() const { return decode + q_last + seqlens; }
};

inline WsLayout ws_layout(int B, int Hq, int Hkv, int D, int max_seqlen) {
  WsLayout l;
  l.decode = round_up(dualflow_decode_attn_workspace_size(B, Hq, Hkv, D, max_seqlen, kPage, 0), 256);
  l.q_last = round_up(static_cast<size_t>(B) * Hq * D * 2, 256);
  l.seqlens = round_up(static_cast<size_t>(B) * 4, 256);
  return l;
}

}  // namespace prefill
}  // namespace df

extern "C" size_t dualflow_prefill_workspace_size(int B, int Hq, int Hkv, int D, int max_seqlen,
                                                  int block_size) {
  if (B < 1 || Hq < 1 || Hkv < 1 || D < 1 || max_seqlen < 1 || block_size != df::prefill::kPage)
    return 0;
  return df::prefill::ws_layout(B, Hq, Hkv, D, max_seqlen).total();
}

extern "C" int dualflow_prefill_num_launches(int with_append, int with_aux) {
  return (with_append ? 1 : 0) + 1 + (with_aux ? 2 : 0);
}

// The tcgen05 attention kernel serves D = 64 and 128 with at least one full
// tile of token rows and 16-byte aligned output rows; anything else takes the
// mma.sync kernel.
static bool tc_kernel_fits(int D, int T, const void* o1, int64_t o_stride_t) {
  return (D == 64 || D == 128) && T >= df::prefill::tc::kRows && df::aligned(o1, 16) &&
         o_stride_t % 8 == 0;
}

extern "C" int dualflow_prefill_kernel(int D, int T, const void* o1, int64_t o_stride_t, int Hq) {
  const int64_t os = o_stride_t ? o_stride_t : static_cast<int64_t>(Hq) * D;
  return tc_kernel_fits(D, T, o1, os) ? DF_PREFILL_KERNEL_TCGEN05 : DF_PREFILL_KERNEL_MMA_SYNC;
}

extern "C" df_status dualflow_prefill_ex(
    const void* q1, int64_t q_stride_t, const void* k_new, const void* v_new, int64_t kv_stride_t,
    const void* q2raw, const void* a, void* k_cache, void* v_cache, const int32_t* block_table,
    int max_blocks_per_seq, const int32_t* cu_seqlens, const int32_t* ctx_lens, int max_q_len,
    int max_seqlen, void* o1, int64_t o_stride_t, void* o2, int B, int T, int Hq, int Hkv, int D,
    int block_size, int num_blocks, float scale, int dtype, int kernel, void* workspace,
    size_t workspace_bytes, int32_t* err_flag, void* stream) {
  using namespace df;
  using namespace df::prefill;
  if (!q1 || !k_cache || !v_cache || !block_table || !cu_seqlens || !o1) return DF_ERR_NULL;
  if ((k_new == nullptr) != (v_new == nullptr)) return DF_ERR_NULL;
  const bool aux = (q2raw != nullptr) && (o2 != nullptr);
  if (B < 1 || T < B || Hq < 1 || Hkv < 1 || D < 1 || num_blocks < 1 || max_blocks_per_seq < 1 ||
      max_q_len < 1 || max_q_len > T || max_seqlen < max_q_len)
    return DF_ERR_SHAPE;
  if (Hq % Hkv != 0) return DF_ERR_SHAPE;
  if (static_cast<int64_t>(max_seqlen) > static_cast<int64_t>(max_blocks_per_seq) * block_size)
    return DF_ERR_SHAPE;
  const int tiles = static_cast<int>(ceil_div(max_q_len, kRows));
  if (B > 65535 || tiles > 65535 || Hq > 65535) return DF_ERR_SHAPE;
  if (dtype != DF_BF16) return DF_ERR_UNSUPPORTED;
  if (block_size != kPage || (D != 64 && D != 128)) return DF_ERR_UNSUPPORTED;
  if (aux && Hq / Hkv > 4) return DF_ERR_UNSUPPORTED;  // the decode kernel's head grouping
  if (static_cast<int64_t>(num_blocks) * Hkv * kPage >= (int64_t(1) << 31)) return DF_ERR_UNSUPPORTED;
  const int64_t qs = q_stride_t ? q_stride_t : static_cast<int64_t>(Hq) * D;
  const int64_t os = o_stride_t ? o_stride_t : static_cast<int64_t>(Hq) * D;
  const int64_t ks = kv_stride_t ? kv_stride_t : static_cast<int64_t>(Hkv) * D;
  if (qs < static_cast<int64_t>(Hq) * D || os < static_cast<int64_t>(Hq) * D ||
      ks < static_cast<int64_t>(Hkv) * D)
    return DF_ERR_SHAPE;
  if (!aligned(q1, 16) || (qs * 2) % 16 != 0 || !aligned(o1, 4) || os % 2 != 0)
    return DF_ERR_ALIGN;
  if (k_new && (!aligned(k_new, 16) || !aligned(v_new, 16) || (ks * 2) % 16 != 0))
    return DF_ERR_ALIGN;
  if (!aligned(k_cache, 16) || !aligned(v_cache, 16)) return DF_ERR_ALIGN;
  if (aux && (!aligned(q2raw, 4) || (a && !aligned(a, 4)) || !aligned(o2, 4))) return DF_ERR_ALIGN;
  if (kernel < DF_PREFILL_KERNEL_AUTO || kernel > DF_PREFILL_KERNEL_TCGEN05) return DF_ERR_SHAPE;
  const bool tc_fits = tc_kernel_fits(D, T, o1, os);
  if (kernel == DF_PREFILL_KERNEL_TCGEN05 && !tc_fits) return DF_ERR_UNSUPPORTED;
  const bool use_tc = kernel == DF_PREFILL_KERNEL_TCGEN05 ||
                      (kernel == DF_PREFILL_KERNEL_AUTO && tc_fits);
  WsLayout wl{};
  if (aux) {
    wl = ws_layout(B, Hq, Hkv, D, max_seqlen);
    if (!workspace || workspace_bytes < wl.total() || !aligned(workspace, 256))
      return DF_ERR_WORKSPACE;
  }

  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // 1. the chunk's K/V rows into the cache
  if (k_new) {
    AppendParams ap;
    ap.k_new = static_cast<const uint8_t*>(k_new);
    ap.v_new = static_cast<const uint8_t*>(v_new);
    ap.new_stride_bytes = ks * 2;
    ap.k_cache = static_cast<uint8_t*>(k_cache);
    ap.v_cache = static_cast<uint8_t*>(v_cache);
    ap.block_table = block_table;
    ap.max_blocks_per_seq = max_blocks_per_seq;
    ap.cu_seqlens = cu_seqlens;
    ap.ctx_lens = ctx_lens;
    ap.B = B;
    ap.T = T;
    ap.Hkv = Hkv;
    ap.row_bytes = D * 2;
    ap.num_blocks = num_blocks;
    ap.max_q_len = max_q_len;
    ap.max_seqlen = max_seqlen;
    ap.err = err_flag;
    const int nvec = Hkv * D * 2 / 16;
    const int threads = nvec >= 256 ? 256 : ((nvec + 31) / 32) * 32;
    if (launch_pdl(append_kernel, dim3(T), dim3(threads), 0, st, ap) != cudaSuccess)
      return DF_ERR_CUDA;
  }

  // 2. causal attention of the primary queries
  CUtensorMap tmK, tmV;
  const uint64_t rows = static_cast<uint64_t>(num_blocks) * Hkv * kPage;
  if (!encode_tmap_bf16_2d(&tmK, k_cache, rows, D, D * 2, kPage, 64) ||
      !encode_tmap_bf16_2d(&tmV, v_cache, rows, D, D * 2, kPage, 64))
    return DF_ERR_CUDA;
  AttnParams p{};
  p.q1 = static_cast<const __nv_bfloat16*>(q1);
  p.q_stride_t = qs;
  p.block_table = block_table;
  p.max_blocks_per_seq = max_blocks_per_seq;
  p.cu_seqlens = cu_seqlens;
  p.ctx_lens = ctx_lens;
  p.o1 = static_cast<__nv_bfloat16*>(o1);
  p.o_stride_t = os;
  p.T = T;
  p.Hkv = Hkv;
  p.G = Hq / Hkv;
  p.num_blocks = num_blocks;
  p.max_q_len = max_q_len;
  p.max_seqlen = max_seqlen;
  p.tiles = use_tc ? static_cast<int>(ceil_div(max_q_len, tc::kRows)) : tiles;
  const float sc = scale > 0.f ? scale : 1.0f / sqrtf(static_cast<float>(D));
  p.scale_log2 = sc * 1.4426950408889634f;
  p.err = err_flag;
  cudaError_t e;
  if (use_tc) {
    CUtensorMap tmQ;  // token rows x (Hq * D) columns; boxes of 128 rows x 64 columns
    if (!encode_tmap_bf16_2d(&tmQ, q1, static_cast<uint64_t>(T), static_cast<uint64_t>(Hq) * D,
                             static_cast<uint64_t>(qs) * 2, tc::kRows, 64))
      return DF_ERR_CUDA;
    e = launch_attn_tc(p, Hq, B, D, &tmQ, &tmK, &tmV, st);
  } else {
    e = (D == 64) ? launch_attn<64>(p, Hq, B, &tmK, &tmV, st)
                  : launch_attn<128>(p, Hq, B, &tmK, &tmV, st);
  }
  if (e != cudaSuccess) return DF_ERR_CUDA;
  if (!aux) return DF_OK;

  // 3. + 4. the auxiliary query of the last prompt position
  uint8_t* w = static_cast<uint8_t*>(workspace);
  GatherParams gp;
  gp.q1 = static_cast<const uint8_t*>(q1);
  gp.q_stride_bytes = qs * 2;
  gp.cu_seqlens = cu_seqlens;
  gp.ctx_lens = ctx_lens;
  gp.T = T;
  gp.max_q_len = max_q_len;
  gp.max_seqlen = max_seqlen;
  gp.row_bytes = Hq * D * 2;
  gp.q_last = w + wl.decode;
  gp.seqlens = reinterpret_cast<int32_t*>(w + wl.decode + wl.q_last);
  if (launch_pdl(gather_last_kernel, dim3(B), dim3(256), 0, st, gp) != cudaSuccess)
    return DF_ERR_CUDA;
  // Split count of the auxiliary step. The decode plan aims at about two
  // waves of split CTAs, rounded up, which serves ragged batches; when every
  // attended length is known equal (no prefix lengths and T = B max_q_len:
  // every chunk is max_q_len tokens), one wave of the decode kernel's 2 CTAs
  // per SM is faster (16 x 8 units of 4097 tokens: 52.8 against 69.6 us),
  // never more splits than the plan (the workspace is sized for it).
  int aux_splits = 0;
  if (ctx_lens == nullptr && static_cast<int64_t>(B) * max_q_len == T) {
    constexpr int kDecodeSlots = 148 * 2;  // the decode kernel's resident CTAs on a B200
    const int units = B * Hkv;
    const int plan = dualflow_decode_attn_num_splits(B, Hkv, max_seqlen, block_size, 0);
    if (units < kDecodeSlots && plan > 1) aux_splits = std::max(1, std::min(plan, kDecodeSlots / units));
  }
  return dualflow_decode_attn(gp.q_last, q2raw, a, 0, k_cache, v_cache, block_table,
                              max_blocks_per_seq, gp.seqlens, max_seqlen, nullptr, o2, 0, B, Hq,
                              Hkv, D, block_size, num_blocks, sc, DF_BF16, aux_splits,
                              wl.decode ? workspace : nullptr, wl.decode, err_flag, stream);
}

extern "C" df_status dualflow_prefill(
    const void* q1, int64_t q_stride_t, const void* k_new, const void* v_new, int64_t kv_stride_t,
    const void* q2raw, const void* a, void* k_cache, void* v_cache, const int32_t* block_table,
    int max_blocks_per_seq, const int32_t* cu_seqlens, const int32_t* ctx_lens, int max_q_len,
    int max_seqlen, void* o1, int64_t o_stride_t, void* o2, int B, int T, int Hq, int Hkv, int D,
    int block_size, int num_blocks, float scale, int dtype, void* workspace,
    size_t workspace_bytes, int32_t* err_flag, void* stream) {
  return dualflow_prefill_ex(q1, q_stride_t, k_new, v_new, kv_stride_t, q2raw, a, k_cache, v_cache,
                             block_table, max_blocks_per_seq, cu_seqlens, ctx_lens, max_q_len,
                             max_seqlen, o1, o_stride_t, o2, B, T, Hq, Hkv, D, block_size,
                             num_blocks, scale, dtype, DF_PREFILL_KERNEL_AUTO, workspace,
                             workspace_bytes, err_flag, stream);
}
