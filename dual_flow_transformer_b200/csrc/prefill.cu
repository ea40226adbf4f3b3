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
//  2. attn_kernel: causal flash attention of the chunk's primary queries over
//     the cache (prefix + chunk). One CTA per (query head, 64-row tile,
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

#include "common.cuh"
#include "host_util.h"

extern "C" size_t dualflow_decode_attn_workspace_size(int B, int Hq, int Hkv, int D,
                                                      int max_seqlen, int block_size,
                                                      int num_splits);
extern "C" df_status dualflow_decode_attn(
    const void* q1, const void* q2raw, const void* a, int64_t q_stride_b, const void* k_cache,
    const void* v_cache, const int32_t* block_table, int max_blocks_per_seq,
    const int32_t* seqlens, int max_seqlen, void* o1, void* o2, int64_t o_stride_b, int B, int Hq,
    int Hkv, int D, int block_size, int num_blocks, float scale, int dtype, int num_splits,
    void* workspace, size_t workspace_bytes, int32_t* err_flag, void* stream);

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
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(attn_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  return launch_pdl(attn_kernel<D>, dim3(Hq, p.tiles, B), dim3(kThreads), smem, stream, *tmK, *tmV,
                    p);
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

extern "C" df_status dualflow_prefill(
    const void* q1, int64_t q_stride_t, const void* k_new, const void* v_new, int64_t kv_stride_t,
    const void* q2raw, const void* a, void* k_cache, void* v_cache, const int32_t* block_table,
    int max_blocks_per_seq, const int32_t* cu_seqlens, const int32_t* ctx_lens, int max_q_len,
    int max_seqlen, void* o1, int64_t o_stride_t, void* o2, int B, int T, int Hq, int Hkv, int D,
    int block_size, int num_blocks, float scale, int dtype, void* workspace,
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
  AttnParams p;
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
  p.tiles = tiles;
  const float sc = scale > 0.f ? scale : 1.0f / sqrtf(static_cast<float>(D));
  p.scale_log2 = sc * 1.4426950408889634f;
  p.err = err_flag;
  cudaError_t e = (D == 64) ? launch_attn<64>(p, Hq, B, &tmK, &tmV, st)
                            : launch_attn<128>(p, Hq, B, &tmK, &tmV, st);
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
  return dualflow_decode_attn(gp.q_last, q2raw, a, 0, k_cache, v_cache, block_table,
                              max_blocks_per_seq, gp.seqlens, max_seqlen, nullptr, o2, 0, B, Hq,
                              Hkv, D, block_size, num_blocks, sc, DF_BF16, 0,
                              wl.decode ? workspace : nullptr, wl.decode, err_flag, stream);
}
