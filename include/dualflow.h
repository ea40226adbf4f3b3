/*
 * dualflow.h -- C ABI of the Dual-Flow Transformer decode-step library
 * (libdualflow.so, NVIDIA B200 / sm_100a).
 *
 * The method (arXiv 2608.12385, "Dual-Flow Transformers"; technical summary
 * page "Sintesi Tecnica: Dual-Flow Transformers", sections "Architettura
 * Core" and "Meccanismi Chiave") runs two residual flows through the same
 * weights. The primary flow is an ordinary causal Transformer and is the only
 * writer of the single persistent KV cache (K1, V1). The auxiliary flow, active
 * at the last prompt position and at every generated position, builds its own
 * query Q2, coupled one way to the primary query Q1 through a learned
 * per-layer vector a_l, and attends to the primary K1/V1 without ever writing
 * the cache or feeding back into the primary flow. Because both flows share
 * the weights and the cache, one pass over each weight matrix and each KV page
 * can serve both ("grouped execution"). This library is that decode step
 * (attention, append, grouped projections, norms), the primary prefill that
 * precedes it (the auxiliary flow joining at the last prompt position), the
 * mixture head that combines both flows' next-token distributions, and the
 * MoE MLP block with router replay.
 *
 * Conventions shared by every entry point
 *  - All tensor pointers are DEVICE pointers owned by the caller. The library
 *    allocates nothing and keeps no state between calls; calls are reentrant.
 *    (One exception, dualflow_decode_attn_noalloc, uses a fixed scratch array
 *    inside the library; its own comment below gives the rules.)
 *  - Every call is asynchronous on `stream` (a cudaStream_t passed as void*;
 *    NULL = legacy default stream). Argument errors are detected on the host
 *    and returned BEFORE any launch. A failed launch returns DF_ERR_CUDA.
 *  - Errors that depend on device data (a length, a page index, a position)
 *    never trap: the kernel skips the bad access and ORs a DF_DEVERR_* bit into
 *    *err_flag (device int32, may be NULL). The caller reads it after syncing.
 *  - Every wait inside a kernel is bounded (about 2 s); a wait that gives up
 *    sets DF_DEVERR_TIMEOUT and the kernel returns.
 *  - bf16 = IEEE bfloat16 (1-8-7), stored as 2-byte values. "Elements" strides
 *    count elements of the tensor's dtype.
 *  - Paged KV cache layout: cache[num_blocks][Hkv][block_size][D], token j of
 *    sequence b in page block_table[b * max_blocks_per_seq + j / block_size],
 *    slot j % block_size. block_size must be 64.
 */
#ifndef DUALFLOW_H
#define DUALFLOW_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  DF_OK = 0,
  DF_ERR_NULL = 1,        /* a required pointer is NULL                        */
  DF_ERR_SHAPE = 2,       /* sizes inconsistent or out of range                */
  DF_ERR_UNSUPPORTED = 3, /* valid request this build does not implement       */
  DF_ERR_WORKSPACE = 4,   /* workspace missing, too small or misaligned        */
  DF_ERR_ALIGN = 5,       /* pointer or stride not aligned as documented       */
  DF_ERR_CUDA = 6         /* a CUDA runtime call or a launch failed            */
} df_status;

typedef enum { DF_FP32 = 0, DF_BF16 = 1 } df_dtype;

typedef enum {
  DF_EPI_NONE = 0,     /* y = x w^T                                             */
  DF_EPI_SWIGLU = 1,   /* y = SiLU(gate) * up (+ b * y_primary on aux rows)     */
  DF_EPI_RESIDUAL = 2  /* y = residual + x w^T (+ c * (x w^T)_primary on aux)   */
} df_epilogue;

/* Bits ORed into *err_flag by kernels (device-side data errors). */
#define DF_DEVERR_SEQLEN   0x1 /* seqlens[b] < 1 (output 0) or above max_seqlen (clamped) */
#define DF_DEVERR_BLOCK    0x2 /* a block_table entry outside [0, num_blocks): page skipped */
#define DF_DEVERR_POSITION 0x4 /* an append position outside the sequence's table: skipped */
#define DF_DEVERR_TIMEOUT  0x8 /* a bounded in-kernel wait gave up: outputs invalid         */

/* Version of this ABI (incremented on any signature change). */
int dualflow_abi_version(void);

/* Human-readable name of a df_status value; never NULL. */
const char* dualflow_status_string(int status);

/* ------------------------------------------------------------------------ */
/* Failure-detection self-test (no counterpart in the pages).                */
/*                                                                           */
/* Every in-kernel wait of this library (on an mbarrier, a grid counter or a */
/* peer CTA) gives up after about 2e9 SM cycles (1-2 s), ORs                 */
/* DF_DEVERR_TIMEOUT into the call's err_flag and lets the kernel return, so */
/* a lost arrival never hangs the GPU. This entry point exercises that       */
/* mechanism without a fault: one launch of one warp waits, with the same    */
/* bounded waits (single thread, then whole warp), on an mbarrier that       */
/* nothing arrives on; after two time-outs (2-4 s) *err_flag has             */
/* DF_DEVERR_TIMEOUT set and the context stays usable.                       */
/* err_flag: int32 in device memory (ORed into). Asynchronous on `stream`.   */
/* ------------------------------------------------------------------------ */
df_status dualflow_selftest_wait_timeout(int32_t* err_flag, void* stream);

/* ------------------------------------------------------------------------ */
/* Dual-flow decode attention (asymmetric shared-KV attention).              */
/*                                                                           */
/* Page "Sintesi Tecnica: Dual-Flow Transformers", section "Meccanismi       */
/* Chiave": the primary query Q1 runs ordinary causal attention over K1/V1;  */
/* the auxiliary query Q2 = Q2raw + a (.) Q1 (element-wise; the pages name   */
/* the coupling vector but print no formula, this additive one-way form is   */
/* the reading taken) attends over the SAME K1/V1. For sequence b, query     */
/* head h, KV head g = h / (Hq / Hkv), flow f:                               */
/*   O_f[b,h] = softmax(scale * q_f K1[b,g]^T) V1[b,g] over the first         */
/*   seqlens[b] tokens of the cache.                                         */
/* Each KV page is read from HBM once for all 2 * Hq/Hkv query rows of its    */
/* KV head. Split over the sequence (flash-decoding) with per-split fp32     */
/* partials in `workspace`, merged by the last split to finish (bf16) or by  */
/* a separate combine kernel (fp32).                                         */
/*                                                                           */
/* q1, q2raw : [B][Hq][D] (dtype), sequence b at q + b*q_stride_b elements   */
/*             (q_stride_b = 0 means Hq*D). 4-byte aligned; q_stride_b even. */
/* a         : [Hq][D] (dtype) or NULL (q2raw is then used as Q2 as is).     */
/* k_cache, v_cache : paged cache (dtype), 16-byte aligned. Read only: this  */
/*             call never writes the cache.                                  */
/* block_table : int32 [B][max_blocks_per_seq]; seqlens : int32 [B], the     */
/*             attended length of each sequence (>= 1, <= max_seqlen).       */
/* max_seqlen : host upper bound of seqlens; <= max_blocks_per_seq*block_size.*/
/* o1, o2    : [B][Hq][D] (dtype) outputs at o + b*o_stride_b (0 = Hq*D).    */
/*             o1 == NULL: aux-only call (q1 still needed for the coupling). */
/*             o2 == NULL or q2raw == NULL: primary-only call.               */
/*             O1 is bit-identical in primary-only, aux-only and dual calls  */
/*             and independent of q2raw/a (even NaN/Inf): the split plan      */
/*             depends only on (B, Hkv, max_seqlen, num_splits).              */
/* scale     : softmax scale; <= 0 selects 1/sqrt(D).                         */
/* dtype     : DF_BF16 (fp32 accumulation; Q2 and softmax weights kept to     */
/*             ~16 mantissa bits through a bf16 hi/lo split) or DF_FP32.      */
/* num_splits: 0 = automatic; otherwise the requested number of splits.      */
/* workspace : device scratch, 256-byte aligned, at least                    */
/*             dualflow_decode_attn_workspace_size(...) bytes (0 when the    */
/*             plan has one split, then workspace may be NULL). bf16: its    */
/*             first bytes are per-(sequence, KV head) arrival counters of   */
/*             the in-kernel split combine, so a new workspace must be       */
/*             ZERO-FILLED once; every completed call leaves them at zero    */
/*             again (re-zero after a call that set a device error code).    */
/*             Calls sharing one workspace must be ordered on the GPU.       */
/* Supported: D in {64, 128}, block_size 64, Hq/Hkv in {1,2,3,4}.            */
/* ------------------------------------------------------------------------ */
int dualflow_decode_attn_num_splits(int B, int Hkv, int max_seqlen, int block_size,
                                    int num_splits);
/* Kernel launches one dualflow_decode_attn call makes with these arguments:*/
/* bf16 1 (the split combine runs in the kernel); fp32 1 (one split) or 2   */
/* (split kernel + combine kernel); 0 for invalid arguments.                 */
int dualflow_decode_attn_num_launches(int B, int Hkv, int max_seqlen, int block_size,
                                      int num_splits, int dtype);
size_t dualflow_decode_attn_workspace_size(int B, int Hq, int Hkv, int D, int max_seqlen,
                                           int block_size, int num_splits);
df_status dualflow_decode_attn(const void* q1, const void* q2raw, const void* a,
                               int64_t q_stride_b, const void* k_cache, const void* v_cache,
                               const int32_t* block_table, int max_blocks_per_seq,
                               const int32_t* seqlens, int max_seqlen, void* o1, void* o2,
                               int64_t o_stride_b, int B, int Hq, int Hkv, int D,
                               int block_size, int num_blocks, float scale, int dtype,
                               int num_splits, void* workspace, size_t workspace_bytes,
                               int32_t* err_flag, void* stream);

/* ------------------------------------------------------------------------ */
/* Decode attention without a caller workspace.                              */
/*                                                                           */
/* The paper has no counterpart: this is a deployment convenience.           */
/* Some callers cannot allocate device memory for a workspace -- a serving    */
/* engine that has given all free device memory to its own KV-page pool      */
/* before decoding starts, or a plain C host program with no device          */
/* allocator. This entry point computes exactly what dualflow_decode_attn    */
/* computes (same arguments minus workspace/workspace_bytes, same results)   */
/* but keeps the split partials in a fixed array inside the library's own    */
/* device memory: DF_DECODE_ATTN_NOALLOC_SCRATCH_BYTES (16 MiB), reserved on  */
/* every GPU that loads the library and held until the process exits. It     */
/* never calls cudaMalloc/cudaFree or any allocating routine.                */
/*  - A request whose workspace would exceed that size (see                  */
/*    dualflow_decode_attn_workspace_size) returns DF_ERR_WORKSPACE before    */
/*    any launch.                                                            */
/*  - The array's device address belongs to a CUDA context. The first call  */
/*    made in a context (the device's primary context, or a driver-API       */
/*    context made current by the caller; again after a device reset) looks  */
/*    it up with cudaGetSymbolAddress, which also loads the library's module */
/*    there, and caches it under the context's unique id; make that first   */
/*    call before any stream capture. A failed lookup: DF_ERR_CUDA.          */
/*  - All calls on a device share the one array, which keeps the last call's */
/*    contents. After every argument check has passed, a bf16 call that      */
/*    splits clears, on its stream, the part that must start at zero (the    */
/*    arrival counters; cudaMemsetAsync, no allocation). A rejected call     */
/*    touches nothing. Calls that overlap on the GPU (different streams, no  */
/*    ordering) race on the array: order them.                              */
/* ------------------------------------------------------------------------ */
#define DF_DECODE_ATTN_NOALLOC_SCRATCH_BYTES (16u * 1024u * 1024u)
df_status dualflow_decode_attn_noalloc(const void* q1, const void* q2raw, const void* a,
                                       int64_t q_stride_b, const void* k_cache,
                                       const void* v_cache, const int32_t* block_table,
                                       int max_blocks_per_seq, const int32_t* seqlens,
                                       int max_seqlen, void* o1, void* o2, int64_t o_stride_b,
                                       int B, int Hq, int Hkv, int D, int block_size,
                                       int num_blocks, float scale, int dtype, int num_splits,
                                       int32_t* err_flag, void* stream);

/* ------------------------------------------------------------------------ */
/* Primary-only KV append.                                                  */
/*                                                                           */
/* Page "Sintesi Tecnica: Dual-Flow Transformers", section "Architettura      */
/* Core": only the primary flow writes the persistent KV cache. Copies       */
/* k_new[b][g][:] and v_new[b][g][:] (every KV head g) into the page          */
/* block_table[b][positions[b] / block_size], slot positions[b] % block_size.*/
/* A bit-exact copy; no other cache byte changes.                            */
/*                                                                           */
/* k_new, v_new : [B][Hkv][D] (dtype) at + b*new_stride_b elements (0 means  */
/*             Hkv*D); 16-byte aligned rows (D*size and stride*size % 16 == 0).*/
/* positions : int32 [B], the slot to write (= cache length before the step).*/
/*             Out-of-table positions or page numbers are skipped and flagged.*/
/* ------------------------------------------------------------------------ */
df_status dualflow_kv_append(const void* k_new, const void* v_new, int64_t new_stride_b,
                             void* k_cache, void* v_cache, const int32_t* block_table,
                             int max_blocks_per_seq, const int32_t* positions, int B, int Hkv,
                             int D, int block_size, int num_blocks, int dtype,
                             int32_t* err_flag, void* stream);

/* ------------------------------------------------------------------------ */
/* Primary prefill (prompt processing), with the auxiliary query at the last */
/* prompt position.                                                          */
/*                                                                           */
/* Page "Sintesi Tecnica: Dual-Flow Transformers", section "Architettura      */
/* Core": the primary flow is a standard causal Transformer that processes   */
/* the whole prompt and writes the persistent cache; the auxiliary flow is   */
/* skipped over the prompt and switched on only at the last prompt position. */
/* Section "Costi di Inferenza vs. Addestramento": prefill costs the same as  */
/* a standard Transformer's.                                                 */
/*                                                                           */
/* Sequence b's chunk is the token rows t in [cu_seqlens[b],                 */
/* cu_seqlens[b+1]) (n_b >= 1 tokens); its cache already holds ctx_lens[b]   */
/* tokens (ctx_lens NULL = 0: a fresh prompt), so chunk token i is position  */
/* p = ctx_lens[b] + i. The call                                             */
/*  1. writes k_new/v_new row t to cache position p (as dualflow_kv_append); */
/*     k_new = v_new = NULL skips this (the cache already holds the chunk);  */
/*  2. O1[t,h] = softmax_j(scale * q1[t,h] . k_j) V over positions j <= p of */
/*     KV head g = h / (Hq/Hkv) (causal; prefix + chunk);                    */
/*  3. if q2raw and o2 are given: O2[b,h] = the decode step's auxiliary      */
/*     output for the last position P = ctx_lens[b] + n_b - 1, i.e. Q2 =     */
/*     q2raw[b] + a (.) q1[last row of b] over positions j <= P (computed by */
/*     the decode attention kernel in auxiliary-only mode, with its own     */
/*     split plan; when ctx_lens is NULL and T = B max_q_len, i.e. every     */
/*     chunk has max_q_len tokens, with the split count that fills one wave  */
/*     of 2 CTAs per SM, capped by that plan).                               */
/*                                                                           */
/* q1        : bf16 [T][Hq][D], token row t at q1 + t*q_stride_t elements    */
/*             (0 = Hq*D); 16-byte aligned, q_stride_t % 8 == 0.              */
/* k_new, v_new : bf16 [T][Hkv][D] at + t*kv_stride_t (0 = Hkv*D), 16-byte   */
/*             aligned, kv_stride_t % 8 == 0; or both NULL.                  */
/* q2raw, a  : bf16 [B][Hq][D] (the auxiliary query of the last position,    */
/*             before coupling) and [Hq][D] (or NULL: no coupling).          */
/* cu_seqlens: int32 [B+1], device; ctx_lens: int32 [B], device, or NULL.    */
/* max_q_len : host bound of every n_b (sets the grid); max_seqlen: host     */
/*             bound of every ctx_lens[b] + n_b, <= max_blocks_per_seq * 64. */
/*             A chunk outside these bounds (or with n_b < 1, or rows past T)*/
/*             sets DF_DEVERR_SEQLEN and is skipped (its rows unwritten).    */
/*             A block_table entry outside [0, num_blocks) sets             */
/*             DF_DEVERR_BLOCK; that sequence's outputs are then invalid.    */
/* o1        : bf16 [T][Hq][D] at + t*o_stride_t (0 = Hq*D), 4-byte aligned. */
/* o2        : bf16 [B][Hq][D] or NULL.                                      */
/* workspace : only with the auxiliary step: 256-byte aligned, at least      */
/*             dualflow_prefill_workspace_size(...) bytes, ZERO-FILLED once  */
/*             (its first bytes are the decode kernel's arrival counters,    */
/*             which every completed call leaves at zero).                   */
/* Supported: dtype DF_BF16, D in {64, 128}, block_size 64; with the         */
/* auxiliary step also Hq/Hkv <= 4. Kernel launches per call:                */
/* dualflow_prefill_num_launches(k_new != NULL, auxiliary step).             */
/* ------------------------------------------------------------------------ */
size_t dualflow_prefill_workspace_size(int B, int Hq, int Hkv, int D, int max_seqlen,
                                       int block_size);
/* Attention kernel of a prefill call. DF_PREFILL_KERNEL_TCGEN05: tensor    */
/* cores with TMEM accumulators, 128-row tiles; used (automatically) when    */
/* D = 64 or 128, T >= 128, o1 is 16-byte aligned and o_stride_t % 8 == 0.   */
/* DF_PREFILL_KERNEL_MMA_SYNC: warp-level mma.sync, 64-row tiles, any        */
/* supported shape. Both compute the same result within the tolerance; the   */
/* cache write and the auxiliary step are the same code.                     */
#define DF_PREFILL_KERNEL_AUTO 0
#define DF_PREFILL_KERNEL_MMA_SYNC 1
#define DF_PREFILL_KERNEL_TCGEN05 2
/* The kernel dualflow_prefill picks for these arguments (o_stride_t 0 = Hq*D). */
int dualflow_prefill_kernel(int D, int T, const void* o1, int64_t o_stride_t, int Hq);
int dualflow_prefill_num_launches(int with_append, int with_aux);
df_status dualflow_prefill(const void* q1, int64_t q_stride_t, const void* k_new,
                           const void* v_new, int64_t kv_stride_t, const void* q2raw,
                           const void* a, void* k_cache, void* v_cache,
                           const int32_t* block_table, int max_blocks_per_seq,
                           const int32_t* cu_seqlens, const int32_t* ctx_lens, int max_q_len,
                           int max_seqlen, void* o1, int64_t o_stride_t, void* o2, int B, int T,
                           int Hq, int Hkv, int D, int block_size, int num_blocks, float scale,
                           int dtype, void* workspace, size_t workspace_bytes, int32_t* err_flag,
                           void* stream);
/* The same call with the attention kernel chosen by the caller (kernel =   */
/* DF_PREFILL_KERNEL_*; TCGEN05 where it does not fit: DF_ERR_UNSUPPORTED;  */
/* another value: DF_ERR_SHAPE).                                             */
df_status dualflow_prefill_ex(const void* q1, int64_t q_stride_t, const void* k_new,
                              const void* v_new, int64_t kv_stride_t, const void* q2raw,
                              const void* a, void* k_cache, void* v_cache,
                              const int32_t* block_table, int max_blocks_per_seq,
                              const int32_t* cu_seqlens, const int32_t* ctx_lens, int max_q_len,
                              int max_seqlen, void* o1, int64_t o_stride_t, void* o2, int B,
                              int T, int Hq, int Hkv, int D, int block_size, int num_blocks,
                              float scale, int dtype, int kernel, void* workspace,
                              size_t workspace_bytes, int32_t* err_flag, void* stream);

/* ------------------------------------------------------------------------ */
/* Grouped shared-weight projection (tcgen05 tensor cores, TMEM accumulator).*/
/*                                                                           */
/* Pages "Sintesi Tecnica" ("Architettura Core": both flows share every      */
/* attention, MLP and output matrix; "Costi di Inferenza": grouped decode     */
/* reads the unique weights once) and the jumtra.com summary ("提案手法の詳細").*/
/* Both flows' rows multiply the same bf16 weight in ONE GEMM:               */
/*   x = [m_primary primary rows ; m_aux auxiliary rows] (bf16 [M][K], row   */
/*   stride ldx), w = bf16 [N][K] (row stride K), fp32 accumulation.          */
/* Auxiliary rows are stored only for output columns < n_aux (n_aux = N:     */
/* all); e.g. the aux flow needs only the Q part of a fused QKV projection.   */
/* Epilogues (the coupling reads are one way, primary -> auxiliary; aux row  */
/* m_primary + j is paired with primary row j, so m_aux must be m_primary    */
/* when a coupling vector is given):                                          */
/*  DF_EPI_NONE     : y[M][N] = x w^T; coupling and residual must be NULL.   */
/*  DF_EPI_SWIGLU   : w = [W_gate (F rows) ; W_up (F rows)], N = 2F;          */
/*                    y[M][F] = SiLU(x W_gate^T) * (x W_up^T), and aux rows   */
/*                    add coupling[n] * y_primary[j][n] (b_l; NULL = none).    */
/*  DF_EPI_RESIDUAL : y[M][N] = residual + x w^T, and aux rows add            */
/*                    coupling[n] * (x w^T)[j][n] before the residual (c_l).   */
/* y and residual may alias (in-place residual add). All bf16.               */
/* w is treated as constant: every launch is a programmatic dependent launch */
/* that starts streaming w BEFORE it waits for the kernel launched ahead of  */
/* it on the stream (x, residual and coupling are read only after the wait),*/
/* so that kernel must not write w.                                          */
/* Supported: M = m_primary + m_aux in [1, 128]; K % 64 == 0; N % 128 == 0    */
/* (SWIGLU: F % 64 == 0); ldx, ldy, ldr multiples of 8 elements; x, w        */
/* 16-byte aligned; n_aux a multiple of 32 or the full output width.          */
/* workspace: >= dualflow_grouped_proj_workspace_size(...) bytes, 256-byte    */
/* aligned, no initial contents required; one workspace may serve            */
/* projections of any shape issued in order on one stream. Launches: the     */
/* GEMM kernel plus, when a tile's k-range is split over CTAs, a reduction    */
/* kernel that sums the fp32 partials in fixed order (deterministic).         */
/* ------------------------------------------------------------------------ */
size_t dualflow_grouped_proj_workspace_size(int M, int N, int K, int epilogue);
/* Number of kernel launches one dualflow_grouped_proj call makes (1 or 2). */
int dualflow_grouped_proj_num_launches(int M, int N, int K, int epilogue);
df_status dualflow_grouped_proj(const void* x, int64_t ldx, int m_primary, int m_aux,
                                const void* w, int N, int K, int n_aux, void* y, int64_t ldy,
                                int epilogue, const void* coupling, const void* residual,
                                int64_t ldr, void* workspace, size_t workspace_bytes,
                                int32_t* err_flag, void* stream);

/* Same projection, and a hint for the projection that will be launched next */
/* on the same stream with the same rows and workspace size: weight w_next   */
/* (bf16 [N_next][K_next], 16-byte aligned, K_next % 64 == 0, N_next % 128   */
/* == 0) and epilogue_next. While this call's tiles finish (the weights have */
/* streamed, HBM is idle), its CTAs prefetch into L2 the first k-blocks that  */
/* each CTA of the next call will read, so the next call starts from L2      */
/* instead of a cold HBM pipeline. Results are identical with or without the */
/* hint; w_next NULL = no hint. The prefetch is a cache hint only: w_next is */
/* never written, and a next call with other arguments is still correct.     */
df_status dualflow_grouped_proj_chain(const void* x, int64_t ldx, int m_primary, int m_aux,
                                      const void* w, int N, int K, int n_aux, void* y,
                                      int64_t ldy, int epilogue, const void* coupling,
                                      const void* residual, int64_t ldr, void* workspace,
                                      size_t workspace_bytes, const void* w_next, int N_next,
                                      int K_next, int epilogue_next, int32_t* err_flag,
                                      void* stream);

/* Batched form: `batch` projections of one shape in one launch (the MoE    */
/* experts: every expert's weights stream once, all experts share one       */
/* pipeline fill and one tail). Entry b reads x + b*x_bstride and             */
/* w + b*w_bstride and writes y + b*y_bstride (elements; 0 = packed). Only    */
/* DF_EPI_NONE and DF_EPI_SWIGLU, no coupling or residual; auxiliary rows     */
/* store every output column. The optional next-projection hint may itself    */
/* be batched (batch_next, w_next_bstride). Without a single-launch plan the  */
/* call runs one projection per entry.                                        */
df_status dualflow_grouped_proj_batched(
    const void* x, int64_t ldx, int64_t x_bstride, int m_primary, int m_aux, const void* w, int N,
    int K, int64_t w_bstride, void* y, int64_t ldy, int64_t y_bstride, int batch, int epilogue,
    void* workspace, size_t workspace_bytes, const void* w_next, int N_next, int K_next,
    int epilogue_next, int batch_next, int64_t w_next_bstride, int32_t* err_flag, void* stream);
/* Kernel launches one batched call makes: 1 with a single-launch plan.      */
int dualflow_grouped_proj_batched_num_launches(int M, int N, int K, int epilogue, int batch);

/* ------------------------------------------------------------------------ */
/* Pre-attention half of the decoder layer in ONE launch.                    */
/*                                                                           */
/* Pages "Sintesi Tecnica" ("Architettura Core": the flows share the         */
/* projection matrices, only the primary flow writes the persistent KV      */
/* cache, the auxiliary flow needs only its query; "Costi di Inferenza":     */
/* grouped decode reads the unique weights once for both flows). With rows   */
/* [0, m_primary) primary and [m_primary, 2 m_primary) auxiliary, M =        */
/* 2 m_primary, q_dim = Hq D, kv_dim = Hkv D, N = q_dim + 2 kv_dim:          */
/*   r   = 1 / sqrt(mean_row(x^2) + eps)          (RMSNorm, unit gain)       */
/*   qkv = bf16(r (x W_qkv^T)): primary rows all N columns, auxiliary rows   */
/*         the q_dim Q columns only (their K / V columns are not written)    */
/*   and, as dualflow_kv_append, primary row b's K and V columns (the same   */
/*   bf16 values) into the cache slot of positions[b].                       */
/* which is dualflow_rmsnorm -> dualflow_grouped_proj (n_aux = q_dim) ->     */
/* dualflow_kv_append computed by one launch of 4-CTA clusters: each         */
/* cluster owns a column tile, its 4 CTAs multiply the 4 quarters of K and   */
/* reduce the partial sums (and the row sums of squares of the norm)        */
/* through distributed shared memory. The row scale multiplies the          */
/* accumulator (the normalised rows are not rounded to bf16 and stored), so */
/* the result matches the three-call form within the bf16 tolerance, not     */
/* bit for bit. Sums are taken in a fixed order (deterministic); primary     */
/* rows never depend on auxiliary rows.                                      */
/*                                                                           */
/* x     : bf16 [M][d_model]; w_qkv : bf16 [N][d_model] (Q rows, K rows, V   */
/* rows), row-major. qkv : bf16 [M][N], written as above (16-byte aligned).  */
/* k_cache, v_cache, block_table, max_blocks_per_seq, positions, block_size, */
/* num_blocks: as dualflow_kv_append (bf16 cache); an out-of-table position  */
/* or page is skipped and flagged in err_flag. w_qkv is read before the wait */
/* for the kernel launched ahead on the stream (programmatic dependent       */
/* launch), so that kernel must not write it. No workspace.                  */
/* Supported (else DF_ERR_UNSUPPORTED; dualflow_layer_pre_attention_supported*/
/* returns 0): 1 <= m_primary <= 64, d_model % 64 == 0, D % 8 == 0, and N at */
/* most 256 x the number of 4-CTA clusters the device holds at once (33 on  */
/* a 148-SM B200: N <= 8448). Needs a current CUDA device. One launch.       */
/* ------------------------------------------------------------------------ */
int dualflow_layer_pre_attention_supported(int m_primary, int d_model, int Hq, int Hkv, int D);
df_status dualflow_layer_pre_attention(const void* x, const void* w_qkv, int m_primary,
                                       int d_model, int Hq, int Hkv, int D, float eps, void* qkv,
                                       void* k_cache, void* v_cache, const int32_t* block_table,
                                       int max_blocks_per_seq, const int32_t* positions,
                                       int block_size, int num_blocks, int32_t* err_flag,
                                       void* stream);

/* ------------------------------------------------------------------------ */
/* Pre-attention half split across two launches: QKV partial products.       */
/*                                                                           */
/* Same operation as dualflow_layer_pre_attention (pages "Sintesi Tecnica",  */
/* "Architettura Core" and "Costi di Inferenza"), but the split sums are     */
/* not reduced here: this launch multiplies and stores, and                  */
/* dualflow_decode_attn_qkv_partials (below) reduces, normalises, rounds     */
/* and appends in its prologue, which removes the reduction's               */
/* distributed-shared-memory round trip from the step. With M = 2 m_primary */
/* and N = (Hq + 2 Hkv) D as in dualflow_layer_pre_attention:                */
/*   part[k][row][n] = sum over K quarter k of x[row][j] w_qkv[n][j]  (fp32) */
/*   ss_part[k][row] = sum over K quarter k of x[row][j]^2            (fp32) */
/* for k = 0..3, the 4 quarters of d_model in order (a quarter past the end  */
/* of K, when d_model / 64 < 4, holds zeros). All M rows and N columns are  */
/* written. Summing the parts in order k = 0..3 from 0 and scaling by        */
/* r = 1 / sqrt(sum_k ss_part[k][row] / d_model + eps) reproduces           */
/* dualflow_layer_pre_attention's qkv bit for bit.                           */
/*                                                                           */
/* x, w_qkv : as dualflow_layer_pre_attention. part : fp32 [4][M][N],        */
/* ss_part : fp32 [4][M], both 16-byte aligned, written completely; N * 4    */
/* must be a multiple of 16 bytes (D % 8 == 0 guarantees it). w_qkv is read  */
/* before the wait for the kernel launched ahead on the stream. Supported:   */
/* as dualflow_layer_pre_attention_supported. One launch, no workspace.      */
/* ------------------------------------------------------------------------ */
df_status dualflow_layer_qkv_partials(const void* x, const void* w_qkv, int m_primary,
                                      int d_model, int Hq, int Hkv, int D, void* part,
                                      void* ss_part, int32_t* err_flag, void* stream);

/* ------------------------------------------------------------------------ */
/* Dual-flow decode attention fed by QKV partial products.                   */
/*                                                                           */
/* Computes what dualflow_layer_pre_attention followed by                    */
/* dualflow_decode_attn (bf16, q_stride_b = N, q2raw = the auxiliary rows'   */
/* qkv) compute, with the same results bit for bit, in one launch: each CTA  */
/* sums `parts` partial products in order, scales by the RMSNorm row scale   */
/* and rounds to bf16 its KV head's Q1 and Q2raw rows (the pre-attention     */
/* formulas above), and the CTA whose split holds position seqlens[b] - 1    */
/* writes primary row b's K and V (same rounding) into that cache slot       */
/* before its page is loaded; the other splits never read that slot.         */
/*                                                                           */
/* part, ss_part, parts : [parts][2 m_primary][(Hq + 2 Hkv) D] and           */
/*            [parts][2 m_primary] fp32 as written by                        */
/*            dualflow_layer_qkv_partials (parts = 4; 1..4 accepted);        */
/*            row b primary, row m_primary + b auxiliary of sequence b.      */
/*            16-byte and 4-byte aligned. d_model, eps: the norm's width     */
/*            and epsilon.                                                   */
/* The other arguments are dualflow_decode_attn's with B = m_primary and     */
/* dtype bf16 (k_cache and v_cache are WRITTEN at the appended slot, so      */
/* they must not be read by another kernel in flight). seqlens[b] counts the */
/* appended token. An out-of-table page is skipped and flagged (             */
/* DF_DEVERR_BLOCK), like a page the attention reads.                        */
/* Supported: as dualflow_decode_attn (bf16). One launch.                    */
/* ------------------------------------------------------------------------ */
df_status dualflow_decode_attn_qkv_partials(
    const float* part, const float* ss_part, int parts, int m_primary, int d_model, float eps,
    const void* a, const void* k_cache, const void* v_cache, const int32_t* block_table,
    int max_blocks_per_seq, const int32_t* seqlens, int max_seqlen, void* o1, void* o2,
    int64_t o_stride_b, int Hq, int Hkv, int D, int block_size, int num_blocks, float scale,
    int num_splits, void* workspace, size_t workspace_bytes, int32_t* err_flag, void* stream);

/* ------------------------------------------------------------------------ */
/* Post-attention half of the decoder layer in ONE persistent launch.        */
/*                                                                           */
/* Pages "Sintesi Tecnica" ("Architettura Core": the flows share the output  */
/* and MLP matrices; "Meccanismi Chiave": one-way coupling b_l at the MLP    */
/* intermediate and c_l at the MLP output; "Costi di Inferenza": grouped     */
/* decode reads the unique weights once for both flows). With rows           */
/* [0, m_primary) primary and [m_primary, 2 m_primary) auxiliary (sequence j */
/* = rows j and m_primary + j), M = 2 m_primary:                             */
/*   x_mid = x + attn W_o^T                                                  */
/*   r     = 1 / sqrt(mean_row(x_mid^2) + eps)   (RMSNorm, unit gain)         */
/*   h     = SiLU(r x_mid W_gate^T) * (r x_mid W_up^T); aux rows += b (.)     */
/*           primary h                                                       */
/*   x_out = x_mid + h W_down^T; aux rows += c (.) (h W_down^T) of primary   */
/* which is dualflow_grouped_proj (residual) -> dualflow_rmsnorm ->          */
/* dualflow_grouped_proj (swiglu, b) -> dualflow_grouped_proj (residual, c)  */
/* computed by one grid of one CTA per SM, launched as clusters of 4 CTAs,   */
/* whose TMA producers stream the three weights back to back. W_o and W_down */
/* are split 4 ways along K over the CTAs of a cluster and their split sums  */
/* are reduced inside the cluster through distributed shared memory; the    */
/* steps that need every column of the step before (x_mid for gate/up, h for */
/* W_down) wait on grid-wide counters in the workspace (bounded waits). The  */
/* norm's row scale multiplies the gate/up accumulators (the normalised rows */
/* are not rounded to bf16 and stored). Each split-k sum is taken in a fixed */
/* order, so the results are deterministic and primary rows never depend on  */
/* auxiliary rows. They match the four-call form within the bf16 tolerance,  */
/* not bit for bit (other split-k orders, no bf16 rounding of the normalised */
/* rows).                                                                    */
/*                                                                           */
/* attn  : bf16 [M][q_dim] (the attention output, O1 rows then O2 rows).      */
/* x     : bf16 [M][d_model] (the layer input, residual of W_o).             */
/* w_o [d_model][q_dim], w_gu [2F][d_model] (gate rows, then up rows),       */
/* w_down [d_model][F]: bf16, row-major. b [F], c [d_model] bf16 or NULL.     */
/* x_mid [M][d_model], h [M][F], x_out [M][d_model]: bf16, written (all rows */
/* packed, 16-byte aligned). w_* are read before the wait for the kernel     */
/* launched ahead on the stream (programmatic dependent launch), so that     */
/* kernel must not write them.                                               */
/* workspace: >= dualflow_layer_post_attention_workspace_size(...) bytes     */
/* (256 + d_model * 16), 256-byte aligned, ZERO-FILLED once: its first 256  */
/* bytes are grid counters that every completed call leaves at zero         */
/* (after a DF_DEVERR_TIMEOUT, zero it again); the rest holds the row sums   */
/* of squares of the norm. Calls sharing one workspace must not overlap on   */
/* the GPU.                                                                  */
/* Supported (else DF_ERR_UNSUPPORTED; the size query returns 0):            */
/* 1 <= m_primary <= 64, d_model % 128 == 0 with d_model / 128 at most the   */
/* number of 4-CTA clusters the device holds at once (33 on a 148-SM B200:   */
/* d_model <= 4224), q_dim % 64 == 0, F % 64 == 0, F <= 112 * 4 * (that     */
/* cluster count). Needs a current CUDA device (the size query too). One    */
/* kernel launch.                                                            */
/* ------------------------------------------------------------------------ */
size_t dualflow_layer_post_attention_workspace_size(int m_primary, int d_model, int q_dim,
                                                    int F);
df_status dualflow_layer_post_attention(const void* attn, const void* x, const void* w_o,
                                        const void* w_gu, const void* w_down, const void* b,
                                        const void* c, int m_primary, int d_model, int q_dim,
                                        int F, float eps, void* x_mid, void* h, void* x_out,
                                        void* workspace, size_t workspace_bytes,
                                        int32_t* err_flag, void* stream);

/* ------------------------------------------------------------------------ */
/* The same launch followed by the NEXT layer's grouped QKV projection of    */
/* x_out, left as partial products (the layer-stack form).                   */
/*                                                                           */
/* Pages "Sintesi Tecnica" ("Architettura Core", "Costi di Inferenza"): in a */
/* stack of layers the next layer's first step reads this layer's output;    */
/* computing it inside this launch lets its weight stream follow W_down's    */
/* through the same pipeline instead of waiting for a new launch. Outputs    */
/* x_mid, h, x_out exactly as dualflow_layer_post_attention (bit for bit),   */
/* and, as dualflow_layer_qkv_partials(x_out, w_qkv_next, ...) would:        */
/*   part[r][row][col] = sum over k in K quarter r of x_out[row][k]           */
/*                       w_qkv_next[col][k]    (fp32, the same MMA order, so  */
/*                       bit for bit equal to that call's)                    */
/*   ss_part[r][row]   = sum over the same k of x_out[row][k]^2 (fp32; other  */
/*                       summation order: equal within fp32 rounding)         */
/* for r = 0..3, all M rows (auxiliary rows' K / V columns included, unused), */
/* col < (Hq + 2 Hkv) D. These feed dualflow_decode_attn_qkv_partials (parts */
/* = 4) of the next layer, which applies that layer's RMSNorm.                */
/* w_qkv_next: bf16 [(Hq + 2 Hkv) D][d_model]; part: fp32 [4][M][(Hq + 2 Hkv)*/
/* D]; ss_part: fp32 [4][M]; all 16-byte aligned, written by the launch and   */
/* read by the next launch on the stream. w_qkv_next is read before the wait  */
/* for the kernel launched ahead (like the other weights).                    */
/* Errors: NULL w_qkv_next / part / ss_part: DF_ERR_NULL; q_dim != Hq * D or */
/* Hq % Hkv != 0: DF_ERR_SHAPE; (Hq + 2 Hkv) D without a divisor among 64,   */
/* 128, 192, 256 giving at most one column tile per 4-CTA cluster, or        */
/* d_model % 256 != 0: DF_ERR_UNSUPPORTED; else as above. One kernel launch; */
/* the same workspace.                                                        */
/* ------------------------------------------------------------------------ */
df_status dualflow_layer_post_attention_qkv(
    const void* attn, const void* x, const void* w_o, const void* w_gu, const void* w_down,
    const void* b, const void* c, int m_primary, int d_model, int q_dim, int F, float eps,
    void* x_mid, void* h, void* x_out, void* workspace, size_t workspace_bytes,
    const void* w_qkv_next, int Hq, int Hkv, int D, void* part, void* ss_part,
    int32_t* err_flag, void* stream);

/* ------------------------------------------------------------------------ */
/* MoE MLP block with router replay.                                         */
/*                                                                           */
/* Page "Sintesi Tecnica: Dual-Flow Transformers", section "Meccanismi        */
/* Chiave" (router replay: the auxiliary flow applies the experts selected   */
/* by the primary router with its own mixing weights) and section            */
/* "Contributi Chiave" (independent expert fan-outs). Readings: one router    */
/* matrix shared by both flows; ids = the primary's top-k_aux experts by      */
/* descending router logit (ties: lower expert index); the primary uses the  */
/* first k, the auxiliary all k_aux (k_aux = k: router replay proper); gates */
/* = softmax of each flow's own router logits over its set; SwiGLU experts.  */
/* A block is: route -> dispatch -> per expert e, dualflow_grouped_proj of    */
/* xe[e] ([128][d], m_primary = 64) with W_gate/up[e] (SWIGLU) and then        */
/* W_down[e] (NONE) into ye[e] -> combine. Each expert's weights stream once  */
/* for both flows; the projections' shapes do not depend on the routing.     */
/* Limits: 1 <= B <= 64 tokens per flow per call, E <= 256,                  */
/* 1 <= k <= k_aux <= min(E, 8), d % 8 == 0, 16-byte aligned rows.             */
/*                                                                           */
/* route:    x bf16 [2B][d] (primary rows, then auxiliary rows; stride ldx,  */
/*           0 = d), w_router bf16 [E][d]. Writes ids int32 [B][k_aux],      */
/*           g1 fp32 [B][k], g2 fp32 [B][k_aux] and, if non-NULL, the router  */
/*           logits fp32 [2B][E] (fp32 dot products of the bf16 rows).        */
/* dispatch: copies, for every expert e, the primary rows of the tokens that  */
/*           chose it (first k choices), in token order, into rows 0.. of    */
/*           xe[e] = xe + e*128*d, and the auxiliary rows (all k_aux choices) */
/*           into rows 64.. ; writes the row of every (token, choice):        */
/*           slot1 [B][k] (0..63), slot2 [B][k_aux] (64..127), and counts     */
/*           [E][2] if non-NULL. ids must be distinct per token; an id        */
/*           outside [0, E) sets DF_DEVERR_BLOCK in err_flag and is skipped.  */
/*           Rows of xe past the counts are left as they were (each output    */
/*           row of a projection depends only on its own input row).          */
/* combine:  y[f*B + t] = sum_j g_f[t][j] * ye[ids[t][j]][slot_f[t][j]]       */
/*           (+ residual[f*B + t]) in fp32, stored bf16; ye bf16 [E][128][d]. */
/* ------------------------------------------------------------------------ */
df_status dualflow_moe_route(const void* x, int64_t ldx, int B, int d, const void* w_router,
                             int E, int k, int k_aux, int32_t* ids, float* g1, float* g2,
                             float* logits, void* stream);
df_status dualflow_moe_dispatch(const void* x, int64_t ldx, int B, int d, const int32_t* ids,
                                int E, int k, int k_aux, void* xe, int32_t* slot1,
                                int32_t* slot2, int32_t* counts, int32_t* err_flag,
                                void* stream);
df_status dualflow_moe_combine(const void* ye, const int32_t* ids, const float* g1,
                               const float* g2, const int32_t* slot1, const int32_t* slot2,
                               int B, int d, int E, int k, int k_aux, const void* residual,
                               int64_t ldr, void* y, int64_t ldy, int32_t* err_flag,
                               void* stream);

/* ------------------------------------------------------------------------ */
/* Mixture head: the mixed next-token distribution of both flows.            */
/*                                                                           */
/* Page "Sintesi Tecnica: Dual-Flow Transformers", section "Meccanismi        */
/* Chiave" (mixture objective): p_mix = alpha p1 + (1 - alpha) p2, the       */
/* weight alpha set by the primary distribution's confidence (collision      */
/* probability) and keeping the primary at least half of the mixture. The    */
/* map is not printed; this library reads it as                               */
/*   alpha_b = 1/2 + 1/2 * sum_v p1[b][v]^2   (in [1/2, 1]).                  */
/* logits : [2B][V] row stride ld (0 = V), dtype DF_BF16 or DF_FP32; rows     */
/*          0..B-1 primary, B..2B-1 auxiliary (the grouped LM-head           */
/*          projection of both flows' final hidden states, one shared         */
/*          output matrix); p1/p2 = softmax of the rows, fp32 arithmetic.      */
/* p_mix  : fp32 [B][V] row stride ldp (0 = V), written.                     */
/* alpha  : fp32 [B] written, or NULL. alpha reads only the primary rows, so  */
/*          it is bit-identical for any auxiliary logits (NaN included).      */
/* Supported: V % 8 == 0; ld % 8 == 0, ldp % 4 == 0; logits and p_mix        */
/* 16-byte aligned. One kernel launch (thread-block clusters of              */
/* dualflow_mixture_head_slices(B, V) CTAs per sequence); no workspace.      */
/* ------------------------------------------------------------------------ */
df_status dualflow_mixture_head(const void* logits, int64_t ld, int B, int V, int dtype,
                                float* p_mix, int64_t ldp, float* alpha, void* stream);
int dualflow_mixture_head_slices(int B, int V);

/* ------------------------------------------------------------------------ */
/* Row RMS normalisation (layer step, pre-attention and pre-MLP).            */
/*                                                                           */
/* y[r][:] = x[r][:] / sqrt(mean(x[r][:]^2) + eps) * gain[:] (gain NULL = 1), */
/* fp32 arithmetic, bf16 in and out. The pages name no normalisation; the    */
/* layer step reads the "Dense LLaMA" family of the summary's "Contributi    */
/* Chiave" as pre-norm RMSNorm. cols % 8 == 0; rows 16-byte aligned.          */
/* ------------------------------------------------------------------------ */
df_status dualflow_rmsnorm(const void* x, int64_t ldx, const void* gain, void* y, int64_t ldy,
                           int rows, int cols, float eps, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* DUALFLOW_H */
