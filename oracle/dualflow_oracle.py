"""Plain fp64 CPU oracle for the Dual-Flow Transformer decode step.

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` may import or run this module.
It shares no code, header, table or helper with the CUDA library, and it
imports nothing from the product package.

Every function follows a definition on the pages describing the method
(arXiv 2608.12385, "Dual-Flow Transformers"), cited as page title + section:

* "Sintesi Tecnica: Dual-Flow Transformers" (gist.science, Italian technical
  summary) -- sections "Architettura Core", "Meccanismi Chiave" and
  "Costi di Inferenza vs. Addestramento".
* "プライマリパスとデコード処理を分離する Dual-Flow Transformers" (jumtra.com news
  summary) -- section "提案手法の詳細".

The pages give the method in prose only: no formulas for the coupling
vectors, no listings, no worked numbers. Where they leave a step open the
oracle takes the plainest reading; each reading is named in the docstring
of the function that takes it:

* Query coupling  q2 = q2raw + a ⊙ q1  (additive, element-wise, one way).
  Pinned only by its special cases (a = 0; q2raw = 0 with a = 1).
  The general formula is a reading: PARITY UNPINNED against the pages.
* MLP coupling    h2 += b ⊙ h1 ;  m2 += c ⊙ m1  (same additive form).
  PARITY UNPINNED against the pages beyond the b = c = 0 reduction.
* Prefill         the primary flow's causal attention over the prompt,
  writing the cache; the auxiliary query only at the last prompt position.
  Both are the pages' statements; the chunked form (a cache that already
  holds a prefix) is the plain extension of the causal mask.
* Layer step      pre-attention and pre-MLP RMSNorm (unit gain, eps 1e-5),
  residual adds, SwiGLU MLP, no positional rotation.
  PARITY UNPINNED against the pages (the pages name no norm, no MLP form);
  the wiring of that reading (which tensor feeds which step) is pinned by a
  hand-derived worked example with every intermediate in closed form.
* MoE router replay  the auxiliary flow uses the primary router's expert
  set with its own gate weights (the pages' statement); the router matrix is
  shared, gates are the softmax of each flow's router logits over the set,
  experts are SwiGLU MLPs, and with a larger auxiliary fan-out the auxiliary
  set is the primary ranking's top k_aux. Those details are readings:
  PARITY UNPINNED against the pages beyond the invariants in the tests.
* Mixture head    p_mix = alpha p1 + (1 - alpha) p2 is the pages' formula;
  the map from the primary's collision probability to alpha is a reading,
  alpha = 1/2 + 1/2 sum(p1^2). Pinned by its limits (uniform and one-hot
  primary) and invariants; the map itself is PARITY UNPINNED against the
  pages beyond those limits.

Attention itself (scores, softmax, weighted sum of V) is the textbook
definition written out, so it is pinned by brute force, closed forms and a
library cross-check in the tests.

All arithmetic is float64. Inputs may be float32 or float64 numpy arrays
(bf16 tensors are widened to float32 exactly by the caller); they are widened
to float64 before any arithmetic.
"""

from __future__ import annotations

import math

import numpy as np

F64 = np.float64

# Largest finite bf16 value: (2 - 2**-7) * 2**127.
_BF16_MAX = (2.0 - 2.0 ** -7) * 2.0 ** 127


def bf16_round(x):
    """Round float64 values to the nearest bfloat16 value, ties to even.

    bfloat16 keeps 8 significant bits (1 implicit + 7 stored) and the float32
    exponent range. The result is returned as float64 (exactly representable).
    Used only where the CUDA path stores a bf16 tensor between two steps, so
    that both sides round at the same interfaces.
    """
    x = np.asarray(x, dtype=F64)
    out = np.empty_like(x)
    finite = np.isfinite(x)
    xf = np.where(finite, x, 0.0)
    m, e = np.frexp(xf)  # xf = m * 2**e with 0.5 <= |m| < 1
    normal = np.abs(xf) >= 2.0 ** -126
    # normal range: keep 8 significant bits
    r_norm = np.ldexp(np.rint(np.ldexp(m, 8)), e - 8)
    # subnormal range: fixed spacing 2**-133
    r_sub = np.rint(xf * 2.0 ** 133) * 2.0 ** -133
    r = np.where(normal, r_norm, r_sub)
    r = np.where(np.abs(r) > _BF16_MAX, np.copysign(np.inf, r), r)
    out[...] = np.where(finite, r, x)
    return out


def couple_query(q1, q2raw, a):
    """Auxiliary query built from the primary query through the vector a_ℓ.

    Page "Sintesi Tecnica: Dual-Flow Transformers", section "Meccanismi Chiave"
    (asymmetric shared-KV attention; lightweight coupling): the auxiliary query
    Q2 is coupled to the primary query Q1 through a learned per-layer vector
    a_ℓ, and information flows only from the primary to the auxiliary flow.
    The pages print no formula. Reading taken: Q2 = Q2raw + a_ℓ ⊙ Q1,
    element-wise, with a_ℓ of shape [Hq, D] shared by every sequence.
    With a = None, q2raw is taken as the already coupled Q2.

    q1, q2raw: [B, Hq, D]; a: [Hq, D] or None. Returns [B, Hq, D] float64.
    """
    q2 = np.asarray(q2raw, dtype=F64)
    if a is None:
        return q2.copy()
    return q2 + np.asarray(a, dtype=F64)[None, :, :] * np.asarray(q1, dtype=F64)


def gather_kv(cache, block_table, b, g, length, block_size):
    """Rows 0..length-1 of KV head g of sequence b from a paged cache.

    The single persistent primary cache ("Architettura Core": only the
    primary flow writes it) is stored in fixed-size pages:
    cache[num_blocks][Hkv][block_size][D]; token j of sequence b lives in page
    block_table[b][j // block_size], slot j % block_size.
    Returns a float64 [length, D] array.
    """
    j = np.arange(length)
    pages = np.asarray(block_table)[b, j // block_size]
    slots = j % block_size
    return np.asarray(cache[pages, g, slots, :], dtype=F64)


def attn_weights(q, k, scale):
    """Softmax attention weights of query rows q [R, D] over keys k [L, D].

    p[r, j] = exp(s[r, j] - max_j s[r, :]) / sum_j exp(s[r, j] - max_j s[r, :]),
    s = scale * q k^T. Plain definition; float64.
    """
    s = scale * (np.asarray(q, dtype=F64) @ np.asarray(k, dtype=F64).T)
    s = s - s.max(axis=1, keepdims=True)
    e = np.exp(s)
    return e / e.sum(axis=1, keepdims=True)


def decode_attn(q1, q2raw, a, k_cache, v_cache, block_table, seqlens, scale=None,
                block_size=None):
    """One decode step of asymmetric shared-KV attention for both flows.

    Page "Sintesi Tecnica: Dual-Flow Transformers", section "Meccanismi
    Chiave": the primary flow runs ordinary causal self-attention; the
    auxiliary query Q2 (coupled to Q1, see ``couple_query``) attends to the
    primary flow's keys and values K1, V1 -- the same cache, no K/V of its own.
    At a decode position the causal mask admits every cached token, so for
    sequence b, query head h and KV head g = h // (Hq / Hkv):

        O_f[b, h] = softmax(scale * q_f K1[b, g]^T) V1[b, g],  f in {1, 2},

    over the first seqlens[b] tokens. scale defaults to 1/sqrt(D).

    q1, q2raw: [B, Hq, D]; a: [Hq, D] or None; caches [num_blocks, Hkv, bs, D];
    block_table [B, max_blocks]; seqlens [B] (each >= 1).
    Returns (o1, o2) as float64 [B, Hq, D]; o2 is None when q2raw is None.
    """
    q1 = np.asarray(q1, dtype=F64)
    B, Hq, D = q1.shape
    Hkv = k_cache.shape[1]
    if block_size is None:
        block_size = k_cache.shape[2]
    if Hq % Hkv != 0:
        raise ValueError("Hq must be a multiple of Hkv")
    G = Hq // Hkv
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    q2 = None if q2raw is None else couple_query(q1, q2raw, a)
    o1 = np.zeros((B, Hq, D), dtype=F64)
    o2 = None if q2 is None else np.zeros((B, Hq, D), dtype=F64)
    for b in range(B):
        L = int(seqlens[b])
        if L < 1:
            raise ValueError("every sequence attends to at least one token")
        for g in range(Hkv):
            K = gather_kv(k_cache, block_table, b, g, L, block_size)
            V = gather_kv(v_cache, block_table, b, g, L, block_size)
            heads = slice(g * G, (g + 1) * G)
            o1[b, heads] = attn_weights(q1[b, heads], K, scale) @ V
            if q2 is not None:
                o2[b, heads] = attn_weights(q2[b, heads], K, scale) @ V
    return o1, o2


def kv_append(k_new, v_new, k_cache, v_cache, block_table, positions, block_size=None):
    """Primary-only append of this step's K1/V1 rows to the paged cache.

    Page "Sintesi Tecnica: Dual-Flow Transformers", section "Architettura
    Core": only the primary flow writes the persistent KV cache; the auxiliary
    flow never writes it. Token position p = positions[b] of sequence b goes to
    page block_table[b][p // block_size], slot p % block_size, for every KV
    head. A plain element copy (no arithmetic): returns new cache arrays with
    the input dtype, leaving every other element untouched.
    """
    kc = np.array(k_cache, copy=True)
    vc = np.array(v_cache, copy=True)
    if block_size is None:
        block_size = kc.shape[2]
    B = k_new.shape[0]
    for b in range(B):
        p = int(positions[b])
        page = int(block_table[b][p // block_size])
        kc[page, :, p % block_size, :] = k_new[b]
        vc[page, :, p % block_size, :] = v_new[b]
    return kc, vc


def prefill(q1, k_new, v_new, k_cache, v_cache, block_table, cu_seqlens, ctx_lens=None,
            q2raw=None, a=None, scale=None, block_size=None):
    """Prompt processing of the primary flow, then the auxiliary query at the
    last prompt position.

    Page "Sintesi Tecnica: Dual-Flow Transformers", section "Architettura
    Core": the primary flow is a standard causal Transformer that processes
    the whole prompt and writes the persistent KV cache; the auxiliary flow is
    skipped while the prompt is processed and switched on only at the last
    prompt position (to predict the first continuation token). Section
    "Costi di Inferenza vs. Addestramento": prefill costs what a standard
    Transformer's does. The page "プライマリパスとデコード処理を分離する
    Dual-Flow Transformers", section "提案手法の詳細", says the same (the auxiliary
    flow is skipped during prompt processing and starts at the final position).

    Sequence b holds the prompt tokens t in [cu_seqlens[b], cu_seqlens[b+1]);
    its cache already holds ctx_lens[b] tokens (0 for a fresh prompt), so
    token i of the chunk sits at position p = ctx_lens[b] + i. Steps:

    1. append: the chunk's K1/V1 rows go to positions ctx_lens[b] + i of the
       paged cache (the ``kv_append`` rule, one position per token);
    2. primary attention, causal: the query at position p attends to cache
       positions j <= p,
           O1[t, h] = softmax_j(scale * q1[t, h] . k_j) V, j in [0, p];
    3. auxiliary query at the last position P = ctx_lens[b] + n_b - 1 only,
       coupled to that position's primary query (``couple_query``) and
       attending to positions j <= P of the same cache:
           O2[b, h] = softmax_j(scale * q2[b, h] . k_j) V.

    q1 [T, Hq, D]; k_new, v_new [T, Hkv, D]; q2raw [B, Hq, D] or None;
    a [Hq, D] or None; caches [num_blocks, Hkv, bs, D]; block_table
    [B, max_blocks]; cu_seqlens [B + 1] with every chunk non-empty.
    Returns (o1 float64 [T, Hq, D], o2 float64 [B, Hq, D] or None,
    k_cache, v_cache) -- the caches as new arrays of the input dtype.
    """
    q1 = np.asarray(q1, dtype=F64)
    T, Hq, D = q1.shape
    Hkv = k_cache.shape[1]
    if block_size is None:
        block_size = k_cache.shape[2]
    if Hq % Hkv != 0:
        raise ValueError("Hq must be a multiple of Hkv")
    G = Hq // Hkv
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    cu = [int(x) for x in cu_seqlens]
    B = len(cu) - 1
    ctx = [0] * B if ctx_lens is None else [int(x) for x in ctx_lens]
    if cu[0] != 0 or cu[-1] != T or any(cu[b + 1] - cu[b] < 1 for b in range(B)):
        raise ValueError("cu_seqlens must split the T tokens into non-empty chunks")

    # 1. primary-only cache write, one position per prompt token (the
    #    ``kv_append`` rule: page table[b][p // bs], slot p % bs, all KV heads)
    kc = np.array(k_cache, copy=True)
    vc = np.array(v_cache, copy=True)
    table = np.asarray(block_table)
    for b in range(B):
        for i in range(cu[b + 1] - cu[b]):
            t, p = cu[b] + i, ctx[b] + i
            page = int(table[b][p // block_size])
            kc[page, :, p % block_size, :] = k_new[t]
            vc[page, :, p % block_size, :] = v_new[t]

    o1 = np.zeros((T, Hq, D), dtype=F64)
    o2 = None if q2raw is None else np.zeros((B, Hq, D), dtype=F64)
    for b in range(B):
        n = cu[b + 1] - cu[b]
        L = ctx[b] + n
        pos = ctx[b] + np.arange(n)                      # position of each query row
        keep = np.arange(L)[None, :] <= pos[:, None]     # causal mask [n, L]
        last = cu[b + 1] - 1
        for g in range(Hkv):
            K = gather_kv(kc, block_table, b, g, L, block_size)
            V = gather_kv(vc, block_table, b, g, L, block_size)
            for h in range(g * G, (g + 1) * G):
                # 2. masked softmax over keys j <= p for every query row
                s = scale * (q1[cu[b]:cu[b + 1], h, :] @ K.T)
                s = np.where(keep, s, -np.inf)
                s = s - s.max(axis=1, keepdims=True)
                e = np.exp(s)
                o1[cu[b]:cu[b + 1], h, :] = (e / e.sum(axis=1, keepdims=True)) @ V
            if q2raw is not None:
                # 3. auxiliary query of the last prompt position, every key
                heads = slice(g * G, (g + 1) * G)
                q2 = couple_query(q1[last:last + 1, heads, :],
                                  np.asarray(q2raw, dtype=F64)[b:b + 1, heads, :],
                                  None if a is None else np.asarray(a, dtype=F64)[heads])
                o2[b, heads] = attn_weights(q2[0], K, scale) @ V
    return o1, o2, kc, vc


def grouped_proj(x, w, m_primary, n_aux=None):
    """Both flows' rows multiplied by the same shared weight matrix.

    Pages "Sintesi Tecnica: Dual-Flow Transformers" ("Architettura Core":
    both flows share all attention, MLP and output matrices; "Costi di
    Inferenza": grouped execution reads the unique weights once) and
    "プライマリパスとデコード処理を分離する Dual-Flow Transformers"
    ("提案手法の詳細": shared matrices allow grouped execution).

    y = x w^T with x = [primary rows; auxiliary rows] of shape [M, K] and
    w of shape [N, K]. Auxiliary rows (index >= m_primary) are defined only
    for columns < n_aux (e.g. the auxiliary flow needs only the Q columns of
    the fused QKV weight because it never writes K/V); the other auxiliary
    entries are returned as NaN ("not computed").
    """
    y = np.asarray(x, dtype=F64) @ np.asarray(w, dtype=F64).T
    if n_aux is not None and n_aux < y.shape[1]:
        y[m_primary:, n_aux:] = np.nan
    return y


def silu(x):
    """SiLU(x) = x * sigmoid(x) = x / (1 + exp(-x)), float64."""
    x = np.asarray(x, dtype=F64)
    return x / (1.0 + np.exp(-x))


def swiglu_couple(gate_up, F, m_primary, b=None):
    """SwiGLU MLP intermediate with the one-way b_ℓ coupling.

    gate_up = [gate | up] of shape [M, 2F] (the fused gate/up projection).
    h = SiLU(gate) ⊙ up for every row. Page "Sintesi Tecnica", section
    "Meccanismi Chiave" (lightweight coupling at the MLP-intermediate level
    through b_ℓ, primary -> auxiliary only). Reading taken (the pages print
    no formula): auxiliary row m_primary + j gets + b ⊙ h[j], where row j is
    the primary row of the same sequence; primary rows are unchanged.
    """
    gu = np.asarray(gate_up, dtype=F64)
    h = silu(gu[:, :F]) * gu[:, F:2 * F]
    if b is not None:
        m_aux = h.shape[0] - m_primary
        h[m_primary:] = h[m_primary:] + np.asarray(b, dtype=F64)[None, :] * h[:m_aux]
    return h


def residual_couple(acc, residual, m_primary, c=None):
    """Projection output plus residual, with the one-way c_ℓ coupling.

    Page "Sintesi Tecnica", section "Meccanismi Chiave" (coupling at the
    MLP-output level through c_ℓ, primary -> auxiliary only). Reading taken:
    auxiliary row m_primary + j gets + c ⊙ acc[j] (the primary row's
    projection output, before its residual add); then every row adds its own
    residual. With c = None this is the plain residual add.
    """
    y = np.asarray(acc, dtype=F64).copy()
    if c is not None:
        m_aux = y.shape[0] - m_primary
        y[m_primary:] = y[m_primary:] + np.asarray(c, dtype=F64)[None, :] * y[:m_aux]
    if residual is not None:
        y = y + np.asarray(residual, dtype=F64)
    return y


def rmsnorm(x, gain=None, eps=1e-5):
    """Row-wise RMS normalisation: x / sqrt(mean(x^2) + eps) (* gain).

    The pages name no normalisation; the layer step reads the "Dense LLaMA"
    model family of section "Contributi Chiave" as the usual pre-norm RMSNorm.
    """
    x = np.asarray(x, dtype=F64)
    y = x / np.sqrt(np.mean(x * x, axis=1, keepdims=True) + eps)
    if gain is not None:
        y = y * np.asarray(gain, dtype=F64)[None, :]
    return y


LAYER_INTERFACES = ("xn", "qkv", "attn", "x_mid", "xn2", "h", "x_out")


def layer_step(x1, x2, w_qkv, w_o, w_gu, w_down, a, b, c, k_cache, v_cache,
               block_table, positions, Hq, Hkv, D, F, round_bf16=True, eps=1e-5,
               rounded=LAYER_INTERFACES):
    """One Dual-Flow decoder layer at one generated position, both flows.

    Composition (pages "Sintesi Tecnica", sections "Architettura Core",
    "Meccanismi Chiave", "Costi di Inferenza"): both flows go through the same
    shared weights; only the primary flow's K/V are appended to the single
    cache; both queries attend over that cache (the auxiliary one after the
    append, so it sees the current token like the primary); coupling flows
    only primary -> auxiliary through a, b, c. Readings: pre-norm RMSNorm,
    SwiGLU MLP, residual adds, no positional rotation.

    x1, x2: [B, d_model] hidden states of the primary and auxiliary flow.
    w_qkv [(Hq + 2 Hkv) D, d_model]; w_o [d_model, Hq D];
    w_gu [2F, d_model] (gate rows then up rows); w_down [d_model, F].
    positions[b]: cache length before this step (the slot the append writes).
    With round_bf16, every intermediate named in `rounded` (by default all
    the tensors a four-call layer step stores as bf16) is rounded to bf16
    here too, in the same order; an implementation that keeps an intermediate
    in fp32 (a normalised row scaled inside a GEMM epilogue instead of stored)
    is compared with that name left out.
    Returns a dict of float64 arrays (and the updated caches).
    """
    exact = lambda t: np.asarray(t, dtype=F64)  # noqa: E731
    rset = frozenset(rounded) if round_bf16 else frozenset()
    unknown = rset - frozenset(LAYER_INTERFACES)
    if unknown:
        raise ValueError("unknown interfaces %s" % sorted(unknown))
    rd = {name: (bf16_round if name in rset else exact) for name in LAYER_INTERFACES}
    x1 = np.asarray(x1, dtype=F64)
    x2 = np.asarray(x2, dtype=F64)
    B = x1.shape[0]
    X = np.concatenate([x1, x2], axis=0)
    qd, kvd = Hq * D, Hkv * D

    xn = rd["xn"](rmsnorm(X, eps=eps))
    qkv = rd["qkv"](grouped_proj(xn, w_qkv, B, n_aux=qd))
    k_new = qkv[:B, qd:qd + kvd].reshape(B, Hkv, D)
    v_new = qkv[:B, qd + kvd:qd + 2 * kvd].reshape(B, Hkv, D)
    kc, vc = kv_append(k_new, v_new, k_cache, v_cache, block_table, positions)
    seqlens = np.asarray(positions) + 1
    q1 = qkv[:B, :qd].reshape(B, Hq, D)
    q2raw = qkv[B:, :qd].reshape(B, Hq, D)
    o1, o2 = decode_attn(q1, q2raw, a, kc, vc, block_table, seqlens)
    attn = rd["attn"](np.concatenate([o1.reshape(B, qd), o2.reshape(B, qd)], axis=0))
    x_mid = rd["x_mid"](residual_couple(grouped_proj(attn, w_o, B), X, B, None))
    xn2 = rd["xn2"](rmsnorm(x_mid, eps=eps))
    h = rd["h"](swiglu_couple(grouped_proj(xn2, w_gu, B), F, B, b))
    x_out = rd["x_out"](residual_couple(grouped_proj(h, w_down, B), x_mid, B, c))
    return {
        "xn": xn, "qkv": qkv, "k_cache": kc, "v_cache": vc, "attn": attn,
        "x_mid": x_mid, "xn2": xn2, "h": h, "x_out": x_out,
    }


# ----------------------------------------------------------------- mixture head

def softmax_rows(logits):
    """Row softmax p_v = exp(l_v - max l) / sum_u exp(l_u - max l), in fp64."""
    l = np.asarray(logits, dtype=F64)
    m = l.max(axis=-1, keepdims=True)
    e = np.exp(l - m)
    return e / e.sum(axis=-1, keepdims=True)


def collision_probability(p):
    """sum_v p_v^2 per row: the chance that two independent draws from p agree
    (1 for a one-hot p, 1/V for a uniform p over V outcomes)."""
    p = np.asarray(p, dtype=F64)
    return (p * p).sum(axis=-1)


def mixture_weight(p1):
    """Weight of the primary distribution in the mixture.

    "Sintesi Tecnica: Dual-Flow Transformers", section "Meccanismi Chiave"
    (mixture objective): the weight follows the primary distribution's
    confidence, measured by its collision probability, and keeps the primary
    at least half of the mixture at inference. The map is not printed; the
    reading taken here is the plainest monotone one onto [1/2, 1]:
        alpha = 1/2 + 1/2 * sum_v p1_v^2.
    """
    return 0.5 + 0.5 * collision_probability(p1)


def mixture_head(logits, B):
    """Mixed next-token distribution of both flows.

    logits: [2B][V], primary rows 0..B-1, auxiliary rows B..2B-1 (the grouped
    LM-head projection's output; same section as `mixture_weight`):
        p1 = softmax(logits[b]), p2 = softmax(logits[B + b]),
        alpha_b = mixture_weight(p1),
        p_mix[b] = alpha_b * p1 + (1 - alpha_b) * p2.
    Returns (p_mix [B][V], alpha [B]), fp64.
    """
    l = np.asarray(logits, dtype=F64)
    p1 = softmax_rows(l[:B])
    p2 = softmax_rows(l[B:2 * B])
    alpha = mixture_weight(p1)
    return alpha[:, None] * p1 + (1.0 - alpha[:, None]) * p2, alpha


# ----------------------------------------------------------------- MoE router replay

def moe_route(x1, x2, w_router, k, k_aux=None, ids=None):
    """Expert selection and gate weights of both flows (router replay).

    "Sintesi Tecnica: Dual-Flow Transformers", section "Meccanismi Chiave"
    (router replay for MoE): the auxiliary flow reuses the set of experts that
    the primary router selected, applied with its own mixing weights; section
    "Contributi Chiave" (phase-specific MoE allocation): the two flows may
    have independent expert fan-outs. Readings taken:
      * router logits r_f = x_f W_router^T (one router matrix shared by both
        flows, like every other matrix of the model);
      * ids = the primary's top-k_aux experts by descending r_1 (ties: lower
        expert index first); the primary uses the first k of them, the
        auxiliary all k_aux (k_aux = k is router replay proper);
      * gates: softmax of each flow's own logits over its set,
        g1 = softmax(r_1[ids[:k]]), g2 = softmax(r_2[ids[:k_aux]]).
    x1, x2: [B][d]; w_router: [E][d]. Returns (ids int [B][k_aux],
    g1 [B][k], g2 [B][k_aux], r1 [B][E], r2 [B][E]), fp64.

    ids (optional, int [B][k_aux]): a selection made elsewhere, used as
    given instead of this function's own ranking. Where two logits are closer
    than the rounding of another implementation's arithmetic, several
    selections are equally correct; the gates and outputs of that selection
    are then checked with the same formulas.
    """
    k_aux = k if k_aux is None else k_aux
    w = np.asarray(w_router, dtype=F64)
    r1 = np.asarray(x1, dtype=F64) @ w.T
    r2 = np.asarray(x2, dtype=F64) @ w.T
    B, E = r1.shape
    if ids is not None:
        ids = np.asarray(ids, dtype=np.int64).reshape(B, k_aux)
    else:
        ids = np.zeros((B, k_aux), dtype=np.int64)
        for t in range(B):
            # stable sort of (-logit, index): descending logit, lower index first on ties
            order = sorted(range(E), key=lambda e: (-r1[t, e], e))
            ids[t] = order[:k_aux]
    g1 = softmax_rows(np.take_along_axis(r1, ids[:, :k], axis=1))
    g2 = softmax_rows(np.take_along_axis(r2, ids, axis=1))
    return ids, g1, g2, r1, r2


def moe_expert(x, w_gu, w_down, round_bf16=True):
    """One SwiGLU expert applied to rows x: W_down (SiLU(x W_gate^T) * (x W_up^T)),
    w_gu = [W_gate; W_up] ([2F][d]), w_down [d][F]. With round_bf16 the
    intermediate and the result are rounded to bf16, where the CUDA path
    stores bf16 tensors."""
    x = np.asarray(x, dtype=F64)
    gu = x @ np.asarray(w_gu, dtype=F64).T
    F = gu.shape[1] // 2
    h = silu(gu[:, :F]) * gu[:, F:]
    if round_bf16:
        h = bf16_round(h)  # the intermediate is stored bf16
    y = h @ np.asarray(w_down, dtype=F64).T
    return bf16_round(y) if round_bf16 else y


def moe_forward(x1, x2, w_router, w_gu, w_down, k, k_aux=None, residual1=None,
                residual2=None, round_bf16=True, ids=None):
    """MoE MLP block of both flows with router replay:
        y1[t] = sum_j g1[t][j] E_{ids[t][j]}(x1[t])       (j < k)
        y2[t] = sum_j g2[t][j] E_{ids[t][j]}(x2[t])       (j < k_aux)
    plus the residual when given, rounded once to bf16 (round_bf16).
    w_gu: [E][2F][d], w_down: [E][d][F]. Returns (y1, y2, ids, g1, g2).
    ids: an expert selection to use as given (see ``moe_route``)."""
    k_aux = k if k_aux is None else k_aux
    ids, g1, g2, _, _ = moe_route(x1, x2, w_router, k, k_aux, ids=ids)
    x1 = np.asarray(x1, dtype=F64)
    x2 = np.asarray(x2, dtype=F64)
    B, d = x1.shape
    y1 = np.zeros((B, d))
    y2 = np.zeros((B, d))
    for e in np.unique(ids):
        t1, j1 = np.nonzero(ids[:, :k] == e)
        if t1.size:
            y1[t1] += g1[t1, j1][:, None] * moe_expert(x1[t1], w_gu[e], w_down[e], round_bf16)
        t2, j2 = np.nonzero(ids == e)
        if t2.size:
            y2[t2] += g2[t2, j2][:, None] * moe_expert(x2[t2], w_gu[e], w_down[e], round_bf16)
    if residual1 is not None:
        y1 = y1 + np.asarray(residual1, dtype=F64)
    if residual2 is not None:
        y2 = y2 + np.asarray(residual2, dtype=F64)
    if round_bf16:
        y1, y2 = bf16_round(y1), bf16_round(y2)
    return y1, y2, ids, g1, g2
