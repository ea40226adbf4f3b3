"""Seeded synthetic inputs for the Dual-Flow decode step.

This module only draws random numbers and lays them out (paged cache,
block tables, lengths). It holds none of the method's arithmetic, so both the
CUDA path and the fp64 oracle can be fed from it. All draws use a CPU
``torch.Generator`` seeded with the workload's seed, in float32, then rounded
to the workload dtype (round-to-nearest-even for bf16), so that every
consumer sees bit-identical host values.

Workloads (the decode-step shapes studied for the method):

* ``tiny``  -- B 1, 2 heads (MHA), head_dim 64, fp32, cache 128 tokens before
  the step, one primary append, then attention over 129 tokens.
* ``mha``   -- B 32, 32 heads (MHA), head_dim 128, bf16, every sequence 2048.
* ``gqa``   -- B 64, 32 query heads per flow on 8 KV heads, head_dim 128, bf16,
  lengths uniform in [1024, 8192], 64-token pages in a random block table.
* ``long``  -- B 8, 32/8 heads, head_dim 128, bf16, lengths uniform in
  [32768, 131072], identity block table (split over the sequence needed).
* ``prefill`` -- primary prefill of 16 fresh prompts of 4096 tokens (the
  layer workload's cache length), 32/8 heads, head_dim 128, bf16, 64-token
  pages in a random block table; auxiliary query at each last position.
* ``layer`` -- full decoder layer at one generated position: d_model 4096,
  32/8 heads, head_dim 128, SwiGLU width 14336, bf16 weights ~ N(0, 0.02),
  B 64 per flow (M = 128 rows), cache 4096 tokens before the step.

Value distributions: K1, V1, Q1, Q2raw, new K/V, hidden states ~ N(0, 1);
a_ℓ, b_ℓ, c_ℓ ~ N(0, 0.1) (standard deviation 0.1); weights ~ N(0, 0.02).
"""

from __future__ import annotations

import dataclasses
import math
from typing import Optional

import torch

BLOCK_SIZE = 64


@dataclasses.dataclass(frozen=True)
class AttnWorkload:
    name: str
    B: int
    Hq: int
    Hkv: int
    D: int
    dtype: str                 # "fp32" or "bf16"
    len_lo: int                # attended length range (inclusive) ...
    len_hi: int                # ... equal bounds = uniform lengths
    random_table: bool = False
    append: bool = False       # cache holds L tokens, append one, attend L + 1
    seed: int = 0

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "fp32" else torch.bfloat16


@dataclasses.dataclass(frozen=True)
class LayerWorkload:
    name: str
    B: int
    d_model: int
    Hq: int
    Hkv: int
    D: int
    F: int
    cache_len: int             # tokens in the cache before the step
    seed: int = 5
    coupled_mlp: bool = True   # b, c ~ N(0, 0.1); False -> b = c = 0


@dataclasses.dataclass(frozen=True)
class MixtureWorkload:
    """Mixture head: grouped LM-head projection of both flows' final hidden
    states (one shared output matrix) and the mixed next-token distribution."""
    name: str
    B: int          # sequences per flow (2B rows in the projection)
    d_model: int
    V: int          # vocabulary (multiple of 128)
    seed: int = 6


@dataclasses.dataclass(frozen=True)
class PrefillWorkload:
    """Primary prefill of prompt chunks (one layer's attention), with the
    auxiliary query at each chunk's last position."""
    name: str
    B: int
    Hq: int
    Hkv: int
    D: int
    len_lo: int                # chunk length range (inclusive)
    len_hi: int
    ctx_lo: int = 0            # tokens already cached before the chunk
    ctx_hi: int = 0
    random_table: bool = True
    seed: int = 8


@dataclasses.dataclass(frozen=True)
class MoEWorkload:
    """MoE MLP block of both flows with router replay (one decode step)."""
    name: str
    B: int          # tokens per flow
    d_model: int
    F: int          # expert SwiGLU width
    E: int          # experts
    k: int          # primary fan-out
    k_aux: int      # auxiliary fan-out (k_aux = k: router replay proper)
    seed: int = 7


WORKLOADS = {
    "tiny": AttnWorkload("tiny", 1, 2, 2, 64, "fp32", 128, 128, append=True, seed=1),
    "mha": AttnWorkload("mha", 32, 32, 32, 128, "bf16", 2048, 2048, seed=2),
    "gqa": AttnWorkload("gqa", 64, 32, 8, 128, "bf16", 1024, 8192, random_table=True, seed=3),
    "long": AttnWorkload("long", 8, 32, 8, 128, "bf16", 32768, 131072, seed=4),
    "layer": LayerWorkload("layer", 64, 4096, 32, 8, 128, 14336, 4096, seed=5),
    "mixture": MixtureWorkload("mixture", 64, 4096, 32000, seed=6),
    "moe": MoEWorkload("moe", 64, 2048, 5632, 8, 2, 2, seed=7),
    "prefill": PrefillWorkload("prefill", 16, 32, 8, 128, 4096, 4096, seed=8),
}


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


def _randn(g, shape, std=1.0, dtype=torch.bfloat16, chunk_rows: Optional[int] = None):
    """N(0, std) in float32, rounded to ``dtype``; drawn in row chunks of the
    leading dimension to bound host memory (the chunking is part of the
    recipe, so values are reproducible)."""
    shape = tuple(int(s) for s in shape)
    out = torch.empty(shape, dtype=dtype)
    if chunk_rows is None or shape[0] <= chunk_rows:
        t = torch.randn(shape, generator=g, dtype=torch.float32)
        if std != 1.0:
            t.mul_(std)
        out.copy_(t)
        return out
    for r0 in range(0, shape[0], chunk_rows):
        r1 = min(shape[0], r0 + chunk_rows)
        t = torch.randn((r1 - r0,) + shape[1:], generator=g, dtype=torch.float32)
        if std != 1.0:
            t.mul_(std)
        out[r0:r1].copy_(t)
    return out


def make_lengths(g, B, lo, hi):
    if lo == hi:
        return torch.full((B,), lo, dtype=torch.int32)
    return torch.randint(lo, hi + 1, (B,), generator=g, dtype=torch.int64).to(torch.int32)


def make_block_table(g, capacities, block_size=BLOCK_SIZE, random_table=False):
    """Block table for sequences holding ``capacities[b]`` tokens.

    Sequence b gets ceil(capacities[b] / block_size) pages. Identity layout:
    pages are numbered consecutively sequence after sequence. Random layout:
    the same pages are assigned in the order of a seeded permutation of all
    page numbers. Unused table entries are -1. Returns (table [B, max_blocks]
    int32, num_blocks).
    """
    nblk = [max(1, math.ceil(int(c) / block_size)) for c in capacities]
    total = sum(nblk)
    maxb = max(nblk)
    order = torch.randperm(total, generator=g).to(torch.int32) if random_table \
        else torch.arange(total, dtype=torch.int32)
    table = torch.full((len(nblk), maxb), -1, dtype=torch.int32)
    k = 0
    for b, n in enumerate(nblk):
        table[b, :n] = order[k:k + n]
        k += n
    return table, total


def make_attn_inputs(w: AttnWorkload, seed: Optional[int] = None, B: Optional[int] = None,
                     lengths=None):
    """Host tensors for one decode-attention step of workload ``w``.

    Returns a dict with: q1, q2raw [B, Hq, D]; a [Hq, D]; k_cache, v_cache
    [num_blocks, Hkv, 64, D]; block_table [B, max_blocks] int32; seqlens [B]
    int32 (attended length after any append); positions [B] int32 (append
    slot = cache length before the step) and k_new, v_new [B, Hkv, D] when the
    workload includes the append. ``lengths`` (optional) replaces the drawn
    lengths (edge-case tests).
    """
    g = _gen(w.seed if seed is None else seed)
    dt = w.torch_dtype
    if lengths is not None:
        lens = torch.as_tensor(lengths, dtype=torch.int32)
        B = lens.numel()
    else:
        B = w.B if B is None else B
        lens = make_lengths(g, B, w.len_lo, w.len_hi)
    if w.append:
        positions = lens.clone()
        seqlens = lens + 1
    else:
        positions = None
        seqlens = lens
    table, nblocks = make_block_table(g, seqlens.tolist(), BLOCK_SIZE, w.random_table)
    q1 = _randn(g, (B, w.Hq, w.D), dtype=dt)
    q2raw = _randn(g, (B, w.Hq, w.D), dtype=dt)
    a = _randn(g, (w.Hq, w.D), std=0.1, dtype=dt)
    kc = _randn(g, (nblocks, w.Hkv, BLOCK_SIZE, w.D), dtype=dt, chunk_rows=1024)
    vc = _randn(g, (nblocks, w.Hkv, BLOCK_SIZE, w.D), dtype=dt, chunk_rows=1024)
    out = dict(q1=q1, q2raw=q2raw, a=a, k_cache=kc, v_cache=vc, block_table=table,
               seqlens=seqlens, num_blocks=nblocks, B=B, Hq=w.Hq, Hkv=w.Hkv, D=w.D,
               dtype=w.dtype)
    if w.append:
        out["positions"] = positions
        out["k_new"] = _randn(g, (B, w.Hkv, w.D), dtype=dt)
        out["v_new"] = _randn(g, (B, w.Hkv, w.D), dtype=dt)
    return out


def make_layer_inputs(w: LayerWorkload, seed: Optional[int] = None, B: Optional[int] = None,
                      with_cache: bool = True):
    """Host tensors for one decoder-layer step of workload ``w`` (bf16).

    x1, x2 [B, d_model]; w_qkv [(Hq + 2 Hkv) D, d_model]; w_o [d_model, Hq D];
    w_gu [2F, d_model] (gate rows, then up rows); w_down [d_model, F];
    a [Hq, D]; b [F]; c [d_model]; paged cache of cache_len + 1 capacity
    (cache_len valid tokens); positions [B] = cache_len.
    """
    g = _gen(w.seed if seed is None else seed)
    B = w.B if B is None else B
    bf = torch.bfloat16
    qd, kvd = w.Hq * w.D, w.Hkv * w.D
    x1 = _randn(g, (B, w.d_model), dtype=bf)
    x2 = _randn(g, (B, w.d_model), dtype=bf)
    w_qkv = _randn(g, (qd + 2 * kvd, w.d_model), std=0.02, dtype=bf, chunk_rows=2048)
    w_o = _randn(g, (w.d_model, qd), std=0.02, dtype=bf, chunk_rows=2048)
    w_gu = _randn(g, (2 * w.F, w.d_model), std=0.02, dtype=bf, chunk_rows=2048)
    w_down = _randn(g, (w.d_model, w.F), std=0.02, dtype=bf, chunk_rows=2048)
    a = _randn(g, (w.Hq, w.D), std=0.1, dtype=bf)
    if w.coupled_mlp:
        b = _randn(g, (w.F,), std=0.1, dtype=bf)
        c = _randn(g, (w.d_model,), std=0.1, dtype=bf)
    else:
        b = torch.zeros(w.F, dtype=bf)
        c = torch.zeros(w.d_model, dtype=bf)
    out = dict(x1=x1, x2=x2, w_qkv=w_qkv, w_o=w_o, w_gu=w_gu, w_down=w_down, a=a, b=b, c=c,
               B=B, d_model=w.d_model, Hq=w.Hq, Hkv=w.Hkv, D=w.D, F=w.F)
    positions = torch.full((B,), w.cache_len, dtype=torch.int32)
    table, nblocks = make_block_table(g, [w.cache_len + 1] * B, BLOCK_SIZE, False)
    out.update(positions=positions, block_table=table, num_blocks=nblocks)
    if with_cache:
        out["k_cache"] = _randn(g, (nblocks, w.Hkv, BLOCK_SIZE, w.D), dtype=bf, chunk_rows=1024)
        out["v_cache"] = _randn(g, (nblocks, w.Hkv, BLOCK_SIZE, w.D), dtype=bf, chunk_rows=1024)
    return out


def to_numpy_f32(t: torch.Tensor):
    """Exact widening of a host bf16/fp32 tensor to a float32 numpy array."""
    return t.detach().to("cpu").to(torch.float32).numpy()


def make_mixture_inputs(w: MixtureWorkload, seed: Optional[int] = None):
    """Host tensors for one mixture-head step of workload ``w`` (bf16):
    h1, h2 [B, d_model] ~ N(0, 1) (final hidden states of the two flows) and
    the shared output matrix w_head [V, d_model] ~ N(0, 0.02), so logits have
    a standard deviation of about 0.02 sqrt(d_model) (1.3 at d_model 4096)."""
    g = _gen(w.seed if seed is None else seed)
    h1 = _randn(g, (w.B, w.d_model))
    h2 = _randn(g, (w.B, w.d_model))
    w_head = _randn(g, (w.V, w.d_model), std=0.02, chunk_rows=2048)
    return dict(h1=h1, h2=h2, w_head=w_head, B=w.B, d_model=w.d_model, V=w.V)


def make_moe_inputs(w: MoEWorkload, seed: Optional[int] = None):
    """Host tensors for one MoE block step of workload ``w`` (bf16): x [2B, d]
    ~ N(0, 1) (primary rows, then auxiliary rows; also the residual), the
    shared router w_router [E, d] ~ N(0, 0.05) (router logits of standard
    deviation ~2.3 at d = 2048), w_gu [E, 2F, d] and w_down [E, d, F]
    ~ N(0, 0.02)."""
    g = _gen(w.seed if seed is None else seed)
    x = _randn(g, (2 * w.B, w.d_model))
    w_router = _randn(g, (w.E, w.d_model), std=0.05)
    w_gu = torch.empty((w.E, 2 * w.F, w.d_model), dtype=torch.bfloat16)
    w_down = torch.empty((w.E, w.d_model, w.F), dtype=torch.bfloat16)
    for e in range(w.E):
        w_gu[e] = _randn(g, (2 * w.F, w.d_model), std=0.02, chunk_rows=2048)
        w_down[e] = _randn(g, (w.d_model, w.F), std=0.02, chunk_rows=2048)
    return dict(x=x, w_router=w_router, w_gu=w_gu, w_down=w_down, B=w.B, d_model=w.d_model,
                F=w.F, E=w.E, k=w.k, k_aux=w.k_aux)


def make_prefill_inputs(w: PrefillWorkload, seed: Optional[int] = None, lengths=None, ctx=None):
    """Host tensors for one prefill call of workload ``w`` (bf16).

    Chunk lengths n_b ~ U{len_lo..len_hi} and cached prefixes c_b ~
    U{ctx_lo..ctx_hi} (or the given ``lengths`` / ``ctx``); the block table
    covers c_b + n_b tokens per sequence. Returns q1 [T, Hq, D], k_new, v_new
    [T, Hkv, D], q2raw [B, Hq, D], a [Hq, D] (std 0.1), k_cache, v_cache
    [num_blocks, Hkv, 64, D] (every slot drawn; the prefix slots are the
    cached tokens), block_table, cu_seqlens [B + 1], ctx_lens [B] (int32),
    max_q_len and max_seqlen.
    """
    g = _gen(w.seed if seed is None else seed)
    dt = torch.bfloat16
    if lengths is not None:
        lens = torch.as_tensor(lengths, dtype=torch.int32)
    else:
        lens = make_lengths(g, w.B, w.len_lo, w.len_hi)
    B = lens.numel()
    if ctx is not None:
        ctx_lens = torch.as_tensor(ctx, dtype=torch.int32)
    elif w.ctx_hi > 0:
        ctx_lens = make_lengths(g, B, w.ctx_lo, w.ctx_hi)
    else:
        ctx_lens = torch.zeros(B, dtype=torch.int32)
    caps = (ctx_lens + lens).tolist()
    table, nblocks = make_block_table(g, caps, BLOCK_SIZE, w.random_table)
    T = int(lens.sum())
    cu = torch.zeros(B + 1, dtype=torch.int32)
    cu[1:] = torch.cumsum(lens, 0).to(torch.int32)
    q1 = _randn(g, (T, w.Hq, w.D), dtype=dt, chunk_rows=4096)
    k_new = _randn(g, (T, w.Hkv, w.D), dtype=dt, chunk_rows=4096)
    v_new = _randn(g, (T, w.Hkv, w.D), dtype=dt, chunk_rows=4096)
    q2raw = _randn(g, (B, w.Hq, w.D), dtype=dt)
    a = _randn(g, (w.Hq, w.D), std=0.1, dtype=dt)
    kc = _randn(g, (nblocks, w.Hkv, BLOCK_SIZE, w.D), dtype=dt, chunk_rows=1024)
    vc = _randn(g, (nblocks, w.Hkv, BLOCK_SIZE, w.D), dtype=dt, chunk_rows=1024)
    return dict(q1=q1, k_new=k_new, v_new=v_new, q2raw=q2raw, a=a, k_cache=kc, v_cache=vc,
                block_table=table, cu_seqlens=cu, ctx_lens=ctx_lens, num_blocks=nblocks, B=B,
                T=T, Hq=w.Hq, Hkv=w.Hkv, D=w.D, max_q_len=int(lens.max()),
                max_seqlen=int(max(caps)))
