"""Thin Python binding over libdualflow.so (argument marshalling only).

Tensors are torch CUDA tensors used as plain device buffers; every
computation runs inside the library's kernels. Outputs and workspaces that
the caller does not pass are allocated here with torch (device memory is
plumbing), never computed here.
"""

from __future__ import annotations

from typing import Optional

import torch

from . import _lib as L


def _lib():
    return L.load()


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else t.data_ptr()


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def dtype_code(dt: torch.dtype) -> int:
    if dt == torch.bfloat16:
        return L.DF_BF16
    if dt == torch.float32:
        return L.DF_FP32
    raise TypeError("unsupported dtype %s (bf16 or fp32)" % dt)


def _heads_view_ok(t: torch.Tensor, Hq: int, D: int) -> bool:
    return t.dim() == 3 and t.shape[1] == Hq and t.shape[2] == D and t.stride(2) == 1 \
        and t.stride(1) == D


# ----------------------------------------------------------------- attention

def decode_attn_num_splits(B, Hkv, max_seqlen, num_splits=0, block_size=64) -> int:
    return _lib().dualflow_decode_attn_num_splits(B, Hkv, max_seqlen, block_size, num_splits)


def decode_attn_num_launches(B, Hkv, max_seqlen, num_splits=0, dtype=torch.bfloat16,
                             block_size=64) -> int:
    return _lib().dualflow_decode_attn_num_launches(B, Hkv, max_seqlen, block_size, num_splits,
                                                    dtype_code(dtype))


def new_attn_workspace(B, Hq, Hkv, D, max_seqlen, num_splits=0, device="cuda"):
    """Zero-filled decode-attention workspace for these sizes (bf16 keeps the
    split-combine arrival counters in it; every completed call leaves them at
    zero, so later calls with the same sizes can reuse it)."""
    n = max(256, decode_attn_workspace_size(B, Hq, Hkv, D, max_seqlen, num_splits))
    return torch.zeros(n, dtype=torch.uint8, device=device)


def decode_attn_workspace_size(B, Hq, Hkv, D, max_seqlen, num_splits=0, block_size=64) -> int:
    return _lib().dualflow_decode_attn_workspace_size(B, Hq, Hkv, D, max_seqlen, block_size,
                                                      num_splits)


def decode_attn(q1, q2raw, a, k_cache, v_cache, block_table, seqlens, max_seqlen, *,
                o1=None, o2=None, primary_out=True, scale=0.0, num_splits=0, workspace=None,
                err_flag=None, stream=None):
    """Dual-flow decode attention; returns (o1, o2).

    q1, q2raw: [B, Hq, D] (heads contiguous; any batch stride, equal for
    both); a: [Hq, D] or None; caches [num_blocks, Hkv, 64, D]; block_table
    int32 [B, max_blocks]; seqlens int32 [B]; max_seqlen: host int.
    primary_out=False makes an auxiliary-only call (o1 not written).
    """
    B, Hq, D = q1.shape
    num_blocks, Hkv, bs, Dk = k_cache.shape
    if Dk != D or tuple(v_cache.shape) != tuple(k_cache.shape):
        raise ValueError("cache shape mismatch")
    if not _heads_view_ok(q1, Hq, D):
        raise ValueError("q1 must be [B, Hq, D] with contiguous heads")
    if q2raw is not None and (not _heads_view_ok(q2raw, Hq, D) or q2raw.stride(0) != q1.stride(0)):
        raise ValueError("q2raw must match q1's layout")
    if not (k_cache.is_contiguous() and v_cache.is_contiguous() and block_table.is_contiguous()):
        raise ValueError("caches and block table must be contiguous")
    dev = q1.device
    if primary_out and o1 is None:
        o1 = torch.empty((B, Hq, D), dtype=q1.dtype, device=dev)
    if not primary_out:
        o1 = None
    if q2raw is not None and o2 is None:
        o2 = torch.empty((B, Hq, D), dtype=q1.dtype, device=dev)
    if q2raw is None:
        o2 = None
    os_b = (o1 if o1 is not None else o2).stride(0)
    for o in (o1, o2):
        if o is not None and (not _heads_view_ok(o, Hq, D) or o.stride(0) != os_b):
            raise ValueError("outputs must be [B, Hq, D] with contiguous heads and equal strides")
    if workspace is None:
        workspace = new_attn_workspace(B, Hq, Hkv, D, max_seqlen, num_splits, dev)
    st = _lib().dualflow_decode_attn(
        _ptr(q1), _ptr(q2raw), _ptr(a), q1.stride(0), _ptr(k_cache), _ptr(v_cache),
        _ptr(block_table), block_table.shape[1], _ptr(seqlens), int(max_seqlen),
        _ptr(o1), _ptr(o2), os_b, B, Hq, Hkv, D, bs, num_blocks, float(scale),
        dtype_code(q1.dtype), int(num_splits), _ptr(workspace),
        0 if workspace is None else workspace.numel() * workspace.element_size(),
        _ptr(err_flag), _stream(stream))
    L.check("dualflow_decode_attn", st)
    return o1, o2


# ----------------------------------------------------------------- prefill

def prefill_workspace_size(B, Hq, Hkv, D, max_seqlen, block_size=64) -> int:
    return _lib().dualflow_prefill_workspace_size(B, Hq, Hkv, D, max_seqlen, block_size)


def prefill_kernel(D, T, o1, Hq) -> str:
    """The attention kernel an automatic prefill call uses for these sizes."""
    k = _lib().dualflow_prefill_kernel(D, T, _ptr(o1), o1.stride(0), Hq)
    return "tcgen05" if k == L.DF_PREFILL_KERNEL_TCGEN05 else "mma_sync"


def prefill_num_launches(with_append=True, with_aux=True) -> int:
    return _lib().dualflow_prefill_num_launches(int(bool(with_append)), int(bool(with_aux)))


def new_prefill_workspace(B, Hq, Hkv, D, max_seqlen, device="cuda"):
    """Zero-filled prefill workspace (the auxiliary step's decode counters
    start at zero and every completed call leaves them there)."""
    n = max(256, prefill_workspace_size(B, Hq, Hkv, D, max_seqlen))
    return torch.zeros(n, dtype=torch.uint8, device=device)


def prefill(q1, k_new, v_new, k_cache, v_cache, block_table, cu_seqlens, max_q_len, max_seqlen,
            *, ctx_lens=None, q2raw=None, a=None, o1=None, o2=None, scale=0.0, workspace=None,
            err_flag=None, stream=None, kernel="auto"):
    """Primary prefill of the chunks cu_seqlens describes; returns (o1, o2).

    q1 [T, Hq, D]; k_new, v_new [T, Hkv, D] (or both None when the cache
    already holds the chunk); caches [num_blocks, Hkv, 64, D]; block_table
    int32 [B, max_blocks]; cu_seqlens int32 [B + 1]; ctx_lens int32 [B] or
    None; q2raw [B, Hq, D] (auxiliary query of each last prompt position) or
    None; a [Hq, D] or None. max_q_len, max_seqlen: host bounds.
    kernel: "auto", "mma_sync" or "tcgen05" (the attention kernel).
    """
    kcode = {"auto": L.DF_PREFILL_KERNEL_AUTO, "mma_sync": L.DF_PREFILL_KERNEL_MMA_SYNC,
             "tcgen05": L.DF_PREFILL_KERNEL_TCGEN05}[kernel]
    T, Hq, D = q1.shape
    num_blocks, Hkv, bs, Dk = k_cache.shape
    B = cu_seqlens.shape[0] - 1
    if Dk != D or tuple(v_cache.shape) != tuple(k_cache.shape):
        raise ValueError("cache shape mismatch")
    if not _heads_view_ok(q1, Hq, D):
        raise ValueError("q1 must be [T, Hq, D] with contiguous heads")
    if (k_new is None) != (v_new is None):
        raise ValueError("give both k_new and v_new or neither")
    if k_new is not None and (tuple(k_new.shape) != (T, Hkv, D) or v_new.stride() != k_new.stride()
                              or not _heads_view_ok(k_new, Hkv, D)):
        raise ValueError("k_new/v_new must be [T, Hkv, D] with contiguous heads")
    if not (k_cache.is_contiguous() and v_cache.is_contiguous() and block_table.is_contiguous()):
        raise ValueError("caches and block table must be contiguous")
    dev = q1.device
    if o1 is None:
        o1 = torch.empty((T, Hq, D), dtype=q1.dtype, device=dev)
    if not _heads_view_ok(o1, Hq, D):
        raise ValueError("o1 must be [T, Hq, D] with contiguous heads")
    if q2raw is None:
        o2 = None
    else:
        if not (q2raw.is_contiguous() and tuple(q2raw.shape) == (B, Hq, D)):
            raise ValueError("q2raw must be a contiguous [B, Hq, D] tensor")
        if o2 is None:
            o2 = torch.empty((B, Hq, D), dtype=q1.dtype, device=dev)
        if not (o2.is_contiguous() and tuple(o2.shape) == (B, Hq, D)):
            raise ValueError("o2 must be a contiguous [B, Hq, D] tensor")
        if workspace is None:
            workspace = new_prefill_workspace(B, Hq, Hkv, D, max_seqlen, dev)
    st = _lib().dualflow_prefill_ex(
        _ptr(q1), q1.stride(0), _ptr(k_new), _ptr(v_new),
        0 if k_new is None else k_new.stride(0), _ptr(q2raw), _ptr(a), _ptr(k_cache),
        _ptr(v_cache), _ptr(block_table), block_table.shape[1], _ptr(cu_seqlens), _ptr(ctx_lens),
        int(max_q_len), int(max_seqlen), _ptr(o1), o1.stride(0), _ptr(o2), B, T, Hq, Hkv, D, bs,
        num_blocks, float(scale), dtype_code(q1.dtype), kcode, _ptr(workspace),
        0 if workspace is None else workspace.numel() * workspace.element_size(),
        _ptr(err_flag), _stream(stream))
    L.check("dualflow_prefill_ex", st)
    return o1, o2


# ----------------------------------------------------------------- append

def kv_append(k_new, v_new, k_cache, v_cache, block_table, positions, *, err_flag=None,
              stream=None):
    """Primary-only append of k_new/v_new [B, Hkv, D] at positions[b]."""
    B, Hkv, D = k_new.shape
    num_blocks, Hkv2, bs, D2 = k_cache.shape
    if (Hkv2, D2) != (Hkv, D) or v_new.shape != k_new.shape or v_new.stride() != k_new.stride():
        raise ValueError("shape mismatch")
    if k_new.stride(2) != 1 or k_new.stride(1) != D:
        raise ValueError("k_new must have contiguous heads")
    st = _lib().dualflow_kv_append(
        _ptr(k_new), _ptr(v_new), k_new.stride(0), _ptr(k_cache), _ptr(v_cache),
        _ptr(block_table), block_table.shape[1], _ptr(positions), B, Hkv, D, bs, num_blocks,
        dtype_code(k_new.dtype), _ptr(err_flag), _stream(stream))
    L.check("dualflow_kv_append", st)


# ----------------------------------------------------------------- projection

EPILOGUES = {"none": L.DF_EPI_NONE, "swiglu": L.DF_EPI_SWIGLU, "residual": L.DF_EPI_RESIDUAL}


def grouped_proj_workspace_size(M, N, K, epilogue="none") -> int:
    return _lib().dualflow_grouped_proj_workspace_size(M, N, K, EPILOGUES[epilogue])


def grouped_proj_num_launches(M, N, K, epilogue="none") -> int:
    return _lib().dualflow_grouped_proj_num_launches(M, N, K, EPILOGUES[epilogue])


def new_proj_workspace(M, N, K, epilogue="none", device="cuda"):
    """Workspace for grouped_proj (fp32 partials of split tiles)."""
    return torch.zeros(max(256, grouped_proj_workspace_size(M, N, K, epilogue)), dtype=torch.uint8,
                       device=device)


def grouped_proj(x, m_primary, w, *, n_aux=None, y=None, epilogue="none", coupling=None,
                 residual=None, workspace=None, err_flag=None, stream=None, next_w=None,
                 next_epilogue="none"):
    """y = epilogue(x w^T) for both flows' rows in one GEMM.

    x: bf16 [M, K] (row stride multiple of 8), rows [0, m_primary) primary,
    the rest auxiliary; w: bf16 [N, K] contiguous. epilogue "swiglu": w is
    [W_gate; W_up] and y is [M, N/2]; "residual": y = residual + x w^T.
    coupling: b (swiglu) or c (residual) vector, bf16, or None.
    next_w / next_epilogue: the projection launched next on this stream (same
    rows and workspace size); its first weight blocks are prefetched into L2
    while this one finishes. A cache hint only: results do not change.
    """
    M, K = x.shape
    N, K2 = w.shape
    if K2 != K or x.stride(1) != 1 or not w.is_contiguous():
        raise ValueError("x [M, K] with unit column stride and w [N, K] contiguous required")
    epi = EPILOGUES[epilogue]
    n_out = N // 2 if epi == L.DF_EPI_SWIGLU else N
    if y is None:
        y = torch.empty((M, n_out), dtype=x.dtype, device=x.device)
    if workspace is None:
        workspace = new_proj_workspace(M, N, K, epilogue, x.device)
    args = (_ptr(x), x.stride(0), int(m_primary), int(M - m_primary), _ptr(w), N, K,
            n_out if n_aux is None else int(n_aux), _ptr(y), y.stride(0), epi, _ptr(coupling),
            _ptr(residual), 0 if residual is None else residual.stride(0), _ptr(workspace),
            workspace.numel() * workspace.element_size())
    if next_w is None:
        st = _lib().dualflow_grouped_proj(*args, _ptr(err_flag), _stream(stream))
        L.check("dualflow_grouped_proj", st)
    else:
        if not next_w.is_contiguous() or next_w.dtype != torch.bfloat16:
            raise ValueError("next_w must be a contiguous bf16 [N, K] weight")
        st = _lib().dualflow_grouped_proj_chain(*args, _ptr(next_w), next_w.shape[0],
                                                next_w.shape[1], EPILOGUES[next_epilogue],
                                                _ptr(err_flag), _stream(stream))
        L.check("dualflow_grouped_proj_chain", st)
    return y


def grouped_proj_batched(x, m_primary, w, *, y=None, epilogue="none", workspace=None,
                         err_flag=None, stream=None, next_w=None, next_epilogue="none"):
    """A batch of projections of one shape in one launch: y[b] = epilogue(x[b]
    w[b]^T) for x bf16 [batch, M, K], w bf16 [batch, N, K] (contiguous), y
    bf16 [batch, M, n_out]; epilogue "none" or "swiglu" (no coupling, no
    residual). next_w ([N', K'] or [batch', N', K']) hints the next projection
    on the stream for an L2 prefetch (results do not change)."""
    batch, M, K = x.shape
    _, N, K2 = w.shape
    if K2 != K or not x.is_contiguous() or not w.is_contiguous():
        raise ValueError("x [batch, M, K] and w [batch, N, K] contiguous required")
    epi = EPILOGUES[epilogue]
    n_out = N // 2 if epi == L.DF_EPI_SWIGLU else N
    if y is None:
        y = torch.empty((batch, M, n_out), dtype=x.dtype, device=x.device)
    if workspace is None:
        workspace = new_proj_workspace(M, N, K, epilogue, x.device)
    if next_w is None:
        nw, nN, nK, nb, nbs = None, 0, 0, 1, 0
    else:
        nw3 = next_w if next_w.dim() == 3 else next_w.unsqueeze(0)
        nb, nN, nK = nw3.shape
        nw, nbs = next_w, nN * nK
    st = _lib().dualflow_grouped_proj_batched(
        _ptr(x), x.stride(1), x.stride(0), int(m_primary), int(M - m_primary), _ptr(w), N, K,
        w.stride(0), _ptr(y), y.stride(1), y.stride(0), batch, epi, _ptr(workspace),
        workspace.numel() * workspace.element_size(), _ptr(nw), nN, nK,
        EPILOGUES[next_epilogue], nb, nbs, _ptr(err_flag), _stream(stream))
    L.check("dualflow_grouped_proj_batched", st)
    return y


def grouped_proj_batched_num_launches(M, N, K, epilogue, batch) -> int:
    return _lib().dualflow_grouped_proj_batched_num_launches(M, N, K, EPILOGUES[epilogue], batch)


# ----------------------------------------------------------------- MoE router replay

MOE_ROWS = 64  # rows per flow in an expert block: at most 64 tokens per call


def moe_route(x, B, w_router, k, k_aux=None, *, ids=None, g1=None, g2=None, logits=None,
              stream=None):
    """Router of both flows (router replay). x: bf16 [2B, d] (primary rows,
    then auxiliary rows); w_router: bf16 [E, d]. Returns (ids int32 [B, k_aux],
    g1 fp32 [B, k], g2 fp32 [B, k_aux]); logits (fp32 [2B, E]) is filled when
    given."""
    k_aux = k if k_aux is None else k_aux
    E, d = w_router.shape
    dev = x.device
    ids = torch.empty((B, k_aux), dtype=torch.int32, device=dev) if ids is None else ids
    g1 = torch.empty((B, k), dtype=torch.float32, device=dev) if g1 is None else g1
    g2 = torch.empty((B, k_aux), dtype=torch.float32, device=dev) if g2 is None else g2
    st = _lib().dualflow_moe_route(_ptr(x), x.stride(0), int(B), int(d), _ptr(w_router), int(E),
                                   int(k), int(k_aux), _ptr(ids), _ptr(g1), _ptr(g2),
                                   _ptr(logits), _stream(stream))
    L.check("dualflow_moe_route", st)
    return ids, g1, g2


def moe_dispatch(x, B, ids, E, k, k_aux=None, *, xe=None, slot1=None, slot2=None, counts=None,
                 err_flag=None, stream=None):
    """Pack each expert's rows: xe bf16 [E, 128, d] (primary rows from 0,
    auxiliary rows from 64), slot1 int32 [B, k], slot2 int32 [B, k_aux]."""
    k_aux = k if k_aux is None else k_aux
    d = x.shape[1]
    dev = x.device
    xe = torch.zeros((E, 2 * MOE_ROWS, d), dtype=torch.bfloat16, device=dev) if xe is None else xe
    slot1 = torch.empty((B, k), dtype=torch.int32, device=dev) if slot1 is None else slot1
    slot2 = torch.empty((B, k_aux), dtype=torch.int32, device=dev) if slot2 is None else slot2
    st = _lib().dualflow_moe_dispatch(_ptr(x), x.stride(0), int(B), int(d), _ptr(ids), int(E),
                                      int(k), int(k_aux), _ptr(xe), _ptr(slot1), _ptr(slot2),
                                      _ptr(counts), _ptr(err_flag), _stream(stream))
    L.check("dualflow_moe_dispatch", st)
    return xe, slot1, slot2


def moe_combine(ye, ids, g1, g2, slot1, slot2, B, k, k_aux=None, *, residual=None, y=None,
                err_flag=None, stream=None):
    """y bf16 [2B, d] = gate-weighted sum of the experts' output rows (+ residual)."""
    k_aux = k if k_aux is None else k_aux
    E, _, d = ye.shape
    if y is None:
        y = torch.empty((2 * B, d), dtype=torch.bfloat16, device=ye.device)
    st = _lib().dualflow_moe_combine(_ptr(ye), _ptr(ids), _ptr(g1), _ptr(g2), _ptr(slot1),
                                     _ptr(slot2), int(B), int(d), int(E), int(k), int(k_aux),
                                     _ptr(residual), 0 if residual is None else residual.stride(0),
                                     _ptr(y), y.stride(0), _ptr(err_flag), _stream(stream))
    L.check("dualflow_moe_combine", st)
    return y


# ----------------------------------------------------------------- mixture head

def mixture_head(logits, B, *, p_mix=None, alpha=None, stream=None):
    """Mixed next-token distribution of both flows.

    logits: [2B, V] bf16 or fp32 (primary rows, then auxiliary rows; unit
    column stride). Returns (p_mix fp32 [B, V], alpha fp32 [B]) with
    p_mix = alpha p1 + (1 - alpha) p2, alpha = 1/2 + 1/2 sum(p1^2).
    """
    rows, V = logits.shape
    if rows < 2 * B or logits.stride(1) != 1:
        raise ValueError("logits must be [2B, V] with unit column stride")
    if p_mix is None:
        p_mix = torch.empty((B, V), dtype=torch.float32, device=logits.device)
    if alpha is None:
        alpha = torch.empty((B,), dtype=torch.float32, device=logits.device)
    st = _lib().dualflow_mixture_head(_ptr(logits), logits.stride(0), int(B), int(V),
                                      dtype_code(logits.dtype), _ptr(p_mix), p_mix.stride(0),
                                      _ptr(alpha), _stream(stream))
    L.check("dualflow_mixture_head", st)
    return p_mix, alpha


def mixture_head_slices(B, V) -> int:
    return _lib().dualflow_mixture_head_slices(int(B), int(V))


# ----------------------------------------------------------------- norm

def rmsnorm(x, gain=None, y=None, eps=1e-5, stream=None):
    rows, cols = x.shape
    if y is None:
        y = torch.empty_like(x)
    st = _lib().dualflow_rmsnorm(_ptr(x), x.stride(0), _ptr(gain), _ptr(y), y.stride(0), rows, cols,
                                 float(eps), _stream(stream))
    L.check("dualflow_rmsnorm", st)
    return y


def layer_pre_attention_supported(m_primary, d_model, Hq, Hkv, D) -> bool:
    return bool(_lib().dualflow_layer_pre_attention_supported(int(m_primary), int(d_model),
                                                               int(Hq), int(Hkv), int(D)))


def layer_pre_attention(x, w_qkv, Hq, Hkv, k_cache, v_cache, block_table, positions, *, eps=1e-5,
                        qkv=None, err_flag=None, stream=None):
    """r = RMSNorm row scale of x; qkv = bf16(r x W_qkv^T) (auxiliary rows: Q
    columns only); the primary rows' K / V columns appended to the cache at
    positions[b], in one launch.

    x: bf16 [2m, d_model] (primary rows first); w_qkv: bf16 [Hq D + 2 Hkv D,
    d_model]; caches bf16 [num_blocks, Hkv, block_size, D]; block_table int32
    [m, max_blocks]; positions int32 [m]. Returns qkv [2m, Hq D + 2 Hkv D]."""
    M, d_model = x.shape
    num_blocks, Hkv2, bs, D = k_cache.shape
    mp = M // 2
    nout = (Hq + 2 * Hkv) * D
    for t in (x, w_qkv, k_cache, v_cache):
        if not t.is_contiguous() or t.dtype != torch.bfloat16:
            raise ValueError("bf16 contiguous tensors required")
    if M % 2 or Hkv2 != Hkv or tuple(w_qkv.shape) != (nout, d_model) or \
            v_cache.shape != k_cache.shape or block_table.shape[0] != mp or \
            positions.numel() != mp:
        raise ValueError("shape mismatch")
    if block_table.dtype != torch.int32 or positions.dtype != torch.int32 or \
            not block_table.is_contiguous():
        raise ValueError("int32 contiguous block_table / positions required")
    if qkv is None:
        qkv = torch.empty((M, nout), dtype=torch.bfloat16, device=x.device)
    if not qkv.is_contiguous() or tuple(qkv.shape) != (M, nout):
        raise ValueError("qkv must be contiguous [2m, N]")
    st = _lib().dualflow_layer_pre_attention(
        _ptr(x), _ptr(w_qkv), mp, d_model, int(Hq), int(Hkv), D, float(eps), _ptr(qkv),
        _ptr(k_cache), _ptr(v_cache), _ptr(block_table), block_table.shape[1], _ptr(positions),
        bs, num_blocks, _ptr(err_flag), _stream(stream))
    L.check("dualflow_layer_pre_attention", st)
    return qkv


def layer_qkv_partials(x, w_qkv, Hq, Hkv, D, *, part=None, ss_part=None, err_flag=None,
                       stream=None):
    """fp32 QKV partial products of the 4 quarters of d_model and the
    quarters' row sums of squares, one launch: returns (part [4, 2m, N],
    ss_part [4, 2m]). Summed in quarter order and scaled by the RMSNorm row
    scale they give layer_pre_attention's qkv bit for bit."""
    M, d_model = x.shape
    nout = (Hq + 2 * Hkv) * D
    for t in (x, w_qkv):
        if not t.is_contiguous() or t.dtype != torch.bfloat16:
            raise ValueError("bf16 contiguous tensors required")
    if M % 2 or tuple(w_qkv.shape) != (nout, d_model):
        raise ValueError("shape mismatch")
    if part is None:
        part = torch.empty((4, M, nout), dtype=torch.float32, device=x.device)
    if ss_part is None:
        ss_part = torch.empty((4, M), dtype=torch.float32, device=x.device)
    if tuple(part.shape) != (4, M, nout) or tuple(ss_part.shape) != (4, M) or \
            part.dtype != torch.float32 or ss_part.dtype != torch.float32 or \
            not part.is_contiguous() or not ss_part.is_contiguous():
        raise ValueError("part must be fp32 [4, 2m, N] and ss_part fp32 [4, 2m], contiguous")
    st = _lib().dualflow_layer_qkv_partials(
        _ptr(x), _ptr(w_qkv), M // 2, d_model, int(Hq), int(Hkv), int(D), _ptr(part),
        _ptr(ss_part), _ptr(err_flag), _stream(stream))
    L.check("dualflow_layer_qkv_partials", st)
    return part, ss_part


def decode_attn_qkv_partials(part, ss_part, d_model, a, k_cache, v_cache, block_table, seqlens,
                             max_seqlen, Hq, *, eps=1e-5, o1=None, o2=None, dual=True, scale=0.0,
                             num_splits=0, workspace=None, err_flag=None, stream=None):
    """Decode attention whose Q1 / Q2raw rows and appended K / V row are built
    in its prologue from layer_qkv_partials' output; returns (o1, o2).
    Equal bit for bit to layer_pre_attention (positions = seqlens - 1)
    followed by decode_attn. dual=False: primary-only (o2 None)."""
    parts, M, nout = part.shape
    mp = M // 2
    num_blocks, Hkv, bs, D = k_cache.shape
    if M % 2 or nout != (Hq + 2 * Hkv) * D or tuple(ss_part.shape) != (parts, M):
        raise ValueError("shape mismatch")
    if part.dtype != torch.float32 or ss_part.dtype != torch.float32 or \
            not part.is_contiguous() or not ss_part.is_contiguous():
        raise ValueError("fp32 contiguous partials required")
    if k_cache.dtype != torch.bfloat16 or v_cache.shape != k_cache.shape or \
            not (k_cache.is_contiguous() and v_cache.is_contiguous() and
                 block_table.is_contiguous()):
        raise ValueError("bf16 contiguous caches and block table required")
    dev = part.device
    if o1 is None:
        o1 = torch.empty((mp, Hq, D), dtype=torch.bfloat16, device=dev)
    if dual and o2 is None:
        o2 = torch.empty((mp, Hq, D), dtype=torch.bfloat16, device=dev)
    if not dual:
        o2 = None
    for o in (o1, o2):
        if o is not None and (not _heads_view_ok(o, Hq, D) or o.stride(0) != o1.stride(0)):
            raise ValueError("outputs must be [m, Hq, D] with contiguous heads and equal strides")
    if workspace is None:
        workspace = new_attn_workspace(mp, Hq, Hkv, D, max_seqlen, num_splits, dev)
    st = _lib().dualflow_decode_attn_qkv_partials(
        _ptr(part), _ptr(ss_part), parts, mp, int(d_model), float(eps), _ptr(a), _ptr(k_cache),
        _ptr(v_cache), _ptr(block_table), block_table.shape[1], _ptr(seqlens), int(max_seqlen),
        _ptr(o1), _ptr(o2), o1.stride(0), int(Hq), Hkv, D, bs, num_blocks, float(scale),
        int(num_splits), _ptr(workspace),
        0 if workspace is None else workspace.numel() * workspace.element_size(),
        _ptr(err_flag), _stream(stream))
    L.check("dualflow_decode_attn_qkv_partials", st)
    return o1, o2


def layer_post_attention_workspace_size(m_primary, d_model, q_dim, F) -> int:
    return _lib().dualflow_layer_post_attention_workspace_size(int(m_primary), int(d_model),
                                                               int(q_dim), int(F))


def new_post_attention_workspace(m_primary, d_model, q_dim, F, device="cuda"):
    """Zero-filled workspace of layer_post_attention (its leading grid counters
    must start at zero; every completed call leaves them at zero)."""
    n = layer_post_attention_workspace_size(m_primary, d_model, q_dim, F)
    if n == 0:
        raise ValueError("layer_post_attention does not support these sizes")
    return torch.zeros(n, dtype=torch.uint8, device=device)


def layer_post_attention(attn, x, w_o, w_gu, w_down, b, c, *, eps=1e-5, x_mid=None, h=None,
                         x_out=None, workspace=None, err_flag=None, stream=None,
                         qkv_next=None):
    """x_mid = x + attn W_o^T; r = RMSNorm row scale of x_mid; h = SiLU(r
    x_mid W_gate^T) * (r x_mid W_up^T) (+ b coupling); x_out = x_mid + h
    W_down^T (+ c coupling), in one launch.

    attn: bf16 [2m, q_dim]; x: bf16 [2m, d_model] (primary rows first); w_o
    [d_model, q_dim], w_gu [2F, d_model], w_down [d_model, F]; b [F], c
    [d_model] or None. Returns (x_out, x_mid, h).

    qkv_next = (w_qkv, Hq, Hkv, D, part, ss_part): the same launch also
    computes the next layer's QKV partial products of x_out into part fp32
    [4, 2m, (Hq + 2 Hkv) D] and ss_part fp32 [4, 2m], as layer_qkv_partials
    (x_out, w_qkv, ...) would (part bit for bit)."""
    M, q_dim = attn.shape
    d_model = x.shape[1]
    F = w_down.shape[1]
    mp = M // 2
    for t in (attn, x, w_o, w_gu, w_down):
        if not t.is_contiguous() or t.dtype != torch.bfloat16:
            raise ValueError("bf16 contiguous tensors required")
    if M % 2 or x.shape[0] != M or tuple(w_o.shape) != (d_model, q_dim) or \
            tuple(w_gu.shape) != (2 * F, d_model):
        raise ValueError("shape mismatch")
    dev = x.device
    bf = torch.bfloat16
    x_mid = torch.empty((M, d_model), dtype=bf, device=dev) if x_mid is None else x_mid
    h = torch.empty((M, F), dtype=bf, device=dev) if h is None else h
    x_out = torch.empty((M, d_model), dtype=bf, device=dev) if x_out is None else x_out
    for t in (x_mid, h, x_out):
        if not t.is_contiguous():
            raise ValueError("outputs must be contiguous")
    if workspace is None:
        workspace = new_post_attention_workspace(mp, d_model, q_dim, F, dev)
    wbytes = workspace.numel() * workspace.element_size()
    if qkv_next is None:
        st = _lib().dualflow_layer_post_attention(
            _ptr(attn), _ptr(x), _ptr(w_o), _ptr(w_gu), _ptr(w_down), _ptr(b), _ptr(c), mp,
            d_model, q_dim, F, float(eps), _ptr(x_mid), _ptr(h), _ptr(x_out), _ptr(workspace),
            wbytes, _ptr(err_flag), _stream(stream))
        L.check("dualflow_layer_post_attention", st)
        return x_out, x_mid, h
    w_qkv, Hq, Hkv, D, part, ss_part = qkv_next
    nout = (Hq + 2 * Hkv) * D
    if not w_qkv.is_contiguous() or w_qkv.dtype != torch.bfloat16 or \
            tuple(w_qkv.shape) != (nout, d_model):
        raise ValueError("w_qkv must be bf16 [(Hq + 2 Hkv) D, d_model], contiguous")
    if tuple(part.shape) != (4, M, nout) or tuple(ss_part.shape) != (4, M) or \
            part.dtype != torch.float32 or ss_part.dtype != torch.float32 or \
            not part.is_contiguous() or not ss_part.is_contiguous():
        raise ValueError("part must be fp32 [4, 2m, N] and ss_part fp32 [4, 2m], contiguous")
    st = _lib().dualflow_layer_post_attention_qkv(
        _ptr(attn), _ptr(x), _ptr(w_o), _ptr(w_gu), _ptr(w_down), _ptr(b), _ptr(c), mp, d_model,
        q_dim, F, float(eps), _ptr(x_mid), _ptr(h), _ptr(x_out), _ptr(workspace), wbytes,
        _ptr(w_qkv), int(Hq), int(Hkv), int(D), _ptr(part), _ptr(ss_part), _ptr(err_flag),
        _stream(stream))
    L.check("dualflow_layer_post_attention_qkv", st)
    return x_out, x_mid, h
