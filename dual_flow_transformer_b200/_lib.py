"""ctypes loader for libdualflow.so.

Argument marshalling only. There is no fallback: if the shared library is
missing or fails to load, importing the API raises, because every step of
the decode path runs in the library's CUDA kernels.
"""

from __future__ import annotations

import ctypes
import os

from . import build as _build

LIB_PATH = _build.LIB_PATH

DF_OK, DF_ERR_NULL, DF_ERR_SHAPE, DF_ERR_UNSUPPORTED, DF_ERR_WORKSPACE, DF_ERR_ALIGN, DF_ERR_CUDA = range(7)
DF_FP32, DF_BF16 = 0, 1
DF_EPI_NONE, DF_EPI_SWIGLU, DF_EPI_RESIDUAL = 0, 1, 2
DF_DEVERR_SEQLEN, DF_DEVERR_BLOCK, DF_DEVERR_POSITION, DF_DEVERR_TIMEOUT = 1, 2, 4, 8
DF_DECODE_ATTN_NOALLOC_SCRATCH_BYTES = 16 * 1024 * 1024
DF_PREFILL_KERNEL_AUTO, DF_PREFILL_KERNEL_MMA_SYNC, DF_PREFILL_KERNEL_TCGEN05 = 0, 1, 2

_c_int, _c_i64, _c_size, _c_float, _vp = (ctypes.c_int, ctypes.c_int64, ctypes.c_size_t,
                                           ctypes.c_float, ctypes.c_void_p)

# name -> (restype, argtypes); the order matches include/dualflow.h
SIGNATURES = {
    "dualflow_abi_version": (_c_int, []),
    "dualflow_status_string": (ctypes.c_char_p, [_c_int]),
    "dualflow_selftest_wait_timeout": (_c_int, [_vp, _vp]),
    "dualflow_decode_attn_num_splits": (_c_int, [_c_int, _c_int, _c_int, _c_int, _c_int]),
    "dualflow_decode_attn_workspace_size": (_c_size, [_c_int] * 7),
    "dualflow_decode_attn_num_launches": (_c_int, [_c_int] * 6),
    "dualflow_decode_attn": (_c_int, [
        _vp, _vp, _vp, _c_i64,          # q1, q2raw, a, q_stride_b
        _vp, _vp,                       # k_cache, v_cache
        _vp, _c_int,                    # block_table, max_blocks_per_seq
        _vp, _c_int,                    # seqlens, max_seqlen
        _vp, _vp, _c_i64,               # o1, o2, o_stride_b
        _c_int, _c_int, _c_int, _c_int, _c_int, _c_int,  # B, Hq, Hkv, D, block_size, num_blocks
        _c_float, _c_int, _c_int,       # scale, dtype, num_splits
        _vp, _c_size, _vp, _vp]),       # workspace, bytes, err_flag, stream
    "dualflow_decode_attn_noalloc": (_c_int, [
        _vp, _vp, _vp, _c_i64, _vp, _vp, _vp, _c_int, _vp, _c_int, _vp, _vp, _c_i64,
        _c_int, _c_int, _c_int, _c_int, _c_int, _c_int, _c_float, _c_int, _c_int,
        _vp, _vp]),                     # err_flag, stream (no workspace)
    "dualflow_kv_append": (_c_int, [
        _vp, _vp, _c_i64, _vp, _vp, _vp, _c_int, _vp,
        _c_int, _c_int, _c_int, _c_int, _c_int, _c_int, _vp, _vp]),
    "dualflow_prefill_workspace_size": (_c_size, [_c_int] * 6),
    "dualflow_prefill_num_launches": (_c_int, [_c_int, _c_int]),
    "dualflow_prefill_kernel": (_c_int, [_c_int, _c_int, _vp, _c_i64, _c_int]),
    "dualflow_prefill_ex": (_c_int, [
        _vp, _c_i64, _vp, _vp, _c_i64, _vp, _vp, _vp, _vp, _vp, _c_int, _vp, _vp, _c_int, _c_int,
        _vp, _c_i64, _vp, _c_int, _c_int, _c_int, _c_int, _c_int, _c_int, _c_int,
        _c_float, _c_int, _c_int,       # scale, dtype, kernel
        _vp, _c_size, _vp, _vp]),
    "dualflow_prefill": (_c_int, [
        _vp, _c_i64, _vp, _vp, _c_i64,  # q1, q_stride_t, k_new, v_new, kv_stride_t
        _vp, _vp, _vp, _vp,             # q2raw, a, k_cache, v_cache
        _vp, _c_int, _vp, _vp,          # block_table, max_blocks_per_seq, cu_seqlens, ctx_lens
        _c_int, _c_int,                 # max_q_len, max_seqlen
        _vp, _c_i64, _vp,               # o1, o_stride_t, o2
        _c_int, _c_int, _c_int, _c_int, _c_int, _c_int, _c_int,  # B, T, Hq, Hkv, D, bs, nblocks
        _c_float, _c_int,               # scale, dtype
        _vp, _c_size, _vp, _vp]),       # workspace, bytes, err_flag, stream
    "dualflow_grouped_proj_workspace_size": (_c_size, [_c_int] * 4),
    "dualflow_grouped_proj_num_launches": (_c_int, [_c_int] * 4),
    "dualflow_grouped_proj": (_c_int, [
        _vp, _c_i64, _c_int, _c_int,    # x, ldx, m_primary, m_aux
        _vp, _c_int, _c_int, _c_int,    # w, N, K, n_aux
        _vp, _c_i64,                    # y, ldy
        _c_int, _vp, _vp, _c_i64,       # epilogue, coupling, residual, ldr
        _vp, _c_size, _vp, _vp]),       # workspace, bytes, err_flag, stream
    "dualflow_grouped_proj_chain": (_c_int, [
        _vp, _c_i64, _c_int, _c_int,    # x, ldx, m_primary, m_aux
        _vp, _c_int, _c_int, _c_int,    # w, N, K, n_aux
        _vp, _c_i64,                    # y, ldy
        _c_int, _vp, _vp, _c_i64,       # epilogue, coupling, residual, ldr
        _vp, _c_size,                   # workspace, bytes
        _vp, _c_int, _c_int, _c_int,    # w_next, N_next, K_next, epilogue_next
        _vp, _vp]),                     # err_flag, stream
    "dualflow_mixture_head": (_c_int, [_vp, _c_i64, _c_int, _c_int, _c_int, _vp, _c_i64, _vp,
                                       _vp]),
    "dualflow_mixture_head_slices": (_c_int, [_c_int, _c_int]),
    "dualflow_moe_route": (_c_int, [_vp, _c_i64, _c_int, _c_int, _vp, _c_int, _c_int, _c_int,
                                    _vp, _vp, _vp, _vp, _vp]),
    "dualflow_moe_dispatch": (_c_int, [_vp, _c_i64, _c_int, _c_int, _vp, _c_int, _c_int, _c_int,
                                       _vp, _vp, _vp, _vp, _vp, _vp]),
    "dualflow_moe_combine": (_c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _c_int, _c_int, _c_int,
                                      _c_int, _c_int, _vp, _c_i64, _vp, _c_i64, _vp, _vp]),
    "dualflow_grouped_proj_batched": (_c_int, [
        _vp, _c_i64, _c_i64, _c_int, _c_int,    # x, ldx, x_bstride, m_primary, m_aux
        _vp, _c_int, _c_int, _c_i64,            # w, N, K, w_bstride
        _vp, _c_i64, _c_i64, _c_int, _c_int,    # y, ldy, y_bstride, batch, epilogue
        _vp, _c_size,                           # workspace, bytes
        _vp, _c_int, _c_int, _c_int, _c_int, _c_i64,  # next: w, N, K, epilogue, batch, bstride
        _vp, _vp]),                             # err_flag, stream
    "dualflow_grouped_proj_batched_num_launches": (_c_int, [_c_int] * 5),
    "dualflow_rmsnorm": (_c_int, [_vp, _c_i64, _vp, _vp, _c_i64, _c_int, _c_int, _c_float, _vp]),
    "dualflow_layer_pre_attention_supported": (_c_int, [_c_int] * 5),
    "dualflow_layer_pre_attention": (_c_int, [
        _vp, _vp, _c_int, _c_int, _c_int, _c_int, _c_int,  # x, w_qkv, m, d, Hq, Hkv, D
        _c_float, _vp, _vp, _vp, _vp, _c_int, _vp,         # eps, qkv, caches, table, mbps, pos
        _c_int, _c_int, _vp, _vp]),                        # block_size, num_blocks, err, stream
    "dualflow_layer_qkv_partials": (_c_int, [
        _vp, _vp, _c_int, _c_int, _c_int, _c_int, _c_int,  # x, w_qkv, m, d, Hq, Hkv, D
        _vp, _vp, _vp, _vp]),                              # part, ss_part, err, stream
    "dualflow_decode_attn_qkv_partials": (_c_int, [
        _vp, _vp, _c_int, _c_int, _c_int, _c_float,  # part, ss_part, parts, m, d_model, eps
        _vp, _vp, _vp, _vp, _c_int,          # a, k_cache, v_cache, block_table, mbps
        _vp, _c_int, _vp, _vp, _c_i64,       # seqlens, max_seqlen, o1, o2, o_stride_b
        _c_int, _c_int, _c_int, _c_int, _c_int,  # Hq, Hkv, D, block_size, num_blocks
        _c_float, _c_int,                    # scale, num_splits
        _vp, _c_size, _vp, _vp]),            # workspace, bytes, err_flag, stream
    "dualflow_layer_post_attention_workspace_size": (_c_size, [_c_int] * 4),
    "dualflow_layer_post_attention": (_c_int, [
        _vp, _vp, _vp, _vp, _vp, _vp, _vp,  # attn, x, w_o, w_gu, w_down, b, c
        _c_int, _c_int, _c_int, _c_int,     # m_primary, d_model, q_dim, F
        _c_float,                           # eps
        _vp, _vp, _vp,                      # x_mid, h, x_out
        _vp, _c_size, _vp, _vp]),           # workspace, bytes, err_flag, stream
    "dualflow_layer_post_attention_qkv": (_c_int, [
        _vp, _vp, _vp, _vp, _vp, _vp, _vp,  # attn, x, w_o, w_gu, w_down, b, c
        _c_int, _c_int, _c_int, _c_int,     # m_primary, d_model, q_dim, F
        _c_float,                           # eps
        _vp, _vp, _vp,                      # x_mid, h, x_out
        _vp, _c_size,                       # workspace, bytes
        _vp, _c_int, _c_int, _c_int,        # w_qkv_next, Hq, Hkv, D
        _vp, _vp, _vp, _vp]),               # part, ss_part, err_flag, stream
}

_lib = None


class DualflowError(RuntimeError):
    def __init__(self, fn, status):
        self.status = status
        super().__init__("%s -> %s" % (fn, status_string(status)))


def load(build_if_missing: bool = True):
    """Load (building first if needed) and return the ctypes handle."""
    global _lib
    if _lib is not None:
        return _lib
    if build_if_missing and not _build.up_to_date():
        _build.build()
    if not os.path.exists(LIB_PATH):
        raise ImportError("libdualflow.so is not built (%s); run __graft_entry__.build()" % LIB_PATH)
    lib = ctypes.CDLL(LIB_PATH)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def status_string(status: int) -> str:
    return load().dualflow_status_string(int(status)).decode()


def check(fn_name: str, status: int):
    if status != DF_OK:
        raise DualflowError(fn_name, status)
