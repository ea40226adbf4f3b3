"""Shared test helpers: tolerances, comparisons and oracle feeding."""

import numpy as np
import torch

import oracle
from dual_flow_transformer_b200 import synth

# Tolerances (stated for the decode step): fp32 inputs max-abs <= 1e-5; bf16
# inputs with fp32 accumulation: max-abs <= 2e-2 and relative <= 1e-2.
#  * Attention outputs (|O| is a weighted mean of V rows, a few units at
#    most) take both literally: every element |gpu - oracle| <= 2e-2, and per
#    output row ||gpu - oracle|| / ||oracle|| <= 1e-2 (assert_attn_close).
#  * Outputs of a bf16 chain whose magnitude reaches 8 and more (projections,
#    the layer step) cannot meet a flat 2e-2: one bf16 step there is 1/16.
#    They take |gpu - oracle| <= 2e-2 + 1e-2 |oracle| per element plus the
#    same row-relative bound (assert_close).
FP32_ATOL = 1e-5
BF16_ATOL = 2e-2
BF16_RTOL = 1e-2

# (what, max-abs, row-relative) of every comparison, for the run's summary
PARITY_LOG = []


def f64(t):
    return synth.to_numpy_f32(t).astype(np.float64) if isinstance(t, torch.Tensor) \
        else np.asarray(t, dtype=np.float64)


def _row_rel(g, r):
    rows_g = g.reshape(-1, g.shape[-1])
    rows_r = r.reshape(-1, r.shape[-1])
    num = np.linalg.norm(rows_g - rows_r, axis=1)
    den = np.maximum(np.linalg.norm(rows_r, axis=1), 1e-30)
    return float((num / den).max()) if num.size else 0.0


def assert_close(gpu, ref, dtype, what="", flat_max_abs=False):
    """Compare a GPU output with the oracle; returns the max-abs error.

    flat_max_abs: bf16 elements must meet |err| <= 2e-2 outright (attention
    outputs); otherwise 2e-2 + 1e-2 |oracle| (long bf16 chains)."""
    g = f64(gpu)
    r = np.asarray(ref, dtype=np.float64)
    assert g.shape == r.shape, (g.shape, r.shape)
    assert np.isfinite(g).all(), "%s: non-finite GPU output" % what
    err = np.abs(g - r)
    mx = float(err.max()) if err.size else 0.0
    if dtype == "fp32":
        PARITY_LOG.append((what, mx, None))
        assert mx <= FP32_ATOL, "%s: max-abs %.3e > %.1e" % (what, mx, FP32_ATOL)
        return mx
    rel = _row_rel(g, r)
    PARITY_LOG.append((what, mx, rel))
    if flat_max_abs:
        assert mx <= BF16_ATOL, "%s: max-abs %.3e > %.1e" % (what, mx, BF16_ATOL)
    else:
        bound = BF16_ATOL + BF16_RTOL * np.abs(r)
        bad = err > bound
        assert not bad.any(), "%s: %d elements outside tolerance, worst err %.3e" % (
            what, int(bad.sum()), mx)
    assert rel <= BF16_RTOL, "%s: row-relative error %.3e > %.1e" % (what, rel, BF16_RTOL)
    return mx


def assert_attn_close(gpu, ref, dtype, what=""):
    """Attention outputs: the stated tolerance taken literally (max-abs 2e-2
    on every element and row-relative 1e-2 for bf16; max-abs 1e-5 for fp32)."""
    return assert_close(gpu, ref, dtype, what, flat_max_abs=True)


def oracle_attn(inp, seqlens=None, k_cache=None, v_cache=None, batches=None):
    """Oracle decode outputs for (a subset of) sequences of a synth input dict."""
    kc = synth.to_numpy_f32(inp["k_cache"] if k_cache is None else k_cache)
    vc = synth.to_numpy_f32(inp["v_cache"] if v_cache is None else v_cache)
    sl = (inp["seqlens"] if seqlens is None else seqlens).numpy()
    tbl = inp["block_table"].numpy()
    q1 = synth.to_numpy_f32(inp["q1"])
    q2 = synth.to_numpy_f32(inp["q2raw"])
    a = synth.to_numpy_f32(inp["a"])
    if batches is not None:
        idx = np.asarray(batches)
        q1, q2, tbl, sl = q1[idx], q2[idx], tbl[idx], sl[idx]
    return oracle.decode_attn(q1, q2, a, kc, vc, tbl, sl)


def to_dev(inp, device):
    out = {}
    for k, v in inp.items():
        out[k] = v.to(device) if isinstance(v, torch.Tensor) else v
    return out
