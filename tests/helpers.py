"""Shared test helpers: tolerances, comparisons and oracle feeding."""

import numpy as np
import torch

import oracle
from dual_flow_transformer_b200 import synth

# Tolerances (stated for the decode step): fp32 inputs max-abs <= 1e-5; bf16
# inputs with fp32 accumulation: |gpu - oracle| <= 2e-2 + 1e-2 |oracle| per
# element, and per output row ||gpu - oracle|| / ||oracle|| <= 1e-2.
FP32_ATOL = 1e-5
BF16_ATOL = 2e-2
BF16_RTOL = 1e-2


def f64(t):
    return synth.to_numpy_f32(t).astype(np.float64) if isinstance(t, torch.Tensor) \
        else np.asarray(t, dtype=np.float64)


def assert_close(gpu, ref, dtype, what=""):
    g = f64(gpu)
    r = np.asarray(ref, dtype=np.float64)
    assert g.shape == r.shape, (g.shape, r.shape)
    assert np.isfinite(g).all(), "%s: non-finite GPU output" % what
    err = np.abs(g - r)
    if dtype == "fp32":
        mx = float(err.max()) if err.size else 0.0
        assert mx <= FP32_ATOL, "%s: max-abs %.3e > %.1e" % (what, mx, FP32_ATOL)
        return mx
    bound = BF16_ATOL + BF16_RTOL * np.abs(r)
    bad = err > bound
    assert not bad.any(), "%s: %d elements outside tolerance, worst err %.3e" % (
        what, int(bad.sum()), float(err.max()))
    rows_g = g.reshape(-1, g.shape[-1])
    rows_r = r.reshape(-1, r.shape[-1])
    num = np.linalg.norm(rows_g - rows_r, axis=1)
    den = np.maximum(np.linalg.norm(rows_r, axis=1), 1e-30)
    rel = float((num / den).max())
    assert rel <= BF16_RTOL, "%s: row-relative error %.3e > %.1e" % (what, rel, BF16_RTOL)
    return float(err.max())


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
