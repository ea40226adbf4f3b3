"""GPU parity of the mixture head (mixed next-token distribution of both
flows) against the fp64 oracle, through the C ABI. Inputs come from seeded
generators; expected values from the oracle only.

p_mix is fp32 and both sides read the same logits (bf16 logits are widened
exactly), so the bar is the fp32 one: max-abs error <= 1e-5 per element and
row-relative L2 error <= 1e-5.
"""

import numpy as np
import pytest
import torch

import oracle
from dual_flow_transformer_b200 import api

pytestmark = pytest.mark.gpu

ABS_TOL = 1e-5
REL_TOL = 1e-5


def _logits(seed, B, V, dtype, scale=3.0):
    g = torch.Generator().manual_seed(seed)
    spread = torch.rand((2 * B, 1), generator=g) * scale + 0.1
    return (torch.randn((2 * B, V), generator=g) * spread).to(dtype)


def _check(p_mix, alpha, logits, B, name):
    ref_p, ref_a = oracle.mixture_head(logits.float().numpy().astype(np.float64), B)
    got_p = p_mix.cpu().numpy().astype(np.float64)
    got_a = alpha.cpu().numpy().astype(np.float64)
    assert np.max(np.abs(got_a - ref_a)) <= ABS_TOL, name + " alpha"
    err = np.abs(got_p - ref_p)
    assert err.max() <= ABS_TOL, "%s max-abs %.3g" % (name, err.max())
    rel = np.linalg.norm(got_p - ref_p, axis=1) / np.linalg.norm(ref_p, axis=1)
    assert rel.max() <= REL_TOL, "%s row-rel %.3g" % (name, rel.max())


CASES = [  # (B, V, dtype)
    (3, 1000, torch.float32),
    (1, 8, torch.float32),
    (1, 32000, torch.bfloat16),      # one sequence: a cluster of 8 slices
    (64, 32000, torch.bfloat16),     # full size: 8 slices per sequence
    (64, 32008, torch.bfloat16),     # ragged last slice
    (5, 50304, torch.float32),
]


@pytest.mark.parametrize("B,V,dtype", CASES)
def test_mixture_parity(cuda_device, B, V, dtype):
    l = _logits(B * 7 + V, B, V, dtype)
    p_mix, alpha = api.mixture_head(l.to(cuda_device), B)
    torch.cuda.synchronize()
    _check(p_mix, alpha, l, B, "B=%d V=%d %s" % (B, V, dtype))


def test_mixture_strided_rows_and_peaked_distributions(cuda_device):
    B, V = 4, 4096
    l = _logits(80, B, V, torch.bfloat16, scale=30.0)
    big = torch.zeros((2 * B, V + 64), dtype=torch.bfloat16, device=cuda_device)
    big[:, :V] = l.to(cuda_device)
    out = torch.full((B, V + 12), -1.0, device=cuda_device)
    assert big[:, :V].stride(0) == V + 64 and out[:, :V].stride(0) == V + 12
    p_mix, alpha = api.mixture_head(big[:, :V], B, p_mix=out[:, :V])
    torch.cuda.synchronize()
    _check(p_mix, alpha, l, B, "strided")
    assert torch.all(out[:, V:] == -1.0)  # nothing written past V


def test_alpha_ignores_auxiliary_logits(cuda_device):
    """alpha reads only the primary rows: NaN or shifted aux logits leave it
    bit-identical (the mixture itself turns NaN only where the aux is NaN)."""
    B, V = 8, 8192
    l = _logits(81, B, V, torch.bfloat16)
    dev = l.to(cuda_device)
    _, a0 = api.mixture_head(dev, B)
    bad = dev.clone()
    bad[B:] = float("nan")
    p_bad, a1 = api.mixture_head(bad, B)
    shifted = dev.clone()
    shifted[B:] += 5.0
    _, a2 = api.mixture_head(shifted, B)
    torch.cuda.synchronize()
    assert torch.equal(a0.view(torch.int32), a1.view(torch.int32))
    assert torch.equal(a0.view(torch.int32), a2.view(torch.int32))
    assert torch.isnan(p_bad).all()


def test_mixture_sums_to_one_at_full_size(cuda_device):
    B, V = 64, 128256
    l = _logits(82, B, V, torch.bfloat16, scale=8.0)
    p_mix, alpha = api.mixture_head(l.to(cuda_device), B)
    torch.cuda.synchronize()
    s = p_mix.double().sum(dim=1)
    assert torch.allclose(s, torch.ones_like(s), atol=1e-5)
    assert bool(((alpha >= 0.5) & (alpha <= 1.0)).all())
    # sampled rows against the oracle
    rows = [0, 31, 63]
    sub = torch.cat([l[rows], l[[B + r for r in rows]]])
    _check(p_mix[rows], alpha[rows], sub, len(rows), "sampled rows")
