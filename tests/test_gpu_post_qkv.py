"""GPU checks of the layer-stack form of the post-attention launch: the same
launch followed by the next layer's QKV projection of x_out, left as the four
K-quarter partial products (dualflow_layer_post_attention_qkv).

Its x_mid, h and x_out must be the plain launch's bit for bit; its partial
products must equal dualflow_layer_qkv_partials(x_out, w_qkv) bit for bit
(the same K quarters, tile MMAs and accumulation order), and its row sums of
squares that call's within fp32 rounding (another summation order). Both
references are themselves checked against the fp64 oracle in their own tests.
"""

import dataclasses

import numpy as np
import pytest
import torch

from dual_flow_transformer_b200 import _lib as L
from dual_flow_transformer_b200 import api

pytestmark = pytest.mark.gpu


@dataclasses.dataclass
class Shape:
    mp: int
    d: int
    Hq: int
    Hkv: int
    D: int
    F: int
    seed: int


SHAPES = {
    "small": Shape(8, 512, 4, 2, 128, 1024, 70),       # QKV tiles of 64 columns
    "mid": Shape(64, 1024, 8, 2, 128, 2048, 71),
    "odd_rows": Shape(5, 256, 2, 1, 64, 640, 72),      # rows past m_primary in the tiles
}
FULL = Shape(64, 4096, 32, 8, 128, 14336, 73)          # the layer workload: 192-column tiles


def _inputs(s, dev):
    g = torch.Generator().manual_seed(s.seed)
    bf = torch.bfloat16
    M, qd, nout = 2 * s.mp, s.Hq * s.D, (s.Hq + 2 * s.Hkv) * s.D
    t = dict(
        attn=torch.randn(M, qd, generator=g).to(bf),
        x=torch.randn(M, s.d, generator=g).to(bf),
        w_o=(torch.randn(s.d, qd, generator=g) * 0.02).to(bf),
        w_gu=(torch.randn(2 * s.F, s.d, generator=g) * 0.02).to(bf),
        w_down=(torch.randn(s.d, s.F, generator=g) * 0.02).to(bf),
        b=(torch.randn(s.F, generator=g) * 0.1).to(bf),
        c=(torch.randn(s.d, generator=g) * 0.1).to(bf),
        w_qkv=(torch.randn(nout, s.d, generator=g) * 0.02).to(bf))
    return {k: v.to(dev) for k, v in t.items()}


def _run(s, d, workspace=None):
    M, nout = 2 * s.mp, (s.Hq + 2 * s.Hkv) * s.D
    part = torch.full((4, M, nout), float("nan"), dtype=torch.float32, device=d["x"].device)
    ss = torch.full((4, M), float("nan"), dtype=torch.float32, device=d["x"].device)
    err = torch.zeros(1, dtype=torch.int32, device=d["x"].device)
    out = api.layer_post_attention(d["attn"], d["x"], d["w_o"], d["w_gu"], d["w_down"], d["b"],
                                   d["c"], err_flag=err, workspace=workspace,
                                   qkv_next=(d["w_qkv"], s.Hq, s.Hkv, s.D, part, ss))
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    return out, part, ss


def _check(s, d):
    (x_out, x_mid, h), part, ss = _run(s, d)
    # the post-attention outputs: the plain launch's, bit for bit
    r_out, r_mid, r_h = api.layer_post_attention(d["attn"], d["x"], d["w_o"], d["w_gu"],
                                                 d["w_down"], d["b"], d["c"])
    assert torch.equal(x_mid, r_mid) and torch.equal(h, r_h) and torch.equal(x_out, r_out)
    # the next layer's partials: the standalone call on x_out
    r_part, r_ss = api.layer_qkv_partials(x_out, d["w_qkv"], s.Hq, s.Hkv, s.D)
    torch.cuda.synchronize()
    assert torch.equal(part, r_part), "partial products differ"
    # two summation orders of the same d/4 positive squares, each within
    # (n - 1) 2^-24 of the exact sum (recursive summation bound)
    n = s.d // 4
    np.testing.assert_allclose(ss.cpu().numpy(), r_ss.cpu().numpy(), rtol=2 * (n - 1) * 2.0**-24,
                               atol=0)
    return x_out, part, ss


@pytest.mark.parametrize("name", list(SHAPES))
def test_qkv_phase_matches_the_two_launches(cuda_device, name):
    _check(SHAPES[name], _inputs(SHAPES[name], cuda_device))


def test_qkv_phase_repeatable_on_one_workspace(cuda_device):
    """Counters rewound after every call: a second call on the same
    workspace gives the same bits."""
    s = SHAPES["small"]
    d = _inputs(s, cuda_device)
    ws = api.new_post_attention_workspace(s.mp, s.d, s.Hq * s.D, s.F, cuda_device)
    a = _run(s, d, ws)
    b = _run(s, d, ws)
    assert torch.equal(a[0][0], b[0][0]) and torch.equal(a[1], b[1]) and torch.equal(a[2], b[2])
    assert int(ws[:256].view(torch.int32).abs().sum().item()) == 0


@pytest.mark.slow
def test_qkv_phase_full_size_layer(cuda_device):
    """The layer workload's sizes: d_model 4096, 32/8 heads of 128, SwiGLU
    14336, 64 sequences per flow (six thousand QKV columns in 32 tiles)."""
    _check(FULL, _inputs(FULL, cuda_device))


def test_qkv_phase_rejects_bad_arguments(cuda_device):
    s = SHAPES["small"]
    d = _inputs(s, cuda_device)
    M, qd, nout = 2 * s.mp, s.Hq * s.D, (s.Hq + 2 * s.Hkv) * s.D
    part = torch.empty((4, M, nout), dtype=torch.float32, device=cuda_device)
    ss = torch.empty((4, M), dtype=torch.float32, device=cuda_device)
    ws = api.new_post_attention_workspace(s.mp, s.d, qd, s.F, cuda_device)
    x_mid = torch.empty_like(d["x"])
    h = torch.empty((M, s.F), dtype=torch.bfloat16, device=cuda_device)
    x_out = torch.empty_like(d["x"])
    p = lambda t: t.data_ptr()  # noqa: E731

    def call(w_qkv, Hq, Hkv, D, part_p, ss_p, d_model=s.d):
        return L.load().dualflow_layer_post_attention_qkv(
            p(d["attn"]), p(d["x"]), p(d["w_o"]), p(d["w_gu"]), p(d["w_down"]), p(d["b"]),
            p(d["c"]), s.mp, d_model, qd, s.F, 1e-5, p(x_mid), p(h), p(x_out), p(ws),
            ws.numel(), w_qkv, Hq, Hkv, D, part_p, ss_p, None, None)

    assert call(None, s.Hq, s.Hkv, s.D, p(part), p(ss)) == L.DF_ERR_NULL
    assert call(p(d["w_qkv"]), s.Hq, s.Hkv, s.D, None, p(ss)) == L.DF_ERR_NULL
    assert call(p(d["w_qkv"]), s.Hq, s.Hkv, s.D, p(part), None) == L.DF_ERR_NULL
    assert call(p(d["w_qkv"]), s.Hq + 1, s.Hkv, s.D, p(part), p(ss)) == L.DF_ERR_SHAPE  # q_dim
    assert call(p(d["w_qkv"]), s.Hq, 3, s.D, p(part), p(ss)) == L.DF_ERR_SHAPE       # Hq % Hkv
    bad = part.data_ptr() + 4
    assert call(p(d["w_qkv"]), s.Hq, s.Hkv, s.D, bad, p(ss)) == L.DF_ERR_ALIGN
    torch.cuda.synchronize()
