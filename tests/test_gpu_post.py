"""GPU parity of the one-launch post-attention half of the decoder layer
(W_o + residual, RMSNorm, SwiGLU gate/up + b coupling, W_down + c coupling +
residual), through the C ABI, against the fp64 oracle (rounding to bf16 at
the interfaces where the kernel stores bf16: x_mid, h, x_out; the kernel
applies the norm's row scale to the gate/up accumulators, so the normalised
rows are not rounded) and against the four-call form.
"""

import dataclasses

import numpy as np
import pytest
import torch

import oracle
from dual_flow_transformer_b200 import _lib as L
from dual_flow_transformer_b200 import api
from tests.helpers import assert_close, f64

pytestmark = pytest.mark.gpu


@dataclasses.dataclass
class Shape:
    mp: int
    d: int
    qd: int
    F: int
    seed: int


SHAPES = {
    "small": Shape(8, 512, 512, 1024, 60),
    "mid": Shape(64, 1024, 512, 2048, 61),
    "odd_rows": Shape(5, 256, 128, 640, 62),
    # 48-column SwiGLU tiles: a 32-column chunk of the last (16-column) tile
    # reaches past F
    "wide": Shape(16, 512, 256, 6016, 64),
}


def _inputs(s, coupled=True):
    g = torch.Generator().manual_seed(s.seed)
    bf = torch.bfloat16
    M = 2 * s.mp
    t = dict(
        attn=torch.randn(M, s.qd, generator=g).to(bf),
        x=torch.randn(M, s.d, generator=g).to(bf),
        w_o=(torch.randn(s.d, s.qd, generator=g) * 0.02).to(bf),
        w_gu=(torch.randn(2 * s.F, s.d, generator=g) * 0.02).to(bf),
        w_down=(torch.randn(s.d, s.F, generator=g) * 0.02).to(bf),
        b=(torch.randn(s.F, generator=g) * 0.1).to(bf),
        c=(torch.randn(s.d, generator=g) * 0.1).to(bf))
    if not coupled:
        t["b"] = None
        t["c"] = None
    return t


def _dev(t, dev):
    return {k: (None if v is None else v.to(dev)) for k, v in t.items()}


def _post(d, err=None, workspace=None):
    return api.layer_post_attention(d["attn"], d["x"], d["w_o"], d["w_gu"], d["w_down"], d["b"],
                                    d["c"], err_flag=err, workspace=workspace)


def _oracle(t, mp):
    """The layer oracle's post-attention steps on the same bf16 inputs, with
    bf16 rounding where this kernel stores bf16 (x_mid, h, x_out)."""
    r = oracle.bf16_round
    X = f64(t["x"])
    b = None if t["b"] is None else f64(t["b"])
    c = None if t["c"] is None else f64(t["c"])
    F = t["w_down"].shape[1]
    x_mid = r(oracle.residual_couple(oracle.grouped_proj(f64(t["attn"]), f64(t["w_o"]), mp), X,
                                     mp, None))
    xn2 = oracle.rmsnorm(x_mid)
    h = r(oracle.swiglu_couple(oracle.grouped_proj(xn2, f64(t["w_gu"]), mp), F, mp, b))
    x_out = r(oracle.residual_couple(oracle.grouped_proj(h, f64(t["w_down"]), mp), x_mid, mp, c))
    return x_mid, h, x_out


@pytest.mark.parametrize("coupled", [True, False])
@pytest.mark.parametrize("name", sorted(SHAPES))
def test_post_attention_matches_oracle(cuda_device, name, coupled):
    s = SHAPES[name]
    t = _inputs(s, coupled)
    d = _dev(t, cuda_device)
    err = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    x_out, x_mid, h = _post(d, err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    r_mid, r_h, r_out = _oracle(t, s.mp)
    assert_close(x_mid.cpu(), r_mid, "bf16", "%s x_mid" % name)
    assert_close(h.cpu(), r_h, "bf16", "%s h" % name)
    assert_close(x_out.cpu(), r_out, "bf16", "%s x_out" % name)


def test_post_attention_matches_the_four_call_form(cuda_device):
    s = SHAPES["mid"]
    d = _dev(_inputs(s), cuda_device)
    x_out, x_mid, h = _post(d)
    M = 2 * s.mp
    ref_mid = api.grouped_proj(d["attn"], s.mp, d["w_o"], epilogue="residual", residual=d["x"])
    ref_xn2 = api.rmsnorm(ref_mid)
    ref_h = api.grouped_proj(ref_xn2, s.mp, d["w_gu"], epilogue="swiglu", coupling=d["b"])
    ref_out = api.grouped_proj(ref_h, s.mp, d["w_down"], epilogue="residual", coupling=d["c"],
                               residual=ref_mid)
    torch.cuda.synchronize()
    for got, ref, what in ((x_mid, ref_mid, "x_mid"), (h, ref_h, "h"), (x_out, ref_out, "x_out")):
        assert got.shape == (M, ref.shape[1])
        assert_close(got.cpu(), f64(ref.cpu()), "bf16", "four-call " + what)


def test_post_attention_deterministic_counters_rewound_and_primary_blind(cuda_device):
    s = SHAPES["mid"]
    t = _inputs(s)
    d = _dev(t, cuda_device)
    ws = api.new_post_attention_workspace(s.mp, s.d, s.qd, s.F, cuda_device)
    err = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    outs = [tuple(o.clone() for o in _post(d, err, ws)) for _ in range(3)]
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    assert torch.count_nonzero(ws[:256]) == 0  # grid counters back at zero
    for o in outs[1:]:
        for a, b in zip(o, outs[0]):
            assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    # the auxiliary flow's inputs do not reach the primary rows
    other = dict(d)
    other["attn"] = d["attn"].clone()
    other["attn"][s.mp:] = float("nan")
    other["x"] = d["x"].clone()
    other["x"][s.mp:] *= 3
    other["b"] = -d["b"]
    other["c"] = d["c"] * 2
    y = _post(other, err, ws)
    torch.cuda.synchronize()
    for a, b in zip(y, outs[0]):
        assert torch.equal(a[:s.mp].view(torch.int16), b[:s.mp].view(torch.int16))
    assert torch.isnan(y[0][s.mp:].float()).all()


def test_post_attention_full_size_layer_shapes(cuda_device):
    """d_model 4096, 32 x 128 attention width, SwiGLU 14336, 64 sequences per
    flow (the layer workload); the oracle recomputes 8 sequences."""
    s = Shape(64, 4096, 4096, 14336, 63)
    t = _inputs(s)
    d = _dev(t, cuda_device)
    err = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    x_out, x_mid, h = _post(d, err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    rows = [0, 9, 31, 63]
    sel = rows + [s.mp + r for r in rows]
    sub = dict(t, attn=t["attn"][sel], x=t["x"][sel])
    r_mid, r_h, r_out = _oracle(sub, len(rows))
    assert_close(x_mid[sel].cpu(), r_mid, "bf16", "full post x_mid")
    assert_close(h[sel].cpu(), r_h, "bf16", "full post h")
    assert_close(x_out[sel].cpu(), r_out, "bf16", "full post x_out")


def test_post_attention_rejects_unsupported_sizes(cuda_device):
    s = SHAPES["small"]
    d = _dev(_inputs(s), cuda_device)
    assert api.layer_post_attention_workspace_size(65, 512, 512, 1024) == 0
    assert api.layer_post_attention_workspace_size(8, 320, 512, 1024) == 0
    # one 128-column W_o / W_down tile per 4-CTA cluster: d_model 8192 needs 64
    assert api.layer_post_attention_workspace_size(8, 8192, 512, 1024) == 0
    # counters + one fp32 sum of squares per (32-column slice, row)
    assert api.layer_post_attention_workspace_size(8, 512, 512, 1024) == 256 + 512 * 16
    ws = torch.zeros(256, dtype=torch.uint8, device=cuda_device)
    with pytest.raises(L.DualflowError) as e:
        _post(d, workspace=ws)
    assert e.value.status == L.DF_ERR_WORKSPACE
