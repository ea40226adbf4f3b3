"""GPU parity of the grouped shared-weight projection (tcgen05) and the fused
epilogues against the fp64 oracle, through the C ABI."""

import numpy as np
import pytest
import torch

import oracle
from dual_flow_transformer_b200 import api, synth
from tests.helpers import assert_close, f64

pytestmark = pytest.mark.gpu


def _rand(g, shape, std=1.0):
    return (torch.randn(shape, generator=g) * std).to(torch.bfloat16)


def _case(seed, mp, ma, N, K, epi="none", coupled=False):
    g = torch.Generator().manual_seed(seed)
    x = _rand(g, (mp + ma, K))
    w = _rand(g, (N, K), 0.02)
    n_out = N // 2 if epi == "swiglu" else N
    cpl = _rand(g, (n_out,), 0.1) if coupled else None
    res = _rand(g, (mp + ma, n_out)) if epi == "residual" else None
    return x, w, cpl, res


def _oracle(x, w, mp, epi, cpl, res, n_aux=None):
    acc = oracle.grouped_proj(f64(x), f64(w), mp)
    if epi == "swiglu":
        return oracle.swiglu_couple(acc, w.shape[0] // 2, mp, None if cpl is None else f64(cpl))
    if epi == "residual":
        return oracle.residual_couple(acc, f64(res), mp, None if cpl is None else f64(cpl))
    return acc


def _gpu(dev, x, w, mp, epi, cpl, res, n_aux=None, y=None):
    return api.grouped_proj(x.to(dev), mp, w.to(dev), n_aux=n_aux, epilogue=epi,
                            coupling=None if cpl is None else cpl.to(dev),
                            residual=None if res is None else res.to(dev), y=y)


SHAPES = [  # (m_primary, m_aux, N, K)
    (64, 64, 256, 512),
    (8, 8, 384, 1024),
    (5, 3, 128, 64),
    (1, 0, 128, 192),
    (64, 64, 128, 8192),   # one tile cut over 128 CTAs (stream-K fixup with many parts)
    (16, 16, 1024, 320),
]


@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("epi,coupled", [("none", False), ("swiglu", False), ("swiglu", True),
                                         ("residual", False), ("residual", True)])
def test_proj_parity(cuda_device, shape, epi, coupled):
    mp, ma, N, K = shape
    if coupled and mp != ma:
        pytest.skip("coupling pairs aux row j with primary row j")
    x, w, cpl, res = _case(sum(shape) + 7 * len(epi) + int(coupled), mp, ma, N, K, epi, coupled)
    y = _gpu(cuda_device, x, w, mp, epi, cpl, res)
    torch.cuda.synchronize()
    ref = _oracle(x, w, mp, epi, cpl, res)
    assert_close(y.cpu(), ref, "bf16", "proj %s %s" % (shape, epi))


def test_aux_columns_mask_and_grouping_is_invisible(cuda_device):
    mp = ma = 32
    x, w, _, _ = _case(7, mp, ma, 512, 256)
    dev = cuda_device
    y = torch.full((mp + ma, 512), 3.0, dtype=torch.bfloat16, device=dev)
    _gpu(dev, x, w, mp, "none", None, None, n_aux=128, y=y)
    alone = _gpu(dev, x[mp:].contiguous(), w, ma, "none", None, None)
    prim = _gpu(dev, x[:mp].contiguous(), w, mp, "none", None, None)
    torch.cuda.synchronize()
    assert torch.all(y[mp:, 128:] == 3.0)  # not stored
    assert torch.equal(y[mp:, :128].view(torch.int16), alone[:, :128].view(torch.int16))
    assert torch.equal(y[:mp].view(torch.int16), prim.view(torch.int16))


def test_deterministic_and_inplace_residual(cuda_device):
    mp = ma = 64
    x, w, c, res = _case(8, mp, ma, 512, 4096, "residual", True)
    dev = cuda_device
    y1 = _gpu(dev, x, w, mp, "residual", c, res)
    y2 = _gpu(dev, x, w, mp, "residual", c, res)
    r = res.to(dev)
    api.grouped_proj(x.to(dev), mp, w.to(dev), epilogue="residual", coupling=c.to(dev), residual=r,
                     y=r)
    torch.cuda.synchronize()
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))
    assert torch.equal(y1.view(torch.int16), r.view(torch.int16))


def test_primary_rows_ignore_aux_rows_and_couplings(cuda_device):
    mp = ma = 64
    x, w, b, _ = _case(9, mp, ma, 512, 1024, "swiglu", True)
    dev = cuda_device
    y1 = _gpu(dev, x, w, mp, "swiglu", b, None)
    x2 = x.clone()
    x2[mp:] = float("nan")
    y2 = _gpu(dev, x2, w, mp, "swiglu", -b, None)
    torch.cuda.synchronize()
    assert torch.equal(y1[:mp].view(torch.int16), y2[:mp].view(torch.int16))


LAYER = synth.WORKLOADS["layer"]
FULL = [("qkv", "w_qkv", "none"), ("o", "w_o", "residual"), ("gu", "w_gu", "swiglu"),
        ("down", "w_down", "residual")]


@pytest.mark.parametrize("name,wkey,epi", FULL)
def test_full_size_layer_projections_sampled(cuda_device, name, wkey, epi):
    """The four shared-weight GEMMs of the 4096/14336 layer at M = 128 rows,
    checked on a sample of output columns (the oracle recomputes only those)."""
    g = torch.Generator().manual_seed(40)
    N, K = {"w_qkv": (6144, 4096), "w_o": (4096, 4096), "w_gu": (2 * 14336, 4096),
            "w_down": (4096, 14336)}[wkey]
    mp = ma = 64
    x = _rand(g, (128, K))
    w = _rand(g, (N, K), 0.02)
    n_out = N // 2 if epi == "swiglu" else N
    cpl = _rand(g, (n_out,), 0.1) if epi != "none" else None
    res = _rand(g, (128, n_out)) if epi == "residual" else None
    y = _gpu(cuda_device, x, w, mp, epi, cpl, res).cpu()
    torch.cuda.synchronize()
    cols = np.unique(np.concatenate([np.arange(0, 64), np.arange(n_out - 64, n_out),
                                     np.random.default_rng(0).integers(0, n_out, 256)]))
    if epi == "swiglu":
        wsel = torch.cat([w[cols], w[n_out + cols]])
        ref = _oracle(x, wsel, mp, "swiglu", cpl[cols], None)
    else:
        ref = _oracle(x, w[cols], mp, epi, None if cpl is None else cpl[cols],
                      None if res is None else res[:, cols])
    assert_close(y[:, cols], ref, "bf16", name)


MEDIUM = [  # (m_primary, m_aux, N, K): shapes that exercise the tile-parallel and
            # cluster split-K plans (several tiles, k-ranges split over clusters)
    (64, 64, 4096, 4096),
    (64, 64, 8192, 4096),
    (16, 16, 6144, 2048),
    (64, 64, 2048, 14336),
    (32, 32, 3200, 4096),   # tile width that does not divide N (tail tile)
]


@pytest.mark.parametrize("shape", MEDIUM)
@pytest.mark.parametrize("epi,coupled", [("none", False), ("swiglu", True), ("residual", True)])
def test_medium_shapes_sampled(cuda_device, shape, epi, coupled):
    mp, ma, N, K = shape
    g = torch.Generator().manual_seed(sum(shape) + len(epi))
    x = _rand(g, (mp + ma, K))
    w = _rand(g, (N, K), 0.02)
    n_out = N // 2 if epi == "swiglu" else N
    cpl = _rand(g, (n_out,), 0.1) if coupled else None
    res = _rand(g, (mp + ma, n_out)) if epi == "residual" else None
    y = _gpu(cuda_device, x, w, mp, epi, cpl, res).cpu()
    torch.cuda.synchronize()
    cols = np.unique(np.concatenate([np.arange(0, 48), np.arange(n_out - 48, n_out),
                                     np.random.default_rng(1).integers(0, n_out, 192)]))
    if epi == "swiglu":
        ref = _oracle(x, torch.cat([w[cols], w[n_out + cols]]), mp, "swiglu", cpl[cols], None)
    else:
        ref = _oracle(x, w[cols], mp, epi, None if cpl is None else cpl[cols],
                      None if res is None else res[:, cols])
    assert_close(y[:, cols], ref, "bf16", "medium %s %s" % (shape, epi))


@pytest.mark.parametrize("cur,nxt", [(("w_o", "residual"), ("w_gu", "swiglu")),
                                     (("w_gu", "swiglu"), ("w_down", "residual")),
                                     (("w_down", "residual"), ("w_qkv", "none"))])
def test_next_projection_hint_changes_no_bit(cuda_device, cur, nxt):
    """The chained entry (L2 prefetch of the next projection's first weight
    blocks) gives the same bits as the plain call, at the layer's shapes; the
    next projection, run after it, is unchanged too."""
    dev = cuda_device
    shapes = {"w_qkv": (6144, 4096), "w_o": (4096, 4096), "w_gu": (2 * 14336, 4096),
              "w_down": (4096, 14336)}
    g = torch.Generator().manual_seed(41)
    (wk, epi), (nk, nepi) = cur, nxt
    N, K = shapes[wk]
    Nn, Kn = shapes[nk]
    n_out = N // 2 if epi == "swiglu" else N
    x = _rand(g, (128, K)).to(dev)
    w = _rand(g, (N, K), 0.02).to(dev)
    wn = _rand(g, (Nn, Kn), 0.02).to(dev)
    xn = _rand(g, (128, Kn)).to(dev)
    cpl = _rand(g, (n_out,), 0.1).to(dev) if epi != "none" else None
    res = _rand(g, (128, n_out)).to(dev) if epi == "residual" else None
    ws = api.new_proj_workspace(128, max(N, Nn), max(K, Kn), "swiglu", dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    kw = dict(epilogue=epi, coupling=cpl, residual=res, workspace=ws, err_flag=err)
    y_plain = api.grouped_proj(x, 64, w, **kw)
    yn_plain = api.grouped_proj(xn, 64, wn, epilogue="none", workspace=ws, err_flag=err)
    y_hint = api.grouped_proj(x, 64, w, next_w=wn, next_epilogue=nepi, **kw)
    yn_hint = api.grouped_proj(xn, 64, wn, epilogue="none", workspace=ws, err_flag=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    assert torch.equal(y_plain.view(torch.int16), y_hint.view(torch.int16))
    assert torch.equal(yn_plain.view(torch.int16), yn_hint.view(torch.int16))


@pytest.mark.parametrize("batch,mp,ma,N,K,epi", [(3, 64, 64, 1024, 512, "swiglu"),
                                                 (8, 64, 64, 2048, 5632, "none"),
                                                 (8, 64, 64, 11264, 2048, "swiglu"),
                                                 (2, 5, 3, 256, 128, "none")])
def test_batched_projection_parity(cuda_device, batch, mp, ma, N, K, epi):
    """One launch for a batch of same-shape projections (the MoE experts):
    every entry matches the oracle, on sampled columns at the larger shapes."""
    g = torch.Generator().manual_seed(batch * 1000 + N)
    x = _rand(g, (batch, mp + ma, K))
    w = _rand(g, (batch, N, K), 0.02)
    err = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    y = api.grouped_proj_batched(x.to(cuda_device), mp, w.to(cuda_device), epilogue=epi,
                                 err_flag=err).cpu()
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    n_out = N // 2 if epi == "swiglu" else N
    cols = np.unique(np.concatenate([np.arange(0, min(48, n_out)),
                                     np.arange(max(0, n_out - 48), n_out),
                                     np.random.default_rng(2).integers(0, n_out, 128)]))
    for b in range(batch):
        if epi == "swiglu":
            ref = _oracle(x[b], torch.cat([w[b][cols], w[b][n_out + cols]]), mp, "swiglu", None, None)
        else:
            ref = _oracle(x[b], w[b][cols], mp, "none", None, None)
        assert_close(y[b][:, cols], ref, "bf16", "batched entry %d" % b)
