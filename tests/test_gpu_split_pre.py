"""GPU checks of the split pre-attention path: the QKV partial products of
the 4 quarters of d_model (dualflow_layer_qkv_partials) and the attention
launch that reduces, normalises, rounds and appends them in its prologue
(dualflow_decode_attn_qkv_partials).

The pair must give, bit for bit, what the one-launch pre-attention
(dualflow_layer_pre_attention) followed by dualflow_decode_attn gives: the
outputs of both flows and the whole cache. The partial products themselves
are checked against the fp64 oracle's product of each quarter.
"""

import dataclasses

import numpy as np
import pytest
import torch

import oracle
from dual_flow_transformer_b200 import _lib as L
from dual_flow_transformer_b200 import api, synth
from tests.helpers import assert_close, f64

pytestmark = pytest.mark.gpu

BASE = synth.WORKLOADS["layer"]
SHAPES = {
    "small": dataclasses.replace(BASE, B=8, d_model=512, Hq=4, Hkv=2, D=128, cache_len=200,
                                 seed=80),
    # D = 64, 5 sequences, one KV head for two query heads
    "odd": dataclasses.replace(BASE, B=5, d_model=256, Hq=2, Hkv=1, D=64, cache_len=70,
                               seed=81),
    # d_model 64: one k-block, three of the four quarters are empty (zeros)
    "one_kblock": dataclasses.replace(BASE, B=3, d_model=64, Hq=2, Hkv=2, D=64, cache_len=10,
                                      seed=82),
    "gqa": dataclasses.replace(BASE, B=16, d_model=1024, Hq=8, Hkv=2, D=128, cache_len=330,
                               seed=83),
    # one query head per KV head: threads that append K / V own no Q columns
    "g1": dataclasses.replace(BASE, B=6, d_model=256, Hq=4, Hkv=4, D=128, cache_len=140,
                              seed=84),
}


def _dev(inp, dev, positions=None):
    keys = ("x1", "x2", "w_qkv", "k_cache", "v_cache", "block_table", "positions", "a")
    d = {k: inp[k].to(dev).contiguous() for k in keys}
    if positions is not None:
        d["positions"] = torch.tensor(positions, dtype=torch.int32, device=dev)
    d["X"] = torch.cat([d["x1"], d["x2"]]).contiguous()
    d["seqlens"] = (d["positions"] + 1).to(torch.int32)
    return d


def _ragged_positions(w):
    """Append positions that start a page (0, 64, 128, ...), end one (63,
    127, ...), the first token (sequence length 1) and the table's last slot,
    cycled over the sequences."""
    cands = [w.cache_len, 0, 63, 64, 127, 128, 1, w.cache_len - 1]
    return [min(cands[i % len(cands)], w.cache_len) for i in range(w.B)]


def _split_path(d, w, dual=True, num_splits=0, err=None):
    part, ss = api.layer_qkv_partials(d["X"], d["w_qkv"], w.Hq, w.Hkv, w.D, err_flag=err)
    max_seqlen = int(d["seqlens"].max())
    o1, o2 = api.decode_attn_qkv_partials(part, ss, w.d_model, d["a"], d["k_cache"],
                                          d["v_cache"], d["block_table"], d["seqlens"],
                                          max_seqlen, w.Hq, dual=dual, num_splits=num_splits,
                                          err_flag=err)
    return o1, o2, part, ss


def _fused_path(d, w, dual=True, num_splits=0, err=None):
    B, qd = w.B, w.Hq * w.D
    qkv = api.layer_pre_attention(d["X"], d["w_qkv"], w.Hq, w.Hkv, d["k_cache"], d["v_cache"],
                                  d["block_table"], d["positions"], err_flag=err)
    max_seqlen = int(d["seqlens"].max())
    o1, o2 = api.decode_attn(qkv[:B, :qd].view(B, w.Hq, w.D),
                             qkv[B:, :qd].view(B, w.Hq, w.D) if dual else None, d["a"],
                             d["k_cache"], d["v_cache"], d["block_table"], d["seqlens"],
                             max_seqlen, num_splits=num_splits, err_flag=err)
    return o1, o2, qkv


def _bits(t):
    return t.contiguous().view(torch.int16).cpu()


def _both(inp, w, dev, positions=None, dual=True, num_splits=0):
    ds = _dev(inp, dev, positions)
    df = _dev(inp, dev, positions)
    e1 = torch.zeros(1, dtype=torch.int32, device=dev)
    e2 = torch.zeros(1, dtype=torch.int32, device=dev)
    s = _split_path(ds, w, dual, num_splits, e1)
    f = _fused_path(df, w, dual, num_splits, e2)
    torch.cuda.synchronize()
    assert int(e1.item()) == 0 and int(e2.item()) == 0
    return ds, df, s, f


@pytest.mark.parametrize("name", sorted(SHAPES))
def test_partials_are_the_quarter_products(cuda_device, name):
    """part[k] = x[:, quarter k] W_qkv[:, quarter k]^T and ss[k] the quarter's
    row sums of squares, against fp64 (fp32 summation bound); summed in
    quarter order from zero and scaled by the row scale they give the
    one-launch pre-attention's qkv bit for bit."""
    w = SHAPES[name]
    inp = synth.make_layer_inputs(w)
    d = _dev(inp, cuda_device)
    err = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    part, ss = api.layer_qkv_partials(d["X"], d["w_qkv"], w.Hq, w.Hkv, w.D, err_flag=err)
    qkv = api.layer_pre_attention(d["X"], d["w_qkv"], w.Hq, w.Hkv, d["k_cache"].clone(),
                                  d["v_cache"].clone(), d["block_table"], d["positions"])
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    X = np.concatenate([f64(inp["x1"]), f64(inp["x2"])])
    W = f64(inp["w_qkv"])
    kb = w.d_model // 64
    got_p = part.cpu().double().numpy()
    got_s = ss.cpu().double().numpy()
    for k in range(4):
        c0, c1 = 64 * (k * kb // 4), 64 * ((k + 1) * kb // 4)
        ref = X[:, c0:c1] @ W[:, c0:c1].T
        bound = (np.abs(X[:, c0:c1]) @ np.abs(W[:, c0:c1]).T) * (c1 - c0 + 1) * 2.0 ** -23
        assert np.all(np.abs(got_p[k] - ref) <= bound + 1e-30), (name, k)
        refs = (X[:, c0:c1] ** 2).sum(axis=1)
        assert np.all(np.abs(got_s[k] - refs) <= refs * (c1 - c0 + 1) * 2.0 ** -23 + 1e-30)
    # the reduction the attention prologue performs, written out in fp32
    pt = part.cpu()
    acc = torch.zeros_like(pt[0])
    sst = torch.zeros_like(ss.cpu()[0])
    for k in range(4):
        acc = acc + pt[k]
        sst = sst + ss.cpu()[k]
    r = 1.0 / torch.sqrt(sst / float(w.d_model) + torch.tensor(1e-5, dtype=torch.float32))
    want = (acc * r[:, None]).to(torch.bfloat16)
    B, qd = w.B, w.Hq * w.D
    g = qkv.cpu()
    assert torch.equal(_bits(want[:B]), _bits(g[:B])), name
    assert torch.equal(_bits(want[B:, :qd]), _bits(g[B:, :qd])), name


@pytest.mark.parametrize("num_splits", [0, 1, 3])
@pytest.mark.parametrize("name", ["small", "odd", "gqa", "g1", "one_kblock"])
def test_split_path_bit_identical_to_fused_pre(cuda_device, name, num_splits):
    w = SHAPES[name]
    inp = synth.make_layer_inputs(w)
    ds, df, s, f = _both(inp, w, cuda_device, positions=_ragged_positions(w),
                         num_splits=num_splits)
    assert torch.equal(_bits(s[0]), _bits(f[0])), "O1"
    assert torch.equal(_bits(s[1]), _bits(f[1])), "O2"
    assert torch.equal(_bits(ds["k_cache"]), _bits(df["k_cache"])), "K cache"
    assert torch.equal(_bits(ds["v_cache"]), _bits(df["v_cache"])), "V cache"


def test_split_path_primary_only(cuda_device):
    w = SHAPES["small"]
    inp = synth.make_layer_inputs(w)
    ds, df, s, f = _both(inp, w, cuda_device, dual=False)
    assert s[1] is None and f[1] is None
    assert torch.equal(_bits(s[0]), _bits(f[0]))
    assert torch.equal(_bits(ds["k_cache"]), _bits(df["k_cache"]))


def test_split_path_matches_oracle_attention(cuda_device):
    """O1 / O2 of the split path against the oracle's attention over the
    cache the path wrote (its Q rows from the oracle's norm and projection):
    bf16 tolerance."""
    w = SHAPES["small"]
    inp = synth.make_layer_inputs(w)
    pos = _ragged_positions(w)
    d = _dev(inp, cuda_device, pos)
    o1, o2, _, _ = _split_path(d, w)
    torch.cuda.synchronize()
    B, qd = w.B, w.Hq * w.D
    X = np.concatenate([f64(inp["x1"]), f64(inp["x2"])])
    qkv = oracle.bf16_round(oracle.grouped_proj(oracle.rmsnorm(X, eps=1e-5), f64(inp["w_qkv"]),
                                                B, n_aux=qd))
    kc = synth.to_numpy_f32(d["k_cache"].cpu())
    vc = synth.to_numpy_f32(d["v_cache"].cpu())
    r1, r2 = oracle.decode_attn(qkv[:B, :qd].reshape(B, w.Hq, w.D),
                                qkv[B:, :qd].reshape(B, w.Hq, w.D), f64(inp["a"]), kc, vc,
                                inp["block_table"].numpy(), np.asarray(pos) + 1)
    assert_close(o1.cpu(), r1, "bf16", "split-path O1")
    assert_close(o2.cpu(), r2, "bf16", "split-path O2")


def test_split_path_full_size_layer(cuda_device):
    """d_model 4096, 32 / 8 heads, 64 sequences, cache 4096 + 1: the launch
    configuration the layer step uses."""
    w = BASE
    inp = synth.make_layer_inputs(w)
    ds, df, s, f = _both(inp, w, cuda_device)
    assert torch.equal(_bits(s[0]), _bits(f[0]))
    assert torch.equal(_bits(s[1]), _bits(f[1]))
    assert torch.equal(_bits(ds["k_cache"]), _bits(df["k_cache"]))
    assert torch.equal(_bits(ds["v_cache"]), _bits(df["v_cache"]))


def test_split_path_flags_out_of_table_append_page(cuda_device):
    """The page holding sequence 0's new position is outside the pool: the
    append and that page's load are skipped and DF_DEVERR_BLOCK is set; the
    other sequences are unaffected."""
    w = SHAPES["small"]
    inp = synth.make_layer_inputs(w)
    d = _dev(inp, cuda_device)
    ref = _dev(inp, cuda_device)
    pos0 = int(d["positions"][0])
    nb = d["k_cache"].shape[0]
    d["block_table"][0, pos0 // 64] = nb
    err = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    o1, o2, _, _ = _split_path(d, w, err=err)
    r = _split_path(ref, w)
    torch.cuda.synchronize()
    assert int(err.item()) & L.DF_DEVERR_BLOCK
    assert torch.equal(_bits(o1[1:]), _bits(r[0][1:]))
    assert torch.equal(_bits(o2[1:]), _bits(r[1][1:]))


def test_split_path_rejects_bad_arguments(cuda_device):
    w = SHAPES["small"]
    inp = synth.make_layer_inputs(w)
    d = _dev(inp, cuda_device)
    part, ss = api.layer_qkv_partials(d["X"], d["w_qkv"], w.Hq, w.Hkv, w.D)
    lib = L.load()
    B = w.B
    o1 = torch.empty(B, w.Hq, w.D, dtype=torch.bfloat16, device=cuda_device)
    args = dict(part=part.data_ptr(), ss=ss.data_ptr(), parts=4, m=B, dm=w.d_model)

    def call(**kw):
        a = dict(args, **kw)
        return lib.dualflow_decode_attn_qkv_partials(
            a["part"], a["ss"], a["parts"], a["m"], a["dm"], 1e-5, None,
            d["k_cache"].data_ptr(), d["v_cache"].data_ptr(), d["block_table"].data_ptr(),
            d["block_table"].shape[1], d["seqlens"].data_ptr(), int(d["seqlens"].max()),
            o1.data_ptr(), None, 0, w.Hq, w.Hkv, w.D, 64, d["k_cache"].shape[0], 0.0, 1,
            None, 0, None, None)

    assert call(part=None) == L.DF_ERR_NULL
    assert call(parts=0) == L.DF_ERR_SHAPE
    assert call(parts=5) == L.DF_ERR_SHAPE
    assert call(part=part.data_ptr() + 4) == L.DF_ERR_ALIGN
    assert lib.dualflow_layer_qkv_partials(d["X"].data_ptr(), d["w_qkv"].data_ptr(), B,
                                           w.d_model, w.Hq, w.Hkv, w.D, part.data_ptr() + 4,
                                           ss.data_ptr(), None, None) == L.DF_ERR_ALIGN
    torch.cuda.synchronize()
