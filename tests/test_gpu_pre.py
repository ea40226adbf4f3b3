"""GPU parity of the one-launch pre-attention half of the decoder layer
(RMSNorm, grouped QKV projection, primary-only KV append), through the C ABI,
against the fp64 oracle (qkv rounded to bf16 where the kernel stores it; the
kernel applies the norm's row scale to the accumulator, so the normalised rows
are not rounded) and against the three-call form.
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
                                 seed=70),
    # D = 64, 5 sequences (rows past M in the tile), a 1-KV-head group
    "odd": dataclasses.replace(BASE, B=5, d_model=256, Hq=2, Hkv=1, D=64, cache_len=70,
                               seed=71),
    # d_model 64: one k-block, so three of a cluster's four ranks have none
    "one_kblock": dataclasses.replace(BASE, B=3, d_model=64, Hq=2, Hkv=2, D=64, cache_len=10,
                                      seed=72),
    "gqa": dataclasses.replace(BASE, B=16, d_model=1024, Hq=8, Hkv=2, D=128, cache_len=130,
                               seed=73),
}


def _inputs(w):
    return synth.make_layer_inputs(w)


def _dev(inp, dev):
    keys = ("x1", "x2", "w_qkv", "k_cache", "v_cache", "block_table", "positions")
    d = {k: inp[k].to(dev).contiguous() for k in keys}
    d["X"] = torch.cat([d["x1"], d["x2"]]).contiguous()
    return d


def _oracle(inp, rows=None):
    """qkv of the oracle's norm + grouped projection (normalised rows kept in
    fp64, qkv rounded to bf16) for the selected sequences."""
    B, qd = inp["B"], inp["Hq"] * inp["D"]
    sel = np.arange(B) if rows is None else np.asarray(rows)
    X = np.concatenate([f64(inp["x1"])[sel], f64(inp["x2"])[sel]])
    xn = oracle.rmsnorm(X, eps=1e-5)
    qkv = oracle.bf16_round(oracle.grouped_proj(xn, f64(inp["w_qkv"]), len(sel), n_aux=qd))
    return qkv


def _run(d, inp, qkv=None, err=None):
    return api.layer_pre_attention(d["X"], d["w_qkv"], inp["Hq"], inp["Hkv"], d["k_cache"],
                                   d["v_cache"], d["block_table"], d["positions"], qkv=qkv,
                                   err_flag=err)


@pytest.mark.parametrize("name", sorted(SHAPES))
def test_pre_attention_matches_oracle_and_appends(cuda_device, name):
    w = SHAPES[name]
    inp = _inputs(w)
    d = _dev(inp, cuda_device)
    B, qd, kvd = inp["B"], inp["Hq"] * inp["D"], inp["Hkv"] * inp["D"]
    nout = qd + 2 * kvd
    assert api.layer_pre_attention_supported(B, w.d_model, w.Hq, w.Hkv, w.D)
    sentinel = torch.full((2 * B, nout), 7.0, dtype=torch.bfloat16, device=cuda_device)
    err = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    k_before, v_before = d["k_cache"].clone(), d["v_cache"].clone()
    qkv = _run(d, inp, qkv=sentinel, err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    ref = _oracle(inp)
    got = qkv.cpu()
    assert_close(got[:B], ref[:B], "bf16", "%s qkv primary" % name)
    assert_close(got[B:, :qd], ref[B:, :qd], "bf16", "%s qkv aux Q" % name)
    # auxiliary rows' K / V columns are never written
    assert torch.all(got[B:, qd:] == 7.0)
    # the append: the primary K / V columns, bit for bit, and nothing else
    # (as 16-bit patterns: the oracle's append is a plain element copy)
    bits = lambda t: t.contiguous().view(torch.int16).numpy()  # noqa: E731
    k_new = got[:B, qd:qd + kvd].reshape(B, inp["Hkv"], inp["D"])
    v_new = got[:B, qd + kvd:].reshape(B, inp["Hkv"], inp["D"])
    k_exp, v_exp = oracle.kv_append(bits(k_new), bits(v_new), bits(k_before.cpu()),
                                    bits(v_before.cpu()), inp["block_table"].numpy(),
                                    inp["positions"].numpy())
    assert np.array_equal(bits(d["k_cache"].cpu()), k_exp)
    assert np.array_equal(bits(d["v_cache"].cpu()), v_exp)


def test_pre_attention_matches_the_three_call_form(cuda_device):
    w = SHAPES["gqa"]
    inp = _inputs(w)
    d = _dev(inp, cuda_device)
    B, qd = inp["B"], inp["Hq"] * inp["D"]
    qkv = _run(d, inp)
    xn = api.rmsnorm(d["X"])
    ref = api.grouped_proj(xn, B, d["w_qkv"], n_aux=qd)
    torch.cuda.synchronize()
    assert_close(qkv[:B].cpu(), f64(ref[:B].cpu()), "bf16", "three-call qkv primary")
    assert_close(qkv[B:, :qd].cpu(), f64(ref[B:, :qd].cpu()), "bf16", "three-call qkv aux Q")


def test_pre_attention_deterministic_and_primary_blind(cuda_device):
    w = SHAPES["small"]
    inp = _inputs(w)
    d = _dev(inp, cuda_device)
    B, qd = inp["B"], inp["Hq"] * inp["D"]
    outs = [_run(d, inp).clone() for _ in range(3)]
    torch.cuda.synchronize()
    for o in outs[1:]:
        assert torch.equal(o.view(torch.int16), outs[0].view(torch.int16))
    k_ref, v_ref = d["k_cache"].clone(), d["v_cache"].clone()
    # auxiliary inputs do not reach the primary rows or the cache
    d2 = dict(d)
    d2["X"] = d["X"].clone()
    d2["X"][B:] = float("nan")
    y = _run(d2, inp)
    torch.cuda.synchronize()
    assert torch.equal(y[:B].view(torch.int16), outs[0][:B].view(torch.int16))
    assert torch.isnan(y[B:, :qd].float()).all()
    assert torch.equal(d["k_cache"], k_ref) and torch.equal(d["v_cache"], v_ref)


def test_pre_attention_full_size_layer_shapes(cuda_device):
    """d_model 4096, 32 query / 8 KV heads of 128, 64 sequences per flow, cache
    4096 + 1 (the layer workload): the oracle recomputes 8 sequences; the
    append is checked for every sequence."""
    inp = _inputs(BASE)
    d = _dev(inp, cuda_device)
    B, qd, kvd = inp["B"], inp["Hq"] * inp["D"], inp["Hkv"] * inp["D"]
    err = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    qkv = _run(d, inp, err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    rows = [0, 9, 31, 63]
    ref = _oracle(inp, rows)
    got = qkv.cpu()
    assert_close(got[rows], ref[:len(rows)], "bf16", "full pre qkv primary")
    assert_close(got[[B + r for r in rows], :qd], ref[len(rows):, :qd], "bf16",
                 "full pre qkv aux Q")
    pos, table = inp["positions"].numpy(), inp["block_table"].numpy()
    kc, vc = d["k_cache"], d["v_cache"]
    for b in range(B):
        p = int(pos[b])
        page = int(table[b][p // synth.BLOCK_SIZE])
        slot = p % synth.BLOCK_SIZE
        assert torch.equal(kc[page, :, slot, :].cpu(),
                           got[b, qd:qd + kvd].view(inp["Hkv"], inp["D"]))
        assert torch.equal(vc[page, :, slot, :].cpu(),
                           got[b, qd + kvd:].view(inp["Hkv"], inp["D"]))


def test_pre_attention_flags_out_of_table_position(cuda_device):
    w = SHAPES["small"]
    inp = _inputs(w)
    d = _dev(inp, cuda_device)
    d["positions"][3] = -1
    k_ref = d["k_cache"].clone()
    err = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    qkv = _run(d, inp, err=err)
    torch.cuda.synchronize()
    assert int(err.item()) & L.DF_DEVERR_POSITION
    # the other sequences' slots are written; sequence 3 writes nothing
    B = inp["B"]
    table, pos = inp["block_table"].numpy(), inp["positions"].numpy()
    changed = torch.nonzero((d["k_cache"] != k_ref).flatten(1).any(1)).flatten().tolist()
    written = {int(table[b][int(pos[b]) // synth.BLOCK_SIZE]) for b in range(B) if b != 3}
    assert set(changed) <= written
    assert torch.isfinite(qkv[:B].float()).all()


def test_pre_attention_rejects_unsupported_sizes(cuda_device):
    assert not api.layer_pre_attention_supported(65, 512, 4, 2, 128)
    assert not api.layer_pre_attention_supported(8, 500, 4, 2, 128)
    assert not api.layer_pre_attention_supported(8, 512, 4, 2, 4)
    # N = (Hq + 2 Hkv) D above 256 columns per co-resident cluster
    assert not api.layer_pre_attention_supported(8, 512, 128, 8, 128)
    w = SHAPES["small"]
    inp = _inputs(w)
    d = _dev(inp, cuda_device)
    qkv = torch.empty(2 * 65, 1024, dtype=torch.bfloat16, device=cuda_device)
    x = torch.zeros(2 * 65, 512, dtype=torch.bfloat16, device=cuda_device)
    p = api._ptr
    st = L.load().dualflow_layer_pre_attention(
        p(x), p(d["w_qkv"]), 65, 512, 4, 2, 128, 1e-5, p(qkv), p(d["k_cache"]), p(d["v_cache"]),
        p(d["block_table"]), d["block_table"].shape[1], p(d["positions"]), synth.BLOCK_SIZE,
        d["k_cache"].shape[0], None, None)
    assert st == L.DF_ERR_UNSUPPORTED
