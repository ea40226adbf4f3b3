"""GPU parity of the decode-attention and KV-append path against the fp64 oracle.

Every call goes through the C ABI (ctypes binding). Inputs come from the seeded
generators; expected values from the oracle only.
"""

import dataclasses

import numpy as np
import pytest
import torch

import oracle
from dual_flow_transformer_b200 import api, synth
from dual_flow_transformer_b200 import _lib as L
from tests.helpers import assert_attn_close, oracle_attn, to_dev

pytestmark = pytest.mark.gpu

W = synth.WORKLOADS


def _small(name, **kw):
    return dataclasses.replace(W[name], **kw)


def _run(inp, dev, num_splits=0, primary_out=True, aux=True, err=None):
    """One decode_attn call. Without an `err` from the caller the device error
    flag (bad lengths or pages, a wait that gave up) must stay clear."""
    d = to_dev(inp, dev)
    max_len = int(inp["seqlens"].max())
    own = err is None
    if own:
        err = torch.zeros(1, dtype=torch.int32, device=dev)
    o1, o2 = api.decode_attn(d["q1"], d["q2raw"] if aux else None, d["a"] if aux else None,
                             d["k_cache"], d["v_cache"], d["block_table"], d["seqlens"], max_len,
                             primary_out=primary_out, num_splits=num_splits, err_flag=err)
    torch.cuda.synchronize()
    if own:
        assert int(err.item()) == 0, "device error flag %d" % int(err.item())
    return o1, o2


# ------------------------------------------------------------------ tiny fp32 workload

def test_tiny_fp32_append_then_attend(cuda_device):
    w = W["tiny"]
    inp = synth.make_attn_inputs(w)
    d = to_dev(inp, cuda_device)
    err = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    api.kv_append(d["k_new"], d["v_new"], d["k_cache"], d["v_cache"], d["block_table"],
                  d["positions"], err_flag=err)
    o1, o2 = api.decode_attn(d["q1"], d["q2raw"], d["a"], d["k_cache"], d["v_cache"],
                             d["block_table"], d["seqlens"], int(inp["seqlens"].max()),
                             err_flag=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    kc, vc = oracle.kv_append(inp["k_new"].numpy(), inp["v_new"].numpy(), inp["k_cache"].numpy(),
                              inp["v_cache"].numpy(), inp["block_table"].numpy(),
                              inp["positions"].numpy())
    assert d["k_cache"].cpu().numpy().tobytes() == kc.tobytes()
    assert d["v_cache"].cpu().numpy().tobytes() == vc.tobytes()
    r1, r2 = oracle.decode_attn(inp["q1"].numpy(), inp["q2raw"].numpy(), inp["a"].numpy(), kc, vc,
                                inp["block_table"].numpy(), inp["seqlens"].numpy())
    assert_attn_close(o1, r1, "fp32", "tiny o1")
    assert_attn_close(o2, r2, "fp32", "tiny o2")


@pytest.mark.parametrize("num_splits", [1, 2, 3])
def test_fp32_split_and_tail(cuda_device, num_splits):
    w = _small("tiny", B=3, Hq=4, Hkv=2, D=128, len_lo=1, len_hi=200, append=False, seed=11)
    inp = synth.make_attn_inputs(w)
    o1, o2 = _run(inp, cuda_device, num_splits=num_splits)
    r1, r2 = oracle_attn(inp)
    assert_attn_close(o1, r1, "fp32", "o1")
    assert_attn_close(o2, r2, "fp32", "o2")


# ------------------------------------------------------------------ bf16 reduced workloads

CASES = {
    # name: workload changes (several pages, ragged tails, random tables)
    "mha_small": dict(name="mha", B=4, Hq=4, Hkv=4, len_lo=300, len_hi=300, seed=21),
    "gqa_small": dict(name="gqa", B=6, Hq=8, Hkv=2, len_lo=1, len_hi=700, seed=22),
    "gqa_g2_d64": dict(name="gqa", B=5, Hq=4, Hkv=2, D=64, len_lo=1, len_hi=400, seed=23),
    "gqa_g3": dict(name="gqa", B=3, Hq=6, Hkv=2, len_lo=60, len_hi=260, seed=24),
    "long_small": dict(name="long", B=2, Hq=4, Hkv=1, len_lo=3000, len_hi=5100, seed=25),
    "edge_lengths": dict(name="gqa", B=8, Hq=8, Hkv=2, len_lo=1, len_hi=130, seed=26),
    # 16..63 pages per unit: several chunks per split at every split count
    "many_pages": dict(name="gqa", B=8, Hq=8, Hkv=2, len_lo=1000, len_hi=4000, seed=29),
}


@pytest.mark.parametrize("case", sorted(CASES))
@pytest.mark.parametrize("num_splits", [0, 1, 4])
def test_bf16_parity(cuda_device, case, num_splits):
    kw = dict(CASES[case])
    w = _small(kw.pop("name"), **kw)
    lengths = [1, 2, 63, 64, 65, 127, 128, 129] if case == "edge_lengths" else None
    inp = synth.make_attn_inputs(w, lengths=lengths)
    o1, o2 = _run(inp, cuda_device, num_splits=num_splits)
    r1, r2 = oracle_attn(inp)
    assert_attn_close(o1, r1, "bf16", case + " o1")
    assert_attn_close(o2, r2, "bf16", case + " o2")


@pytest.mark.parametrize("num_splits", [0, 1])
def test_bf16_workspace_reuse_is_deterministic(cuda_device, num_splits):
    """Back-to-back calls on one workspace give the same bits: the arrival
    counters return to zero after every call, every call rewrites the split
    partials it reads, and the combine order is fixed."""
    kw = dict(CASES["many_pages"])
    w = _small(kw.pop("name"), **kw)
    inp = synth.make_attn_inputs(w)
    d = to_dev(inp, cuda_device)
    max_len = int(inp["seqlens"].max())
    ws = api.new_attn_workspace(w.B, w.Hq, w.Hkv, w.D, max_len, num_splits, cuda_device)
    err = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    outs = []
    for _ in range(3):
        o1, o2 = api.decode_attn(d["q1"], d["q2raw"], d["a"], d["k_cache"], d["v_cache"],
                                 d["block_table"], d["seqlens"], max_len, num_splits=num_splits,
                                 workspace=ws, err_flag=err)
        outs.append((o1.clone(), o2.clone()))
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    for o1, o2 in outs[1:]:
        assert torch.equal(o1.view(torch.int16), outs[0][0].view(torch.int16))
        assert torch.equal(o2.view(torch.int16), outs[0][1].view(torch.int16))
    r1, r2 = oracle_attn(inp)
    assert_attn_close(outs[0][0], r1, "bf16", "o1")
    assert_attn_close(outs[0][1], r2, "bf16", "o2")


def test_bf16_stale_nan_tail_slots_do_not_leak(cuda_device):
    """Slots past each sequence's end hold NaN bit patterns: masked tokens
    (zero weight) must not turn the output into NaN."""
    w = _small("gqa", B=4, Hq=8, Hkv=2, len_lo=70, len_hi=190, seed=27)
    inp = synth.make_attn_inputs(w)
    kc, vc, tbl, sl = inp["k_cache"], inp["v_cache"], inp["block_table"], inp["seqlens"]
    for b in range(w.B):
        L_b = int(sl[b])
        last = int(tbl[b, (L_b - 1) // 64])
        kc[last, :, L_b % 64 or 64:] = float("nan")
        vc[last, :, L_b % 64 or 64:] = float("nan")
    o1, o2 = _run(inp, cuda_device)
    r1, r2 = oracle_attn(inp)
    assert_attn_close(o1, r1, "bf16", "o1")
    assert_attn_close(o2, r2, "bf16", "o2")


# ------------------------------------------------------------------ asymmetry invariants

def test_primary_output_bit_identical_whatever_the_aux_inputs(cuda_device):
    w = _small("gqa", B=6, Hq=8, Hkv=2, len_lo=100, len_hi=900, seed=28)
    inp = synth.make_attn_inputs(w)
    base, _ = _run(inp, cuda_device, aux=False)
    dual, _ = _run(inp, cuda_device)
    bad = dict(inp)
    bad["q2raw"] = inp["q2raw"].clone()
    bad["q2raw"][0, 1, 5] = float("nan")
    bad["q2raw"][2, 3, 0] = float("inf")
    bad["a"] = inp["a"].clone()
    bad["a"][4, 7] = float("nan")
    noisy, o2bad = _run(bad, cuda_device)
    other = dict(inp)
    other["q2raw"] = inp["q2raw"] * 3
    other["a"] = -inp["a"]
    shifted, _ = _run(other, cuda_device)
    for t in (dual, noisy, shifted):
        assert torch.equal(t.view(torch.int16), base.view(torch.int16))
    assert torch.isnan(o2bad[0].float()).any()


def test_aux_only_call_leaves_cache_and_primary_output_untouched(cuda_device):
    w = _small("gqa", B=3, Hq=8, Hkv=2, len_lo=100, len_hi=300, seed=29)
    inp = synth.make_attn_inputs(w)
    d = to_dev(inp, cuda_device)
    kbytes = d["k_cache"].view(torch.int16).clone()
    vbytes = d["v_cache"].view(torch.int16).clone()
    sentinel = torch.full_like(d["q1"], 7.0)
    o1, o2 = api.decode_attn(d["q1"], d["q2raw"], d["a"], d["k_cache"], d["v_cache"],
                             d["block_table"], d["seqlens"], int(inp["seqlens"].max()),
                             primary_out=False)
    torch.cuda.synchronize()
    assert o1 is None
    assert torch.equal(d["k_cache"].view(torch.int16), kbytes)
    assert torch.equal(d["v_cache"].view(torch.int16), vbytes)
    assert torch.equal(sentinel, torch.full_like(d["q1"], 7.0))
    _, r2 = oracle_attn(inp)
    assert_attn_close(o2, r2, "bf16", "aux-only o2")


def test_split_count_independent_of_aux_inputs():
    for B, Hkv, L in [(1, 1, 129), (64, 8, 4097), (8, 8, 131072), (32, 32, 2048)]:
        assert api.decode_attn_num_splits(B, Hkv, L) >= 1


# ------------------------------------------------------------------ device-side errors

def test_bad_lengths_and_pages_are_flagged_not_trapped(cuda_device):
    w = _small("gqa", B=3, Hq=8, Hkv=2, len_lo=100, len_hi=200, seed=30)
    inp = synth.make_attn_inputs(w)
    inp["seqlens"][1] = 0
    err = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    o1, o2 = _run(inp, cuda_device, err=err, num_splits=1)
    assert int(err.item()) & L.DF_DEVERR_SEQLEN
    assert torch.count_nonzero(o1[1]) == 0 and torch.count_nonzero(o2[1]) == 0
    good = [0, 2]
    r1, r2 = oracle_attn(inp, batches=good)
    assert_attn_close(o1[good], r1, "bf16", "o1 of good sequences")
    bad = synth.make_attn_inputs(w)
    bad["block_table"][2, 0] = 10 ** 6
    err.zero_()
    _run(bad, cuda_device, err=err)
    assert int(err.item()) & L.DF_DEVERR_BLOCK


def test_append_bad_position_flagged(cuda_device):
    w = W["tiny"]
    inp = synth.make_attn_inputs(w)
    d = to_dev(inp, cuda_device)
    before = d["k_cache"].clone()
    d["positions"][0] = 10 ** 6
    err = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    api.kv_append(d["k_new"], d["v_new"], d["k_cache"], d["v_cache"], d["block_table"],
                  d["positions"], err_flag=err)
    torch.cuda.synchronize()
    assert int(err.item()) & L.DF_DEVERR_POSITION
    assert torch.equal(before, d["k_cache"])


# ------------------------------------------------------------------ append, bf16, strided source

def test_bf16_append_from_strided_rows_bit_exact(cuda_device):
    g = torch.Generator().manual_seed(31)
    B, Hkv, D = 5, 2, 128
    table, nblocks = synth.make_block_table(g, [300, 10, 64, 65, 1], random_table=True)
    kc = torch.randn(nblocks, Hkv, 64, D, generator=g).to(torch.bfloat16)
    vc = torch.randn(nblocks, Hkv, 64, D, generator=g).to(torch.bfloat16)
    wide = torch.randn(B, 3 * Hkv * D, generator=g).to(torch.bfloat16)  # like a fused QKV row
    k_new = wide[:, Hkv * D:2 * Hkv * D].view(B, Hkv, D)
    v_new = wide[:, 2 * Hkv * D:].view(B, Hkv, D)
    pos = torch.tensor([299, 9, 63, 64, 0], dtype=torch.int32)
    dev = cuda_device
    dkc, dvc, dwide = kc.to(dev), vc.to(dev), wide.to(dev)
    api.kv_append(dwide[:, Hkv * D:2 * Hkv * D].view(B, Hkv, D), dwide[:, 2 * Hkv * D:].view(B, Hkv, D),
                  dkc, dvc, table.to(dev), pos.to(dev))
    torch.cuda.synchronize()
    ek, ev = oracle.kv_append(k_new.view(torch.int16).numpy(), v_new.view(torch.int16).numpy(),
                              kc.view(torch.int16).numpy(), vc.view(torch.int16).numpy(),
                              table.numpy(), pos.numpy())
    assert dkc.cpu().view(torch.int16).numpy().tobytes() == ek.tobytes()
    assert dvc.cpu().view(torch.int16).numpy().tobytes() == ev.tobytes()


# ------------------------------------------------------------------ full-size workloads

@pytest.mark.parametrize("name", ["mha", "gqa", "long"])
def test_full_size_workloads_every_sequence(cuda_device, name):
    """The full attention workloads in the launch configuration the benchmark
    times; the oracle recomputes every sequence (every split count and tail)."""
    w = W[name]
    inp = synth.make_attn_inputs(w)
    o1, o2 = _run(inp, cuda_device)
    r1, r2 = oracle_attn(inp)
    assert_attn_close(o1, r1, "bf16", "full %s O1" % name)
    assert_attn_close(o2, r2, "bf16", "full %s O2" % name)


def test_tiny_workload_reported(cuda_device):
    """The fp32 tiny workload (append, then attention over 129 tokens) in the
    parity summary beside the full-size ones."""
    w = W["tiny"]
    inp = synth.make_attn_inputs(w)
    d = to_dev(inp, cuda_device)
    api.kv_append(d["k_new"], d["v_new"], d["k_cache"], d["v_cache"], d["block_table"],
                  d["positions"])
    o1, o2 = api.decode_attn(d["q1"], d["q2raw"], d["a"], d["k_cache"], d["v_cache"],
                             d["block_table"], d["seqlens"], int(inp["seqlens"].max()))
    torch.cuda.synchronize()
    kc, vc = oracle.kv_append(inp["k_new"].numpy(), inp["v_new"].numpy(), inp["k_cache"].numpy(),
                              inp["v_cache"].numpy(), inp["block_table"].numpy(),
                              inp["positions"].numpy())
    r1, r2 = oracle.decode_attn(inp["q1"].numpy(), inp["q2raw"].numpy(), inp["a"].numpy(), kc, vc,
                                inp["block_table"].numpy(), inp["seqlens"].numpy())
    assert_attn_close(o1, r1, "fp32", "full tiny O1")
    assert_attn_close(o2, r2, "fp32", "full tiny O2")


@pytest.mark.parametrize("num_splits", [0, 1])
def test_permuting_the_batch_permutes_the_outputs(cuda_device, num_splits):
    """Every sequence's outputs depend on that sequence alone, whatever order
    the grid takes the sequences in (unsplit plans take them longest first,
    ties in index order): the batch reversed gives the outputs reversed, bit
    for bit. Ragged lengths with ties; 40 sequences x 8 KV heads = 320 units,
    one CTA each in the automatic plan."""
    w = _small("gqa", B=40, Hq=16, Hkv=8, len_lo=64, len_hi=700, seed=31)
    lengths = [300, 64, 700, 300, 65, 700, 128, 1, 511, 300] * 4
    inp = synth.make_attn_inputs(w, lengths=lengths)
    perm = torch.arange(len(lengths) - 1, -1, -1)
    rev = dict(inp)
    for k in ("q1", "q2raw", "block_table", "seqlens"):
        rev[k] = inp[k][perm].contiguous()
    o1, o2 = _run(inp, cuda_device, num_splits=num_splits)
    r1, r2 = _run(rev, cuda_device, num_splits=num_splits)
    dev_perm = perm.to(cuda_device)
    assert torch.equal(r1, o1[dev_perm]) and torch.equal(r2, o2[dev_perm])
    r1o, r2o = oracle_attn(inp)
    assert_attn_close(o1, r1o, "bf16", "permuted batch o1")
    assert_attn_close(o2, r2o, "bf16", "permuted batch o2")
