"""GPU parity of the primary prefill (cache write, causal attention, auxiliary
query at the last prompt position) against the fp64 oracle, through the C ABI.

Inputs come from the seeded generators; expected values from the oracle only.
"""

import dataclasses
import math

import numpy as np
import pytest
import torch

import oracle
from dual_flow_transformer_b200 import api, synth
from dual_flow_transformer_b200 import _lib as L
from tests.helpers import assert_attn_close

pytestmark = pytest.mark.gpu

W = synth.WORKLOADS["prefill"]
f32 = synth.to_numpy_f32


def _w(**kw):
    return dataclasses.replace(W, **kw)


def _dev(inp, dev):
    return {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}


def _run(d, aux=True, append=True, err=None, check_err=True, **kw):
    own = err is None
    if own:
        err = torch.zeros(1, dtype=torch.int32, device=d["q1"].device)
    o1, o2 = api.prefill(d["q1"], d["k_new"] if append else None, d["v_new"] if append else None,
                         d["k_cache"], d["v_cache"], d["block_table"], d["cu_seqlens"],
                         d["max_q_len"], d["max_seqlen"], ctx_lens=d["ctx_lens"],
                         q2raw=d["q2raw"] if aux else None, a=d["a"] if aux else None,
                         err_flag=err, **kw)
    torch.cuda.synchronize()
    if own and check_err:
        assert int(err.item()) == 0, "device error flag %d" % int(err.item())
    return o1, o2


def _oracle(inp, aux=True):
    return oracle.prefill(f32(inp["q1"]), f32(inp["k_new"]), f32(inp["v_new"]),
                          f32(inp["k_cache"]), f32(inp["v_cache"]), inp["block_table"].numpy(),
                          inp["cu_seqlens"].numpy(), inp["ctx_lens"].numpy(),
                          q2raw=f32(inp["q2raw"]) if aux else None,
                          a=f32(inp["a"]) if aux else None)


def _check_all(inp, d, o1, o2, what):
    r1, r2, kc, vc = _oracle(inp, aux=o2 is not None)
    assert_attn_close(o1, r1, "bf16", what + " O1")
    if o2 is not None:
        assert_attn_close(o2, r2, "bf16", what + " O2")
    # byte copies: equal values, NaN slots (stale-slot tests) equal as NaN
    assert np.array_equal(f32(d["k_cache"]), kc, equal_nan=True), what + ": K cache differs"
    assert np.array_equal(f32(d["v_cache"]), vc, equal_nan=True), what + ": V cache differs"
    return r1, r2


KERNELS = ["mma_sync", "tcgen05"]


@pytest.mark.parametrize("kernel", KERNELS)
@pytest.mark.parametrize("Hq,Hkv,D,lengths,ctx", [
    (8, 2, 128, (1, 63, 65, 200), (0, 37, 64, 130)),   # ragged chunks, prefixes, tile edges
    (16, 4, 64, (130, 7), (0, 0)),                     # D 64, 4 query heads per KV head
    (8, 2, 64, (300, 129, 1), (40, 0, 7)),             # D 64: row tiles, prefixes, one token
    (4, 4, 128, (256, 129), (0, 0)),                   # MHA, fresh prompts
    (6, 2, 128, (64, 128, 191), (1, 63, 0)),           # G = 3
    (8, 2, 128, (127, 128, 129, 300), (0, 5, 200, 64)),  # 128-row tile edges
    # odd groups: the tcgen05 kernel pairs row tiles 2y, 2y + 1 of one head
    # (different causal ends; 3 tiles leave the second tile of the last pair
    # empty)
    (2, 2, 128, (300, 129, 384), (70, 0, 5)),          # MHA, 3 row tiles, prefixes
    (3, 1, 128, (200, 260, 385), (0, 130, 0)),         # G = 3, 4 row tiles (last: 1 row)
])
def test_prefill_matches_oracle(cuda_device, Hq, Hkv, D, lengths, ctx, kernel):
    inp = synth.make_prefill_inputs(_w(Hq=Hq, Hkv=Hkv, D=D), lengths=lengths, ctx=ctx)
    d = _dev(inp, cuda_device)
    o1, o2 = _run(d, kernel=kernel)
    _check_all(inp, d, o1, o2, "%s G=%d D=%d" % (kernel, Hq // Hkv, D))


def test_automatic_kernel_choice(cuda_device):
    o1 = torch.empty((256, 8, 128), dtype=torch.bfloat16, device=cuda_device)
    assert api.prefill_kernel(128, 256, o1, 8) == "tcgen05"
    assert api.prefill_kernel(64, 256, o1[:, :, :64], 8) == "tcgen05"
    assert api.prefill_kernel(64, 100, o1[:100, :, :64], 8) == "mma_sync"
    assert api.prefill_kernel(96, 256, o1[:, :, :96], 8) == "mma_sync"
    assert api.prefill_kernel(128, 100, o1[:100], 8) == "mma_sync"


def test_both_kernels_agree_within_tolerance(cuda_device):
    inp = synth.make_prefill_inputs(_w(Hq=8, Hkv=2), lengths=(400, 250), ctx=(30, 0))
    d = _dev(inp, cuda_device)
    a1, a2 = _run(d, kernel="mma_sync")
    b1, b2 = _run(d, kernel="tcgen05", append=False)
    assert torch.equal(a2, b2)   # the auxiliary step is the same code
    r1, _, _, _ = _oracle(inp)
    assert_attn_close(a1, r1, "bf16", "mma_sync O1")
    assert_attn_close(b1, r1, "bf16", "tcgen05 O1")


def test_aux_output_is_the_decode_step_of_the_last_position(cuda_device):
    inp = synth.make_prefill_inputs(_w(Hq=8, Hkv=2), lengths=(70, 300), ctx=(10, 0))
    d = _dev(inp, cuda_device)
    o1, o2 = _run(d)
    last = (inp["cu_seqlens"][1:] - 1).long()
    seqlens = (inp["ctx_lens"] + inp["cu_seqlens"][1:] - inp["cu_seqlens"][:-1]).to(cuda_device)
    q_last = d["q1"][last.to(cuda_device)].contiguous()
    d1, d2 = api.decode_attn(q_last, d["q2raw"], d["a"], d["k_cache"], d["v_cache"],
                             d["block_table"], seqlens, inp["max_seqlen"])
    torch.cuda.synchronize()
    assert torch.equal(d2, o2)          # the same kernel on the same cache
    r1, _, _, _ = _oracle(inp)
    assert_attn_close(d1, r1[last.numpy()], "bf16", "decode O1 at the last position")
    assert_attn_close(o1[last.to(cuda_device)], r1[last.numpy()], "bf16", "prefill O1 last rows")


def test_uniform_batch_aux_step_takes_one_wave_of_splits(cuda_device):
    """Fresh prompts of one length without ctx_lens: the auxiliary step runs
    the decode kernel with the split count that fills one wave (2 CTAs per
    SM, capped by the decode plan), so it equals that decode call bit for
    bit, and the oracle's decode step within the tolerance. 16 prompts x 8
    KV heads = 128 units of 2600 tokens: the plan's 5 splits against 2."""
    B, Hkv, n = 16, 8, 2600
    inp = synth.make_prefill_inputs(_w(Hq=8, Hkv=Hkv, D=64), lengths=(n,) * B, ctx=(0,) * B)
    d = _dev(inp, cuda_device)
    o1, o2 = api.prefill(d["q1"], d["k_new"], d["v_new"], d["k_cache"], d["v_cache"],
                         d["block_table"], d["cu_seqlens"], inp["max_q_len"], inp["max_seqlen"],
                         q2raw=d["q2raw"], a=d["a"])
    plan = api.decode_attn_num_splits(B, Hkv, inp["max_seqlen"])
    splits = min(plan, 296 // (B * Hkv))
    assert plan > splits >= 1
    last = (inp["cu_seqlens"][1:] - 1).long()
    seqlens = torch.full((B,), n, dtype=torch.int32, device=cuda_device)
    q_last = d["q1"][last.to(cuda_device)].contiguous()
    _, d2 = api.decode_attn(q_last, d["q2raw"], d["a"], d["k_cache"], d["v_cache"],
                            d["block_table"], seqlens, inp["max_seqlen"], num_splits=splits)
    torch.cuda.synchronize()
    assert torch.equal(d2, o2)
    cu = inp["cu_seqlens"].tolist()
    scale = 1.0 / math.sqrt(64)
    for b in (0, 7, 15):
        q2 = oracle.couple_query(f32(inp["q1"][cu[b + 1] - 1])[None], f32(inp["q2raw"][b])[None],
                                 f32(inp["a"]))[0]
        for h in (0, 5):
            K = f32(inp["k_new"][cu[b]:cu[b + 1], h])
            V = f32(inp["v_new"][cu[b]:cu[b + 1], h])
            ref = oracle.attn_weights(q2[h][None], K, scale) @ V
            assert_attn_close(o2[b, h][None], ref, "bf16", "uniform batch O2 b=%d h=%d" % (b, h))


def test_primary_output_ignores_aux_inputs_even_nan(cuda_device):
    inp = synth.make_prefill_inputs(_w(Hq=8, Hkv=2), lengths=(100, 33), ctx=(5, 0))
    d = _dev(inp, cuda_device)
    base, _ = _run(d, aux=False)
    d = _dev(inp, cuda_device)
    d["q2raw"] = torch.full_like(d["q2raw"], float("nan"))
    o1, o2 = _run(d)
    assert torch.equal(o1, base)
    assert torch.isnan(o2.float()).all()


@pytest.mark.parametrize("kernel", KERNELS)
def test_stale_nan_slots_around_the_chunk_are_masked(cuda_device, kernel):
    """Every cache slot that is neither prefix nor chunk holds NaN: the tail
    of the last page must not leak into any output."""
    inp = synth.make_prefill_inputs(_w(Hq=8, Hkv=2), lengths=(37, 100, 1), ctx=(3, 0, 70))
    kc, vc = inp["k_cache"].clone(), inp["v_cache"].clone()
    nan_k = torch.full_like(kc, float("nan"))
    nan_v = torch.full_like(vc, float("nan"))
    tbl = inp["block_table"]
    for b, c in enumerate(inp["ctx_lens"].tolist()):
        for p in range(c):
            page, slot = int(tbl[b, p // 64]), p % 64
            nan_k[page, :, slot] = kc[page, :, slot]
            nan_v[page, :, slot] = vc[page, :, slot]
    inp["k_cache"], inp["v_cache"] = nan_k, nan_v
    d = _dev(inp, cuda_device)
    o1, o2 = _run(d, kernel=kernel)
    assert torch.isfinite(o1.float()).all() and torch.isfinite(o2.float()).all()
    _check_all(inp, d, o1, o2, "%s NaN stale slots" % kernel)


@pytest.mark.parametrize("kernel", KERNELS)
def test_chunked_prefill_equals_whole_prompt(cuda_device, kernel):
    inp = synth.make_prefill_inputs(_w(Hq=8, Hkv=2), lengths=(300,), ctx=(0,))
    r1, r2, _, _ = _oracle(inp)
    d = _dev(inp, cuda_device)
    m = 129
    first = dict(d, q1=d["q1"][:m], k_new=d["k_new"][:m], v_new=d["v_new"][:m],
                 cu_seqlens=torch.tensor([0, m], dtype=torch.int32, device=cuda_device),
                 max_q_len=m)
    a1, _ = _run(first, aux=False, kernel=kernel)
    second = dict(d, q1=d["q1"][m:], k_new=d["k_new"][m:], v_new=d["v_new"][m:],
                  cu_seqlens=torch.tensor([0, 300 - m], dtype=torch.int32, device=cuda_device),
                  ctx_lens=torch.tensor([m], dtype=torch.int32, device=cuda_device),
                  max_q_len=300 - m)
    a2, b2 = _run(second, kernel=kernel)
    assert_attn_close(torch.cat([a1, a2]), r1, "bf16", "chunked O1")
    assert_attn_close(b2, r2, "bf16", "chunked O2")


def test_without_append_reads_the_cached_chunk(cuda_device):
    inp = synth.make_prefill_inputs(_w(Hq=8, Hkv=2), lengths=(90, 17), ctx=(20, 0))
    d = _dev(inp, cuda_device)
    o1, o2 = _run(d)
    p1, p2 = _run(d, append=False)
    assert torch.equal(p1, o1) and torch.equal(p2, o2)


def test_invalid_chunk_is_flagged_and_the_others_are_computed(cuda_device):
    """An empty chunk in the middle: DF_DEVERR_SEQLEN, zero auxiliary output
    for it, correct rows for the other sequences."""
    inp = synth.make_prefill_inputs(_w(Hq=8, Hkv=2), lengths=(5, 1, 7), ctx=(0, 0, 9))
    inp["cu_seqlens"] = torch.tensor([0, 5, 5, 12], dtype=torch.int32)
    inp["T"] = 12
    for k in ("q1", "k_new", "v_new"):
        inp[k] = inp[k][:12].contiguous()
    d = _dev(inp, cuda_device)
    err = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    o1, o2 = _run(d, err=err)
    assert int(err.item()) & L.DF_DEVERR_SEQLEN
    assert not bool(o2[1].any())
    for b, (t0, t1) in ((0, (0, 5)), (2, (5, 12))):
        one = dict(inp, q1=inp["q1"][t0:t1], k_new=inp["k_new"][t0:t1],
                   v_new=inp["v_new"][t0:t1], q2raw=inp["q2raw"][b:b + 1],
                   block_table=inp["block_table"][b:b + 1],
                   cu_seqlens=torch.tensor([0, t1 - t0], dtype=torch.int32),
                   ctx_lens=inp["ctx_lens"][b:b + 1])
        r1, r2, _, _ = _oracle(one)
        assert_attn_close(o1[t0:t1], r1, "bf16", "sequence %d O1" % b)
        assert_attn_close(o2[b:b + 1], r2, "bf16", "sequence %d O2" % b)


@pytest.mark.parametrize("kernel", KERNELS)
def test_out_of_range_page_is_flagged(cuda_device, kernel):
    inp = synth.make_prefill_inputs(_w(Hq=8, Hkv=2), lengths=(200,), ctx=(0,))
    inp["block_table"] = inp["block_table"].clone()
    inp["block_table"][0, 1] = inp["num_blocks"] + 5
    d = _dev(inp, cuda_device)
    err = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    _run(d, err=err, kernel=kernel)
    assert int(err.item()) & L.DF_DEVERR_BLOCK
    assert not int(err.item()) & L.DF_DEVERR_TIMEOUT


def test_launch_count():
    assert api.prefill_num_launches(True, True) == 4
    assert api.prefill_num_launches(False, False) == 1


@pytest.mark.slow
@pytest.mark.parametrize("Hq,Hkv", [(32, 8), (32, 32), (24, 8)])
def test_full_size_prefill_sampled_rows(cuda_device, Hq, Hkv):
    """The timed workload (16 prompts of 4096 tokens, D 128; 32/8 heads, and
    the odd groups of MHA and G = 3 that pair row tiles): every row of the
    cache written bit-exactly is checked on sampled tokens, and sampled
    output rows against the oracle's attention of that row."""
    w = _w(Hq=Hq, Hkv=Hkv)
    inp = synth.make_prefill_inputs(w)
    d = _dev(inp, cuda_device)
    o1, o2 = _run(d)   # automatic choice: the tcgen05 kernel at these sizes
    kc, vc = d["k_cache"].cpu(), d["v_cache"].cpu()
    tbl, cu = inp["block_table"], inp["cu_seqlens"].tolist()
    G = w.Hq // w.Hkv
    scale = 1.0 / math.sqrt(w.D)
    rng = np.random.default_rng(0)
    for b in (0, 7, 15):
        t0, n = cu[b], cu[b + 1] - cu[b]
        for i in sorted({0, 1, 63, 64, 65, n - 1} | set(rng.integers(0, n, 4).tolist())):
            t = t0 + i
            page, slot = int(tbl[b, i // 64]), i % 64
            assert torch.equal(kc[page, :, slot], inp["k_new"][t])
            assert torch.equal(vc[page, :, slot], inp["v_new"][t])
            for h in (0, 13, w.Hq - 1):
                g = h // G
                K = f32(inp["k_new"][t0:t + 1, g])
                V = f32(inp["v_new"][t0:t + 1, g])
                ref = oracle.attn_weights(f32(inp["q1"][t, h])[None], K, scale) @ V
                assert_attn_close(o1[t, h][None], ref, "bf16", "row b=%d i=%d h=%d" % (b, i, h))
        last = t0 + n - 1
        q2 = oracle.couple_query(f32(inp["q1"][last])[None], f32(inp["q2raw"][b])[None],
                                 f32(inp["a"]))[0]
        for h in (0, w.Hq - 1):
            g = h // G
            K = f32(inp["k_new"][t0:last + 1, g])
            V = f32(inp["v_new"][t0:last + 1, g])
            ref = oracle.attn_weights(q2[h][None], K, scale) @ V
            assert_attn_close(o2[b, h][None], ref, "bf16", "aux b=%d h=%d" % (b, h))
