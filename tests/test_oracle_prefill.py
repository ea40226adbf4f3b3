"""Pins of the oracle's prefill (primary prompt processing + auxiliary query
at the last prompt position) against things other than itself: pure-Python
loops, torch's scaled-dot-product attention in float64, closed forms, and
the decode step and append it must agree with.

Method: "Sintesi Tecnica: Dual-Flow Transformers", section "Architettura
Core" -- the primary flow processes the prompt causally and writes the
cache; the auxiliary flow is skipped during prefill and runs only at the last
prompt position.
"""

import math

import numpy as np
import pytest
import torch

import oracle
from tests import brute


def _case(seed, lens=(5, 7), ctx=(0, 3), Hq=4, Hkv=2, D=8, bs=4, spare=3):
    """Random prompts in a shuffled paged cache; prefixes of ctx tokens are
    already in the cache. Returns the prefill arguments and the logical
    (position-ordered) prefix keys/values per sequence for the checks."""
    rng = np.random.default_rng(seed)
    B = len(lens)
    T = sum(lens)
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    pages_per = [-(-(c + n) // bs) for c, n in zip(ctx, lens)]
    mb = max(pages_per)
    nblk = sum(pages_per) + spare
    perm = rng.permutation(nblk)
    table = np.zeros((B, mb), dtype=np.int64)
    k = 0
    for b in range(B):
        for j in range(pages_per[b]):
            table[b, j] = perm[k]
            k += 1
    kc = rng.standard_normal((nblk, Hkv, bs, D))
    vc = rng.standard_normal((nblk, Hkv, bs, D))
    prefix_k = [[kc[table[b, j // bs], :, j % bs, :].copy() for j in range(ctx[b])]
                for b in range(B)]
    prefix_v = [[vc[table[b, j // bs], :, j % bs, :].copy() for j in range(ctx[b])]
                for b in range(B)]
    q1 = rng.standard_normal((T, Hq, D))
    kn = rng.standard_normal((T, Hkv, D))
    vn = rng.standard_normal((T, Hkv, D))
    q2 = rng.standard_normal((B, Hq, D))
    a = 0.1 * rng.standard_normal((Hq, D))
    return dict(q1=q1, k_new=kn, v_new=vn, k_cache=kc, v_cache=vc, block_table=table,
                cu_seqlens=cu, ctx_lens=np.asarray(ctx), q2raw=q2, a=a), prefix_k, prefix_v


@pytest.mark.parametrize("seed", [0, 1])
def test_prefill_matches_brute_force_loops(seed):
    args, pk, pv = _case(seed)
    o1, o2, _, _ = oracle.prefill(**args)
    q1, kn, vn, cu = args["q1"], args["k_new"], args["v_new"], args["cu_seqlens"]
    Hq, D = q1.shape[1:]
    Hkv = kn.shape[1]
    G = Hq // Hkv
    scale = 1.0 / math.sqrt(D)
    for b in range(len(cu) - 1):
        c = int(args["ctx_lens"][b])
        t0, t1 = int(cu[b]), int(cu[b + 1])
        for h in range(Hq):
            g = h // G
            keys = [list(x[g]) for x in pk[b]] + [list(kn[t, g]) for t in range(t0, t1)]
            vals = [list(x[g]) for x in pv[b]] + [list(vn[t, g]) for t in range(t0, t1)]
            rows = brute.causal_prefill([list(q1[t, h]) for t in range(t0, t1)], keys, vals,
                                        c, scale)
            np.testing.assert_allclose(o1[t0:t1, h], np.array(rows), rtol=0, atol=1e-12)
            q2 = [args["q2raw"][b, h, d] + args["a"][h, d] * q1[t1 - 1, h, d] for d in range(D)]
            np.testing.assert_allclose(o2[b, h], brute.softmax_attention(q2, keys, vals, scale),
                                       rtol=0, atol=1e-12)


def _sdpa(q, k, v, mask=None, causal=False):
    """torch SDPA in float64 on [heads, n, D] tensors."""
    return torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q), torch.from_numpy(k), torch.from_numpy(v),
        attn_mask=None if mask is None else torch.from_numpy(mask), is_causal=causal).numpy()


def test_fresh_prompt_matches_torch_causal_sdpa():
    args, _, _ = _case(3, lens=(9, 16), ctx=(0, 0), Hq=6, Hkv=2, D=16, bs=4)
    o1, _, _, _ = oracle.prefill(**args)
    cu, G = args["cu_seqlens"], 3
    for b in range(2):
        t0, t1 = int(cu[b]), int(cu[b + 1])
        q = args["q1"][t0:t1].transpose(1, 0, 2)
        k = np.repeat(args["k_new"][t0:t1].transpose(1, 0, 2), G, axis=0)
        v = np.repeat(args["v_new"][t0:t1].transpose(1, 0, 2), G, axis=0)
        ref = _sdpa(q, k, v, causal=True)
        np.testing.assert_allclose(o1[t0:t1].transpose(1, 0, 2), ref, rtol=0, atol=1e-12)


def test_prompt_after_a_prefix_matches_sdpa_with_offset_mask():
    args, pk, pv = _case(4, lens=(6, 5), ctx=(7, 2), Hq=2, Hkv=2, D=8, bs=4)
    o1, _, _, _ = oracle.prefill(**args)
    cu = args["cu_seqlens"]
    for b in range(2):
        c = int(args["ctx_lens"][b])
        t0, t1 = int(cu[b]), int(cu[b + 1])
        n = t1 - t0
        keys = np.concatenate([np.array(pk[b]).reshape(c, 2, 8), args["k_new"][t0:t1]], 0)
        vals = np.concatenate([np.array(pv[b]).reshape(c, 2, 8), args["v_new"][t0:t1]], 0)
        # row i may see key j iff j <= c + i: the lower triangle shifted by c
        mask = np.tril(np.ones((n, c + n), dtype=bool), k=c)
        ref = _sdpa(args["q1"][t0:t1].transpose(1, 0, 2), keys.transpose(1, 0, 2),
                    vals.transpose(1, 0, 2), mask=mask)
        np.testing.assert_allclose(o1[t0:t1].transpose(1, 0, 2), ref, rtol=0, atol=1e-12)


def test_first_token_of_a_fresh_prompt_returns_its_value_row():
    args, _, _ = _case(5, lens=(4, 3), ctx=(0, 0))
    o1, _, _, _ = oracle.prefill(**args)
    G = 2
    for t0 in (0, 4):
        for h in range(4):
            assert np.array_equal(o1[t0, h], args["v_new"][t0, h // G])


def test_last_prompt_position_equals_a_decode_step():
    args, _, _ = _case(6, lens=(9, 4), ctx=(2, 5))
    o1, o2, kc, vc = oracle.prefill(**args)
    cu = args["cu_seqlens"]
    last = cu[1:] - 1
    seqlens = args["ctx_lens"] + np.diff(cu)
    d1, d2 = oracle.decode_attn(args["q1"][last], args["q2raw"], args["a"], kc, vc,
                                args["block_table"], seqlens)
    np.testing.assert_allclose(o1[last], d1, rtol=0, atol=1e-12)
    np.testing.assert_allclose(o2, d2, rtol=0, atol=1e-12)


def test_prefill_cache_equals_token_by_token_appends():
    args, _, _ = _case(7, lens=(6, 5), ctx=(1, 4))
    _, _, kc, vc = oracle.prefill(**args)
    ek, ev = args["k_cache"], args["v_cache"]
    cu = args["cu_seqlens"]
    for b in range(2):
        for i in range(int(cu[b + 1] - cu[b])):
            t = int(cu[b]) + i
            ek, ev = oracle.kv_append(args["k_new"][t:t + 1], args["v_new"][t:t + 1], ek, ev,
                                      args["block_table"][b:b + 1], [int(args["ctx_lens"][b]) + i])
    assert np.array_equal(kc, ek) and np.array_equal(vc, ev)
    # the prefix and every page outside the sequences' tables are untouched
    used = set()
    for b in range(2):
        for p in range(int(args["ctx_lens"][b]), int(args["ctx_lens"][b] + cu[b + 1] - cu[b])):
            used.add((int(args["block_table"][b, p // 4]), p % 4))
    for page in range(kc.shape[0]):
        for slot in range(4):
            if (page, slot) not in used:
                assert np.array_equal(kc[page, :, slot], args["k_cache"][page, :, slot])


def test_chunked_prefill_equals_whole_prompt():
    args, _, _ = _case(8, lens=(11,), ctx=(0,), bs=4)
    o1, o2, kc, vc = oracle.prefill(**args)
    m = 6
    first = dict(args, q1=args["q1"][:m], k_new=args["k_new"][:m], v_new=args["v_new"][:m],
                 cu_seqlens=np.array([0, m]), q2raw=None)
    a1, _, kc1, vc1 = oracle.prefill(**first)
    second = dict(args, q1=args["q1"][m:], k_new=args["k_new"][m:], v_new=args["v_new"][m:],
                  cu_seqlens=np.array([0, 11 - m]), ctx_lens=np.array([m]), k_cache=kc1,
                  v_cache=vc1)
    a2, b2, kc2, vc2 = oracle.prefill(**second)
    np.testing.assert_allclose(np.concatenate([a1, a2]), o1, rtol=0, atol=1e-12)
    np.testing.assert_allclose(b2, o2, rtol=0, atol=1e-12)
    assert np.array_equal(kc2, kc) and np.array_equal(vc2, vc)


def test_aux_at_last_position_coupling_limits():
    args, _, _ = _case(9)
    cu = args["cu_seqlens"]
    last = cu[1:] - 1
    o1, _, _, _ = oracle.prefill(**args)
    # q2raw = 0, a = 1: the auxiliary query is the primary one -> O2 = O1[last]
    _, o2, _, _ = oracle.prefill(**dict(args, q2raw=np.zeros_like(args["q2raw"]),
                                        a=np.ones_like(args["a"])))
    np.testing.assert_allclose(o2, o1[last], rtol=0, atol=1e-12)
    # a = 0: plain attention of the raw auxiliary query over every prompt key
    _, o2z, kc, vc = oracle.prefill(**dict(args, a=np.zeros_like(args["a"])))
    seqlens = args["ctx_lens"] + np.diff(cu)
    d1, _ = oracle.decode_attn(args["q2raw"], None, None, kc, vc, args["block_table"], seqlens)
    np.testing.assert_allclose(o2z, d1, rtol=0, atol=1e-12)


def test_primary_prefill_ignores_aux_inputs_even_nan():
    args, _, _ = _case(10)
    o1, _, kc, vc = oracle.prefill(**args)
    n1, n2, nkc, nvc = oracle.prefill(**dict(args, q2raw=np.full_like(args["q2raw"], np.nan)))
    assert np.array_equal(o1, n1) and np.isnan(n2).all()
    assert np.array_equal(kc, nkc) and np.array_equal(vc, nvc)
    p1, p2, _, _ = oracle.prefill(**dict(args, q2raw=None))
    assert np.array_equal(o1, p1) and p2 is None


def _golden_num(s):
    table = {"sqrt2ln2": math.sqrt(2) * math.log(2), "sqrt2ln3": math.sqrt(2) * math.log(3)}
    if s in table:
        return table[s]
    if "/" in s:
        n, d = s.split("/")
        return float(int(n)) / float(int(d))
    return float(s)


def _golden_arr(x):
    return np.vectorize(_golden_num, otypes=[np.float64])(np.array(x, dtype=object))


def test_golden_prefill_worked_example():
    import json
    import os
    spec = json.load(open(os.path.join(os.path.dirname(__file__), "golden",
                                       "prefill_worked_example.json")))
    bs = spec["block_size"]
    table = np.array(spec["block_table"])
    kc = np.full((3, 1, bs, 2), 9.0)   # page 2 is spare: its marker must survive
    vc = np.full((3, 1, bs, 2), 9.0)
    for j, (kr, vr) in enumerate(zip(spec["cached_k"], spec["cached_v"])):
        kc[table[0, j // bs], 0, j % bs] = _golden_arr(kr)
        vc[table[0, j // bs], 0, j % bs] = _golden_arr(vr)
    o1, o2, kc2, vc2 = oracle.prefill(
        _golden_arr(spec["q1"]), _golden_arr(spec["k_new"]), _golden_arr(spec["v_new"]), kc, vc,
        table, np.array(spec["cu_seqlens"]), np.array(spec["ctx_lens"]),
        q2raw=_golden_arr(spec["q2raw"]), a=_golden_arr(spec["a"]))
    np.testing.assert_allclose(o1, _golden_arr(spec["o1"]), rtol=0, atol=1e-12)
    np.testing.assert_allclose(o2, _golden_arr(spec["o2"]), rtol=0, atol=1e-12)
    for page, rows in spec["k_pages_after"].items():
        np.testing.assert_array_equal(kc2[int(page), 0], _golden_arr(rows))
    for page, rows in spec["v_pages_after"].items():
        np.testing.assert_array_equal(vc2[int(page), 0], _golden_arr(rows))
    assert (kc2[2] == 9.0).all() and (vc2[2] == 9.0).all()
