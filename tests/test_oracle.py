"""Pins for the fp64 oracle (CPU only).

Each test checks the oracle against something other than itself: values
worked out by hand from the method's definition (tests/golden), closed
forms, invariants the pages state, brute force with explicit loops, or a
library routine (torch SDPA in float64, scipy's logistic function, torch's
bf16 conversion). Chosen so that a dropped term, a wrong sign, a wrong
head/page index or a transposed operand in the oracle fails at least one.
"""

import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from tests import brute

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _num(s):
    table = {"sqrt2ln3": math.sqrt(2) * math.log(3), "sqrt2ln3/2": math.sqrt(2) * math.log(3) / 2,
             "ln2": math.log(2), "ln3": math.log(3)}
    if s in table:
        return table[s]
    if "/" in s:
        num, den = s.split("/")
        return float(int(num)) / float(int(den))
    return float(s)


def _arr(x):
    return np.vectorize(_num, otypes=[np.float64])(np.array(x, dtype=object))


def _paged(keys_list, Hkv=1, bs=64):
    """[L][D] (one KV head) -> one page cache [1, Hkv, bs, D] + table."""
    k = np.array(keys_list, dtype=np.float64)
    L, D = k.shape
    cache = np.zeros((1, Hkv, bs, D))
    cache[0, 0, :L] = k
    return cache, np.zeros((1, 1), dtype=np.int32)


# ---------------------------------------------------------------- golden

def test_golden_closed_form_attention():
    spec = json.load(open(os.path.join(GOLDEN, "closed_form_attention.json")))
    for case in spec["cases"]:
        kc, table = _paged(_arr(case["keys"]))
        vc, _ = _paged(_arr(case["values"]))
        q1, q2raw, a = _arr(case["q1"]), _arr(case["q2raw"]), _arr(case["a"])
        L = len(case["keys"])
        o1, o2 = oracle.decode_attn(q1, q2raw, a, kc, vc, table, [L])
        np.testing.assert_allclose(o1, _arr(case["o1"]), rtol=0, atol=1e-12, err_msg=case["name"])
        np.testing.assert_allclose(o2, _arr(case["o2"]), rtol=0, atol=1e-12, err_msg=case["name"])


def test_golden_gqa_head_mapping():
    spec = json.load(open(os.path.join(GOLDEN, "closed_form_gqa.json")))
    Hq, Hkv, D = spec["Hq"], spec["Hkv"], spec["D"]
    rng = np.random.default_rng(0)
    vals = _arr(spec["values_per_kv_head"])
    kc = np.zeros((1, Hkv, 64, D))
    vc = np.zeros((1, Hkv, 64, D))
    kc[0, :, 0] = rng.standard_normal((Hkv, D))
    vc[0, :, 0] = vals
    q1 = rng.standard_normal((1, Hq, D))
    q2 = rng.standard_normal((1, Hq, D))
    a = rng.standard_normal((Hq, D))
    o1, o2 = oracle.decode_attn(q1, q2, a, kc, vc, np.zeros((1, 1), np.int32), [1])
    exp = _arr(spec["o_expected_per_query_head"])
    np.testing.assert_array_equal(o1[0], exp)
    np.testing.assert_array_equal(o2[0], exp)


# ---------------------------------------------------------------- brute force

def _random_case(rng, B=2, Hq=4, Hkv=2, D=8, bs=4, lens=(5, 11), random_table=True):
    nblk = [math.ceil(L / bs) for L in lens]
    total = sum(nblk)
    order = rng.permutation(total) if random_table else np.arange(total)
    table = -np.ones((B, max(nblk)), dtype=np.int32)
    k = 0
    for b, n in enumerate(nblk):
        table[b, :n] = order[k:k + n]
        k += n
    kc = rng.standard_normal((total, Hkv, bs, D))
    vc = rng.standard_normal((total, Hkv, bs, D))
    q1 = rng.standard_normal((B, Hq, D))
    q2 = rng.standard_normal((B, Hq, D))
    a = 0.5 * rng.standard_normal((Hq, D))
    return q1, q2, a, kc, vc, table, list(lens)


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_decode_matches_brute_force_loops(seed):
    rng = np.random.default_rng(seed)
    q1, q2, a, kc, vc, table, lens = _random_case(rng)
    o1, o2 = oracle.decode_attn(q1, q2, a, kc, vc, table, lens, block_size=4)
    b1, b2 = brute.dual_decode(q1.tolist(), q2.tolist(), a.tolist(), kc.tolist(), vc.tolist(),
                               table.tolist(), lens, 4, 4, 2)
    np.testing.assert_allclose(o1, np.array(b1), rtol=0, atol=1e-12)
    np.testing.assert_allclose(o2, np.array(b2), rtol=0, atol=1e-12)


# ---------------------------------------------------------------- closed forms

def test_single_token_returns_its_value_row():
    rng = np.random.default_rng(3)
    q1, q2, a, kc, vc, table, _ = _random_case(rng, B=1, Hq=2, Hkv=2, lens=(1,))
    o1, o2 = oracle.decode_attn(q1, q2, a, kc, vc, table, [1], block_size=4)
    page = table[0, 0]
    for h in range(2):
        np.testing.assert_array_equal(o1[0, h], vc[page, h, 0])
        np.testing.assert_array_equal(o2[0, h], vc[page, h, 0])


def test_identical_keys_give_mean_of_values():
    rng = np.random.default_rng(4)
    L, D = 37, 16
    kc = np.zeros((1, 1, 64, D))
    kc[0, 0, :L] = rng.standard_normal(D)[None, :]
    vc = np.zeros((1, 1, 64, D))
    vc[0, 0, :L] = rng.standard_normal((L, D))
    q1 = rng.standard_normal((1, 1, D))
    q2 = rng.standard_normal((1, 1, D))
    o1, o2 = oracle.decode_attn(q1, q2, None, kc, vc, np.zeros((1, 1), np.int32), [L])
    mean = vc[0, 0, :L].mean(axis=0)
    np.testing.assert_allclose(o1[0, 0], mean, atol=1e-13)
    np.testing.assert_allclose(o2[0, 0], mean, atol=1e-13)


def test_dominant_key_selects_its_value():
    rng = np.random.default_rng(5)
    L, D = 20, 8
    kc = np.zeros((1, 1, 64, D))
    kc[0, 0, :L] = 0.01 * rng.standard_normal((L, D))
    q = np.zeros((1, 1, D))
    q[0, 0, 0] = 1.0
    kc[0, 0, 7, 0] = 400.0  # score 400/sqrt(8) above the rest
    vc = np.zeros((1, 1, 64, D))
    vc[0, 0, :L] = rng.standard_normal((L, D))
    o1, _ = oracle.decode_attn(q, None, None, kc, vc, np.zeros((1, 1), np.int32), [L])
    np.testing.assert_allclose(o1[0, 0], vc[0, 0, 7], atol=1e-12)


def test_weights_are_a_distribution():
    rng = np.random.default_rng(6)
    p = oracle.attn_weights(rng.standard_normal((5, 32)) * 4, rng.standard_normal((300, 32)), 0.3)
    assert np.all(p >= 0)
    np.testing.assert_allclose(p.sum(axis=1), 1.0, atol=1e-14)


def test_primary_equals_last_row_of_causal_attention():
    """Textbook check: the primary flow at a decode position is ordinary causal
    self-attention, i.e. the last row of full causal attention over the
    sequence (torch SDPA in float64 on the CPU as the library cross-check)."""
    rng = np.random.default_rng(7)
    H, L, D = 3, 150, 32
    Q = rng.standard_normal((H, L, D))
    K = rng.standard_normal((H, L, D))
    V = rng.standard_normal((H, L, D))
    full = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(Q)[None], torch.from_numpy(K)[None], torch.from_numpy(V)[None],
        is_causal=True)[0].numpy()
    bs = 64
    nblk = math.ceil(L / bs)
    kc = np.zeros((nblk, H, bs, D))
    vc = np.zeros((nblk, H, bs, D))
    for j in range(L):
        kc[j // bs, :, j % bs] = K[:, j]
        vc[j // bs, :, j % bs] = V[:, j]
    table = np.arange(nblk, dtype=np.int32)[None]
    o1, _ = oracle.decode_attn(Q[None, :, L - 1], None, None, kc, vc, table, [L])
    np.testing.assert_allclose(o1[0], full[:, L - 1], rtol=0, atol=1e-12)


# ---------------------------------------------------------------- coupling special cases

def test_zero_coupling_is_plain_attention_of_raw_aux_query():
    rng = np.random.default_rng(8)
    q1, q2, a, kc, vc, table, lens = _random_case(rng)
    _, o2 = oracle.decode_attn(q1, q2, np.zeros_like(a), kc, vc, table, lens, block_size=4)
    ref, _ = oracle.decode_attn(q2, None, None, kc, vc, table, lens, block_size=4)
    np.testing.assert_array_equal(o2, ref)


def test_unit_coupling_of_zero_raw_query_reproduces_primary():
    rng = np.random.default_rng(9)
    q1, q2, a, kc, vc, table, lens = _random_case(rng)
    o1, o2 = oracle.decode_attn(q1, np.zeros_like(q2), np.ones_like(a), kc, vc, table, lens,
                                block_size=4)
    np.testing.assert_array_equal(o1, o2)


def test_coupling_is_elementwise_per_head():
    q1 = np.arange(12, dtype=np.float64).reshape(1, 2, 6)
    q2 = np.ones((1, 2, 6))
    a = np.full((2, 6), 2.0)
    a[1, 3] = -1.0
    q = oracle.couple_query(q1, q2, a)
    assert q[0, 0, 5] == 1 + 2 * 5
    assert q[0, 1, 3] == 1 - 9
    assert q[0, 1, 0] == 1 + 2 * 6


# ---------------------------------------------------------------- asymmetry invariants

def test_primary_output_ignores_aux_inputs_even_nan():
    rng = np.random.default_rng(10)
    q1, q2, a, kc, vc, table, lens = _random_case(rng)
    o1_ref, _ = oracle.decode_attn(q1, None, None, kc, vc, table, lens, block_size=4)
    q2_bad = q2.copy()
    q2_bad[0, 1, 2] = np.nan
    q2_bad[1, 0, 0] = np.inf
    a_bad = a.copy()
    a_bad[2, 3] = np.nan
    o1, o2 = oracle.decode_attn(q1, q2_bad, a_bad, kc, vc, table, lens, block_size=4)
    np.testing.assert_array_equal(o1, o1_ref)
    assert np.isnan(o2[0, 1]).all()


def test_paging_is_invisible():
    rng = np.random.default_rng(11)
    q1, q2, a, kc, vc, table, lens = _random_case(rng, random_table=True)
    # lay the same logical tokens out contiguously and compare
    B, Hkv, bs, D = len(lens), kc.shape[1], kc.shape[2], kc.shape[3]
    nblk = table.shape[1]
    kc2 = np.zeros((B * nblk, Hkv, bs, D))
    vc2 = np.zeros_like(kc2)
    t2 = np.zeros((B, nblk), dtype=np.int32)
    for b in range(B):
        for j in range(math.ceil(lens[b] / bs)):
            kc2[b * nblk + j] = kc[table[b, j]]
            vc2[b * nblk + j] = vc[table[b, j]]
            t2[b, j] = b * nblk + j
    r1 = oracle.decode_attn(q1, q2, a, kc, vc, table, lens, block_size=4)
    r2 = oracle.decode_attn(q1, q2, a, kc2, vc2, t2, lens, block_size=4)
    np.testing.assert_array_equal(r1[0], r2[0])
    np.testing.assert_array_equal(r1[1], r2[1])


def test_gqa_equals_mha_with_repeated_kv_heads():
    rng = np.random.default_rng(12)
    q1, q2, a, kc, vc, table, lens = _random_case(rng, Hq=6, Hkv=2)
    G = 3
    kr = np.repeat(kc, G, axis=1)
    vr = np.repeat(vc, G, axis=1)
    g1, g2 = oracle.decode_attn(q1, q2, a, kc, vc, table, lens, block_size=4)
    m1, m2 = oracle.decode_attn(q1, q2, a, kr, vr, table, lens, block_size=4)
    np.testing.assert_allclose(g1, m1, atol=1e-14)
    np.testing.assert_allclose(g2, m2, atol=1e-14)


# ---------------------------------------------------------------- append

def test_kv_append_writes_only_the_slot():
    rng = np.random.default_rng(13)
    kc = rng.standard_normal((6, 2, 4, 3)).astype(np.float32)
    vc = rng.standard_normal((6, 2, 4, 3)).astype(np.float32)
    kc0, vc0 = kc.copy(), vc.copy()
    table = np.array([[4, 1, -1], [0, 5, 2]], dtype=np.int32)
    pos = [5, 8]
    kn = rng.standard_normal((2, 2, 3)).astype(np.float32)
    vn = rng.standard_normal((2, 2, 3)).astype(np.float32)
    k2, v2 = oracle.kv_append(kn, vn, kc, vc, table, pos)
    np.testing.assert_array_equal(kc, kc0)  # inputs untouched
    expect_k, expect_v = kc0.copy(), vc0.copy()
    # by hand: seq 0 pos 5 -> table[0][1] = page 1, slot 1; seq 1 pos 8 -> page 2, slot 0
    expect_k[1, :, 1] = kn[0]
    expect_v[1, :, 1] = vn[0]
    expect_k[2, :, 0] = kn[1]
    expect_v[2, :, 0] = vn[1]
    assert k2.dtype == np.float32
    assert k2.tobytes() == expect_k.tobytes()
    assert v2.tobytes() == expect_v.tobytes()


# ---------------------------------------------------------------- projection / MLP pieces

def test_grouped_proj_matches_loops_and_grouping_changes_nothing():
    rng = np.random.default_rng(14)
    x = rng.standard_normal((6, 5))
    w = rng.standard_normal((7, 5))
    y = oracle.grouped_proj(x, w, 3, n_aux=4)
    ref = np.array(brute.matmul_nt(x.tolist(), w.tolist()))
    np.testing.assert_allclose(y[:3], ref[:3], atol=1e-13)
    np.testing.assert_allclose(y[3:, :4], ref[3:, :4], atol=1e-13)
    assert np.isnan(y[3:, 4:]).all()
    alone = oracle.grouped_proj(x[3:], w, 3)
    np.testing.assert_array_equal(alone[:, :4], y[3:, :4])


def test_silu_against_logistic_and_limits():
    from scipy.special import expit
    x = np.linspace(-30, 30, 1001)
    np.testing.assert_allclose(oracle.silu(x), x * expit(x), rtol=1e-14, atol=1e-300)
    assert oracle.silu(np.array([0.0]))[0] == 0.0
    assert abs(oracle.silu(np.array([40.0]))[0] - 40.0) < 1e-15
    assert abs(oracle.silu(np.array([-40.0]))[0]) < 1e-15


def test_swiglu_coupling_by_hand():
    gate = np.array([[0.0, 2.0], [1.0, -1.0]])
    up = np.array([[3.0, 4.0], [5.0, 6.0]])
    b = np.array([10.0, -1.0])
    h = oracle.swiglu_couple(np.concatenate([gate, up], axis=1), 2, 1, b)
    s = lambda v: v / (1 + math.exp(-v))
    h1 = [s(0.0) * 3, s(2.0) * 4]
    np.testing.assert_allclose(h[0], h1, atol=1e-15)
    np.testing.assert_allclose(h[1], [s(1.0) * 5 + 10 * h1[0], s(-1.0) * 6 - h1[1]], atol=1e-14)
    h0 = oracle.swiglu_couple(np.concatenate([gate, up], axis=1), 2, 1, np.zeros(2))
    np.testing.assert_array_equal(h0, oracle.swiglu_couple(np.concatenate([gate, up], 1), 2, 1))


def test_residual_coupling_by_hand():
    acc = np.array([[1.0, 2.0], [3.0, 4.0]])
    res = np.array([[0.5, 0.5], [-1.0, 1.0]])
    c = np.array([2.0, -3.0])
    y = oracle.residual_couple(acc, res, 1, c)
    np.testing.assert_array_equal(y, [[1.5, 2.5], [3 + 2 * 1 - 1, 4 - 3 * 2 + 1]])


def test_rmsnorm_closed_form():
    x = np.full((1, 8), 3.0)
    y = oracle.rmsnorm(x, eps=1e-5)
    np.testing.assert_allclose(y, 3.0 / math.sqrt(9.0 + 1e-5), rtol=1e-15)
    rng = np.random.default_rng(15)
    z = oracle.rmsnorm(rng.standard_normal((4, 4096)) * 7, eps=0.0)
    np.testing.assert_allclose(np.sqrt((z * z).mean(axis=1)), 1.0, rtol=1e-13)


# ---------------------------------------------------------------- bf16 rounding

def test_bf16_round_matches_torch_conversion():
    rng = np.random.default_rng(16)
    x = np.concatenate([rng.standard_normal(20000) * 10.0 ** rng.integers(-30, 30, 20000),
                        [0.0, -0.0, 1.0, 3.0e38, -3.0e38, 1e-39]]).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(oracle.bf16_round(x.astype(np.float64)), ref)


def test_bf16_round_ties_to_even():
    # 1 + 2^-8 is halfway between 1 and 1 + 2^-7: even mantissa is 1.
    assert oracle.bf16_round(np.array([1 + 2 ** -8]))[0] == 1.0
    # 1 + 3*2^-8 is halfway between 1 + 2^-7 (odd) and 1 + 2^-6 (even).
    assert oracle.bf16_round(np.array([1 + 3 * 2 ** -8]))[0] == 1 + 2 ** -6
    # one fp64 ulp above the tie rounds up (direct rounding, no fp32 detour)
    assert oracle.bf16_round(np.array([1 + 2 ** -8 + 2 ** -40]))[0] == 1 + 2 ** -7


# ---------------------------------------------------------------- layer step

def _tiny_layer(rng, B=3, d=16, Hq=2, Hkv=1, D=8, F=12, L=5):
    bf = oracle.bf16_round
    qd, kvd = Hq * D, Hkv * D
    p = dict(
        x1=bf(rng.standard_normal((B, d))), x2=bf(rng.standard_normal((B, d))),
        w_qkv=bf(0.2 * rng.standard_normal((qd + 2 * kvd, d))),
        w_o=bf(0.2 * rng.standard_normal((d, qd))),
        w_gu=bf(0.2 * rng.standard_normal((2 * F, d))),
        w_down=bf(0.2 * rng.standard_normal((d, F))),
        a=bf(0.1 * rng.standard_normal((Hq, D))), b=bf(0.1 * rng.standard_normal(F)),
        c=bf(0.1 * rng.standard_normal(d)))
    bs = 4
    nblk = math.ceil((L + 1) / bs)
    p["k_cache"] = bf(rng.standard_normal((B * nblk, Hkv, bs, D)))
    p["v_cache"] = bf(rng.standard_normal((B * nblk, Hkv, bs, D)))
    p["block_table"] = np.arange(B * nblk, dtype=np.int32).reshape(B, nblk)
    p["positions"] = np.full(B, L, dtype=np.int32)
    return p, dict(Hq=Hq, Hkv=Hkv, D=D, F=F)


def test_layer_primary_is_self_sufficient():
    rng = np.random.default_rng(17)
    p, dims = _tiny_layer(rng)
    r1 = oracle.layer_step(**p, **dims)
    q = dict(p)
    q["x2"] = rng.standard_normal(p["x2"].shape) * 5
    q["a"] = rng.standard_normal(p["a"].shape)
    q["b"] = rng.standard_normal(p["b"].shape)
    q["c"] = rng.standard_normal(p["c"].shape)
    r2 = oracle.layer_step(**q, **dims)
    B = p["x1"].shape[0]
    np.testing.assert_array_equal(r1["x_out"][:B], r2["x_out"][:B])
    np.testing.assert_array_equal(r1["k_cache"], r2["k_cache"])
    np.testing.assert_array_equal(r1["v_cache"], r2["v_cache"])


def test_layer_uncoupled_twin_flow_equals_primary():
    rng = np.random.default_rng(18)
    p, dims = _tiny_layer(rng)
    p["x2"] = p["x1"].copy()
    for k in ("a", "b", "c"):
        p[k] = np.zeros_like(p[k])
    r = oracle.layer_step(**p, **dims)
    B = p["x1"].shape[0]
    np.testing.assert_array_equal(r["x_out"][B:], r["x_out"][:B])


def test_layer_with_empty_cache_attends_to_current_token_only():
    rng = np.random.default_rng(19)
    p, dims = _tiny_layer(rng, L=0)
    r = oracle.layer_step(**p, **dims)
    B, Hq, Hkv, D = p["x1"].shape[0], dims["Hq"], dims["Hkv"], dims["D"]
    qd, kvd = Hq * D, Hkv * D
    v_new = r["qkv"][:B, qd + kvd:qd + 2 * kvd].reshape(B, Hkv, D)
    expect = oracle.bf16_round(np.repeat(v_new, Hq // Hkv, axis=1).reshape(B, qd))
    np.testing.assert_array_equal(r["attn"][:B], expect)
    np.testing.assert_array_equal(r["attn"][B:], expect)


def test_layer_cache_gets_primary_rows_only():
    rng = np.random.default_rng(20)
    p, dims = _tiny_layer(rng)
    r = oracle.layer_step(**p, **dims)
    B, qd, kvd = p["x1"].shape[0], dims["Hq"] * dims["D"], dims["Hkv"] * dims["D"]
    kn = r["qkv"][:B, qd:qd + kvd].reshape(B, dims["Hkv"], dims["D"])
    vn = r["qkv"][:B, qd + kvd:].reshape(B, dims["Hkv"], dims["D"])
    ek, ev = oracle.kv_append(kn, vn, p["k_cache"], p["v_cache"], p["block_table"], p["positions"])
    np.testing.assert_array_equal(r["k_cache"], ek)
    np.testing.assert_array_equal(r["v_cache"], ev)


def test_layer_with_zero_output_weights_is_identity_on_hidden_state():
    """Closed form: with W_o = W_down = 0 both sublayers add nothing, so each
    flow's hidden state passes through both residual connections unchanged."""
    rng = np.random.default_rng(21)
    p, dims = _tiny_layer(rng)
    p["w_o"] = np.zeros_like(p["w_o"])
    p["w_down"] = np.zeros_like(p["w_down"])
    r = oracle.layer_step(**p, **dims)
    np.testing.assert_array_equal(r["x_out"], np.concatenate([p["x1"], p["x2"]]))
    np.testing.assert_array_equal(r["x_mid"], np.concatenate([p["x1"], p["x2"]]))


# ---------------------------------------------------------------- mixture head

def test_golden_mixture_worked_examples():
    with open(os.path.join(GOLDEN, "mixture_worked_example.json")) as f:
        cases = json.load(f)["cases"]
    for c in cases:
        logits = _arr(c["logits"])
        p_mix, alpha = oracle.mixture_head(logits, 1)
        np.testing.assert_allclose(alpha, _arr(c["alpha"]), rtol=0, atol=1e-14, err_msg=c["name"])
        np.testing.assert_allclose(p_mix, _arr(c["p_mix"]), rtol=0, atol=1e-14, err_msg=c["name"])


def test_mixture_of_identical_flows_is_the_flow():
    rng = np.random.default_rng(70)
    l = rng.normal(size=(3, 50)) * 3
    p_mix, alpha = oracle.mixture_head(np.concatenate([l, l]), 3)
    e = np.exp(l - l.max(axis=1, keepdims=True))
    np.testing.assert_allclose(p_mix, e / e.sum(axis=1, keepdims=True), rtol=1e-13, atol=0)
    assert np.all(alpha > 0.5) and np.all(alpha < 1.0)


def test_mixture_weight_limits():
    V = 1000
    # uniform primary: collision probability 1/V, alpha = 1/2 + 1/(2V)
    l = np.concatenate([np.full((1, V), -2.5), np.zeros((1, V))])
    _, alpha = oracle.mixture_head(l, 1)
    assert alpha[0] == pytest.approx(0.5 + 0.5 / V, abs=1e-15)
    # one-hot primary (a logit 1000 above the rest): alpha = 1, the mixture is
    # the primary distribution (a swapped weight would give the aux one)
    l1 = np.zeros(V)
    l1[17] = 1000.0
    l2 = np.linspace(-1, 1, V)
    p_mix, alpha = oracle.mixture_head(np.stack([l1, l2]), 1)
    assert alpha[0] == 1.0
    assert p_mix[0, 17] == 1.0 and np.all(np.delete(p_mix[0], 17) == 0.0)


def test_mixture_invariants_and_primary_only_weight():
    rng = np.random.default_rng(71)
    B, V = 4, 257
    l = rng.normal(size=(2 * B, V)) * rng.uniform(0.1, 6, size=(2 * B, 1))
    p_mix, alpha = oracle.mixture_head(l, B)
    np.testing.assert_allclose(p_mix.sum(axis=1), 1.0, rtol=0, atol=1e-13)
    assert np.all(p_mix >= 0) and np.all((alpha >= 0.5) & (alpha <= 1.0))
    # alpha reads only the primary rows: any aux logits (NaN included) leave it unchanged
    l_bad = l.copy()
    l_bad[B:] = np.nan
    _, alpha_bad = oracle.mixture_head(l_bad, B)
    np.testing.assert_array_equal(alpha, alpha_bad)
    # a flow swap is visible: exchanging the rows changes the mixture
    p_swap, _ = oracle.mixture_head(np.concatenate([l[B:], l[:B]]), B)
    assert not np.allclose(p_swap, p_mix)


# ---------------------------------------------------------------- MoE router replay

def _moe_fixture_experts(u):
    E = len(u)
    w_gu = np.zeros((E, 2, 2))
    w_gu[:, 0, 0] = 40.0          # gate row (40, 0)
    w_gu[:, 1, 0] = u             # up row (u_e, 0)
    w_down = np.zeros((E, 2, 1))
    w_down[:, 0, 0] = 1.0         # down column (1, 0)
    return w_gu, w_down


def test_golden_moe_router_replay():
    with open(os.path.join(GOLDEN, "moe_router_replay_worked_example.json")) as f:
        fx = json.load(f)
    w_r = _arr(fx["w_router"])
    u = _arr(fx["u"])
    w_gu, w_down = _moe_fixture_experts(u)
    S = 40.0 / (1.0 + math.exp(-40.0))
    for c in fx["cases"]:
        y1, y2, ids, g1, g2 = oracle.moe_forward(_arr(fx["x1"]), _arr(fx["x2"]), w_r, w_gu, w_down,
                                                 c["k"], c["k_aux"], round_bf16=False)
        np.testing.assert_array_equal(ids, np.array(c["ids"]), err_msg=c["name"])
        np.testing.assert_allclose(g1, _arr(c["g1"]), rtol=0, atol=1e-15, err_msg=c["name"])
        np.testing.assert_allclose(g2, _arr(c["g2"]), rtol=0, atol=1e-15, err_msg=c["name"])
        np.testing.assert_allclose(y1, S * _arr(c["y1_over_S"]), rtol=1e-14, atol=0, err_msg=c["name"])
        np.testing.assert_allclose(y2, S * _arr(c["y2_over_S"]), rtol=1e-14, atol=0, err_msg=c["name"])


def _moe_case(seed, B=6, d=32, E=5, F=16):
    rng = np.random.default_rng(seed)
    return (rng.normal(size=(B, d)), rng.normal(size=(B, d)), rng.normal(size=(E, d)),
            rng.normal(size=(E, 2 * F, d)) * 0.2, rng.normal(size=(E, d, F)) * 0.2)


def test_moe_identical_flows_and_primary_blind_to_aux():
    x1, x2, wr, wgu, wd = _moe_case(90)
    y1, y2, ids, g1, g2 = oracle.moe_forward(x1, x1, wr, wgu, wd, 2)
    np.testing.assert_array_equal(y1, y2)
    np.testing.assert_array_equal(g1, g2)
    ya, _, ida, ga, _ = oracle.moe_forward(x1, x2, wr, wgu, wd, 2, 4)
    bad = np.full_like(x2, np.nan)
    yb, y2b, idb, gb, g2b = oracle.moe_forward(x1, bad, wr, wgu, wd, 2, 4)
    np.testing.assert_array_equal(ida, idb)
    np.testing.assert_array_equal(ga, gb)
    np.testing.assert_array_equal(ya, yb)
    assert np.isnan(y2b).all() and np.isnan(g2b).all()
    np.testing.assert_allclose(g1.sum(axis=1), 1.0, atol=1e-15)


def test_moe_relabelled_experts_give_the_same_outputs():
    x1, x2, wr, wgu, wd = _moe_case(91)
    perm = np.array([3, 0, 4, 1, 2])
    y1, y2, ids, _, _ = oracle.moe_forward(x1, x2, wr, wgu, wd, 2, 3)
    z1, z2, jds, _, _ = oracle.moe_forward(x1, x2, wr[perm], wgu[perm], wd[perm], 2, 3)
    np.testing.assert_allclose(z1, y1, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(z2, y2, rtol=1e-12, atol=1e-12)
    np.testing.assert_array_equal(perm[jds], ids)   # same experts under the new labels


def test_moe_limits_reduce_to_the_dense_mlp():
    x1, x2, wr, wgu, wd = _moe_case(92, E=4)
    # a zero router: every logit ties, gates are uniform over k = E experts;
    # with identical experts the block is that expert
    same_gu = np.repeat(wgu[:1], 4, axis=0)
    same_d = np.repeat(wd[:1], 4, axis=0)
    y1, _, ids, g1, _ = oracle.moe_forward(x1, x2, np.zeros_like(wr), same_gu, same_d, 4,
                                           round_bf16=False)
    np.testing.assert_array_equal(ids, np.tile(np.arange(4), (x1.shape[0], 1)))
    np.testing.assert_allclose(g1, 0.25, atol=1e-15)
    # one expert, k = 1: the dense SwiGLU MLP (matmul, SiLU(gate) * up, matmul)
    y1, y2, _, _, _ = oracle.moe_forward(x1, x2, wr[:1], wgu[:1], wd[:1], 1, round_bf16=False)
    gu = oracle.grouped_proj(np.concatenate([x1, x2]), wgu[0], x1.shape[0])
    h = oracle.swiglu_couple(gu, wgu.shape[1] // 2, x1.shape[0])
    dense = oracle.grouped_proj(h, wd[0], x1.shape[0])
    np.testing.assert_allclose(np.concatenate([y1, y2]), dense, rtol=1e-12, atol=1e-12)


def test_moe_given_selection():
    # The selection passed in replaces the oracle's own ranking: its own ids
    # reproduce every output bit for bit; the same set in another order
    # permutes the gates with it and leaves each flow's sum over the set as it
    # was; a different set changes the outputs.
    x1, x2, wr, wgu, wd = _moe_case(93)
    y1, y2, ids, g1, g2 = oracle.moe_forward(x1, x2, wr, wgu, wd, 2, 2, round_bf16=False)
    z1, z2, jds, h1, h2 = oracle.moe_forward(x1, x2, wr, wgu, wd, 2, 2, round_bf16=False, ids=ids)
    for a, b in ((y1, z1), (y2, z2), (ids, jds), (g1, h1), (g2, h2)):
        np.testing.assert_array_equal(a, b)
    swapped = ids[:, ::-1].copy()
    s1, s2, _, sg1, sg2 = oracle.moe_forward(x1, x2, wr, wgu, wd, 2, 2, round_bf16=False,
                                             ids=swapped)
    np.testing.assert_allclose(sg1, g1[:, ::-1], rtol=0, atol=1e-15)
    np.testing.assert_allclose(sg2, g2[:, ::-1], rtol=0, atol=1e-15)
    np.testing.assert_allclose(s1, y1, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(s2, y2, rtol=1e-12, atol=1e-12)
    other = ids.copy()
    other[:, 1] = [next(e for e in range(5) if e not in ids[t]) for t in range(ids.shape[0])]
    o1, _, _, og1, _ = oracle.moe_forward(x1, x2, wr, wgu, wd, 2, 2, round_bf16=False, ids=other)
    assert np.abs(o1 - y1).max() > 1e-3
    r1 = x1 @ wr.T
    np.testing.assert_allclose(og1, oracle.softmax_rows(np.take_along_axis(r1, other, axis=1)),
                               rtol=0, atol=1e-15)
