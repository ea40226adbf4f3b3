"""Pins of the oracle's decoder-layer composition (CPU only).

The layer step chains RMSNorm -> grouped QKV -> primary-only append -> dual
attention -> grouped W_o + residual -> RMSNorm -> grouped gate/up (SwiGLU +
b coupling) -> grouped down + c coupling + residual. The invariants in
test_oracle.py (self-sufficient primary, twin flows, empty cache, zero output
weights) do not see the wiring between those steps; the hand-derived worked
example below does: every intermediate has a closed form, written out step by
step in tests/golden/layer_worked_example.json. The mutation runs plant
plausible wiring mistakes in a copy of the oracle's layer step and check that
the worked example catches each one.
"""

import inspect
import json
import math
import os
import textwrap

import numpy as np
import pytest

import oracle
from oracle import dualflow_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "layer_worked_example.json")

# The names the fixture's closed forms may use, and nothing else.
_NAMES = {"s": math.e / (1.0 + math.e), "ln3": math.log(3.0), "sqrt2": math.sqrt(2.0)}


def _val(expr):
    return float(eval(expr, {"__builtins__": {}}, dict(_NAMES)))  # noqa: S307 (fixture text)


def _arr(rows):
    return np.array([[_val(x) for x in r] for r in rows], dtype=np.float64) \
        if isinstance(rows[0], list) else np.array([_val(x) for x in rows], dtype=np.float64)


def _spec():
    with open(GOLDEN) as f:
        return json.load(f)


def _inputs(spec):
    z = spec["sizes"]
    bs, D, Hkv = z["block_size"], z["D"], z["Hkv"]
    kc = np.full((1, Hkv, bs, D), 9.0)  # slot 1 holds a marker the append must overwrite
    vc = np.full((1, Hkv, bs, D), 9.0)
    kc[0, 0, 0] = _arr(spec["cached_k"])[0]
    vc[0, 0, 0] = _arr(spec["cached_v"])[0]
    return dict(x1=_arr(spec["x1"]), x2=_arr(spec["x2"]), w_qkv=_arr(spec["w_qkv"]),
                w_o=_arr(spec["w_o"]), w_gu=_arr(spec["w_gu"]), w_down=_arr(spec["w_down"]),
                a=_arr(spec["a"]), b=_arr(spec["b"]), c=_arr(spec["c"]), k_cache=kc,
                v_cache=vc, block_table=np.array(spec["block_table"], dtype=np.int32),
                positions=np.array(spec["positions"], dtype=np.int32), Hq=z["Hq"], Hkv=Hkv,
                D=D, F=z["F"], round_bf16=False, eps=z["eps"])


def _mismatches(out, spec, tol=1e-12):
    """Names of the intermediates of ``out`` that differ from the fixture."""
    ex = spec["expected"]
    qd = spec["sizes"]["Hq"] * spec["sizes"]["D"]
    got = {
        "xn": out["xn"], "qkv_primary": out["qkv"][:1], "q2raw": out["qkv"][1:, :qd],
        "k_page_after": out["k_cache"][0, 0], "v_page_after": out["v_cache"][0, 0],
        "attn": out["attn"], "x_mid": out["x_mid"], "xn2": out["xn2"], "h": out["h"],
        "x_out": out["x_out"],
    }
    bad = []
    for name, g in got.items():
        want = _arr(ex[name])
        g = np.asarray(g, dtype=np.float64)
        if g.shape != want.shape or not np.all(np.abs(g - want) <= tol):
            bad.append(name)
    return bad


def test_fixture_closed_forms_match_their_decimals():
    spec = _spec()
    dec = spec["expected_decimal"]
    assert abs(_NAMES["s"] - dec["s"]) < 1e-15
    np.testing.assert_allclose(_arr(spec["expected"]["h"]), dec["h"], rtol=0, atol=1e-13)
    np.testing.assert_allclose(_arr(spec["expected"]["x_out"]), dec["x_out"], rtol=0, atol=1e-13)


def test_layer_step_worked_example():
    spec = _spec()
    out = oracle.layer_step(**_inputs(spec))
    assert _mismatches(out, spec) == []
    # the auxiliary rows' K/V columns are never computed (it never writes the cache)
    qd = spec["sizes"]["Hq"] * spec["sizes"]["D"]
    assert np.isnan(out["qkv"][1:, qd:]).all()


def test_layer_step_defaults():
    # eps of the worked example is 0 (exact closed forms); the layer's own
    # default is the stated reading (1e-5) and bf16 rounding at the stored
    # interfaces is on by default.
    sig = inspect.signature(oracle.layer_step)
    assert sig.parameters["eps"].default == 1e-5
    assert sig.parameters["round_bf16"].default is True


def test_layer_step_worked_example_with_bf16_interfaces():
    # xn, the primary Q/V columns, x_mid and the primary O are bf16-exact here,
    # so rounding at the stored interfaces leaves them unchanged; xn2 = 0.2,
    # 1.4 become the nearest bf16 values 205/1024 and 179/128.
    spec = _spec()
    inp = _inputs(spec)
    inp["round_bf16"] = True
    out = oracle.layer_step(**inp)
    np.testing.assert_array_equal(out["xn"], [[1, 1], [1, -1]])
    np.testing.assert_array_equal(out["qkv"][0, [0, 1, 4, 5]], [1, 1, 2, 0])
    np.testing.assert_array_equal(out["xn2"][0], [205 / 1024, 179 / 128])
    np.testing.assert_array_equal(out["xn2"][1], [-205 / 1024, -179 / 128])


# Plausible wiring mistakes, each planted as a text substitution in a copy of
# the oracle's layer step (only that copy is changed, and only on the CPU).
MUTATIONS = {
    "MLP fed from the first norm xn": ("grouped_proj(xn2, w_gu, B)", "grouped_proj(xn, w_gu, B)"),
    "QKV built from X, not xn": ("grouped_proj(xn, w_qkv, B, n_aux=qd)",
                                 "grouped_proj(X, w_qkv, B, n_aux=qd)"),
    "second norm dropped": ('xn2 = rd["xn2"](rmsnorm(x_mid, eps=eps))', 'xn2 = rd["xn2"](x_mid)'),
    "attention residual taken from xn": ("grouped_proj(attn, w_o, B), X, B, None)",
                                         "grouped_proj(attn, w_o, B), xn, B, None)"),
    "MLP residual taken from X": ("grouped_proj(h, w_down, B), x_mid, B, c)",
                                  "grouped_proj(h, w_down, B), X, B, c)"),
    "auxiliary query read from the primary rows": ("q2raw = qkv[B:, :qd]", "q2raw = qkv[:B, :qd]"),
    "K and V columns swapped": ("k_new = qkv[:B, qd:qd + kvd]", "k_new = qkv[:B, qd + kvd:qd + 2 * kvd]"),
    "attention before the append": ("decode_attn(q1, q2raw, a, kc, vc, block_table, seqlens)",
                                    "decode_attn(q1, q2raw, a, k_cache, v_cache, block_table, "
                                    "np.asarray(positions))"),
    "c coupling dropped": ("x_mid, B, c)", "x_mid, B, None)"),
    "b coupling dropped": ("F, B, b)", "F, B, None)"),
    "coupling vector a ignored": ("decode_attn(q1, q2raw, a,", "decode_attn(q1, q2raw, None,"),
}


def _mutant(old, new):
    src = textwrap.dedent(inspect.getsource(O.layer_step))
    assert src.count(old) == 1, "mutation pattern not found once: %r" % old
    ns = dict(vars(O))
    exec(compile(src.replace(old, new), "<mutant layer_step>", "exec"), ns)  # noqa: S102
    return ns["layer_step"]


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_worked_example_catches_planted_wiring_mistake(name):
    spec = _spec()
    old, new = MUTATIONS[name]
    out = _mutant(old, new)(**_inputs(spec))
    assert _mismatches(out, spec), "planted mistake not caught: %s" % name


def test_unmutated_copy_passes():
    # the mutation harness itself: a copy with a no-op substitution is exact
    spec = _spec()
    same = 'xn2 = rd["xn2"](rmsnorm(x_mid, eps=eps))'
    out = _mutant(same, same)(**_inputs(spec))
    assert _mismatches(out, spec) == []


def test_rounded_interfaces_option():
    # `rounded` names the intermediates rounded to bf16: all of them by
    # default, none equals round_bf16=False, one left out differs from the
    # default only from that point on (here xn2: x_mid is unchanged, h is not).
    spec = _spec()
    inp = _inputs(spec)
    inp["round_bf16"] = True
    inp["eps"] = 1e-5
    full = oracle.layer_step(**inp)
    same = oracle.layer_step(**dict(inp, rounded=oracle.LAYER_INTERFACES))
    none = oracle.layer_step(**dict(inp, rounded=()))
    exact = oracle.layer_step(**dict(inp, round_bf16=False))
    keep = oracle.layer_step(**dict(inp, rounded=tuple(n for n in oracle.LAYER_INTERFACES
                                                        if n != "xn2")))
    for k in ("xn", "qkv", "attn", "x_mid", "xn2", "h", "x_out"):
        np.testing.assert_array_equal(full[k], same[k])
        np.testing.assert_array_equal(none[k], exact[k])
    np.testing.assert_array_equal(keep["x_mid"], full["x_mid"])
    assert not np.array_equal(keep["xn2"], full["xn2"])
    np.testing.assert_array_equal(keep["xn2"], oracle.rmsnorm(full["x_mid"], eps=1e-5))
    with pytest.raises(ValueError):
        oracle.layer_step(**dict(inp, rounded=("xn3",)))
