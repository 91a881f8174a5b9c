"""Pins of the CPU oracle against what the pages and the mathematics fix.

Each test checks the oracle against something other than itself: a
hand-derived closed form, brute-force enumeration, a plain-Python
evaluation, an identity of the definition, or an invariant.  The last test
plants plausible mistakes in the oracle and checks that the pins catch them.
"""
import itertools
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest

from oracle import moe_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
LN2, LN3 = math.log(2.0), math.log(3.0)


def _ev(v):
    """Evaluate a fixture entry: number, 'p/q', 'p/q*ln3', 'ln2', 'ln3'."""
    if isinstance(v, (int, float)):
        return float(v)
    if isinstance(v, list):
        return [_ev(u) for u in v]
    s = v.strip()
    if s == "ln3":
        return LN3
    if s == "ln2":
        return LN2
    if s.endswith("*ln3"):
        return float(Fraction(s[:-4])) * LN3
    return float(Fraction(s))


def _golden_layer():
    with open(os.path.join(GOLDEN, "worked_layer.json")) as f:
        g = json.load(f)
    inp = {k: (np.array(_ev(v), dtype=np.float64) if isinstance(v, list) else v)
           for k, v in g["inputs"].items()}
    exp = {k: np.array(_ev(v), dtype=np.float64) for k, v in g["expected"].items()}
    return inp, exp


def _run_golden(forward):
    inp, _ = _golden_layer()
    return forward(inp["x"], inp["w_router"], inp["w_gate"], inp["w_up"], inp["w_down"], inp["k"],
                   ws_gate=inp["ws_gate"], ws_up=inp["ws_up"], ws_down=inp["ws_down"],
                   routed_scaling_factor=inp["routed_scaling_factor"])


def _golden_mismatches(forward):
    _, exp = _golden_layer()
    try:
        out = _run_golden(forward)
    except Exception as e:  # a planted mistake may also break shapes
        return [f"raised {type(e).__name__}"]
    bad = []
    if not np.array_equal(np.asarray(out["topk_idx"]), exp["topk_idx"].astype(np.int64)):
        bad.append("topk_idx")
    for key in ("topk_w", "R", "Sh", "y"):
        if not np.allclose(out[key], exp[key], rtol=1e-13, atol=1e-13):
            bad.append(key)
    return bad


# ---------------------------------------------------------------- closed forms

def test_golden_worked_layer_closed_form():
    assert _golden_mismatches(O.moe_forward) == []


def test_golden_router_scores_are_sigmoid():
    inp, exp = _golden_layer()
    idx, w, scores, logits = O.route(inp["x"], inp["w_router"], None, inp["k"])
    assert np.allclose(scores[0], exp["scores_token0"], rtol=1e-15, atol=0)
    assert np.allclose(logits[0], [LN3, 0.0, LN2], rtol=1e-15, atol=0)


def test_silu_and_sigmoid_special_values():
    assert O.sigmoid(0.0) == 0.5
    assert O.silu(0.0) == 0.0
    assert math.isclose(float(O.sigmoid(LN3)), 0.75, rel_tol=1e-15)
    assert math.isclose(float(O.silu(-LN3)), -0.25 * LN3, rel_tol=1e-15)
    # silu(z) - silu(-z) = z for every z (sigma(z) + sigma(-z) = 1)
    z = np.linspace(-20, 20, 101)
    assert np.allclose(O.silu(z) - O.silu(-z), z, rtol=1e-14, atol=1e-14)


# ---------------------------------------------------------------- definitions

def _rand_layer(rng, T, d, E, F, Fs, scale=0.3):
    f = lambda *s: rng.standard_normal(s) * scale
    return dict(x=rng.standard_normal((T, d)), w_router=f(E, d), w_gate=f(E, F, d),
                w_up=f(E, F, d), w_down=f(E, d, F),
                ws_gate=f(Fs, d) if Fs else None, ws_up=f(Fs, d) if Fs else None,
                ws_down=f(d, Fs) if Fs else None)


def _fwd(L, k, **kw):
    return O.moe_forward(L["x"], L["w_router"], L["w_gate"], L["w_up"], L["w_down"], k,
                         ws_gate=L["ws_gate"], ws_up=L["ws_up"], ws_down=L["ws_down"], **kw)


def test_normalised_weights_sum_to_one():
    rng = np.random.default_rng(1)
    for (E, k) in [(16, 4), (8, 1), (8, 8), (256, 8), (64, 16)]:
        L = _rand_layer(rng, 50, 32, E, 8, 0)
        _, w, _, _ = O.route(L["x"], L["w_router"], None, k)
        assert np.all(np.abs(w.sum(axis=1) - 1.0) <= 1e-12)
        assert np.all(w > 0)


def test_routed_output_is_exactly_scale_times_weighted_sum():
    rng = np.random.default_rng(2)
    L = _rand_layer(rng, 20, 16, 8, 4, 4)
    L0 = dict(L, ws_gate=np.zeros_like(L["ws_gate"]), ws_up=np.zeros_like(L["ws_up"]),
              ws_down=np.zeros_like(L["ws_down"]))
    a = _fwd(L0, 3, routed_scaling_factor=2.5)
    b = _fwd(L0, 3, routed_scaling_factor=1.0)
    # shared weights zero isolate the routed path: y = 2.5 R bit for bit
    assert np.array_equal(a["Sh"], np.zeros_like(a["Sh"]))
    assert np.array_equal(a["y"], 2.5 * b["y"])
    assert np.array_equal(a["y"], 2.5 * a["R"])
    # with the shared expert on, the scale touches the routed part only
    c = _fwd(L, 3, routed_scaling_factor=2.5)
    assert np.allclose(c["y"] - c["Sh"], 2.5 * c["R"], rtol=1e-13, atol=1e-14)
    assert np.allclose(c["y"], a["y"] + c["Sh"], rtol=1e-13, atol=1e-14)


def test_k_equal_one_gives_unit_weight():
    rng = np.random.default_rng(3)
    L = _rand_layer(rng, 40, 16, 8, 4, 0)
    idx, w, scores, _ = O.route(L["x"], L["w_router"], None, 1)
    assert np.all(w == 1.0)
    assert np.array_equal(idx[:, 0], np.argmax(scores, axis=1))


def test_k_equal_E_normalises_over_all_experts():
    rng = np.random.default_rng(4)
    L = _rand_layer(rng, 30, 16, 6, 4, 0)
    idx, w, scores, _ = O.route(L["x"], L["w_router"], None, 6)
    full = scores / scores.sum(axis=1, keepdims=True)
    assert np.allclose(w, np.take_along_axis(full, idx, axis=1), rtol=1e-15, atol=0)
    assert all(sorted(r) == list(range(6)) for r in idx.tolist())


def _py_logits_scores(x, w_router):
    T, d = len(x), len(x[0])
    lg = [[math.fsum(x[t][i] * w_router[e][i] for i in range(d)) for e in range(len(w_router))]
          for t in range(T)]
    sc = [[1.0 / (1.0 + math.exp(-v)) for v in row] for row in lg]
    return lg, sc


def _brute_force_topk(scores_row, k):
    """Subset of size k with the largest score sum; ties -> lexicographically smallest."""
    best, best_sum = None, None
    for sub in itertools.combinations(range(len(scores_row)), k):
        s = math.fsum(scores_row[e] for e in sub)
        if best is None or s > best_sum:
            best, best_sum = sub, s
    return best


@pytest.mark.parametrize("E", [2, 3, 4, 5, 6, 7, 8])
def test_selection_matches_brute_force_enumeration(E):
    rng = np.random.default_rng(10 + E)
    d, T = 6, 40
    # small dyadic integers: every logit is exact in any summation order, and
    # many exact ties occur, which pins the lower-index tie-break too
    x = rng.integers(-2, 3, size=(T, d)).astype(np.float64)
    wr = rng.integers(-2, 3, size=(E, d)).astype(np.float64) * 0.5
    wr[E - 1] = wr[0]  # an injected duplicate expert: identical scores
    _, sc = _py_logits_scores(x.tolist(), wr.tolist())
    for k in range(1, E + 1):
        idx, w, scores, _ = O.route(x, wr, None, k)
        for t in range(T):
            bf = _brute_force_topk(sc[t], k)
            assert tuple(sorted(idx[t].tolist())) == bf, (E, k, t)
            # listed by descending score, equal scores by ascending index
            key = [(-scores[t, e], e) for e in idx[t]]
            assert key == sorted(key)


def test_router_bias_shifts_logits_before_sigmoid():
    rng = np.random.default_rng(5)
    L = _rand_layer(rng, 25, 16, 8, 4, 0)
    b = rng.standard_normal(8)
    idx, w, scores, logits = O.route(L["x"], L["w_router"], b, 3)
    _, _, _, l0 = O.route(L["x"], L["w_router"], None, 3)
    assert np.allclose(logits, l0 + b[None, :], rtol=0, atol=1e-15)
    assert np.allclose(scores, 1 / (1 + np.exp(-(l0 + b))), rtol=1e-15, atol=0)


def _py_swiglu(xrow, wg, wu, wd):
    F, d = len(wg), len(xrow)
    h = []
    for f in range(F):
        g = math.fsum(wg[f][i] * xrow[i] for i in range(d))
        u = math.fsum(wu[f][i] * xrow[i] for i in range(d))
        h.append(g / (1.0 + math.exp(-g)) * u)
    return [math.fsum(wd[o][f] * h[f] for f in range(F)) for o in range(len(wd))]


def test_single_expert_reduces_to_dense_swiglu_mlp():
    """E=1, k=1: y = 2.5 * MLP(x) + MLP_shared(x), against plain-Python loops."""
    rng = np.random.default_rng(6)
    T, d, F, Fs = 5, 7, 3, 4
    L = _rand_layer(rng, T, d, 1, F, Fs, scale=0.5)
    out = _fwd(L, 1)
    for t in range(T):
        xr = L["x"][t].tolist()
        m = _py_swiglu(xr, L["w_gate"][0].tolist(), L["w_up"][0].tolist(), L["w_down"][0].tolist())
        s = _py_swiglu(xr, L["ws_gate"].tolist(), L["ws_up"].tolist(), L["ws_down"].tolist())
        ref = [2.5 * a + b for a, b in zip(m, s)]
        assert np.allclose(out["y"][t], ref, rtol=1e-12, atol=1e-14)
    assert np.all(out["topk_w"] == 1.0)


def test_full_layer_against_plain_python_per_token():
    """Small random layer, every token evaluated by definition in plain Python."""
    rng = np.random.default_rng(7)
    T, d, E, k, F, Fs = 6, 5, 5, 2, 3, 2
    L = _rand_layer(rng, T, d, E, F, Fs, scale=0.7)
    out = _fwd(L, k)
    lg, sc = _py_logits_scores(L["x"].tolist(), L["w_router"].tolist())
    for t in range(T):
        sel = _brute_force_topk(sc[t], k)
        tot = math.fsum(sc[t][e] for e in sel)
        acc = [0.0] * d
        for e in sel:
            o = _py_swiglu(L["x"][t].tolist(), L["w_gate"][e].tolist(), L["w_up"][e].tolist(),
                           L["w_down"][e].tolist())
            acc = [a + sc[t][e] / tot * v for a, v in zip(acc, o)]
        s = _py_swiglu(L["x"][t].tolist(), L["ws_gate"].tolist(), L["ws_up"].tolist(),
                       L["ws_down"].tolist())
        ref = [2.5 * a + b for a, b in zip(acc, s)]
        assert np.allclose(out["y"][t], ref, rtol=1e-12, atol=1e-14)


def test_unnormalised_weights_are_the_selected_sigmoid_scores():
    """norm_topk_prob off (a config key of the spec sheet; both Laguna models set it on):
    each weight is the selected expert's own sigmoid score, with no division by the sum.
    Every token evaluated by definition in plain Python."""
    rng = np.random.default_rng(21)
    T, d, E, k, F, Fs = 6, 5, 6, 3, 3, 2
    L = _rand_layer(rng, T, d, E, F, Fs, scale=0.7)
    out = _fwd(L, k, norm_topk_prob=False)
    _, sc = _py_logits_scores(L["x"].tolist(), L["w_router"].tolist())
    for t in range(T):
        sel = _brute_force_topk(sc[t], k)
        assert sorted(out["topk_idx"][t].tolist()) == list(sel)
        got_w = dict(zip(out["topk_idx"][t].tolist(), out["topk_w"][t].tolist()))
        assert all(math.isclose(got_w[e], sc[t][e], rel_tol=1e-14) for e in sel)
        acc = [0.0] * d
        for e in sel:
            o = _py_swiglu(L["x"][t].tolist(), L["w_gate"][e].tolist(), L["w_up"][e].tolist(),
                           L["w_down"][e].tolist())
            acc = [a + sc[t][e] * v for a, v in zip(acc, o)]
        s = _py_swiglu(L["x"][t].tolist(), L["ws_gate"].tolist(), L["ws_up"].tolist(),
                       L["ws_down"].tolist())
        ref = [2.5 * a + b for a, b in zip(acc, s)]
        assert np.allclose(out["y"][t], ref, rtol=1e-12, atol=1e-14)
    # the sum over the selection is not 1 (it is with normalisation on)
    assert np.all(np.abs(out["topk_w"].sum(axis=1) - 1.0) > 1e-3)


# ---------------------------------------------------------------- invariants

def test_token_permutation_equivariance():
    rng = np.random.default_rng(8)
    L = _rand_layer(rng, 33, 16, 8, 4, 4)
    p = rng.permutation(33)
    a = _fwd(L, 3)
    b = _fwd(dict(L, x=L["x"][p]), 3)
    assert np.allclose(b["y"], a["y"][p], rtol=1e-12, atol=1e-14)
    assert np.array_equal(b["topk_idx"], a["topk_idx"][p])


def test_expert_relabel_invariance():
    rng = np.random.default_rng(9)
    L = _rand_layer(rng, 33, 16, 8, 4, 4)
    pi = rng.permutation(8)            # expert e becomes pi[e]
    inv = np.argsort(pi)
    M = dict(L)
    for key in ("w_router", "w_gate", "w_up", "w_down"):
        M[key] = L[key][inv]
    a = _fwd(L, 3)
    b = _fwd(M, 3)
    assert np.allclose(b["y"], a["y"], rtol=1e-12, atol=1e-14)
    assert [sorted(r) for r in b["topk_idx"].tolist()] == \
           [sorted(pi[r].tolist()) for r in a["topk_idx"]]


def test_linear_in_down_projection():
    rng = np.random.default_rng(11)
    L = _rand_layer(rng, 17, 16, 8, 4, 0)
    a = _fwd(L, 2)
    b = _fwd(dict(L, w_down=2.0 * L["w_down"]), 2)
    c = _fwd(dict(L, w_down=-0.75 * L["w_down"]), 2)
    assert np.array_equal(b["R"], 2.0 * a["R"])
    assert np.allclose(c["R"], -0.75 * a["R"], rtol=1e-13, atol=1e-15)


def test_tokens_are_independent():
    rng = np.random.default_rng(12)
    L = _rand_layer(rng, 40, 16, 8, 4, 4)
    a = _fwd(L, 3)
    sub = np.array([3, 17, 39, 0])
    b = _fwd(dict(L, x=L["x"][sub]), 3)
    assert np.allclose(b["y"], a["y"][sub], rtol=1e-12, atol=1e-14)


def test_expert_order_against_brute_force():
    rng = np.random.default_rng(13)
    for (T, E, k) in [(1, 4, 2), (37, 16, 4), (200, 8, 8), (64, 64, 1)]:
        idx = np.stack([rng.permutation(E)[:k] for _ in range(T)])
        counts, offsets, perm = O.expert_order(idx, E)
        assert counts.sum() == T * k and offsets[-1] == T * k
        assert sorted(perm.tolist()) == list(range(T * k))        # a bijection
        for e in range(E):
            want = [t * k + j for t in range(T) for j in range(k) if idx[t, j] == e]
            assert perm[offsets[e]:offsets[e + 1]].tolist() == want
            assert counts[e] == len(want)


# ---------------------------------------------------------------- selection-only bias

@pytest.mark.parametrize("E", [3, 5, 8])
def test_selection_bias_chooses_by_biased_score_weights_unbiased(E):
    """Auxiliary-loss-free variant: the k experts maximise sum(sigmoid(l) + b) (brute force,
    lexicographic-min on ties), the weights are the unbiased sigmoid scores normalised over them
    (plain Python)."""
    rng = np.random.default_rng(30 + E)
    d, T = 6, 30
    x = rng.standard_normal((T, d))
    wr = rng.standard_normal((E, d)) * 0.4
    b = rng.standard_normal(E) * 0.15
    _, sc = _py_logits_scores(x.tolist(), wr.tolist())
    for k in range(1, E + 1):
        idx, w, keys, _ = O.route(x, wr, None, k, selection_bias=b)
        for t in range(T):
            biased = [sc[t][e] + b[e] for e in range(E)]
            bf = _brute_force_topk(biased, k)
            assert tuple(sorted(idx[t].tolist())) == bf, (E, k, t)
            tot = math.fsum(sc[t][e] for e in bf)
            for j, e in enumerate(idx[t]):
                assert abs(w[t, j] - sc[t][e] / tot) <= 1e-15
                assert keys[t, e] == sc[t][e] + b[e] or abs(keys[t, e] - (sc[t][e] + b[e])) < 1e-15


def test_selection_bias_zero_is_the_plain_router_and_a_large_bias_forces_an_expert():
    rng = np.random.default_rng(40)
    L = _rand_layer(rng, 25, 16, 8, 4, 4)
    a = _fwd(L, 3)
    z = _fwd(L, 3, selection_bias=np.zeros(8))
    assert np.array_equal(z["topk_idx"], a["topk_idx"]) and np.array_equal(z["y"], a["y"])
    b = np.zeros(8)
    b[5] = 2.0  # sigmoid scores lie in (0, 1): +2 puts expert 5 first for every token
    f = _fwd(L, 3, selection_bias=b)
    assert np.all(f["topk_idx"][:, 0] == 5)
    _, _, s, _ = O.route(L["x"], L["w_router"], None, 3)
    sel = np.take_along_axis(s, f["topk_idx"], axis=1)
    assert np.allclose(f["topk_w"], sel / sel.sum(axis=1, keepdims=True), rtol=0, atol=1e-15)
    # the pin is sensitive: weights from the biased scores, or selection on biased logits,
    # give other results
    keys = s + b[None, :]
    wrong_w = np.take_along_axis(keys, f["topk_idx"], axis=1)
    assert not np.allclose(f["topk_w"], wrong_w / wrong_w.sum(axis=1, keepdims=True))
    lg = O.router_logits(L["x"], L["w_router"], None)
    b2 = rng.standard_normal(8) * 0.3
    sel_keys = O.select_topk(O.sigmoid(lg) + b2[None, :], 3)
    sel_logits = O.select_topk(lg + b2[None, :], 3)
    got = O.route(L["x"], L["w_router"], None, 3, selection_bias=b2)[0]
    assert np.array_equal(got, sel_keys) and not np.array_equal(got, sel_logits)


# ---------------------------------------------------------------- e4m3 (FP8 experts)

def test_e4m3_code_table_follows_the_format():
    v = O.e4m3_value(np.arange(256))
    assert v[0x38] == 1.0 and v[0xB8] == -1.0 and v[0x40] == 2.0 and v[0x3C] == 1.5
    assert v[0x7E] == 448.0 and np.isnan(v[0x7F]) and np.isnan(v[0xFF])
    assert v[0x08] == 2.0 ** -6 and v[0x01] == 2.0 ** -9 and v[0x07] == 7 * 2.0 ** -9
    assert v[0x00] == 0.0 and v[0x80] == 0.0
    assert np.all(np.diff(v[:0x7F]) > 0)           # codes 0..0x7E strictly increasing
    assert np.array_equal(v[0x80:0xFF], -v[:0x7F])


def _e4m3_brute(x):
    """Nearest finite e4m3 value by exhaustive search; ties to the even code; |x| > 448 -> 448."""
    codes = np.array([c for c in range(256) if not np.isnan(O.e4m3_value(c))])
    vals = O.e4m3_value(codes)
    out = []
    for xv in np.asarray(x, dtype=np.float64):
        xs = min(max(xv, -448.0), 448.0)
        dist = np.abs(vals - xs)
        best = codes[dist == dist.min()]
        if len(best) > 1:
            nz = [c for c in best if O.e4m3_value(c) != 0.0] or list(best)
            even = [c for c in nz if c % 2 == 0]
            best = even if even else nz
            if O.e4m3_value(best[0]) == 0.0:  # zero keeps the input's sign
                best = [0x80 if np.signbit(xv) else 0x00]
        out.append(best[0])
    return np.array(out)


def test_e4m3_rounding_against_exhaustive_search():
    rng = np.random.default_rng(50)
    mag = 2.0 ** rng.uniform(-12, 10, 3000)
    x = (mag * rng.choice([-1.0, 1.0], 3000)).astype(np.float32)
    got = O.e4m3_round(x)
    want = _e4m3_brute(x)
    same = (got == want) | ((O.e4m3_value(got) == 0) & (O.e4m3_value(want) == 0))
    assert same.all(), x[~same][:5]


def test_e4m3_ties_go_to_even_and_large_values_saturate():
    v = O.e4m3_value(np.arange(0x7F))
    mids = ((v[:-1] + v[1:]) / 2).astype(np.float32)
    exact = mids.astype(np.float64) == (v[:-1] + v[1:]) / 2   # midpoints exact in float32
    codes = O.e4m3_round(mids[exact])
    assert np.all(codes % 2 == 0)
    big = np.array([449, 464, 480, 500, 1e6, 3e38], np.float32)
    assert np.all(O.e4m3_round(big) == 0x7E) and np.all(O.e4m3_round(-big) == 0xFE)


def test_power_of_two_row_scales():
    """pow2 scales: the smallest power of two >= amax / 448, so every scaled value lies in
    (-448, 448] and scaling is exact (codes depend on each element alone)."""
    rng = np.random.default_rng(53)
    a = (rng.standard_normal((30, 64)) * 10.0 ** rng.uniform(-4, 3, (30, 1))).astype(np.float32)
    a[0, :] = 0.0
    a[1, :] = 0.0
    a[1, :3] = [448.0, -1.0, 2.0]      # amax / 448 = 1 exactly: the scale stays 1
    codes, s = O.quantize_rows_e4m3(a, pow2=True)
    mant, ex = np.frexp(s.astype(np.float64))
    assert np.all(mant == 0.5)                                     # powers of two
    t = np.max(np.abs(a), axis=1).astype(np.float32) / np.float32(448.0)
    nz = t > 0
    assert np.all(s[nz] >= t[nz]) and np.all(s[nz] / 2 < t[nz]) and s[0] == 1.0 and s[1] == 1.0
    assert np.all(np.abs(O.e4m3_value(codes)) <= 448.0)
    # exact scaling: the codes equal those of each element divided by the scale
    want = O.e4m3_round((a.astype(np.float64) / s[:, None]).astype(np.float32))
    same = (codes == want) | ((O.e4m3_value(codes) == 0) & (O.e4m3_value(want) == 0))
    assert same.all()


def test_per_row_quantization_error_bound():
    rng = np.random.default_rng(51)
    a = (rng.standard_normal((40, 300)) * 10.0 ** rng.uniform(-3, 2, (40, 1))).astype(np.float32)
    a[3] = 0.0
    codes, s = O.quantize_rows_e4m3(a)
    deq = O.dequantize_rows_e4m3(codes, s)
    assert s[3] == 1.0 and np.all(deq[3] == 0)
    assert np.all(np.abs(O.e4m3_value(codes)).max(axis=1)[np.arange(40) != 3] == 448.0)
    # round to nearest: at most half a quantum (2^-4 relative to the binade, 2^-10 below 2^-6)
    scaled = a.astype(np.float64) / s[:, None].astype(np.float64)
    quantum = np.where(np.abs(scaled) < 2.0 ** -6, 2.0 ** -9,
                       np.ldexp(1.0, np.frexp(np.abs(scaled))[1] - 4))
    assert np.all(np.abs(deq / s[:, None] - scaled) <= quantum / 2 * (1 + 1e-6) + 1e-30)


def test_fp8_forward_against_plain_python_per_token():
    """The FP8-weight layer, token by token in plain Python: per-token x scale, per-row weight
    scales, h rounded to fp16 then quantized per row, routing and combine as in the 16-bit
    layer."""
    rng = np.random.default_rng(52)
    T, d, E, k, F, Fs = 5, 8, 3, 2, 4, 4
    L = _rand_layer(rng, T, d, E, F, Fs, scale=0.5)
    L = {key: (None if v is None else v.astype(np.float32)) for key, v in L.items()}
    fp8 = O.quantize_experts_fp8(L["w_gate"], L["w_up"], L["w_down"],
                                 L["ws_gate"], L["ws_up"], L["ws_down"])
    out = O.moe_forward_fp8(L["x"], L["w_router"], fp8, k)
    ref_route = O.route(L["x"], L["w_router"], None, k)

    def q_row(vals, pow2=False):
        amax = max(abs(float(v)) for v in vals)
        sc = float(np.float32(np.float32(amax) / np.float32(448.0))) if amax > 0 else 1.0
        if pow2 and amax > 0:
            sc = 2.0 ** math.ceil(math.log2(sc))  # exact for these (normal) values
        rc = np.float32(np.float32(1.0) / np.float32(sc))
        codes = [int(O.e4m3_round(np.float32(np.float32(v) * rc))) for v in vals]
        return [float(O.e4m3_value(c)) * sc for c in codes]

    def mat(w):  # dequantized rows of a weight matrix
        return [q_row(r) for r in w.tolist()]

    def ffn(xq, g, u, dn):
        h = []
        for f in range(len(g)):
            a = math.fsum(xq[i] * g[f][i] for i in range(len(xq)))
            b = math.fsum(xq[i] * u[f][i] for i in range(len(xq)))
            h.append(float(np.float32(np.float16(a / (1.0 + math.exp(-a)) * b))))
        hq = q_row(h, pow2=True)
        return [math.fsum(hq[j] * dn[o][j] for j in range(len(hq))) for o in range(len(dn))]

    for t in range(T):
        xq = q_row(L["x"][t].tolist())
        acc = [0.0] * d
        for j in range(k):
            e = int(ref_route[0][t, j])
            o = ffn(xq, mat(L["w_gate"][e]), mat(L["w_up"][e]), mat(L["w_down"][e]))
            acc = [a + ref_route[1][t, j] * v for a, v in zip(acc, o)]
        sh = ffn(xq, mat(L["ws_gate"]), mat(L["ws_up"]), mat(L["ws_down"]))
        want = [2.5 * a + b for a, b in zip(acc, sh)]
        assert np.allclose(out["y"][t], want, rtol=1e-12, atol=1e-14), t


# ---------------------------------------------------------------- padding mask

def test_padding_token_gets_shared_expert_only():
    """A masked token is not routed: y_t equals the shared expert alone, evaluated in plain
    Python; its slots carry the not-routed id and zero weight."""
    rng = np.random.default_rng(21)
    T, d, E, k, F, Fs = 9, 6, 5, 2, 3, 4
    L = _rand_layer(rng, T, d, E, F, Fs, scale=0.6)
    mask = np.array([1, 0, 1, 1, 0, 0, 1, 0, 1], dtype=np.uint8)
    out = _fwd(L, k, token_mask=mask)
    for t in np.nonzero(mask == 0)[0]:
        s = _py_swiglu(L["x"][t].tolist(), L["ws_gate"].tolist(), L["ws_up"].tolist(),
                       L["ws_down"].tolist())
        assert np.allclose(out["y"][t], s, rtol=1e-12, atol=1e-14)
        assert np.all(out["R"][t] == 0.0)
        assert np.all(out["topk_idx"][t] == O.NOT_ROUTED) and np.all(out["topk_w"][t] == 0.0)
    # the pin is sensitive: routing the masked tokens would change their outputs
    full = _fwd(L, k)
    assert not np.allclose(full["y"][mask == 0], out["y"][mask == 0])
    # the same layer without a shared expert gives exact zeros for masked tokens
    L0 = dict(L, ws_gate=None, ws_up=None, ws_down=None)
    out0 = _fwd(L0, k, token_mask=mask)
    assert np.all(out0["y"][mask == 0] == 0.0)


def test_mask_leaves_other_tokens_unchanged():
    """Tokens are independent, so masking some changes nothing for the others."""
    rng = np.random.default_rng(22)
    L = _rand_layer(rng, 40, 16, 8, 4, 4)
    mask = (rng.random(40) < 0.6).astype(np.uint8)
    a = _fwd(L, 3)
    b = _fwd(L, 3, token_mask=mask)
    keep = mask == 1
    assert np.array_equal(b["y"][keep], a["y"][keep])
    assert np.array_equal(b["topk_idx"][keep], a["topk_idx"][keep])
    assert np.array_equal(b["topk_w"][keep], a["topk_w"][keep])
    ones = _fwd(L, 3, token_mask=np.ones(40, np.uint8))
    assert np.array_equal(ones["y"], a["y"])


def test_expert_order_skips_unrouted_pairs():
    """Counts cover the routed pairs only; perm is a bijection onto them, in (t, j) order."""
    rng = np.random.default_rng(23)
    T, E, k = 50, 8, 3
    idx = np.stack([rng.permutation(E)[:k] for _ in range(T)])
    pad = rng.random(T) < 0.3
    idx[pad] = O.NOT_ROUTED
    counts, offsets, perm = O.expert_order(idx, E)
    routed = [t * k + j for t in range(T) for j in range(k) if not pad[t]]
    assert counts.sum() == len(routed) == k * int((~pad).sum()) and offsets[-1] == len(routed)
    assert sorted(perm.tolist()) == routed
    for e in range(E):
        want = [t * k + j for t in range(T) for j in range(k) if idx[t, j] == e]
        assert perm[offsets[e]:offsets[e + 1]].tolist() == want
    none, noff, nperm = O.expert_order(np.full((4, 2), O.NOT_ROUTED), E)
    assert none.sum() == 0 and noff[-1] == 0 and nperm.size == 0


def test_bf16_widening_is_exact():
    bits = np.array([0x3F80, 0xBF80, 0x0000, 0x8000, 0x3E80, 0x4049, 0x7F7F, 0x0080], np.uint16)
    want = [1.0, -1.0, 0.0, -0.0, 0.25, 3.140625, 3.3895313892515355e38, 2.0 ** -126]
    assert O.bf16_to_f64(bits).tolist() == want


# ---------------------------------------------------------------- planted mistakes

def _variant_forward(mistake):
    """The oracle's forward with one plausible mistake planted (CPU only)."""
    def fwd(x, w_router, w_gate, w_up, w_down, k, *, ws_gate=None, ws_up=None, ws_down=None,
            routed_scaling_factor=2.5, router_bias=None, norm_topk_prob=True):
        X = O.bf16_to_f64(x)
        logits = O.router_logits(x, w_router, router_bias)
        if mistake == "softmax_router":
            ex = np.exp(logits - logits.max(axis=1, keepdims=True))
            scores = ex / ex.sum(axis=1, keepdims=True)
        else:
            scores = O.sigmoid(logits)
        if mistake == "ties_to_higher_index":
            rev = np.argsort(-logits[:, ::-1], axis=1, kind="stable")
            idx = (logits.shape[1] - 1 - rev)[:, :k]
        else:
            idx = O.select_topk(logits, k)
        sel = np.take_along_axis(scores, idx, axis=1)
        w = sel if mistake == "no_normalisation" else sel / sel.sum(axis=1, keepdims=True)

        def ffn(xr, wg, wu, wd):
            g = xr @ np.asarray(wg, float).T
            u = xr @ np.asarray(wu, float).T
            if mistake == "silu_on_up":
                h = g * O.silu(u)
            elif mistake == "no_gate_nonlinearity":
                h = g * u
            else:
                h = O.silu(g) * u
            return h @ np.asarray(wd, float).T

        T, d = X.shape
        R = np.zeros((T, d))
        for t in range(T):
            for j in range(k):
                e = idx[t, j]
                R[t] += w[t, j] * ffn(X[t:t + 1], w_gate[e], w_up[e], w_down[e])[0]
        Sh = ffn(X, ws_gate, ws_up, ws_down)
        if mistake == "scale_on_shared_too":
            y = routed_scaling_factor * (R + Sh)
        elif mistake == "shared_dropped":
            y = routed_scaling_factor * R
        elif mistake == "scale_dropped":
            y = R + Sh
        else:
            y = routed_scaling_factor * R + Sh
        return {"y": y, "R": R, "Sh": Sh if mistake != "shared_dropped" else Sh, "topk_idx": idx,
                "topk_w": w}
    return fwd


@pytest.mark.parametrize("mistake", ["softmax_router", "ties_to_higher_index", "no_normalisation",
                                     "silu_on_up", "no_gate_nonlinearity", "scale_on_shared_too",
                                     "shared_dropped", "scale_dropped"])
def test_pins_catch_planted_mistakes(mistake):
    assert _golden_mismatches(_variant_forward("none")) == []
    assert _golden_mismatches(_variant_forward(mistake)) != []
