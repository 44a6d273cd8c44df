"""Pins of the CPU oracle against facts fixed outside the oracle itself.

Each test checks the oracle against one of: a closed form, a hand-derived
example (tests/golden), an exact-arithmetic reference (Python ``fractions`` /
``math.fsum``), numpy's own binary16 conversion (an independent decoder), or
a brute-force enumeration of all products on tiny inputs.  The method is the
Effort approximate matvec of the Hacker News thread "Show HN: Speeding up
LLM inference 2x times (possibly)" (item 40067677): rows sorted by |w|
descending, probes, chart = v * probes, cutoff = topK(chart, effort), and the
multiply over the used leading part of each row.
"""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest

from oracle import effort_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def f16bits(a):
    return np.asarray(a, dtype=np.float16).view(np.uint16)


# ---------------------------------------------------------------- decoder pins
@pytest.mark.parametrize("bits,value", [
    (0x0000, 0.0), (0x3C00, 1.0), (0xBC00, -1.0), (0x4000, 2.0),
    (0x0001, 2.0 ** -24), (0x03FF, 1023 * 2.0 ** -24), (0x0400, 2.0 ** -14),
    (0x7BFF, 65504.0), (0x3555, 0.333251953125), (0xC500, -5.0),
])
def test_fp16_decoder_closed_forms(bits, value):
    assert O.fp16_bits_to_float64(np.array([bits], np.uint16))[0] == value


def test_fp16_decoder_signed_zero_inf_nan():
    d = O.fp16_bits_to_float64(np.array([0x8000, 0x7C00, 0xFC00, 0x7E00], np.uint16))
    assert d[0] == 0.0 and math.copysign(1.0, d[0]) == -1.0
    assert d[1] == math.inf and d[2] == -math.inf and math.isnan(d[3])


def test_fp16_decoder_matches_numpy_on_all_patterns():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    mine = O.fp16_bits_to_float64(bits)
    ref = bits.view(np.float16).astype(np.float64)
    finite = np.isfinite(ref)
    assert np.array_equal(mine[finite], ref[finite])
    assert np.array_equal(np.signbit(mine[finite]), np.signbit(ref[finite]))
    assert np.array_equal(np.isnan(mine), np.isnan(ref))


# ------------------------------------------------------------ keep / K / probes
@pytest.mark.parametrize("out_dim,keep,n", [
    (4096, 1.0, 4096), (14336, 0.75, 10752), (1024, 0.8, 819), (3, 0.5, 2),
    (4, 0.5, 2), (10, 0.05, 1), (10, 0.04, 0),
])
def test_kept_count(out_dim, keep, n):
    assert O.kept_count(out_dim, keep) == n


@pytest.mark.parametrize("effort,N,K", [
    (0.25, 512 * 512, 65536), (0.1, 100, 10), (0.5, 3, 2), (0.5, 1, 1),
    (1.0, 4096 * 14336, 4096 * 14336), (0.01, 12, 0), (1.0 / 3.0, 12, 4),
])
def test_effort_K(effort, N, K):
    # llround of the double product; fl32(0.1) * 100 = 10.0000001 -> 10; 1.5 -> 2
    assert O.effort_K(effort, N, 1) == K


def test_probe_layout_closed_forms():
    r, w = O.probe_layout(16)
    assert list(r) == list(range(16)) and list(w) == [1] * 16
    r, w = O.probe_layout(4096)
    assert list(r) == [256 * k + 128 for k in range(16)] and list(w) == [256] * 16
    r, w = O.probe_layout(32)
    assert list(r) == [2 * k + 1 for k in range(16)] and list(w) == [2] * 16
    r, w = O.probe_layout(10)
    assert list(w) == [0, 1, 0, 1, 1, 0, 1, 1, 0, 1, 0, 1, 1, 0, 1, 1]
    assert [x for x in r if x >= 0] == [0, 1, 2, 3, 4, 5, 6, 7, 8, 9]
    for n in (1, 7, 100, 14336, 10752):
        r, w = O.probe_layout(n)
        assert w.sum() == n and np.all(r[w > 0] < n) and np.all(np.diff(r[w > 0]) > 0)


# ---------------------------------------------------------------- sort pins
def test_sort_rows_ties_and_signs():
    W = f16bits([[0.5, -1.0, 1.0, 0.25, -0.5]])
    idx, val, mag = O.sort_matrix_rows(W)
    assert list(idx[0]) == [1, 2, 0, 4, 3]
    assert list(val[0]) == [-1.0, 1.0, 0.5, -0.5, 0.25]


def test_keep_tie_break_lower_column_kept():
    prep = O.Prepared(f16bits([[1.0, -1.0, 1.0, 0.5]]), keep_fraction=0.5)
    assert prep.n == 2 and list(np.nonzero(prep.kept[0])[0]) == [0, 1]


def test_sort_rows_against_python_sorted():
    rng = np.random.default_rng(5)
    W = (rng.integers(-6, 7, size=(6, 23)) * 0.125).astype(np.float16)
    idx, _, _ = O.sort_matrix_rows(W.view(np.uint16))
    for i in range(W.shape[0]):
        ref = sorted(range(W.shape[1]), key=lambda j: (-abs(float(W[i, j])), j))
        assert list(idx[i]) == ref


# ---------------------------------------------------------------- fp32 chart
def test_chart_single_rounding_rne():
    # (1 + 2^-23) * (1 + 2^-10) = 1 + 2^-10 + 2^-23 + 2^-33 -> RNE drops 2^-33
    v = np.array([np.float32(1.0) + np.float32(2.0 ** -23)], np.float32)
    p = np.array([[1.0 + 2.0 ** -10] + [0.0] * 15])
    x = O.cutoff_chart(v, p)
    assert x.dtype == np.float32 and float(x[0, 0]) == 1.0 + 2.0 ** -10 + 2.0 ** -23


def test_chart_keeps_subnormal_products():
    v = np.array([2.0 ** -110], np.float32)
    p = np.array([[2.0 ** -24] + [0.0] * 15])
    assert float(O.cutoff_chart(v, p)[0, 0]) == 2.0 ** -134


# ---------------------------------------------------------------- topK pins
def brute_cutoff(chart, weights, K):
    """max{x : sum of weights of entries >= x is >= K} by enumeration."""
    vals = sorted(set(float(x) for x in chart.reshape(-1)))
    best = None
    for x in vals:
        tot = sum(int(weights[k]) for (i, k), y in np.ndenumerate(chart) if float(y) >= x)
        if tot >= K:
            best = x if best is None or x > best else best
    return best


def test_topk_hand_examples():
    ch = np.array([[4, 3], [2, 1]], np.float32)
    w = np.array([1, 1])
    assert [float(O.top_k_cutoff(ch, w, K, 4)) for K in (1, 2, 3)] == [4.0, 3.0, 2.0]
    assert float(O.top_k_cutoff(ch, w, 4, 4)) == 0.0
    assert float(O.top_k_cutoff(ch, w, 0, 4)) == math.inf
    w2 = np.array([2, 1])
    assert [float(O.top_k_cutoff(ch, w2, K, 6)) for K in (1, 2, 3, 4, 5)] == [4, 4, 3, 2, 2]
    tie = np.array([[2, 2], [2, 1]], np.float32)
    assert float(O.top_k_cutoff(tie, w, 1, 4)) == 2.0
    assert float(O.top_k_cutoff(tie, w, 3, 4)) == 2.0


def test_topk_against_enumeration():
    rng = np.random.default_rng(11)
    for trial in range(30):
        I, P = rng.integers(1, 6), rng.integers(1, 5)
        chart = (rng.integers(0, 6, size=(I, P)) * 0.5).astype(np.float32)
        weights = rng.integers(0, 4, size=P)
        total = int(weights.sum()) * I
        for K in range(1, total):
            assert float(O.top_k_cutoff(chart, weights, K, total)) == brute_cutoff(chart, weights, K)


# ------------------------------------------------------------- golden example
def load_golden():
    with open(os.path.join(GOLDEN, "hand_3x4.json")) as f:
        return json.load(f)


@pytest.mark.parametrize("case", load_golden()["cases"], ids=lambda c: f"e{c['effort']}_k{c['keep']}")
def test_golden_hand_example(case):
    g = load_golden()
    prep = O.Prepared(f16bits(g["W"]), case["keep"])
    r = O.effort_gemv(prep, np.array(g["v"], np.float32), case["effort"])
    c = math.inf if case["c"] == "inf" else case["c"]
    assert r.K == case["K"] and float(r.c) == c and r.count == case["count"]
    assert list(r.L) == case["L"] and list(r.out) == case["out"]


# ------------------------------------------------------------- method pins
def small_problem(seed, I=24, Od=40, dist="normal"):
    rng = np.random.default_rng(seed)
    W = (rng.standard_normal((I, Od)) * 0.02).astype(np.float16)
    if dist == "t3":
        v = (rng.standard_t(3, I) / math.sqrt(3)).astype(np.float32)
    else:
        v = rng.standard_normal(I).astype(np.float32)
    return W.view(np.uint16), v


def exact_dense(W_bits, v):
    """W^T v with exact rational arithmetic, rounded once to float64."""
    W = W_bits.view(np.float16)
    out = []
    for j in range(W.shape[1]):
        s = sum(Fraction(float(v[i])) * Fraction(float(W[i, j])) for i in range(W.shape[0]))
        out.append(float(s))
    return np.array(out)


def test_effort_one_is_dense_gemv():
    W, v = small_problem(1, 12, 20)
    r = O.effort_gemv(O.Prepared(W, 1.0), v, 1.0)
    assert r.count == W.size and float(r.c) == 0.0
    np.testing.assert_allclose(r.out, exact_dense(W, v), rtol=1e-13, atol=1e-15)


def test_effort_one_non_square_orientation():
    # out has out_dim entries and row i multiplies v[i]: a transposed operand fails here
    W, v = small_problem(2, 7, 13)
    r = O.effort_gemv(O.Prepared(W, 1.0), v, 1.0)
    assert r.out.shape == (13,)
    np.testing.assert_allclose(r.out, exact_dense(W, v), rtol=1e-13, atol=1e-15)


@pytest.mark.parametrize("seed,I,Od", [(4, 11, 17), (5, 1, 9), (6, 23, 3)])
def test_dense_gemv_against_exact_rational(seed, I, Od):
    # the dense baseline W^T v of the method, on non-square shapes (a
    # transposed operand or a dropped row fails), fp32 and fp16 v
    W, v = small_problem(seed, I, Od)
    np.testing.assert_allclose(O.dense_gemv(W, v), exact_dense(W, v), rtol=1e-13, atol=1e-15)
    v16 = v.astype(np.float16)
    np.testing.assert_allclose(O.dense_gemv(W, v16), exact_dense(W, v16.astype(np.float32)), rtol=1e-13, atol=1e-15)


def test_keep_closed_form_effort_one():
    W, v = small_problem(3, 9, 16)
    keep = 0.75
    n = O.kept_count(16, keep)
    Wf = W.view(np.float16)
    ref = [Fraction(0)] * 16
    for i in range(9):
        order = sorted(range(16), key=lambda j: (-abs(float(Wf[i, j])), j))[:n]
        for j in order:
            ref[j] += Fraction(float(v[i])) * Fraction(float(Wf[i, j]))
    r = O.effort_gemv(O.Prepared(W, keep), v, 1.0)
    assert r.count == 9 * n
    np.testing.assert_allclose(r.out, [float(x) for x in ref], rtol=1e-13, atol=1e-15)


def brute_selection(W_bits, v, keep, c):
    """Used set for cutoff c by enumerating every product with Python floats."""
    Wf = W_bits.view(np.float16)
    I, Od = Wf.shape
    n = O.kept_count(Od, keep)
    S = set()
    for i in range(I):
        order = sorted(range(Od), key=lambda j: (-abs(float(Wf[i, j])), j))[:n]
        for j in order:
            prod = np.float32(abs(float(v[i]))) * np.float32(abs(float(Wf[i, j])))
            if prod >= c:
                S.add((i, j))
    return S


@pytest.mark.parametrize("seed,keep,effort", [(4, 1.0, 0.25), (5, 1.0, 0.15), (6, 0.75, 0.4), (7, 1.0, 0.5)])
def test_brute_force_product_set(seed, keep, effort):
    W, v = small_problem(seed, 16, 32)
    prep = O.Prepared(W, keep)
    r = O.effort_gemv(prep, v, effort)
    S = brute_selection(W, v, keep, np.float32(r.c))
    assert set(zip(*np.nonzero(r.mask))) == S
    # the used set is the top-|S| of all kept products, and the next one is below c
    Wf = W.view(np.float16)
    prods = sorted(((np.float32(abs(float(v[i]))) * np.float32(abs(float(Wf[i, j]))), (i, j))
                    for i in range(16) for j in range(32) if prep.kept[i, j]), reverse=True)
    top = prods[: len(S)]
    assert all(p >= r.c for p, _ in top)
    if len(S) < len(prods):
        assert prods[len(S)][0] < r.c


def test_cutoff_is_a_chart_value_and_meets_K():
    W, v = small_problem(8, 32, 64)
    prep = O.Prepared(W, 1.0)
    for e in (0.12, 0.25, 0.4):
        r = O.effort_gemv(prep, v, e)
        chart = O.cutoff_chart(v, prep.probes)
        wts = np.broadcast_to(prep.weights, chart.shape)
        assert np.any(chart == r.c)
        assert wts[chart >= r.c].sum() >= r.K > wts[chart > r.c].sum()


def test_nested_and_monotone():
    W, v = small_problem(9, 48, 64, "t3")
    prep = O.Prepared(W, 1.0)
    efforts = [0.15, 0.25, 0.4, 0.5, 1.0]
    rs = [O.effort_gemv(prep, v, e) for e in efforts]
    for a, b in zip(rs, rs[1:]):
        assert a.c >= b.c
        assert np.all(b.mask[a.mask])  # S(e1) subset of S(e2)
        assert a.count <= b.count


def test_row_prefix_property():
    W, v = small_problem(10, 40, 48, "t3")
    prep = O.Prepared(W, 0.75)
    for e in (0.15, 0.3, 0.6):
        r = O.effort_gemv(prep, v, e)
        L = O.row_prefix_lengths(prep, r.mask)
        assert np.array_equal(L, r.L)


def test_dropped_weights_never_used():
    W, v = small_problem(12, 20, 30)
    prep = O.Prepared(W, 0.6)
    for e in (0.1, 0.5, 1.0):
        r = O.effort_gemv(prep, v, e)
        assert not np.any(r.mask & ~prep.kept)


@pytest.mark.parametrize("shape,dist", [((256, 512), "normal"), ((512, 256), "t3")])
def test_count_scales_with_effort(shape, dist):
    W, v = small_problem(13, shape[0], shape[1], dist)
    prep = O.Prepared(W, 1.0)
    for e in (0.12, 0.15, 0.25, 0.4, 0.5):
        r = O.effort_gemv(prep, v, e)
        assert abs(r.count - r.K) <= 0.01 * r.K + shape[1], (e, r.count, r.K)


def test_effort_and_input_validation():
    W, v = small_problem(14, 4, 8)
    prep = O.Prepared(W, 1.0)
    for bad in (0.0, -0.1, 1.5, float("nan")):
        with pytest.raises(ValueError):
            O.effort_gemv(prep, v, bad)
    with pytest.raises(ValueError):
        O.effort_gemv(prep, np.array([1, np.inf, 0, 0], np.float32), 0.5)
    with pytest.raises(ValueError):
        O.Prepared(np.array([[0x7C00, 0]], np.uint16))
    with pytest.raises(ValueError):
        O.Prepared(W, 0.0)


def test_zero_vector_entries_and_fp16_v():
    W, v = small_problem(15, 16, 16)
    v[::3] = 0.0
    prep = O.Prepared(W, 1.0)
    r = O.effort_gemv(prep, v, 0.3)
    assert not np.any(r.mask[::3])  # zero rows only enter when c == 0
    r16 = O.effort_gemv(prep, v.astype(np.float16), 0.3)
    v16 = v.astype(np.float16).astype(np.float32)
    r32 = O.effort_gemv(prep, v16, 0.3)
    assert r16.c == r32.c and np.array_equal(r16.mask, r32.mask)
