"""Pins of the Q8 oracle against things other than itself.

* With power-of-two scales every Q8 weight is a binary16 value, and the Q8
  oracle must give the pinned fp16 oracle's c, used set and out bit for bit.
* With arbitrary scales, on tiny inputs: the chart recomputed from Python's
  own sort of each row, the cutoff by enumeration, the used set from every
  product, and out as an exact rational sum.
* effort 1 against the exact rational W^T v; invariances that the
  arithmetic fixes (an exact power-of-two rescaling of s_i against v_i, the
  sign of s_i); a zero scale; argument checks.
"""
import math
from fractions import Fraction

import numpy as np
import pytest

from dynamic_approximate_gemv_b200 import inputs
from oracle import effort_oracle as F
from oracle import effort_q8_oracle as Q
from tests.test_oracle_pins import brute_cutoff


def q8_problem(seed, I, Od, pow2=False, dist="normal"):
    rng = np.random.default_rng(seed)
    q = rng.integers(-127, 128, size=(I, Od)).astype(np.int8)
    q[rng.random((I, Od)) < 0.1] = 0  # some exact zeros and ties
    sign = np.where(rng.random(I) < 0.3, -1.0, 1.0)  # some negative scales
    if pow2:
        s = (sign * 2.0 ** -rng.integers(7, 13, size=I)).astype(np.float16)
    else:
        s = (sign * rng.uniform(1e-4, 1e-3, size=I)).astype(np.float16)
    if dist == "t3":
        v = (rng.standard_t(3, I) / math.sqrt(3)).astype(np.float32)
    else:
        v = rng.standard_normal(I).astype(np.float32)
    return q, s.view(np.uint16), v


def exact_w(q, s_bits):
    s = s_bits.view(np.float16)
    return [[Fraction(float(s[i])) * int(q[i, j]) for j in range(q.shape[1])] for i in range(q.shape[0])]


# ------------------------------------------------- reduction to the fp16 oracle
@pytest.mark.parametrize("seed,I,Od,keep,effort,dist", [
    (1, 24, 40, 1.0, 0.25, "normal"), (2, 31, 57, 0.75, 0.4, "t3"), (3, 9, 130, 1.0, 0.12, "t3"),
    (4, 64, 64, 0.5, 0.5, "normal"), (5, 17, 23, 1.0, 1.0, "normal")])
def test_power_of_two_scales_reduce_to_fp16_oracle(seed, I, Od, keep, effort, dist):
    q, s_bits, v = q8_problem(seed, I, Od, pow2=True, dist=dist)
    W = Q.q8_to_float64(q, s_bits)
    W16 = W.astype(np.float16)
    assert np.array_equal(W16.astype(np.float64), W), "the weights must be binary16 values here"
    a = Q.effort_gemv(Q.PreparedQ8(q, s_bits, keep), v, effort)
    b = F.effort_gemv(F.Prepared(W16.view(np.uint16), keep), v, effort)
    assert a.K == b.K and np.float32(a.c).view(np.uint32) == np.float32(b.c).view(np.uint32)
    assert np.array_equal(a.mask, b.mask)
    assert np.array_equal(a.out, b.out)


# ------------------------------------------------------------- brute force
@pytest.mark.parametrize("seed,keep,effort", [(11, 1.0, 0.25), (12, 0.75, 0.4), (13, 0.5, 0.15), (14, 1.0, 0.6)])
def test_brute_force_arbitrary_scales(seed, keep, effort):
    I, Od = 6, 9
    q, s_bits, v = q8_problem(seed, I, Od)
    Wx = exact_w(q, s_bits)
    n = F.kept_count(Od, keep)
    ranks, weights = F.probe_layout(n)
    # the chart from Python's own sort of each row (|w| descending, lower column first)
    chart = np.zeros((I, 16), np.float32)
    kept = set()
    for i in range(I):
        order = sorted(range(Od), key=lambda j: (-abs(Wx[i][j]), j))
        kept |= {(i, j) for j in order[:n]}
        for k in range(16):
            if weights[k] > 0:
                p = np.float32(float(abs(Wx[i][order[ranks[k]]])))
                chart[i, k] = np.float32(abs(v[i])) * p
    K = F.effort_K(effort, I, Od)
    c_ref = 0.0 if K >= I * n else brute_cutoff(chart, weights, K)
    r = Q.effort_gemv(Q.PreparedQ8(q, s_bits, keep), v, effort)
    assert float(r.c) == c_ref
    # every product against the cutoff
    used = {(i, j) for (i, j) in kept
            if np.float32(abs(v[i])) * np.float32(float(abs(Wx[i][j]))) >= np.float32(c_ref)}
    assert {(int(i), int(j)) for i, j in zip(*np.nonzero(r.mask))} == used
    ref = [sum((Fraction(float(v[i])) * Wx[i][j] for i in range(I) if (i, j) in used), Fraction(0))
           for j in range(Od)]
    np.testing.assert_allclose(r.out, [float(x) for x in ref], rtol=1e-13, atol=1e-15)


def test_effort_one_is_exact_dense():
    q, s_bits, v = q8_problem(21, 13, 19)
    Wx = exact_w(q, s_bits)
    r = Q.effort_gemv(Q.PreparedQ8(q, s_bits, 1.0), v, 1.0)
    ref = [float(sum(Fraction(float(v[i])) * Wx[i][j] for i in range(13))) for j in range(19)]
    assert r.count == 13 * 19 and float(r.c) == 0.0
    np.testing.assert_allclose(r.out, ref, rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(Q.dense_gemv(q, s_bits, v), ref, rtol=1e-13, atol=1e-15)


# ------------------------------------------------------------- invariances
def test_power_of_two_rescaling_of_a_row_changes_nothing():
    # w_ij * 2 and v_i / 2: every product |v_i||w_ij| is the same number
    q, s_bits, v = q8_problem(31, 20, 33, dist="t3")
    s = s_bits.view(np.float16).copy()
    s2, v2 = s.copy(), v.copy()
    s2[[1, 5, 9]] *= np.float16(2.0)
    v2[[1, 5, 9]] /= np.float32(2.0)
    a = Q.effort_gemv(Q.PreparedQ8(q, s.view(np.uint16), 1.0), v, 0.3)
    b = Q.effort_gemv(Q.PreparedQ8(q, s2.view(np.uint16), 1.0), v2, 0.3)
    assert float(a.c) == float(b.c) and np.array_equal(a.mask, b.mask)
    np.testing.assert_allclose(a.out, b.out, rtol=1e-13, atol=1e-15)


def test_sign_of_a_scale_flips_its_row_only():
    q, s_bits, v = q8_problem(32, 12, 25)
    r4 = int(np.argmax(np.abs(v)))  # the row with the largest |v_i| has used entries
    s = s_bits.view(np.float16).copy()
    sn = s.copy()
    sn[r4] = -sn[r4]
    a = Q.effort_gemv(Q.PreparedQ8(q, s.view(np.uint16), 1.0), v, 0.35)
    b = Q.effort_gemv(Q.PreparedQ8(q, sn.view(np.uint16), 1.0), v, 0.35)
    assert float(a.c) == float(b.c) and np.array_equal(a.mask, b.mask) and a.mask[r4].any()
    wx = exact_w(q, s.view(np.uint16))[r4]
    row = np.array([float(Fraction(float(v[r4])) * wx[j]) if a.mask[r4, j] else 0.0 for j in range(25)])
    np.testing.assert_allclose(b.out, a.out - 2 * row, rtol=1e-12, atol=1e-15)


def test_selection_rounds_the_product_once():
    # fl32(|v_i| |w_ij|) with |w_ij| = |s_i q_ij| exact: one rounding of the
    # exact product (exact in float64: 24 + 11 + 8 bits), not two.  The
    # cutoff is set to a product where rounding |v_i| s_i first would land
    # one unit lower.
    for trial in range(200):
        q, s_bits, v = q8_problem(1000 + trial, 4, 8)
        s = s_bits.view(np.float16).astype(np.float64)
        exact = np.abs(v.astype(np.float64))[:, None] * np.abs(s)[:, None] * np.abs(q.astype(np.float64))
        once = exact.astype(np.float32)
        twice = ((np.abs(v) * np.abs(s).astype(np.float32)).astype(np.float32)[:, None] *
                 np.abs(q.astype(np.float32))).astype(np.float32)
        diff = np.argwhere(twice < once)
        if len(diff):
            i, j = diff[0]
            c = once[i, j]
            prep = Q.PreparedQ8(q, s_bits, 1.0)
            m = Q.selected_mask(prep, v, c)
            assert np.array_equal(m, once >= c)
            assert m[i, j]
            return
    pytest.fail("no product found where the two roundings differ")


def test_zero_scale_row_orders_by_column():
    q, s_bits, v = q8_problem(33, 5, 12)
    s = s_bits.view(np.float16).copy()
    s[2] = np.float16(0.0)
    prep = Q.PreparedQ8(q, s.view(np.uint16), 0.5)
    assert list(prep.W_idx[2]) == list(range(12))  # all |w| = 0: lower column first
    assert prep.kept[2].tolist() == [True] * 6 + [False] * 6
    r = Q.effort_gemv(prep, v, 1.0)
    assert np.all(r.mask[2] == prep.kept[2])  # c = 0: every kept entry is used, adding +0


def test_generated_q8_weights_dequantise_near_the_draw():
    q, s = inputs.q8_weights(16, 300, 5)
    w = inputs.weights(16, 300, 5).astype(np.float64)  # the same draw, rounded to fp16
    W = Q.q8_to_float64(q, s.view(np.uint16))
    assert q.dtype == np.int8 and np.abs(q).max() <= 127
    assert np.max(np.abs(W - w)) <= 0.6 * float(s.astype(np.float64).max()) + 1e-4


def test_argument_checks():
    q, s_bits, v = q8_problem(34, 4, 6)
    with pytest.raises(ValueError):
        Q.PreparedQ8(q.astype(np.int16), s_bits)
    with pytest.raises(ValueError):
        Q.PreparedQ8(q, s_bits[:3])
    bad = s_bits.copy()
    bad[1] = 0x7C00  # +inf
    with pytest.raises(ValueError):
        Q.PreparedQ8(q, bad)
    with pytest.raises(ValueError):
        Q.effort_gemv(Q.PreparedQ8(q, s_bits), v, 0.0)
