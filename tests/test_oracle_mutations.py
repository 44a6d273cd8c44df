"""Planted mistakes in the oracle must be caught by its pins.

Each case patches one plausible error into the CPU oracle (a flipped
comparison, a lost sign, a wrong rank, a transposed operand, ...) and checks
that the pin suite of test_oracle_pins.py fails on the patched oracle.  The
mistakes are planted in the oracle only, on the CPU.
"""
import math

import numpy as np
import pytest

from oracle import effort_oracle as O
from tests import test_oracle_pins as pins


def run_pin_suite():
    """Run a representative set of pins; True iff every one passes."""
    checks = [
        lambda: [pins.test_golden_hand_example(c) for c in pins.load_golden()["cases"]],
        pins.test_effort_one_is_dense_gemv,
        pins.test_effort_one_non_square_orientation,
        pins.test_keep_closed_form_effort_one,
        lambda: pins.test_brute_force_product_set(4, 1.0, 0.25),
        lambda: pins.test_brute_force_product_set(6, 0.75, 0.4),
        pins.test_probe_layout_closed_forms,
        pins.test_topk_hand_examples,
        pins.test_topk_against_enumeration,
        pins.test_sort_rows_ties_and_signs,
        pins.test_keep_tie_break_lower_column_kept,
        pins.test_chart_single_rounding_rne,
        pins.test_chart_keeps_subnormal_products,
        pins.test_fp16_decoder_matches_numpy_on_all_patterns,
        pins.test_cutoff_is_a_chart_value_and_meets_K,
        lambda: [pins.test_effort_K(e, N, K) for e, N, K in
                 [(0.25, 512 * 512, 65536), (0.5, 3, 2), (0.5, 1, 1), (0.01, 12, 0)]],
        lambda: [pins.test_kept_count(o, k, n) for o, k, n in [(3, 0.5, 2), (1024, 0.8, 819), (10, 0.04, 0)]],
        pins.test_row_prefix_property,
        lambda: pins.test_count_scales_with_effort((256, 512), "normal"),
    ]
    for chk in checks:
        try:
            chk()
        except (AssertionError, ValueError, IndexError):
            return False
    return True


def mut_strict_compare(mp):
    def bad(prep, v32, c):
        a = np.abs(v32.astype(np.float32))[:, None]
        wabs = np.abs(O.fp16_bits_to_float64(prep.W_bits)).astype(np.float32)
        return prep.kept & ((a * wabs).astype(np.float32) > np.float32(c))
    mp.setattr(O, "selected_mask", bad)


def mut_ties_high_column_first(mp):
    def bad(W_bits):
        W_bits = np.asarray(W_bits, dtype=np.uint16)
        mag = O.fp16_magnitude_key(W_bits)
        Od = W_bits.shape[1]
        idx = np.argsort(-(mag * (Od + 1) + np.arange(Od)[None, :]), axis=1, kind="stable")
        vals = O.fp16_bits_to_float64(W_bits)
        val = np.take_along_axis(vals, idx, axis=1)
        return idx, val, np.abs(val)
    mp.setattr(O, "sort_matrix_rows", bad)


def mut_probe_at_segment_start(mp):
    def bad(n, P=O.P_PROBES):
        b = [(k * n) // P for k in range(P + 1)]
        w = [b[k] - b[k - 1] for k in range(1, P + 1)]
        r = [b[k - 1] if w[k - 1] > 0 else -1 for k in range(1, P + 1)]
        return np.array(r), np.array(w)
    mp.setattr(O, "probe_layout", bad)


def mut_lost_sign(mp):
    def bad(prep, v32, mask):
        W = O.fp16_bits_to_float64(prep.W_bits)
        return np.where(mask, np.abs(v32.astype(np.float64))[:, None] * W, 0.0).sum(axis=0)
    mp.setattr(O, "approx_mul", bad)


def mut_transposed(mp):
    # reduces over the wrong axis: one sum per input row instead of per output column
    def bad(prep, v32, mask):
        W = O.fp16_bits_to_float64(prep.W_bits)
        s = np.where(mask, v32.astype(np.float64)[:, None] * W, 0.0).sum(axis=1)
        out = np.zeros(prep.out_dim)
        m = min(s.size, prep.out_dim)
        out[:m] = s[:m]
        return out
    mp.setattr(O, "approx_mul", bad)


def mut_unweighted_topk(mp):
    orig = O.top_k_cutoff

    def bad(chart, weights, K, kept_total):
        return orig(chart, np.ones_like(weights), K, kept_total)
    mp.setattr(O, "top_k_cutoff", bad)


def mut_K_floor(mp):
    def bad(effort, in_dim, out_dim):
        return int(math.floor(float(np.float32(effort)) * in_dim * out_dim))
    mp.setattr(O, "effort_K", bad)


def mut_chart_double(mp):
    def bad(v32, probes):
        return np.abs(v32.astype(np.float64))[:, None] * probes
    mp.setattr(O, "cutoff_chart", bad)


def mut_keep_floor(mp):
    mp.setattr(O, "kept_count", lambda out_dim, keep: int(math.floor(float(np.float32(keep)) * out_dim)))


def mut_subnormal_decode(mp):
    orig = O.fp16_bits_to_float64

    def bad(bits):
        b = np.asarray(bits, dtype=np.uint16).astype(np.int64)
        out = orig(bits)
        expo = (b >> 10) & 0x1F
        frac = (b & 0x3FF).astype(np.float64)
        sign = np.where((b >> 15) & 1, -1.0, 1.0)
        return np.where(expo == 0, sign * (1.0 + frac / 1024.0) * 2.0 ** -15 * (frac > 0), out)
    mp.setattr(O, "fp16_bits_to_float64", bad)


def mut_off_by_one_kept(mp):
    orig = O.kept_count
    mp.setattr(O, "kept_count", lambda out_dim, keep: max(0, orig(out_dim, keep) - 1) if keep < 1 else orig(out_dim, keep))


def mut_drop_last_row(mp):
    def bad(prep, v32, mask):
        W = O.fp16_bits_to_float64(prep.W_bits)
        contrib = np.where(mask, v32.astype(np.float64)[:, None] * W, 0.0)
        return contrib[:-1].sum(axis=0)
    mp.setattr(O, "approx_mul", bad)


MUTATIONS = [mut_strict_compare, mut_ties_high_column_first, mut_probe_at_segment_start,
             mut_lost_sign, mut_transposed, mut_unweighted_topk, mut_K_floor, mut_chart_double,
             mut_keep_floor, mut_subnormal_decode, mut_off_by_one_kept, mut_drop_last_row]


def test_unmutated_oracle_passes_suite():
    assert run_pin_suite()


@pytest.mark.parametrize("mutate", MUTATIONS, ids=lambda f: f.__name__)
def test_planted_mistake_is_caught(mutate, monkeypatch):
    mutate(monkeypatch)
    assert not run_pin_suite(), f"pins did not catch {mutate.__name__}"
