"""Planted mistakes in the Q8 oracle must be caught by its pins.

Each case patches one plausible error into the Q8 oracle (on the CPU) and
checks that the pins of test_oracle_q8_pins.py fail on the patched oracle.
"""
import numpy as np
import pytest

from oracle import effort_oracle as F
from oracle import effort_q8_oracle as Q
from tests import test_oracle_q8_pins as pins


def run_pin_suite():
    checks = [
        lambda: pins.test_power_of_two_scales_reduce_to_fp16_oracle(1, 24, 40, 1.0, 0.25, "normal"),
        lambda: pins.test_power_of_two_scales_reduce_to_fp16_oracle(2, 31, 57, 0.75, 0.4, "t3"),
        lambda: pins.test_brute_force_arbitrary_scales(11, 1.0, 0.25),
        lambda: pins.test_brute_force_arbitrary_scales(12, 0.75, 0.4),
        lambda: pins.test_brute_force_arbitrary_scales(13, 0.5, 0.15),
        pins.test_effort_one_is_exact_dense,
        pins.test_power_of_two_rescaling_of_a_row_changes_nothing,
        pins.test_sign_of_a_scale_flips_its_row_only,
        pins.test_zero_scale_row_orders_by_column,
        pins.test_selection_rounds_the_product_once,
    ]
    for chk in checks:
        try:
            chk()
        except (AssertionError, ValueError, IndexError):
            return False
    return True


def mut_product_rounded_twice(mp):
    # fl32(fl32(|v| s) |q|) instead of fl32(|v| |w|)
    def bad(prep, v32, c):
        s = F.fp16_bits_to_float64(prep.s_bits).astype(np.float32)
        a = (np.abs(v32.astype(np.float32)) * np.abs(s)).astype(np.float32)[:, None]
        prod = (a * np.abs(prep.q.astype(np.float32))).astype(np.float32)
        return prep.kept & (prod >= np.float32(c))
    mp.setattr(Q, "selected_mask", bad)


def mut_scale_sign_dropped(mp):
    def bad(q, s_bits):
        return np.abs(F.fp16_bits_to_float64(np.asarray(s_bits, dtype=np.uint16)))[:, None] * q.astype(np.float64)
    mp.setattr(Q, "q8_to_float64", bad)


def mut_strict_compare(mp):
    def bad(prep, v32, c):
        a = np.abs(v32.astype(np.float32))[:, None]
        return prep.kept & ((a * np.abs(prep.W).astype(np.float32)).astype(np.float32) > np.float32(c))
    mp.setattr(Q, "selected_mask", bad)


def mut_multiply_without_scale(mp):
    def bad(prep, v32, mask):
        contrib = np.where(mask, v32.astype(np.float64)[:, None] * prep.q.astype(np.float64), 0.0)
        return contrib.sum(axis=0)
    mp.setattr(Q, "approx_mul", bad)


def mut_order_by_q_descending_ties_high(mp):
    # order by |q| with ties to the higher column (wrong for ties and zero scales)
    orig = Q.PreparedQ8.__init__

    def bad(self, q, s_bits, keep_fraction=1.0, P=Q.P_PROBES):
        orig(self, q, s_bits, keep_fraction, P)
        mag = np.abs(self.q.astype(np.int64))
        idx = np.argsort(-mag[:, ::-1], axis=1, kind="stable")
        self.W_idx = self.q.shape[1] - 1 - idx
        self.W_val = np.take_along_axis(self.W, self.W_idx, axis=1)
        self.W_mag = np.abs(self.W_val)
        self.probes, self.weights = F.get_probes(self.W_mag, self.n, P)
        self.kept = np.zeros(self.q.shape, dtype=bool)
        np.put_along_axis(self.kept, self.W_idx[:, : self.n], True, axis=1)
    mp.setattr(Q.PreparedQ8, "__init__", bad)


def mut_probe_from_q(mp):
    # probes taken as |q| (scale forgotten in the chart)
    orig = Q.PreparedQ8.__init__

    def bad(self, q, s_bits, keep_fraction=1.0, P=Q.P_PROBES):
        orig(self, q, s_bits, keep_fraction, P)
        qmag = np.take_along_axis(np.abs(self.q.astype(np.float64)), self.W_idx, axis=1)
        self.probes, self.weights = F.get_probes(qmag, self.n, P)
    mp.setattr(Q.PreparedQ8, "__init__", bad)


MUTATIONS = [mut_product_rounded_twice, mut_scale_sign_dropped, mut_strict_compare, mut_multiply_without_scale,
             mut_order_by_q_descending_ties_high, mut_probe_from_q]


def test_pins_pass_on_the_oracle():
    assert run_pin_suite()


@pytest.mark.parametrize("mutation", MUTATIONS, ids=lambda m: m.__name__)
def test_planted_mistake_is_caught(mutation, monkeypatch):
    mutation(monkeypatch)
    assert not run_pin_suite(), f"{mutation.__name__} went unnoticed"
