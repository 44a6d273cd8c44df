"""Per-matrix effort schedules for the decode chain (host logic, CPU only).

The pages treat effort as a setting that may change per layer, per matrix and
per token (the author's replies in Hacker News item 40067677).  The library
takes the effort on every call; `bench.effort_for` turns a schedule into the
effort of one matvec and `bench.chain_token` passes it through.  The GPU side
of a scheduled chain is checked against the oracle in test_gpu_chain.py.
"""
import os
import sys

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def test_number_is_one_effort_for_every_matvec():
    assert bench.effort_for(0.25, 0, "q") == 0.25
    assert bench.effort_for(1, 31, "w2") == 1.0


def test_mapping_by_name_and_by_layer_and_name():
    sched = {"q": 0.5, "w2": 0.2, (3, "q"): 0.1}
    assert bench.effort_for(sched, 0, "q") == 0.5
    assert bench.effort_for(sched, 3, "q") == 0.1  # the (layer, name) entry wins
    assert bench.effort_for(sched, 3, "w2") == 0.2
    with pytest.raises(KeyError):
        bench.effort_for(sched, 0, "k")


def test_callable_and_range_check():
    assert bench.effort_for(lambda l, n: 0.1 * l, 2, "v") == pytest.approx(0.2)
    for bad in (-0.01, 1.5, float("nan")):
        with pytest.raises(ValueError):
            bench.effort_for(bad, 0, "q")


def test_equalizer_keeps_the_weighted_mean_near_a_quarter():
    dims = (4096, 1024, 14336)
    params = {n: dims[a] * dims[b] for n, a, b in bench.CHAIN_MATS}
    mean = sum(bench.CHAIN_EQUALIZER[n] * params[n] for n in params) / sum(params.values())
    assert set(bench.CHAIN_EQUALIZER) == set(params)
    assert abs(mean - 0.25) < 0.005


class _FakeMatrix:
    """Stands in for a prepared matrix: records the effort of each call."""

    def __init__(self, out_dim, log, key):
        self.out_dim, self.log, self.key = out_dim, log, key

    def gemv(self, x, effort):
        self.log.append((self.key, effort))
        return torch.ones(self.out_dim)


def test_chain_token_passes_each_matvecs_scheduled_effort():
    dims = (8, 2, 16)
    log = []
    mats = [{n: _FakeMatrix(dims[b], log, (l, n)) for n, a, b in bench.CHAIN_MATS} for l in range(3)]
    sched = lambda l, n: round(0.1 * l + 0.01 * [m for m, _, _ in bench.CHAIN_MATS].index(n), 2)
    x = bench.chain_token(None, mats, torch.ones(dims[0]), sched)
    assert x.shape == (dims[0],)
    assert [k for k, _ in log] == [(l, n) for l in range(3) for n in ("q", "k", "v", "o", "w1", "w3", "w2")]
    for (l, n), e in log:
        assert e == sched(l, n)
