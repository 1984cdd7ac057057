"""The split-K slice count of the tensor-core GEMM (host code, no GPU): the
launch's units (output tiles x K slices) run on persistent CTAs or CTA pairs,
each taking units `workers` apart, so a round that only a few workers reach
costs as much as a full one."""

import ctypes
import itertools

import pytest

from rnn_joint_network_02_b200 import frnnt


def _auto():
    f = frnnt.lib().frnnt_test_auto_splits
    f.argtypes = [ctypes.c_int] * 3
    f.restype = ctypes.c_int
    return f


def _rounds_and_per(mn, workers, kblocks, s):
    per = -(-kblocks // s)
    real = -(-kblocks // per)
    return -(-(mn * real) // workers), per, real


@pytest.mark.parametrize("mn,workers,kblocks,want", [
    (12, 74, 4624, 6),      # medium dW_o on CTA pairs: one full round (13 slices left 8 pairs a third round)
    (12, 74, 40000, 6),     # long dW_o
    (64, 74, 4994, 8),      # large dW_o: 512 units in 7 rounds instead of 64 on 74 pairs
    (20, 148, 100, 7),      # dW_f of medium on one-CTA tiles
    (3, 148, 4624, 49),     # the duration head's 64-row GEMM: 147 units in one round
    (16, 74, 31, 4),        # a short K keeps its slices long
])
def test_slice_counts_of_the_measured_shapes(mn, workers, kblocks, want):
    assert _auto()(mn, workers, kblocks) == want


def test_degenerate_inputs_take_one_slice():
    auto = _auto()
    for args in [(0, 148, 100), (5, 0, 100), (5, 148, 0), (5, 148, 1)]:
        assert auto(*args) == 1, args


def test_the_choice_fills_the_workers_no_worse_than_any_other_slice_count():
    """Against every slice count that rounding to whole K blocks can produce,
    the chosen one has the smallest modelled time, rounds x (K blocks per unit
    + 64), and at that time the fewest slices."""
    auto = _auto()
    for mn, workers, kblocks in itertools.product([1, 3, 12, 20, 64, 150], [74, 148], [2, 31, 100, 777, 4624]):
        s = auto(mn, workers, kblocks)
        assert 1 <= s <= kblocks
        r, per, real = _rounds_and_per(mn, workers, kblocks, s)
        assert real == s
        cost = r * (per + 64)
        for t in range(1, kblocks + 1):
            rt, pt, realt = _rounds_and_per(mn, workers, kblocks, t)
            if realt != t:
                continue
            ct = rt * (pt + 64)
            assert cost <= ct, (mn, workers, kblocks, s, t)
            if ct == cost:
                assert s <= t, (mn, workers, kblocks, s, t)
            if rt > 16:
                break
