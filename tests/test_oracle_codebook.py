"""Pins of the oracle's NF4 codebook against what the pages print and what
the mathematics fixes ("第 04 篇：QLoRA 原理" §3.3, §4.2, §4.3)."""
import math

import numpy as np
import pytest
from scipy import stats

import oracle
from conftest import read_golden


def printed_levels():
    vals = [float(v) for v in read_golden("nf4_levels.txt")]
    assert len(vals) == 16
    return np.array(vals, np.float64)


def test_norm_ppf_matches_library():
    ps = np.concatenate([np.linspace(0.001, 0.999, 211), [0.5, 0.9677083333, 1e-9, 1 - 1e-9]])
    for p in ps:
        ref = stats.norm.ppf(p)
        got = oracle.norm_ppf(p)
        assert abs(got - ref) <= 1e-12 * max(1.0, abs(ref)), (p, got, ref)


def test_runtime_levels_are_the_printed_table():
    got = oracle.levels()
    assert np.array_equal(got, printed_levels().astype(np.float32))


def test_built_codebook_reproduces_printed_table():
    built = oracle.build_codebook()
    err = np.max(np.abs(built - printed_levels()))
    # the table has 7 decimals; the quantile construction lands within 2e-7
    assert err <= 2e-7, err


def test_codebook_structure():
    c = printed_levels()
    built = oracle.build_codebook()
    for table in (c, built):
        assert table[7] == 0.0                     # exact zero
        assert table[0] == -1.0 and table[15] == 1.0
        assert np.all(np.diff(table) > 0)          # strictly increasing
        assert np.sum(table < 0) == 7 and np.sum(table > 0) == 8
        # not mirror-symmetric: the positive half has one more level
        assert not np.allclose(np.sort(-table[table < 0]), table[table > 0][:7])
    gaps = np.diff(c)
    # denser near zero than in the tails (both sides)
    assert gaps[7] < gaps[14] and gaps[6] < gaps[0]


def test_built_levels_have_equal_probability_bins():
    """Each half of the built codebook sits on equally spaced probabilities of
    the standard normal (closed form: Phi of the un-normalised levels)."""
    built = oracle.build_codebook()
    delta = 1 - 0.5 * (1 / 32 + 1 / 30)
    vmax = stats.norm.ppf(delta)
    pos = built[built > 0] * vmax
    neg = -built[built < 0] * vmax
    p_pos = np.sort(stats.norm.cdf(pos))
    p_neg = np.sort(stats.norm.cdf(neg))
    assert np.allclose(np.diff(np.concatenate([[0.5], p_pos])), (delta - 0.5) / 8, atol=1e-12)
    assert np.allclose(np.diff(np.concatenate([[0.5], p_neg])), (delta - 0.5) / 7, atol=1e-12)


def test_midpoints_separate_neighbours():
    c = oracle.levels()
    m = oracle.midpoints()
    assert m.dtype == np.float32 and m.size == 15
    assert np.all(m > c[:-1]) and np.all(m < c[1:])
    # within half an ulp of the exact mid-value
    exact = (c[:-1].astype(np.float64) + c[1:].astype(np.float64)) / 2
    assert np.all(np.abs(m - exact) <= np.spacing(np.abs(m).astype(np.float32)))
