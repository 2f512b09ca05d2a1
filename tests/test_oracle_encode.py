"""Pins of the oracle's first-level quantiser: blockwise absmax, nearest
level, nibble packing ("第 04 篇：QLoRA 原理" §2.1, §3.2, §3.4, §4.3)."""
import numpy as np
import pytest

import oracle
import workloads


def brute_force_codes(w, block=64):
    """Nearest level by exhaustive search in fp64, element by element."""
    c = oracle.levels().astype(np.float64)
    flat = np.asarray(w, np.float32).reshape(-1)
    out = []
    for b0 in range(0, flat.size, block):
        blk = flat[b0:b0 + block]
        a = max(abs(float(v)) for v in blk)
        for v in blk:
            if a == 0.0:
                out.append(7)
                continue
            x = float(np.float32(v) / np.float32(a))       # IEEE fp32 division
            d = [abs(x - cj) for cj in c]
            out.append(int(np.argmin(d)))                  # first (lower) on ties
    return np.array(out, np.uint8)


@pytest.mark.parametrize("shape,seed", [((3, 64), 1), ((5, 128), 2), ((2, 192), 3)])
def test_nearest_level_by_brute_force(shape, seed):
    w = np.random.default_rng(seed).standard_normal(shape).astype(np.float32) * 0.02
    amax = oracle.absmax(w)
    codes = oracle.encode(w, amax)
    assert np.array_equal(codes, brute_force_codes(w))


def test_special_blocks_by_brute_force():
    w = workloads.special_blocks(4)
    amax = oracle.absmax(w)
    codes = oracle.encode(w, amax)
    assert np.array_equal(codes, brute_force_codes(w))


def test_absmax_is_block_maximum_and_short_last_block():
    rng = np.random.default_rng(4)
    w = rng.standard_normal(64 * 5 + 17).astype(np.float32)
    amax = oracle.absmax(w)
    assert amax.size == 6
    for b in range(6):
        assert amax[b] == np.max(np.abs(w[b * 64:(b + 1) * 64]))


def test_extreme_elements_and_zero():
    rng = np.random.default_rng(5)
    w = rng.standard_normal((4, 64)).astype(np.float32)
    w[0, 3] = 0.0
    amax = oracle.absmax(w)
    codes = oracle.encode(w, amax).reshape(4, 64)
    assert codes[0, 3] == 7
    for row in range(4):
        i = int(np.argmax(np.abs(w[row])))
        assert codes[row, i] == (15 if w[row, i] > 0 else 0)


def test_all_zero_block():
    w = np.zeros(128, np.float32)
    w[64:] = 1.0
    amax = oracle.absmax(w)
    assert amax[0] == 0.0
    codes = oracle.encode(w, amax)
    assert np.all(codes[:64] == 7) and np.all(codes[64:] == 15)


def test_round_trip_of_codebook_points():
    """w = c_j * 2^e in a block whose absmax is 2^e encodes to j."""
    c = oracle.levels()
    for e in (-12, -3, 0, 5):
        blk = np.zeros(64, np.float32)
        blk[:16] = c * np.float32(2.0 ** e)
        blk[16:] = c[np.arange(48) % 16] * np.float32(2.0 ** e)
        codes = oracle.encode(blk, oracle.absmax(blk))
        assert np.array_equal(codes, np.arange(64) % 16)


def test_threshold_ties_go_to_lower_level():
    m = oracle.midpoints()
    blk = np.zeros(64, np.float32)
    blk[0] = 1.0                                    # absmax 1, so x = w exactly
    blk[1:16] = m
    codes = oracle.encode(blk, oracle.absmax(blk))
    assert np.array_equal(codes[1:16], np.arange(15))
    # one ulp above each threshold goes to the upper level
    blk[1:16] = np.nextafter(m, np.float32(2.0))
    codes = oracle.encode(blk, oracle.absmax(blk))
    assert np.array_equal(codes[1:16], np.arange(1, 16))


def test_error_bound_half_local_gap():
    """|w - c[code] a_b| <= a_b * (half the larger neighbouring gap) + rounding."""
    c = oracle.levels().astype(np.float64)
    w = workloads.weight(32, 256, outliers=True)
    amax = oracle.absmax(w)
    codes = oracle.encode(w, amax)
    flat = w.reshape(-1).astype(np.float64)
    a = np.repeat(amax.astype(np.float64), 64)
    gaps = np.diff(c)
    left = np.concatenate([[0.0], gaps])[codes]
    right = np.concatenate([gaps, [0.0]])[codes]
    bound = a * np.maximum(left, right) / 2 + a * 2.0 ** -23
    assert np.all(np.abs(flat - c[codes] * a) <= bound)
    # the largest half gap of the table (-1 .. -0.6962) caps every element
    assert np.max(gaps) / 2 == pytest.approx(0.1519036, abs=1e-6)
    assert np.all(np.abs(flat / np.where(a > 0, a, 1) - c[codes]) <= np.max(gaps) / 2 + 1e-6)


def test_pack_order_and_unpack():
    codes = np.array([1, 2, 3, 15, 0, 7, 9], np.uint8)
    packed = oracle.pack(codes)
    assert list(packed) == [0x12, 0x3F, 0x07, 0x90]
    assert np.array_equal(oracle.unpack(packed, 7), codes)


def test_thresholds_fit_sixteenth_buckets():
    """The spacing the GPU encoder's division-free code search relies on:
    consecutive thresholds are more than 1/16 apart (so a bucket
    [-1 + b/16, -1 + (b+1)/16) holds at most one) and none lies within 1e-3 of
    a bucket edge (so rounding x by a few ulp never moves it past a threshold
    when it moves it to the next bucket)."""
    m = oracle.midpoints().astype(np.float64)
    assert np.all(np.diff(m) > 1.0 / 16)
    edges = -1.0 + np.arange(33) / 16.0
    assert np.min(np.abs(m[:, None] - edges[None, :])) >= 1e-3
