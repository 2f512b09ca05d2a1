"""Pins of the oracle's double quantisation, dequantisation and storage
accounting ("第 04 篇：QLoRA 原理" §5.1-§5.4, §6.1, §8.1; compassingai.com
QLoRA concept page, "雙重量化")."""
import math

import numpy as np
import pytest
import torch

import oracle
import workloads
from conftest import golden_table


@pytest.mark.parametrize("n", [1, 2, 3, 5, 255, 256, 257, 4097, 100003])
def test_dq_mean_is_the_exact_mean_rounded(n):
    a = np.abs(np.random.default_rng(n).standard_normal(n).astype(np.float32)) * 0.05
    mu = oracle.dq_mean(a)
    exact = math.fsum(float(v) for v in a) / n
    assert mu == np.float32(exact)


def test_dq_codes_extremes_and_bound():
    w = workloads.weight(64, 512, outliers=True, index=3)
    qt = oracle.quantize(w)
    amax, q, a2, mu = qt["absmax"], qt["q"], qt["a2"], float(qt["mu"])
    assert np.all(np.abs(q.astype(np.int32)) <= 127)
    s_hat = oracle.dq_scales(q, a2, mu)
    for g in range(a2.size):
        lo, hi = g * 256, min((g + 1) * 256, amax.size)
        d = amax[lo:hi].astype(np.float64) - mu
        assert a2[g] == np.float32(np.max(np.abs(amax[lo:hi] - np.float32(mu))))
        # the scale that attains a2 gets +-127
        i = lo + int(np.argmax(np.abs(d)))
        assert abs(int(q[i])) == 127
        # reconstruction within half a step, plus rounding of the fp32 ops
        err = np.abs(s_hat[lo:hi].astype(np.float64) - amax[lo:hi])
        tol = a2[g] / 254.0 + 4 * np.spacing(np.float32(max(mu, float(np.max(amax[lo:hi])))))
        assert np.all(err <= tol)


def test_dq_constant_group_has_zero_codes():
    amax = np.full(300, 0.125, np.float32)
    mu = oracle.dq_mean(amax)
    assert mu == np.float32(0.125)
    q, a2 = oracle.dq_quantize(amax, mu)
    assert np.all(q == 0) and np.all(a2 == 0)
    assert np.all(oracle.dq_scales(q, a2, mu) == np.float32(0.125))


def test_dq_short_tail_group():
    rng = np.random.default_rng(9)
    amax = np.abs(rng.standard_normal(256 * 2 + 40)).astype(np.float32)
    q, a2 = oracle.dq_quantize(amax, oracle.dq_mean(amax))
    assert a2.size == 3
    tail = amax[512:] - oracle.dq_mean(amax)
    assert a2[2] == np.max(np.abs(tail))


def test_bf16_rounding_matches_library():
    rng = np.random.default_rng(11)
    vals = np.concatenate([
        rng.standard_normal(4000).astype(np.float32),
        (rng.standard_normal(1000) * 1e-40).astype(np.float32),       # subnormals
        np.array([0.0, -0.0, 1.0, -1.0, 3.0e38, -3.0e38, np.inf, -np.inf], np.float32),
        # exact ties between two bfloat16 values: 1 + 2^-8 (to even: 1),
        # 1 + 3*2^-8 (to even: 1 + 2^-6)
        np.array([1 + 2 ** -8, 1 + 3 * 2 ** -8, -(1 + 2 ** -8)], np.float32),
    ])
    got = oracle.bf16_bits(vals)
    ref = torch.from_numpy(vals).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got, ref)


def test_dequantize_error_bound():
    """|w - w_hat| <= a_b * half gap + |c| |s_hat - a_b| + bf16 rounding."""
    c = oracle.levels().astype(np.float64)
    w = workloads.weight(48, 384, outliers=True, index=2)
    qt = oracle.quantize(w)
    w_hat = oracle.dequantize(qt, w.shape).reshape(-1).astype(np.float64)
    s_hat = np.repeat(oracle.dq_scales(qt["q"], qt["a2"], float(qt["mu"])).astype(np.float64), 64)
    a = np.repeat(qt["absmax"].astype(np.float64), 64)
    codes = qt["codes"]
    gaps = np.diff(c)
    half = np.maximum(np.concatenate([[0.0], gaps])[codes], np.concatenate([gaps, [0.0]])[codes]) / 2
    bound = a * half + np.abs(c[codes]) * np.abs(s_hat - a) + np.abs(w_hat) * 2.0 ** -8 + 1e-12
    assert np.all(np.abs(w.reshape(-1) - w_hat) <= bound)


def test_dequantize_round_trip_with_common_scale():
    """Every block with the same power-of-two absmax: the scales double-quantise
    exactly (a2 = 0), so w_hat = bf16(w) for codebook points times the scale."""
    c = oracle.levels()
    idx = np.random.default_rng(3).integers(0, 16, size=(8, 128))
    idx[:, 0] = 15                               # every block contains +1 * 2^-4
    idx[:, 64] = 0
    w = (c[idx] * np.float32(2.0 ** -4)).astype(np.float32)
    qt = oracle.quantize(w)
    assert np.all(qt["a2"] == 0) and np.all(qt["q"] == 0)
    assert np.array_equal(qt["codes"].reshape(w.shape), idx.astype(np.uint8))
    w_hat = oracle.dequantize(qt, w.shape)
    ref = torch.from_numpy(w).to(torch.bfloat16).float().numpy()
    assert np.array_equal(w_hat, ref)


def test_all_zero_block_dequantizes_to_zero():
    w = workloads.weight(4, 128)
    w[1, :64] = 0.0
    qt = oracle.quantize(w)
    w_hat = oracle.dequantize(qt, w.shape)
    assert np.all(w_hat[1, :64] == 0.0)


def test_storage_accounting_matches_pages():
    g = golden_table("storage_accounting.txt")
    n = int(g["params_65b"])
    b1, b2 = int(g["block_size_1"]), int(g["block_size_2"])
    assert (b1, b2) == (oracle.NF4_BLOCK, oracle.DQ_BLOCK)
    total = oracle.packed_bytes(n)
    assert round(total / 1e9, 2) == g["nf4_dq_65b_gb"]
    assert round(total / 2 ** 30, 2) == g["nf4_dq_65b_gib"]
    # scale metadata per weight, without and with double quantisation
    without = 32 / b1
    assert without == g["scale_bits_without_dq"]
    with_dq = (total - n / 2) * 8 / n
    assert round(without - with_dq, 2) == g["dq_saving_bits"]
    saved_bytes = (without - with_dq) * n / 8
    assert round(saved_bytes / 1e9, 1) == g["dq_saving_65b_gb"]
    assert round(saved_bytes / 2 ** 30, 2) == g["dq_saving_65b_gib"]
