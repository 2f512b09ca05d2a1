"""Pins of the oracle's encoding without double quantisation: the codes with
one fp32 scale per block of 64 weights, stored as is ("第 04 篇：QLoRA 原理"
§5.1, the block-wise quantisation that double quantisation then compresses).
The code search and the block absmax are the pinned ones of the
double-quantised encoding; what is new is the storage and the decode from
plain fp32 scales, pinned here against the pages' storage figures, exact
power-of-two cases, the error bound and the already pinned two-level decode."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from conftest import golden_table


def test_storage_without_dq_matches_pages():
    g = golden_table("storage_accounting.txt")
    n = int(g["params_65b"])
    b1 = int(g["block_size_1"])
    assert b1 == oracle.NF4_BLOCK
    # 4 bits of code plus 32 bits per block of 64: the 0.5 bit of §5.1
    per_weight = oracle.packed_bytes_nodq(64 * 1024) * 8 / (64 * 1024)
    assert per_weight - 4 == g["scale_bits_without_dq"]
    # what double quantisation saves at 65B (§5.3: about 3.0 GB, 2.82 GiB)
    saved = oracle.packed_bytes_nodq(n) - oracle.packed_bytes(n)
    assert round(saved / 1e9, 1) == g["dq_saving_65b_gb"]
    assert round(saved / 2 ** 30, 2) == g["dq_saving_65b_gib"]


def test_power_of_two_block_scales_round_trip():
    """Each block holds codebook points times its own power of two, +1 among
    them: its scale is that power exactly and every weight decodes to
    bf16(w)."""
    c = oracle.levels()
    rng = np.random.default_rng(5)
    idx = rng.integers(0, 16, size=(6, 256))
    idx[:, ::64] = 15                                  # +1 in every block
    k = rng.integers(-12, 3, size=(6, 4))              # one exponent per block
    scale = np.repeat(np.float32(2.0) ** k.astype(np.float32), 64, axis=1)
    w = (c[idx] * scale).astype(np.float32)
    qt = oracle.quantize_nodq(w)
    assert np.array_equal(qt["absmax"], (np.float32(2.0) ** k.astype(np.float32)).reshape(-1))
    assert np.array_equal(qt["codes"].reshape(w.shape), idx.astype(np.uint8))
    w_hat = oracle.dequantize(qt, w.shape)
    ref = torch.from_numpy(w).to(torch.bfloat16).float().numpy()
    assert np.array_equal(w_hat, ref)


def test_error_bound_without_dq():
    """|w - w_hat| <= a_b * half the local level gap + bf16 rounding: no
    scale error term, unlike the double-quantised encoding."""
    c = oracle.levels().astype(np.float64)
    w = workloads.weight(40, 448, outliers=True, index=3)
    qt = oracle.quantize_nodq(w)
    w_hat = oracle.dequantize(qt, w.shape).reshape(-1).astype(np.float64)
    a = np.repeat(qt["absmax"].astype(np.float64), 64)
    codes = qt["codes"]
    gaps = np.diff(c)
    half = np.maximum(np.concatenate([[0.0], gaps])[codes], np.concatenate([gaps, [0.0]])[codes]) / 2
    bound = a * half + np.abs(w_hat) * 2.0 ** -8 + 1e-12
    assert np.all(np.abs(w.reshape(-1) - w_hat) <= bound)
    # and the scale is the block's absmax itself
    assert np.array_equal(qt["absmax"], np.abs(w).reshape(-1, 64).max(axis=1))


def test_fp32_scale_decode_is_the_two_level_decode_given_restored_scales():
    w = workloads.weight(16, 512, outliers=True, index=4)
    qt = oracle.quantize(w)
    restored = oracle.dq_scales(qt["q"], qt["a2"], float(qt["mu"]))
    a = oracle.dequantize_scales_bits(qt["packed"], restored, w.size)
    b = oracle.dequantize_bits(qt["packed"], qt["q"], qt["a2"], float(qt["mu"]), w.size)
    assert np.array_equal(a, b)


def test_all_zero_block_without_dq():
    w = workloads.weight(2, 192)
    w[1, 64:128] = 0.0
    qt = oracle.quantize_nodq(w)
    assert qt["absmax"][4] == 0.0
    assert np.all(qt["codes"].reshape(w.shape)[1, 64:128] == 7)
    assert np.all(oracle.dequantize(qt, w.shape)[1, 64:128] == 0.0)


@pytest.mark.parametrize("shape", [(1, 64), (3, 640)])
def test_codes_are_the_double_quantised_encodings_codes(shape):
    """Both encodings code each weight against its block's own absmax."""
    w = workloads.weight(*shape, outliers=True, index=6)
    assert np.array_equal(oracle.quantize_nodq(w)["packed"], oracle.quantize(w)["packed"])
