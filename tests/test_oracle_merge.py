"""Pins of the oracle's adapter merge ("第 04 篇：QLoRA 原理" §12.3: W + s B A,
then encode again; the re-rounding the page warns about).

merge_lora states fp32(W_hat + s * sum_j B[:, j] A[j, :]) with the rank-r sum in
fp64 in ascending j.  Pinned by: the zero adapter (the dequantised base comes
back unchanged), an adapter whose product is exact in fp32 (a closed form),
the fp64 summation order on products whose running sum must round, the
re-quantisation of an unchanged base (the encoding of W_hat itself) and the
trainable shapes."""
import numpy as np
import torch

import oracle
import workloads


def _base(d_out=64, d_in=128, seed=0):
    W = workloads.weight(d_out, d_in, index=seed)
    qt = oracle.quantize(W)
    return qt, oracle.dequantize(qt, W.shape)


def test_zero_adapter_returns_the_base():
    qt, W_hat = _base()
    A = workloads.lora_a(8, 128, 0)
    B = torch.zeros(64, 8, dtype=torch.bfloat16)
    merged = oracle.merge_lora(W_hat, A, B, 2.0)
    assert merged.dtype == np.float32 and np.array_equal(merged, W_hat)
    again = oracle.merge_requantize(qt, W_hat.shape, A, B, 2.0)
    direct = oracle.quantize(W_hat)
    for k in ("packed", "q", "a2"):
        assert np.array_equal(again[k], direct[k])


def test_exact_rank_one_update_closed_form():
    """B = 1 in column 0 and A's row 0 a set of small bf16 values: s B A is
    exact, and so is its sum with W_hat (both bf16, close exponents)."""
    qt, W_hat = _base()
    r = 3
    B = torch.zeros(64, r, dtype=torch.bfloat16)
    B[:, 0] = 1.0
    A = torch.zeros(r, 128, dtype=torch.bfloat16)
    A[0] = torch.linspace(-0.25, 0.25, 128).bfloat16()
    merged = oracle.merge_lora(W_hat, A, B, 0.5)
    expect = (W_hat.astype(np.float64) + 0.5 * A[0].float().numpy().astype(np.float64)[None, :])
    assert np.array_equal(merged, expect.astype(np.float32))
    assert np.array_equal(merged.astype(np.float64), expect)  # no rounding at all


def test_rank_sum_in_fp64_ascending_order():
    """Products 2^60, 1, -2^60: summed in fp64 from j = 0 the 1 is lost
    (2^60 + 1 rounds to 2^60), so the update is 0, not 1."""
    W_hat = np.full((4, 64), 0.5, np.float32)
    B = torch.tensor([[2.0 ** 30, 1.0, -2.0 ** 30]] * 4, dtype=torch.bfloat16)
    A = torch.tensor([[2.0 ** 30] * 64, [1.0] * 64, [2.0 ** 30] * 64], dtype=torch.bfloat16)
    merged = oracle.merge_lora(W_hat, A, B, 1.0)
    assert np.all(merged == np.float32(0.5))
    # reversed, -2^60 + 1 rounds to -2^60 and cancels the same way
    merged_rev = oracle.merge_lora(W_hat, A.flip(0), B.flip(1), 1.0)
    assert np.all(merged_rev == np.float32(0.5))
    B2 = torch.tensor([[1.0, 2.0 ** 30, -2.0 ** 30]] * 4, dtype=torch.bfloat16)
    A2 = torch.tensor([[1.0] * 64, [2.0 ** 30] * 64, [2.0 ** 30] * 64], dtype=torch.bfloat16)
    merged_first = oracle.merge_lora(W_hat, A2, B2, 1.0)
    assert np.all(merged_first == np.float32(0.5))  # 1 + 2^60 -> 2^60, then 0
    B3 = torch.tensor([[2.0 ** 30, -2.0 ** 30, 1.0]] * 4, dtype=torch.bfloat16)
    A3 = torch.tensor([[2.0 ** 30] * 64, [2.0 ** 30] * 64, [1.0] * 64], dtype=torch.bfloat16)
    merged_last = oracle.merge_lora(W_hat, A3, B3, 1.0)
    assert np.all(merged_last == np.float32(1.5))  # 2^60 - 2^60 = 0, then + 1


def test_scaling_enters_as_fp32_and_rounds_once():
    W_hat = np.zeros((8, 64), np.float32)
    B = torch.ones(8, 1, dtype=torch.bfloat16)
    A = torch.ones(1, 64, dtype=torch.bfloat16)
    s = 0.1  # fp32(0.1) = 0.100000001490116...
    merged = oracle.merge_lora(W_hat, A, B, s)
    assert np.all(merged == np.float32(0.1))
    assert np.float64(merged[0, 0]) != 0.1


def test_merged_shape_matches_the_base():
    qt, W_hat = _base(48, 192, 3)
    A = workloads.lora_a(16, 192, 3)
    B = workloads.lora_b(48, 16, 3)
    merged = oracle.merge_lora(W_hat, A, B, 1.0)
    assert merged.shape == (48, 192)
    # the update is the rank-16 product: W' - W_hat has rank <= 16
    diff = merged.astype(np.float64) - W_hat.astype(np.float64)
    assert np.linalg.matrix_rank(diff, tol=1e-6 * np.abs(diff).max()) <= 16
