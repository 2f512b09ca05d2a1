"""Pins of the oracle's layer arithmetic (forward, backward) against a library
statement of the same layer (torch modules + autograd in fp64), central finite
differences and special cases ("第 04 篇：QLoRA 原理" §2.2, §2.4, §6.3-§6.5;
compassingai.com QLoRA concept page, compute graph and LoRA shapes)."""
import numpy as np
import pytest
import torch

import oracle
import workloads


def small_case(d_in=64, d_out=128, m=3, r=2, seed=0, b_std=0.3):
    c = workloads.linear_case(d_out, d_in, m, r, alpha=2 * r, index=seed, b_std=b_std)
    qt = oracle.quantize(c.W)
    W_hat = oracle.dequantize(qt, c.W.shape)
    return c, W_hat


def library_layer(W_hat, A, B, scaling):
    """The adapted linear as separate library modules: frozen base, LoRA down,
    LoRA up, summed with the scaling (fp64)."""
    d_out, d_in = W_hat.shape
    r = A.shape[0]
    base = torch.nn.Linear(d_in, d_out, bias=False).double()
    down = torch.nn.Linear(d_in, r, bias=False).double()
    up = torch.nn.Linear(r, d_out, bias=False).double()
    with torch.no_grad():
        base.weight.copy_(torch.from_numpy(np.asarray(W_hat, np.float64)))
        down.weight.copy_(A.double())
        up.weight.copy_(B.double())
    base.weight.requires_grad_(False)
    return base, down, up


@pytest.mark.parametrize("d_in,d_out,m,r", [(64, 128, 3, 2), (128, 64, 5, 8), (192, 256, 17, 16)])
def test_forward_backward_match_autograd(d_in, d_out, m, r):
    c, W_hat = small_case(d_in, d_out, m, r)
    base, down, up = library_layer(W_hat, c.A, c.B, c.scaling)
    x = c.X.double().clone().requires_grad_(True)
    y = base(x) + c.scaling * up(down(x))
    y.backward(c.dY.double())
    Y, _ = oracle.forward(W_hat, c.A, c.B, c.X, c.scaling)
    dX, dA, dB = oracle.backward(W_hat, c.A, c.B, c.X, c.dY, c.scaling)
    np.testing.assert_allclose(Y, y.detach().numpy(), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(dX, x.grad.numpy(), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(dA, down.weight.grad.numpy(), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(dB, up.weight.grad.numpy(), rtol=1e-12, atol=1e-12)
    assert base.weight.grad is None                # no weight gradient of the base
    trainable = sum(p.numel() for mod in (base, down, up) for p in mod.parameters() if p.requires_grad)
    assert trainable == r * (d_in + d_out) == oracle.trainable_parameters(d_in, d_out, r)


def test_gradients_match_central_differences():
    c, W_hat = small_case(64, 128, 3, 2)
    X = c.X.double().numpy()
    A = c.A.double().numpy()
    B = c.B.double().numpy()
    dY = c.dY.double().numpy()
    s = c.scaling

    def loss(X_, A_, B_):
        return float(np.sum(dY * oracle.forward(W_hat, A_, B_, X_, s)[0]))

    dX, dA, dB = oracle.backward(W_hat, A, B, X, dY, s)
    h = 1e-3
    rng = np.random.default_rng(0)
    for name, arr, grad in (("X", X, dX), ("A", A, dA), ("B", B, dB)):
        for _ in range(12):
            idx = tuple(int(rng.integers(0, n)) for n in arr.shape)
            plus, minus = arr.copy(), arr.copy()
            plus[idx] += h
            minus[idx] -= h
            args_p = {"X": (plus, A, B), "A": (X, plus, B), "B": (X, A, plus)}[name]
            args_m = {"X": (minus, A, B), "A": (X, minus, B), "B": (X, A, minus)}[name]
            fd = (loss(*args_p) - loss(*args_m)) / (2 * h)
            assert abs(fd - grad[idx]) <= 1e-6 * max(1.0, abs(grad[idx])), (name, idx, fd, grad[idx])


def test_zero_b_reduces_to_the_base_product():
    c, W_hat = small_case(128, 64, 4, 8)
    B0 = torch.zeros_like(c.B)
    Y, T = oracle.forward(W_hat, c.A, B0, c.X, c.scaling)
    ref = torch.nn.functional.linear(c.X.double(), torch.from_numpy(W_hat.astype(np.float64)))
    np.testing.assert_allclose(Y, ref.numpy(), rtol=1e-12, atol=1e-12)
    dX, dA, dB = oracle.backward(W_hat, c.A, B0, c.X, c.dY, c.scaling)
    assert np.all(dA == 0)
    ref_dx = c.dY.double() @ torch.from_numpy(W_hat.astype(np.float64))
    np.testing.assert_allclose(dX, ref_dx.numpy(), rtol=1e-12, atol=1e-12)


def test_zero_a_gives_zero_db():
    c, W_hat = small_case(128, 64, 4, 8)
    A0 = torch.zeros_like(c.A)
    _, _, dB = oracle.backward(W_hat, A0, c.B, c.X, c.dY, c.scaling)
    assert np.all(dB == 0)


def test_linearity_in_x():
    c, W_hat = small_case(64, 128, 6, 4)
    X1 = c.X.double().numpy()
    X2 = np.random.default_rng(2).standard_normal(X1.shape)
    Y1 = oracle.forward(W_hat, c.A, c.B, X1, c.scaling)[0]
    Y2 = oracle.forward(W_hat, c.A, c.B, X2, c.scaling)[0]
    Y12 = oracle.forward(W_hat, c.A, c.B, 2.5 * X1 - 0.75 * X2, c.scaling)[0]
    np.testing.assert_allclose(Y12, 2.5 * Y1 - 0.75 * Y2, rtol=1e-10, atol=1e-10)


def test_row_subset_helpers_agree_with_full():
    c, W_hat = small_case(128, 64, 9, 4)
    rows = np.array([0, 4, 8])
    Y, _ = oracle.forward(W_hat, c.A, c.B, c.X, c.scaling)
    dX, dA, dB = oracle.backward(W_hat, c.A, c.B, c.X, c.dY, c.scaling)
    np.testing.assert_array_equal(oracle.output_rows(W_hat, c.A, c.B, c.X[rows], c.scaling), Y[rows])
    np.testing.assert_allclose(oracle.input_grad_rows(W_hat, c.A, c.B, c.dY[rows], c.scaling), dX[rows],
                               rtol=1e-13, atol=1e-13)
    lA, lB = oracle.lora_grads(c.A, c.B, c.X, c.dY, c.scaling)
    np.testing.assert_array_equal(lA, dA)
    np.testing.assert_array_equal(lB, dB)
