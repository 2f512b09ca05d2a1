"""Pins of the oracle's AdamW step (the adapter's optimizer update, "第 04 篇：
QLoRA 原理" §7.3: fp32 first and second moments per trainable parameter).

The pages print no update formula; the oracle states decoupled-weight-decay
AdamW with bias-corrected moments.  It is pinned to a library routine
(torch.optim.AdamW run in float64) over several steps, to the closed form of
the first step, and to the pure-decay case."""
import numpy as np
import pytest
import torch

import oracle


def _torch_adamw(p0, grads, lr, betas, eps, wd):
    p = torch.nn.Parameter(torch.from_numpy(p0.copy()))
    opt = torch.optim.AdamW([p], lr=lr, betas=betas, eps=eps, weight_decay=wd)
    out = []
    for g in grads:
        p.grad = torch.from_numpy(g.copy())
        opt.step()
        st = opt.state[p]
        out.append((p.detach().numpy().copy(), st["exp_avg"].numpy().copy(), st["exp_avg_sq"].numpy().copy()))
    return out


@pytest.mark.parametrize("wd", [0.0, 0.01])
def test_matches_torch_adamw_over_steps(wd):
    rng = np.random.default_rng(3)
    p = rng.standard_normal(257) * 0.05
    grads = [rng.standard_normal(257) * 10.0 ** rng.uniform(-4, 0) for _ in range(6)]
    ref = _torch_adamw(p, grads, 2e-4, (0.9, 0.999), 1e-8, wd)
    m = np.zeros_like(p)
    v = np.zeros_like(p)
    for t, (g, (rp, rm, rv)) in enumerate(zip(grads, ref), start=1):
        p, m, v = oracle.adamw_step(p, g, m, v, t, 2e-4, 0.9, 0.999, 1e-8, wd)
        np.testing.assert_allclose(m, rm, rtol=1e-12, atol=0)
        np.testing.assert_allclose(v, rv, rtol=1e-12, atol=0)
        np.testing.assert_allclose(p, rp, rtol=1e-12, atol=1e-18)


def test_first_step_closed_form():
    """With zero moments and no decay the first step moves each entry by
    lr * g / (|g| + eps): the bias corrections undo (1 - b1) and (1 - b2)."""
    rng = np.random.default_rng(4)
    p = rng.standard_normal(64)
    g = rng.standard_normal(64) * 1e-3
    lr, eps = 1e-3, 1e-8
    p1, m1, v1 = oracle.adamw_step(p, g, np.zeros(64), np.zeros(64), 1, lr, 0.9, 0.999, eps, 0.0)
    np.testing.assert_allclose(p1, p - lr * g / (np.abs(g) + eps), rtol=1e-12)
    np.testing.assert_allclose(m1, 0.1 * g, rtol=1e-15)
    np.testing.assert_allclose(v1, 0.001 * g * g, rtol=1e-12)


def test_zero_gradient_is_pure_decay():
    p = np.linspace(-1, 1, 9)
    m = np.full(9, 0.5)
    v = np.full(9, 0.25)
    p1, m1, v1 = oracle.adamw_step(p, np.zeros(9), m, v, 3, 0.1, 0.9, 0.999, 1e-8, 0.5)
    np.testing.assert_allclose(m1, 0.45, rtol=1e-15)
    np.testing.assert_allclose(v1, 0.24975, rtol=1e-15)
    step = (0.1 / (1 - 0.9 ** 3)) * m1 / (np.sqrt(v1) / np.sqrt(1 - 0.999 ** 3) + 1e-8)
    np.testing.assert_allclose(p1, p * (1 - 0.05) - step, rtol=1e-12, atol=1e-15)
    with pytest.raises(ValueError):
        oracle.adamw_step(p, np.zeros(9), m, v, 0, 0.1)
