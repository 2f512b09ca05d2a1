"""Comparison helpers shared by the GPU parity tests.

Floating-point outputs (Y, dX, dA, dB) are compared normwise per tensor:
    max |got - ref| / max |ref|   <= 2e-2
    mean |got - ref| / mean |ref| <= 2e-3
(the tolerance the layer is specified to, with the relative error read as
normwise because element-wise ratios are undefined where ref is ~0).

The outputs are bfloat16 by specification, so the fp64 reference is rounded to
bfloat16 (round to nearest even) before the comparison: the best answer the
output format can hold then scores zero error."""
import numpy as np
import torch

MAX_REL = 2e-2
MEAN_REL = 2e-3


def to_np(t) -> np.ndarray:
    if isinstance(t, torch.Tensor):
        return t.detach().float().cpu().numpy().astype(np.float64)
    return np.asarray(t, np.float64)


def rel_errors(got, ref):
    got, ref = to_np(got), to_np(ref)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    d = np.abs(got - ref)
    max_ref = float(np.max(np.abs(ref))) if ref.size else 0.0
    mean_ref = float(np.mean(np.abs(ref))) if ref.size else 0.0
    max_rel = float(np.max(d)) / max_ref if max_ref > 0 else float(np.max(d, initial=0.0))
    mean_rel = float(np.mean(d)) / mean_ref if mean_ref > 0 else float(np.mean(d) if d.size else 0.0)
    return max_rel, mean_rel


def bf16_round(ref) -> np.ndarray:
    return torch.from_numpy(to_np(ref)).to(torch.bfloat16).double().numpy()


def assert_close(got, ref, name="", max_rel=MAX_REL, mean_rel=MEAN_REL, round_ref=True):
    mx, mn = rel_errors(got, bf16_round(ref) if round_ref else ref)
    assert mx <= max_rel and mn <= mean_rel, "%s: max rel %.3e (<= %.1e), mean rel %.3e (<= %.1e)" % (
        name, mx, max_rel, mn, mean_rel)
    return mx, mn
