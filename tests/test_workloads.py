"""The seeded input generators follow the recipe their module states (and the
five workloads have the shapes they are named for), and they stay free of the
method: the generator module imports neither the oracle nor the CUDA
package, so the two sides compared by the parity tests share only their
random inputs."""
import ast
import os

import numpy as np
import pytest
import torch

import workloads

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_weight_is_seeded_normal_with_exact_outliers():
    w0 = workloads.weight(256, 512, sigma=0.02, outliers=False, index=3)
    assert w0.dtype == np.float32 and w0.shape == (256, 512)
    assert np.array_equal(w0, workloads.weight(256, 512, sigma=0.02, outliers=False, index=3))
    assert abs(float(w0.mean())) < 1e-3 and abs(float(w0.std()) - 0.02) < 5e-4
    w1 = workloads.weight(256, 512, sigma=0.02, outliers=True, index=3)
    diff = np.flatnonzero(w1 != w0)
    assert diff.size == 256 * 512 // 1000  # 0.1 % of the entries
    assert np.array_equal(w1.reshape(-1)[diff], w0.reshape(-1)[diff] * np.float32(10.0))
    assert not np.array_equal(w0, workloads.weight(256, 512, index=4))


@pytest.mark.parametrize("gen,shape,std", [
    (lambda: workloads.lora_a(64, 4096, 0), (64, 4096), 1 / 64),
    (lambda: workloads.lora_b(4096, 64, 0), (4096, 64), 0.01),
    (lambda: workloads.activations(64, 4096), (64, 4096), 1.0),
    (lambda: workloads.grad_output(64, 4096, 0), (64, 4096), 1.0),
])
def test_adapter_and_activation_draws(gen, shape, std):
    t = gen()
    assert t.dtype == torch.bfloat16 and tuple(t.shape) == shape and t.is_contiguous()
    x = t.float().numpy()
    assert abs(float(x.std()) - std) < 0.02 * std and abs(float(x.mean())) < 0.02 * std
    assert torch.equal(t, gen())  # seeded


def test_bf16_rounding_is_round_to_nearest_even():
    a = np.array([1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -(1.0 + 2.0 ** -8)], np.float32)
    got = workloads._bf16(a).float().numpy()
    assert np.array_equal(got, np.array([1.0, 1.0 + 2.0 ** -6, -1.0], np.float32))


def test_workload_shapes():
    w = workloads.WORKLOADS
    assert set(w) == {"linear512_r8_m16", "q_proj4096_r64_m1-4-16", "llama7b_mlp_r64_m4096",
                      "llama7b_layer_r16_m8192", "llama65b_layer_r64_m2048"}
    assert [(m.d_out, m.d_in) for m in w["llama7b_mlp_r64_m4096"].modules] == [(11008, 4096), (11008, 4096),
                                                                               (4096, 11008)]
    assert len(w["llama7b_layer_r16_m8192"].modules) == 7 and w["llama7b_layer_r16_m8192"].tokens == (8192,)
    l65 = w["llama65b_layer_r64_m2048"]
    assert sum(m.d_out * m.d_in for m in l65.modules) == 4 * 8192 * 8192 + 3 * 8192 * 22016
    assert l65.sigma == 0.015 and l65.outliers and l65.quantize_timed and l65.tokens == (2048,)
    q = w["q_proj4096_r64_m1-4-16"]
    assert q.tokens == (1, 4, 16) and q.backward == "dx" and q.scaling == 16 / 64
    assert w["linear512_r8_m16"].scaling == 2.0


def test_generators_hold_no_method_code():
    tree = ast.parse(open(os.path.join(ROOT, "workloads.py")).read())
    imported = set()
    for node in ast.walk(tree):
        if isinstance(node, ast.Import):
            imported.update(a.name.split(".")[0] for a in node.names)
        elif isinstance(node, ast.ImportFrom) and node.module:
            imported.add(node.module.split(".")[0])
    assert imported <= {"__future__", "dataclasses", "typing", "numpy", "torch"}, imported
